"""Parity of the tcgen05 (PREFILL) expert-FFN kernels with the CPU oracle on
small inputs: boundaries of the 192-row token tiles (one expert receiving
exactly 191, 192, 193, 383, 384, 385, ... rows) in the PREFILL and HYBRID
forms, several H and I, the shared expert, and agreement of every form with
the oracle."""
import numpy as np
import pytest
import torch

import mixture_experts_ffn_sort_b200 as moe
import oracle
from mixture_experts_ffn_sort_b200 import workloads as wl

from _gpu_util import assert_moe_close, bf16_tensor

pytestmark = pytest.mark.gpu


def dev(a, dtype=None):
    t = torch.from_numpy(np.ascontiguousarray(a)).cuda()
    return t if dtype is None else t.to(dtype)


def _ffn(x, K, ex, off, sr, wt, mode, sh=None):
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    y, ys = moe.moe_expert_ffn(bf16_tensor(x), K, moe.Experts.from_host(ex), dev(off), dev(sr),
                               dev(wt, torch.float32), moe.Experts.from_host(sh) if sh else None,
                               mode=mode, status=status)
    torch.cuda.synchronize()
    assert status.item() == 0, status.item()
    return y, ys


def test_prefill_tiny_single_expert():
    T, H, I, E, K = 16, 128, 128, 2, 1
    ex = wl.draw_experts(2, 60, E, I, H, 0.05, threads=1)
    x = wl.random_rows_bf16(T, H, seed=1)
    ids = np.zeros((T, K), np.int32)
    off, sr, inv, _ = oracle.sort(ids, E)
    wt = np.ones((T, K))
    y, _ = _ffn(x, K, ex, off, sr, wt, moe.MOE_MODE_PREFILL)
    assert_moe_close(y, oracle.ffn_sorted(x, K, ex, off, sr, wt), "y_sorted")


# The prefill kernels' token tile is 192 rows (the MMA's N); an expert's rows
# are split into tiles of 192 and a ragged last tile.
TILE_ROWS = 192


@pytest.mark.parametrize("n_hot", [1, 15, 16, 17, 31, 32, 33, TILE_ROWS - 1, TILE_ROWS, TILE_ROWS + 1, 255, 256, 257,
                                   2 * TILE_ROWS - 1, 2 * TILE_ROWS, 2 * TILE_ROWS + 1, 513, 3 * TILE_ROWS + 1])
@pytest.mark.parametrize("mode", [moe.MOE_MODE_PREFILL, moe.MOE_MODE_HYBRID])
def test_prefill_token_tile_boundaries(n_hot, mode):
    """The hot expert receives exactly n_hot rows (slot 0 of every token)."""
    T, H, I, E, K = n_hot, 256, 128, 5, 2
    ex = wl.draw_experts(3, 61, E, I, H, 0.05, threads=2)
    x = wl.random_rows_bf16(T, H, seed=n_hot)
    ids = wl.skewed_ids(T, K, E, hot=1, seed=n_hot)
    off, sr, inv, _ = oracle.sort(ids, E)
    assert off[2] - off[1] == n_hot
    wt = np.random.default_rng(n_hot).random((T, K)).astype(np.float32).astype(np.float64)
    y, _ = _ffn(x, K, ex, off, sr, wt, mode)
    assert_moe_close(y, oracle.ffn_sorted(x, K, ex, off, sr, wt), "y_sorted")


@pytest.mark.parametrize("T,H,I,E,K,Is", [(64, 512, 256, 8, 2, 0), (200, 1024, 384, 16, 4, 256),
                                          (40, 384, 128, 3, 3, 128), (600, 128, 512, 6, 2, 0)])
def test_prefill_shapes_with_shared(T, H, I, E, K, Is):
    ex = wl.draw_experts(4, 62, E, I, H, 0.05, threads=4)
    sh = wl.draw_experts(4, 63, 1, Is, H, 0.05, threads=1) if Is else None
    x = wl.random_rows_bf16(T, H, seed=T)
    lg = np.random.default_rng(T).standard_normal((T, E)).astype(np.float32)
    ids, wt = oracle.route(lg, K)
    off, sr, inv, _ = oracle.sort(ids, E)
    wt32 = wt.astype(np.float32).astype(np.float64)
    y, ys = _ffn(x, K, ex, off, sr, wt32, moe.MOE_MODE_PREFILL, sh)
    assert_moe_close(y, oracle.ffn_sorted(x, K, ex, off, sr, wt32), "y_sorted")
    if sh:
        assert_moe_close(ys, oracle.ffn_shared(x, sh), "y_shared")


@pytest.mark.parametrize("mode", [moe.MOE_MODE_DECODE, moe.MOE_MODE_PREFILL, moe.MOE_MODE_HYBRID])
def test_both_modes_full_pipeline(mode):
    T, H, I, E, K = 300, 512, 256, 16, 4
    ex = wl.draw_experts(5, 64, E, I, H, 0.05, threads=4)
    sh = wl.draw_experts(5, 65, 1, 128, H, 0.05, threads=1)
    x = wl.random_rows_bf16(T, H, seed=5)
    lg = np.random.default_rng(6).standard_normal((T, E)).astype(np.float32)
    mask = (np.random.default_rng(7).random((T, K)) < 0.05).astype(np.uint8)
    layer = moe.MoEFFN(moe.Experts.from_host(ex), T, K, moe.Experts.from_host(sh), mode=mode)
    out = layer(bf16_tensor(x), dev(lg), dev(mask))
    torch.cuda.synchronize()
    assert layer.status.item() == 0
    assert_moe_close(out, oracle.moe(x, lg, K, ex, sh, mask)["out"], "out")


def test_prefill_special_codes():
    T, H, I, E, K = 40, 256, 128, 2, 1
    for ex in (wl.subnormal_experts(E, I, H, seed=7), wl.all_code_experts(E, I, H, seed=8)):
        x = wl.random_rows_bf16(T, H, seed=9)
        lg = np.random.default_rng(10).standard_normal((T, E)).astype(np.float32)
        layer = moe.MoEFFN(moe.Experts.from_host(ex), T, K, mode=moe.MOE_MODE_PREFILL)
        out = layer(bf16_tensor(x), dev(lg))
        torch.cuda.synchronize()
        assert_moe_close(out, oracle.moe(x, lg, K, ex)["out"], "out")


@pytest.mark.parametrize("T,H,I,E,K,Is,zf", [(300, 512, 256, 16, 4, 128, 0.05), (64, 256, 128, 8, 2, 0, 0.0),
                                             (1000, 1024, 256, 32, 6, 256, 0.01), (193, 384, 128, 5, 2, 0, 0.0)])
@pytest.mark.parametrize("out_dtype", [moe.MOE_OUT_BF16, moe.MOE_OUT_F32])
def test_fused_ffn_combine(T, H, I, E, K, Is, zf, out_dtype):
    """moe_expert_ffn_combine (the down epilogue reducing into the fp32 output
    rows) against the oracle, with zero-weight routes and a shared expert."""
    ex = wl.draw_experts(8, 66, E, I, H, 0.05, threads=4)
    sh = wl.draw_experts(8, 67, 1, Is, H, 0.05, threads=1) if Is else None
    x = wl.random_rows_bf16(T, H, seed=T + 1)
    lg = np.random.default_rng(T + 2).standard_normal((T, E)).astype(np.float32)
    mask = (np.random.default_rng(T + 3).random((T, K)) < zf).astype(np.uint8) if zf else None
    layer = moe.MoEFFN(moe.Experts.from_host(ex), T, K, moe.Experts.from_host(sh) if sh else None,
                       out_dtype=out_dtype, fused_combine=True)
    out = layer(bf16_tensor(x), dev(lg), dev(mask) if mask is not None else None)
    torch.cuda.synchronize()
    assert layer.status.item() == 0
    assert out.dtype == (torch.bfloat16 if out_dtype == moe.MOE_OUT_BF16 else torch.float32)
    assert_moe_close(out, oracle.moe(x, lg, K, ex, sh, mask)["out"], "fused out")


def test_fused_ffn_combine_matches_two_calls():
    """The fused call and moe_expert_ffn + moe_combine agree to fp32 summation
    order (same bf16 rows, different order of the fp32 additions)."""
    T, H, I, E, K, Is = 500, 512, 256, 16, 4, 128
    ex = wl.draw_experts(9, 68, E, I, H, 0.05, threads=4)
    sh = wl.draw_experts(9, 69, 1, Is, H, 0.05, threads=1)
    x = wl.random_rows_bf16(T, H, seed=9)
    lg = np.random.default_rng(10).standard_normal((T, E)).astype(np.float32)
    a = moe.MoEFFN(moe.Experts.from_host(ex), T, K, moe.Experts.from_host(sh), mode=moe.MOE_MODE_PREFILL,
                   out_dtype=moe.MOE_OUT_F32)
    b = moe.MoEFFN(moe.Experts.from_host(ex), T, K, moe.Experts.from_host(sh), out_dtype=moe.MOE_OUT_F32,
                   fused_combine=True)
    oa = a(bf16_tensor(x), dev(lg)).double().cpu().numpy()
    ob = b(bf16_tensor(x), dev(lg)).double().cpu().numpy()
    torch.cuda.synchronize()
    ys = a.y_sorted.float().abs().cpu().numpy()
    inv = a.inv_route.cpu().numpy().reshape(T, K)
    bound = ys[inv].sum(axis=1) + np.abs(a.y_shared.float().cpu().numpy())
    assert np.all(np.abs(oa - ob) <= (K + 2) * 2.0 ** -23 * bound + 1e-30)
