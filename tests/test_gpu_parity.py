"""Parity of the CUDA path (through the C ABI) with the CPU oracle.

Routing ids and the sort maps must match bit for bit; route weights within
1e-5 relative; FFN outputs within rel-L2 <= 5e-3 and max-abs <= 1e-2 *
max|oracle| + 1e-3.  The five workloads run in the launch configuration the
benchmark uses (AUTO mode) and the FFN in each of its forms; the first four
are compared on every row and token, the largest (32768 tokens at width
8192) on every routing and sort output and on a seeded sample of 2048 tokens
and 2048 sorted rows plus every expert's first row.
"""
import numpy as np
import pytest
import torch

import mixture_experts_ffn_sort_b200 as moe
import oracle
from mixture_experts_ffn_sort_b200 import workloads as wl

from _gpu_util import (W_ATOL, W_RTOL, DeviceWorkload, assert_moe_close, bf16_numpy, bf16_tensor,
                       device_workload, oracle_maps, sample_tokens, to_f64, workload)

pytestmark = pytest.mark.gpu

ALL = wl.SHAPE_ORDER
FULL = {"tiny", "decode", "decode_skew", "prefill"}   # compared on every row
SAMPLE_ROWS = 2048
MODES = [moe.MOE_MODE_DECODE, moe.MOE_MODE_PREFILL, moe.MOE_MODE_HYBRID]


@pytest.fixture(scope="module", params=ALL)
def cfg(request):
    return request.param


_oracle_cache = {}


def oracle_full(name):
    if name not in _oracle_cache:
        _oracle_cache.clear()
        _oracle_cache[name] = oracle.workload(workload(name))
    return _oracle_cache[name]


def dev(a, dtype=None):
    t = torch.from_numpy(np.ascontiguousarray(a)).cuda()
    return t if dtype is None else t.to(dtype)


def oracle_y_rows(w, maps, positions):
    """Oracle y_sorted rows at the given sorted positions (w[r] * FFN_e(x[t]))."""
    off, sr, wt = maps["offsets"], maps["sorted_route"], maps["w"].ravel()
    K = w.shape.K
    experts = np.searchsorted(off, positions, side="right") - 1
    out = np.empty((len(positions), w.shape.H))
    for e in np.unique(experts):
        idx = np.nonzero(experts == e)[0]
        r = sr[positions[idx]]
        y = oracle.expert_rows(w.x, w.routed, int(e), (r // K).astype(np.int32))
        out[idx] = y * wt[r][:, None]
    return out


# ---------------------------------------------------------------- the five workloads

def test_route(cfg):
    w, dw, m = workload(cfg), device_workload(cfg), oracle_maps(cfg)
    ids, wts = moe.moe_route(dw.logits, w.shape.K, dw.zero_mask)
    torch.cuda.synchronize()
    assert np.array_equal(ids.cpu().numpy(), m["ids"])
    np.testing.assert_allclose(wts.cpu().numpy(), m["w"], rtol=W_RTOL, atol=W_ATOL)
    if w.zero_mask is not None:
        assert np.all(wts.cpu().numpy()[w.zero_mask == 1] == 0.0)


def test_sort(cfg):
    w, m = workload(cfg), oracle_maps(cfg)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    off, sr, inv = moe.moe_sort(dev(m["ids"]), w.shape.E, status)
    torch.cuda.synchronize()
    assert np.array_equal(off.cpu().numpy(), m["offsets"])
    assert np.array_equal(sr.cpu().numpy(), m["sorted_route"])
    assert np.array_equal(inv.cpu().numpy(), m["inv_route"])
    assert status.item() == 0


@pytest.mark.parametrize("mode", MODES)
def test_expert_ffn(cfg, mode):
    if cfg == "prefill_large" and mode == moe.MOE_MODE_DECODE:
        pytest.skip("the weight-streaming form re-reads a hot expert's weights per 8-row group")
    w, dw, m = workload(cfg), device_workload(cfg), oracle_maps(cfg)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    y, ys = moe.moe_expert_ffn(dw.x, w.shape.K, dw.routed, dev(m["offsets"]), dev(m["sorted_route"]),
                               dev(m["w"], torch.float32), dw.shared, mode=mode, status=status)
    torch.cuda.synchronize()
    assert status.item() == 0
    R = w.shape.R
    if cfg in FULL:
        ref = oracle_full(cfg)["y_sorted"]
        assert_moe_close(y, ref, "y_sorted")
        if w.shared is not None:
            assert_moe_close(ys, oracle_full(cfg)["y_shared"], "y_shared")
    else:
        pos = np.unique(np.concatenate([sample_tokens(R, SAMPLE_ROWS, seed=1), m["offsets"][:-1].clip(0, R - 1)]))
        assert_moe_close(to_f64(y[torch.from_numpy(pos).long().cuda()]), oracle_y_rows(w, m, pos), "y_sorted rows")
        if w.shared is not None:
            tk = sample_tokens(w.shape.T, 256, seed=2)
            ref = oracle.expert_rows(w.x, w.shared, 0, tk)
            assert_moe_close(to_f64(ys[torch.from_numpy(tk).long().cuda()]), ref, "y_shared rows")


def test_pipeline(cfg):
    w, dw = workload(cfg), device_workload(cfg)
    layer = moe.MoEFFN(dw.routed, w.shape.T, w.shape.K, dw.shared)
    out = layer(dw.x, dw.logits, dw.zero_mask)
    torch.cuda.synchronize()
    assert layer.status.item() == 0
    if cfg in FULL:
        assert_moe_close(out, oracle_full(cfg)["out"], "out")
    else:
        tk = sample_tokens(w.shape.T, SAMPLE_ROWS, seed=3)
        ref = oracle.moe_tokens(w.x, w.logits, w.shape.K, w.routed, w.shared, w.zero_mask, tokens=tk)
        assert_moe_close(to_f64(out[torch.from_numpy(tk).long().cuda()]), ref, "out rows")


def test_pipeline_fused_combine(cfg):
    """The layer with moe_expert_ffn_combine (no y_sorted) on the workloads the
    tensor-core form serves: every token of the 8192-token prefill, sampled
    tokens of the large one."""
    if cfg not in ("prefill", "prefill_large", "decode_skew"):
        pytest.skip("the fused combine runs the tensor-core form")
    w, dw = workload(cfg), device_workload(cfg)
    layer = moe.MoEFFN(dw.routed, w.shape.T, w.shape.K, dw.shared, fused_combine=True)
    out = layer(dw.x, dw.logits, dw.zero_mask)
    torch.cuda.synchronize()
    assert layer.status.item() == 0
    if cfg in FULL:
        assert_moe_close(out, oracle_full(cfg)["out"], "out")
    else:
        tk = sample_tokens(w.shape.T, SAMPLE_ROWS, seed=3)
        ref = oracle.moe_tokens(w.x, w.logits, w.shape.K, w.routed, w.shared, w.zero_mask, tokens=tk)
        assert_moe_close(to_f64(out[torch.from_numpy(tk).long().cuda()]), ref, "out rows")


# ---------------------------------------------------------------- edge cases

def _small(T, H, I, E, K, seed=0, shared_I=0, std=0.05):
    ex = wl.draw_experts(seed, 50, E, I, H, std, threads=4)
    sh = wl.draw_experts(seed, 51, 1, shared_I, H, std, threads=1) if shared_I else None
    x = wl.random_rows_bf16(T, H, seed=seed + 3)
    lg = np.random.default_rng(seed + 4).standard_normal((T, E)).astype(np.float32)
    return x, lg, ex, sh


def _run_pipeline(x, lg, K, ex, sh=None, zero_mask=None, out_dtype=moe.MOE_OUT_BF16, mode=moe.MOE_MODE_AUTO):
    T = x.shape[0]
    layer = moe.MoEFFN(moe.Experts.from_host(ex), T, K, moe.Experts.from_host(sh) if sh else None,
                       mode=mode, out_dtype=out_dtype)
    out = layer(bf16_tensor(x), dev(lg), dev(zero_mask) if zero_mask is not None else None)
    torch.cuda.synchronize()
    assert layer.status.item() == 0
    return out, layer


@pytest.mark.parametrize("T,H,I,E,K,Is", [(1, 128, 128, 4, 1, 0), (3, 256, 128, 8, 8, 0), (37, 384, 256, 16, 3, 128),
                                          (300, 128, 128, 4, 2, 0), (5, 1024, 384, 1, 1, 256),
                                          (129, 512, 128, 32, 4, 0)])
@pytest.mark.parametrize("mode", MODES)
def test_edge_shapes(T, H, I, E, K, Is, mode):
    x, lg, ex, sh = _small(T, H, I, E, K, seed=T, shared_I=Is)
    out, _ = _run_pipeline(x, lg, K, ex, sh, mode=mode)
    ref = oracle.moe(x, lg, K, ex, sh)["out"]
    assert_moe_close(out, ref, "out")
    out32, _ = _run_pipeline(x, lg, K, ex, sh, out_dtype=moe.MOE_OUT_F32, mode=mode)
    assert out32.dtype == torch.float32
    assert_moe_close(out32, ref, "out f32")


@pytest.mark.parametrize("n_hot", [7, 8, 9, 15, 16, 17, 31, 32, 33, 65, 127, 128, 129])
@pytest.mark.parametrize("mode", MODES)
def test_group_size_boundaries(n_hot, mode):
    """One expert receives exactly n_hot routes (around the kernels' token tiles)."""
    T, H, I, E, K = n_hot, 256, 128, 6, 2
    ex = wl.draw_experts(7, 52, E, I, H, 0.05, threads=4)
    x = wl.random_rows_bf16(T, H, seed=n_hot)
    ids = wl.skewed_ids(T, K, E, hot=2, seed=n_hot)
    off, sr, inv, _ = oracle.sort(ids, E)
    wt = np.random.default_rng(n_hot).random((T, K))
    y, _ = moe.moe_expert_ffn(bf16_tensor(x), K, moe.Experts.from_host(ex), dev(off), dev(sr), dev(wt, torch.float32),
                              mode=mode)
    torch.cuda.synchronize()
    ref = oracle.ffn_sorted(x, K, ex, off, sr, wt.astype(np.float32).astype(np.float64))
    assert_moe_close(y, ref, "y_sorted")


@pytest.mark.parametrize("kind", ["subnormal", "all_codes"])
@pytest.mark.parametrize("mode", MODES)
def test_special_fp8_codes(kind, mode):
    T, H, I, E, K = 24, 256, 128, 2, 1
    ex = (wl.subnormal_experts if kind == "subnormal" else wl.all_code_experts)(E, I, H, seed=3)
    x = wl.random_rows_bf16(T, H, seed=11)
    lg = np.random.default_rng(5).standard_normal((T, E)).astype(np.float32)
    out, _ = _run_pipeline(x, lg, K, ex, mode=mode)
    assert_moe_close(out, oracle.moe(x, lg, K, ex)["out"], kind)


@pytest.mark.parametrize("mode", MODES)
def test_zero_weight_routes_contribute_zero(mode):
    T, H, I, E, K = 64, 256, 128, 8, 3
    x, lg, ex, _ = _small(T, H, I, E, K, seed=9)
    mask = (np.random.default_rng(1).random((T, K)) < 0.3).astype(np.uint8)
    out, layer = _run_pipeline(x, lg, K, ex, zero_mask=mask, mode=mode)
    inv = layer.inv_route.cpu().numpy().reshape(T, K)
    y = layer.y_sorted.float().cpu().numpy()
    assert np.all(y[inv[mask == 1]] == 0.0)
    assert_moe_close(out, oracle.moe(x, lg, K, ex, zero_mask=mask)["out"], "out")


@pytest.mark.parametrize("mode", MODES)
def test_token_permutation_is_bit_exact(mode):
    T, H, I, E, K = 96, 256, 256, 8, 2
    x, lg, ex, _ = _small(T, H, I, E, K, seed=13)
    perm = np.random.default_rng(2).permutation(T)
    a, _ = _run_pipeline(x, lg, K, ex, mode=mode)
    a = bf16_numpy(a)
    b, _ = _run_pipeline(x[perm], lg[perm], K, ex, mode=mode)
    assert np.array_equal(a[perm], bf16_numpy(b))


def test_route_ties():
    lg = wl.tie_logits(200, 64, seed=3, levels=3)
    ids, wts = moe.moe_route(dev(lg), 8)
    oid, ow = oracle.route(lg, 8)
    assert np.array_equal(ids.cpu().numpy(), oid)
    np.testing.assert_allclose(wts.cpu().numpy(), ow, rtol=W_RTOL, atol=W_ATOL)


# Single-block sort (R <= 16384) and tiled sort (2048-route tiles of 8 x 256):
# exact tiles, a partial last tile, a partial last warp, R just above the
# single-block limit, one expert, E = MOE_MAX_E.
@pytest.mark.parametrize("T,K,E", [(1024, 32, 1024), (700, 10, 512), (5000, 8, 3), (1, 1, 1), (16384, 1, 64),
                                   (16385, 1, 7), (4097, 4, 513), (20480, 1, 1), (2305, 8, 256), (512, 8, 256)])
def test_sort_shapes(T, K, E):
    ids = wl.random_ids(T, K, E, seed=T, distinct=E >= K) if E >= K else \
        np.random.default_rng(0).integers(0, E, (T, K)).astype(np.int32)
    off, sr, inv = moe.moe_sort(dev(ids), E)
    o = oracle.sort(ids, E)
    assert np.array_equal(off.cpu().numpy(), o[0])
    assert np.array_equal(sr.cpu().numpy(), o[1])
    assert np.array_equal(inv.cpu().numpy(), o[2])


@pytest.mark.parametrize("T", [100, 4000, 6000])
def test_sort_out_of_range_ids_are_skipped(T):
    K, E = 4, 16
    ids = wl.random_ids(T, K, E, seed=5)
    ids[3, 1] = 16
    ids[T - 1, 0] = -2
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    off, sr, inv = moe.moe_sort(dev(ids), E, status)
    o = oracle.sort(ids, E)
    assert status.item() & moe.MOE_STATUS_BAD_ID
    assert np.array_equal(off.cpu().numpy(), o[0])
    assert np.array_equal(sr.cpu().numpy(), o[1])
    assert np.array_equal(inv.cpu().numpy(), o[2])


def test_ffn_flags_corrupt_offsets():
    T, H, I, E, K = 8, 128, 128, 2, 1
    ex = wl.draw_experts(1, 53, E, I, H, 0.05, threads=1)
    x = wl.random_rows_bf16(T, H, seed=1)
    off = np.array([0, 5, 99], np.int32)             # offsets[E] beyond T*K
    sr = np.arange(T, dtype=np.int32)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    moe.moe_expert_ffn(bf16_tensor(x), K, moe.Experts.from_host(ex), dev(off), dev(sr),
                       torch.ones(T, 1, device="cuda"), status=status)
    torch.cuda.synchronize()
    assert status.item() & moe.MOE_STATUS_BAD_MAP


@pytest.mark.parametrize("K,shared", [(1, False), (4, True), (11, False)])
def test_combine_step(K, shared):
    T, E, H = 333, 16, 264
    ids = wl.random_ids(T, K, E, seed=K)
    off, sr, inv, _ = oracle.sort(ids, E)
    ys = wl.random_rows_bf16(T * K, H, seed=K)
    sh = wl.random_rows_bf16(T, H, seed=K + 1) if shared else None
    ref = oracle.combine_bf16(ys, inv, sh, T, K)
    terms = oracle.combine(np.abs(oracle.bf16_array(ys)), inv,
                           np.abs(oracle.bf16_array(sh)) if shared else None, T, K)   # sum of |terms|
    o32 = moe.moe_combine(bf16_tensor(ys), dev(inv), bf16_tensor(sh) if shared else None, T, K, moe.MOE_OUT_F32)
    o16 = moe.moe_combine(bf16_tensor(ys), dev(inv), bf16_tensor(sh) if shared else None, T, K, moe.MOE_OUT_BF16)
    torch.cuda.synchronize()
    g32 = to_f64(o32)
    bound = (K + 2) * 2.0 ** -24 * terms       # fp32 summation of K+1 terms
    assert np.all(np.abs(g32 - ref) <= bound)
    g16 = to_f64(o16)
    assert np.all(np.abs(g16 - ref) <= 2.0 ** -8 * np.abs(ref) + 2 * bound)


def test_combine_skips_and_flags_corrupt_positions():
    """inv_route entries outside [0, T*K) (other than -1) are skipped, never
    read, and set MOE_STATUS_BAD_MAP; the rest sums as if they were -1."""
    T, K, E, H = 100, 4, 8, 64
    ids = wl.random_ids(T, K, E, seed=31)
    off, sr, inv, _ = oracle.sort(ids, E)
    ys = wl.random_rows_bf16(T * K, H, seed=31)
    bad = inv.copy()
    bad[5] = T * K                 # one past the end
    bad[17] = 1 << 30              # far out of range
    bad[42] = -3                   # negative, not the skip marker
    clean = bad.copy()
    clean[[5, 17, 42]] = -1
    ref = oracle.combine(oracle.bf16_array(ys), clean, None, T, K)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    o32 = moe.moe_combine(bf16_tensor(ys), dev(bad), None, T, K, moe.MOE_OUT_F32, status=status)
    torch.cuda.synchronize()
    assert status.item() & moe.MOE_STATUS_BAD_MAP
    terms = oracle.combine(np.abs(oracle.bf16_array(ys)), clean, None, T, K)
    assert np.all(np.abs(to_f64(o32) - ref) <= (K + 2) * 2.0 ** -24 * terms)
    status.zero_()
    moe.moe_combine(bf16_tensor(ys), dev(inv), None, T, K, moe.MOE_OUT_F32, status=status)
    torch.cuda.synchronize()
    assert status.item() == 0


def test_outputs_fully_written():
    """NaN-poisoned outputs and scratch: every row the maps cover is written."""
    T, H, I, E, K = 50, 256, 256, 8, 2
    x, lg, ex, sh = _small(T, H, I, E, K, seed=21, shared_I=128)
    layer = moe.MoEFFN(moe.Experts.from_host(ex), T, K, moe.Experts.from_host(sh))
    for t in (layer.y_sorted, layer.y_shared, layer.out):
        t.fill_(float("nan"))
    layer.ffn_ws.fill_(0xFF)
    out = layer(bf16_tensor(x), dev(lg))
    torch.cuda.synchronize()
    assert torch.isfinite(layer.y_sorted.float()).all()
    assert torch.isfinite(layer.y_shared.float()).all()
    assert_moe_close(out, oracle.moe(x, lg, K, ex, sh)["out"], "out")


def test_graph_replay_with_changing_routes():
    """The four calls captured once in a CUDA graph, replayed on new inputs
    (new routes and zero weights each time), as the aiter PR's replay test."""
    T, H, I, E, K = 64, 512, 256, 32, 4
    ex = wl.draw_experts(3, 54, E, I, H, 0.05, threads=4)
    layer = moe.MoEFFN(moe.Experts.from_host(ex), T, K)
    x_s = torch.zeros(T, H, dtype=torch.bfloat16, device="cuda")
    lg_s = torch.zeros(T, E, dtype=torch.float32, device="cuda")
    zm_s = torch.zeros(T, K, dtype=torch.uint8, device="cuda")
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        layer(x_s, lg_s, zm_s)            # first call outside capture (one-time set-up)
    torch.cuda.current_stream().wait_stream(s)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        layer(x_s, lg_s, zm_s)
    for it in range(3):
        x = wl.random_rows_bf16(T, H, seed=100 + it)
        lg = np.random.default_rng(200 + it).standard_normal((T, E)).astype(np.float32)
        zm = (np.random.default_rng(300 + it).random((T, K)) < 0.1).astype(np.uint8)
        x_s.copy_(bf16_tensor(x))
        lg_s.copy_(dev(lg))
        zm_s.copy_(dev(zm))
        g.replay()
        torch.cuda.synchronize()
        assert_moe_close(layer.out, oracle.moe(x, lg, K, ex, zero_mask=zm)["out"], "replay %d" % it)
