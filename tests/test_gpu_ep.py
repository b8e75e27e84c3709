"""Expert-parallel decode on one GPU: the ranks are run one after another
(no collective), and their fp32 partial outputs must add up to the
single-device layer and to the oracle."""
import numpy as np
import pytest
import torch

import mixture_experts_ffn_sort_b200 as moe
import oracle
from mixture_experts_ffn_sort_b200 import ep
from mixture_experts_ffn_sort_b200 import workloads as wl

from _gpu_util import assert_moe_close, bf16_tensor

pytestmark = pytest.mark.gpu


def _sum_of_ranks(w, world, mode):
    dev = torch.device("cuda")
    full = moe.Experts.from_host(w.routed, dev)
    shared = moe.Experts.from_host(w.shared, dev) if w.shared is not None else None
    x, lg = bf16_tensor(w.x), torch.from_numpy(w.logits).to(dev)
    zm = torch.from_numpy(w.zero_mask).to(dev) if w.zero_mask is not None else None
    T, E = w.logits.shape
    K = w.shape.K
    total = torch.zeros((T, w.x.shape[1]), dtype=torch.float32, device=dev)
    for r in range(world):
        layer = ep.ExpertParallelMoE(ep.local_experts(full, r, world), E, T, K, r, world, shared, mode=mode,
                                     device=dev)
        total += layer.partial(x, lg, zm)
        torch.cuda.synchronize()
        assert layer.status.item() == 0
    single = moe.MoEFFN(full, T, K, shared, mode=mode, out_dtype=moe.MOE_OUT_F32, device=dev)(x, lg, zm)
    torch.cuda.synchronize()
    return total, single


@pytest.mark.parametrize("world", [1, 2, 4, 8])
def test_ep_decode_workload(world):
    w = wl.make_workload("decode")
    total, single = _sum_of_ranks(w, world, moe.MOE_MODE_DECODE)
    # Same rows, added in another order: fp32 rounding only.
    torch.testing.assert_close(total, single, rtol=1e-5, atol=1e-5)
    ids, wt = oracle.route(w.logits, w.shape.K)
    tk = np.arange(0, w.logits.shape[0], 4, dtype=np.int32)
    ref = oracle.moe_tokens_routed(w.x, ids[tk], wt[tk], w.routed, None, tokens=tk)
    assert_moe_close(total.double().cpu().numpy()[tk], ref, "ep x%d" % world)


@pytest.mark.parametrize("world", [2, 4])
@pytest.mark.parametrize("mode", [moe.MOE_MODE_DECODE, moe.MOE_MODE_PREFILL])
def test_ep_with_shared_expert(world, mode):
    """The shared expert is added once (by rank 0)."""
    T, H, I, E, K, Is = 37, 384, 256, 16, 3, 128
    rng = np.random.default_rng(5)

    class W:
        pass
    w = W()
    w.x = wl.random_rows_bf16(T, H, seed=3)
    w.logits = rng.standard_normal((T, E)).astype(np.float32)
    w.routed = wl.draw_experts(7, 4, E, I, H)
    w.shared = wl.draw_experts(7, 5, 1, Is, H)
    w.zero_mask = None
    w.shape = type("S", (), {"K": K})()
    total, single = _sum_of_ranks(w, world, mode)
    torch.testing.assert_close(total, single, rtol=1e-5, atol=1e-5)
    ref = oracle.moe(w.x, w.logits, K, w.routed, w.shared)["out"]
    assert_moe_close(total.double().cpu().numpy(), ref, "ep shared x%d" % world)


def _exchange_emulated(layers, xs, lgs, zms):
    """Run the prefill ranks in one process: each exchange is a concatenation
    of the senders' row blocks in rank order, as all_to_all_single lays them out."""
    G = len(layers)
    disp = [layers[r].dispatch(xs[r], lgs[r], zms[r]) for r in range(G)]
    starts = [np.concatenate([[0], np.cumsum(d[3])]) for d in disp]  # rank s: first row for each destination
    ys = []
    for d in range(G):
        rx = torch.cat([disp[s][0][starts[s][d]:starts[s][d + 1]] for s in range(G)])
        rw = torch.cat([disp[s][1][starts[s][d]:starts[s][d + 1]] for s in range(G)])
        rc = torch.stack([disp[s][2][d] for s in range(G)])
        ys.append((layers[d].expert_rows(rx, rw, rc), [disp[s][3][d] for s in range(G)]))
    outs = []
    for s in range(G):
        back = []
        for d in range(G):
            y, from_each = ys[d]
            b = int(sum(from_each[:s]))
            back.append(y[b:b + from_each[s]])
        outs.append(layers[s].finish(torch.cat(back), xs[s], moe.MOE_OUT_F32))
    torch.cuda.synchronize()
    return outs


@pytest.mark.parametrize("world", [1, 2, 4])
def test_ep_prefill_all_to_all(world):
    """Token-sharded expert parallelism: every rank's output equals the
    single-device layer on its tokens and the oracle."""
    H, I, E, K, Is = 256, 128, 16, 3, 128
    Ts = [40, 33, 57, 21][:world]
    dev = torch.device("cuda")
    routed = wl.draw_experts(11, 4, E, I, H)
    shared = wl.draw_experts(11, 5, 1, Is, H)
    full = moe.Experts.from_host(routed, dev)
    sh = moe.Experts.from_host(shared, dev)
    xs_np = [wl.random_rows_bf16(T, H, seed=30 + r) for r, T in enumerate(Ts)]
    lg_np = [np.random.default_rng(40 + r).standard_normal((T, E)).astype(np.float32) for r, T in enumerate(Ts)]
    zm_np = [(np.random.default_rng(50 + r).random((T, K)) < 0.05).astype(np.uint8) for r, T in enumerate(Ts)]
    layers = [ep.ExpertParallelPrefill(ep.local_experts(full, r, world), E, Ts[r], K, r, world, sh, device=dev)
              for r in range(world)]
    outs = _exchange_emulated(layers, [bf16_tensor(a) for a in xs_np], [torch.from_numpy(a).to(dev) for a in lg_np],
                              [torch.from_numpy(a).to(dev) for a in zm_np])
    for r in range(world):
        assert layers[r].status.item() == 0
        single = moe.MoEFFN(full, Ts[r], K, sh, out_dtype=moe.MOE_OUT_F32, device=dev)(
            bf16_tensor(xs_np[r]), torch.from_numpy(lg_np[r]).to(dev), torch.from_numpy(zm_np[r]).to(dev))
        torch.cuda.synchronize()
        torch.testing.assert_close(outs[r], single, rtol=2e-2, atol=2e-3)
        ref = oracle.moe(xs_np[r], lg_np[r], K, routed, shared, zero_mask=zm_np[r])["out"]
        assert_moe_close(outs[r].double().cpu().numpy(), ref, "ep prefill rank %d of %d" % (r, world))
