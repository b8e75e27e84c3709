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
