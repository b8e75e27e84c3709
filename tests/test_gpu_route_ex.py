"""GPU parity of the routing variants (moe_route_ex) with the CPU oracle.

Where the choice is taken on computed scores (a selection bias or a group
limit), the kernel ranks by its fp32 scores and the oracle by fp64 ones: a
token may then pick differently only between experts whose scores tie to fp32
rounding.  Such a token must be rare, and its choice must be as good as the
oracle's (the same selection scores, rank by rank, to a few fp32 ulps); its
weights are the oracle's weights for the kernel's choice.  Without bias and
groups the ranking compares the fp32 logits and must match exactly.
"""
import numpy as np
import pytest
import torch

import mixture_experts_ffn_sort_b200 as moe
import oracle
from mixture_experts_ffn_sort_b200 import workloads as wl

from _gpu_util import W_ATOL, W_RTOL

pytestmark = pytest.mark.gpu

SIG, SMX = oracle.SCORE_SIGMOID, oracle.SCORE_SOFTMAX
# Two selection scores "tie to fp32 rounding" within this many units of 2^-24.
TIE_ULPS = 8.0


def _logits(T, E, seed, scale=1.0):
    return (np.random.default_rng(seed).standard_normal((T, E)) * scale).astype(np.float32)


def _run(lg, K, score=SMX, bias=None, n_group=1, topk_group=None, renormalize=True, scaling=1.0,
         zero_mask=None):
    tg = n_group if topk_group is None else topk_group
    ids, w = moe.moe_route_ex(torch.from_numpy(lg).cuda(), K, score=score,
                              sel_bias=None if bias is None else torch.from_numpy(bias).cuda(),
                              n_group=n_group, topk_group=tg, renormalize=renormalize, scaling=scaling,
                              zero_mask=None if zero_mask is None else torch.from_numpy(zero_mask).cuda())
    torch.cuda.synchronize()
    oid, ow = oracle.route_ex(lg, K, score=score, bias=bias, n_group=n_group, topk_group=tg,
                              renormalize=renormalize, scaling=scaling, zero_mask=zero_mask)
    return ids.cpu().numpy(), w.cpu().numpy(), oid, ow


def _check(lg, K, score=SMX, bias=None, n_group=1, topk_group=None, renormalize=True, scaling=1.0,
           zero_mask=None, max_tie_frac=0.01):
    ids, w, oid, ow = _run(lg, K, score, bias, n_group, topk_group, renormalize, scaling, zero_mask)
    T, E = lg.shape
    assert ids.shape == (T, K) and np.all((ids >= 0) & (ids < E))
    assert all(len(set(r)) == K for r in ids), "repeated expert in a token's choice"
    differ = np.any(ids != oid, axis=1)
    if bias is None and n_group == 1:
        assert not differ.any(), "ranking by the fp32 logit must match exactly"
    elif differ.any():
        assert differ.mean() <= max_tie_frac, "%d of %d tokens differ" % (differ.sum(), T)
        c = oracle.route_select_scores(lg, score, bias)
        for t in np.nonzero(differ)[0]:
            cg, co = c[t, ids[t]], c[t, oid[t]]
            tol = TIE_ULPS * 2.0 ** -24 * np.maximum(1.0, np.abs(co))
            assert np.all(np.abs(np.sort(cg)[::-1] - co) <= tol), (t, ids[t], oid[t])
            assert np.all(np.diff(cg) <= tol[1:]), "kernel order not descending (token %d)" % t
    ref_w = oracle.route_weights(lg, ids, score=score, renormalize=renormalize, scaling=scaling)
    if zero_mask is not None:
        ref_w[zero_mask != 0] = 0.0
        assert np.all(w[zero_mask != 0] == 0.0)
    np.testing.assert_allclose(w, ref_w, rtol=W_RTOL, atol=W_ATOL)
    return differ.sum()


def test_route_ex_default_matches_route():
    lg = wl.tie_logits(300, 64, seed=1, levels=3)
    ids, w = moe.moe_route(torch.from_numpy(lg).cuda(), 8)
    ids2, w2 = moe.moe_route_ex(torch.from_numpy(lg).cuda(), 8)
    assert torch.equal(ids, ids2)
    torch.testing.assert_close(w2, w, rtol=W_RTOL, atol=W_ATOL)
    _check(lg, 8)


@pytest.mark.parametrize("T,E,K,scaling,renorm", [(1000, 128, 6, 2.5, False), (777, 128, 6, 2.5, True),
                                                  (64, 32, 32, 1.0, True), (500, 20, 3, 0.75, False)])
def test_route_ex_sigmoid(T, E, K, scaling, renorm):
    """Nemotron-style sigmoid top-k with a routed scaling factor."""
    _check(_logits(T, E, T + E, scale=2.0), K, score=SIG, renormalize=renorm, scaling=scaling)


def test_route_ex_sigmoid_ties_go_to_lower_id():
    _check(wl.tie_logits(400, 48, seed=5, levels=3), 7, score=SIG, scaling=2.0)


def test_route_ex_zero_bias_ties_go_to_lower_id():
    """A zero bias makes the ranking use the computed scores; equal logits
    still give equal scores, so ties resolve to the lower id exactly."""
    lg = wl.tie_logits(400, 48, seed=6, levels=3)
    ids, _, oid, _ = _run(lg, 7, score=SIG, bias=np.zeros(48, np.float32))
    assert np.array_equal(ids, oid)


@pytest.mark.parametrize("score", [SIG, SMX])
def test_route_ex_deepseek_v3_shape(score):
    """256 experts in 8 groups, 4 kept, top-8, selection bias, scaling 2.5."""
    rng = np.random.default_rng(21)
    bias = (rng.standard_normal(256) * 0.02).astype(np.float32)
    _check(_logits(2048, 256, 22), 8, score=score, bias=bias, n_group=8, topk_group=4, scaling=2.5)


@pytest.mark.parametrize("E,n_group,topk_group,K", [(96, 3, 2, 5), (40, 5, 2, 4), (1000, 8, 3, 10),
                                                    (64, 32, 16, 8), (16, 16, 5, 3), (512, 8, 4, 10),
                                                    (24, 2, 1, 12)])
def test_route_ex_group_shapes(E, n_group, topk_group, K):
    """Group sizes that are not multiples of the warp, one expert per group,
    32 groups (one per lane), and E up to 1000."""
    rng = np.random.default_rng(E + K)
    bias = (rng.random(E) * 0.2 - 0.1).astype(np.float32)
    _check(_logits(600, E, E * 7), K, score=SIG, bias=bias, n_group=n_group, topk_group=topk_group,
           scaling=1.5)
    _check(_logits(300, E, E * 9), K, score=SMX, n_group=n_group, topk_group=topk_group)


def test_route_ex_bias_without_groups_and_zero_mask():
    rng = np.random.default_rng(31)
    E, K = 160, 6
    bias = (rng.standard_normal(E) * 0.05).astype(np.float32)
    mask = (rng.random((900, K)) < 0.05).astype(np.uint8)
    _check(_logits(900, E, 32), K, score=SIG, bias=bias, scaling=2.5, zero_mask=mask)


def test_route_ex_large_bias_forces_the_set():
    E, K = 64, 4
    bias = np.zeros(E, np.float32)
    S = [5, 17, 40, 63]
    bias[S] = 50.0
    lg = _logits(200, E, 33)
    ids, w, _, _ = _run(lg, K, score=SIG, bias=bias)
    assert all(set(r) == set(S) for r in ids)
    _check(lg, K, score=SIG, bias=bias)


@pytest.mark.parametrize("router", ["sigmoid", "grouped"])
@pytest.mark.parametrize("workload,mode", [("tiny", moe.MOE_MODE_AUTO), ("decode", moe.MOE_MODE_DECODE),
                                           ("decode", moe.MOE_MODE_PREFILL)])
def test_layer_with_router_variant(workload, mode, router):
    """The whole path with a routing variant: the layer's expert choice agrees
    with the oracle router (up to fp32 score ties) and its output equals the
    brute-force oracle FFN for that choice and the oracle's weights."""
    from _gpu_util import assert_moe_close, device_workload
    shape = wl.SHAPES[workload]
    dw = device_workload(workload)
    w = dw.w
    cfg = dict(wl.ROUTERS[router])
    use_bias = cfg.pop("bias", False)
    bias = wl.selection_bias(shape.E, shape.seed) if use_bias else None
    dev = torch.device("cuda")
    route_cfg = dict(cfg, sel_bias=None if bias is None else torch.from_numpy(bias).to(dev))
    layer = moe.MoEFFN(dw.routed, shape.T, shape.K, dw.shared, mode=mode, device=dev, route_cfg=route_cfg)
    out = layer(dw.x, dw.logits, dw.zero_mask)
    torch.cuda.synchronize()
    assert layer.status.item() == 0
    ids = layer.topk_ids.cpu().numpy()
    oid, _ = oracle.route_ex(w.logits, shape.K, bias=bias, zero_mask=w.zero_mask, **cfg)
    differ = np.any(ids != oid, axis=1)
    assert differ.mean() <= 0.01
    wt = oracle.route_weights(w.logits, ids, score=cfg["score"], renormalize=cfg["renormalize"],
                              scaling=cfg["scaling"])
    if w.zero_mask is not None:
        wt[w.zero_mask != 0] = 0.0
    np.testing.assert_allclose(layer.topk_w.cpu().numpy(), wt, rtol=W_RTOL, atol=W_ATOL)
    ref = oracle.moe_tokens_routed(w.x, ids, wt, w.routed, w.shared)
    assert_moe_close(out, ref, "%s/%s" % (workload, router))
