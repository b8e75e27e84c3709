"""GPU parity of the fused router (moe_router: gate GEMM + top-K) with the CPU
oracle (fp64 gate GEMM, rounded to the fp32 logit type, then the routing step).

The kernel sums the bf16 products on the tensor cores in fp32, so its logits
differ from the exact ones by fp32 rounding: at most LOGIT_RTOL times
sum_h |x_h w_h| per logit, checked on every logit.  A token may therefore
choose differently from the oracle only between experts whose scores lie that
close (at most 2 * LOGIT_RTOL * sum|x w| apart, every score here changes by at
most the logit change); its choice must be as good as the oracle's, rank by
rank, within that window, and most tokens must match exactly.  Where the
choices agree the weights agree to the same window.
"""
import numpy as np
import pytest
import torch

import mixture_experts_ffn_sort_b200 as moe
import oracle
from mixture_experts_ffn_sort_b200 import workloads as wl

pytestmark = pytest.mark.gpu

SIG, SMX = oracle.SCORE_SIGMOID, oracle.SCORE_SOFTMAX
# fp32 accumulation of up to 16384 bf16 products: observed errors are far
# below this bound on sum |x w| (which itself is far below the worst case).
LOGIT_RTOL = 1e-5


def _abs_dot(x_bits, w_bits):
    xa = np.abs(oracle.bf16_array(x_bits))
    wa = np.abs(oracle.bf16_array(w_bits))
    return xa @ wa.T


def _run(x, w, K, tokens=None, want_logits=True, **kw):
    """Kernel on all T tokens; the oracle on `tokens` (all if None)."""
    T, H = x.shape
    E = w.shape[0]
    route_kw = dict(kw)
    bias = route_kw.pop("bias", None)
    zero_mask = route_kw.pop("zero_mask", None)
    dev_lg = torch.full((T, E), float("nan"), dtype=torch.float32, device="cuda") if want_logits else None
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    xt = torch.from_numpy(x.view(np.int16)).cuda()
    wt = torch.from_numpy(w.view(np.int16)).cuda()
    ids, wts = moe.moe_router(xt, wt, K, sel_bias=None if bias is None else torch.from_numpy(bias).cuda(),
                              zero_mask=None if zero_mask is None else torch.from_numpy(zero_mask).cuda(),
                              logits=dev_lg, status=status, **route_kw)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    tok = np.arange(T) if tokens is None else np.asarray(tokens)
    okw = dict(route_kw)
    okw.pop("topk_group", None)
    tg = kw.get("topk_group") or kw.get("n_group", 1)
    zm = None if zero_mask is None else zero_mask[tok]
    l64, l32, oid, ow = oracle.router(x[tok], w, K, bias=bias, topk_group=tg, zero_mask=zm, **okw)
    return dict(ids=ids.cpu().numpy()[tok], w=wts.cpu().numpy()[tok],
                logits=None if dev_lg is None else dev_lg.cpu().numpy()[tok],
                l64=l64, l32=l32, oid=oid, ow=ow, absdot=_abs_dot(x[tok], w), bias=bias)


def _check(r, K, E, score=SMX, n_group=1, scaling=1.0, min_match=0.95, **_):
    tol = LOGIT_RTOL * r["absdot"] + 1e-6           # per logit
    if r["logits"] is not None:
        err = np.abs(r["logits"].astype(np.float64) - r["l64"])
        assert np.all(err <= tol), "logit error %.3g above bound at %s" % (err.max(), np.unravel_index(
            np.argmax(err - tol), err.shape))
    ids, oid = r["ids"], r["oid"]
    n = ids.shape[0]
    assert np.all((ids >= 0) & (ids < E))
    assert all(len(set(row)) == K for row in ids), "repeated expert in a token's choice"
    same = np.all(ids == oid, axis=1)
    assert same.mean() >= min_match, "%d of %d tokens differ" % ((~same).sum(), n)
    # Selection scores of the oracle (fp64 from its fp32 logits); every
    # variant's score moves by at most the logit error.
    c = oracle.route_select_scores(r["l32"], score, r["bias"])
    win = 2.0 * tol.max(axis=1) + 1e-6               # per token
    for t in np.nonzero(~same)[0]:
        if n_group > 1:
            continue  # a near-tie between groups may change the eligible set; ids checked above
        cg, co = c[t, ids[t]], c[t, oid[t]]
        assert np.all(np.abs(cg - co) <= win[t]), (t, ids[t], oid[t], cg - co)
    wtol = scaling * (2.0 * win[:, None] + 2e-6)
    assert np.all(np.abs(r["w"][same] - r["ow"][same]) <= wtol[same]), np.abs(r["w"][same] - r["ow"][same]).max()


# (T, H, E, K): cluster sizes 1, 2, 4 and 8, ragged token tiles, expert counts
# that are not a multiple of 16 or of the cluster's slice, one K stage.
SHAPES = [(16, 256, 8, 2), (64, 2048, 256, 8), (300, 1024, 512, 10), (200, 256, 40, 6),
          (129, 512, 100, 7), (1000, 64, 128, 4), (130, 4096, 512, 10), (7, 128, 300, 32)]


@pytest.mark.parametrize("T,H,E,K", SHAPES)
def test_router_plain_softmax(T, H, E, K):
    x = wl.random_rows_bf16(T, H, seed=T + H)
    w = wl.router_weight(E, H, seed=E)
    r = _run(x, w, K)
    _check(r, K, E)


@pytest.mark.parametrize("variant", ["sigmoid", "grouped", "softmax_norenorm", "softmax_bias"])
def test_router_variants(variant):
    T, H, E, K = 384, 2048, 256, 8
    x = wl.random_rows_bf16(T, H, seed=11)
    w = wl.router_weight(E, H, seed=12)
    kw = dict(sigmoid=dict(score=SIG, scaling=2.5),
              grouped=dict(score=SIG, n_group=8, topk_group=4, scaling=2.5, bias=wl.selection_bias(E, 1, 0.05)),
              softmax_norenorm=dict(score=SMX, renormalize=False),
              softmax_bias=dict(score=SMX, bias=wl.selection_bias(E, 2, 0.001)))[variant]
    r = _run(x, w, K, **kw)
    _check(r, K, E, **kw)


def test_router_zero_mask_and_no_logit_copy():
    T, H, E, K = 256, 1024, 64, 6
    x = wl.random_rows_bf16(T, H, seed=21)
    w = wl.router_weight(E, H, seed=22)
    zm = (np.random.default_rng(23).random((T, K)) < 0.1).astype(np.uint8)
    r = _run(x, w, K, want_logits=False, zero_mask=zm)
    _check(r, K, E)
    same = np.all(r["ids"] == r["oid"], axis=1)
    assert np.all(r["w"][zm.astype(bool) & same[:, None]] == 0.0)


def test_router_full_size_sampled():
    """8192 tokens x H 4096 x 512 experts, top-10 (the prefill router), in the
    launch configuration of the full-size call; the oracle on 192 sampled tokens
    from every part of the batch."""
    T, H, E, K = 8192, 4096, 512, 10
    x = wl.random_rows_bf16(T, H, seed=31)
    w = wl.router_weight(E, H, seed=32)
    tok = np.unique(np.concatenate([np.arange(64), np.arange(T - 64, T),
                                    np.random.default_rng(33).choice(T, 64, replace=False)]))
    r = _run(x, w, K, tokens=tok)
    _check(r, K, E)


def test_router_zero_tokens_is_a_no_op():
    w = torch.zeros((8, 128), dtype=torch.int16, device="cuda")
    x = torch.zeros((0, 128), dtype=torch.int16, device="cuda")
    ids, wts = moe.moe_router(x, w, 2)
    assert ids.shape == (0, 2) and wts.shape == (0, 2)


def test_router_feeds_the_path():
    """moe_router -> moe_sort -> moe_expert_ffn -> moe_combine (the layer's
    forward_fused) on the tiny workload equals the oracle's method with the
    oracle's own router."""
    wk = wl.make_workload("tiny")
    T, H, E, K = wk.shape.T, wk.shape.H, wk.shape.E, wk.shape.K
    w = wl.router_weight(E, H, seed=41)
    layer = moe.MoEFFN(moe.Experts.from_host(wk.routed), T, K,
                       w_router=torch.from_numpy(w.view(np.int16)).cuda())
    xt = torch.from_numpy(wk.x.view(np.int16)).cuda()
    out = layer.forward_fused(xt).float().cpu().numpy()
    l64, l32, oid, ow = oracle.router(wk.x, w, K)
    assert np.array_equal(layer.topk_ids.cpu().numpy(), oid)
    ref = oracle.moe_tokens_routed(wk.x, oid, ow, wk.routed)
    rel = np.linalg.norm(out - ref) / np.linalg.norm(ref)
    assert rel < 5e-3, rel


def test_router_graph_replay_with_changing_tokens():
    """The layer's fused-router forward captured once in a CUDA graph and
    replayed on new token rows: the routing follows x (the oracle's router on
    each new batch) and the output matches the oracle's method."""
    T, H, I, E, K = 64, 512, 256, 32, 4
    ex = wl.draw_experts(3, 55, E, I, H, 0.05, threads=4)
    wr = wl.router_weight(E, H, seed=56)
    layer = moe.MoEFFN(moe.Experts.from_host(ex), T, K, w_router=torch.from_numpy(wr.view(np.int16)).cuda())
    x_s = torch.zeros(T, H, dtype=torch.int16, device="cuda")
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        layer.forward_fused(x_s)          # first call outside capture (one-time set-up)
    torch.cuda.current_stream().wait_stream(s)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        layer.forward_fused(x_s)
    # Batches whose oracle top-K+1 logits are at least 1e-3 apart (a margin far
    # above the fp32 accumulation error), so the choice is unique.
    for it, seed in enumerate((402, 409, 412)):
        x = wl.random_rows_bf16(T, H, seed=seed)
        x_s.copy_(torch.from_numpy(x.view(np.int16)).cuda())
        g.replay()
        torch.cuda.synchronize()
        _, _, oid, ow = oracle.router(x, wr, K)
        assert np.array_equal(layer.topk_ids.cpu().numpy(), oid), "replay %d: ids" % it
        ref = oracle.moe_tokens_routed(x, oid, ow, ex)
        got = layer.out.double().cpu().numpy()
        rel = np.linalg.norm(got - ref) / np.linalg.norm(ref)
        assert rel < 5e-3, (it, rel)
