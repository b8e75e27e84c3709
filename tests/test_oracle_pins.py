"""Pins of the CPU oracle to things other than itself (CPU only).

Each test checks one oracle function against a library routine (torch's FP8
and bf16 casts, torch.nn.functional, numpy's stable argsort, scipy's softmax,
Python's sorted), a closed form, an invariant of the method, or brute force on
tiny inputs.  The mistakes they are chosen to catch are named in each test.
"""
import numpy as np
import pytest
import scipy.special
import torch
import torch.nn.functional as F

import oracle
from mixture_experts_ffn_sort_b200 import workloads as wl


def _fp8_dense(codes: np.ndarray, scales: np.ndarray) -> torch.Tensor:
    """Library decode: torch's E4M3FN -> float64, times the block scale expanded
    with a Kronecker product (rows and cols of one block share one scale)."""
    v = torch.from_numpy(np.ascontiguousarray(codes)).view(torch.float8_e4m3fn).to(torch.float64)
    s = torch.from_numpy(np.kron(scales.astype(np.float64), np.ones((128, 128))))
    return v * s


def _torch_mlp(x64: torch.Tensor, ex, e: int) -> torch.Tensor:
    """The eager SwiGLU MLP (down(silu(gate(x)) * up(x))) with torch Linear ops."""
    wg = _fp8_dense(ex.w_gate[e], ex.s_gate[e])
    wu = _fp8_dense(ex.w_up[e], ex.s_up[e])
    wd = _fp8_dense(ex.w_down[e], ex.s_down[e])
    return F.linear(F.silu(F.linear(x64, wg)) * F.linear(x64, wu), wd)


def _x64(x_bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(x_bits.view(np.int16).copy()).view(torch.bfloat16).to(torch.float64)


# ------------------------------------------------------------------ formats

def test_e4m3fn_every_code_matches_torch_cast():
    """All 256 codes against torch's float8_e4m3fn -> float32 conversion
    (catches a wrong bias, a subnormal rule or a sign slip)."""
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = np.array([oracle.e4m3fn_value(c) for c in range(256)])
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])
    assert np.array_equal(np.signbit(got[~nan]), np.signbit(ref[~nan]))


def test_e4m3fn_closed_forms():
    """Values fixed by the E4M3FN definition (bias 7, 3 mantissa bits, no inf)."""
    assert oracle.e4m3fn_value(0x00) == 0.0
    assert oracle.e4m3fn_value(0x01) == 2.0 ** -9          # smallest subnormal
    assert oracle.e4m3fn_value(0x07) == 7 * 2.0 ** -9      # largest subnormal
    assert oracle.e4m3fn_value(0x08) == 2.0 ** -6          # smallest normal
    assert oracle.e4m3fn_value(0x38) == 1.0
    assert oracle.e4m3fn_value(0x3C) == 1.5
    assert oracle.e4m3fn_value(0x7E) == 448.0              # largest finite
    assert oracle.e4m3fn_value(0xFE) == -448.0
    assert np.isnan(oracle.e4m3fn_value(0x7F)) and np.isnan(oracle.e4m3fn_value(0xFF))
    assert np.signbit(oracle.e4m3fn_value(0x80))


def test_bf16_matches_torch_cast():
    rng = np.random.default_rng(1)
    bits = rng.integers(0, 1 << 16, size=2000, dtype=np.uint32).astype(np.uint16)
    bits[:4] = [0x3F80, 0xC000, 0x0001, 0x7F7F]
    ref = torch.from_numpy(bits.view(np.int16).copy()).view(torch.bfloat16).to(torch.float64).numpy()
    got = np.array([oracle.bf16_value(int(b)) for b in bits])
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])
    assert got[0] == 1.0 and got[1] == -2.0 and got[2] == 2.0 ** -133


# ------------------------------------------------------------------ route

def _sorted_topk(l: np.ndarray, K: int):
    return [e for _, e in sorted((-float(v), e) for e, v in enumerate(l))][:K]


@pytest.mark.parametrize("T,E,K,levels", [(40, 8, 2, None), (30, 256, 8, None),
                                          (50, 6, 3, 2), (50, 33, 7, 3), (5, 16, 16, None)])
def test_route_ids_match_python_sorted(T, E, K, levels):
    """Top-K, descending, ties to the lower id: against Python's sorted on
    (-logit, id) (catches ascending order, a wrong tie rule, repeated picks)."""
    lg = (wl.tie_logits(T, E, seed=T, levels=levels) if levels
          else np.random.default_rng(T).standard_normal((T, E)).astype(np.float32))
    ids, w = oracle.route(lg, K)
    for t in range(T):
        assert list(ids[t]) == _sorted_topk(lg[t], K)


def test_route_ranking_equals_probability_ranking():
    """Ranking by logit equals ranking the fp64 softmax (scipy) probabilities."""
    lg = np.random.default_rng(7).standard_normal((200, 64)).astype(np.float32) * 3
    ids, _ = oracle.route(lg, 10)
    p = scipy.special.softmax(lg.astype(np.float64), axis=1)
    ref = np.argsort(-p, axis=1, kind="stable")[:, :10]
    assert np.array_equal(ids, ref)


def test_route_weights_full_k_is_softmax():
    """With K = E the renormalisation is a no-op: w equals scipy's softmax."""
    lg = np.random.default_rng(3).standard_normal((20, 12)).astype(np.float32) * 2
    ids, w = oracle.route(lg, 12)
    p = scipy.special.softmax(lg.astype(np.float64), axis=1)
    np.testing.assert_allclose(w, np.take_along_axis(p, ids, axis=1), rtol=1e-13, atol=0)


def test_route_weight_closed_forms():
    """Renormalised weights sum to 1, and w_i / w_j = exp(l_i - l_j) (softmax
    ratio); adding a constant to a token's logits changes nothing."""
    lg = np.random.default_rng(4).standard_normal((64, 40)).astype(np.float32)
    ids, w = oracle.route(lg, 6)
    np.testing.assert_allclose(w.sum(1), 1.0, rtol=0, atol=1e-14)
    l_sel = np.take_along_axis(lg.astype(np.float64), ids, axis=1)
    np.testing.assert_allclose(w[:, 1:] / w[:, :1], np.exp(l_sel[:, 1:] - l_sel[:, :1]), rtol=1e-12)
    ids2, w2 = oracle.route(lg + np.float32(8.0), 6)
    assert np.array_equal(ids, ids2)
    np.testing.assert_allclose(w2, w, rtol=1e-5)   # the shifted fp32 logits round


def test_route_zero_mask_forces_zero_without_renormalising():
    lg = np.random.default_rng(5).standard_normal((30, 16)).astype(np.float32)
    mask = np.zeros((30, 4), np.uint8)
    mask[::3, 1] = 1
    ids0, w0 = oracle.route(lg, 4)
    ids1, w1 = oracle.route(lg, 4, mask)
    assert np.array_equal(ids0, ids1)
    assert np.all(w1[mask == 1] == 0.0)
    assert np.array_equal(w1[mask == 0], w0[mask == 0])


# ------------------------------------------------------------------ routing variants

SIG = oracle.SCORE_SIGMOID


def _sigmoid64(lg: np.ndarray) -> np.ndarray:
    return scipy.special.expit(lg.astype(np.float64))


def test_route_ex_default_is_route():
    """Softmax, no bias, one group, renormalised, scale 1 is the plain router."""
    lg = wl.tie_logits(60, 24, seed=6, levels=3)
    ids0, w0 = oracle.route(lg, 5)
    ids1, w1 = oracle.route_ex(lg, 5)
    assert np.array_equal(ids0, ids1)
    np.testing.assert_allclose(w1, w0, rtol=1e-15, atol=0)


def test_route_ex_sigmoid_closed_forms():
    """Sigmoid scores (scipy's expit): with K = E and renormalisation the weights
    are sigmoid / sum(sigmoid); without it, scaling * sigmoid; the order is the
    logit order, ties to the lower id (catches a softmax left in, a missing or
    doubled scaling, a dropped renormalisation)."""
    lg = np.random.default_rng(8).standard_normal((30, 10)).astype(np.float32) * 2
    sg = _sigmoid64(lg)
    ids, w = oracle.route_ex(lg, 10, score=SIG)
    for t in range(30):
        assert list(ids[t]) == _sorted_topk(lg[t], 10)
    np.testing.assert_allclose(w, np.take_along_axis(sg / sg.sum(1, keepdims=True), ids, 1), rtol=1e-13)
    ids, w = oracle.route_ex(lg, 4, score=SIG, renormalize=False, scaling=2.5)
    np.testing.assert_allclose(w, 2.5 * np.take_along_axis(sg, ids, 1), rtol=1e-13)
    ids, w = oracle.route_ex(lg, 4, score=SIG, scaling=2.5)
    np.testing.assert_allclose(w.sum(1), 2.5, rtol=1e-14)


def test_route_ex_bias_selects_but_does_not_weigh():
    """A large selection bias on a set S forces S (ordered by score + bias),
    while the weights stay the unbiased sigmoid scores of S, renormalised."""
    rng = np.random.default_rng(9)
    T, E, K = 40, 32, 4
    lg = rng.standard_normal((T, E)).astype(np.float32)
    S = np.array([3, 17, 22, 30])
    bias = np.zeros(E, np.float32)
    bias[S] = np.float32(10.0) + rng.random(K).astype(np.float32)
    ids, w = oracle.route_ex(lg, K, score=SIG, bias=bias)
    sg = _sigmoid64(lg)
    for t in range(T):
        order = sorted(S, key=lambda e: (-(sg[t, e] + float(bias[e])), e))
        assert list(ids[t]) == order
        np.testing.assert_allclose(w[t], sg[t, order] / sg[t, S].sum(), rtol=1e-13)


def _brute_group_route(c: np.ndarray, n_group: int, topk_group: int, K: int):
    """Exhaustive search: the group subset of largest total group score (a
    group's score: sum of its two largest c), then the K-subset of its experts
    of largest total c, listed by c descending."""
    import itertools
    E = c.size
    G = E // n_group
    gs = [sum(sorted(c[g * G:(g + 1) * G])[-2:]) for g in range(n_group)]
    groups = max(itertools.combinations(range(n_group), topk_group), key=lambda gg: sum(gs[g] for g in gg))
    pool = [e for g in groups for e in range(g * G, (g + 1) * G)]
    best = max(itertools.combinations(pool, K), key=lambda ee: sum(c[e] for e in ee))
    return sorted(best, key=lambda e: -c[e])


@pytest.mark.parametrize("E,n_group,topk_group,K", [(12, 4, 2, 3), (16, 8, 3, 4), (18, 3, 1, 2), (8, 8, 5, 5)])
def test_route_ex_groups_match_exhaustive_search(E, n_group, topk_group, K):
    """Group-limited selection against an exhaustive search over group and
    expert subsets on tiny, tie-free inputs (catches a top-1 group score, the
    groups scored on the unbiased scores, experts taken outside the kept
    groups)."""
    rng = np.random.default_rng(E * 100 + K)
    T = 25
    lg = rng.standard_normal((T, E)).astype(np.float32)
    bias = (rng.random(E) * 0.3 - 0.1).astype(np.float32)
    ids, w = oracle.route_ex(lg, K, score=SIG, bias=bias, n_group=n_group, topk_group=topk_group)
    c = _sigmoid64(lg) + bias.astype(np.float64)
    for t in range(T):
        assert list(ids[t]) == _brute_group_route(c[t], n_group, topk_group, K)


def test_route_ex_all_groups_kept_is_no_group_limit():
    lg = np.random.default_rng(11).standard_normal((50, 64)).astype(np.float32)
    bias = (np.random.default_rng(12).random(64) * 0.2).astype(np.float32)
    a = oracle.route_ex(lg, 8, score=SIG, bias=bias, n_group=8, topk_group=8, scaling=1.5)
    b = oracle.route_ex(lg, 8, score=SIG, bias=bias, scaling=1.5)
    assert np.array_equal(a[0], b[0])
    np.testing.assert_array_equal(a[1], b[1])


def test_route_ex_matches_transformers_deepseek_v3_router():
    """The published DeepSeek-V3 router as the transformers library implements
    it (sigmoid, selection-only correction bias, group-limited top-k,
    renormalised, scaled), in float64 on tie-free inputs with a non-negative
    bias (the library fills masked experts with 0, which only matters when an
    eligible score is negative).  The library returns its picks unordered, so
    sets and per-expert weights are compared."""
    mod = pytest.importorskip("transformers.models.deepseek_v3.modeling_deepseek_v3")
    from transformers import DeepseekV3Config
    E, n_group, topk_group, K, scale = 64, 8, 4, 6, 2.5
    cfg = DeepseekV3Config(hidden_size=32, intermediate_size=64, moe_intermediate_size=16,
                           n_routed_experts=E, n_shared_experts=1, num_experts_per_tok=K,
                           n_group=n_group, topk_group=topk_group, norm_topk_prob=True,
                           routed_scaling_factor=scale, num_hidden_layers=1, num_attention_heads=4,
                           num_key_value_heads=4)
    moe = mod.DeepseekV3MoE(cfg).double()
    rng = np.random.default_rng(13)
    lg = rng.standard_normal((100, E)).astype(np.float32)
    bias = (rng.random(E) * 0.05).astype(np.float32)
    with torch.no_grad():
        moe.gate.e_score_correction_bias.copy_(torch.from_numpy(bias.astype(np.float64)))
        li, lw = moe.route_tokens_to_experts(torch.from_numpy(lg.astype(np.float64)))
    ids, w = oracle.route_ex(lg, K, score=SIG, bias=bias, n_group=n_group, topk_group=topk_group,
                             scaling=scale)
    li, lw = li.numpy(), lw.numpy()
    for t in range(100):
        assert set(ids[t]) == set(li[t])
        ref = dict(zip(li[t], lw[t]))
        np.testing.assert_allclose(w[t], [ref[e] for e in ids[t]], rtol=1e-12)


def test_moe_tokens_routed_with_the_plain_router_is_moe_tokens(tiny):
    """The FFN with a given routing, fed the plain router's choice, is the
    routed brute-force oracle bit for bit."""
    w = tiny
    tk = np.arange(w.x.shape[0], dtype=np.int32)[::3]
    ids, wt = oracle.route(w.logits, w.shape.K, w.zero_mask)
    a = oracle.moe_tokens(w.x, w.logits, w.shape.K, w.routed, w.shared, w.zero_mask, tokens=tk)
    b = oracle.moe_tokens_routed(w.x, ids[tk], wt[tk], w.routed, w.shared, tokens=tk)
    np.testing.assert_array_equal(a, b)


def test_route_ex_weights_and_scores_helpers():
    """route_weights on the oracle's own choice reproduces its weights; the
    selection scores are sigmoid + bias (scipy)."""
    rng = np.random.default_rng(14)
    lg = rng.standard_normal((20, 48)).astype(np.float32)
    bias = (rng.random(48) * 0.1).astype(np.float32)
    ids, w = oracle.route_ex(lg, 5, score=SIG, bias=bias, n_group=4, topk_group=2, scaling=3.0)
    np.testing.assert_allclose(oracle.route_weights(lg, ids, score=SIG, scaling=3.0), w, rtol=1e-15)
    np.testing.assert_allclose(oracle.route_select_scores(lg, SIG, bias), _sigmoid64(lg) + bias, rtol=1e-15)
    p = scipy.special.softmax(lg.astype(np.float64), axis=1)
    np.testing.assert_allclose(oracle.route_select_scores(lg, oracle.SCORE_SOFTMAX), p, rtol=1e-13)


# ------------------------------------------------------------------ sort

@pytest.mark.parametrize("T,K,E,distinct", [(0, 4, 8, True), (1, 1, 1, True), (37, 3, 5, True),
                                            (200, 8, 64, True), (100, 5, 7, False),
                                            (513, 10, 512, True)])
def test_sort_matches_numpy_stable_argsort(T, K, E, distinct):
    ids = wl.random_ids(T, K, E, seed=T + K, distinct=distinct) if T else np.zeros((0, K), np.int32)
    off, sr, inv, bad = oracle.sort(ids, E)
    flat = ids.ravel()
    assert bad == 0
    assert np.array_equal(sr, np.argsort(flat, kind="stable"))
    assert np.array_equal(off, np.concatenate([[0], np.cumsum(np.bincount(flat, minlength=E))]))
    assert np.array_equal(inv[sr], np.arange(T * K))


def test_sort_all_routes_on_one_expert():
    ids = np.full((50, 1), 3, np.int32)
    off, sr, inv, bad = oracle.sort(ids, 8)
    assert list(off) == [0, 0, 0, 0, 50, 50, 50, 50, 50]
    assert np.array_equal(sr, np.arange(50)) and np.array_equal(inv, np.arange(50))


def test_sort_skips_out_of_range_ids():
    ids = np.array([[0, 9], [-1, 2], [2, 0]], np.int32)
    off, sr, inv, bad = oracle.sort(ids, 4)
    assert bad == 2
    assert list(off) == [0, 2, 2, 4, 4]
    assert list(sr) == [0, 5, 3, 4, -1, -1]
    assert list(inv) == [0, -1, -1, 2, 3, 1]


# ------------------------------------------------------------------ FFN

def test_swiglu_matches_torch_silu():
    """silu(gate) * up against torch.nn.functional.silu (catches a swapped
    gate/up, sigmoid(g)*u, or a sign error in the exponent)."""
    rng = np.random.default_rng(6)
    g = rng.standard_normal(1000) * 6
    u = rng.standard_normal(1000) * 3
    ref = (F.silu(torch.from_numpy(g)) * torch.from_numpy(u)).numpy()
    np.testing.assert_allclose(oracle.swiglu(g, u), ref, rtol=1e-14, atol=1e-300)
    h = oracle.swiglu(np.array([0.0, 1.0, 2.0, -50.0]), np.array([5.0, 2.0, 1.0, 1.0]))
    assert h[0] == 0.0
    assert abs(h[1] - 2.0 / (1.0 + np.exp(-1.0))) < 1e-15       # silu(1) * 2
    assert abs(h[2] - 2.0 / (1.0 + np.exp(-2.0))) < 1e-15       # silu(2) * 1
    assert abs(h[3]) < 1e-20


@pytest.mark.parametrize("H,I", [(256, 384), (384, 128)])
def test_expert_ffn_matches_torch_mlp(H, I):
    """One expert against the eager torch MLP built from torch-decoded weights.
    H != I and per-block random scales catch transposed operands, a transposed
    scale grid, or a scale applied to the wrong block."""
    ex = wl.draw_experts(seed=11, tag=99, n=2, I=I, H=H, std=0.05, threads=1)
    for e in range(2):
        ex.s_gate[e] *= np.exp2(np.random.default_rng(e).integers(-3, 4, ex.s_gate[e].shape))
        ex.s_down[e] *= np.exp2(np.random.default_rng(9 + e).integers(-3, 4, ex.s_down[e].shape))
    x = wl.random_rows_bf16(5, H, seed=2)
    for e in range(2):
        got = oracle.expert_rows(x, ex, e, np.arange(5))
        ref = _torch_mlp(_x64(x), ex, e).numpy()
        np.testing.assert_allclose(got, ref, rtol=1e-10, atol=1e-12 * np.abs(ref).max())


def test_expert_ffn_subnormal_and_all_codes():
    """Blocks of E4M3FN subnormals only, and blocks using every finite code."""
    for ex in (wl.subnormal_experts(1, 128, 256), wl.all_code_experts(1, 128, 256)):
        x = wl.random_rows_bf16(3, 256, seed=5)
        got = oracle.expert_rows(x, ex, 0, np.arange(3))
        ref = _torch_mlp(_x64(x), ex, 0).numpy()
        np.testing.assert_allclose(got, ref, rtol=1e-10, atol=1e-12 * np.abs(ref).max())


# ------------------------------------------------------------------ whole path

@pytest.fixture(scope="module")
def tiny():
    return wl.make_workload("tiny", threads=1)


def test_structured_equals_brute_force(tiny):
    """Route -> sort -> grouped FFN -> combine equals the per-token definition."""
    o = oracle.workload(tiny)
    b = oracle.moe_tokens(tiny.x, tiny.logits, tiny.shape.K, tiny.routed)
    np.testing.assert_allclose(o["out"], b, rtol=1e-12, atol=1e-14)
    assert o["bad"] == 0


def test_brute_force_tiny_against_library_chain():
    """The whole chain on tiny inputs from library pieces: Python sorted for the
    top-K, scipy softmax, torch Linear/SiLU for each expert."""
    T, H, I, E, K = 4, 128, 128, 5, 2
    ex = wl.draw_experts(seed=4, tag=98, n=E, I=I, H=H, std=0.05, threads=1)
    x = wl.random_rows_bf16(T, H, seed=8)
    lg = np.random.default_rng(12).standard_normal((T, E)).astype(np.float32)
    got = oracle.moe_tokens(x, lg, K, ex)
    x64 = _x64(x)
    for t in range(T):
        p = scipy.special.softmax(lg[t].astype(np.float64))
        sel = _sorted_topk(lg[t], K)
        ref = sum(p[e] / p[sel].sum() * _torch_mlp(x64[t:t + 1], ex, e)[0].numpy() for e in sel)
        np.testing.assert_allclose(got[t], ref, rtol=1e-10, atol=1e-13)


def test_full_topk_equals_softmax_mixture():
    """K = E: the routed sum is the full softmax mixture sum_e p_e FFN_e(x)."""
    T, H, I, E = 3, 128, 128, 4
    ex = wl.draw_experts(seed=5, tag=97, n=E, I=I, H=H, std=0.05, threads=1)
    x = wl.random_rows_bf16(T, H, seed=9)
    lg = np.random.default_rng(13).standard_normal((T, E)).astype(np.float32)
    got = oracle.moe_tokens(x, lg, E, ex)
    p = scipy.special.softmax(lg.astype(np.float64), axis=1)
    ref = sum(p[:, e:e + 1] * oracle.expert_rows(x, ex, e, np.arange(T)) for e in range(E))
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-14)


def test_zero_weight_route_contributes_nothing(tiny):
    """A masked route adds exactly 0: replacing its expert's weights by other
    finite values leaves the output bit-identical."""
    T, K = tiny.shape.T, tiny.shape.K
    ids, _ = oracle.route(tiny.logits, K)
    mask = np.zeros((T, K), np.uint8)
    mask[:, 0] = 1
    hot = ids[:, 0]
    # Every slot-0 expert is masked everywhere; only experts never used unmasked change.
    used_unmasked = set(ids[:, 1:].ravel().tolist())
    victims = [e for e in set(hot.tolist()) if e not in used_unmasked]
    assert victims
    a = oracle.moe(tiny.x, tiny.logits, K, tiny.routed, zero_mask=mask)["out"]
    ex2 = wl.FP8Experts(*(np.copy(v) for v in (tiny.routed.w_gate, tiny.routed.s_gate,
                                                tiny.routed.w_up, tiny.routed.s_up,
                                                tiny.routed.w_down, tiny.routed.s_down)))
    for e in victims:
        ex2.w_down[e] = 0x7E                  # 448: large but finite
        ex2.s_down[e] = 3.0
    b = oracle.moe(tiny.x, tiny.logits, K, ex2, zero_mask=mask)["out"]
    assert np.array_equal(a, b)


def test_token_permutation_permutes_rows(tiny):
    perm = np.random.default_rng(1).permutation(tiny.shape.T)
    a = oracle.moe(tiny.x, tiny.logits, tiny.shape.K, tiny.routed)["out"]
    b = oracle.moe(tiny.x[perm], tiny.logits[perm], tiny.shape.K, tiny.routed)["out"]
    assert np.array_equal(a[perm], b)


def test_shared_expert_is_added_with_weight_one():
    T, H, I, E, K = 6, 128, 128, 4, 2
    ex = wl.draw_experts(seed=6, tag=96, n=E, I=I, H=H, std=0.05, threads=1)
    sh = wl.draw_experts(seed=6, tag=95, n=1, I=256, H=H, std=0.05, threads=1)
    x = wl.random_rows_bf16(T, H, seed=10)
    lg = np.random.default_rng(14).standard_normal((T, E)).astype(np.float32)
    with_s = oracle.moe(x, lg, K, ex, sh)
    without = oracle.moe(x, lg, K, ex)
    ref = _torch_mlp(_x64(x), sh, 0).numpy()
    np.testing.assert_allclose(with_s["out"] - without["out"], ref, rtol=1e-9, atol=1e-12)
    np.testing.assert_allclose(with_s["y_shared"], ref, rtol=1e-10, atol=1e-13)


def test_combine_closed_form():
    """y for route r, column n = (r+1)(n+1): out[t, n] = (n+1) * sum_j (tK+j+1)
    exactly (catches a dropped or doubled slot and a wrong inverse lookup)."""
    T, K, E, H = 9, 3, 5, 16
    ids = wl.random_ids(T, K, E, seed=3)
    off, sr, inv, _ = oracle.sort(ids, E)
    y = np.empty((T * K, H))
    for p in range(T * K):
        y[p] = (sr[p] + 1) * (np.arange(H) + 1.0)
    out = oracle.combine(y, inv, None, T, K)
    for t in range(T):
        s = sum(t * K + j + 1 for j in range(K))
        assert np.array_equal(out[t], s * (np.arange(H) + 1.0))
    sh = np.full((T, H), 0.5)
    assert np.array_equal(oracle.combine(y, inv, sh, T, K), out + 0.5)


def test_combine_bf16_matches_float_combine():
    T, K, E, H = 7, 4, 6, 32
    ids = wl.random_ids(T, K, E, seed=4)
    _, _, inv, _ = oracle.sort(ids, E)
    ys = wl.random_rows_bf16(T * K, H, seed=6)
    sh = wl.random_rows_bf16(T, H, seed=7)
    a = oracle.combine_bf16(ys, inv, sh, T, K)
    b = oracle.combine(oracle.bf16_array(ys), inv, oracle.bf16_array(sh), T, K)
    assert np.array_equal(a, b)


def test_oracle_matches_stored_golden(tiny):
    """The stored oracle output of the tiny workload (tests/golden/make_golden.py)."""
    import os
    path = os.path.join(os.path.dirname(__file__), "golden", "tiny_oracle.txt")
    rows = {}
    for line in open(path):
        if line.startswith("#"):
            continue
        key, *vals = line.split()
        rows[key] = vals
    o = oracle.workload(tiny)
    assert list(map(int, rows["ids"])) == list(o["ids"].ravel())
    assert list(map(int, rows["offsets"])) == list(o["offsets"])
    assert list(map(int, rows["sorted_route"])) == list(o["sorted_route"])
    np.testing.assert_allclose(np.array(rows["w"], float), o["w"].ravel(), rtol=1e-15)
    for t in range(4):
        np.testing.assert_allclose(np.array(rows["out%d" % t], float), o["out"][t, :16],
                                   rtol=1e-13, atol=1e-15)


def test_route_ex_matches_stored_golden(tiny):
    """The stored routing-variant output of the tiny workload (tests/golden/make_golden.py)."""
    import os
    path = os.path.join(os.path.dirname(__file__), "golden", "tiny_route_ex.txt")
    rows = {}
    for line in open(path):
        if not line.startswith("#"):
            key, *vals = line.split()
            rows[key] = vals
    bias = wl.selection_bias(tiny.shape.E, seed=1, std=0.05)
    ids, w = oracle.route_ex(tiny.logits, tiny.shape.K, score=SIG, bias=bias, n_group=4, topk_group=2,
                             scaling=2.5)
    assert list(map(int, rows["ids"])) == list(ids.ravel())
    np.testing.assert_allclose(np.array(rows["w"], float), w.ravel(), rtol=1e-15)


# ------------------------------------------------------------------ router gate GEMM

def test_router_logits_match_library_matmul():
    """The fp64 gate GEMM against numpy's matmul of torch's bf16 -> float64
    widening: catches a transposed operand (T != E != H), a wrong stride or a
    dropped term."""
    x = wl.random_rows_bf16(37, 192, seed=3)
    w = wl.router_weight(21, 192, seed=4)
    got = oracle.router_logits(x, w)
    ref = _x64(x).numpy() @ _x64(w).numpy().T
    assert got.shape == (37, 21)
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-12)


def test_router_logits_closed_forms():
    """One-hot tokens pick a column of w_router; small-integer inputs give
    exact integer logits (every product and sum is exact in fp64)."""
    H, E = 64, 5
    w = wl.router_weight(E, H, seed=5)
    x = np.zeros((3, H), np.uint16)
    for t, h in enumerate((0, 17, 63)):
        x[t, h] = 0x3F80  # 1.0
    got = oracle.router_logits(x, w)
    w64 = oracle.bf16_array(w)
    for t, h in enumerate((0, 17, 63)):
        assert np.array_equal(got[t], w64[:, h])
    rng = np.random.default_rng(6)
    xi = rng.integers(-8, 9, (4, H)).astype(np.float32)
    wi = rng.integers(-8, 9, (E, H)).astype(np.float32)
    got = oracle.router_logits(wl.to_bf16_bits(xi), wl.to_bf16_bits(wi))
    exact = [[sum(int(a) * int(b) for a, b in zip(xi[t], wi[e])) for e in range(E)] for t in range(4)]
    assert np.array_equal(got, np.array(exact, np.float64))


def test_router_routes_the_rounded_logits():
    """router() is the gate GEMM rounded to the fp32 logit type and then the
    routing step: the plain router's ids are the K largest fp32 logits (ties to
    the lower id, Python's sorted), and its weights the renormalised softmax."""
    x = wl.random_rows_bf16(9, 128, seed=7)
    w = wl.router_weight(16, 128, seed=8)
    l64, l32, ids, wt = oracle.router(x, w, 4)
    assert l32.dtype == np.float32 and np.array_equal(l32, l64.astype(np.float32))
    for t in range(9):
        order = sorted(range(16), key=lambda e: (-float(l32[t, e]), e))[:4]
        assert list(ids[t]) == order
        p = scipy.special.softmax(l32[t].astype(np.float64))
        np.testing.assert_allclose(wt[t], p[order] / p[order].sum(), rtol=1e-12)


def test_router_logits_permutations_and_linearity():
    """Permuting tokens permutes logit rows, permuting experts permutes
    columns (bit-identical), and the GEMM is linear in x: logits of a
    power-of-two multiple of x are that multiple (exact in fp64)."""
    x = wl.random_rows_bf16(11, 128, seed=9)
    w = wl.router_weight(7, 128, seed=10)
    base = oracle.router_logits(x, w)
    pt = np.random.default_rng(1).permutation(11)
    pe = np.random.default_rng(2).permutation(7)
    assert np.array_equal(oracle.router_logits(x[pt], w), base[pt])
    assert np.array_equal(oracle.router_logits(x, w[pe]), base[:, pe])
    x4 = wl.to_bf16_bits(oracle.bf16_array(x).astype(np.float32) * np.float32(4.0))
    assert np.array_equal(oracle.router_logits(x4, w), 4.0 * base)


# ------------------------------------------------------------------ W8A8 form (FP8 activations)

def _torch_e4m3(v32: np.ndarray) -> np.ndarray:
    """Library rounding: torch's float32 -> float8_e4m3fn cast (round to nearest
    even; it gives NaN at and above 464 instead of saturating)."""
    t = torch.from_numpy(np.ascontiguousarray(v32, dtype=np.float32))
    return t.to(torch.float8_e4m3fn).to(torch.float64).numpy()


def test_e4m3fn_round_matches_torch_cast():
    """Catches a wrong tie rule, a wrong binade or subnormal step, a lost sign."""
    rng = np.random.default_rng(11)
    mags = np.exp2(rng.uniform(-13.0, np.log2(463.0), 20000))
    vals = (mags * rng.choice([-1.0, 1.0], mags.size)).astype(np.float32)
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8).view(torch.float8_e4m3fn).to(torch.float64)
    finite = np.unique(np.abs(codes.numpy()[np.isfinite(codes.numpy())]))
    mids = ((finite[1:] + finite[:-1]) / 2).astype(np.float32)  # exact in fp32
    for v in (vals, finite.astype(np.float32), mids, -mids):
        np.testing.assert_array_equal(oracle.e4m3fn_round(v.astype(np.float64)), _torch_e4m3(v))


def test_e4m3fn_round_saturates():
    """The saturating conversion: everything at or above 448 in magnitude gives 448."""
    r = oracle.e4m3fn_round(np.array([448.0, 463.99, 464.0, 1e9, -500.0, -448.0]))
    np.testing.assert_array_equal(r, [448.0, 448.0, 448.0, 448.0, -448.0, -448.0])
    assert np.isnan(oracle.e4m3fn_round(np.array([np.nan]))[0])


def _k_by_search(amax: float) -> int:
    """Brute force: the largest k in [-126, 126] with amax * 2^k <= 448."""
    if amax == 0:
        return 0
    ks = [k for k in range(-126, 127) if amax * 2.0 ** k <= 448.0]
    return max(ks) if ks else -126


def test_act_scale_exp_is_the_largest_fitting_power_of_two():
    """Catches an off-by-one exponent (a block scaled into saturation, or one
    binade too low) and a wrong 1.75 boundary."""
    rng = np.random.default_rng(12)
    amaxes = list(np.exp2(rng.uniform(-40, 40, 2000))) + [1.75, np.nextafter(1.75, 2), 1.0, 2.0, 448.0,
                                                          224.0, np.nextafter(224.0, 0), 3.5, 0.0]
    for a in amaxes:
        k = oracle.act_scale_exp(a)
        assert k == _k_by_search(a), a
        if a:
            assert 224.0 < a * 2.0 ** k <= 448.0


def test_act_quantize_matches_torch_blocks():
    """Blocks of 128 (x) and 64 (h): each block scaled by its own power of two,
    rounded with torch's cast, scaled back.  Catches a block boundary or a
    scale taken from the wrong block."""
    rng = np.random.default_rng(13)
    for block in (128, 64):
        v = rng.standard_normal(16 * block) * np.exp2(rng.integers(-20, 20, 16 * block // block).repeat(block))
        v32 = v.astype(np.float32).astype(np.float64)  # fp32-exact inputs (as bf16 and fp32 activations are)
        ref = np.empty_like(v32)
        for b0 in range(0, v32.size, block):
            blk = v32[b0:b0 + block]
            k = _k_by_search(np.abs(blk).max())
            ref[b0:b0 + block] = _torch_e4m3((blk * 2.0 ** k).astype(np.float32)) * 2.0 ** -k
        np.testing.assert_array_equal(oracle.act_quantize(v32, block), ref)


def _quant_torch(v64: np.ndarray, block: int) -> np.ndarray:
    out = np.empty_like(v64)
    for b0 in range(0, v64.size, block):
        blk = v64[b0:b0 + block]
        k = _k_by_search(np.abs(blk).max())
        out[b0:b0 + block] = _torch_e4m3((blk * 2.0 ** k).astype(np.float32)) * 2.0 ** -k
    return out


def test_ffn_w8a8_matches_torch_chain():
    """The W8A8 expert FFN against torch ops: x quantised per 128 columns
    (torch cast), F.linear with the block-scaled FP8 weights, F.silu, h
    quantised per 64 features, F.linear.  h passes through fp32 before torch's
    cast, which can move a value across a rounding midpoint in rare elements,
    so the comparison is relative-L2 at 1e-4 (the quantisation error itself is
    about 1e-2)."""
    E, I, H, T, K = 3, 128, 256, 6, 2
    ex = wl.draw_experts(21, 71, E, I, H, 0.05, threads=1)
    x = wl.random_rows_bf16(T, H, seed=22)
    ids = np.array([[0, 1], [2, 0], [1, 2], [0, 2], [1, 0], [2, 1]], np.int32)
    off, sr, inv, _ = oracle.sort(ids, E)
    w = np.ones((T, K))
    y = oracle.ffn_sorted_w8a8(x, K, ex, off, sr, w)
    x64 = _x64(x).numpy()
    for p, r in enumerate(sr):
        t, e = r // K, ids.ravel()[r]
        xq = torch.from_numpy(_quant_torch(x64[t], 128))
        wg, wu, wd = (_fp8_dense(ex.w_gate[e], ex.s_gate[e]), _fp8_dense(ex.w_up[e], ex.s_up[e]),
                      _fp8_dense(ex.w_down[e], ex.s_down[e]))
        h = (F.silu(F.linear(xq, wg)) * F.linear(xq, wu)).numpy()
        ref = F.linear(torch.from_numpy(_quant_torch(h, 64)), wd).numpy()
        assert np.linalg.norm(y[p] - ref) <= 1e-4 * np.linalg.norm(ref)


def test_ffn_w8a8_is_the_exact_ffn_when_quantisation_is_exact():
    """Inputs for which both quantisations are exact, so the W8A8 FFN must
    equal the fp64 FFN: x[t, :128] = c_t (c_t in 4..7), gate rows of E4M3FN
    ones over those columns, so g = 128 c_t and silu(g) = g in fp64
    (e^-g < 2^-53); x[t, 128] = d_t 2^-20 and up row i one power-of-two code
    p_i in column 128, so u = p_i d_t 2^-20 and h = g u has at most three
    significant bits.  The second x block is 2^-20 below the first, and the
    two 64-feature blocks of h are 2^15 apart (codes 2^7, 2^8 against 2^-9,
    2^-8): a scale taken from the wrong block, or h quantised in blocks of
    128, flushes or rounds the small values and breaks the equality."""
    E, I, H, T, K = 1, 128, 256, 4, 1
    ex = wl.draw_experts(23, 72, E, I, H, 0.05, threads=1)
    rng = np.random.default_rng(24)
    ex.w_gate[:] = 0
    ex.w_gate[0, :, :128] = 0x38  # 1.0
    ex.s_gate[:] = 1.0
    ex.w_up[:] = 0
    ex.w_up[0, :64, 128] = rng.choice([0x70, 0x78], 64)  # 2^7, 2^8
    ex.w_up[0, 64:, 128] = rng.choice([0x01, 0x02], 64)  # 2^-9, 2^-8 (subnormal codes)
    ex.s_up[:] = 1.0
    xs = np.zeros((T, H), np.float32)
    xs[:, :128] = rng.integers(4, 8, (T, 1))
    xs[:, 128:] = rng.choice([1.0, 2.0, 4.0], (T, 128)) * 2.0 ** -20
    x = (xs.view(np.uint32) >> 16).astype(np.uint16)
    assert np.array_equal(oracle.bf16_array(x), xs.astype(np.float64))
    ids = np.zeros((T, K), np.int32)
    off, sr, inv, _ = oracle.sort(ids, E)
    w = np.ones((T, K))
    exact = oracle.ffn_sorted(x, K, ex, off, sr, w)
    assert np.abs(exact).max() > 0
    np.testing.assert_allclose(oracle.ffn_sorted_w8a8(x, K, ex, off, sr, w), exact, rtol=1e-12, atol=0)


def test_ffn_shared_w8a8_is_the_routed_form_with_every_token_on_one_expert():
    """The shared expert's W8A8 rows equal the routed W8A8 rows of a one-expert
    layer where every token is routed to that expert with weight 1."""
    T, H, I = 5, 256, 128
    sh = wl.draw_experts(25, 73, 1, I, H, 0.05, threads=1)
    x = wl.random_rows_bf16(T, H, seed=26)
    ids = np.zeros((T, 1), np.int32)
    off, sr, inv, _ = oracle.sort(ids, 1)
    routed = oracle.ffn_sorted_w8a8(x, 1, sh, off, sr, np.ones((T, 1)))
    np.testing.assert_array_equal(oracle.ffn_shared_w8a8(x, sh), routed[inv])
