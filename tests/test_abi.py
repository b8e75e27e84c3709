"""The C-ABI library loads and exports every symbol include/*.h declares, and
its host-side contract checks reject bad arguments before touching the device
(CPU only: every call here returns from validation, none reaches a kernel)."""
import ctypes
import glob
import os
import re

import pytest

import mixture_experts_ffn_sort_b200 as moe

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    from mixture_experts_ffn_sort_b200 import build
    build.build()
    return moe.lib()


def declared_symbols():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        text = open(h).read()
        for m in re.finditer(r"MOE_API\s+[\w\s\*]+?\b(moe_\w+)\s*\(", text):
            names.add(m.group(1))
    return names


def test_every_declared_symbol_is_exported(L):
    names = declared_symbols()
    assert {"moe_route", "moe_sort", "moe_expert_ffn", "moe_combine"} <= names
    for n in names:
        assert hasattr(L, n), n
    assert names == set(moe.EXPORTED)


def test_no_other_symbols_exported(L):
    out = os.popen("nm -D --defined-only %s" % moe.LIB_PATH).read()
    exported = {l.split()[-1] for l in out.splitlines() if " T " in l}
    assert exported == set(moe.EXPORTED)


def test_abi_version(L):
    assert L.moe_abi_version() == 2


def test_workspace_queries(L):
    assert L.moe_sort_workspace_bytes(64, 8, 256) == 0            # single-block sort
    assert L.moe_sort_workspace_bytes(32768, 10, 512) == 160 * 512 * 4
    assert L.moe_ffn_workspace_bytes(64, 8, 2048, 256, 512, 0, 0) == 512 * 512 * 2
    assert L.moe_ffn_workspace_bytes(16, 2, 256, 8, 128, 0, 0) == 8192
    # The tensor-core forms add the f16 copy of x and its row scales.
    assert L.moe_ffn_workspace_bytes(8192, 10, 4096, 512, 256, 256, 0) == \
        81920 * 512 + 8192 * 512 + 8192 * 4096 * 2 + 8192 * 4
    assert L.moe_ffn_workspace_bytes(64, 8, 2048, 256, 512, 0, moe.MOE_MODE_PREFILL) == \
        512 * 512 * 2 + 64 * 2048 * 2 + 256
    # The fused FFN + combine: no y_sorted, an fp32 accumulator for a bf16 output.
    base = 81920 * 512 + 8192 * 512 + 8192 * 4096 * 2 + 8192 * 4
    assert L.moe_ffn_combine_workspace_bytes(8192, 10, 4096, 512, 256, 256, moe.MOE_OUT_F32) == base
    assert L.moe_ffn_combine_workspace_bytes(8192, 10, 4096, 512, 256, 256, moe.MOE_OUT_BF16) == \
        base + 8192 * 4096 * 4


def test_ffn_resolve_mode(L):
    D, PF, HY = moe.MOE_MODE_DECODE, moe.MOE_MODE_PREFILL, moe.MOE_MODE_HYBRID
    # Explicit modes resolve to themselves at any size.
    assert L.moe_ffn_resolve_mode(32768, 10, 512, D) == D
    assert L.moe_ffn_resolve_mode(1, 1, 8, PF) == PF
    assert L.moe_ffn_resolve_mode(1, 1, 8, HY) == HY
    # AUTO: decode while routes per expert stay at most 8 and routes at most
    # 8192; hybrid up to 32 routes per expert; prefill beyond.
    assert L.moe_ffn_resolve_mode(16, 2, 8, 0) == D          # 4 routes per expert
    assert L.moe_ffn_resolve_mode(64, 8, 256, 0) == D        # 2
    assert L.moe_ffn_resolve_mode(256, 8, 256, 0) == D       # 8: the limit
    assert L.moe_ffn_resolve_mode(257, 8, 256, 0) == HY
    assert L.moe_ffn_resolve_mode(512, 8, 256, 0) == HY      # 16
    assert L.moe_ffn_resolve_mode(1024, 8, 256, 0) == HY     # 32: the limit
    assert L.moe_ffn_resolve_mode(1025, 8, 256, 0) == PF
    assert L.moe_ffn_resolve_mode(1024, 8, 1024, 0) == D     # 8192 routes
    assert L.moe_ffn_resolve_mode(1025, 8, 1024, 0) == HY    # 8200 routes, 8.0 per expert
    assert L.moe_ffn_resolve_mode(8192, 10, 512, 0) == PF
    assert L.moe_ffn_resolve_mode(0, 8, 256, 0) == D
    assert moe.moe_ffn_resolve_mode(512, 8, 256) == HY
    for args in ((4, 2, 8, 4), (-1, 2, 8, 0), (4, 0, 8, 0), (4, 2, 0, 0)):
        assert L.moe_ffn_resolve_mode(*args) == moe.MOE_ERR_INVALID_ARG
        assert "moe_ffn_resolve_mode" in L.moe_last_error().decode()
    with pytest.raises(moe.MoEError):
        moe.moe_ffn_resolve_mode(4, 2, 8, 7)


P = ctypes.c_void_p


def _err(L):
    return L.moe_last_error().decode()


@pytest.mark.parametrize("T,E,K,code", [(4, 8, 0, moe.MOE_ERR_INVALID_ARG), (4, 8, 9, moe.MOE_ERR_INVALID_ARG),
                                        (4, 1025, 2, moe.MOE_ERR_UNSUPPORTED_SHAPE),
                                        (4, 64, 33, moe.MOE_ERR_INVALID_ARG), (-1, 8, 2, moe.MOE_ERR_INVALID_ARG)])
def test_route_rejects_bad_sizes(L, T, E, K, code):
    assert L.moe_route(P(16), T, E, K, None, P(16), P(16), None) == code
    assert _err(L)


def test_route_top_k_message_names_bounds(L):
    assert L.moe_route(P(16), 4, 8, 9, None, P(16), P(16), None) == moe.MOE_ERR_INVALID_ARG
    assert "top_k=9 must be in 1..=8" in _err(L)


def test_route_zero_tokens_is_a_no_op(L):
    assert L.moe_route(None, 0, 8, 2, None, None, None, None) == moe.MOE_OK
    assert _err(L) == ""


def test_route_null_and_misaligned(L):
    assert L.moe_route(None, 4, 8, 2, None, P(16), P(16), None) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_route(P(0x1008), 4, 8, 2, None, P(16), P(16), None) == moe.MOE_ERR_MISALIGNED


def _rcfg(score=0, bias=None, n_group=1, topk_group=1, renorm=1, scaling=1.0):
    return ctypes.byref(moe._RouteConfig(score, bias, n_group, topk_group, renorm, scaling))


@pytest.mark.parametrize("cfg,why", [
    (dict(score=2), "unknown score"), (dict(n_group=0), "n_group < 1"), (dict(n_group=33), "n_group > 32"),
    (dict(n_group=3), "n_group does not divide E"), (dict(n_group=4, topk_group=0), "topk_group < 1"),
    (dict(n_group=4, topk_group=5), "topk_group > n_group"),
    (dict(n_group=8, topk_group=1), "kept groups hold fewer than K experts"),
    (dict(renorm=2), "renormalize not 0/1"), (dict(scaling=0.0), "scaling 0"),
    (dict(scaling=float("inf")), "scaling inf"), (dict(scaling=float("nan")), "scaling nan")])
def test_route_ex_rejects_bad_config(L, cfg, why):
    # E = 16, K = 4: n_group 8 with one kept group leaves 2 experts < K.
    assert L.moe_route_ex(P(16), 4, 16, 4, _rcfg(**cfg), None, P(16), P(16), None) == moe.MOE_ERR_INVALID_ARG, why


def test_route_ex_checks(L):
    assert L.moe_route_ex(P(16), 4, 16, 4, None, None, P(16), P(16), None) == moe.MOE_ERR_INVALID_ARG
    assert b"cfg" in L.moe_last_error()
    assert L.moe_route_ex(P(16), 4, 16, 17, _rcfg(), None, P(16), P(16), None) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_route_ex(None, 0, 16, 4, _rcfg(n_group=4, topk_group=2), None, None, None, None) == moe.MOE_OK
    assert L.moe_route_ex(P(0x1008), 4, 16, 4, _rcfg(), None, P(16), P(16), None) == moe.MOE_ERR_MISALIGNED
    assert L.moe_route_ex(P(16), 4, 16, 4, _rcfg(bias=0x1002), None, P(16), P(16), None) == moe.MOE_ERR_MISALIGNED


def test_sort_checks(L):
    assert L.moe_sort(P(16), 4, 2, 8, None, P(16), P(16), None, 0, None, None) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_sort(P(16), 4, 2, 8, P(20), P(16), P(16), None, 0, None, None) == moe.MOE_ERR_MISALIGNED
    # Large sorts need the workspace the query reports.
    assert L.moe_sort(P(16), 4096, 8, 64, P(16), P(16), P(16), P(16), 10, None, None) == \
        moe.MOE_ERR_WORKSPACE_TOO_SMALL
    assert "need" in _err(L)


def _experts(inter=128, n=4, base=0x10000):
    return moe._Experts(base, base + 0x100, base + 0x200, base + 0x300, base + 0x400, base + 0x500, n, inter)


def test_expert_ffn_checks(L):
    ex = _experts()
    ws = L.moe_ffn_workspace_bytes(8, 2, 256, 4, 128, 0, 0)
    args = lambda **kw: dict(dict(x=P(16), T=8, H=256, K=2, routed=ctypes.byref(ex), shared=None,
                                  off=P(16), sr=P(16), w=P(16), y=P(16), ys=None, mode=0, ws=P(16),
                                  wsb=ws, status=None, stream=None), **kw)

    def call(**kw):
        a = args(**kw)
        return L.moe_expert_ffn(a["x"], a["T"], a["H"], a["K"], a["routed"], a["shared"], a["off"], a["sr"],
                                a["w"], a["y"], a["ys"], a["mode"], a["ws"], a["wsb"], a["status"], a["stream"])

    assert call(H=200) == moe.MOE_ERR_UNSUPPORTED_SHAPE
    assert call(H=16384) == moe.MOE_ERR_UNSUPPORTED_SHAPE
    assert call(mode=7) == moe.MOE_ERR_INVALID_ARG
    assert call(K=33) == moe.MOE_ERR_INVALID_ARG
    assert call(x=P(24)) == moe.MOE_ERR_MISALIGNED
    assert call(status=P(0x1002)) == moe.MOE_ERR_MISALIGNED
    assert call(wsb=ws - 1) == moe.MOE_ERR_WORKSPACE_TOO_SMALL
    assert call(y=None) == moe.MOE_ERR_INVALID_ARG
    bad_inter = _experts(inter=192)
    assert call(routed=ctypes.byref(bad_inter)) == moe.MOE_ERR_UNSUPPORTED_SHAPE
    two = _experts(n=2)
    assert call(shared=ctypes.byref(two), ys=P(16)) == moe.MOE_ERR_INVALID_ARG   # shared must hold 1 expert
    assert call(T=0) == moe.MOE_OK
    assert L.moe_expert_ffn(P(16), 8, 256, 2, None, None, P(16), P(16), P(16), P(16), None, 0, P(16), ws,
                            None, None) == moe.MOE_ERR_INVALID_ARG


def test_expert_ffn_w8a8_checks(L):
    ex = _experts()
    ws = L.moe_ffn_w8a8_workspace_bytes(8, 2, 128, 0)
    # codes (8*2*128 bytes) and 64-feature block scales (16 rows x 2 x 4 bytes), each 256-aligned
    assert ws == 2048 + 256
    assert L.moe_ffn_w8a8_workspace_bytes(8, 2, 128, 256) == ws + 2048 + 256
    assert L.moe_ffn_w8a8_workspace_bytes(-1, 2, 128, 0) == 0
    args = lambda **kw: dict(dict(x=P(16), T=8, H=256, K=2, routed=ctypes.byref(ex), shared=None,
                                  off=P(16), sr=P(16), w=P(16), y=P(16), ys=None, ws=P(16),
                                  wsb=ws, status=None, stream=None), **kw)

    def call(**kw):
        a = args(**kw)
        return L.moe_expert_ffn_w8a8(a["x"], a["T"], a["H"], a["K"], a["routed"], a["shared"], a["off"], a["sr"],
                                     a["w"], a["y"], a["ys"], a["ws"], a["wsb"], a["status"], a["stream"])

    assert call(H=200) == moe.MOE_ERR_UNSUPPORTED_SHAPE
    assert call(K=33) == moe.MOE_ERR_INVALID_ARG
    assert call(x=P(24)) == moe.MOE_ERR_MISALIGNED
    assert call(status=P(0x1002)) == moe.MOE_ERR_MISALIGNED
    assert call(wsb=ws - 1) == moe.MOE_ERR_WORKSPACE_TOO_SMALL
    assert "need" in _err(L)
    assert call(y=None) == moe.MOE_ERR_INVALID_ARG
    assert call(routed=None) == moe.MOE_ERR_INVALID_ARG
    two = _experts(n=2)
    assert call(shared=ctypes.byref(two), ys=P(16)) == moe.MOE_ERR_INVALID_ARG
    assert call(T=0) == moe.MOE_OK


def test_combine_checks(L):
    assert L.moe_combine(P(16), P(16), None, 4, 2, 12, P(16), 0, None, None) == moe.MOE_ERR_UNSUPPORTED_SHAPE
    assert L.moe_combine(P(16), P(16), None, 4, 2, 16, P(16), 3, None, None) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_combine(P(16), P(16), P(40), 4, 2, 16, P(16), 0, None, None) == moe.MOE_ERR_MISALIGNED
    assert L.moe_combine(P(16), P(16), None, 4, 2, 16, P(16), 0, P(18), None) == moe.MOE_ERR_MISALIGNED
    assert L.moe_combine(None, None, None, 0, 2, 16, None, 0, None, None) == moe.MOE_OK


def test_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    monkeypatch.setattr(moe, "LIB_PATH", str(tmp_path / "missing.so"))
    monkeypatch.setattr(moe, "_L", None)
    with pytest.raises(RuntimeError, match="missing"):
        moe.lib()


def test_router_checks(L):
    base = dict(x=P(16), T=4, H=128, w=P(16), E=16, K=4, cfg=None, zm=None, ids=P(16), wt=P(16), lg=None,
                status=None)

    def call(**kw):
        a = dict(base, **kw)
        return L.moe_router(a["x"], a["T"], a["H"], a["w"], a["E"], a["K"], a["cfg"], a["zm"], a["ids"], a["wt"],
                            a["lg"], a["status"], None)

    assert call(E=moe.MOE_ROUTER_MAX_E + 1) == moe.MOE_ERR_UNSUPPORTED_SHAPE
    assert "moe_router" in _err(L)
    for H in (0, 96, 16384 + 64):
        assert call(H=H) == moe.MOE_ERR_UNSUPPORTED_SHAPE, H
    assert call(K=17) == moe.MOE_ERR_INVALID_ARG
    assert call(cfg=_rcfg(n_group=3)) == moe.MOE_ERR_INVALID_ARG
    assert call(cfg=_rcfg(scaling=0.0)) == moe.MOE_ERR_INVALID_ARG
    assert call(x=None) == moe.MOE_ERR_INVALID_ARG
    assert call(ids=None) == moe.MOE_ERR_INVALID_ARG
    assert call(x=P(24)) == moe.MOE_ERR_MISALIGNED
    assert call(w=P(0x1008)) == moe.MOE_ERR_MISALIGNED
    assert call(lg=P(0x1004)) == moe.MOE_ERR_MISALIGNED
    assert call(status=P(0x1002)) == moe.MOE_ERR_MISALIGNED
    assert call(T=0, x=None, w=None, ids=None, wt=None) == moe.MOE_OK
    assert call(T=-1) == moe.MOE_ERR_INVALID_ARG


def test_selftest_bounded_wait_checks(L):
    assert L.moe_selftest_bounded_wait(None, P(16), None) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_selftest_bounded_wait(P(16), None, None) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_selftest_bounded_wait(P(0x1002), P(16), None) == moe.MOE_ERR_MISALIGNED
    assert L.moe_selftest_bounded_wait(P(16), P(0x1004), None) == moe.MOE_ERR_MISALIGNED


def test_router_plan_invariants_hold_over_a_wide_grid(L):
    """moe_router's launch plan satisfies the kernel's indexing invariants for
    every valid size: H in steps of 64 up to the limit, E from 1 to 512, batch
    sizes below, at and above one 128-token tile and up to a full wave, and
    both chunking limits.  Host only: the plan is computed and checked, nothing
    is launched."""
    fields = (ctypes.c_int32 * 9)()
    bad = []
    for kch in (1, 4):
        for T in (1, 7, 8, 100, 127, 128, 129, 1000, 8192, 32768):
            for H in range(64, 16384 + 1, 64):
                for E in range(1, 513):
                    if L.moe_router_plan_check(T, H, E, kch, fields) != moe.MOE_OK:
                        bad.append((T, H, E, kch, L.moe_last_error().decode()))
                        if len(bad) > 5:
                            break
    assert not bad, bad
    # The fields are what the kernel is launched with.
    assert L.moe_router_plan_check(8192, 4096, 512, 1, fields) == moe.MOE_OK
    tiles, cn, ne = fields[0], fields[1], fields[2]
    assert tiles == 64 and cn * ne >= 512 and ne % 16 == 0


def test_router_plan_check_rejects_bad_arguments(L):
    assert L.moe_router_plan_check(0, 128, 8, 1, None) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_router_plan_check(4, 100, 8, 1, None) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_router_plan_check(4, 128, 513, 1, None) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_router_plan_check(4, 128, 8, 3, None) == moe.MOE_ERR_INVALID_ARG
