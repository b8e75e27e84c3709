"""CPU oracle of the routed MoE FFN -- TEST INFRASTRUCTURE ONLY.

Only tests/, __graft_entry__.smoke() and bench.py's cpu_baseline / reference
leg may import this package.  The CUDA library and its Python binding never
import, link or call it, and it imports nothing from them: the two sides share
only the seeded input generator (mixture_experts_ffn_sort_b200.workloads),
which holds none of the method's arithmetic.

The arithmetic lives in moe_oracle.c (plain C, fp64); this module compiles it
with gcc and wraps it with ctypes.  Every function cites its source in the C
file.  Parity status: every function here is pinned by tests/test_oracle_pins.py
(closed forms, library routines, brute force, invariants).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.c")
_LIB = os.path.join(_HERE, "libmoe_oracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile moe_oracle.c into libmoe_oracle.so (gcc -O2 -fopenmp)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".%d.tmp" % os.getpid()
        cmd = ["gcc", "-O2", "-std=c99", "-fopenmp", "-fPIC", "-shared", "-o", tmp, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB)
    return _LIB


class _Experts(ctypes.Structure):
    _fields_ = [
        ("w_gate", ctypes.c_void_p), ("s_gate", ctypes.c_void_p),
        ("w_up", ctypes.c_void_p), ("s_up", ctypes.c_void_p),
        ("w_down", ctypes.c_void_p), ("s_down", ctypes.c_void_p),
        ("n_experts", ctypes.c_int), ("inter", ctypes.c_int),
    ]


def lib():
    global _lib
    with _lock:
        if _lib is None:
            build()
            L = ctypes.CDLL(_LIB)
            P, I = ctypes.c_void_p, ctypes.c_int
            L.oracle_e4m3fn_value.restype = ctypes.c_double
            L.oracle_e4m3fn_value.argtypes = [ctypes.c_uint8]
            L.oracle_bf16_value.restype = ctypes.c_double
            L.oracle_bf16_value.argtypes = [ctypes.c_uint16]
            L.oracle_set_threads.argtypes = [I]
            L.oracle_set_threads.restype = I
            L.oracle_get_threads.restype = I
            L.oracle_route.argtypes = [P, I, I, I, P, P, P]
            L.oracle_route_ex.argtypes = [P, I, I, I, I, P, I, I, I, ctypes.c_double, P, P, P]
            L.oracle_route_weights.argtypes = [P, I, I, I, I, I, ctypes.c_double, P, P]
            L.oracle_route_select_scores.argtypes = [P, I, I, I, P, P]
            L.oracle_router_logits.argtypes = [P, P, I, I, I, P]
            L.oracle_sort.argtypes = [P, I, I, I, P, P, P]
            L.oracle_sort.restype = I
            L.oracle_ffn_sorted.argtypes = [P, I, I, I, P, P, P, P, P]
            L.oracle_ffn_shared.argtypes = [P, I, I, P, P]
            L.oracle_combine.argtypes = [P, P, P, I, I, I, P]
            L.oracle_combine_bf16.argtypes = [P, P, P, I, I, I, P]
            L.oracle_moe.argtypes = [P, P, I, I, I, I, P, P, P, P, P, P, P, P, P, P, P]
            L.oracle_moe.restype = I
            L.oracle_moe_tokens.argtypes = [P, P, I, I, I, I, P, P, P, P, I, P]
            L.oracle_expert_rows.argtypes = [P, I, P, I, P, I, P]
            L.oracle_moe_tokens_routed.argtypes = [P, I, I, P, P, P, P, P, I, P]
            L.oracle_swiglu.argtypes = [P, P, I, P]
            L.oracle_e4m3fn_round.restype = ctypes.c_double
            L.oracle_e4m3fn_round.argtypes = [ctypes.c_double]
            L.oracle_e4m3fn_round_array.argtypes = [P, I, P]
            L.oracle_act_scale_exp.restype = I
            L.oracle_act_scale_exp.argtypes = [ctypes.c_double]
            L.oracle_act_quantize.argtypes = [P, I, I, P]
            L.oracle_ffn_sorted_w8a8.argtypes = [P, I, I, I, P, P, P, P, P]
            L.oracle_ffn_shared_w8a8.argtypes = [P, I, I, P, P]
            L.oracle_set_threads(int(os.environ.get("ORACLE_THREADS", os.cpu_count() or 1)))
            _lib = L
    return _lib


def _p(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def set_threads(n: int) -> int:
    return lib().oracle_set_threads(int(n))


def threads() -> int:
    return lib().oracle_get_threads()


def e4m3fn_value(code: int) -> float:
    return lib().oracle_e4m3fn_value(int(code))


def bf16_value(bits: int) -> float:
    return lib().oracle_bf16_value(int(bits))


def bf16_array(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns -> float64: a bf16 is the upper half of a binary32."""
    b = _c(bits, np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


class _ExpertsRef:
    """Keeps numpy arrays alive while a ctypes struct points into them."""

    def __init__(self, ex):
        self.arrays = [_c(ex.w_gate, np.uint8), _c(ex.s_gate, np.float32),
                       _c(ex.w_up, np.uint8), _c(ex.s_up, np.float32),
                       _c(ex.w_down, np.uint8), _c(ex.s_down, np.float32)]
        a = self.arrays
        self.struct = _Experts(_p(a[0]), _p(a[1]), _p(a[2]), _p(a[3]), _p(a[4]), _p(a[5]),
                               int(a[0].shape[0]), int(a[0].shape[1]))

    def ref(self):
        return ctypes.byref(self.struct)


def route(logits: np.ndarray, K: int, zero_mask: Optional[np.ndarray] = None):
    """-> (ids int32 [T,K], w float64 [T,K])."""
    lg = _c(logits, np.float32)
    T, E = lg.shape
    ids = np.empty((T, K), np.int32)
    w = np.empty((T, K), np.float64)
    zm = None if zero_mask is None else _c(zero_mask, np.uint8)
    lib().oracle_route(_p(lg), T, E, K, _p(zm), _p(ids), _p(w))
    return ids, w


SCORE_SOFTMAX, SCORE_SIGMOID = 0, 1


def route_ex(logits: np.ndarray, K: int, score: int = SCORE_SOFTMAX, bias: Optional[np.ndarray] = None,
             n_group: int = 1, topk_group: int = 1, renormalize: bool = True, scaling: float = 1.0,
             zero_mask: Optional[np.ndarray] = None):
    """Routing variants -> (ids int32 [T,K], w float64 [T,K])."""
    lg = _c(logits, np.float32)
    T, E = lg.shape
    if n_group > 1:
        assert E % n_group == 0 and n_group <= 64 and 1 <= topk_group <= n_group
        assert topk_group * (E // n_group) >= K
    ids = np.empty((T, K), np.int32)
    w = np.empty((T, K), np.float64)
    b = None if bias is None else _c(bias, np.float32)
    zm = None if zero_mask is None else _c(zero_mask, np.uint8)
    lib().oracle_route_ex(_p(lg), T, E, K, int(score), _p(b), int(n_group), int(topk_group),
                          int(bool(renormalize)), float(scaling), _p(zm), _p(ids), _p(w))
    return ids, w


def route_weights(logits: np.ndarray, ids: np.ndarray, score: int = SCORE_SOFTMAX,
                  renormalize: bool = True, scaling: float = 1.0) -> np.ndarray:
    """float64 [T,K]: the routing variants' weights for the given expert choice."""
    lg = _c(logits, np.float32)
    T, E = lg.shape
    idc = _c(ids, np.int32)
    K = idc.shape[1]
    w = np.empty((T, K), np.float64)
    lib().oracle_route_weights(_p(lg), T, E, K, int(score), int(bool(renormalize)), float(scaling),
                               _p(idc), _p(w))
    return w


def route_select_scores(logits: np.ndarray, score: int, bias: Optional[np.ndarray] = None) -> np.ndarray:
    """float64 [T,E]: the selection score s_e + bias_e of every expert."""
    lg = _c(logits, np.float32)
    T, E = lg.shape
    c = np.empty((T, E), np.float64)
    b = None if bias is None else _c(bias, np.float32)
    lib().oracle_route_select_scores(_p(lg), T, E, int(score), _p(b), _p(c))
    return c


def router_logits(x_bits: np.ndarray, w_router_bits: np.ndarray) -> np.ndarray:
    """float64 [T,E]: the router's gate GEMM x . w_router^T of bf16 bit patterns
    x [T,H] and w_router [E,H], in fp64."""
    xb = _c(x_bits, np.uint16)
    wb = _c(w_router_bits, np.uint16)
    T, H = xb.shape
    E = wb.shape[0]
    assert wb.shape[1] == H
    out = np.empty((T, E), np.float64)
    lib().oracle_router_logits(_p(xb), _p(wb), T, H, E, _p(out))
    return out


def router(x_bits: np.ndarray, w_router_bits: np.ndarray, K: int, **route_kw):
    """The fused router: fp64 gate GEMM, rounded to the route step's fp32 logit
    type, then route_ex.  -> (logits64 [T,E], logits32 [T,E], ids [T,K], w [T,K])."""
    l64 = router_logits(x_bits, w_router_bits)
    l32 = l64.astype(np.float32)
    ids, w = route_ex(l32, K, **route_kw)
    return l64, l32, ids, w


def sort(ids: np.ndarray, E: int):
    """-> (offsets [E+1], sorted_route [R], inv_route [R], n_out_of_range)."""
    ids = _c(ids, np.int32)
    T, K = ids.shape
    off = np.empty(E + 1, np.int32)
    sr = np.empty(T * K, np.int32)
    inv = np.empty(T * K, np.int32)
    bad = lib().oracle_sort(_p(ids), T, K, E, _p(off), _p(sr), _p(inv))
    return off, sr, inv, bad


def ffn_sorted(x: np.ndarray, K: int, experts, offsets, sorted_route, w) -> np.ndarray:
    """y_sorted float64 [T*K, H]: row p = w[r] * FFN_e(x[r // K]) for r = sorted_route[p]."""
    x = _c(x, np.uint16)
    T, H = x.shape
    ex = _ExpertsRef(experts)
    off, sr, wv = _c(offsets, np.int32), _c(sorted_route, np.int32), _c(w, np.float64).ravel()
    y = np.zeros((T * K, H), np.float64)
    lib().oracle_ffn_sorted(_p(x), T, H, K, ex.ref(), _p(off), _p(sr), _p(wv), _p(y))
    return y


def ffn_shared(x: np.ndarray, shared) -> np.ndarray:
    x = _c(x, np.uint16)
    T, H = x.shape
    ex = _ExpertsRef(shared)
    y = np.empty((T, H), np.float64)
    lib().oracle_ffn_shared(_p(x), T, H, ex.ref(), _p(y))
    return y


# ---------------------------------------------------------------- W8A8 form (FP8 activations)

XQ_BLOCK, HQ_BLOCK = 128, 64


def e4m3fn_round(v) -> np.ndarray:
    """Nearest E4M3FN value (ties to even, saturating at 448) of each element."""
    a = _c(np.atleast_1d(v), np.float64)
    out = np.empty_like(a)
    lib().oracle_e4m3fn_round_array(_p(a), a.size, _p(out))
    return out.reshape(np.shape(v))


def act_scale_exp(amax: float) -> int:
    """k with amax * 2^k in (224, 448] (0 for amax == 0, k in [-126, 126])."""
    return int(lib().oracle_act_scale_exp(float(amax)))


def act_quantize(v: np.ndarray, block: int) -> np.ndarray:
    """Blocks of `block` values -> e4m3fn(v * 2^k) * 2^-k, k from each block's largest |v|."""
    a = _c(v, np.float64).ravel()
    out = np.empty_like(a)
    lib().oracle_act_quantize(_p(a), a.size, int(block), _p(out))
    return out.reshape(np.shape(v))


def ffn_sorted_w8a8(x: np.ndarray, K: int, experts, offsets, sorted_route, w) -> np.ndarray:
    """ffn_sorted in the W8A8 form: x quantised per 128-column block, h per 64-feature block."""
    x = _c(x, np.uint16)
    T, H = x.shape
    ex = _ExpertsRef(experts)
    off, sr, wv = _c(offsets, np.int32), _c(sorted_route, np.int32), _c(w, np.float64).ravel()
    y = np.zeros((T * K, H), np.float64)
    lib().oracle_ffn_sorted_w8a8(_p(x), T, H, K, ex.ref(), _p(off), _p(sr), _p(wv), _p(y))
    return y


def ffn_shared_w8a8(x: np.ndarray, shared) -> np.ndarray:
    x = _c(x, np.uint16)
    T, H = x.shape
    ex = _ExpertsRef(shared)
    y = np.empty((T, H), np.float64)
    lib().oracle_ffn_shared_w8a8(_p(x), T, H, ex.ref(), _p(y))
    return y


def combine(y_sorted: np.ndarray, inv_route: np.ndarray, y_shared: Optional[np.ndarray],
            T: int, K: int) -> np.ndarray:
    ys = _c(y_sorted, np.float64)
    H = ys.shape[1]
    inv = _c(inv_route, np.int32)
    sh = None if y_shared is None else _c(y_shared, np.float64)
    out = np.empty((T, H), np.float64)
    lib().oracle_combine(_p(ys), _p(inv), _p(sh), T, K, H, _p(out))
    return out


def combine_bf16(y_sorted: np.ndarray, inv_route: np.ndarray, y_shared: Optional[np.ndarray],
                 T: int, K: int) -> np.ndarray:
    ys = _c(y_sorted, np.uint16)
    H = ys.shape[1]
    inv = _c(inv_route, np.int32)
    sh = None if y_shared is None else _c(y_shared, np.uint16)
    out = np.empty((T, H), np.float64)
    lib().oracle_combine_bf16(_p(ys), _p(inv), _p(sh), T, K, H, _p(out))
    return out


def moe(x, logits, K, routed, shared=None, zero_mask=None) -> dict:
    """Structured oracle: every intermediate of route -> sort -> FFN -> combine."""
    x = _c(x, np.uint16)
    lg = _c(logits, np.float32)
    T, H = x.shape
    E = lg.shape[1]
    R = T * K
    r = _ExpertsRef(routed)
    s = _ExpertsRef(shared) if shared is not None else None
    zm = None if zero_mask is None else _c(zero_mask, np.uint8)
    o = dict(ids=np.empty((T, K), np.int32), w=np.empty((T, K), np.float64),
             offsets=np.empty(E + 1, np.int32), sorted_route=np.empty(R, np.int32),
             inv_route=np.empty(R, np.int32), y_sorted=np.zeros((R, H), np.float64),
             y_shared=np.zeros((T, H), np.float64) if s else None,
             out=np.empty((T, H), np.float64))
    o["bad"] = lib().oracle_moe(
        _p(x), _p(lg), T, H, E, K, _p(zm), r.ref(), s.ref() if s else None,
        _p(o["ids"]), _p(o["w"]), _p(o["offsets"]), _p(o["sorted_route"]), _p(o["inv_route"]),
        _p(o["y_sorted"]), _p(o["y_shared"]), _p(o["out"]))
    return o


def moe_tokens(x, logits, K, routed, shared=None, zero_mask=None, tokens=None) -> np.ndarray:
    """Brute-force oracle rows out[i] for token tokens[i] (all tokens if None)."""
    x = _c(x, np.uint16)
    lg = _c(logits, np.float32)
    T, H = x.shape
    E = lg.shape[1]
    r = _ExpertsRef(routed)
    s = _ExpertsRef(shared) if shared is not None else None
    zm = None if zero_mask is None else _c(zero_mask, np.uint8)
    tk = None if tokens is None else _c(tokens, np.int32)
    n = T if tk is None else tk.size
    out = np.empty((n, H), np.float64)
    lib().oracle_moe_tokens(_p(x), _p(lg), T, H, E, K, _p(zm), r.ref(), s.ref() if s else None,
                            _p(tk), n, _p(out))
    return out


def moe_tokens_routed(x, ids, w, routed, shared=None, tokens=None) -> np.ndarray:
    """Brute-force rows out[i] for token tokens[i] with the routing given:
    ids / w [n, K] are token tokens[i]'s experts and weights (any router)."""
    x = _c(x, np.uint16)
    H = x.shape[1]
    idc, wc = _c(ids, np.int32), _c(w, np.float64)
    n, K = idc.shape
    r = _ExpertsRef(routed)
    s = _ExpertsRef(shared) if shared is not None else None
    tk = None if tokens is None else _c(tokens, np.int32)
    assert tk is None or tk.size == n
    out = np.empty((n, H), np.float64)
    lib().oracle_moe_tokens_routed(_p(x), H, K, _p(idc), _p(wc), r.ref(), s.ref() if s else None,
                                   _p(tk), n, _p(out))
    return out


def expert_rows(x, experts, e: int, rows) -> np.ndarray:
    """FFN_e(x[rows[i]]) for each i (no routing, no affinity)."""
    x = _c(x, np.uint16)
    H = x.shape[1]
    ex = _ExpertsRef(experts)
    rw = _c(rows, np.int32)
    y = np.empty((rw.size, H), np.float64)
    lib().oracle_expert_rows(_p(x), H, ex.ref(), int(e), _p(rw), rw.size, _p(y))
    return y


def swiglu(g: np.ndarray, u: np.ndarray) -> np.ndarray:
    g, u = _c(g, np.float64).ravel(), _c(u, np.float64).ravel()
    h = np.empty_like(g)
    lib().oracle_swiglu(_p(g), _p(u), g.size, _p(h))
    return h


def workload(wl) -> dict:
    """Structured oracle of a mixture_experts_ffn_sort_b200.workloads.Workload."""
    return moe(wl.x, wl.logits, wl.shape.K, wl.routed, wl.shared, wl.zero_mask)
