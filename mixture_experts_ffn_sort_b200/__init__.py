"""Routed MoE FFN for NVIDIA B200: Python binding of libmoe_ffn_b200.so.

The library (include/moe_ffn.h) exports moe_route, moe_sort, moe_expert_ffn
and moe_combine.  This module marshals torch tensors into those calls: device
pointers, sizes and the current CUDA stream.  Every step of the computation
runs in the library's kernels; torch only allocates device memory.  There is no
fallback: if the library is missing, every call raises.
"""
from __future__ import annotations

import ctypes
import os
import threading
from dataclasses import dataclass
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoe_ffn_b200.so")

MOE_OK = 0
MOE_ERR_INVALID_ARG = -1
MOE_ERR_UNSUPPORTED_SHAPE = -2
MOE_ERR_MISALIGNED = -3
MOE_ERR_WORKSPACE_TOO_SMALL = -4
MOE_ERR_CUDA = -5
MOE_MODE_AUTO, MOE_MODE_DECODE, MOE_MODE_PREFILL, MOE_MODE_HYBRID = 0, 1, 2, 3
MOE_HYBRID_ROW_SPLIT = 8
MOE_OUT_BF16, MOE_OUT_F32 = 0, 1
MOE_STATUS_BAD_ID, MOE_STATUS_BAD_MAP, MOE_STATUS_TIMEOUT = 1, 2, 4
MOE_MAX_E, MOE_MAX_K = 1024, 32

EXPORTED = ("moe_last_error", "moe_abi_version", "moe_route", "moe_route_ex", "moe_router", "moe_sort_workspace_bytes",
            "moe_sort", "moe_selftest_bounded_wait", "moe_router_plan_check",
            "moe_sort_static_ws", "moe_ffn_resolve_mode", "moe_ffn_workspace_bytes", "moe_expert_ffn", "moe_combine",
            "moe_ffn_combine_workspace_bytes", "moe_expert_ffn_combine", "moe_ffn_w8a8_workspace_bytes",
            "moe_expert_ffn_w8a8")


class MoEError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__("MoE call failed (%d): %s" % (code, msg))
        self.code = code


class _Experts(ctypes.Structure):
    _fields_ = [("w_gate", ctypes.c_void_p), ("w_up", ctypes.c_void_p), ("w_down", ctypes.c_void_p),
                ("s_gate", ctypes.c_void_p), ("s_up", ctypes.c_void_p), ("s_down", ctypes.c_void_p),
                ("n_experts", ctypes.c_int), ("inter", ctypes.c_int)]


class _RouteConfig(ctypes.Structure):
    _fields_ = [("score", ctypes.c_int), ("sel_bias", ctypes.c_void_p), ("n_group", ctypes.c_int),
                ("topk_group", ctypes.c_int), ("renormalize", ctypes.c_int), ("scaling", ctypes.c_float)]


_lock = threading.Lock()
_L = None


def lib() -> ctypes.CDLL:
    """Load the CUDA library (raises if it has not been built)."""
    global _L
    with _lock:
        if _L is None:
            if not os.path.exists(LIB_PATH):
                raise RuntimeError("%s is missing: build it with "
                                   "`python -m mixture_experts_ffn_sort_b200.build`" % LIB_PATH)
            L = ctypes.CDLL(LIB_PATH)
            P, I, S = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
            L.moe_last_error.restype = ctypes.c_char_p
            L.moe_abi_version.restype = I
            L.moe_route.argtypes = [P, I, I, I, P, P, P, P]
            L.moe_route_ex.argtypes = [P, I, I, I, ctypes.POINTER(_RouteConfig), P, P, P, P]
            L.moe_route_ex.restype = I
            L.moe_router.argtypes = [P, I, I, P, I, I, ctypes.POINTER(_RouteConfig), P, P, P, P, P, P]
            L.moe_router.restype = I
            L.moe_router_plan_check.argtypes = [I, I, I, I, P]
            L.moe_router_plan_check.restype = I
            L.moe_selftest_bounded_wait.argtypes = [P, P, P]
            L.moe_selftest_bounded_wait.restype = I
            L.moe_route.restype = I
            L.moe_sort_workspace_bytes.argtypes = [I, I, I]
            L.moe_sort_workspace_bytes.restype = S
            L.moe_sort.argtypes = [P, I, I, I, P, P, P, P, S, P, P]
            L.moe_sort.restype = I
            L.moe_sort_static_ws.argtypes = [P, I, I, I, P, P, P, P, P]
            L.moe_sort_static_ws.restype = I
            L.moe_ffn_resolve_mode.argtypes = [I, I, I, I]
            L.moe_ffn_resolve_mode.restype = I
            L.moe_ffn_workspace_bytes.argtypes = [I, I, I, I, I, I, I]
            L.moe_ffn_workspace_bytes.restype = S
            L.moe_expert_ffn.argtypes = [P, I, I, I, P, P, P, P, P, P, P, I, P, S, P, P]
            L.moe_expert_ffn.restype = I
            L.moe_ffn_combine_workspace_bytes.argtypes = [I, I, I, I, I, I, I]
            L.moe_ffn_combine_workspace_bytes.restype = S
            L.moe_expert_ffn_combine.argtypes = [P, I, I, I, P, P, P, P, P, P, I, P, S, P, P]
            L.moe_expert_ffn_combine.restype = I
            L.moe_ffn_w8a8_workspace_bytes.argtypes = [I, I, I, I]
            L.moe_ffn_w8a8_workspace_bytes.restype = S
            L.moe_expert_ffn_w8a8.argtypes = [P, I, I, I, P, P, P, P, P, P, P, P, S, P, P]
            L.moe_expert_ffn_w8a8.restype = I
            L.moe_combine.argtypes = [P, P, P, I, I, I, P, I, P, P]
            L.moe_combine.restype = I
            _L = L
    return _L


def _check(rc: int):
    if rc != MOE_OK:
        raise MoEError(rc, lib().moe_last_error().decode())


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _need_cuda(*ts):
    for t in ts:
        if t is not None and not t.is_cuda:
            raise ValueError("tensors must be CUDA tensors")


@dataclass
class Experts:
    """Block-scaled FP8 experts resident on the device (see moe_fp8_experts).

    w_gate, w_up: uint8 [n, I, H]; w_down: uint8 [n, H, I];
    s_gate, s_up: float32 [n, I/128, H/128]; s_down: float32 [n, H/128, I/128].
    """

    w_gate: torch.Tensor
    s_gate: torch.Tensor
    w_up: torch.Tensor
    s_up: torch.Tensor
    w_down: torch.Tensor
    s_down: torch.Tensor

    @property
    def n(self) -> int:
        return self.w_gate.shape[0]

    @property
    def inter(self) -> int:
        return self.w_gate.shape[1]

    def struct(self) -> _Experts:
        return _Experts(self.w_gate.data_ptr(), self.w_up.data_ptr(), self.w_down.data_ptr(),
                        self.s_gate.data_ptr(), self.s_up.data_ptr(), self.s_down.data_ptr(),
                        self.n, self.inter)

    @staticmethod
    def from_host(ex, device="cuda") -> "Experts":
        """Copy host experts (any object with numpy w_*/s_* arrays) to the device."""
        def t(a):
            return torch.from_numpy(a).to(device)
        return Experts(t(ex.w_gate), t(ex.s_gate), t(ex.w_up), t(ex.s_up), t(ex.w_down), t(ex.s_down))


# ---------------------------------------------------------------- the four calls

def moe_route(logits: torch.Tensor, K: int, zero_mask: Optional[torch.Tensor] = None,
              topk_ids: Optional[torch.Tensor] = None, topk_w: Optional[torch.Tensor] = None,
              stream=None):
    """logits [T, E] f32 -> (topk_ids [T, K] i32, topk_w [T, K] f32)."""
    _need_cuda(logits, zero_mask)
    T, E = logits.shape
    if topk_ids is None:
        topk_ids = torch.empty((T, K), dtype=torch.int32, device=logits.device)
    if topk_w is None:
        topk_w = torch.empty((T, K), dtype=torch.float32, device=logits.device)
    _check(lib().moe_route(_ptr(logits), T, E, K, _ptr(zero_mask), _ptr(topk_ids), _ptr(topk_w),
                           _stream(stream)))
    return topk_ids, topk_w


MOE_SCORE_SOFTMAX, MOE_SCORE_SIGMOID = 0, 1


def moe_route_ex(logits: torch.Tensor, K: int, score: int = MOE_SCORE_SOFTMAX,
                 sel_bias: Optional[torch.Tensor] = None, n_group: int = 1, topk_group: Optional[int] = None,
                 renormalize: bool = True, scaling: float = 1.0, zero_mask: Optional[torch.Tensor] = None,
                 topk_ids: Optional[torch.Tensor] = None, topk_w: Optional[torch.Tensor] = None, stream=None):
    """Routing variants: logits [T, E] f32 -> (topk_ids [T, K] i32, topk_w [T, K] f32).
    sel_bias [E] f32 (selection only); n_group / topk_group: group-limited choice."""
    _need_cuda(logits, zero_mask, sel_bias)
    T, E = logits.shape
    if topk_ids is None:
        topk_ids = torch.empty((T, K), dtype=torch.int32, device=logits.device)
    if topk_w is None:
        topk_w = torch.empty((T, K), dtype=torch.float32, device=logits.device)
    cfg = _RouteConfig(int(score), _ptr(sel_bias), int(n_group),
                       int(n_group if topk_group is None else topk_group), int(bool(renormalize)), float(scaling))
    _check(lib().moe_route_ex(_ptr(logits), T, E, K, ctypes.byref(cfg), _ptr(zero_mask), _ptr(topk_ids),
                              _ptr(topk_w), _stream(stream)))
    return topk_ids, topk_w



MOE_ROUTER_MAX_E = 512


def moe_router(x: torch.Tensor, w_router: torch.Tensor, K: int, score: int = MOE_SCORE_SOFTMAX,
               sel_bias: Optional[torch.Tensor] = None, n_group: int = 1, topk_group: Optional[int] = None,
               renormalize: bool = True, scaling: float = 1.0, zero_mask: Optional[torch.Tensor] = None,
               logits: Optional[torch.Tensor] = None, status: Optional[torch.Tensor] = None,
               topk_ids: Optional[torch.Tensor] = None, topk_w: Optional[torch.Tensor] = None, stream=None):
    """Fused router: x [T, H] bf16 and w_router [E, H] bf16 -> (topk_ids [T, K] i32, topk_w [T, K] f32),
    the gate GEMM and the routing of moe_route_ex in one kernel.  logits [T, E] f32, if given,
    receives the fp32 logits."""
    _need_cuda(x, w_router, zero_mask, sel_bias, logits, status)
    T, H = x.shape
    E = w_router.shape[0]
    if topk_ids is None:
        topk_ids = torch.empty((T, K), dtype=torch.int32, device=x.device)
    if topk_w is None:
        topk_w = torch.empty((T, K), dtype=torch.float32, device=x.device)
    cfg = _RouteConfig(int(score), _ptr(sel_bias), int(n_group),
                       int(n_group if topk_group is None else topk_group), int(bool(renormalize)), float(scaling))
    _check(lib().moe_router(_ptr(x), T, H, _ptr(w_router), E, K, ctypes.byref(cfg), _ptr(zero_mask),
                            _ptr(topk_ids), _ptr(topk_w), _ptr(logits), _ptr(status), _stream(stream)))
    return topk_ids, topk_w


def moe_selftest_bounded_wait(stream=None):
    """Make the library's bounded wait run out on purpose (about 2 s): returns
    (status word, [elapsed ns of the two waits]) after a synchronize."""
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    elapsed = torch.zeros(2, dtype=torch.int64, device="cuda")
    _check(lib().moe_selftest_bounded_wait(_ptr(status), _ptr(elapsed), _stream(stream)))
    torch.cuda.synchronize()
    return int(status.item()), [int(v) for v in elapsed.cpu().tolist()]

def moe_sort_workspace_bytes(T: int, K: int, E: int) -> int:
    return int(lib().moe_sort_workspace_bytes(T, K, E))


def moe_sort(topk_ids: torch.Tensor, E: int, status: Optional[torch.Tensor] = None,
             expert_offsets=None, sorted_route=None, inv_route=None, workspace=None, stream=None):
    """topk_ids [T, K] i32 -> (expert_offsets [E+1], sorted_route [T*K], inv_route [T*K])."""
    _need_cuda(topk_ids, status)
    T, K = topk_ids.shape
    dev = topk_ids.device
    if expert_offsets is None:
        expert_offsets = torch.empty(E + 1, dtype=torch.int32, device=dev)
    if sorted_route is None:
        sorted_route = torch.empty(T * K, dtype=torch.int32, device=dev)
    if inv_route is None:
        inv_route = torch.empty(T * K, dtype=torch.int32, device=dev)
    need = moe_sort_workspace_bytes(T, K, E)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=dev)
    _check(lib().moe_sort(_ptr(topk_ids), T, K, E, _ptr(expert_offsets), _ptr(sorted_route),
                          _ptr(inv_route), _ptr(workspace), workspace.numel(), _ptr(status),
                          _stream(stream)))
    return expert_offsets, sorted_route, inv_route


def moe_ffn_resolve_mode(T: int, K: int, E: int, mode: int = MOE_MODE_AUTO) -> int:
    """The FFN form (MOE_MODE_DECODE, MOE_MODE_PREFILL or MOE_MODE_HYBRID) moe_expert_ffn runs for `mode`."""
    rc = int(lib().moe_ffn_resolve_mode(T, K, E, mode))
    _check(min(rc, 0))
    return rc


def moe_ffn_workspace_bytes(T, K, H, E, I, I_shared=0, mode=MOE_MODE_AUTO) -> int:
    return int(lib().moe_ffn_workspace_bytes(T, K, H, E, I, I_shared, mode))


def moe_expert_ffn(x: torch.Tensor, K: int, routed: Experts, expert_offsets: torch.Tensor,
                   sorted_route: torch.Tensor, topk_w: torch.Tensor, shared: Optional[Experts] = None,
                   mode: int = MOE_MODE_AUTO, status: Optional[torch.Tensor] = None,
                   y_sorted=None, y_shared=None, workspace=None, stream=None):
    """x [T, H] bf16 -> (y_sorted [T*K, H] bf16, y_shared [T, H] bf16 or None)."""
    _need_cuda(x, expert_offsets, sorted_route, topk_w, status)
    T, H = x.shape
    dev = x.device
    if y_sorted is None:
        y_sorted = torch.empty((T * K, H), dtype=torch.bfloat16, device=dev)
    if shared is not None and y_shared is None:
        y_shared = torch.empty((T, H), dtype=torch.bfloat16, device=dev)
    need = moe_ffn_workspace_bytes(T, K, H, routed.n, routed.inter, shared.inter if shared else 0, mode)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=dev)
    rs = routed.struct()
    ss = shared.struct() if shared is not None else None
    _check(lib().moe_expert_ffn(_ptr(x), T, H, K, ctypes.byref(rs),
                                ctypes.byref(ss) if ss is not None else None,
                                _ptr(expert_offsets), _ptr(sorted_route), _ptr(topk_w), _ptr(y_sorted),
                                _ptr(y_shared) if shared is not None else None, mode, _ptr(workspace),
                                workspace.numel(), _ptr(status), _stream(stream)))
    return y_sorted, (y_shared if shared is not None else None)


def moe_ffn_w8a8_workspace_bytes(T: int, K: int, I: int, I_shared: int = 0) -> int:
    return int(lib().moe_ffn_w8a8_workspace_bytes(T, K, I, I_shared))


def moe_expert_ffn_w8a8(x: torch.Tensor, K: int, routed: Experts, expert_offsets: torch.Tensor,
                        sorted_route: torch.Tensor, topk_w: torch.Tensor, shared: Optional[Experts] = None,
                        status: Optional[torch.Tensor] = None, y_sorted=None, y_shared=None, workspace=None,
                        stream=None):
    """moe_expert_ffn with FP8 activations (the opt-in W8A8 form)."""
    _need_cuda(x, expert_offsets, sorted_route, topk_w, status)
    T, H = x.shape
    dev = x.device
    if y_sorted is None:
        y_sorted = torch.empty((T * K, H), dtype=torch.bfloat16, device=dev)
    if shared is not None and y_shared is None:
        y_shared = torch.empty((T, H), dtype=torch.bfloat16, device=dev)
    need = moe_ffn_w8a8_workspace_bytes(T, K, routed.inter, shared.inter if shared else 0)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=dev)
    rs = routed.struct()
    ss = shared.struct() if shared is not None else None
    _check(lib().moe_expert_ffn_w8a8(_ptr(x), T, H, K, ctypes.byref(rs),
                                     ctypes.byref(ss) if ss is not None else None,
                                     _ptr(expert_offsets), _ptr(sorted_route), _ptr(topk_w), _ptr(y_sorted),
                                     _ptr(y_shared) if shared is not None else None, _ptr(workspace),
                                     workspace.numel(), _ptr(status), _stream(stream)))
    return y_sorted, (y_shared if shared is not None else None)


def moe_ffn_combine_workspace_bytes(T, K, H, E, I, I_shared=0, out_dtype=MOE_OUT_BF16) -> int:
    return int(lib().moe_ffn_combine_workspace_bytes(T, K, H, E, I, I_shared, out_dtype))


def moe_expert_ffn_combine(x: torch.Tensor, K: int, routed: Experts, expert_offsets: torch.Tensor,
                           sorted_route: torch.Tensor, topk_w: torch.Tensor, shared: Optional[Experts] = None,
                           out_dtype: int = MOE_OUT_BF16, status: Optional[torch.Tensor] = None, out=None,
                           workspace=None, stream=None):
    """x [T, H] bf16 -> out [T, H] (bf16 or f32): the expert FFN and the combine
    in one call (tensor-core kernels; fp32 reductions in no fixed order)."""
    _need_cuda(x, expert_offsets, sorted_route, topk_w, status)
    T, H = x.shape
    dev = x.device
    if out is None:
        dt = torch.bfloat16 if out_dtype == MOE_OUT_BF16 else torch.float32
        out = torch.empty((T, H), dtype=dt, device=dev)
    need = moe_ffn_combine_workspace_bytes(T, K, H, routed.n, routed.inter, shared.inter if shared else 0, out_dtype)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=dev)
    rs = routed.struct()
    ss = shared.struct() if shared is not None else None
    _check(lib().moe_expert_ffn_combine(_ptr(x), T, H, K, ctypes.byref(rs),
                                        ctypes.byref(ss) if ss is not None else None, _ptr(expert_offsets),
                                        _ptr(sorted_route), _ptr(topk_w), _ptr(out), out_dtype, _ptr(workspace),
                                        workspace.numel(), _ptr(status), _stream(stream)))
    return out


def moe_combine(y_sorted: torch.Tensor, inv_route: torch.Tensor, y_shared: Optional[torch.Tensor],
                T: int, K: int, out_dtype: int = MOE_OUT_BF16, out=None, stream=None,
                status: Optional[torch.Tensor] = None):
    """-> out [T, H] (bf16 or f32).  status: optional int32 device word that
    receives MOE_STATUS_BAD_MAP for an out-of-range inv_route entry."""
    _need_cuda(y_sorted, inv_route, y_shared, status)
    H = y_sorted.shape[1]
    if out is None:
        dt = torch.bfloat16 if out_dtype == MOE_OUT_BF16 else torch.float32
        out = torch.empty((T, H), dtype=dt, device=y_sorted.device)
    _check(lib().moe_combine(_ptr(y_sorted), _ptr(inv_route), _ptr(y_shared), T, K, H, _ptr(out),
                             out_dtype, _ptr(status), _stream(stream)))
    return out


# ---------------------------------------------------------------- whole layer

class MoEFFN:
    """The routed MoE FFN of one layer on fixed shapes: route -> sort -> expert
    FFN -> combine, with every buffer allocated once (no allocation per call,
    so a call can be captured in a CUDA graph after the first one).
    route_cfg: keyword arguments of moe_route_ex (score, sel_bias, n_group,
    topk_group, renormalize, scaling) for a routing variant; None routes with
    moe_route.  w_router: bf16 [E, H] gate vectors for forward_fused, which
    routes with the fused router (moe_router) from x alone.  fused_combine:
    run the expert FFN and the combine as one call (moe_expert_ffn_combine:
    tensor-core kernels, no y_sorted, fp32 reductions in no fixed order).
    w8a8: FP8 activations (moe_expert_ffn_w8a8, weight-streaming kernels);
    `mode` is then ignored."""

    def __init__(self, routed: Experts, T: int, K: int, shared: Optional[Experts] = None,
                 mode: int = MOE_MODE_AUTO, out_dtype: int = MOE_OUT_BF16, device="cuda",
                 route_cfg: Optional[dict] = None, w_router: Optional[torch.Tensor] = None,
                 fused_combine: bool = False, w8a8: bool = False):
        if fused_combine and w8a8:
            raise ValueError("fused_combine and w8a8 are separate forms")
        self.routed, self.shared, self.T, self.K = routed, shared, T, K
        self.fused_combine = fused_combine
        self.w8a8 = w8a8
        self.w_router = w_router
        self.route_cfg = dict(route_cfg) if route_cfg else None
        self.E, self.I, self.H = routed.n, routed.inter, routed.w_gate.shape[2]
        self.mode, self.out_dtype = mode, out_dtype
        d = device
        R = T * K
        self.topk_ids = torch.empty((T, K), dtype=torch.int32, device=d)
        self.topk_w = torch.empty((T, K), dtype=torch.float32, device=d)
        self.offsets = torch.empty(self.E + 1, dtype=torch.int32, device=d)
        self.sorted_route = torch.empty(R, dtype=torch.int32, device=d)
        self.inv_route = torch.empty(R, dtype=torch.int32, device=d)
        self.sort_ws = torch.empty(max(16, moe_sort_workspace_bytes(T, K, self.E)), dtype=torch.uint8, device=d)
        if fused_combine:
            self.ffn_ws = torch.empty(max(16, moe_ffn_combine_workspace_bytes(
                T, K, self.H, self.E, self.I, shared.inter if shared else 0, out_dtype)), dtype=torch.uint8, device=d)
            self.y_sorted, self.y_shared = None, None
        else:
            Is = shared.inter if shared else 0
            need = (moe_ffn_w8a8_workspace_bytes(T, K, self.I, Is) if w8a8 else
                    moe_ffn_workspace_bytes(T, K, self.H, self.E, self.I, Is, mode))
            self.ffn_ws = torch.empty(max(16, need), dtype=torch.uint8, device=d)
            self.y_sorted = torch.empty((R, self.H), dtype=torch.bfloat16, device=d)
            self.y_shared = torch.empty((T, self.H), dtype=torch.bfloat16, device=d) if shared else None
        dt = torch.bfloat16 if out_dtype == MOE_OUT_BF16 else torch.float32
        self.out = torch.empty((T, self.H), dtype=dt, device=d)
        self.status = torch.zeros(1, dtype=torch.int32, device=d)

    # Number of the library's kernel launches one forward makes.
    def launches(self) -> int:
        R = self.T * self.K
        # The decode form runs the shared expert as a second kernel pair; the
        # prefill form runs it inside its two kernels.
        sort = 1 if R <= 16384 else 3
        if self.fused_combine:
            # f16 copy of x, gate/up, down with the reductions, fp32 -> bf16.
            return 1 + sort + 3 + (1 if self.out_dtype == MOE_OUT_BF16 else 0)
        form = MOE_MODE_DECODE if self.w8a8 else moe_ffn_resolve_mode(self.T, self.K, self.E, self.mode)
        # The tensor-core form also launches the f16 copy of x.
        ffn = {MOE_MODE_DECODE: 2 + (2 if self.shared is not None else 0), MOE_MODE_PREFILL: 3,
               MOE_MODE_HYBRID: 5}[form]
        return 1 + sort + ffn + 1

    def forward(self, x: torch.Tensor, logits: torch.Tensor, zero_mask: Optional[torch.Tensor] = None,
                stream=None) -> torch.Tensor:
        if self.route_cfg is None:
            moe_route(logits, self.K, zero_mask, self.topk_ids, self.topk_w, stream=stream)
        else:
            moe_route_ex(logits, self.K, zero_mask=zero_mask, topk_ids=self.topk_ids, topk_w=self.topk_w,
                         stream=stream, **self.route_cfg)
        return self._experts(x, stream)

    def forward_fused(self, x: torch.Tensor, zero_mask: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
        """The same layer with the router's gate GEMM fused into the routing step."""
        if self.w_router is None:
            raise ValueError("forward_fused needs w_router")
        moe_router(x, self.w_router, self.K, zero_mask=zero_mask, topk_ids=self.topk_ids, topk_w=self.topk_w,
                   stream=stream, **(self.route_cfg or {}))
        return self._experts(x, stream)

    def _experts(self, x: torch.Tensor, stream) -> torch.Tensor:
        moe_sort(self.topk_ids, self.E, self.status, self.offsets, self.sorted_route, self.inv_route,
                 self.sort_ws, stream=stream)
        if self.fused_combine:
            return moe_expert_ffn_combine(x, self.K, self.routed, self.offsets, self.sorted_route, self.topk_w,
                                          self.shared, self.out_dtype, self.status, self.out, self.ffn_ws,
                                          stream=stream)
        if self.w8a8:
            moe_expert_ffn_w8a8(x, self.K, self.routed, self.offsets, self.sorted_route, self.topk_w, self.shared,
                                self.status, self.y_sorted, self.y_shared, self.ffn_ws, stream=stream)
        else:
            moe_expert_ffn(x, self.K, self.routed, self.offsets, self.sorted_route, self.topk_w, self.shared,
                           self.mode, self.status, self.y_sorted, self.y_shared, self.ffn_ws, stream=stream)
        moe_combine(self.y_sorted, self.inv_route, self.y_shared, self.T, self.K, self.out_dtype, self.out,
                    stream=stream, status=self.status)
        return self.out

    __call__ = forward
