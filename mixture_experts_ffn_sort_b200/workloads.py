"""Seeded synthetic inputs for the routed MoE FFN.

This module draws inputs only: activations, router logits, expert weights
quantised to FP8 E4M3FN with one fp32 scale per 128x128 block, and the
zero-weight route mask.  It holds none of the MoE arithmetic (no softmax, no
top-k, no sort, no FP8 decode, no FFN); both the CUDA path and the CPU oracle
consume what it returns, and neither is imported here.

Shapes follow the workloads the source pages describe:
  * FP8 W8A16 MoE decode kernel (dstair/gated-deltanet-nki-trainium,
    "FP8 MoE decode kernel" section): 256 experts, top-8, H=2048, I=512,
    E4M3FN weights with 128x128 block scales.
  * gfx950 fused MXFP4 MoE prefill (ROCm/aiter PR #5988, latency table):
    width 4096/8192, intermediate 256, 512 routed experts top-10 plus one
    always-on shared expert, 8K-32K tokens, zero routing weights in the
    replay tests.

Every tensor has its own numpy PCG64 stream keyed by (seed, tag, index), so a
tensor is the same whatever else is drawn and experts can be drawn in
parallel threads without changing a single value.
"""
from __future__ import annotations

import os
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, field
from typing import Optional

import numpy as np
import torch

E4M3_MAX = 448.0
BLOCK = 128

# Stream tags: one independent stream per tensor kind.
_TAG_X, _TAG_LOGITS, _TAG_BIAS, _TAG_ROUTED, _TAG_SHARED, _TAG_MASK = 1, 2, 3, 4, 5, 6
_TAG_IDS, _TAG_YS, _TAG_PROBE, _TAG_SEL_BIAS, _TAG_ROUTER_W = 7, 8, 9, 10, 11


def _rng(seed: int, tag: int, index: int = 0) -> np.random.Generator:
    return np.random.default_rng([int(seed), int(tag), int(index)])


@dataclass(frozen=True)
class MoEShape:
    """One workload: T tokens of width H, E experts of intermediate I, top-K."""

    name: str
    T: int
    H: int
    I: int
    E: int
    K: int
    I_shared: int = 0          # 0: no shared expert
    bias: str = "none"         # "none" | "normal" | "zipf": per-expert logit offset
    bias_param: float = 0.0    # std of the normal bias, or the Zipf exponent s
    zero_frac: float = 0.0     # Bernoulli rate of routes whose weight is forced to 0
    weight_std: float = 0.02
    seed: int = 0

    @property
    def R(self) -> int:
        return self.T * self.K


# The five workloads.  The router bias is part of the data: it is added to the
# N(0,1) logits before they reach the route step.
SHAPES = {
    "tiny": MoEShape("tiny", T=16, H=256, I=128, E=8, K=2),
    "decode": MoEShape("decode", T=64, H=2048, I=512, E=256, K=8),
    "decode_skew": MoEShape("decode_skew", T=512, H=2048, I=512, E=256, K=8,
                            bias="normal", bias_param=1.5),
    "prefill": MoEShape("prefill", T=8192, H=4096, I=256, E=512, K=10,
                        I_shared=256, zero_frac=0.01),
    "prefill_large": MoEShape("prefill_large", T=32768, H=8192, I=256, E=512, K=10,
                              I_shared=256, bias="zipf", bias_param=1.1),
}
SHAPE_ORDER = ["tiny", "decode", "decode_skew", "prefill", "prefill_large"]


@dataclass
class FP8Experts:
    """Block-scaled FP8 expert weights, rows = output features, K contiguous.

    w_gate, w_up: uint8 E4M3FN codes [n, I, H]; w_down: [n, H, I].
    s_gate, s_up: float32 [n, I/128, H/128]; s_down: [n, H/128, I/128].
    """

    w_gate: np.ndarray
    s_gate: np.ndarray
    w_up: np.ndarray
    s_up: np.ndarray
    w_down: np.ndarray
    s_down: np.ndarray

    @property
    def n(self) -> int:
        return self.w_gate.shape[0]

    @property
    def inter(self) -> int:
        return self.w_gate.shape[1]

    @property
    def hidden(self) -> int:
        return self.w_gate.shape[2]


@dataclass
class Workload:
    shape: MoEShape
    x: np.ndarray                      # uint16 bf16 bit patterns [T, H]
    logits: np.ndarray                 # float32 [T, E]
    routed: FP8Experts
    shared: Optional[FP8Experts] = None
    zero_mask: Optional[np.ndarray] = None   # uint8 [T, K], 1 = weight forced to 0
    meta: dict = field(default_factory=dict)


def to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """float32 -> bf16 (round to nearest even, torch's cast), returned as uint16 bits."""
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def quantize_blocks(w: np.ndarray):
    """Offline weight preparation: float32 [rows, cols] -> (E4M3FN codes, block scales).

    One fp32 scale per 128x128 block, s = amax/448 (1 where the block is all
    zero); codes = torch's round-to-nearest-even E4M3FN cast of w/s, clamped
    to +-448 first so no code is NaN.
    """
    rows, cols = w.shape
    assert rows % BLOCK == 0 and cols % BLOCK == 0
    blk = w.reshape(rows // BLOCK, BLOCK, cols // BLOCK, BLOCK)
    amax = np.abs(blk).max(axis=(1, 3)).astype(np.float32)
    s = np.where(amax > 0, amax / np.float32(E4M3_MAX), np.float32(1.0)).astype(np.float32)
    q = blk / s[:, None, :, None]
    np.clip(q, -E4M3_MAX, E4M3_MAX, out=q)
    codes = torch.from_numpy(np.ascontiguousarray(q.reshape(rows, cols), dtype=np.float32))
    codes = codes.to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    return codes, s


def _draw_expert(seed: int, tag: int, e: int, I: int, H: int, std: float):
    rng = _rng(seed, tag, e)
    wg = rng.standard_normal((I, H), dtype=np.float32) * np.float32(std)
    wu = rng.standard_normal((I, H), dtype=np.float32) * np.float32(std)
    wd = rng.standard_normal((H, I), dtype=np.float32) * np.float32(std)
    return quantize_blocks(wg), quantize_blocks(wu), quantize_blocks(wd)


def draw_experts(seed: int, tag: int, n: int, I: int, H: int, std: float = 0.02,
                 threads: Optional[int] = None) -> FP8Experts:
    """n experts with N(0, std) weights quantised per 128x128 block."""
    ex = FP8Experts(
        w_gate=np.empty((n, I, H), np.uint8), s_gate=np.empty((n, I // BLOCK, H // BLOCK), np.float32),
        w_up=np.empty((n, I, H), np.uint8), s_up=np.empty((n, I // BLOCK, H // BLOCK), np.float32),
        w_down=np.empty((n, H, I), np.uint8), s_down=np.empty((n, H // BLOCK, I // BLOCK), np.float32),
    )

    def one(e):
        (qg, sg), (qu, su), (qd, sd) = _draw_expert(seed, tag, e, I, H, std)
        ex.w_gate[e], ex.s_gate[e] = qg, sg
        ex.w_up[e], ex.s_up[e] = qu, su
        ex.w_down[e], ex.s_down[e] = qd, sd

    threads = threads or min(16, os.cpu_count() or 1)
    if threads <= 1 or n == 1:
        for e in range(n):
            one(e)
    else:
        with ThreadPoolExecutor(threads) as pool:
            list(pool.map(one, range(n)))
    return ex


def logit_bias(shape: MoEShape) -> Optional[np.ndarray]:
    """Per-expert logit offset that skews expert load.

    "normal": bias[e] ~ N(0, bias_param).
    "zipf":   expert e gets rank 1 + pi(e) for a seeded permutation pi and
              bias[e] = -s * ln(rank), so exp(bias) is a Zipf(s) law over ranks.
    """
    if shape.bias == "none":
        return None
    rng = _rng(shape.seed, _TAG_BIAS)
    if shape.bias == "normal":
        return (rng.standard_normal(shape.E, dtype=np.float32) * np.float32(shape.bias_param))
    if shape.bias == "zipf":
        rank = 1 + rng.permutation(shape.E)
        return (-shape.bias_param * np.log(rank.astype(np.float64))).astype(np.float32)
    raise ValueError(shape.bias)


def make_workload(shape, seed: Optional[int] = None, threads: Optional[int] = None,
                  with_weights: bool = True) -> Workload:
    """Draw the full input set of one workload."""
    if isinstance(shape, str):
        shape = SHAPES[shape]
    if seed is not None:
        shape = MoEShape(**{**shape.__dict__, "seed": seed})
    T, H, I, E, K, s = shape.T, shape.H, shape.I, shape.E, shape.K, shape.seed
    x = to_bf16_bits(_rng(s, _TAG_X).standard_normal((T, H), dtype=np.float32))
    logits = _rng(s, _TAG_LOGITS).standard_normal((T, E), dtype=np.float32)
    b = logit_bias(shape)
    if b is not None:
        logits = (logits + b[None, :]).astype(np.float32)
    zero_mask = None
    if shape.zero_frac > 0:
        zero_mask = (_rng(s, _TAG_MASK).random((T, K)) < shape.zero_frac).astype(np.uint8)
    if with_weights:
        routed = draw_experts(s, _TAG_ROUTED, E, I, H, shape.weight_std, threads)
        shared = (draw_experts(s, _TAG_SHARED, 1, shape.I_shared, H, shape.weight_std, threads)
                  if shape.I_shared else None)
    else:
        routed, shared = None, None
    return Workload(shape=shape, x=x, logits=logits, routed=routed, shared=shared,
                    zero_mask=zero_mask, meta={"bias": b})


# ---------------------------------------------------------------------------
# Probe inputs for single-step tests and edge cases.

def selection_bias(E: int, seed: int = 0, std: float = 0.02) -> np.ndarray:
    """float32 [E] selection-only router bias ~ N(0, std) (the learned
    load-balancing correction of a DeepSeek-V3-style router, drawn)."""
    return (_rng(seed, _TAG_SEL_BIAS).standard_normal(E) * std).astype(np.float32)



def router_weight(E: int, H: int, seed: int = 0) -> np.ndarray:
    """uint16 bf16 bits [E, H]: the router's gate vectors ~ N(0, 1/H), so that
    for x ~ N(0, 1) the logits x . w_e are ~ N(0, 1), the logit distribution
    the routing workloads draw directly."""
    w = _rng(seed, _TAG_ROUTER_W).standard_normal((E, H), dtype=np.float32) * np.float32(1.0 / np.sqrt(H))
    return to_bf16_bits(w)

# Router variants of the benchmark and the end-to-end tests, by name: keyword
# arguments of moe_route_ex / oracle.route_ex (a selection bias, when used, is
# selection_bias(E, seed)).  "softmax" is the plain router.
ROUTERS = {
    "softmax": None,
    "sigmoid": dict(score=1, n_group=1, topk_group=1, renormalize=True, scaling=2.5),
    "grouped": dict(score=1, n_group=8, topk_group=4, renormalize=True, scaling=2.5, bias=True),
}


def random_ids(T: int, K: int, E: int, seed: int = 0, distinct: bool = True) -> np.ndarray:
    """int32 [T, K] expert ids; distinct within a token unless distinct=False."""
    rng = _rng(seed, _TAG_IDS)
    if distinct:
        ids = np.argsort(rng.random((T, E)), axis=1)[:, :K]
    else:
        ids = rng.integers(0, E, size=(T, K))
    return np.ascontiguousarray(ids, dtype=np.int32)


def skewed_ids(T: int, K: int, E: int, hot: int, seed: int = 0) -> np.ndarray:
    """Every token routes slot 0 to expert `hot`; the other slots are random and distinct."""
    rng = _rng(seed, _TAG_IDS, 1)
    ids = np.empty((T, K), np.int32)
    others = np.array([e for e in range(E) if e != hot])
    for t in range(T):
        ids[t, 0] = hot
        ids[t, 1:] = rng.permutation(others)[: K - 1]
    return ids


def random_rows_bf16(n: int, H: int, seed: int = 0, std: float = 1.0) -> np.ndarray:
    """uint16 bf16 bits [n, H] drawn N(0, std)."""
    return to_bf16_bits(_rng(seed, _TAG_YS).standard_normal((n, H), dtype=np.float32) * np.float32(std))


def tie_logits(T: int, E: int, seed: int = 0, levels: int = 3) -> np.ndarray:
    """float32 [T, E] logits drawn from {0, ..., levels-1}: many exact ties."""
    rng = _rng(seed, _TAG_PROBE)
    return rng.integers(0, levels, size=(T, E)).astype(np.float32)


def subnormal_experts(n: int, I: int, H: int, seed: int = 0) -> FP8Experts:
    """Experts whose codes are all E4M3FN subnormals or zero (exponent field 0),
    with block scales of order 1, so the subnormal values dominate the result."""
    rng = _rng(seed, _TAG_PROBE, 1)

    def codes(r, c):
        mant = rng.integers(0, 8, size=(n, r, c), dtype=np.uint8)
        sign = rng.integers(0, 2, size=(n, r, c), dtype=np.uint8) << 7
        return (mant | sign).astype(np.uint8)

    def scales(r, c):
        return (0.5 + rng.random((n, r // BLOCK, c // BLOCK))).astype(np.float32)

    return FP8Experts(codes(I, H), scales(I, H), codes(I, H), scales(I, H),
                      codes(H, I), scales(H, I))


def all_code_experts(n: int, I: int, H: int, seed: int = 0) -> FP8Experts:
    """Experts whose codes are uniform over all 254 finite E4M3FN codes, with
    block scales in [2^-12, 2^-8] so every product stays finite."""
    rng = _rng(seed, _TAG_PROBE, 2)
    finite = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], dtype=np.uint8)

    def codes(r, c):
        return finite[rng.integers(0, finite.size, size=(n, r, c))]

    def scales(r, c):
        return np.exp2(rng.uniform(-12, -8, size=(n, r // BLOCK, c // BLOCK))).astype(np.float32)

    return FP8Experts(codes(I, H), scales(I, H), codes(I, H), scales(I, H),
                      codes(H, I), scales(H, I))
