"""Host-side pieces of bench.py (CPU only): the oracle leg of the fused-router
option and the reference arm's JSON line."""
import json
import os
import subprocess
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
import oracle  # noqa: E402
from mixture_experts_ffn_sort_b200 import workloads as wl  # noqa: E402


def test_fused_router_oracle_rows_route_from_x():
    """With the fused router the oracle rows are the method on the logits of
    the router's gate GEMM of x (not the workload's drawn logits)."""
    shape = wl.SHAPES["tiny"]
    w = wl.make_workload("tiny")
    tk = np.arange(shape.T, dtype=np.int32)
    got = bench.oracle_rows(w, shape, tk, "softmax", fused_router=True)
    _, _, ids, wt = oracle.router(w.x, wl.router_weight(shape.E, shape.H, shape.seed), shape.K,
                                  zero_mask=w.zero_mask)
    ref = oracle.moe_tokens_routed(w.x, ids, wt, w.routed, w.shared, tokens=tk)
    assert np.array_equal(got, ref)
    plain = bench.oracle_rows(w, shape, tk, "softmax")
    assert not np.array_equal(got, plain)


def test_reference_arm_line_with_fused_router():
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload", "tiny",
                        "--fused-router", "--steps", "1", "--warmup", "0"], capture_output=True, text=True,
                       cwd=ROOT, timeout=300)
    assert r.returncode == 0, r.stderr
    line = json.loads(r.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["value"] > 0
    assert "moe_router" in line["config"]["logits"] and line["config"]["logit_bias"] is None


def test_ffn_roofline_objects():
    """The FFN roofline: touched-expert bytes over HBM for the weight-streaming
    and hybrid forms, bf16 FLOPs over the tensor cores for the prefill form,
    with the DRAM traffic of the committed ncu summary while the FFN kernels'
    sources still match it."""
    peaks = {"hbm": 6544.0, "bf16_sus": 1388.3, "src": "test"}
    dec = wl.SHAPES["decode"]
    r = bench.ffn_roofline(dec, "decode", touched=222, flops=0, ffn_ms=0.119, peaks=peaks)
    algo = 222 * bench.expert_bytes(dec.H, dec.I)
    assert r["bound"] == "hbm" and r["algorithmic_bytes"] == algo
    assert abs(r["achieved"] - algo / 0.119e-3 / 1e9) < 1e-6 * r["achieved"]
    assert abs(r["frac"] - r["achieved"] / 6544.0) < 1e-12 and abs(r["frac_of_spec"] - r["achieved"] / 8000.0) < 1e-12
    assert r["traffic"] is not None
    pre = wl.SHAPES["prefill"]
    r = bench.ffn_roofline(pre, "prefill", touched=512, flops=5.62e11, ffn_ms=0.8, peaks=peaks)
    assert r["bound"] == "tensor" and abs(r["achieved"] - 5.62e11 / 0.8e-3 / 1e12) < 1e-9
    assert abs(r["frac_of_spec"] - r["achieved"] / 2250.0) < 1e-12 and r["traffic"] is not None
    skew = wl.SHAPES["decode_skew"]
    r = bench.ffn_roofline(skew, "hybrid", touched=106, flops=0, ffn_ms=0.143, peaks=peaks)
    assert r["bound"] == "hbm" and r["traffic"] is not None
