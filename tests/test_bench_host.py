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
