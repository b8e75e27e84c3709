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


def test_ffn_roofline_objects(tmp_path):
    """The FFN roofline: touched-expert bytes over HBM for the weight-streaming
    and hybrid forms, bf16 FLOPs over the burst tensor-core peak for the
    prefill form (its FFN time is a synchronised single replay), with the DRAM
    traffic of an ncu summary only while the FFN kernels' sources still match
    the hash recorded in it."""
    peaks = {"hbm": 6544.0, "bf16": 1657.0, "bf16_sus": 1388.3, "src": "test"}
    prof = tmp_path / "profiles"
    prof.mkdir()
    for kind, name in (("decode", "decode"), ("prefill", "prefill"), ("hybrid", "decode_skew")):
        (prof / ("ffn_%s_%s.md" % (kind, name))).write_text(
            "traffic_bytes_per_call: 1.5e9\nsources_sha256: %s\n" % bench.sources_hash(kind))
    dec = wl.SHAPES["decode"]
    r = bench.ffn_roofline(dec, "decode", touched=222, flops=0, ffn_ms=0.119, peaks=peaks, root=str(tmp_path))
    algo = 222 * bench.expert_bytes(dec.H, dec.I)
    assert r["bound"] == "hbm" and r["algorithmic_bytes"] == algo
    assert abs(r["achieved"] - algo / 0.119e-3 / 1e9) < 1e-6 * r["achieved"]
    assert abs(r["frac"] - r["achieved"] / 6544.0) < 1e-12 and abs(r["frac_of_spec"] - r["achieved"] / 8000.0) < 1e-12
    assert r["traffic"] == 1.5e9
    pre = wl.SHAPES["prefill"]
    r = bench.ffn_roofline(pre, "prefill", touched=512, flops=5.62e11, ffn_ms=0.8, peaks=peaks, root=str(tmp_path))
    assert r["bound"] == "tensor" and abs(r["achieved"] - 5.62e11 / 0.8e-3 / 1e12) < 1e-9
    assert r["peak"] == 1657.0 and abs(r["frac"] - r["achieved"] / 1657.0) < 1e-12
    assert abs(r["frac_of_sustained"] - r["achieved"] / 1388.3) < 1e-12
    assert abs(r["frac_of_spec"] - r["achieved"] / 2250.0) < 1e-12 and r["traffic"] == 1.5e9
    skew = wl.SHAPES["decode_skew"]
    r = bench.ffn_roofline(skew, "hybrid", touched=106, flops=0, ffn_ms=0.143, peaks=peaks, root=str(tmp_path))
    assert r["bound"] == "hbm" and r["traffic"] == 1.5e9
    # The W8A8 form reads its own summary (same workload, profile kind "w8a8").
    (prof / "ffn_w8a8_decode.md").write_text("traffic_bytes_per_call: 7.0e8\nsources_sha256: %s\n"
                                              % bench.sources_hash("w8a8"))
    r = bench.ffn_roofline(dec, "decode", touched=222, flops=0, ffn_ms=0.123, peaks=peaks, root=str(tmp_path),
                           profile_kind="w8a8")
    assert r["bound"] == "hbm" and r["traffic"] == 7.0e8
    # A summary taken on other kernel sources gives no traffic.
    (prof / "ffn_decode_decode.md").write_text("traffic_bytes_per_call: 1.5e9\nsources_sha256: 0123abcd\n")
    r = bench.ffn_roofline(dec, "decode", touched=222, flops=0, ffn_ms=0.119, peaks=peaks, root=str(tmp_path))
    assert r["traffic"] is None


def test_reference_and_our_arm_share_the_config():
    """Both arms report the same config object (run settings live outside it)."""
    shape = wl.SHAPES["decode"]
    line = bench.run_reference(type("A", (), dict(steps=1, warmup=0, gpus=1, router="softmax",
                                                   fused_router=False))(), wl.SHAPES["tiny"])
    assert line["config"] == bench.config_of(wl.SHAPES["tiny"])
    assert set(bench.config_of(shape)) >= {"workload", "T", "H", "I", "E", "K"}
    assert not {"parallelism", "l2", "timing"} & set(bench.config_of(shape))
