"""Benchmark of the routed MoE FFN hot path on B200.

One step = one pass of the whole path over one batch: moe_route -> moe_sort ->
moe_expert_ffn -> moe_combine, replayed from a CUDA graph.  The default
workload is the decode MoE (T=64 tokens, H=2048, I=512, 256 experts, top-8,
FP8 E4M3 weights with 128x128 block scales, bf16 activations).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload decode|tiny|decode_skew|prefill|prefill_large]

Prints one JSON line (rank 0).  With N > 1 (torchrun), every rank runs an
independent replica of the workload (the path has no cross-token exchange);
the time is the max over ranks and the value counts all ranks' tokens.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from mixture_experts_ffn_sort_b200 import workloads as wl  # noqa: E402

METRIC = "MoE FFN tokens/s at 1 B200; % HBM roofline (decode) / % BF16 TC peak (prefill)"
UNIT = "tokens/s"
# Bytes of one expert's FP8 weights and fp32 block scales, used for the decode roofline.


# Nominal B200 figures, reported beside the measured-peak fractions: HBM3e
# bandwidth and dense bf16 tensor-core throughput.
SPEC_HBM_GBS = 8000.0
SPEC_BF16_TFLOPS = 2250.0


def expert_bytes(H, I):
    return 3 * H * I + 3 * (H // 128) * (I // 128) * 4


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return dict(hbm=d["hbm_gbs"], bf16=d["bf16_tflops"], bf16_sus=d["bf16_tflops_sustained"],
                    src="measured")
    return dict(hbm=6650.0, bf16=1590.0, bf16_sus=1400.0, src="fallback")


def profile_traffic(workload, kind, root=ROOT):
    """DRAM bytes per FFN call from the committed ncu summary of this workload,
    if the kernel sources it was taken on are unchanged (else None)."""
    path = os.path.join(root, "profiles", "ffn_%s_%s.md" % (kind, workload))
    if not os.path.exists(path):
        return None
    text = open(path).read()
    m = re.search(r"traffic_bytes_per_call:\s*([0-9.eE+]+)", text)
    h = re.search(r"sources_sha256:\s*([0-9a-f]+)", text)
    if not m or not h or h.group(1) != sources_hash(kind):
        return None
    return float(m.group(1))


FFN_SOURCES = {"decode": ("ffn_decode.cu", "device_common.cuh", "launch.h"),
               "w8a8": ("ffn_decode.cu", "device_common.cuh", "launch.h"),
               "prefill": ("ffn_prefill.cu", "device_common.cuh", "launch.h"),
               "hybrid": ("ffn_decode.cu", "ffn_prefill.cu", "device_common.cuh", "launch.h")}


def sources_hash(kind="decode"):
    """Hash of the code of the FFN kernels a profile summary was taken on
    (comments and layout left out, so editing a comment keeps the summary)."""
    d = os.path.join(ROOT, "mixture_experts_ffn_sort_b200", "csrc")
    hs = hashlib.sha256()
    for f in FFN_SOURCES[kind]:
        path = os.path.join(d, f)
        if os.path.exists(path):
            text = open(path).read()
            text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
            text = re.sub(r"//[^\n]*", " ", text)
            hs.update(" ".join(text.split()).encode())
    return hs.hexdigest()[:16]


class ClockSampler:
    """SM clock, power and clock-event (throttle) reasons of one GPU, sampled
    every 5 ms by a thread through NVML (read-only queries; nvidia-smi every
    50 ms if NVML is unavailable).  Samples are time-stamped, so each timed
    region gets its own summary."""

    NAMES = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
    Q = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
         "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
         "clocks_event_reasons.sw_power_cap")

    def __init__(self, index, pci_bus_id=None, period_s=0.005):
        self.index, self.pci, self.period = index, pci_bus_id, period_s
        self.samples = []  # (time, sm MHz, max MHz, power W, {reason names})
        self.proc, self.stop, self.source = None, threading.Event(), None

    def __enter__(self):
        try:
            import pynvml
            pynvml.nvmlInit()
            try:
                h = pynvml.nvmlDeviceGetHandleByPciBusId(self.pci) if self.pci else None
            except pynvml.NVMLError:
                h = None
            if h is None:
                h = pynvml.nvmlDeviceGetHandleByIndex(self.index)
            self.nvml, self.h = pynvml, h
            bits = (pynvml.nvmlClocksEventReasonHwSlowdown, pynvml.nvmlClocksEventReasonHwThermalSlowdown,
                    pynvml.nvmlClocksEventReasonSwThermalSlowdown, pynvml.nvmlClocksEventReasonSwPowerCap)
            self.bits = list(zip(self.NAMES, bits))
            self.source = "nvml, %.0f ms" % (self.period * 1e3)
            self.t = threading.Thread(target=self._nvml_loop, daemon=True)
            self.t.start()
            return self
        except Exception:
            pass
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.index), "--query-gpu=" + self.Q,
                                          "--format=csv,noheader,nounits", "-lms", "50"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.source = "nvidia-smi, 50 ms"
            self.t = threading.Thread(target=self._smi_loop, daemon=True)
            self.t.start()
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def _nvml_loop(self):
        n = self.nvml
        mx = n.nvmlDeviceGetMaxClockInfo(self.h, n.NVML_CLOCK_SM)
        while not self.stop.is_set():
            try:
                sm = n.nvmlDeviceGetClockInfo(self.h, n.NVML_CLOCK_SM)
                pw = n.nvmlDeviceGetPowerUsage(self.h) / 1000.0
                r = n.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                self.samples.append((time.monotonic(), float(sm), float(mx), pw,
                                     {name for name, b in self.bits if r & b}))
            except Exception:
                pass
            time.sleep(self.period)

    def _smi_loop(self):
        for line in self.proc.stdout:
            f = [x.strip() for x in line.strip().split(",")]
            if len(f) < 8:
                continue
            try:
                self.samples.append((time.monotonic(), float(f[0]), float(f[1]), float(f[2]),
                                     {n for n, v in zip(self.NAMES, f[4:8]) if v.lower().startswith("active")}))
            except ValueError:
                continue

    def wait_first(self, timeout_s=3.0):
        t0 = time.monotonic()
        while not self.samples and time.monotonic() - t0 < timeout_s and self.source:
            time.sleep(0.01)

    def __exit__(self, *a):
        self.stop.set()
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self, t0=None, t1=None):
        """Median SM clock, max clock and throttle reasons of the samples taken
        in [t0, t1] (all samples when no interval is given)."""
        sm, mx, pw, reasons = [], [], [], set()
        for ts, c, m, p, rs in list(self.samples):
            if (t0 is not None and ts < t0) or (t1 is not None and ts > t1):
                continue
            sm.append(c)
            mx.append(m)
            pw.append(p)
            reasons |= rs
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0, "source": self.source}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "power_w_max": max(pw),
                "reasons": sorted(reasons), "samples": len(sm), "source": self.source}


def ffn_roofline(shape, form_kind, touched, flops, ffn_ms, peaks, root=ROOT, profile_kind=None):
    """The roofline object of the FFN call: touched-expert bytes against HBM
    for the weight-streaming and hybrid forms (form_kind "decode" / "hybrid"),
    bf16 FLOPs against the tensor cores for the prefill form.  The FFN time is
    a median of single synchronised replays, a kernel timed on its own, so
    the tensor-core fraction is against the burst bf16 peak (the sustained
    one, for a kernel inside a seconds-long loop, is reported beside it)."""
    H, I = shape.H, shape.I
    if form_kind in ("decode", "hybrid"):
        algo = touched * expert_bytes(H, I) + (expert_bytes(H, shape.I_shared) if shape.I_shared else 0)
        ach = algo / (ffn_ms * 1e-3) / 1e9
        return {"bound": "hbm", "achieved": ach, "peak": peaks["hbm"], "unit": "GB/s",
                "frac": ach / peaks["hbm"], "traffic": profile_traffic(shape.name, profile_kind or form_kind, root),
                "kernel": "moe_expert_ffn (gate/up + down kernels)", "algorithmic_bytes": algo,
                "touched_experts": touched, "peak_source": peaks["src"] + " copy bandwidth",
                "spec_peak": SPEC_HBM_GBS, "frac_of_spec": ach / SPEC_HBM_GBS}
    ach = flops / (ffn_ms * 1e-3) / 1e12
    pk = peaks["bf16"]
    return {"bound": "tensor", "achieved": ach, "peak": pk, "unit": "TFLOP/s", "frac": ach / pk,
            "traffic": profile_traffic(shape.name, "prefill", root), "kernel": "moe_expert_ffn", "flops": flops,
            "peak_source": peaks["src"] + " burst bf16",
            "peak_sustained": peaks["bf16_sus"], "frac_of_sustained": ach / peaks["bf16_sus"],
            "spec_peak": SPEC_BF16_TFLOPS, "frac_of_spec": ach / SPEC_BF16_TFLOPS}


# The arithmetic each FFN form computes in ("dtype" of the line and its description).
ARITHMETIC = {
    "decode": ("f16", "E4M3 weights taken exactly as f16 MMA operands, activations as f16 after an exact "
                      "power-of-two row scale, fp32 accumulate, fp32 block scale per 128-column partial; "
                      "bf16 h, y_sorted and out"),
    "prefill": ("f16+bf16", "gate/up: f16 MMA on f16(e4m3 x block scale x 2^ka) and f16(x x 2^k_t), power-of-two "
                            "row scales undone in the epilogue; down: bf16 MMA on bf16(e4m3 x block scale) and bf16 "
                            "h; fp32 accumulate in TMEM; bf16 h, y_sorted and out"),
    "w8a8": ("e4m3", "E4M3FN weights and E4M3FN activations (x in 128-column, h in 64-feature blocks with "
                     "power-of-two scales) in m16n8k32 MMAs, fp32 accumulate, fp32 weight and activation block "
                     "scales per partial sum; bf16 y_sorted and out"),
    "hybrid": ("f16+bf16", "experts with few rows as the decode form (f16 MMA on exact E4M3), the others as the "
                           "prefill form (f16 gate/up, bf16 down); fp32 accumulate; bf16 h, y_sorted and out"),
}


# ---------------------------------------------------------------- reference arm (CPU oracle)

def oracle_route_kwargs(router, shape):
    """The oracle's route_ex arguments for a router preset (None: plain router)."""
    cfg = wl.ROUTERS[router]
    if cfg is None:
        return None
    kw = {k: v for k, v in cfg.items() if k != "bias"}
    kw["bias"] = wl.selection_bias(shape.E, shape.seed) if cfg.get("bias") else None
    return kw


def oracle_rows(w, shape, tk, router, fused_router=False):
    """Brute-force oracle rows of the sampled tokens tk, routed by `router`
    (fused_router: the logits are the router's gate GEMM of x, computed here)."""
    import oracle
    kw = oracle_route_kwargs(router, shape)
    if kw is None and not fused_router:
        return oracle.moe_tokens(w.x, w.logits, shape.K, w.routed, w.shared, w.zero_mask, tokens=tk)
    zm = None if w.zero_mask is None else w.zero_mask[tk]
    if fused_router:
        lg = oracle.router_logits(w.x[tk], wl.router_weight(shape.E, shape.H, shape.seed)).astype(np.float32)
    else:
        lg = w.logits[tk]
    ids, wt = oracle.route_ex(lg, shape.K, zero_mask=zm, **(kw or {}))
    return oracle.moe_tokens_routed(w.x, ids, wt, w.routed, w.shared, tokens=tk)


def run_reference(args, shape):
    import oracle
    w = wl.make_workload(shape.name)
    cores = oracle.threads()
    tk = np.arange(min(shape.T, 64 if shape.T > 512 else shape.T), dtype=np.int32)

    def one():
        t0 = time.perf_counter()
        oracle_rows(w, shape, tk, args.router, args.fused_router)
        return time.perf_counter() - t0

    for _ in range(args.warmup):
        one()
    ts = [one() for _ in range(args.steps)]
    tot = sum(ts)
    value = len(tk) * len(ts) / tot
    sample = "%d of the %d tokens per step (brute-force per-token oracle, fp64)" % (len(tk), shape.T)
    return {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": 1e3 * tot / len(ts), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "impl": "reference", "config": config_of(shape, args.router, args.fused_router),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def cpu_baseline(shape, router="softmax", fused_router=False, budget_s=10.0):
    """The oracle as it stands, on the host cores, on a bounded sample."""
    import oracle
    w = wl.make_workload(shape.name)
    tk = np.arange(min(shape.T, 64), dtype=np.int32)
    n, t0 = 0, time.perf_counter()
    while time.perf_counter() - t0 < budget_s or n == 0:
        oracle_rows(w, shape, tk, router, fused_router)
        n += 1
    dt = time.perf_counter() - t0
    return {"value": n * len(tk) / dt, "unit": UNIT, "cores": oracle.threads(), "kind": "oracle",
            "sample": "%d x %d tokens of the workload, %.1f s, brute-force per-token oracle in fp64"
                      % (n, len(tk), dt)}


# ---------------------------------------------------------------- replicas

def dist_env():
    """(rank, world size, local rank) from the torchrun environment (1 process: 0, 1, 0)."""
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def max_over_ranks(v, device="cpu"):
    """Largest v over all ranks of the process group (v itself without one)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(v)
    t = torch.tensor([float(v)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.item()


def job_tokens_per_s(T, world, ms_per_step):
    """Whole-job throughput: every replica processes T tokens per step."""
    return T * world / (ms_per_step * 1e-3)


def config_of(shape, router="softmax", fused_router=False):
    c = {"workload": shape.name, "T": shape.T, "H": shape.H, "I": shape.I, "E": shape.E, "K": shape.K,
         "I_shared": shape.I_shared, "weights": "fp8 e4m3fn, fp32 scale per 128x128 block",
         "activations": "bf16", "logit_bias": shape.bias, "zero_route_frac": shape.zero_frac,
         "seed": shape.seed, "router": router}
    if wl.ROUTERS[router] is not None:
        c["router_cfg"] = {k: v for k, v in wl.ROUTERS[router].items() if k != "bias"}
        c["router_cfg"]["selection_bias"] = "N(0, 0.02) per expert" if wl.ROUTERS[router].get("bias") else None
    c["logits"] = ("x . W_r^T on the device (moe_router: gate GEMM fused with the routing; W_r bf16 "
                   "[E, H] ~ N(0, 1/H))" if fused_router else "given, f32 [T, E]")
    if fused_router:
        c["logit_bias"] = None  # the router computes the logits; no drawn bias is added
    return c


# ---------------------------------------------------------------- our arm

# Windows of `steps` replays timed one by one; the step time is their median.
N_WINDOWS = 7
# Workloads timed after the headline one with the same protocol (the line's
# "workloads" object): the skewed high-batch decode and both prefills.
EXTRA_WORKLOADS = ("decode_skew", "prefill", "prefill_large")
DEFAULT_STEPS = {"tiny": 500, "decode": 500, "decode_skew": 200, "prefill": 30, "prefill_large": 10}


class Eager:
    """Stands in for a CUDA graph: replay() launches every call directly."""

    def __init__(self, fn):
        self.fn = fn

    def replay(self):
        self.fn()


def measure(args, shape, steps, dev, world, clk, want_e2e):
    """One workload: build the layer, capture a step in a CUDA graph, warm up,
    time N_WINDOWS windows of `steps` replays (barrier and synchronize around
    each, max over ranks), then the per-call breakdown from an instrumented
    graph.  Returns the workload's record, plus the end-to-end measurement
    through the public API when want_e2e."""
    import torch
    import torch.distributed as dist
    import mixture_experts_ffn_sort_b200 as moe

    w = wl.make_workload(shape.name)
    T, K, E, H, I = shape.T, shape.K, shape.E, shape.H, shape.I
    x = torch.from_numpy(w.x.view(np.int16)).view(torch.bfloat16).to(dev)
    logits = torch.from_numpy(w.logits).to(dev)
    zmask = torch.from_numpy(w.zero_mask).to(dev) if w.zero_mask is not None else None
    routed = moe.Experts.from_host(w.routed, dev)
    shared = moe.Experts.from_host(w.shared, dev) if w.shared is not None else None
    route_cfg = None
    kw = wl.ROUTERS[args.router]
    if kw is not None:
        route_cfg = {k: v for k, v in kw.items() if k != "bias"}
        route_cfg["sel_bias"] = (torch.from_numpy(wl.selection_bias(E, shape.seed)).to(dev)
                                 if kw.get("bias") else None)
    wr = (torch.from_numpy(wl.router_weight(E, H, shape.seed).view(np.int16)).view(torch.bfloat16).to(dev)
          if args.fused_router else None)
    layer = moe.MoEFFN(routed, T, K, shared, mode=args.mode, device=dev, route_cfg=route_cfg, w_router=wr,
                       fused_combine=args.fused_combine, w8a8=args.w8a8)
    stream = torch.cuda.Stream(device=dev)

    def run(lay, xx, ll):
        if args.fused_router:
            lay.forward_fused(xx, zmask)
        else:
            lay(xx, ll, zmask)

    def step():
        run(layer, x, logits)

    def barrier():
        if world > 1:
            dist.barrier()

    with torch.cuda.stream(stream):
        step()  # first call outside any capture (one-time set-up)
    stream.synchronize()

    def instrumented():
        ev[0].record()
        if args.fused_router:
            moe.moe_router(x, wr, K, zero_mask=zmask, topk_ids=layer.topk_ids, topk_w=layer.topk_w,
                           **(route_cfg or {}))
        elif route_cfg is None:
            moe.moe_route(logits, K, zmask, layer.topk_ids, layer.topk_w)
        else:
            moe.moe_route_ex(logits, K, zero_mask=zmask, topk_ids=layer.topk_ids, topk_w=layer.topk_w,
                             **route_cfg)
        ev[1].record()
        moe.moe_sort(layer.topk_ids, E, layer.status, layer.offsets, layer.sorted_route, layer.inv_route,
                     layer.sort_ws)
        ev[2].record()
        if args.fused_combine:
            moe.moe_expert_ffn_combine(x, K, routed, layer.offsets, layer.sorted_route, layer.topk_w, shared,
                                       moe.MOE_OUT_BF16, layer.status, layer.out, layer.ffn_ws)
            ev[3].record()
        else:
            if args.w8a8:
                moe.moe_expert_ffn_w8a8(x, K, routed, layer.offsets, layer.sorted_route, layer.topk_w, shared,
                                        layer.status, layer.y_sorted, layer.y_shared, layer.ffn_ws)
            else:
                moe.moe_expert_ffn(x, K, routed, layer.offsets, layer.sorted_route, layer.topk_w, shared,
                                   args.mode, layer.status, layer.y_sorted, layer.y_shared, layer.ffn_ws)
            ev[3].record()
            moe.moe_combine(layer.y_sorted, layer.inv_route, layer.y_shared, T, K, moe.MOE_OUT_BF16, layer.out,
                            status=layer.status)
        ev[4].record()

    # Graph of one step; the timed windows replay it.  A second graph records
    # events around each call, for the per-call breakdown.
    ev = [torch.cuda.Event(enable_timing=True, external=not args.eager) for _ in range(5)]
    if args.eager:
        g, g2 = Eager(step), Eager(instrumented)
    else:
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            step()
        g2 = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g2, stream=stream):
            instrumented()
    t_warm = time.monotonic()
    with torch.cuda.stream(stream):
        for _ in range(max(3, args.warmup)):
            g.replay()
        g2.replay()
    stream.synchronize()
    if layer.status.item() != 0:
        raise RuntimeError("%s: status word %d after warm-up" % (shape.name, layer.status.item()))

    windows = []
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t_timed = time.monotonic()
    for _ in range(N_WINDOWS):
        barrier()
        torch.cuda.synchronize(dev)
        start.record(stream)
        with torch.cuda.stream(stream):
            for _ in range(steps):
                g.replay()
        end.record(stream)
        torch.cuda.synchronize(dev)
        barrier()
        windows.append(start.elapsed_time(end) / steps)
    t_done = time.monotonic()
    t_local = statistics.median(windows)
    # Per-call breakdown from the instrumented graph (same stream, after the timed windows).
    parts = {k: [] for k in ("route", "sort", "ffn", "combine")}
    with torch.cuda.stream(stream):
        for _ in range(min(max(steps, 20), 200)):
            g2.replay()
            stream.synchronize()
            for i, k in enumerate(parts):
                parts[k].append(ev[i].elapsed_time(ev[i + 1]))
    t_max = max_over_ranks(t_local, dev)
    if layer.status.item() != 0:
        raise RuntimeError("%s: status word %d after the timed windows" % (shape.name, layer.status.item()))

    peaks = load_peaks()
    off = layer.offsets.cpu().numpy()
    touched = int(np.count_nonzero(np.diff(off)))
    ffn_ms = statistics.median(parts["ffn"])
    R_nz = int(np.count_nonzero(layer.topk_w.cpu().numpy()))
    flops = (R_nz + (T if shape.I_shared else 0)) * 6 * H * I
    form = (moe.MOE_MODE_PREFILL if args.fused_combine else
            moe.MOE_MODE_DECODE if args.w8a8 else moe.moe_ffn_resolve_mode(T, K, E, args.mode))
    form_kind = {moe.MOE_MODE_DECODE: "decode", moe.MOE_MODE_PREFILL: "prefill",
                 moe.MOE_MODE_HYBRID: "hybrid"}[form]
    roof = ffn_roofline(shape, form_kind, touched=touched, flops=flops, ffn_ms=ffn_ms, peaks=peaks,
                        profile_kind="w8a8" if args.w8a8 else None)
    if form_kind == "hybrid":
        # The tensor-core share of the same call, for reference.
        roof["flops"] = flops
        roof["tflops"] = flops / (ffn_ms * 1e-3) / 1e12
    if args.fused_router:
        # The fused router's own roofline: a bf16 GEMM of 2 T H E flops (its
        # top-K epilogue adds no HBM traffic beyond the ids and weights).
        r_ms = statistics.median(parts["route"])
        r_flops = 2.0 * T * H * E
        r_ach = r_flops / (r_ms * 1e-3) / 1e12
        roof["router"] = {"kernel": "moe_router (gate GEMM + top-K)", "bound": "tensor", "flops": r_flops,
                          "achieved": r_ach, "peak": peaks["bf16"], "unit": "TFLOP/s",
                          "frac": r_ach / peaks["bf16"]}
    weights_gb = (touched if form_kind != "prefill" else E) * expert_bytes(H, I) / 1e9
    rec = {"workload": shape.name, "value": job_tokens_per_s(T, world, t_max), "unit": UNIT,
           "ms_per_step": t_max, "steps": steps, "windows": N_WINDOWS,
           "window_ms_per_step": {"min": min(windows), "median": t_local, "max": max(windows)},
           "spread": (max(windows) - min(windows)) / t_local,
           "form": form_kind + ("+combine (moe_expert_ffn_combine: fp32 reductions, unordered)"
                                if args.fused_combine else " W8A8 (moe_expert_ffn_w8a8)" if args.w8a8 else ""),
           "dtype": ARITHMETIC["w8a8" if args.w8a8 else form_kind][0],
           "arithmetic": ARITHMETIC["w8a8" if args.w8a8 else form_kind][1],
           "l2": "inputs larger than L2 (%s expert weights %.2f GB > 126 MB)"
                 % ("touched" if form_kind != "prefill" else "all", weights_gb),
           "roofline": roof, "breakdown_ms": {k: statistics.median(v) for k, v in parts.items()},
           "gpu_launches": layer.launches() * steps * N_WINDOWS,
           "clocks": clk.summary(t_timed, t_done) if clk.summary(t_timed, t_done)["samples"]
           else dict(clk.summary(t_warm, time.monotonic()), note="no sample inside the timed windows; "
                     "samples from warm-up to the breakdown")}
    e2e = None
    if want_e2e:
        e2e = measure_e2e(args, w, shape, layer, routed, shared, route_cfg, wr, x, logits, run, dev, world, stream)
    del g, g2
    return rec, e2e


def measure_e2e(args, w, shape, layer, routed, shared, route_cfg, wr, x, logits, run, dev, world, stream):
    """End to end through the public API with host buffers: every step copies
    its x and logits in from pinned host memory and its output back out.  Two
    sets of device buffers (a second layer object over the same weights) let
    step i+1's input copy and step i-1's output copy overlap step i's compute:
    copy-in, compute and copy-out streams ordered by events."""
    import torch
    import mixture_experts_ffn_sort_b200 as moe
    T, K, H = shape.T, shape.K, shape.H
    xh = torch.from_numpy(w.x.view(np.int16)).view(torch.bfloat16).pin_memory()
    lh = torch.from_numpy(w.logits).pin_memory()
    oh = [torch.empty((T, H), dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    layers = [layer, moe.MoEFFN(routed, T, K, shared, mode=args.mode, device=dev, route_cfg=route_cfg,
                                w_router=wr, fused_combine=args.fused_combine, w8a8=args.w8a8)]
    xs, ls = [x, torch.empty_like(x)], [logits, torch.empty_like(logits)]
    h2d, d2h = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    in_ready, in_free, out_ready, out_free = ([torch.cuda.Event(), torch.cuda.Event()] for _ in range(4))
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    n_e2e = min(args.steps * N_WINDOWS, 500)
    with torch.cuda.stream(stream):
        xs[1].copy_(xh)
        ls[1].copy_(lh)
        run(layers[1], xs[1], ls[1])  # first call of the second layer outside the timed region
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    torch.cuda.synchronize(dev)
    e0.record(stream)
    h2d.wait_event(e0)
    for i in range(n_e2e):
        b = i % 2
        with torch.cuda.stream(h2d):
            if i >= 2:
                h2d.wait_event(in_free[b])
            xs[b].copy_(xh, non_blocking=True)
            if not args.fused_router:  # the fused router computes the logits from x
                ls[b].copy_(lh, non_blocking=True)
            in_ready[b].record(h2d)
        with torch.cuda.stream(stream):
            stream.wait_event(in_ready[b])
            if i >= 2:
                stream.wait_event(out_free[b])
            run(layers[b], xs[b], ls[b])
            in_free[b].record(stream)
            out_ready[b].record(stream)
        with torch.cuda.stream(d2h):
            d2h.wait_event(out_ready[b])
            oh[b].copy_(layers[b].out, non_blocking=True)
            out_free[b].record(d2h)
    stream.wait_stream(d2h)
    stream.wait_stream(h2d)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / n_e2e, dev)
    for lay in layers:
        if lay.status.item() != 0:
            raise RuntimeError("status word %d after the end-to-end run" % lay.status.item())
    return {"value": job_tokens_per_s(T, world, e2e_ms), "unit": UNIT,
            "h2d_bytes_per_step": x.numel() * 2 + (0 if args.fused_router else logits.numel() * 4),
            "d2h_bytes_per_step": layer.out.numel() * 2, "steps": n_e2e}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None, help="replays per timed window (7 windows)")
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="decode", choices=wl.SHAPE_ORDER)
    ap.add_argument("--extra-workloads", default=",".join(EXTRA_WORKLOADS),
                    help="comma-separated workloads timed after the headline one (\"none\" for none)")
    ap.add_argument("--mode", type=int, default=0, help="moe_expert_ffn mode: 0 AUTO, 1 DECODE, 2 PREFILL, 3 HYBRID")
    ap.add_argument("--router", default="softmax", choices=sorted(wl.ROUTERS),
                    help="routing variant: softmax top-k (moe_route) or a moe_route_ex preset")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--fused-router", action="store_true",
                    help="route from x with the fused router (gate GEMM + top-K) instead of given logits")
    ap.add_argument("--eager", action="store_true",
                    help="launch every call directly instead of replaying CUDA graphs (for profilers)")
    ap.add_argument("--w8a8", action="store_true",
                    help="FP8 activations (moe_expert_ffn_w8a8, the opt-in W8A8 form) instead of moe_expert_ffn")
    ap.add_argument("--fused-combine", action="store_true",
                    help="expert FFN and combine in one call (moe_expert_ffn_combine; tensor-core form)")
    args = ap.parse_args()
    shape = wl.SHAPES[args.workload]
    rank, world, local = dist_env()

    if args.impl == "reference":
        if args.steps is None:
            args.steps = 3
        if rank == 0:
            print(json.dumps(run_reference(args, shape)), flush=True)
        return

    import torch
    import torch.distributed as dist

    extras = [n for n in args.extra_workloads.split(",") if n and n != "none" and n != shape.name]
    for n in extras:
        if n not in wl.SHAPES:
            raise SystemExit("unknown workload %r" % n)
    steps_given = args.steps is not None
    if not steps_given:
        args.steps = DEFAULT_STEPS[shape.name]
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)

    props = torch.cuda.get_device_properties(dev)
    pci = ("%08x:%02x:%02x.0" % (props.pci_domain_id, props.pci_bus_id, props.pci_device_id)
           if hasattr(props, "pci_bus_id") else None)
    with ClockSampler(local, pci) as clk:
        clk.wait_first()
        head, e2e = measure(args, shape, args.steps, dev, world, clk, want_e2e=True)
        others = {}
        for n in extras:
            torch.cuda.empty_cache()
            rec, _ = measure(args, wl.SHAPES[n], args.steps if steps_given else DEFAULT_STEPS[n], dev, world, clk,
                             want_e2e=False)
            others[n] = rec
    out = {"metric": METRIC, "value": head["value"], "unit": UNIT, "n_gpus": world,
           "steps": args.steps, "warmup": args.warmup, "ms_per_step": head["ms_per_step"],
           "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": head["dtype"],
           "data": "synthetic",
           "config": config_of(shape, args.router, args.fused_router),
           "parallelism": "replicas x%d" % world, "l2": head["l2"],
           "timing": "median of %d windows of %d %s of one step (CUDA events on the launching stream, "
                     "barrier and synchronize around each window, max over ranks)"
                     % (N_WINDOWS, args.steps, "eager launches" if args.eager else "CUDA-graph replays"),
           "window_ms_per_step": head["window_ms_per_step"], "spread": head["spread"],
           "arithmetic": head["arithmetic"], "form": head["form"],
           "roofline": head["roofline"], "breakdown_ms": head["breakdown_ms"],
           "e2e": e2e, "gpu_launches": head["gpu_launches"], "clocks": head["clocks"],
           "workloads": others}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline(shape, args.router, args.fused_router)
    if rank == 0:
        print(json.dumps(out), flush=True)
    if world > 1:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
