"""Helpers of the GPU parity tests: device copies of generator inputs, the
tolerance of the FFN outputs, and cached workloads / oracle results."""
import functools

import numpy as np
import torch

import oracle
from mixture_experts_ffn_sort_b200 import workloads as wl

# FFN output tolerance: rel-L2 <= 5e-3 and max-abs <= 1e-2 * max|oracle| + 1e-3.
REL_L2 = 5e-3
MAX_ABS_REL = 1e-2
MAX_ABS_FLOOR = 1e-3
# Route weights: fp32 exp / sum against the fp64 oracle.
W_ATOL = 1e-6
W_RTOL = 1e-5


def assert_moe_close(got, ref, what="", chunk_rows=4096):
    """Every element of `got` (tensor or array) against the oracle's `ref`;
    large outputs are compared in row chunks (same result, bounded memory)."""
    r_all = np.asarray(ref)
    assert tuple(got.shape) == r_all.shape, (tuple(got.shape), r_all.shape)
    n = r_all.shape[0] if r_all.ndim else 1
    step = max(1, chunk_rows) if r_all.ndim >= 2 else max(n, 1)
    se = sr = 0.0
    mx = rmax = 0.0
    for i in range(0, max(n, 1), step):
        if torch.is_tensor(got):
            g = got[i:i + step].detach().double().cpu().numpy() if r_all.ndim else got.detach().double().cpu().numpy()
        else:
            g = np.asarray(got[i:i + step] if r_all.ndim else got, np.float64)
        r = np.asarray(r_all[i:i + step] if r_all.ndim else r_all, np.float64)
        assert np.all(np.isfinite(g)), "%s: non-finite output" % what
        err = g - r
        se += float(np.sum(err * err))
        sr += float(np.sum(r * r))
        if err.size:
            mx = max(mx, float(np.abs(err).max()))
            rmax = max(rmax, float(np.abs(r).max()))
    rel = np.sqrt(se / sr) if sr > 0 else np.sqrt(se)
    bound = MAX_ABS_REL * rmax + MAX_ABS_FLOOR
    assert rel <= REL_L2, "%s: rel-L2 %.3e > %.1e" % (what, rel, REL_L2)
    assert mx <= bound, "%s: max-abs %.3e > %.3e" % (what, mx, bound)
    return rel, mx


def bf16_tensor(bits: np.ndarray, device="cuda") -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(device)


def bf16_numpy(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().view(torch.int16).numpy().view(np.uint16)


def to_f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().double().cpu().numpy()


@functools.lru_cache(maxsize=2)
def workload(name: str):
    return wl.make_workload(name)


class DeviceWorkload:
    def __init__(self, w, device="cuda"):
        import mixture_experts_ffn_sort_b200 as moe
        self.w = w
        self.x = bf16_tensor(w.x, device)
        self.logits = torch.from_numpy(w.logits).to(device)
        self.zero_mask = torch.from_numpy(w.zero_mask).to(device) if w.zero_mask is not None else None
        self.routed = moe.Experts.from_host(w.routed, device)
        self.shared = moe.Experts.from_host(w.shared, device) if w.shared is not None else None


@functools.lru_cache(maxsize=1)
def device_workload(name: str):
    return DeviceWorkload(workload(name))


@functools.lru_cache(maxsize=3)
def oracle_maps(name: str):
    """Oracle route + sort of a workload (cheap at every size)."""
    w = workload(name)
    ids, wts = oracle.route(w.logits, w.shape.K, w.zero_mask)
    off, sr, inv, bad = oracle.sort(ids, w.shape.E)
    return dict(ids=ids, w=wts, offsets=off, sorted_route=sr, inv_route=inv, bad=bad)


def sample_tokens(T: int, n: int, seed: int = 0) -> np.ndarray:
    if n >= T:
        return np.arange(T, dtype=np.int32)
    rng = np.random.default_rng(seed)
    s = np.sort(rng.choice(T, size=n, replace=False)).astype(np.int32)
    s[0], s[-1] = 0, T - 1
    return np.unique(s)
