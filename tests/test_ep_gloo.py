"""Expert-parallel decode host path on CPU: the expert partition and the
cross-rank sum of partial outputs over a world-size-2 gloo group.

Each rank computes its partial output with the oracle restricted to its
experts (the other experts' route weights set to zero; rank 0 alone adds the
shared expert), the partials are summed by ep.reduce_partials over gloo, and
the sum must be the oracle's full layer output.
"""
import json
import os
import socket
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _problem():
    from mixture_experts_ffn_sort_b200 import workloads as wl
    T, H, I, E, K, Is = 12, 256, 128, 16, 3, 128
    rng = np.random.default_rng(21)
    x = wl.random_rows_bf16(T, H, seed=4)
    logits = rng.standard_normal((T, E)).astype(np.float32)
    return x, logits, K, wl.draw_experts(9, 4, E, I, H, threads=1), wl.draw_experts(9, 5, 1, Is, H, threads=1)


def _rank_main(rank, world, port, out_dir):
    import torch
    import torch.distributed as dist
    from datetime import timedelta

    import oracle
    from mixture_experts_ffn_sort_b200 import ep
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        oracle.set_threads(1)
        x, logits, K, routed, shared = _problem()
        E = logits.shape[1]
        b, e = ep.expert_range(E, rank, world)
        ids, w = oracle.route(logits, K)
        w_local = np.where((ids >= b) & (ids < e), w, 0.0)
        part = oracle.moe_tokens_routed(x, ids, w_local, routed, shared if rank == 0 else None)
        total = ep.reduce_partials(torch.from_numpy(part))
        with open(os.path.join(out_dir, "rank%d.json" % rank), "w") as f:
            json.dump({"range": [b, e], "out": total.numpy().tolist()}, f)
    finally:
        dist.destroy_process_group()


def test_expert_parallel_partials_sum_to_the_layer_gloo(tmp_path):
    import oracle
    world = 2
    mp.start_processes(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True,
                       start_method="spawn")
    x, logits, K, routed, shared = _problem()
    ref = oracle.moe(x, logits, K, routed, shared)["out"]
    ranges = []
    for rank in range(world):
        d = json.load(open(tmp_path / ("rank%d.json" % rank)))
        ranges.append(d["range"])
        np.testing.assert_allclose(np.array(d["out"]), ref, rtol=1e-12, atol=1e-12)
    assert ranges == [[0, 8], [8, 16]]


def test_expert_range_checks():
    from mixture_experts_ffn_sort_b200 import ep
    assert ep.expert_range(256, 0, 8) == (0, 32)
    assert ep.expert_range(256, 7, 8) == (224, 256)
    for bad in ((20, 0, 8), (256, 8, 8), (256, -1, 8), (256, 0, 0)):
        with pytest.raises(ValueError):
            ep.expert_range(*bad)
