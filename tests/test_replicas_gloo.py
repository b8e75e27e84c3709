"""The multi-GPU host path on CPU: world-size-2 process groups over gloo.

The MoE FFN path shards as independent replicas (tokens never interact), so
the only cross-rank steps are the benchmark's barrier, its max-over-ranks
timing and the rank-0-only report; these tests run them as two CPU ranks.
"""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, values, out_dir):
    import torch.distributed as dist
    from datetime import timedelta
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        r, w, local = bench.dist_env()
        dist.barrier()
        got = bench.max_over_ranks(values[rank])
        with open(os.path.join(out_dir, "rank%d.json" % rank), "w") as f:
            json.dump({"env": [r, w, local], "max": got,
                       "value": bench.job_tokens_per_s(64, w, got)}, f)
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_job_value_gloo(tmp_path):
    world, values = 2, [1.25, 3.5]
    mp.start_processes(_rank_main, args=(world, _free_port(), values, str(tmp_path)), nprocs=world,
                       join=True, start_method="spawn")
    for rank in range(world):
        d = json.load(open(tmp_path / ("rank%d.json" % rank)))
        assert d["env"] == [rank, world, rank]
        assert d["max"] == max(values)                       # every rank sees the slowest rank's time
        assert d["value"] == pytest.approx(64 * world / (max(values) * 1e-3))


def test_single_process_needs_no_group(monkeypatch):
    for k in ("RANK", "WORLD_SIZE", "LOCAL_RANK"):
        monkeypatch.delenv(k, raising=False)
    assert bench.dist_env() == (0, 1, 0)
    assert bench.max_over_ranks(2.5) == 2.5
    assert bench.job_tokens_per_s(512, 1, 2.0) == pytest.approx(256000.0)


def test_reference_arm_under_torchrun_prints_one_line():
    """torchrun with 2 ranks: rank 0 alone runs the oracle and prints; rank 1 exits 0."""
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(_free_port()), os.path.join(ROOT, "bench.py"),
           "--impl", "reference", "--workload", "tiny", "--gpus", "2", "--steps", "2", "--warmup", "1"]
    env = dict(os.environ, OMP_NUM_THREADS="1")
    p = subprocess.run(cmd, capture_output=True, text=True, timeout=300, env=env, cwd=ROOT)
    assert p.returncode == 0, p.stderr[-2000:]
    lines = [l for l in p.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, p.stdout
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["steps"] == 2 and d["warmup"] == 1
    assert d["value"] > 0 and d["e2e"]["value"] == d["value"]
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
