"""The row exchange of expert-parallel prefill (ep.all_to_all_rows) over a
world-size-2 gloo group on CPU: uneven blocks, an empty block, the count
exchange, and the round trip back to the senders' order."""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rows(rank, dest, n, H):
    import torch
    return torch.arange(n * H, dtype=torch.float32).view(n, H) + 1000.0 * rank + 100.0 * dest


def _rank_main(rank, world, port, q):
    import torch
    import torch.distributed as dist
    from datetime import timedelta

    from mixture_experts_ffn_sort_b200 import ep
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        H = 8
        n = [[3, 0], [2, 5]]  # rows rank s sends to rank d
        send = torch.cat([_rows(rank, d, n[rank][d], H) for d in range(world)])
        counts = torch.tensor([[n[rank][d]] for d in range(world)], dtype=torch.int32)
        recv_counts = torch.empty_like(counts)
        dist.all_to_all_single(recv_counts, counts)
        recv_rows = recv_counts.view(-1).tolist()
        assert recv_rows == [n[s][rank] for s in range(world)], recv_rows
        got = ep.all_to_all_rows(send, [n[rank][d] for d in range(world)], recv_rows)
        want = torch.cat([_rows(s, rank, n[s][rank], H) for s in range(world)])
        assert torch.equal(got, want)
        back = ep.all_to_all_rows(got * 2, recv_rows, [n[rank][d] for d in range(world)])
        assert torch.equal(back, send * 2)
        q.put((rank, "ok"))
    except Exception as e:  # reported to the parent
        q.put((rank, repr(e)))
    finally:
        dist.destroy_process_group()


def test_all_to_all_rows_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
    assert res == {0: "ok", 1: "ok"}, res
