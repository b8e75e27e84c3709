"""Expert-parallel prefill's host path end to end over a world-size-2 gloo
group on CPU: ep.ExpertParallelPrefill.forward with its real exchanges
(counts, rows, weights, results: all_to_all_single over gloo) and the
library's four calls replaced by stand-ins built on the oracle (route, sort,
per-row expert FFN, combine; x travels as its bf16 bit patterns).  Every
rank's output must equal the oracle's whole layer on that rank's tokens, so
the dispatch metadata, the split sizes, the order of the returned rows and the
final inverse-map combine are all checked."""
import os
import socket
import sys

import numpy as np
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

H, I, E, K, IS = 256, 128, 16, 3, 128
TS = [23, 17]


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _inputs(rank):
    from mixture_experts_ffn_sort_b200 import workloads as wl
    T = TS[rank]
    x = wl.random_rows_bf16(T, H, seed=60 + rank)
    lg = np.random.default_rng(70 + rank).standard_normal((T, E)).astype(np.float32)
    zm = (np.random.default_rng(80 + rank).random((T, K)) < 0.1).astype(np.uint8)
    return x, lg, zm


def _stand_ins():
    """CPU stand-ins of the library calls ep uses, on the oracle."""
    import torch

    import oracle

    def route(logits, K, zero_mask, ids, w, stream=None):
        oid, ow = oracle.route(logits.numpy(), K, None if zero_mask is None else zero_mask.numpy())
        ids.copy_(torch.from_numpy(oid))
        w.copy_(torch.from_numpy(ow.astype(np.float32)))
        return ids, w

    def sort(ids, E, status, offsets, sorted_route, inv_route, workspace, stream=None):
        off, sr, inv, _ = oracle.sort(ids.numpy(), E)
        offsets.copy_(torch.from_numpy(off))
        sorted_route.copy_(torch.from_numpy(sr))
        inv_route.copy_(torch.from_numpy(inv))
        return offsets, sorted_route, inv_route

    def combine(y_sorted, inv_route, y_shared, T, K, out_dtype=0, out=None, stream=None):
        if y_sorted.dtype == torch.int32:  # a row gather of bf16 bit patterns (K = 1)
            assert K == 1 and y_shared is None
            return y_sorted[inv_route.long()]
        sh = None if y_shared is None else y_shared.numpy()
        return torch.from_numpy(oracle.combine(y_sorted.double().numpy(), inv_route.numpy(), sh, T, K))

    def expert_ffn(x, K, routed, offsets, sorted_route, topk_w, shared=None, mode=0, status=None,
                   y_sorted=None, y_shared=None, workspace=None, stream=None):
        xb = x.numpy().astype(np.uint16)
        y = oracle.ffn_sorted(xb, K, routed, offsets.numpy(), sorted_route.numpy(), topk_w.double().numpy())
        ys = oracle.ffn_shared(xb, shared) if shared is not None else None
        return torch.from_numpy(y), (torch.from_numpy(ys) if ys is not None else None)

    return route, sort, combine, expert_ffn


def _rank_main(rank, world, port, q):
    import torch
    import torch.distributed as dist
    from datetime import timedelta

    import mixture_experts_ffn_sort_b200 as moe
    import oracle
    from mixture_experts_ffn_sort_b200 import ep
    from mixture_experts_ffn_sort_b200 import workloads as wl
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        oracle.set_threads(1)
        ep.moe_route, ep.moe_sort, ep.moe_combine, ep.moe_expert_ffn = _stand_ins()
        routed = wl.draw_experts(13, 4, E, I, H, threads=1)
        shared = wl.draw_experts(13, 5, 1, IS, H, threads=1)
        full = moe.Experts(routed.w_gate, routed.s_gate, routed.w_up, routed.s_up, routed.w_down, routed.s_down)
        sh = moe.Experts(shared.w_gate, shared.s_gate, shared.w_up, shared.s_up, shared.w_down, shared.s_down)
        x, lg, zm = _inputs(rank)
        layer = ep.ExpertParallelPrefill(ep.local_experts(full, rank, world), E, TS[rank], K, rank, world, sh,
                                         device="cpu")
        out = layer(torch.from_numpy(x.astype(np.int32)), torch.from_numpy(lg), torch.from_numpy(zm))
        ref = oracle.moe(x, lg, K, routed, shared, zero_mask=zm)["out"]
        err = float(np.abs(out.numpy() - ref).max() / np.abs(ref).max())
        q.put((rank, "ok" if err < 1e-5 else "max rel err %.3g" % err))
    except Exception as e:  # reported to the parent
        import traceback
        q.put((rank, traceback.format_exc()[-2000:]))
    finally:
        dist.destroy_process_group()


def test_ep_prefill_forward_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=300) for _ in procs)
    for p in procs:
        p.join(timeout=60)
    assert res == {0: "ok", 1: "ok"}, res
