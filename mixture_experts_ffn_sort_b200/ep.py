"""Expert parallelism over a process group (NCCL on GPUs): decode with an
all-reduce of partial outputs, prefill with all-to-all dispatch and combine.

The pages' decode kernel shards the experts across devices: every device
routes all tokens the same way, applies only the experts it holds, and the
partial outputs are summed across devices before the shared expert is added
(dstair/gated-deltanet-nki-trainium, "FP8 MoE decode kernel", "Interface" and
"Serving contract": local routed experts, expert-sum, an all-reduce across the
expert-parallel group).  This module does that with the library's own calls:

    route (all experts) -> sort (all experts) -> zero y_sorted
    -> expert FFN on this rank's experts only (a view of the global offsets)
    -> combine in fp32 (only this rank's rows are nonzero; rank 0 adds the
       shared expert) -> all-reduce (sum) over the group

so no kernel is specific to it.  Rank r of G holds experts
[r*E/G, (r+1)*E/G); E must be a multiple of 4*G (each rank's slice of the
offsets must start 16-byte aligned).  The partial sums are fp32; the result
equals the single-device layer up to the order of the fp32 additions.
"""
import contextlib
from typing import Optional, Tuple

import torch

from . import (MOE_MODE_AUTO, MOE_MODE_DECODE, MOE_OUT_BF16, MOE_OUT_F32, Experts, moe_combine, moe_expert_ffn,
               moe_ffn_workspace_bytes, moe_route, moe_sort, moe_sort_workspace_bytes)


def expert_range(E: int, rank: int, world: int) -> Tuple[int, int]:
    """[begin, end) of the experts rank `rank` of `world` holds."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("rank %d of %d" % (rank, world))
    if E % (4 * world):
        raise ValueError("E=%d must be a multiple of 4 * world (%d)" % (E, 4 * world))
    n = E // world
    return rank * n, (rank + 1) * n


def local_experts(full: Experts, rank: int, world: int) -> Experts:
    """This rank's slice of a full set of experts (views, no copy)."""
    b, e = expert_range(full.n, rank, world)
    return Experts(full.w_gate[b:e], full.s_gate[b:e], full.w_up[b:e], full.s_up[b:e],
                   full.w_down[b:e], full.s_down[b:e])


def reduce_partials(partial: torch.Tensor, group=None) -> torch.Tensor:
    """Sum the ranks' partial outputs in place (no-op without a group)."""
    import torch.distributed as dist
    if group is not None or (dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1):
        dist.all_reduce(partial, op=dist.ReduceOp.SUM, group=group)
    return partial


class ExpertParallelMoE:
    """One rank of an expert-parallel MoE FFN layer on fixed shapes.

    routed: this rank's experts (see local_experts); E: the total number of
    experts; shared: the shared expert, applied by rank 0 only.  Buffers are
    allocated once.  forward() returns the fp32 layer output summed over the
    group; partial() returns this rank's share without the collective.
    """

    def __init__(self, routed: Experts, E: int, T: int, K: int, rank: int, world: int,
                 shared: Optional[Experts] = None, mode: int = MOE_MODE_DECODE, device="cuda", group=None):
        self.e_begin, self.e_end = expert_range(E, rank, world)
        if routed.n != self.e_end - self.e_begin:
            raise ValueError("rank %d holds %d experts, expected %d" % (rank, routed.n, self.e_end - self.e_begin))
        self.routed, self.E, self.T, self.K, self.rank, self.world = routed, E, T, K, rank, world
        self.shared = shared if rank == 0 else None
        self.mode, self.group = mode, group
        H = routed.w_gate.shape[2]
        d = device
        R = T * K
        self.topk_ids = torch.empty((T, K), dtype=torch.int32, device=d)
        self.topk_w = torch.empty((T, K), dtype=torch.float32, device=d)
        self.offsets = torch.empty(E + 1, dtype=torch.int32, device=d)
        self.sorted_route = torch.empty(R, dtype=torch.int32, device=d)
        self.inv_route = torch.empty(R, dtype=torch.int32, device=d)
        self.sort_ws = torch.empty(max(16, moe_sort_workspace_bytes(T, K, E)), dtype=torch.uint8, device=d)
        self.ffn_ws = torch.empty(max(16, moe_ffn_workspace_bytes(
            T, K, H, routed.n, routed.inter, self.shared.inter if self.shared else 0, mode)), dtype=torch.uint8, device=d)
        self.y_sorted = torch.empty((R, H), dtype=torch.bfloat16, device=d)
        self.y_shared = torch.empty((T, H), dtype=torch.bfloat16, device=d) if self.shared else None
        self.out = torch.empty((T, H), dtype=torch.float32, device=d)
        self.status = torch.zeros(1, dtype=torch.int32, device=d)

    def partial(self, x: torch.Tensor, logits: torch.Tensor, zero_mask: Optional[torch.Tensor] = None,
                stream=None) -> torch.Tensor:
        moe_route(logits, self.K, zero_mask, self.topk_ids, self.topk_w, stream=stream)
        moe_sort(self.topk_ids, self.E, self.status, self.offsets, self.sorted_route, self.inv_route,
                 self.sort_ws, stream=stream)
        # Rows of the other ranks' experts stay zero in the combine.
        with torch.cuda.stream(stream) if stream is not None else contextlib.nullcontext():
            self.y_sorted.zero_()
        local_offsets = self.offsets[self.e_begin:self.e_end + 1]
        moe_expert_ffn(x, self.K, self.routed, local_offsets, self.sorted_route, self.topk_w, self.shared,
                       self.mode, self.status, self.y_sorted, self.y_shared, self.ffn_ws, stream=stream)
        return moe_combine(self.y_sorted, self.inv_route, self.y_shared, self.T, self.K, MOE_OUT_F32, self.out,
                           stream=stream)

    def forward(self, x: torch.Tensor, logits: torch.Tensor, zero_mask: Optional[torch.Tensor] = None,
                stream=None) -> torch.Tensor:
        return reduce_partials(self.partial(x, logits, zero_mask, stream), self.group)

    __call__ = forward


# ---------------------------------------------------------------- prefill: all-to-all dispatch and combine

def all_to_all_rows(send: torch.Tensor, send_rows, recv_rows, group=None) -> torch.Tensor:
    """Exchange row blocks: block d of `send` (send_rows[d] rows) goes to rank
    d; the result holds recv_rows[s] rows from each rank s, in rank order."""
    import torch.distributed as dist
    out = torch.empty((int(sum(recv_rows)),) + tuple(send.shape[1:]), dtype=send.dtype, device=send.device)
    dist.all_to_all_single(out, send.contiguous(), output_split_sizes=[int(v) for v in recv_rows],
                           input_split_sizes=[int(v) for v in send_rows], group=group)
    return out


class ExpertParallelPrefill:
    """One rank of a token-sharded, expert-parallel MoE FFN (the all-to-all-v
    dispatch and combine of the NKI library's MoE kernels: Build All2All
    Dispatch Metadata, Permute / Unpermute Routed Tokens).

    Every rank routes and sorts its own T tokens over all E experts, sends each
    route's x row and weight to the rank holding its expert (rows of one
    destination are contiguous in the sorted order), runs its experts on the
    rows it receives (as tokens with K = 1: sort by local expert, expert FFN
    with the route weight in the down epilogue, un-permute), sends the
    results back, where they arrive in the sender's sorted order -- its
    y_sorted -- and combines them through its inverse route map, adding its
    own shared expert.  The library's kernels do all of that but the
    exchanges (all_to_all_single) and the bookkeeping of counts (integer
    tensors; the row counts are read back to the host to size the exchange).

    The steps are also callable one by one (dispatch, expert_rows, finish),
    which is how one process can stand in for several ranks.
    """

    def __init__(self, routed: Experts, E: int, T: int, K: int, rank: int, world: int,
                 shared: Optional[Experts] = None, mode: int = MOE_MODE_AUTO, device="cuda", group=None):
        self.e_begin, self.e_end = expert_range(E, rank, world)
        if routed.n != self.e_end - self.e_begin:
            raise ValueError("rank %d holds %d experts, expected %d" % (rank, routed.n, self.e_end - self.e_begin))
        self.routed, self.shared, self.E, self.T, self.K = routed, shared, E, T, K
        self.rank, self.world, self.mode, self.group, self.dev = rank, world, mode, group, device
        self.El = E // world
        self.H = routed.w_gate.shape[2]
        d = device
        R = T * K
        self.topk_ids = torch.empty((T, K), dtype=torch.int32, device=d)
        self.topk_w = torch.empty((T, K), dtype=torch.float32, device=d)
        self.offsets = torch.empty(E + 1, dtype=torch.int32, device=d)
        self.sorted_route = torch.empty(R, dtype=torch.int32, device=d)
        self.inv_route = torch.empty(R, dtype=torch.int32, device=d)
        self.sort_ws = torch.empty(max(16, moe_sort_workspace_bytes(T, K, E)), dtype=torch.uint8, device=d)
        self.no_rows = torch.zeros(self.El + 1, dtype=torch.int32, device=d)  # offsets of an empty routed set
        self.status = torch.zeros(1, dtype=torch.int32, device=d)

    def dispatch(self, x: torch.Tensor, logits: torch.Tensor, zero_mask: Optional[torch.Tensor] = None):
        """Route and sort this rank's tokens.  Returns (rows [R, H] bf16 and
        weights [R] f32 in sorted order, per-expert route counts [world, El]
        i32 on the device, rows per destination rank as a host list)."""
        moe_route(logits, self.K, zero_mask, self.topk_ids, self.topk_w)
        moe_sort(self.topk_ids, self.E, self.status, self.offsets, self.sorted_route, self.inv_route, self.sort_ws)
        R = self.T * self.K
        # Row p of the sorted order is route sorted_route[p] = t * K + j: token t.
        src_token = torch.div(self.sorted_route, self.K, rounding_mode="floor").to(torch.int32)
        rows = moe_combine(x, src_token, None, R, 1, MOE_OUT_BF16)  # a gather: one term per output row
        wts = self.topk_w.view(-1)[self.sorted_route.long()]
        counts = (self.offsets[1:] - self.offsets[:-1]).view(self.world, self.El).contiguous()
        ends = self.offsets[::self.El].cpu().tolist()  # dispatch metadata: one read-back
        send_rows = [ends[d + 1] - ends[d] for d in range(self.world)]
        return rows, wts, counts, send_rows

    def expert_rows(self, recv_x: torch.Tensor, recv_w: torch.Tensor, recv_counts: torch.Tensor) -> torch.Tensor:
        """Run this rank's experts on the rows it received (recv_counts
        [world, El]: rows per source rank and local expert, the rows of each
        source grouped by expert in that order).  Returns the weighted output
        rows [Rr, H] bf16 in the received order."""
        Rr = recv_x.shape[0]
        H, El = self.H, self.El
        if Rr == 0:
            return torch.empty((0, H), dtype=torch.bfloat16, device=recv_x.device)
        dev = recv_x.device
        local = torch.arange(El, dtype=torch.int32, device=dev).repeat(self.world)
        ids = torch.repeat_interleave(local, recv_counts.reshape(-1).long()).view(Rr, 1)
        offs = torch.empty(El + 1, dtype=torch.int32, device=dev)
        srt = torch.empty(Rr, dtype=torch.int32, device=dev)
        inv = torch.empty(Rr, dtype=torch.int32, device=dev)
        ws = torch.empty(max(16, moe_sort_workspace_bytes(Rr, 1, El)), dtype=torch.uint8, device=dev)
        moe_sort(ids, El, self.status, offs, srt, inv, ws)
        y, _ = moe_expert_ffn(recv_x, 1, self.routed, offs, srt, recv_w.contiguous().view(Rr, 1), None, self.mode,
                              self.status)
        return moe_combine(y, inv, None, Rr, 1, MOE_OUT_BF16)  # back to the received order

    def finish(self, y_back: torch.Tensor, x: torch.Tensor, out_dtype: int = MOE_OUT_BF16) -> torch.Tensor:
        """Combine the returned rows (this rank's y_sorted) through the inverse
        route map, with this rank's shared expert on its own tokens."""
        y_shared = None
        if self.shared is not None:
            # The shared expert alone: an expert set with no routed rows.
            _, y_shared = moe_expert_ffn(x, self.K, self.routed, self.no_rows, self.sorted_route, self.topk_w,
                                         self.shared, self.mode, self.status)
        return moe_combine(y_back, self.inv_route, y_shared, self.T, self.K, out_dtype)

    def forward(self, x: torch.Tensor, logits: torch.Tensor, zero_mask: Optional[torch.Tensor] = None,
                out_dtype: int = MOE_OUT_BF16) -> torch.Tensor:
        import torch.distributed as dist
        rows, wts, counts, send_rows = self.dispatch(x, logits, zero_mask)
        recv_counts = torch.empty_like(counts)
        dist.all_to_all_single(recv_counts, counts, group=self.group)
        recv_rows = recv_counts.sum(dim=1).cpu().tolist()
        recv_x = all_to_all_rows(rows, send_rows, recv_rows, self.group)
        recv_w = all_to_all_rows(wts, send_rows, recv_rows, self.group)
        y = self.expert_rows(recv_x, recv_w, recv_counts)
        y_back = all_to_all_rows(y, recv_rows, send_rows, self.group)
        return self.finish(y_back, x, out_dtype)

    __call__ = forward
