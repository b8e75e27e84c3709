"""Expert-parallel decode over a process group (NCCL on GPUs).

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

from . import (MOE_MODE_DECODE, MOE_OUT_F32, Experts, moe_combine, moe_expert_ffn, moe_ffn_workspace_bytes,
               moe_route, moe_sort, moe_sort_workspace_bytes)


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
