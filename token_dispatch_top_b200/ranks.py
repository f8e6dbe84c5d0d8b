"""The path across P GPUs, one process per GPU: host plumbing around the
per-rank entry points of libzb (argument marshalling and collectives only;
every step of the path runs in the library's kernels).

ISER-MoE ("Methodology / HALO-Q Scheduler", stage 1) has the ranks exchange
their route counts and then plan alike; MoonEP ("What MoonEP enforces and
how") has each rank write its rows straight into the fixed-shape receive
buffers of the other ranks.  On rank i of a process group of P ranks:

1. ``zb.count`` on the rank's own ids;
2. ``zb.exchange_counts``: an all-gather of the P count rows (NCCL);
3. ``zb.plan_rank``: the same plan tables on every rank, the rows of rank
   i's own entries;
4. ``zb.dispatch_rank``: rank i's rows stored into every rank's receive
   buffer, addressed through the P base pointers of a symmetric-memory
   allocation (plain stores over NVLink; no bulk or multicast copies);
5. a stream-ordered barrier (a one-element all-reduce), after which every
   rank's buffer holds all its rows for the expert computation;
6. after the experts have written their outputs into the symmetric output
   buffer and a second barrier, ``zb.combine_rank`` gathers rank i's tokens
   from every rank's outputs (plain loads), and a third barrier keeps the
   next invocation from overwriting outputs another rank still reads.

No kernel of this path waits on another rank: the ranks meet only in the
collectives.  Every rank takes the same collective steps in the same order.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import zb


class RankGroup:
    """Rank ``dist.get_rank(group)`` of a P-GPU group running the path with
    its own ``cfg.S`` tokens; ``cfg.P`` must equal the group's size."""

    def __init__(self, cfg: zb.Config, group=None, device=None):
        import torch.distributed._symmetric_memory as symm_mem
        self.group = group if group is not None else dist.group.WORLD
        self.rank = dist.get_rank(self.group)
        P = dist.get_world_size(self.group)
        if cfg.P != P:
            raise zb.ZbError(zb.ERR_INVALID, f"cfg.P = {cfg.P}, but the group has {P} ranks")
        self.cfg = cfg
        self.device = torch.device("cuda", torch.cuda.current_device()) \
            if device is None else torch.device(device)
        self.plan = zb.RankPlan(cfg, self.rank, self.device)
        # receive buffer and expert outputs, addressable by every rank
        self.buf = symm_mem.empty(cfg.cap, cfg.H, dtype=torch.bfloat16, device=self.device)
        self.y = symm_mem.empty(cfg.cap, cfg.H, dtype=torch.bfloat16, device=self.device)
        self._buf_h = symm_mem.rendezvous(self.buf, self.group)
        self._y_h = symm_mem.rendezvous(self.y, self.group)
        self.buf_ptrs = list(self._buf_h.buffer_ptrs)
        self.y_ptrs = list(self._y_h.buffer_ptrs)
        self._tick = torch.zeros(1, dtype=torch.int32, device=self.device)

    def barrier(self) -> None:
        """Stream-ordered: work after it on this stream starts once every rank
        has enqueued and run everything before its own barrier."""
        dist.all_reduce(self._tick, group=self.group)

    def plan_and_dispatch(self, topk_ids: torch.Tensor, hidden: torch.Tensor,
                          placement: torch.Tensor | None = None) -> None:
        """Steps 1-4 and the barrier: afterwards ``self.buf`` holds this
        rank's received rows, grouped by ``self.plan.cu_seqlens[rank]``."""
        zb.count(self.plan, topk_ids)
        zb.exchange_counts(self.plan.counts, self.plan.table, self.group)
        zb.plan_rank(self.plan, topk_ids, placement)
        zb.dispatch_rank(self.plan, hidden, self.buf_ptrs)
        self.barrier()

    def combine(self, topk_weights: torch.Tensor, out: torch.Tensor) -> None:
        """Step 5 once the expert outputs are in ``self.y`` on every rank."""
        self.barrier()
        zb.combine_rank(self.plan, self.y_ptrs, topk_weights, out)
        self.barrier()
