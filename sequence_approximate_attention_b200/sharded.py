"""Sharded prefill: the host blocks of one layer spread over ranks (one process per
GPU), the library's kernels on every rank, the exchange by torch.distributed.

The pages' system (APB-V technical summary, 1. Framework design, "Context splitting &
ZigZag arrangement"; 2. System optimisations, "Overlapped communication"): each
physical host runs a pair of virtual hosts (h, 2W-1-h), sends its passing blocks to
the later hosts and its partial query results to be merged, and these transfers run
while attention computes.  Per rank and layer:

    compute stream                         comm stream
                                           broadcast anchor rows k, v [0, A)
    SELECT  score/select own hosts,
            passing rows -> own part  ---> all-gather passing K, V
    LOCAL   own blocks (causal),
            text pieces -> own slots  ---> all-gather text partials (O, lse)
    REMOTE  (waits for the passing and anchor) own hosts over [anchor | passing],
            merged with the local partials
    MERGE   (waits for the text partials) text rows from all ranks' slots

With ``overlap=False`` (the one-pass form) the rank waits for the passing exchange
after SELECT and runs ATTEND, one pass per own host over [anchor | passing | own
block], instead of LOCAL + REMOTE: on NVLink the exchange is short next to the
attention, and one pass saves the fp32 row partials and the second online softmax.

Every rank issues the same collectives in the same order.  The exchange buffers
live in the plan's sharded workspace, rank-major, so every collective is an
in-place all-gather of one contiguous run per rank.  With NCCL they run on a
separate CUDA stream ordered by events; with gloo (CPU tensors) they run in line.
The plan object is anything with ``set_shard``, ``shard_layout``, ``shard_stage``,
``device`` and the size attributes of :class:`Plan`.
"""

from typing import Optional, Sequence

import torch
import torch.distributed as dist

from . import _lib

__all__ = ["ShardedPrefill"]


class ShardedPrefill:
    """One rank's side of the sharded prefill of a plan (see the module docstring)."""

    def __init__(self, plan, rank: int, world: int, owner: Sequence[int], group=None, overlap: bool = True):
        if len(owner) != plan.n_hosts:
            raise ValueError("owner needs one rank per host")
        self.plan, self.rank, self.world, self.group = plan, int(rank), int(world), group
        self.overlap = bool(overlap)
        self.owner = [int(x) for x in owner]
        plan.set_shard(self.rank, self.world, self.owner)
        L = plan.shard_layout()
        self.layout = L
        self.ws = torch.zeros(max(int(L.workspace_bytes), 256), dtype=torch.uint8, device=plan.device)

        def run(off, per_rank):
            whole = self.ws[int(off): int(off) + self.world * int(per_rank)]
            mine = whole[self.rank * int(per_rank): (self.rank + 1) * int(per_rank)]
            return whole, mine

        self.pass_k, self.pass_k_mine = run(L.pass_k_offset, L.pass_bytes_per_rank)
        self.pass_v, self.pass_v_mine = run(L.pass_v_offset, L.pass_bytes_per_rank)
        self.text_o, self.text_o_mine = run(L.text_o_offset, L.text_o_bytes_per_rank)
        self.text_lse, self.text_lse_mine = run(L.text_lse_offset, L.text_lse_bytes_per_rank)
        self.anchor_src = self.owner[0]
        self.cuda = plan.device.type == "cuda"
        self.comm = torch.cuda.Stream(device=plan.device) if self.cuda else None
        self.launches = 0  # library kernel launches enqueued by forward() so far

    # -- collectives (same sequence on every rank)
    def _gather(self, whole: torch.Tensor, mine: torch.Tensor) -> None:
        if whole.numel():
            dist.all_gather_into_tensor(whole, mine, group=self.group)

    def _broadcast_anchor(self, k: torch.Tensor, v: torch.Tensor) -> None:
        # rows [0, A) belong to host 0: read by its owner's stages only, written here
        # on every other rank, where no stage before REMOTE / ATTEND reads them
        A = self.plan.anchor
        if A > 0 and self.plan.n_hosts > 1:
            dist.broadcast(k[:A], src=self.anchor_src, group=self.group)
            dist.broadcast(v[:A], src=self.anchor_src, group=self.group)

    def _exchange_passing(self) -> None:
        self._gather(self.pass_k, self.pass_k_mine)
        self._gather(self.pass_v, self.pass_v_mine)

    def _exchange_text(self) -> None:
        self._gather(self.text_o, self.text_o_mine)
        self._gather(self.text_lse, self.text_lse_mine)

    def _on_comm(self, after: "torch.cuda.Event", fn, *args):
        """Run fn on the comm stream after `after`; returns the event that marks its end."""
        if not self.cuda:
            fn(*args)
            return None
        with torch.cuda.stream(self.comm):
            self.comm.wait_event(after)
            fn(*args)
            done = torch.cuda.Event()
            done.record(self.comm)
        return done

    def forward(self, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, o: Optional[torch.Tensor] = None,
                lse: Optional[torch.Tensor] = None):
        """One layer on this rank.  q/k/v are full-size [N+T, heads, d] buffers holding
        this rank's host rows and the text rows (the anchor rows arrive by broadcast);
        their other rows must be finite (zeros will do).  Returns (o, lse) with this
        rank's host rows and all text rows final."""
        plan = self.plan
        if o is None:
            o = torch.empty_like(q)
        if lse is None:
            lse = torch.empty((plan.hq, plan.n_total), dtype=torch.float32, device=plan.device)
        cur = torch.cuda.current_stream(plan.device) if self.cuda else None
        stage_fn = plan.shard_stage

        def stage(*a):
            stage_fn(*a)
            self.launches += _lib.launches_of_last_call()

        def mark():
            if not self.cuda:
                return None
            e = torch.cuda.Event()
            e.record(cur)
            return e

        if self.cuda:
            k.record_stream(self.comm)
            v.record_stream(self.comm)
        self._on_comm(mark(), self._broadcast_anchor, k, v)
        stage(_lib.SPAVA_SHARD_SELECT, q, k, v, None, None, self.ws)
        pass_done = self._on_comm(mark(), self._exchange_passing)
        if self.overlap:
            stage(_lib.SPAVA_SHARD_LOCAL, q, k, v, o, lse, self.ws)
            text_done = self._on_comm(mark(), self._exchange_text)
            if pass_done is not None:
                cur.wait_event(pass_done)
            stage(_lib.SPAVA_SHARD_REMOTE, q, k, v, o, lse, self.ws)
        else:
            if pass_done is not None:
                cur.wait_event(pass_done)
            stage(_lib.SPAVA_SHARD_ATTEND, q, k, v, o, lse, self.ws)
            text_done = self._on_comm(mark(), self._exchange_text)
        if text_done is not None:
            cur.wait_event(text_done)
        stage(_lib.SPAVA_SHARD_MERGE, None, None, None, o, lse, self.ws)
        return o, lse

    def owned_rows(self):
        """[(row0, row1), ...] visual rows whose output this rank computes."""
        off = self.plan.offsets
        return [(off[h], off[h + 1]) for h in range(self.plan.n_hosts) if self.owner[h] == self.rank]
