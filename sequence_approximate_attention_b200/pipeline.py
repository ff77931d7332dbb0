"""Prefill from pinned host memory with the copies overlapped with the compute.

``HostPrefillPipeline.submit`` takes one layer's q, k, v in pinned host memory and
host buffers for o and lse.  It enqueues, on three CUDA streams of its own,

    copy-in:   q, k, v host -> one of two device input sets
    compute:   spava_attn_prefill (or the two-stage flow) on that set
    copy-out:  o, lse of that set -> host

and returns at once, so the host->device copy of call n+1 and the device->host copy
of call n-1 run while call n computes (PCIe moves both directions at once).  Events
order the reuse of the two sets: inputs of set s are overwritten only after the
compute of the call two back has finished with them, outputs of set s only after
they have been copied out.  ``wait`` makes a stream wait for everything submitted;
host buffers handed to ``submit`` must stay untouched until then.

Only copies and stream ordering happen here; the prefill itself is the library's
single C-ABI call on the compute stream.
"""

from typing import Optional

import torch

from . import Plan, attn_prefill, attn_prefill_two_stage

__all__ = ["HostPrefillPipeline"]


def _expect_host(t: torch.Tensor, name: str, dtype, shape) -> None:
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.device.type != "cpu" or not t.is_pinned():
        raise ValueError(f"{name} must be in pinned host memory")
    if t.dtype != dtype or tuple(t.shape) != tuple(shape) or not t.is_contiguous():
        raise ValueError(f"{name}: expected contiguous {dtype} {tuple(shape)}, got {t.dtype} {tuple(t.shape)}")


class HostPrefillPipeline:
    """Double-buffered prefill of host-resident layers on one device (see module doc)."""

    def __init__(self, plan: Plan, two_stage: bool = False):
        self.plan = plan
        self.two_stage = two_stage
        dev = plan.device
        qs, ks = plan.qkv_shapes()
        bf16 = torch.bfloat16
        self._q = [torch.empty(qs, dtype=bf16, device=dev) for _ in range(2)]
        self._k = [torch.empty(ks, dtype=bf16, device=dev) for _ in range(2)]
        self._v = [torch.empty(ks, dtype=bf16, device=dev) for _ in range(2)]
        self._o = [torch.empty(qs, dtype=bf16, device=dev) for _ in range(2)]
        self._lse = [torch.empty((plan.hq, plan.n_total), dtype=torch.float32, device=dev) for _ in range(2)]
        self._ws = plan.new_workspace(two_stage)
        self._copy_in = torch.cuda.Stream(dev)
        self._compute = torch.cuda.Stream(dev)
        self._copy_out = torch.cuda.Stream(dev)
        self._in_ready = [torch.cuda.Event() for _ in range(2)]
        self._done = [torch.cuda.Event() for _ in range(2)]
        self._out_done = [torch.cuda.Event() for _ in range(2)]
        self._n = 0

    @property
    def h2d_bytes(self) -> int:
        return sum(t.numel() * t.element_size() for t in (self._q[0], self._k[0], self._v[0]))

    @property
    def d2h_bytes(self) -> int:
        return self._o[0].numel() * 2 + self._lse[0].numel() * 4

    def submit(self, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, o: torch.Tensor, lse: torch.Tensor) -> None:
        """Enqueue one layer: q, k, v pinned host inputs; o, lse pinned host outputs."""
        plan = self.plan
        qs, ks = plan.qkv_shapes()
        _expect_host(q, "q", torch.bfloat16, qs)
        _expect_host(k, "k", torch.bfloat16, ks)
        _expect_host(v, "v", torch.bfloat16, ks)
        _expect_host(o, "o", torch.bfloat16, qs)
        _expect_host(lse, "lse", torch.float32, (plan.hq, plan.n_total))
        s = self._n & 1
        # copy-in: after the caller's prior work and after the compute two calls back
        self._copy_in.wait_stream(torch.cuda.current_stream(plan.device))
        self._copy_in.wait_event(self._done[s])
        with torch.cuda.stream(self._copy_in):
            self._q[s].copy_(q, non_blocking=True)
            self._k[s].copy_(k, non_blocking=True)
            self._v[s].copy_(v, non_blocking=True)
        self._in_ready[s].record(self._copy_in)
        # compute: inputs in place, outputs of this set copied out two calls back
        self._compute.wait_event(self._in_ready[s])
        self._compute.wait_event(self._out_done[s])
        prefill = attn_prefill_two_stage if self.two_stage else attn_prefill
        prefill(plan, self._q[s], self._k[s], self._v[s], o=self._o[s], lse=self._lse[s], workspace=self._ws,
                stream=self._compute)
        self._done[s].record(self._compute)
        # copy-out
        self._copy_out.wait_event(self._done[s])
        with torch.cuda.stream(self._copy_out):
            o.copy_(self._o[s], non_blocking=True)
            lse.copy_(self._lse[s], non_blocking=True)
        self._out_done[s].record(self._copy_out)
        self._n += 1

    def wait(self, stream: Optional[torch.cuda.Stream] = None) -> None:
        """Make `stream` (default: the current one) wait for every submitted layer."""
        st = torch.cuda.current_stream(self.plan.device) if stream is None else stream
        for e in self._out_done:
            st.wait_event(e)

    def synchronize(self) -> None:
        """Block the host until every submitted layer's outputs are in host memory."""
        self._copy_out.synchronize()
