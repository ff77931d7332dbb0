"""A synthetic multi-layer prefill: the attention blocks of a decoder with random
weights, for a time-to-first-token style comparison of the approximate-attention
prefill against dense causal attention on the same layers.

Each layer, on hidden states x [N+T, hidden] (bf16), entirely in the library's kernels:

    q, k, v = split((x / rms(x)) W_qkv^T)   spava_qkv_projection: tcgen05 GEMM whose
                                             epilogue applies the RMSNorm row scale and
                                             writes q, k, v in the [tokens, heads, d]
                                             layouts the attention reads
    o = attention(q, k, v)                   spava_attn_prefill (or the two-stage flow,
                                             or spava_dense_causal for the comparison)
    x = x + o W_o^T                          spava_out_projection: tcgen05 GEMM with the
                                             residual add in its epilogue, in place

Weights are random (seeded, scaled by fan_in^-1/2) and stored with rows = output
features (W_qkv [(hq + 2 hkv) d, hidden], W_o [hidden, hq d]); there is no rotary
embedding, no norm gain and no MLP: the layers carry the work the method changes
(attention) and the linear maps around it.
"""

from typing import List, Optional

import torch

from . import (Plan, attn_prefill, attn_prefill_two_stage, check_layer_error, dense_causal, layer_workspace,
               out_projection, qkv_projection)

__all__ = ["LayerStack"]


class LayerStack:
    """``n_layers`` attention blocks sharing one plan (sizes, heads, hosts)."""

    def __init__(self, plan: Plan, hidden: int, n_layers: int, seed: int = 0, two_stage: bool = False,
                 rms_eps: float = 1e-6):
        if n_layers < 1 or hidden < 1:
            raise ValueError("need at least one layer and a positive hidden size")
        self.plan = plan
        self.hidden = hidden
        self.two_stage = two_stage
        self.rms_eps = rms_eps
        dev = plan.device
        g = torch.Generator(device="cpu").manual_seed(seed)
        qd, kd = plan.hq * plan.head_dim, plan.hkv * plan.head_dim

        def w(n_out, n_in):
            return (torch.randn(n_out, n_in, generator=g) * n_in ** -0.5).to(torch.bfloat16).to(dev)

        self.layers: List[dict] = [{"w_qkv": w(qd + 2 * kd, hidden), "w_o": w(hidden, qd)} for _ in range(n_layers)]
        self.ws = plan.new_workspace(two_stage)
        self.ws_dense = self.ws if not two_stage else plan.new_workspace(False)
        NT = plan.n_total
        self.ws_layer = layer_workspace(NT, dev)
        qs, ks = plan.qkv_shapes()
        self._x = torch.empty((NT, hidden), dtype=torch.bfloat16, device=dev)
        self._q = torch.empty(qs, dtype=torch.bfloat16, device=dev)
        self._k = torch.empty(ks, dtype=torch.bfloat16, device=dev)
        self._v = torch.empty(ks, dtype=torch.bfloat16, device=dev)
        self._o = torch.empty(qs, dtype=torch.bfloat16, device=dev)
        self._lse = torch.empty((plan.hq, NT), dtype=torch.float32, device=dev)

    def forward(self, x: torch.Tensor, dense: bool = False, record: Optional[list] = None) -> torch.Tensor:
        """All layers on x [N+T, hidden] bf16 (device), on the current stream; returns the
        final hidden states (the stack's own buffer: copy it to keep it past the next
        call).  ``dense`` swaps the approximate prefill for the dense causal kernel.
        With a list in ``record`` each layer appends a dict of clones of its input x,
        q, k, v, o, lse and, for the approximate prefill, its selection (for tests)."""
        plan = self.plan
        if x.shape != (plan.n_total, self.hidden) or x.dtype != torch.bfloat16:
            raise ValueError(f"x must be bf16 [{plan.n_total}, {self.hidden}]")
        self._x.copy_(x)
        for L in self.layers:
            x_in = self._x.clone() if record is not None else None
            qkv_projection(self._x, L["w_qkv"], plan.hq, plan.hkv, plan.head_dim, self._q, self._k, self._v,
                           self.ws_layer, self.rms_eps)
            idx = None
            if dense:
                dense_causal(plan, self._q, self._k, self._v, o=self._o, lse=self._lse, workspace=self.ws_dense)
            else:
                prefill = attn_prefill_two_stage if self.two_stage else attn_prefill
                if record is not None and plan.n_hosts > 1 and plan.passing > 0:
                    idx = torch.empty(plan.idx_shape(), dtype=torch.int32, device=self._x.device)
                prefill(plan, self._q, self._k, self._v, o=self._o, lse=self._lse, workspace=self.ws, idx_out=idx)
            out_projection(self._o, L["w_o"], self._x, self.ws_layer)
            if record is not None:
                record.append({"x": x_in, "q": self._q.clone(), "k": self._k.clone(), "v": self._v.clone(),
                               "o": self._o.clone(), "lse": self._lse.clone(), "sel": idx})
        return self._x

    def check_errors(self) -> None:
        """Raise if a bounded device wait of a projection ran out (synchronises)."""
        check_layer_error(self.ws_layer)

    def flops(self) -> dict:
        """Projection FLOPs per layer (the attention's are counted by the caller)."""
        NT, qd, kd = self.plan.n_total, self.plan.hq * self.plan.head_dim, self.plan.hkv * self.plan.head_dim
        return {"projections": 2.0 * NT * self.hidden * (2 * qd + 2 * kd),
                "qkv": 2.0 * NT * self.hidden * (qd + 2 * kd), "out": 2.0 * NT * qd * self.hidden}
