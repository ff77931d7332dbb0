"""A synthetic multi-layer prefill: the attention blocks of a decoder with random
weights, for a time-to-first-token style comparison of the approximate-attention
prefill against dense causal attention on the same layers.

Each layer, on hidden states x [N+T, hidden] (bf16):

    h = rms_norm(x)
    q = h W_q, k = h W_k, v = h W_v          (plain GEMMs: cuBLAS through torch.matmul)
    o = attention(q, k, v)                   (the library: spava_attn_prefill, or
                                              spava_dense_causal for the comparison)
    x = x + o W_o

The attention is the library's C-ABI call on the same plan and workspace for every
layer; the projections are plain library GEMMs.  Weights are random (seeded,
scaled by hidden^-1/2); there is no rotary embedding and no MLP: the layers carry the
work the method changes (attention) and the linear maps around it.
"""

from typing import List

import torch

from . import Plan, attn_prefill, attn_prefill_two_stage, dense_causal

__all__ = ["LayerStack"]


class LayerStack:
    """``n_layers`` attention blocks sharing one plan (sizes, heads, hosts)."""

    def __init__(self, plan: Plan, hidden: int, n_layers: int, seed: int = 0, two_stage: bool = False):
        if n_layers < 1 or hidden < 1:
            raise ValueError("need at least one layer and a positive hidden size")
        self.plan = plan
        self.hidden = hidden
        self.two_stage = two_stage
        dev = plan.device
        g = torch.Generator(device="cpu").manual_seed(seed)
        qd, kd = plan.hq * plan.head_dim, plan.hkv * plan.head_dim

        def w(n_in, n_out):
            return (torch.randn(n_in, n_out, generator=g) * n_in ** -0.5).to(torch.bfloat16).to(dev)

        self.layers: List[dict] = [
            {"wq": w(hidden, qd), "wk": w(hidden, kd), "wv": w(hidden, kd), "wo": w(qd, hidden)}
            for _ in range(n_layers)]
        self.ws = plan.new_workspace(two_stage)
        self.ws_dense = self.ws if not two_stage else plan.new_workspace(False)
        NT = plan.n_total
        qs, ks = plan.qkv_shapes()
        self._q = torch.empty(qs, dtype=torch.bfloat16, device=dev)
        self._k = torch.empty(ks, dtype=torch.bfloat16, device=dev)
        self._v = torch.empty(ks, dtype=torch.bfloat16, device=dev)
        self._o = torch.empty(qs, dtype=torch.bfloat16, device=dev)
        self._lse = torch.empty((plan.hq, NT), dtype=torch.float32, device=dev)

    def forward(self, x: torch.Tensor, dense: bool = False) -> torch.Tensor:
        """All layers on x [N+T, hidden] bf16 (device), on the current stream; returns the
        new hidden states.  ``dense`` swaps the approximate prefill for the dense causal
        kernel."""
        plan = self.plan
        if x.shape != (plan.n_total, self.hidden) or x.dtype != torch.bfloat16:
            raise ValueError(f"x must be bf16 [{plan.n_total}, {self.hidden}]")
        NT = plan.n_total
        for L in self.layers:
            h = x.float()
            h = (h * torch.rsqrt(h.pow(2).mean(dim=1, keepdim=True) + 1e-6)).to(torch.bfloat16)
            torch.matmul(h, L["wq"], out=self._q.view(NT, -1))
            torch.matmul(h, L["wk"], out=self._k.view(NT, -1))
            torch.matmul(h, L["wv"], out=self._v.view(NT, -1))
            if dense:
                dense_causal(plan, self._q, self._k, self._v, o=self._o, lse=self._lse, workspace=self.ws_dense)
            else:
                prefill = attn_prefill_two_stage if self.two_stage else attn_prefill
                prefill(plan, self._q, self._k, self._v, o=self._o, lse=self._lse, workspace=self.ws)
            x = x + torch.matmul(self._o.view(NT, -1), L["wo"])
        return x

    def flops(self) -> dict:
        """Projection FLOPs per layer (the attention's are counted by the caller)."""
        NT, qd, kd = self.plan.n_total, self.plan.hq * self.plan.head_dim, self.plan.hkv * self.plan.head_dim
        return {"projections": 2.0 * NT * self.hidden * (2 * qd + 2 * kd)}
