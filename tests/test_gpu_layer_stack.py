"""LayerStack (the synthetic multi-layer prefill): its orchestration against the same
steps written out here, and the degenerate case where approximate and dense attention
coincide.

* One layer equals: RMSNorm in fp32, three projections, spava_attn_prefill on the
  projected q/k/v, output projection, residual -- computed here step by step with the
  stack's own weights (to bf16 rounding: the library GEMMs may pick other kernels).
* With one host the approximate prefill is dense causal attention, so a 3-layer
  stack gives the same hidden states either way (within bf16 rounding).
* Hidden states stay finite through the layers.
"""

import pytest
import torch

from workloads import CONFIGS, generate

from .helpers import make_plan

pytestmark = pytest.mark.gpu

sab = pytest.importorskip("sequence_approximate_attention_b200")

CFG = CONFIGS["tiny"].with_(n_visual=1024, n_hosts=4, head_dim=128, hq=8, hkv=2, anchor=64, passing=64,
                            probe_r=32, n_text=40)


def _stack(cfg, n_layers):
    from sequence_approximate_attention_b200.layer_stack import LayerStack

    g = generate(cfg)
    plan = make_plan(sab, cfg, g["host_sizes"])
    hidden = cfg.hq * cfg.head_dim
    stack = LayerStack(plan, hidden, n_layers, seed=3)
    x = (torch.randn(plan.n_total, hidden, generator=torch.Generator().manual_seed(4)) * 0.5).to(torch.bfloat16).cuda()
    return plan, stack, x


def test_one_layer_matches_the_steps():
    plan, stack, x = _stack(CFG, 1)
    got = stack.forward(x)
    L = stack.layers[0]
    NT = plan.n_total
    h = x.float()
    h = (h * torch.rsqrt(h.pow(2).mean(dim=1, keepdim=True) + 1e-6)).to(torch.bfloat16)
    q = torch.matmul(h, L["wq"]).view(NT, plan.hq, plan.head_dim).contiguous()
    k = torch.matmul(h, L["wk"]).view(NT, plan.hkv, plan.head_dim).contiguous()
    v = torch.matmul(h, L["wv"]).view(NT, plan.hkv, plan.head_dim).contiguous()
    o, _ = sab.attn_prefill(plan, q, k, v)
    want = x + torch.matmul(o.view(NT, -1), L["wo"])
    torch.cuda.synchronize()
    torch.testing.assert_close(got.float(), want.float(), atol=3e-2, rtol=2e-2)
    plan.close()


def test_one_host_stack_equals_dense():
    plan, stack, x = _stack(CFG.with_(n_hosts=1), 3)
    a = stack.forward(x).float()
    b = stack.forward(x, dense=True).float()
    torch.cuda.synchronize()
    assert torch.isfinite(a).all() and torch.isfinite(b).all()
    assert (a - b).abs().max().item() <= 5e-2 * max(1.0, b.abs().max().item())
    plan.close()


def test_stack_stays_finite():
    plan, stack, x = _stack(CFG, 4)
    y = stack.forward(x)
    torch.cuda.synchronize()
    assert torch.isfinite(y.float()).all()
    assert stack.flops()["projections"] > 0
    plan.close()
