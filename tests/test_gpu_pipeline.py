"""HostPrefillPipeline: layers submitted back to back from pinned host memory come back
identical to spava_attn_prefill on the same inputs.

The pipeline reuses two device input/output sets across calls on three streams; a
missing ordering edge would let a copy overwrite a set that a prefill still reads (or
copy out a set before its prefill wrote it), which shows as a mismatch here.  The
kernels are deterministic, so the comparison is exact.  The O-vs-oracle accuracy of
the same kernels is covered by test_gpu_parity.py.
"""

import pytest
import torch

from workloads import CONFIGS, generate

from .helpers import make_plan

pytestmark = pytest.mark.gpu

sab = pytest.importorskip("sequence_approximate_attention_b200")

TINY = CONFIGS["tiny"]
CASES = {
    "tiny_text40": TINY.with_(n_text=40),
    "d128_g7_text": TINY.with_(n_visual=1024, n_hosts=4, head_dim=128, hq=14, hkv=2, anchor=64, passing=64,
                               probe_r=32, n_text=77, kv_kind="frame", frame=64),
}


def _pinned(bits):
    return torch.from_numpy(bits.view("int16")).view(torch.bfloat16).pin_memory()


@pytest.mark.parametrize("two_stage", [False, True])
@pytest.mark.parametrize("name", list(CASES))
def test_pipeline_matches_single_calls(name, two_stage):
    from sequence_approximate_attention_b200.pipeline import HostPrefillPipeline

    cfg = CASES[name]
    layers = [generate(cfg, seed=cfg.seed + 11 * n) for n in range(5)]
    plan = make_plan(sab, cfg, layers[0]["host_sizes"])
    pipe = HostPrefillPipeline(plan, two_stage=two_stage)
    host_in = [{x: _pinned(g[x]) for x in ("q", "k", "v")} for g in layers]
    qs, _ = plan.qkv_shapes()
    outs = [(torch.empty(qs, dtype=torch.bfloat16).pin_memory(),
             torch.empty((plan.hq, plan.n_total), dtype=torch.float32).pin_memory()) for _ in layers]
    for hi, (o_h, l_h) in zip(host_in, outs):
        pipe.submit(hi["q"], hi["k"], hi["v"], o_h, l_h)
    pipe.synchronize()
    prefill = sab.attn_prefill_two_stage if two_stage else sab.attn_prefill
    for n, (hi, (o_h, l_h)) in enumerate(zip(host_in, outs)):
        d = {x: hi[x].cuda() for x in hi}
        o_ref, l_ref = prefill(plan, d["q"], d["k"], d["v"])
        torch.cuda.synchronize()
        assert torch.equal(o_h.view(torch.int16), o_ref.cpu().view(torch.int16)), (name, n)
        assert torch.equal(l_h, l_ref.cpu()), (name, n)
    plan.close()


def test_pipeline_rejects_pageable_host_memory():
    from sequence_approximate_attention_b200.pipeline import HostPrefillPipeline

    cfg = CASES["tiny_text40"]
    g = generate(cfg)
    plan = make_plan(sab, cfg, g["host_sizes"])
    pipe = HostPrefillPipeline(plan)
    qs, ks = plan.qkv_shapes()
    q = torch.zeros(qs, dtype=torch.bfloat16)  # pageable
    k = torch.zeros(ks, dtype=torch.bfloat16).pin_memory()
    o = torch.empty(qs, dtype=torch.bfloat16).pin_memory()
    lse = torch.empty((plan.hq, plan.n_total), dtype=torch.float32).pin_memory()
    with pytest.raises(ValueError, match="pinned"):
        pipe.submit(q, k, k, o, lse)
    plan.close()
