"""spava_attn_prefill_noalloc: the prefill for callers that cannot allocate device
memory when they call (their device memory is owned by a pooling allocator, they run
under a hard memory cap, or their interface has no way to pass a workspace).  It
keeps its scratch in a static device array inside the library instead of a
caller-provided workspace.

Checked through the C ABI: two calls in a row must both agree with the workspace
entry point (spava_attn_prefill) within the parity tolerances, and a plan whose
scratch does not fit the static array is refused before anything is enqueued.
This file is collected last on purpose; it must pass alone and after the others.
"""

import ctypes

import pytest
import torch

from workloads import CONFIGS

from .helpers import LSE_TOL, O_TOL, inputs, make_plan

pytestmark = pytest.mark.gpu

sab = pytest.importorskip("sequence_approximate_attention_b200")

TINY = CONFIGS["tiny"]
CASES = {
    "tiny_text40": (TINY.with_(n_text=40), None),
    "d128_g7_uneven": (TINY.with_(n_visual=1024, n_hosts=4, head_dim=128, hq=14, hkv=2, anchor=64, passing=64,
                                  probe_r=32, n_text=77, kv_kind="frame", frame=64, seed=7),
                       [192, 320, 256, 256]),
}


def _p(t):
    return ctypes.c_void_p(t.data_ptr())


@pytest.mark.parametrize("name", list(CASES))
def test_noalloc_matches_workspace_entry_point(name):
    cfg, sizes = CASES[name]
    g, _, dev = inputs(cfg)
    plan = make_plan(sab, cfg, sizes if sizes is not None else g["host_sizes"])
    lib = plan.lib
    assert plan.workspace_bytes <= lib_limit()
    o_ref, lse_ref = sab.attn_prefill(plan, dev["q"], dev["k"], dev["v"])
    torch.cuda.synchronize()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for call in range(2):
        o = torch.full_like(o_ref, float("nan"))
        lse = torch.full_like(lse_ref, float("nan"))
        st = lib.spava_attn_prefill_noalloc(plan.handle, _p(dev["q"]), _p(dev["k"]), _p(dev["v"]), _p(o),
                                            _p(lse), stream)
        assert st == 0, lib.spava_last_error().decode()
        torch.cuda.synchronize()
        do = (o.float() - o_ref.float()).abs().max().item()
        dl = (lse - lse_ref).abs().max().item()
        assert do <= O_TOL and dl <= LSE_TOL, (name, call, do, dl)
    plan.close()


def lib_limit():
    return 32 * 1024 * 1024


def test_noalloc_refuses_plans_beyond_the_static_scratch():
    cfg = CONFIGS["128k"]
    plan = sab.Plan(cfg.n_visual, cfg.n_text, cfg.n_hosts, None, cfg.anchor, cfg.passing, cfg.probe_r,
                    cfg.hq, cfg.hkv, cfg.head_dim)
    assert plan.workspace_bytes > lib_limit()
    dummy = torch.zeros(1024, dtype=torch.bfloat16, device="cuda")
    st = plan.lib.spava_attn_prefill_noalloc(plan.handle, _p(dummy), _p(dummy), _p(dummy), _p(dummy), _p(dummy),
                                             None)
    assert st == 2
    msg = plan.lib.spava_last_error().decode()
    assert "static scratch" in msg and str(plan.workspace_bytes) in msg
    plan.close()
