"""spava_attn_prefill_noalloc: the prefill for callers that cannot allocate device
memory when they call (their device memory is owned by a pooling allocator, they run
under a hard memory cap, or their interface has no way to pass a workspace).  It
keeps its scratch in a static device array inside the library instead of a
caller-provided workspace.

Checked through the C ABI:
  * two calls in a row agree with the workspace entry point (spava_attn_prefill)
    within the parity tolerances, and with the fp64 oracle re-run with the
    selection the workspace entry point made;
  * between those two calls another plan, with a different layout of the shared
    array (other H, d, head counts and text length), runs through the same array:
    the second call must still be right, so whatever has to start at zero is
    cleared by the call itself, not left over from the previous call;
  * a call allocates nothing: after a warm-up call, neither torch's allocator nor
    the device's free memory moves across a call;
  * a plan whose scratch does not fit the static array is refused before anything
    is enqueued.  The limit is read from include/spava.h.
This file is collected last on purpose; it must pass alone and after the others.
"""

import ctypes
import math
import os
import re

import numpy as np
import pytest
import torch

from oracle import spava_oracle as orc
from workloads import CONFIGS

from .helpers import LSE_TOL, O_TOL, compare_attention, inputs, make_plan

pytestmark = pytest.mark.gpu

sab = pytest.importorskip("sequence_approximate_attention_b200")

TINY = CONFIGS["tiny"]
CASES = {
    "tiny_text40": (TINY.with_(n_text=40), None),
    "d128_g7_uneven": (TINY.with_(n_visual=1024, n_hosts=4, head_dim=128, hq=14, hkv=2, anchor=64, passing=64,
                                  probe_r=32, n_text=77, kv_kind="frame", frame=64, seed=7),
                       [192, 320, 256, 256]),
}
OTHER = {"tiny_text40": "d128_g7_uneven", "d128_g7_uneven": "tiny_text40"}

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "spava.h")


def lib_limit():
    """SPAVA_NOALLOC_SCRATCH_BYTES as the header defines it."""
    text = open(HEADER).read()
    m = re.search(r"#define\s+SPAVA_NOALLOC_SCRATCH_BYTES\s+\((\d+)u\s*\*\s*(\d+)u\s*\*\s*(\d+)u\)", text)
    assert m, "SPAVA_NOALLOC_SCRATCH_BYTES not found in include/spava.h"
    return int(m.group(1)) * int(m.group(2)) * int(m.group(3))


def _p(t):
    return ctypes.c_void_p(t.data_ptr())


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


class Case:
    """A plan with its inputs, the workspace entry point's output and selection, and
    the oracle's output for that selection."""

    def __init__(self, name):
        cfg, sizes = CASES[name]
        self.name = name
        g, f64, self.dev = inputs(cfg)
        sizes = sizes if sizes is not None else g["host_sizes"]
        self.plan = make_plan(sab, cfg, sizes)
        assert self.plan.workspace_bytes <= lib_limit()
        idx = torch.full(self.plan.idx_shape(), -1, dtype=torch.int32, device="cuda")
        self.o_ref, self.lse_ref = sab.attn_prefill(self.plan, self.dev["q"], self.dev["k"], self.dev["v"],
                                                    idx_out=idx)
        torch.cuda.synchronize()
        off = orc.host_offsets(np.asarray(sizes, dtype=np.int64))
        self.O_orc, self.L_orc = orc.approx_attention(f64["q"], f64["k"], f64["v"], off, cfg.anchor,
                                                      idx.cpu().numpy().astype(np.int64),
                                                      1.0 / math.sqrt(cfg.head_dim))

    def call(self):
        o = torch.full_like(self.o_ref, float("nan"))
        lse = torch.full_like(self.lse_ref, float("nan"))
        st = self.plan.lib.spava_attn_prefill_noalloc(self.plan.handle, _p(self.dev["q"]), _p(self.dev["k"]),
                                                      _p(self.dev["v"]), _p(o), _p(lse), _stream())
        assert st == 0, self.plan.lib.spava_last_error().decode()
        torch.cuda.synchronize()
        return o, lse

    def check(self, o, lse, what):
        do = (o.float() - self.o_ref.float()).abs().max().item()
        dl = (lse - self.lse_ref).abs().max().item()
        assert do <= O_TOL and dl <= LSE_TOL, (self.name, what, do, dl)
        compare_attention(o, lse, self.O_orc, self.L_orc, f"{self.name} {what} vs oracle")

    def close(self):
        self.plan.close()


@pytest.mark.parametrize("name", list(CASES))
def test_noalloc_matches_workspace_entry_point_and_oracle(name):
    case, other = Case(name), Case(OTHER[name])
    o, lse = case.call()
    case.check(o, lse, "first call")
    # another layout of the shared array in between
    o2, lse2 = other.call()
    other.check(o2, lse2, "interleaved call")
    o, lse = case.call()
    case.check(o, lse, "second call")
    case.close()
    other.close()


def test_noalloc_allocates_nothing():
    case = Case("d128_g7_uneven")
    case.call()  # warm-up: loads the module's kernels, sets their shared-memory limits
    torch.cuda.synchronize()
    alloc0 = torch.cuda.memory_allocated()
    free0, _ = torch.cuda.mem_get_info()
    o = torch.empty_like(case.o_ref)
    lse = torch.empty_like(case.lse_ref)
    torch.cuda.synchronize()
    alloc1 = torch.cuda.memory_allocated()
    free1, _ = torch.cuda.mem_get_info()
    for _ in range(2):
        st = case.plan.lib.spava_attn_prefill_noalloc(case.plan.handle, _p(case.dev["q"]), _p(case.dev["k"]),
                                                      _p(case.dev["v"]), _p(o), _p(lse), _stream())
        assert st == 0, case.plan.lib.spava_last_error().decode()
    torch.cuda.synchronize()
    assert torch.cuda.memory_allocated() == alloc1
    free2, _ = torch.cuda.mem_get_info()
    assert free2 == free1, (free0, free1, free2)
    assert alloc1 >= alloc0
    case.check(o, lse, "no-allocation call")
    case.close()


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
    assert "static scratch" in msg and str(plan.workspace_bytes) in msg and str(lib_limit()) in msg
    plan.close()
