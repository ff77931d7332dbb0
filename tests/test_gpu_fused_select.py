"""The prefill's one-launch scoring + selection + gather (spava_plan_set_fused_select,
ssg_kernel.cuh) against the two-kernel path (score kernel, then select + gather) and
the fp64 oracle.

* Scores, indices, O and lse of the two paths are bit-identical: the fused launch
  computes the same maxima and applies the same selection rule, and the attention
  pass that follows is deterministic, so any wrong gathered row would show in O.
* The selection equals the oracle's selection run on the GPU's fp32 scores, bit for
  bit, also with many exactly tied scores (duplicated key rows) cut by the P-th place.
* Shapes cover many small units spread over many CTAs, probe queries in two chunks
  (G = 7), candidate runs longer than the 8192 keys the worker threads hold in
  registers, P = 1 with an odd anchor, and P equal to whole blocks.
* Repeated calls on one workspace give the same result (the unit counters are
  cleared by every call).
* With the load thread told to issue nothing, every wait of the launch (MMA issuers,
  epilogue, publisher, worker group) runs out: the call reports SPAVA_ERR_TIMEOUT and
  the plan then runs correctly.
"""

import math

import numpy as np
import pytest
import torch

from oracle import spava_oracle as orc
from workloads import CONFIGS

from .helpers import compare_attention, inputs, make_plan, score_tolerance, to_device_bf16

# The fused launch's CTAs wait on one another (bounded, 2 s per wait); a test that ran
# far past that would mean a wait the kernel cannot bound, so it is ended rather than
# left to block the rest of the suite.
pytestmark = [pytest.mark.gpu, pytest.mark.timeout(300, method="thread")]

sab = pytest.importorskip("sequence_approximate_attention_b200")

TINY = CONFIGS["tiny"]

CASES = {
    # 15 x 4 units of 2 tiles each: about one score tile per CTA, gather tasks everywhere
    "many_units_d64": TINY.with_(n_visual=4096, n_hosts=16, hq=8, hkv=4, head_dim=64, anchor=32, passing=64,
                                 probe_r=32, n_text=12, seed=31),
    # G = 7, R = 64: two probe chunks of 32 tokens (224 MMA columns), two query buffers
    "d128_g7_two_chunks": TINY.with_(n_visual=1536, n_hosts=3, head_dim=128, hq=14, hkv=2, anchor=64,
                                     passing=96, probe_r=64, n_text=7, kv_kind="frame", frame=64,
                                     salient_frac=0.05, seed=32),
    # 9216 candidates per unit: the selection re-reads scores from L2 on every pass
    "long_blocks": TINY.with_(n_visual=27648, n_hosts=3, hq=2, hkv=1, head_dim=64, anchor=0, passing=700,
                              probe_r=16, n_text=0, seed=33),
    "p1_odd_anchor": TINY.with_(n_visual=1024, n_hosts=4, passing=1, anchor=5, n_text=3, seed=34),
    "p_whole_block": TINY.with_(n_visual=512, n_hosts=4, anchor=0, passing=128, n_text=9, seed=35),
    "d128_p1024": TINY.with_(n_visual=8192, n_hosts=4, head_dim=128, hq=8, hkv=2, anchor=512, passing=1024,
                             probe_r=64, n_text=0, seed=36),
}


def _run(plan, dev, fused, ws):
    plan.set_fused_select(fused)
    scores = torch.full(plan.scores_shape(), float("nan"), device="cuda")
    idx = torch.full(plan.idx_shape(), -1, dtype=torch.int32, device="cuda")
    o, lse = sab.attn_prefill(plan, dev["q"], dev["k"], dev["v"], scores_out=scores, idx_out=idx, workspace=ws)
    sab.check_device_error(plan, ws)
    torch.cuda.synchronize()
    return scores, idx, o, lse


def _check_against_three_launch(cfg, dev, f64, sizes):
    plan = make_plan(sab, cfg, sizes)
    off = orc.host_offsets(sizes)
    H = cfg.n_hosts
    n_sc = int(off[H - 1])
    ws = plan.new_workspace()
    s1, i1, o1, l1 = _run(plan, dev, True, ws)
    s0, i0, o0, l0 = _run(plan, dev, False, ws)
    a, b = s1[:, :n_sc].cpu().numpy(), s0[:, :n_sc].cpu().numpy()
    np.testing.assert_array_equal(a.view(np.uint32), b.view(np.uint32))
    sel = i1.cpu().numpy().astype(np.int64)
    np.testing.assert_array_equal(sel, i0.cpu().numpy())
    np.testing.assert_array_equal(sel, orc.select_passing(s1.cpu().numpy(), off, cfg.anchor, cfg.passing))
    assert torch.equal(o1.view(torch.int16), o0.view(torch.int16))
    assert torch.equal(l1, l0)
    # the same workspace again: counters and flags start from zero on every call
    s2, i2, o2, l2 = _run(plan, dev, True, ws)
    assert torch.equal(i2, i1) and torch.equal(o2.view(torch.int16), o1.view(torch.int16))
    plan.close()
    return s1, sel, o1, l1, off


@pytest.mark.parametrize("name", list(CASES))
def test_fused_equals_three_launch_and_oracle(name):
    cfg = CASES[name].with_(uneven=None)
    g, f64, dev = inputs(cfg)
    sizes = g["host_sizes"]
    scores, sel, o, lse, off = _check_against_three_launch(cfg, dev, f64, sizes)
    scale = 1.0 / math.sqrt(cfg.head_dim)
    n_sc = int(off[cfg.n_hosts - 1])
    ref = orc.probe_scores(f64["q"], f64["k"], off, cfg.probe_r, scale)
    tol = score_tolerance(f64["q"], f64["k"], off, cfg.probe_r, scale)
    err = np.abs(scores.cpu().numpy()[:, :n_sc] - ref[:, :n_sc])
    assert (err <= tol[:, :n_sc]).all(), f"score error {err.max()}"
    if cfg.n_visual * cfg.hq <= 1 << 15:
        O_ref, L_ref = orc.approx_attention(f64["q"], f64["k"], f64["v"], off, cfg.anchor, sel, scale)
        compare_attention(o, lse, O_ref, L_ref, name)


@pytest.mark.parametrize("dup", [2, 4, 16])
def test_fused_selection_with_exact_ties(dup):
    """Key rows repeated in runs of `dup`: every run scores identically wherever all its
    keys see the same probe rows, so the P-th place falls inside tie groups; the fused
    selection must take the lowest indices of a tied group, as the oracle does."""
    cfg = TINY.with_(n_visual=2048, n_hosts=4, hq=4, hkv=2, head_dim=64, anchor=16, passing=100, probe_r=16,
                     n_text=0, seed=40 + dup)
    g, f64, dev = inputs(cfg)
    kb = g["k"].copy()
    n = cfg.n_visual
    src = (np.arange(n) // dup) * dup
    kb[:n] = kb[src]
    dev["k"] = to_device_bf16(kb)
    f64["k"] = orc.bf16_bits_to_f64(kb)
    scores, sel, _, _, off = _check_against_three_launch(cfg, dev, f64, g["host_sizes"])
    sc = scores.cpu().numpy()
    # ties were really exercised: some P-th score occurs more than once in its block
    tied = 0
    for h in range(cfg.n_hosts - 1):
        lo = int(off[h]) + (cfg.anchor if h == 0 else 0)
        for r in range(cfg.hkv):
            seg = np.sort(sc[r, lo:int(off[h + 1])])[::-1]
            tied += int(np.sum(seg == seg[cfg.passing - 1]) > 1)
    assert tied > 0


def test_fused_bounded_waits_report_timeout():
    cfg = TINY.with_(n_visual=2048, n_hosts=4, hq=4, hkv=2, head_dim=64, anchor=16, passing=64, probe_r=16,
                     n_text=5, seed=50)
    g, f64, dev = inputs(cfg)
    plan = make_plan(sab, cfg, g["host_sizes"])
    plan.set_fused_select(True)
    ws = plan.new_workspace()
    plan.set_debug(wait_limit_ns=20_000_000, stall_producer=True)
    sab.attn_prefill(plan, dev["q"], dev["k"], dev["v"], workspace=ws)
    with pytest.raises(sab.SpavaError) as ei:
        sab.check_device_error(plan, ws)
    assert ei.value.status == 4
    plan.set_debug(0, False)
    idx = torch.empty(plan.idx_shape(), dtype=torch.int32, device="cuda")
    o, lse = sab.attn_prefill(plan, dev["q"], dev["k"], dev["v"], idx_out=idx, workspace=ws)
    sab.check_device_error(plan, ws)
    off = orc.host_offsets(g["host_sizes"])
    O_ref, L_ref = orc.approx_attention(f64["q"], f64["k"], f64["v"], off, cfg.anchor,
                                        idx.cpu().numpy().astype(np.int64), 1 / math.sqrt(cfg.head_dim))
    compare_attention(o, lse, O_ref, L_ref, "fused, after timeout")
    plan.close()
