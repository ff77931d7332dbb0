"""GPU parity of probability scores (spava_plan_set_score_kind "prob"): each probe
row's attention probability over the keys of its own block it sees, then the max over
probe rows and the head reduction, in the standalone scoring and in both prefill flows.

Scores are compared in the log domain: |log p_gpu - log p_oracle| stays within the
logit tolerance (fp32 accumulation of exact bf16 products) plus 5e-4 for the probe
row's lse, which the attention kernel computes in fp32; the sum over heads keeps the
same relative bound.  Selection: bit-exact on the GPU's own fp32 scores; against the
fp64 scores a swap is allowed only between keys within that relative bound of the
P-th best score.  O/lse against the oracle re-run with the GPU's indices.
"""

import math

import numpy as np
import pytest
import torch

from oracle import spava_oracle as orc
from workloads import CONFIGS

from .helpers import compare_attention, inputs, make_plan, score_tolerance

pytestmark = pytest.mark.gpu

sab = pytest.importorskip("sequence_approximate_attention_b200")

TINY = CONFIGS["tiny"]
CASES = {
    "tiny": (TINY, None),
    "d128_g7_uneven": (TINY.with_(n_visual=1024, n_hosts=4, head_dim=128, hq=14, hkv=2, anchor=64,
                                  passing=64, probe_r=32, n_text=77, kv_kind="frame", frame=64,
                                  salient_frac=0.05, seed=7), [192, 320, 256, 256]),
    "d128_g16_r128": (TINY.with_(n_visual=768, n_hosts=3, head_dim=128, hq=16, hkv=1, anchor=32,
                                 passing=96, probe_r=128, n_text=0, seed=9), None),
}
LSE_ERR = 5e-4


def _setup(name, mode):
    cfg, sizes = CASES[name]
    cfg = cfg.with_(uneven=None)
    g, f64, dev = inputs(cfg)
    sizes = np.asarray(sizes if sizes is not None else g["host_sizes"], dtype=np.int32)
    plan = make_plan(sab, cfg, sizes)
    plan.set_score_reduce(mode)
    plan.set_score_kind("prob")
    off = orc.host_offsets(sizes)
    scale = 1.0 / math.sqrt(cfg.head_dim)
    per_head = mode == "per_query_head"
    ref = orc.probe_scores(f64["q"], f64["k"], off, cfg.probe_r, scale,
                           head_reduce="none" if per_head else mode, score_kind="prob")
    G = cfg.hq // cfg.hkv
    tol_log = score_tolerance(f64["q"], f64["k"], off, cfg.probe_r, scale) + LSE_ERR
    if per_head:
        tol_log = np.repeat(tol_log, G, axis=0)   # the group's bound holds for each of its heads
    return cfg, f64, dev, plan, off, scale, ref, tol_log


def _check_scores(sc, ref, tol_log, cols, what):
    assert np.isfinite(sc[:, cols]).all() and (sc[:, cols] > 0).all(), what
    err = np.abs(np.log(sc[:, cols].astype(np.float64)) - np.log(ref[:, cols]))
    assert (err <= tol_log[:, cols]).all(), (what, float(err.max()))


def _check_selection_relative(sel, ref, off, anchor, passing, rel):
    want = orc.select_passing(ref, off, anchor, passing)
    for h in range(want.shape[0]):
        lo = int(off[h]) + (anchor if h == 0 else 0)
        hi = int(off[h + 1])
        for g in range(want.shape[1]):
            a, b = set(want[h, g].tolist()), set(sel[h, g].tolist())
            if a == b:
                continue
            pth = np.sort(ref[g, lo:hi])[::-1][passing - 1]
            for j in a ^ b:
                assert abs(ref[g, j] - pth) <= rel * pth, (h, g, j, ref[g, j], pth)


@pytest.mark.parametrize("mode", ["max", "sum", "per_query_head"])
@pytest.mark.parametrize("name", list(CASES))
def test_prob_score_select(name, mode):
    cfg, f64, dev, plan, off, scale, ref, tol_log = _setup(name, mode)
    scores, idx = sab.score_select(plan, dev["q"], dev["k"])
    torch.cuda.synchronize()
    sc = scores.cpu().numpy()
    _check_scores(sc, ref, tol_log, slice(0, cfg.n_visual), (name, mode))
    np.testing.assert_array_equal(idx.cpu().numpy(), orc.select_passing(sc, off, cfg.anchor, cfg.passing))
    plan.close()


@pytest.mark.parametrize("two_stage", [False, True])
@pytest.mark.parametrize("mode", ["max", "sum", "per_query_head"])
@pytest.mark.parametrize("name", list(CASES))
def test_prob_prefill(name, mode, two_stage):
    cfg, f64, dev, plan, off, scale, ref, tol_log = _setup(name, mode)
    ws = plan.new_workspace(two_stage=two_stage)
    scores = torch.full(plan.scores_shape(), float("nan"), device="cuda")
    idx = torch.full(plan.idx_shape(), -1, dtype=torch.int32, device="cuda")
    prefill = sab.attn_prefill_two_stage if two_stage else sab.attn_prefill
    o, lse = prefill(plan, dev["q"], dev["k"], dev["v"], scores_out=scores, idx_out=idx, workspace=ws)
    sab.check_device_error(plan, ws)
    torch.cuda.synchronize()
    n_sc = int(off[cfg.n_hosts - 1])
    sc = scores.cpu().numpy()
    _check_scores(sc, ref, tol_log, slice(0, n_sc), (name, mode, two_stage))
    sel = idx.cpu().numpy().astype(np.int64)
    np.testing.assert_array_equal(sel, orc.select_passing(sc, off, cfg.anchor, cfg.passing))
    _check_selection_relative(sel, ref, off, cfg.anchor, cfg.passing, rel=2 * float(tol_log.max()))
    O_ref, L_ref = orc.approx_attention(f64["q"], f64["k"], f64["v"], off, cfg.anchor, sel, scale)
    compare_attention(o, lse, O_ref, L_ref, f"{name} prob {mode} two_stage={two_stage}")
    plan.close()
