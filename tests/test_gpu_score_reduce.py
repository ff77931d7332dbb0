"""GPU parity of the switchable head reduction of the probe scores (sum and mean of the
per-head maxima beside the default max, and per-query-head selection), through
spava_plan_set_score_reduce.

Standalone scoring (spava_score_select) and both prefill flows (the score kernel, and
the fused local-pass scores of the two-stage flow) against the fp64 oracle with the
same ``head_reduce``: scores within G times the per-head tolerance for the sum (the
per-head errors add) and within it for the mean; selection bit-exact on the GPU's own
fp32 scores and near-tie-only against the fp64 scores; O/lse against the oracle re-run
with the GPU's indices.  The cases cover G = 2, 7 (one 224-column chunk) and 16 with
R = 128 (eight 16-row probe chunks).
"""

import math

import numpy as np
import pytest
import torch

from oracle import spava_oracle as orc
from workloads import CONFIGS

from .helpers import adversarial_scores, check_selection_vs_fp64, compare_attention, inputs, make_plan, score_tolerance

pytestmark = pytest.mark.gpu

sab = pytest.importorskip("sequence_approximate_attention_b200")

TINY = CONFIGS["tiny"]
CASES = {
    "tiny": (TINY, None),
    "tiny_h8": (TINY.with_(n_hosts=8, anchor=16, passing=16, probe_r=16), None),
    "d128_g7_uneven": (TINY.with_(n_visual=1024, n_hosts=4, head_dim=128, hq=14, hkv=2, anchor=64,
                                  passing=64, probe_r=32, n_text=77, kv_kind="frame", frame=64,
                                  salient_frac=0.05, seed=7), [192, 320, 256, 256]),
    "d128_g16_r128": (TINY.with_(n_visual=768, n_hosts=3, head_dim=128, hq=16, hkv=1, anchor=32,
                                 passing=96, probe_r=128, n_text=0, seed=9), None),
}


def _setup(name, mode):
    cfg, sizes = CASES[name]
    cfg = cfg.with_(uneven=None)
    g, f64, dev = inputs(cfg)
    sizes = np.asarray(sizes if sizes is not None else g["host_sizes"], dtype=np.int32)
    plan = make_plan(sab, cfg, sizes)
    plan.set_score_reduce(mode)
    off = orc.host_offsets(sizes)
    scale = 1.0 / math.sqrt(cfg.head_dim)
    per_head = mode == "per_query_head"
    ref = orc.probe_scores(f64["q"], f64["k"], off, cfg.probe_r, scale, head_reduce="none" if per_head else mode)
    G = cfg.hq // cfg.hkv
    tol = score_tolerance(f64["q"], f64["k"], off, cfg.probe_r, scale) * (G if mode == "sum" else 1)
    if per_head:
        tol = np.repeat(tol, G, axis=0)   # the group's bound holds for each of its heads
    return cfg, f64, dev, plan, off, scale, ref, tol


@pytest.mark.parametrize("mode", ["sum", "mean", "per_query_head"])
@pytest.mark.parametrize("name", list(CASES))
def test_score_select_head_reduce(name, mode):
    cfg, f64, dev, plan, off, scale, ref, tol = _setup(name, mode)
    scores, idx = sab.score_select(plan, dev["q"], dev["k"])
    torch.cuda.synchronize()
    sc = scores.cpu().numpy()
    err = np.abs(sc - ref)
    assert (err <= tol).all(), (name, mode, float(err.max()))
    np.testing.assert_array_equal(idx.cpu().numpy(), orc.select_passing(sc, off, cfg.anchor, cfg.passing))
    plan.close()


@pytest.mark.parametrize("two_stage", [False, True])
@pytest.mark.parametrize("mode", ["sum", "mean", "per_query_head"])
@pytest.mark.parametrize("name", list(CASES))
def test_prefill_head_reduce(name, mode, two_stage):
    cfg, f64, dev, plan, off, scale, ref, tol = _setup(name, mode)
    ws = plan.new_workspace(two_stage=two_stage)
    scores = torch.full(plan.scores_shape(), float("nan"), device="cuda")
    idx = torch.full(plan.idx_shape(), -1, dtype=torch.int32, device="cuda")
    prefill = sab.attn_prefill_two_stage if two_stage else sab.attn_prefill
    o, lse = prefill(plan, dev["q"], dev["k"], dev["v"], scores_out=scores, idx_out=idx, workspace=ws)
    sab.check_device_error(plan, ws)
    torch.cuda.synchronize()
    n_sc = int(off[cfg.n_hosts - 1])
    sc = scores.cpu().numpy()
    err = np.abs(sc[:, :n_sc] - ref[:, :n_sc])
    assert (err <= tol[:, :n_sc]).all(), (name, mode, two_stage, float(np.nanmax(err)))
    sel = idx.cpu().numpy().astype(np.int64)
    np.testing.assert_array_equal(sel, orc.select_passing(sc, off, cfg.anchor, cfg.passing))
    check_selection_vs_fp64(sel, ref, off, cfg.anchor, cfg.passing)
    O_ref, L_ref = orc.approx_attention(f64["q"], f64["k"], f64["v"], off, cfg.anchor, sel, scale)
    compare_attention(o, lse, O_ref, L_ref, f"{name} {mode} two_stage={two_stage}")
    plan.close()


def test_unknown_mode_is_refused():
    cfg, sizes = CASES["tiny"]
    g, _, _ = inputs(cfg)
    plan = make_plan(sab, cfg, g["host_sizes"])
    with pytest.raises(ValueError):
        plan.set_score_reduce("median")
    assert plan.lib.spava_plan_set_score_reduce(plan.handle, 7) == 1   # SPAVA_ERR_INVALID_ARG
    plan.close()


@pytest.mark.parametrize("name", ["tiny", "d128_g7_uneven"])
def test_gather_per_query_head(name):
    """Standalone gather with one selection row per query head: k_pass[c][h][j] =
    k[idx[h][c][j]][c // G], byte for byte."""
    cfg, f64, dev, plan, off, scale, ref, tol = _setup(name, "per_query_head")
    G = cfg.hq // cfg.hkv
    scores, idx = sab.score_select(plan, dev["q"], dev["k"])
    kp, vp = sab.gather_passing(plan, dev["k"], dev["v"], idx)
    torch.cuda.synchronize()
    idx_h = idx.cpu().numpy()
    k16, v16 = dev["k"].cpu().view(torch.int16), dev["v"].cpu().view(torch.int16)
    kp16, vp16 = kp.cpu().view(torch.int16), vp.cpu().view(torch.int16)
    assert kp.shape == (cfg.hq, cfg.n_hosts - 1, cfg.passing, cfg.head_dim)
    for c in range(cfg.hq):
        for h in range(cfg.n_hosts - 1):
            rows = torch.from_numpy(idx_h[h, c].astype(np.int64))
            assert torch.equal(kp16[c, h], k16[rows, c // G]), (name, c, h)
            assert torch.equal(vp16[c, h], v16[rows, c // G]), (name, c, h)
    plan.close()


@pytest.mark.parametrize("sizes,anchor,passing", [([8192] * 3, 1024, 1024), ([300, 500, 224], 10, 290),
                                                  ([1000, 24], 0, 1)])
def test_per_query_head_select_bit_exact_with_ties(sizes, anchor, passing):
    """Selection rows per query head (hq = 8 rows of scores) through the given-scores
    path, on adversarial scores (exact ties, +-0, huge values, a near-equal ramp):
    bit-exact against the oracle's selection of the same fp32 scores."""
    rng = np.random.default_rng(len(sizes) * 7 + passing)
    hq, hkv = 8, 2
    N = int(sum(sizes))
    cfg = TINY.with_(n_visual=N, n_hosts=len(sizes), anchor=anchor, passing=passing, probe_r=16,
                     hq=hq, hkv=hkv, head_dim=64)
    plan = make_plan(sab, cfg, sizes)
    plan.set_score_reduce("per_query_head")
    s = adversarial_scores(rng, hq, N)
    scores = torch.from_numpy(s).cuda()
    _, idx = sab.score_select(plan, None, None, scores=scores, scores_given=True)
    torch.cuda.synchronize()
    off = orc.host_offsets(sizes)
    assert idx.shape == (len(sizes) - 1, hq, passing)
    np.testing.assert_array_equal(idx.cpu().numpy(), orc.select_passing(s, off, anchor, passing))
    plan.close()
