"""Shared helpers for the parity tests: seeded inputs on the device and the
acceptance checks (selection, O, lse) against the oracle."""

import math

import numpy as np
import torch

from oracle import spava_oracle as orc
from workloads import generate

O_TOL = 2e-2      # max |dO| (bf16 output vs fp64 oracle)
LSE_TOL = 1e-3    # max |dlse|
SWAP_GAP = 1e-4   # a selection may differ only where the P-th/(P+1)-th oracle scores are this close


def to_device_bf16(bits: np.ndarray, device="cuda") -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).to(device).view(torch.bfloat16)


def make_plan(sab, cfg, host_sizes):
    return sab.Plan(cfg.n_visual, cfg.n_text, cfg.n_hosts, list(map(int, host_sizes)), cfg.anchor,
                    cfg.passing, cfg.probe_r, cfg.hq, cfg.hkv, cfg.head_dim)


def inputs(cfg, seed=None):
    g = generate(cfg, seed=seed)
    f64 = {x: orc.bf16_bits_to_f64(g[x]) for x in ("q", "k", "v")}
    dev = {x: to_device_bf16(g[x]) for x in ("q", "k", "v")}
    return g, f64, dev


def score_tolerance(q64, k64, off, probe_r, scale):
    """|d score| bound for fp32 accumulation of exact bf16 products: 1e-5 * scale *
    max over the probe (row, head) of sum_t |q_t k_t| (plus a tiny floor)."""
    hq, hkv = q64.shape[1], k64.shape[1]
    G = hq // hkv
    tol = np.empty((hkv, int(off[-1])))
    for h in range(len(off) - 1):
        a, e = int(off[h]), int(off[h + 1])
        for g in range(hkv):
            qa = np.abs(q64[e - probe_r:e, g * G:(g + 1) * G, :]).reshape(-1, q64.shape[2])
            ka = np.abs(k64[a:e, g, :])
            tol[g, a:e] = (ka @ qa.T).max(axis=1)
    return 1e-5 * scale * tol + 1e-6


def check_selection_vs_fp64(sel_gpu, scores64, off, anchor, passing):
    """GPU selection may differ from the fp64 oracle's only at near-ties: every
    differing key must score within SWAP_GAP of the P-th best oracle score."""
    ref = orc.select_passing(scores64, off, anchor, passing)
    n_diff = 0
    for h in range(ref.shape[0]):
        lo = int(off[h]) + (anchor if h == 0 else 0)
        hi = int(off[h + 1])
        for g in range(ref.shape[1]):
            a, b = set(ref[h, g].tolist()), set(sel_gpu[h, g].tolist())
            if a == b:
                continue
            s = np.sort(scores64[g, lo:hi])[::-1]
            pth = s[passing - 1]
            for j in a ^ b:
                assert abs(scores64[g, j] - pth) < SWAP_GAP, (h, g, j, scores64[g, j], pth)
            n_diff += len(a ^ b) // 2
    return n_diff


def compare_attention(o_gpu, lse_gpu, O_ref, L_ref, what=""):
    o = o_gpu.float().cpu().numpy().astype(np.float64)
    lse = lse_gpu.float().cpu().numpy().astype(np.float64)
    assert np.isfinite(o).all() and np.isfinite(lse).all(), what
    do = np.abs(o - O_ref).max()
    dl = np.abs(lse - L_ref).max()
    assert do <= O_TOL, f"{what}: max |dO| = {do}"
    assert dl <= LSE_TOL, f"{what}: max |dlse| = {dl}"
    return do, dl


def default_scale(cfg):
    return 1.0 / math.sqrt(cfg.head_dim)


def adversarial_scores(rng, rows, N):
    """fp32 scores [rows, N] built to break a selection: heavy exact ties, +-0, one row
    all equal, values near the fp32 limits, and a ramp whose steps are one or two ulps."""
    s = rng.integers(-4, 5, size=(rows, N)).astype(np.float32)   # heavy exact ties
    s[0, ::7] = -0.0
    s[0, 3::7] = 0.0
    if rows > 1:
        s[1] = 2.5                                               # all equal
    if rows > 2:
        s[2] = rng.standard_normal(N).astype(np.float32) * np.float32(1e30)
        s[2, 100:110] = np.float32(3.0e38)
        s[2, 200:210] = np.float32(-3.0e38)
    if rows > 3:
        s[3] = np.float32(1.0) + np.arange(N, dtype=np.float32) * np.float32(1e-7)  # near-equal ramp
    return s
