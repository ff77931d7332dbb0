"""Pins for the fp64 oracle (CPU only).

The pages print no worked example and no formula, so the oracle is pinned to
things outside itself:
  * hand-derived prefills (tests/golden/hand_examples.json);
  * one host degenerates to standard causal attention (APB-V "Limitations"),
    checked against torch's scaled_dot_product_attention in fp64;
  * passing everything (P = B, A = 0) also equals dense causal attention;
  * A = 0, P = 0 equals block-diagonal causal attention (torch SDPA with an
    explicit mask);
  * a second formulation with an explicit (tokens x tokens) visibility mask;
  * brute-force selection and scoring in pure Python on tiny inputs;
  * lse-merge associativity, and output sanity bounds.
"""

import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import spava_oracle as orc
from workloads import CONFIGS, bf16_round_bits, generate, host_sizes_for

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "hand_examples.json")


def _rand_qkv(rng, NT, hq, hkv, d):
    q = rng.standard_normal((NT, hq, d))
    k = rng.standard_normal((NT, hkv, d))
    v = rng.standard_normal((NT, hkv, d))
    return q, k, v


def _sdpa(q, k, v, scale, mask=None, causal=False):
    """torch SDPA (fp64, CPU) on [tokens, heads, d] with GQA by repeat."""
    hq, hkv = q.shape[1], k.shape[1]
    G = hq // hkv
    Q = torch.from_numpy(q).permute(1, 0, 2)
    K = torch.from_numpy(k).permute(1, 0, 2).repeat_interleave(G, dim=0)
    V = torch.from_numpy(v).permute(1, 0, 2).repeat_interleave(G, dim=0)
    m = None if mask is None else torch.from_numpy(mask)
    o = torch.nn.functional.scaled_dot_product_attention(Q, K, V, attn_mask=m, is_causal=causal,
                                                         scale=scale)
    return o.permute(1, 0, 2).numpy()


def _lse_from_mask(q, k, scale, mask):
    hq, hkv = q.shape[1], k.shape[1]
    G = hq // hkv
    out = np.empty((hq, q.shape[0]))
    for c in range(hq):
        s = q[:, c, :] @ k[:, c // G, :].T * scale
        s = np.where(mask, s, -np.inf)
        m = s.max(axis=1)
        out[c] = m + np.log(np.exp(s - m[:, None]).sum(axis=1))
    return out


# ---------------------------------------------------------------- golden, by hand
def _golden():
    with open(GOLDEN) as f:
        return json.load(f)["examples"]


@pytest.mark.parametrize("ex", _golden(), ids=lambda e: e["name"])
def test_hand_examples(ex):
    q = np.asarray(ex["q"], dtype=np.float64)[:, :, None]
    k = np.asarray(ex["k"], dtype=np.float64)[:, :, None]
    v = np.asarray(ex["v"], dtype=np.float64)[:, :, None]
    assert q.shape[1] == ex["hq"] and k.shape[1] == ex["hkv"]
    res = orc.prefill(q, k, v, ex["host_sizes"], ex["anchor"], ex["passing"], ex["probe_r"],
                      scale=ex["softmax_scale"])
    np.testing.assert_array_equal(res["scores"], np.asarray(ex["expected_scores"], dtype=np.float64))
    np.testing.assert_array_equal(res["sel"], np.asarray(ex["expected_sel"]))
    off = res["offsets"]
    for row, keys in ex["expected_keys"].items():
        got = orc.key_set(off, ex["anchor"], res["sel"], 0, int(row), ex["n_visual"])
        assert sorted(got.tolist()) == keys, row
    env = {"e": math.e, "log": math.log}
    O = np.array([[eval(s, {"__builtins__": {}}, env) for s in r] for r in ex["expected_O"]])
    L = np.array([[eval(s, {"__builtins__": {}}, env) for s in r] for r in ex["expected_lse"]])
    np.testing.assert_allclose(res["O"][:, :, 0], O, rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(res["lse"].T, L, rtol=1e-13, atol=1e-13)


# ---------------------------------------------------------------- degenerate cases
@pytest.mark.parametrize("anchor,passing,n_text", [(0, 0, 0), (16, 8, 0), (64, 32, 17)])
def test_one_host_is_dense_causal(anchor, passing, n_text):
    rng = np.random.default_rng(11)
    N, hq, hkv, d = 192, 4, 2, 16
    q, k, v = _rand_qkv(rng, N + n_text, hq, hkv, d)
    scale = 1 / math.sqrt(d)
    res = orc.prefill(q, k, v, [N], anchor, passing, 8, scale=scale)
    ref = _sdpa(q, k, v, scale, causal=True)
    np.testing.assert_allclose(res["O"], ref, rtol=1e-11, atol=1e-12)
    mask = np.tril(np.ones((N + n_text, N + n_text), dtype=bool))
    np.testing.assert_allclose(res["lse"], _lse_from_mask(q, k, scale, mask), rtol=1e-12, atol=1e-12)
    O2, L2 = orc.dense_causal(q, k, v, scale)
    np.testing.assert_allclose(res["O"], O2, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("H,n_text", [(2, 0), (4, 5), (8, 0)])
def test_passing_everything_is_dense_causal(H, n_text):
    rng = np.random.default_rng(H)
    B, hq, hkv, d = 32, 6, 2, 8
    N = B * H
    q, k, v = _rand_qkv(rng, N + n_text, hq, hkv, d)
    scale = 0.3
    res = orc.prefill(q, k, v, [B] * H, 0, B, 4, scale=scale)
    np.testing.assert_allclose(res["O"], _sdpa(q, k, v, scale, causal=True), rtol=1e-11, atol=1e-12)


@pytest.mark.parametrize("H", [2, 3])
def test_no_anchor_no_passing_is_block_diagonal(H):
    rng = np.random.default_rng(5)
    sizes = [24, 40, 16][:H]
    N = sum(sizes)
    hq, hkv, d = 4, 4, 8
    q, k, v = _rand_qkv(rng, N, hq, hkv, d)
    scale = 0.25
    off = orc.host_offsets(sizes)
    blk = np.zeros((N, N), dtype=bool)
    for h in range(H):
        a, e = off[h], off[h + 1]
        blk[a:e, a:e] = np.tril(np.ones((e - a, e - a), dtype=bool))
    res = orc.prefill(q, k, v, sizes, 0, 0, 4, scale=scale)
    np.testing.assert_allclose(res["O"], _sdpa(q, k, v, scale, mask=blk), rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(res["lse"], _lse_from_mask(q, k, scale, blk), rtol=1e-12, atol=1e-12)


# ---------------------------------------------------------------- explicit-mask formulation
def _explicit_mask(off, anchor, sel, g, N, NT):
    """Visibility matrix built cell by cell from the method's description."""
    M = np.zeros((NT, NT), dtype=bool)
    H = len(off) - 1
    for i in range(NT):
        if i >= N:
            M[i, :i + 1] = True
            continue
        h = int(np.searchsorted(off, i, side="right") - 1)
        if h == 0:
            M[i, :i + 1] = True
            continue
        M[i, :anchor] = True
        for hp in range(h):
            for j in sel[hp, g]:
                M[i, j] = True
        M[i, off[h]:i + 1] = True
    return M


@pytest.mark.parametrize("H", [1, 2, 4, 8])
def test_blockwise_equals_explicit_mask(H):
    cfg = CONFIGS["tiny"].with_(n_hosts=H, n_text=7)
    g = generate(cfg)
    q, k, v = (orc.bf16_bits_to_f64(g[x]) for x in ("q", "k", "v"))
    B = cfg.n_visual // H
    P = min(cfg.passing, B // 2)
    A = min(cfg.anchor, B - P)
    scale = 1 / math.sqrt(cfg.head_dim)
    res = orc.prefill(q, k, v, g["host_sizes"], A, P, min(cfg.probe_r, B), scale=scale)
    off = res["offsets"]
    G = cfg.hq // cfg.hkv
    NT = cfg.n_total
    for gi in range(cfg.hkv):
        M = _explicit_mask(off, A, res["sel"], gi, cfg.n_visual, NT)
        for c in range(gi * G, (gi + 1) * G):
            s = q[:, c, :] @ k[:, gi, :].T * scale
            s = np.where(M, s, -np.inf)
            m = s.max(axis=1, keepdims=True)
            p = np.exp(s - m)
            l = p.sum(axis=1, keepdims=True)
            np.testing.assert_allclose(res["O"][:, c, :], (p @ v[:, gi, :]) / l, rtol=1e-11, atol=1e-12)
            np.testing.assert_allclose(res["lse"][c], (m + np.log(l))[:, 0], rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("H", [2, 4])
def test_per_query_head_selection_explicit_mask(H):
    """Per-query-head selection (head_reduce="none"): every query head attends through
    its own selection row; checked against an explicit mask per query head."""
    cfg = CONFIGS["tiny"].with_(n_hosts=H, n_text=5, hq=6, hkv=2)
    g = generate(cfg)
    q, k, v = (orc.bf16_bits_to_f64(g[x]) for x in ("q", "k", "v"))
    B = cfg.n_visual // H
    P = min(cfg.passing, B // 2)
    A = min(cfg.anchor, B - P)
    scale = 1 / math.sqrt(cfg.head_dim)
    res = orc.prefill(q, k, v, g["host_sizes"], A, P, min(cfg.probe_r, B), scale=scale, head_reduce="none")
    assert res["scores"].shape == (cfg.hq, cfg.n_visual) and res["sel"].shape == (H - 1, cfg.hq, P)
    off = res["offsets"]
    G = cfg.hq // cfg.hkv
    for c in range(cfg.hq):
        gi = c // G
        M = _explicit_mask(off, A, res["sel"], c, cfg.n_visual, cfg.n_total)
        s = q[:, c, :] @ k[:, gi, :].T * scale
        s = np.where(M, s, -np.inf)
        m = s.max(axis=1, keepdims=True)
        p = np.exp(s - m)
        l = p.sum(axis=1, keepdims=True)
        np.testing.assert_allclose(res["O"][:, c, :], (p @ v[:, gi, :]) / l, rtol=1e-11, atol=1e-12)
        np.testing.assert_allclose(res["lse"][c], (m + np.log(l))[:, 0], rtol=1e-12, atol=1e-12)


def test_per_query_head_scores_and_duplicate_heads():
    """Row c of the per-query-head scores is the max-mode score of the problem made of
    query head c alone; with every query head of a group a copy of the first, the
    per-query-head prefill equals the default (max over heads) one."""
    cfg = CONFIGS["tiny"].with_(n_hosts=4, n_text=3, hq=6, hkv=2)
    g = generate(cfg)
    q, k, v = (orc.bf16_bits_to_f64(g[x]) for x in ("q", "k", "v"))
    off = orc.host_offsets(g["host_sizes"])
    scale = 1 / math.sqrt(cfg.head_dim)
    G = cfg.hq // cfg.hkv
    per = orc.probe_scores(q, k, off, cfg.probe_r, scale, "none")
    for t in range(G):
        heads = [gg * G + t for gg in range(cfg.hkv)]
        np.testing.assert_array_equal(per[heads], orc.probe_scores(q[:, heads], k, off, cfg.probe_r, scale, "max"))
    qd = q.copy()
    for gg in range(cfg.hkv):
        for t in range(1, G):
            qd[:, gg * G + t] = qd[:, gg * G]
    a = orc.prefill(qd, k, v, g["host_sizes"], cfg.anchor, cfg.passing, cfg.probe_r, scale=scale)
    b = orc.prefill(qd, k, v, g["host_sizes"], cfg.anchor, cfg.passing, cfg.probe_r, scale=scale,
                    head_reduce="none")
    for c in range(cfg.hq):
        np.testing.assert_array_equal(b["sel"][:, c], a["sel"][:, c // G])
    np.testing.assert_allclose(b["O"], a["O"], rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(b["lse"], a["lse"], rtol=1e-13, atol=1e-13)


def test_rows_formulation_matches_blockwise():
    cfg = CONFIGS["tiny"].with_(n_text=5)
    g = generate(cfg)
    q, k, v = (orc.bf16_bits_to_f64(g[x]) for x in ("q", "k", "v"))
    scale = 1 / math.sqrt(cfg.head_dim)
    full = orc.prefill(q, k, v, g["host_sizes"], cfg.anchor, cfg.passing, cfg.probe_r, scale=scale)
    rng = np.random.default_rng(0)
    rows = rng.integers(0, cfg.n_total, 64)
    heads = rng.integers(0, cfg.hq, 64)
    O, L = orc.attention_rows(q, k, v, full["offsets"], cfg.anchor, full["sel"], scale, rows, heads)
    np.testing.assert_allclose(O, full["O"][rows, heads], rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(L, full["lse"][heads, rows], rtol=1e-12, atol=1e-12)


def test_row_range_matches_full():
    cfg = CONFIGS["tiny"].with_(n_text=20, n_hosts=4)
    g = generate(cfg)
    q, k, v = (orc.bf16_bits_to_f64(g[x]) for x in ("q", "k", "v"))
    scale = 1 / math.sqrt(cfg.head_dim)
    full = orc.prefill(q, k, v, g["host_sizes"], cfg.anchor, cfg.passing, cfg.probe_r, scale=scale)
    for r0, r1 in [(100, 300), (500, 532), (0, 7)]:
        O, L = orc.approx_attention(q, k, v, full["offsets"], cfg.anchor, full["sel"], scale,
                                    row_chunk=64, row_range=(r0, r1))
        np.testing.assert_allclose(O[r0:r1], full["O"][r0:r1], rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(L[:, r0:r1], full["lse"][:, r0:r1], rtol=1e-12, atol=1e-12)
        assert np.isnan(O[r1:]).all() and np.isnan(O[:r0]).all()
        Oc, Lc = orc.approx_attention(q, k, v, full["offsets"], cfg.anchor, full["sel"], scale,
                                      row_chunk=64, row_range=(r0, r1), compact=True)
        assert Oc.shape == (r1 - r0,) + O.shape[1:] and Lc.shape == (L.shape[0], r1 - r0)
        np.testing.assert_array_equal(Oc, O[r0:r1])
        np.testing.assert_array_equal(Lc, L[:, r0:r1])


# ---------------------------------------------------------------- brute force: scores, select
def test_scores_brute_force():
    rng = np.random.default_rng(3)
    sizes = [12, 9, 10]
    hq, hkv, d, R = 6, 2, 4, 5
    N = sum(sizes)
    q, k, _ = _rand_qkv(rng, N, hq, hkv, d)
    scale = 0.7
    off = orc.host_offsets(sizes)
    got = orc.probe_scores(q, k, off, R, scale)
    G = hq // hkv
    for h in range(len(sizes)):
        a, e = int(off[h]), int(off[h + 1])
        for g in range(hkv):
            for j in range(a, e):
                best = -math.inf
                for i in range(e - R, e):
                    if i < j:
                        continue
                    for c in range(g * G, (g + 1) * G):
                        dot = sum(q[i, c, t] * k[j, g, t] for t in range(d))
                        best = max(best, dot * scale)
                assert got[g, j] == pytest.approx(best, rel=1e-13, abs=1e-13)
                # invariant: never below the last row's own logit (every head)
                for c in range(g * G, (g + 1) * G):
                    assert got[g, j] >= q[e - 1, c] @ k[j, g] * scale - 1e-12


@pytest.mark.parametrize("mode", ["sum", "mean"])
def test_scores_head_reduce_brute_force(mode):
    """Switchable reading R1: per-head max over the probe rows, then sum or mean over
    the group's heads -- a pure-Python triple loop on tiny inputs."""
    rng = np.random.default_rng(5)
    sizes = [11, 14, 9]
    hq, hkv, d, R = 6, 2, 4, 5
    q, k, _ = _rand_qkv(rng, sum(sizes), hq, hkv, d)
    scale = 0.6
    off = orc.host_offsets(sizes)
    got = orc.probe_scores(q, k, off, R, scale, head_reduce=mode)
    G = hq // hkv
    for h in range(len(sizes)):
        a, e = int(off[h]), int(off[h + 1])
        for g in range(hkv):
            for j in range(a, e):
                total = 0.0
                for c in range(g * G, (g + 1) * G):
                    best = -math.inf
                    for i in range(max(j, e - R), e):
                        best = max(best, sum(q[i, c, t] * k[j, g, t] for t in range(d)) * scale)
                    total += best
                want = total if mode == "sum" else total / G
                assert got[g, j] == pytest.approx(want, rel=1e-13, abs=1e-13)


def test_scores_head_reduce_decomposes_over_heads():
    """sum over heads = the sum of max-mode scores of the one-head-per-group problems
    (query head t of every group alone); the modes agree when a group has one head;
    mean = sum / G."""
    cfg = CONFIGS["tiny"].with_(hq=6, hkv=2, head_dim=16, n_visual=192, n_hosts=3, anchor=16, passing=8,
                                probe_r=8)
    g = generate(cfg)
    q, k = orc.bf16_bits_to_f64(g["q"]), orc.bf16_bits_to_f64(g["k"])
    off = orc.host_offsets(g["host_sizes"])
    scale = 1.0 / math.sqrt(cfg.head_dim)
    G = cfg.hq // cfg.hkv
    s_sum = orc.probe_scores(q, k, off, cfg.probe_r, scale, "sum")
    parts = [orc.probe_scores(q[:, [gg * G + t for gg in range(cfg.hkv)]],
                              k, off, cfg.probe_r, scale, "max") for t in range(G)]
    np.testing.assert_allclose(s_sum, sum(parts), rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(orc.probe_scores(q, k, off, cfg.probe_r, scale, "mean"), s_sum / G,
                               rtol=1e-14, atol=1e-14)
    one = [gg * G for gg in range(cfg.hkv)]
    q1 = q[:, one]
    ref = orc.probe_scores(q1, k, off, cfg.probe_r, scale, "max")
    for mode in ("sum", "mean"):
        np.testing.assert_array_equal(orc.probe_scores(q1, k, off, cfg.probe_r, scale, mode), ref)
    with pytest.raises(ValueError):
        orc.probe_scores(q, k, off, cfg.probe_r, scale, "median")


@pytest.mark.parametrize("mode", ["max", "sum"])
def test_prob_scores_brute_force(mode):
    """score_kind="prob": each probe row's softmax over the block keys it sees, then
    the max over probe rows and the head reduction -- pure-Python loops."""
    rng = np.random.default_rng(6)
    sizes = [10, 13, 9]
    hq, hkv, d, R = 4, 2, 3, 4
    q, k, _ = _rand_qkv(rng, sum(sizes), hq, hkv, d)
    scale = 0.8
    off = orc.host_offsets(sizes)
    got = orc.probe_scores(q, k, off, R, scale, head_reduce=mode, score_kind="prob")
    G = hq // hkv
    for h in range(len(sizes)):
        a, e = int(off[h]), int(off[h + 1])
        for g in range(hkv):
            for j in range(a, e):
                per = []
                for c in range(g * G, (g + 1) * G):
                    best = 0.0
                    for i in range(max(j, e - R), e):
                        logit = [sum(q[i, c, t] * k[jj, g, t] for t in range(d)) * scale for jj in range(a, i + 1)]
                        z = sum(math.exp(x - max(logit)) for x in logit)
                        best = max(best, math.exp(logit[j - a] - max(logit)) / z)
                    per.append(best)
                want = max(per) if mode == "max" else sum(per)
                assert got[g, j] == pytest.approx(want, rel=1e-12, abs=1e-15)


def test_prob_scores_invariants():
    """Probabilities: within (0, 1]; for every head the scores of a host's keys add up
    to at least 1 (they dominate the last probe row's distribution); with one probe row
    the selection equals the logit selection (a monotone map of the same row)."""
    cfg = CONFIGS["tiny"].with_(n_hosts=4, hq=4, hkv=2)
    g = generate(cfg)
    q, k = orc.bf16_bits_to_f64(g["q"]), orc.bf16_bits_to_f64(g["k"])
    off = orc.host_offsets(g["host_sizes"])
    scale = 1.0 / math.sqrt(cfg.head_dim)
    per = orc.probe_scores(q, k, off, cfg.probe_r, scale, "none", "prob")
    assert (per > 0).all() and (per <= 1 + 1e-12).all()
    for h in range(cfg.n_hosts):
        a, e = int(off[h]), int(off[h + 1])
        assert (per[:, a:e].sum(axis=1) >= 1 - 1e-12).all()
    sp = orc.probe_scores(q, k, off, 1, scale, "none", "prob")
    sl = orc.probe_scores(q, k, off, 1, scale, "none", "logit")
    np.testing.assert_array_equal(orc.select_passing(sp, off, cfg.anchor, cfg.passing),
                                  orc.select_passing(sl, off, cfg.anchor, cfg.passing))
    with pytest.raises(ValueError):
        orc.probe_scores(q, k, off, cfg.probe_r, scale, "max", "softmax")


def _brute_select(vals, lo, P):
    order = sorted(range(len(vals)), key=lambda t: (-float(vals[t]), t))
    return sorted(lo + t for t in order[:P])


@pytest.mark.parametrize("dtype", [np.float32, np.float64])
def test_select_brute_force_with_ties(dtype):
    rng = np.random.default_rng(9)
    sizes = [40, 33, 27, 35]
    off = orc.host_offsets(sizes)
    hkv, A, P = 3, 6, 9
    N = int(off[-1])
    base = rng.integers(-3, 4, size=(hkv, N)).astype(dtype)   # many exact ties
    base[0, 7:20] = 0.0
    base[0, 8] = -0.0                                           # -0 equals +0
    base[1, :] = 1.0                                            # all equal
    base[2, 50:60] = np.float32(3.4e38)                         # very large
    sel = orc.select_passing(base, off, A, P)
    assert sel.shape == (len(sizes) - 1, hkv, P)
    for h in range(len(sizes) - 1):
        lo = int(off[h]) + (A if h == 0 else 0)
        hi = int(off[h + 1])
        for g in range(hkv):
            want = _brute_select(base[g, lo:hi], lo, P)
            assert sel[h, g].tolist() == want
            chosen = set(want)
            rest = [j for j in range(lo, hi) if j not in chosen]
            assert min(base[g, j] for j in chosen) >= max(base[g, j] for j in rest)
    # all-equal segment: the lowest P candidate indices
    assert sel[0, 1].tolist() == list(range(A, A + P))


def test_anchor_is_never_a_candidate():
    off = orc.host_offsets([20, 20])
    s = np.zeros((1, 40))
    s[0, :5] = 100.0
    sel = orc.select_passing(s, off, 5, 3)
    assert sel[0, 0].tolist() == [5, 6, 7]


# ---------------------------------------------------------------- merge, sanity
def test_lse_merge_associative():
    rng = np.random.default_rng(1)
    d, L = 8, 50
    kk = rng.standard_normal((L, d))
    vv = rng.standard_normal((L, d))
    qq = rng.standard_normal(d)

    def attend(idx):
        s = kk[idx] @ qq
        m = s.max()
        p = np.exp(s - m)
        return p @ vv[idx] / p.sum(), m + np.log(p.sum())

    full_o, full_l = attend(np.arange(L))
    for cut in (1, 17, 49):
        o1, l1 = attend(np.arange(cut))
        o2, l2 = attend(np.arange(cut, L))
        o, l = orc.lse_merge(o1, np.float64(l1), o2, np.float64(l2))
        np.testing.assert_allclose(o, full_o, rtol=1e-12, atol=1e-12)
        assert abs(l - full_l) < 1e-12
    # three-way split merged in two orders
    parts = [attend(np.arange(0, 10)), attend(np.arange(10, 30)), attend(np.arange(30, L))]
    a = orc.lse_merge(*orc.lse_merge(parts[0][0], parts[0][1], parts[1][0], parts[1][1]),
                      parts[2][0], parts[2][1])
    b = orc.lse_merge(parts[0][0], parts[0][1],
                      *orc.lse_merge(parts[1][0], parts[1][1], parts[2][0], parts[2][1]))
    np.testing.assert_allclose(a[0], b[0], rtol=1e-12, atol=1e-12)


def test_output_within_attended_value_range():
    cfg = CONFIGS["tiny"].with_(n_text=9)
    g = generate(cfg)
    q, k, v = (orc.bf16_bits_to_f64(g[x]) for x in ("q", "k", "v"))
    scale = 1 / math.sqrt(cfg.head_dim)
    res = orc.prefill(q, k, v, g["host_sizes"], cfg.anchor, cfg.passing, cfg.probe_r, scale=scale)
    G = cfg.hq // cfg.hkv
    for i in range(0, cfg.n_total, 7):
        for c in range(cfg.hq):
            keys = orc.key_set(res["offsets"], cfg.anchor, res["sel"], c // G, i, cfg.n_visual)
            vals = v[keys, c // G, :]
            assert (res["O"][i, c] <= vals.max(axis=0) + 1e-12).all()
            assert (res["O"][i, c] >= vals.min(axis=0) - 1e-12).all()


# ---------------------------------------------------------------- generator
def test_generator_recipe():
    cfg = CONFIGS["tiny"]
    a, b = generate(cfg), generate(cfg)
    for x in ("q", "k", "v"):
        assert a[x].dtype == np.uint16 and np.array_equal(a[x], b[x])
    assert a["q"].shape == (512, 4, 64) and a["k"].shape == (512, 2, 64)
    st = CONFIGS["stress"]
    sizes = host_sizes_for(st, np.random.default_rng(st.seed))
    assert sizes.sum() == st.n_visual and sizes.min() >= 4096 and sizes.max() <= 12288
    assert (sizes % 64 == 0).all() and sizes[0] >= st.anchor + st.passing
    # bf16 rounding: exact values survive, ties go to even
    x = np.array([1.0, -2.5, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8], dtype=np.float32)
    bits = bf16_round_bits(x)
    back = orc.bf16_bits_to_f64(bits)
    assert back.tolist() == [1.0, -2.5, 1.0, 1.0 + 2 ** -6]


def test_frame_structure():
    cfg = CONFIGS["tiny"].with_(kv_kind="frame", frame=64, salient_frac=0.05)
    g = generate(cfg)
    k = orc.bf16_bits_to_f64(g["k"])
    # tokens of one frame are close to each other (noise 0.3), frames differ
    assert len(g["salient"]) == round(0.05 * cfg.n_visual)
    plain = np.setdiff1d(np.arange(cfg.n_visual), g["salient"])
    f0 = plain[plain < 64]
    spread = np.abs(k[f0, 0] - k[f0, 0].mean(axis=0)).mean()
    assert 0.15 < spread < 0.35


# ---------------------------------------------------------------- sharding (multi-host form)
def test_zigzag_pages_example():
    """The pages' description of the arrangement (German explainer, "Lastverteilung"):
    the first worker takes the first and the last block, the second the second and the
    one before last, and so on (tests/golden/zigzag_pairing.json, written out by hand)."""
    with open(os.path.join(os.path.dirname(__file__), "golden", "zigzag_pairing.json")) as f:
        cases = json.load(f)["cases"]
    for c in cases:
        assert orc.zigzag_owners(c["blocks"], c["workers"]).tolist() == c["owner"], c
    with pytest.raises(ValueError):
        orc.zigzag_owners(6, 4)


@pytest.mark.parametrize("world", [1, 2, 3, 4, 8])
@pytest.mark.parametrize("rounds", [1, 2, 3])
def test_zigzag_balances_passing_lengths(world, rounds):
    """"Approximate attention load balancing": ZigZag makes the total length of the
    passing blocks each physical host attends to equal (host h attends to h * P passing
    rows); every rank runs the same number of hosts.  The contiguous split does not
    balance (later ranks carry more) once there are two ranks."""
    H, P = 2 * world * rounds, 7
    zz = orc.zigzag_owners(H, world)
    load = np.zeros(world, dtype=np.int64)
    for h in range(H):
        load[zz[h]] += h * P
    assert (load == load[0]).all()
    assert (np.bincount(zz, minlength=world) == 2 * rounds).all()
    ct = orc.contiguous_owners(H, world)
    lc = np.zeros(world, dtype=np.int64)
    for h in range(H):
        lc[ct[h]] += h * P
    assert (world == 1) or (np.diff(lc) > 0).all()


@pytest.mark.parametrize("policy", ["zigzag", "contiguous", "random"])
@pytest.mark.parametrize("head_reduce", ["max", "none"])
def test_sharded_attention_equals_single(policy, head_reduce):
    """The multi-host form (local causal part and [anchor | passing] part merged
    through the lse per host; the text rows' per-host partials from their owners,
    merged after the exchange) equals the one-pass approximate attention."""
    H, world = 8, 2
    cfg = CONFIGS["tiny"].with_(n_visual=256, n_hosts=H, n_text=11, hq=4, hkv=2, head_dim=16, anchor=8,
                                passing=5, probe_r=16)
    g = generate(cfg)
    q, k, v = (orc.bf16_bits_to_f64(g[x]) for x in ("q", "k", "v"))
    scale = 1 / math.sqrt(cfg.head_dim)
    res = orc.prefill(q, k, v, g["host_sizes"], cfg.anchor, cfg.passing, cfg.probe_r, scale=scale,
                      head_reduce=head_reduce)
    if policy == "zigzag":
        owner = orc.zigzag_owners(H, world)
    elif policy == "contiguous":
        owner = orc.contiguous_owners(H, world)
    else:
        owner = np.random.default_rng(5).integers(0, 3, size=H)
    O, L = orc.sharded_attention(q, k, v, res["offsets"], cfg.anchor, res["sel"], scale, owner)
    np.testing.assert_allclose(O, res["O"], rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(L, res["lse"], rtol=1e-12, atol=1e-12)


def test_host_costs_count_attended_pairs():
    """Summed over the hosts, the per-host costs are the (query, key) pairs the
    approximate attention evaluates: counted here row by row from the key sets."""
    sizes, A, P, T = [40, 24, 56, 32], 6, 5, 9
    N = sum(sizes)
    off = orc.host_offsets(sizes)
    sel = np.zeros((len(sizes) - 1, 1, P), dtype=np.int64)
    for h in range(len(sizes) - 1):
        lo = int(off[h]) + (A if h == 0 else 0)
        sel[h, 0] = np.arange(lo, lo + P)
    pairs = sum(len(orc.key_set(off, A, sel, 0, i, N)) for i in range(N + T))
    cost = orc.host_costs(sizes, A, P, T)
    assert int(cost.sum()) == pairs
    assert (np.diff(orc.host_costs([32] * 6, A, P, 0)) > 0).all()   # later hosts carry more


@pytest.mark.parametrize("world", [2, 3])
@pytest.mark.parametrize("seed", [0, 1, 2, 3])
def test_longest_first_within_graham_bound_of_optimum(world, seed):
    """Longest-first list scheduling: every rank's load is at most the mean plus the
    largest cost, and the largest load is within 4/3 - 1/(3W) of the optimum, found here
    by trying every assignment (Graham's bound for this rule)."""
    import itertools
    rng = np.random.default_rng(seed)
    cost = rng.integers(1, 50, size=7)
    own = orc.longest_first_owners(cost, world)
    load = np.bincount(own, weights=cost, minlength=world)
    assert load.max() <= cost.sum() / world + cost.max()
    best = min(np.bincount(np.array(a), weights=cost, minlength=world).max()
               for a in itertools.product(range(world), repeat=len(cost)))
    assert load.max() <= (4 / 3 - 1 / (3 * world)) * best + 1e-9


def test_oracle_pool_matches_direct_calls():
    """The process pool that full-size GPU tests use for whole-tile comparisons returns
    exactly what approx_attention gives for the same row ranges."""
    from . import oracle_pool
    cfg = CONFIGS["tiny"].with_(n_text=20, n_hosts=4)
    g = generate(cfg)
    q, k, v = (orc.bf16_bits_to_f64(g[x]) for x in ("q", "k", "v"))
    scale = 1 / math.sqrt(cfg.head_dim)
    full = orc.prefill(q, k, v, g["host_sizes"], cfg.anchor, cfg.passing, cfg.probe_r, scale=scale)
    ranges = [(0, 128), (256, 384), (384, 512), (512, 532)]
    res = oracle_pool.attention_rows_ranges(g, full["offsets"], cfg.anchor, full["sel"], scale, ranges, workers=2)
    for (r0, r1), (O, L) in zip(ranges, res):
        np.testing.assert_allclose(O, full["O"][r0:r1], rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(L, full["lse"][:, r0:r1], rtol=1e-12, atol=1e-12)
