"""Parity at the full sizes of the five workloads, through the C ABI, in the launch
configuration bench.py times (one plan, one workspace, one spava_attn_prefill).

Every score of hosts 0..H-2 is checked against the fp64 oracle; the selection is
checked bit-exactly against the oracle's selection on the GPU's own fp32 scores and
for near-tie-only differences against the fp64 selection; O and lse are checked
element by element, every head, on whole 128-row tiles of the kernel -- the first, a
middle and the last tile of every host block -- and on every text row, against the
oracle re-run with the GPU's indices (the oracle runs in a spawn-started process
pool, tests/oracle_pool.py); further sampled (row, head) outputs cover block starts,
tile boundaries, probe rows and random rows.  The 256k workload also runs the dense
causal kernel on the same inputs, checked on four whole tiles.
"""

import math

import numpy as np
import pytest
import torch

from oracle import spava_oracle as orc
from workloads import CONFIGS, generate

from . import oracle_pool
from .helpers import LSE_TOL, O_TOL, check_selection_vs_fp64, to_device_bf16

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

sab = pytest.importorskip("sequence_approximate_attention_b200")


class LazyF64:
    """bf16 bits viewed as float64, converted where indexed (keeps host memory low)."""

    def __init__(self, bits):
        self.bits = bits
        self.shape = bits.shape

    def __getitem__(self, key):
        b = np.ascontiguousarray(self.bits[key], dtype=np.uint16)
        return (b.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


def _score_tolerance_and_ref(q, k, off, R, scale, hosts):
    hq, hkv = q.shape[1], k.shape[1]
    G = hq // hkv
    ref = {}
    tol = {}
    for h in hosts:
        a, e = int(off[h]), int(off[h + 1])
        keys = np.arange(a, e)
        rows = np.arange(e - R, e)
        vis = rows[:, None] >= keys[None, :]
        qh = q[e - R:e]                                   # [R, hq, d]
        for g in range(hkv):
            qg = qh[:, g * G:(g + 1) * G, :].reshape(-1, qh.shape[2])   # [(R*G), d], row = (r, c)
            kb = k[a:e, g, :]
            s = (qg @ kb.T).reshape(R, G, -1) * scale
            s = np.where(vis[:, None, :], s, -np.inf)
            ref[(h, g)] = s.max(axis=(0, 1))
            tol[(h, g)] = 1e-5 * scale * (np.abs(qg) @ np.abs(kb).T).max(axis=0) + 1e-6
    return ref, tol


def _sample_rows(cfg, off, rng, n_random=48):
    rows = set()
    for h in range(cfg.n_hosts):
        a, e = int(off[h]), int(off[h + 1])
        for r in (a, a + 1, a + 127, a + 128, a + 255, a + 256, e - cfg.probe_r, e - 2, e - 1):
            if a <= r < e:
                rows.add(r)
    for r in (cfg.n_visual, cfg.n_visual + cfg.n_text // 2, cfg.n_visual + cfg.n_text - 1):
        if cfg.n_text and r < cfg.n_visual + cfg.n_text:
            rows.add(r)
    rows.update(int(x) for x in rng.integers(0, cfg.n_visual + cfg.n_text, n_random))
    rows = sorted(rows)
    heads = [int((i * 7 + 3) % cfg.hq) for i in range(len(rows))]
    return rows, heads


def _whole_tiles(cfg, off):
    """Row ranges of whole 128-row tiles of the attention kernel (tiles start at each
    block's first row): the first, a middle and the last tile of every host block,
    and all text rows."""
    ranges = []
    for h in range(cfg.n_hosts):
        a, e = int(off[h]), int(off[h + 1])
        B = e - a
        for t in sorted({0, 128 * ((B // 128) // 2), 128 * ((B - 1) // 128)}):
            ranges.append((a + t, min(e, a + t + 128)))
    if cfg.n_text:
        ranges.append((cfg.n_visual, cfg.n_visual + cfg.n_text))
    return ranges


def _compare_ranges(o_dev, lse_dev, ranges, refs, what):
    """Every head of every row of the ranges against the oracle; returns the number of
    (row, head) outputs compared."""
    n, worst_o, worst_l = 0, 0.0, 0.0
    for (r0, r1), (O_ref, L_ref) in zip(ranges, refs):
        o = o_dev[r0:r1].float().cpu().numpy()
        lse = lse_dev[:, r0:r1].cpu().numpy()
        assert np.isfinite(o).all() and np.isfinite(lse).all(), (what, r0, r1)
        worst_o = max(worst_o, float(np.abs(o - O_ref).max()))
        worst_l = max(worst_l, float(np.abs(lse - L_ref).max()))
        n += O_ref.shape[0] * O_ref.shape[1]
    assert worst_o <= O_TOL and worst_l <= LSE_TOL, (what, n, worst_o, worst_l)
    return n


@pytest.fixture(scope="module", params=["qwen64k", "128k", "stress", "256k"])
def fullsize_run(request):
    cfg = CONFIGS[request.param]
    g = generate(cfg)
    sizes = [int(x) for x in g["host_sizes"]]
    dev = {x: to_device_bf16(g[x]) for x in ("q", "k", "v")}
    plan = sab.Plan(cfg.n_visual, cfg.n_text, cfg.n_hosts, sizes, cfg.anchor, cfg.passing, cfg.probe_r,
                    cfg.hq, cfg.hkv, cfg.head_dim)
    ws = plan.new_workspace()
    scores = torch.empty((cfg.hkv, cfg.n_visual), dtype=torch.float32, device="cuda")
    idx = torch.empty(plan.idx_shape(), dtype=torch.int32, device="cuda")
    o, lse = sab.attn_prefill(plan, dev["q"], dev["k"], dev["v"], scores_out=scores, idx_out=idx, workspace=ws)
    sab.check_device_error(plan, ws)
    res = {"cfg": cfg, "g": g, "sizes": sizes, "plan": plan, "dev": dev, "ws": ws,
           "scores": scores.cpu().numpy(), "idx": idx.cpu().numpy().astype(np.int64),
           "o": o, "lse": lse}
    yield res
    plan.close()
    del dev, o, lse
    torch.cuda.empty_cache()


def test_fullsize_scores_and_selection(fullsize_run):
    r = fullsize_run
    cfg = r["cfg"]
    off = orc.host_offsets(r["sizes"])
    q, k = LazyF64(r["g"]["q"]), LazyF64(r["g"]["k"])
    scale = 1.0 / math.sqrt(cfg.head_dim)
    hosts = range(cfg.n_hosts - 1)
    ref, tol = _score_tolerance_and_ref(q, k, off, cfg.probe_r, scale, hosts)
    sc = r["scores"]
    ref64 = np.full_like(sc, np.nan, dtype=np.float64)
    for (h, g), v in ref.items():
        a, e = int(off[h]), int(off[h + 1])
        err = np.abs(sc[g, a:e] - v)
        assert (err <= tol[(h, g)]).all(), (cfg.name, h, g, float(err.max()))
        ref64[g, a:e] = v
    np.testing.assert_array_equal(r["idx"], orc.select_passing(sc, off, cfg.anchor, cfg.passing))
    # fp64 selection: differences only at near-ties (rows of host H-1 are unused)
    ref64[:, int(off[cfg.n_hosts - 1]):] = 0.0
    check_selection_vs_fp64(r["idx"], ref64, off, cfg.anchor, cfg.passing)


def test_fullsize_sampled_outputs(fullsize_run):
    r = fullsize_run
    cfg = r["cfg"]
    off = orc.host_offsets(r["sizes"])
    q, k, v = (LazyF64(r["g"][x]) for x in ("q", "k", "v"))
    rng = np.random.default_rng(cfg.seed)
    rows, heads = _sample_rows(cfg, off, rng)
    O_ref, L_ref = orc.attention_rows(q, k, v, off, cfg.anchor, r["idx"], 1.0 / math.sqrt(cfg.head_dim), rows, heads)
    rt = torch.tensor(rows, device="cuda")
    ht = torch.tensor(heads, device="cuda")
    o = r["o"][rt, ht].float().cpu().numpy()
    lse = r["lse"][ht, rt].cpu().numpy()
    assert np.isfinite(o).all() and np.isfinite(lse).all()
    do = np.abs(o - O_ref).max()
    dl = np.abs(lse - L_ref).max()
    assert do <= O_TOL and dl <= LSE_TOL, (cfg.name, do, dl)
    # every output is finite (no NaN/inf anywhere in the full tensors)
    assert torch.isfinite(r["o"].float()).all().item() and torch.isfinite(r["lse"]).all().item()


# (row, head) outputs compared element by element per workload: (tiles + text rows) x heads
WHOLE_TILE_OUTPUTS = {"qwen64k": (24 * 128 + 128) * 28, "128k": (48 * 128 + 256) * 32,
                      "stress": None, "256k": (96 * 128 + 256) * 32}


def test_fullsize_whole_tiles(fullsize_run):
    r = fullsize_run
    cfg = r["cfg"]
    off = orc.host_offsets(r["sizes"])
    ranges = _whole_tiles(cfg, off)
    refs = oracle_pool.attention_rows_ranges(r["g"], off, cfg.anchor, r["idx"], 1.0 / math.sqrt(cfg.head_dim),
                                             ranges)
    n = _compare_ranges(r["o"], r["lse"], ranges, refs, cfg.name)
    expected = WHOLE_TILE_OUTPUTS[cfg.name]
    if expected is None:  # uneven blocks: the last tile of a block may be partial
        expected = sum(r1 - r0 for r0, r1 in ranges) * cfg.hq
    assert n == expected, (cfg.name, n, expected)


def test_fullsize_dense_causal_256k(fullsize_run):
    r = fullsize_run
    cfg = r["cfg"]
    if cfg.name != "256k":
        pytest.skip("the dense causal comparison runs on the 256k workload")
    dev = r["dev"]
    o, lse = sab.dense_causal(r["plan"], dev["q"], dev["k"], dev["v"], workspace=r["ws"])
    sab.check_device_error(r["plan"], r["ws"])
    off = orc.host_offsets([cfg.n_visual])   # one host: dense causal
    q, k, v = (LazyF64(r["g"][x]) for x in ("q", "k", "v"))
    NT = cfg.n_visual + cfg.n_text
    rows = [0, 1, 127, 128, 4095, 100000, 200000, NT - 300, NT - 1]
    heads = [(i * 5) % cfg.hq for i in range(len(rows))]
    O_ref, L_ref = orc.attention_rows(q, k, v, off, 0, None, 1.0 / math.sqrt(cfg.head_dim), rows, heads)
    rt, ht = torch.tensor(rows, device="cuda"), torch.tensor(heads, device="cuda")
    do = np.abs(o[rt, ht].float().cpu().numpy() - O_ref).max()
    dl = np.abs(lse[ht, rt].cpu().numpy() - L_ref).max()
    assert do <= O_TOL and dl <= LSE_TOL, (do, dl)
    # four whole 128-row tiles of the dense kernel, every head: the first, two in the
    # middle and the last (partial) one
    last = 128 * ((NT - 1) // 128)
    ranges = [(0, 128), (100096, 100224), (200064, 200192), (last, NT)]
    refs = oracle_pool.attention_rows_ranges(r["g"], off, 0, None, 1.0 / math.sqrt(cfg.head_dim), ranges)
    n = _compare_ranges(o, lse, ranges, refs, "dense 256k")
    assert n == (3 * 128 + NT - last) * cfg.hq


def test_fullsize_two_stage_flow(fullsize_run):
    """The two-stage flow (local pass with fused probe scores, remote pass merged
    through the lse) on the same full-size inputs: fused scores within tolerance of the
    oracle, selection bit-exact on its own scores, sampled outputs against the oracle
    re-run with its indices."""
    r = fullsize_run
    cfg = r["cfg"]
    if cfg.name not in ("128k", "stress"):
        pytest.skip("two-stage flow checked at full size on the 128k and stress workloads")
    dev, plan = r["dev"], r["plan"]
    ws = plan.new_workspace(two_stage=True)
    scores = torch.empty((cfg.hkv, cfg.n_visual), dtype=torch.float32, device="cuda")
    idx = torch.empty(plan.idx_shape(), dtype=torch.int32, device="cuda")
    o, lse = sab.attn_prefill_two_stage(plan, dev["q"], dev["k"], dev["v"], scores_out=scores, idx_out=idx,
                                        workspace=ws)
    sab.check_device_error(plan, ws)
    off = orc.host_offsets(r["sizes"])
    q, k, v = (LazyF64(r["g"][x]) for x in ("q", "k", "v"))
    scale = 1.0 / math.sqrt(cfg.head_dim)
    sc = scores.cpu().numpy()
    hosts = range(cfg.n_hosts - 1)
    ref, tol = _score_tolerance_and_ref(q, k, off, cfg.probe_r, scale, hosts)
    for (h, g), val in ref.items():
        a, e = int(off[h]), int(off[h + 1])
        assert (np.abs(sc[g, a:e] - val) <= tol[(h, g)]).all(), (cfg.name, h, g)
    sel = idx.cpu().numpy().astype(np.int64)
    np.testing.assert_array_equal(sel, orc.select_passing(sc, off, cfg.anchor, cfg.passing))
    rng = np.random.default_rng(cfg.seed + 1)
    rows, heads = _sample_rows(cfg, off, rng)
    O_ref, L_ref = orc.attention_rows(q, k, v, off, cfg.anchor, sel, scale, rows, heads)
    rt, ht = torch.tensor(rows, device="cuda"), torch.tensor(heads, device="cuda")
    do = np.abs(o[rt, ht].float().cpu().numpy() - O_ref).max()
    dl = np.abs(lse[ht, rt].cpu().numpy() - L_ref).max()
    assert do <= O_TOL and dl <= LSE_TOL, (cfg.name, do, dl)
    del ws
    torch.cuda.empty_cache()


@pytest.mark.parametrize("reduce,kind", [("per_query_head", "logit"), ("max", "prob")])
def test_fullsize_score_variants_qwen64k(reduce, kind):
    """The score variants at full size (qwen64k, 28/4 heads): per-query-head selection
    (scores, indices and passing buffers per query head) and probability scores (probe
    rows' lse by the attention kernel, then the score kernel).  Every score of hosts
    0..H-2 against the fp64 oracle (probabilities in the log domain), selection
    bit-exact on the GPU's own scores, sampled outputs against the oracle re-run with
    the GPU's indices."""
    cfg = CONFIGS["qwen64k"]
    g = generate(cfg)
    sizes = [int(x) for x in g["host_sizes"]]
    dev = {x: to_device_bf16(g[x]) for x in ("q", "k", "v")}
    plan = sab.Plan(cfg.n_visual, cfg.n_text, cfg.n_hosts, sizes, cfg.anchor, cfg.passing, cfg.probe_r,
                    cfg.hq, cfg.hkv, cfg.head_dim)
    plan.set_score_reduce(reduce)
    plan.set_score_kind(kind)
    ws = plan.new_workspace()
    scores = torch.empty(plan.scores_shape(), dtype=torch.float32, device="cuda")
    idx = torch.empty(plan.idx_shape(), dtype=torch.int32, device="cuda")
    o, lse = sab.attn_prefill(plan, dev["q"], dev["k"], dev["v"], scores_out=scores, idx_out=idx, workspace=ws)
    sab.check_device_error(plan, ws)
    off = orc.host_offsets(sizes)
    q, k, v = (LazyF64(g[x]) for x in ("q", "k", "v"))
    scale = 1.0 / math.sqrt(cfg.head_dim)
    G = cfg.hq // cfg.hkv
    sc = scores.cpu().numpy()
    for h in range(cfg.n_hosts - 1):
        a, e = int(off[h]), int(off[h + 1])
        sub = orc.host_offsets([e - a])
        qh, kh = q[a:e], k[a:e]
        ref = orc.probe_scores(qh, kh, sub, cfg.probe_r, scale, "none" if reduce == "per_query_head" else reduce, kind)
        _, tol = _score_tolerance_and_ref(qh, kh, sub, cfg.probe_r, scale, [0])
        t = np.stack([tol[(0, gg)] for gg in range(cfg.hkv)])
        if reduce == "per_query_head":
            t = np.repeat(t, G, axis=0)
        got = sc[:, a:e].astype(np.float64)
        if kind == "prob":
            err = np.abs(np.log(got) - np.log(ref))
            assert (err <= t + 5e-4).all(), (h, float(err.max()))
        else:
            assert (np.abs(got - ref) <= t).all(), (h, float(np.abs(got - ref).max()))
    sel = idx.cpu().numpy().astype(np.int64)
    np.testing.assert_array_equal(sel, orc.select_passing(sc, off, cfg.anchor, cfg.passing))
    rng = np.random.default_rng(cfg.seed + 2)
    rows, heads = _sample_rows(cfg, off, rng, n_random=24)
    O_ref, L_ref = orc.attention_rows(q, k, v, off, cfg.anchor, sel, scale, rows, heads)
    rt, ht = torch.tensor(rows, device="cuda"), torch.tensor(heads, device="cuda")
    do = np.abs(o[rt, ht].float().cpu().numpy() - O_ref).max()
    dl = np.abs(lse[ht, rt].cpu().numpy() - L_ref).max()
    assert do <= O_TOL and dl <= LSE_TOL, (reduce, kind, do, dl)
    plan.close()
    del dev, o, lse, ws
    torch.cuda.empty_cache()


@pytest.mark.parametrize("flow", ["two_stage", "one_pass"])
def test_fullsize_sharded_emulated(fullsize_run, flow):
    """The sharded prefill at full size, its W ranks run one after another on this GPU
    (128k: W = 8, ZigZag; stress: W = 4, ZigZag, uneven blocks), the exchange moved by
    device copies between the stages: every host's selection equals the one-GPU
    prefill's bit for bit; O and lse of every row within the bf16 tolerances of the
    one-GPU prefill's; sampled outputs against the oracle."""
    r = fullsize_run
    cfg = r["cfg"]
    worlds = {"128k": 8, "stress": 4}
    if cfg.name not in worlds:
        pytest.skip("sharded prefill checked at full size on the 128k and stress workloads")
    W, dev = worlds[cfg.name], r["dev"]
    owner = sab.shard_owners(cfg.n_hosts, W, "zigzag")
    ranks = []
    for rk in range(W):
        p = sab.Plan(cfg.n_visual, cfg.n_text, cfg.n_hosts, r["sizes"], cfg.anchor, cfg.passing, cfg.probe_r,
                     cfg.hq, cfg.hkv, cfg.head_dim)
        p.set_shard(rk, W, owner)
        ranks.append((p, p.shard_layout(), torch.zeros(p.shard_workspace_bytes, dtype=torch.uint8, device="cuda")))
    o = torch.zeros_like(dev["q"])
    lse = torch.zeros_like(r["lse"])
    L0 = ranks[0][1]

    def exchange(off, per):
        off, per = int(off), int(per)
        for rk, (_, _, ws) in enumerate(ranks):
            for _, _, ws2 in ranks:
                if ws2 is not ws:
                    ws2[off + rk * per: off + (rk + 1) * per].copy_(ws[off + rk * per: off + (rk + 1) * per])

    from sequence_approximate_attention_b200 import _lib
    stages = ((_lib.SPAVA_SHARD_SELECT, _lib.SPAVA_SHARD_LOCAL, _lib.SPAVA_SHARD_REMOTE, _lib.SPAVA_SHARD_MERGE)
              if flow == "two_stage" else (_lib.SPAVA_SHARD_SELECT, _lib.SPAVA_SHARD_ATTEND, _lib.SPAVA_SHARD_MERGE))
    for sid in stages:
        for p, _, ws in ranks:
            sab.shard_stage(p, sid, dev["q"], dev["k"], dev["v"], o, lse, ws)
        if sid == _lib.SPAVA_SHARD_SELECT:
            exchange(L0.pass_k_offset, L0.pass_bytes_per_rank)
            exchange(L0.pass_v_offset, L0.pass_bytes_per_rank)
        elif sid in (_lib.SPAVA_SHARD_LOCAL, _lib.SPAVA_SHARD_ATTEND):
            exchange(L0.text_o_offset, L0.text_o_bytes_per_rank)
            exchange(L0.text_lse_offset, L0.text_lse_bytes_per_rank)
    for p, _, ws in ranks:
        sab.check_device_error(p, ws)
    H, P, hkv = cfg.n_hosts, cfg.passing, cfg.hkv
    sel = np.empty_like(r["idx"])
    for h in range(H - 1):
        p, L, ws = ranks[owner[h]]
        idx = ws[int(L.idx_offset): int(L.idx_offset) + (H - 1) * hkv * P * 4].view(torch.int32).view(H - 1, hkv, P)
        sel[h] = idx[h].cpu().numpy()
    np.testing.assert_array_equal(sel, r["idx"])
    do = (o.float() - r["o"].float()).abs().max().item()
    dl = (lse - r["lse"]).abs().max().item()
    assert do <= O_TOL and dl <= LSE_TOL, (cfg.name, do, dl)
    off = orc.host_offsets(r["sizes"])
    q, k, v = (LazyF64(r["g"][x]) for x in ("q", "k", "v"))
    rows, heads = _sample_rows(cfg, off, np.random.default_rng(cfg.seed + 2))
    O_ref, L_ref = orc.attention_rows(q, k, v, off, cfg.anchor, sel, 1.0 / math.sqrt(cfg.head_dim), rows, heads)
    rt, ht = torch.tensor(rows, device="cuda"), torch.tensor(heads, device="cuda")
    assert np.abs(o[rt, ht].float().cpu().numpy() - O_ref).max() <= O_TOL
    assert np.abs(lse[ht, rt].cpu().numpy() - L_ref).max() <= LSE_TOL
    for p, _, _ in ranks:
        p.close()
    del ranks, o, lse
    torch.cuda.empty_cache()
