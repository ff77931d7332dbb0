"""GPU parity of the sharded prefill's stages (spava_plan_set_shard / spava_shard_stage),
in both forms (LOCAL + REMOTE, or the one-pass ATTEND), with the ranks emulated one
after another on one GPU.

Every emulated rank has its own plan, workspace and full-size q/k/v/o/lse buffers in
which only its own host rows and the text rows hold the inputs; every other row holds
finite garbage (large random values), so any use of a row the rank does not own
shows up in the result.  Between the stages the test moves the bytes a collective
would move (each rank's contiguous part of the exchange buffers to every rank, the
anchor rows from the owner of host 0); no kernel waits for another.

Checked: the selection of every host equals the one-GPU spava_score_select's bit for
bit (same score kernel tiles) and its scores are within the fp32 bound of the oracle's;
the assembled O/lse (host rows from their owner, text rows from any rank -- identical
on all) against the oracle's approximate attention with those indices; the text rows
equal on every rank; nothing non-finite anywhere.
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
from sequence_approximate_attention_b200 import _lib  # noqa: E402

TINY = CONFIGS["tiny"]
BASE = TINY.with_(n_visual=1024, n_hosts=4, head_dim=128, hq=8, hkv=2, anchor=64, passing=64, probe_r=32,
                  n_text=40)
CASES = {
    # name: (cfg, host sizes or None, owner, score reduce, score kind)
    "zigzag_w2": (BASE, None, [0, 1, 1, 0], "max", "logit"),
    "contiguous_w2": (BASE, None, [0, 0, 1, 1], "max", "logit"),
    "zigzag_w4_uneven_d64_no_text": (BASE.with_(n_hosts=8, head_dim=64, n_text=0, anchor=16, passing=48),
                                     [96, 160, 128, 112, 144, 128, 100, 156], [0, 1, 2, 3, 3, 2, 1, 0],
                                     "max", "logit"),
    "w3_uneven_slots": (BASE.with_(n_hosts=6, n_visual=1152, n_text=300, passing=40),
                        None, [2, 0, 1, 2, 0, 1], "max", "logit"),
    "per_query_head_w2": (BASE, None, [1, 0, 0, 1], "per_query_head", "logit"),
    "mean_w2": (BASE.with_(hq=14, hkv=2), [192, 320, 256, 256], [0, 1, 1, 0], "mean", "logit"),
    "prob_w2": (BASE, None, [0, 1, 1, 0], "max", "prob"),
    "one_host": (BASE.with_(n_hosts=1), None, [0], "max", "logit"),
    "no_anchor_no_passing_w2": (BASE.with_(anchor=0, passing=0), None, [0, 1, 1, 0], "max", "logit"),
    "idle_rank_w3": (BASE, None, [0, 0, 2, 2], "max", "logit"),   # rank 1 runs no host
    # owners from the oracle's longest-first rule on these uneven blocks (3 ranks)
    "longest_first_w3_uneven": (BASE.with_(n_hosts=8, head_dim=64, anchor=16, passing=48),
                                [96, 160, 128, 112, 144, 128, 100, 156], "longest_first:3", "max", "logit"),
}


def _owner(cfg, sizes, owner):
    if isinstance(owner, str):
        world = int(owner.split(":")[1])
        cost = orc.host_costs(sizes, cfg.anchor, cfg.passing, cfg.n_text)
        return orc.longest_first_owners(cost, world).tolist()
    return owner


def _garbage_like(t, rng_seed):
    g = torch.Generator(device="cpu").manual_seed(rng_seed)
    return (torch.randn(t.shape, generator=g) * 40.0).to(torch.bfloat16).to(t.device)


def _run_emulated(name, flow="two_stage"):
    cfg, sizes, owner, mode, kind = CASES[name]
    cfg = cfg.with_(uneven=None)
    g, f64, dev = inputs(cfg)
    sizes = np.asarray(sizes if sizes is not None else g["host_sizes"], dtype=np.int32)
    off = orc.host_offsets(sizes)
    owner = _owner(cfg, sizes, owner)
    H, N, NT, A = cfg.n_hosts, cfg.n_visual, cfg.n_total, cfg.anchor
    world = max(owner) + 1
    ranks = []
    for r in range(world):
        plan = make_plan(sab, cfg, sizes)
        plan.set_score_reduce(mode)
        plan.set_score_kind(kind)
        plan.set_shard(r, world, owner)
        L = plan.shard_layout()
        ws = torch.zeros(int(L.workspace_bytes), dtype=torch.uint8, device="cuda")
        bufs = {}
        for x in ("q", "k", "v"):
            t = _garbage_like(dev[x], 100 * r + ord(x))
            for h in range(H):
                if owner[h] == r:
                    t[off[h]:off[h + 1]] = dev[x][off[h]:off[h + 1]]
            t[N:] = dev[x][N:]
            bufs[x] = t
        o = _garbage_like(dev["q"], 7 + r)
        lse = torch.full((cfg.hq, NT), float("nan"), device="cuda")
        ranks.append(dict(plan=plan, L=L, ws=ws, o=o, lse=lse, **bufs))

    def stage(sid):
        for R in ranks:
            sab.shard_stage(R["plan"], sid, R["q"], R["k"], R["v"], R["o"], R["lse"], R["ws"])

    def allgather(off_name, per_name):
        L0 = ranks[0]["L"]
        o0, per = int(getattr(L0, off_name)), int(getattr(L0, per_name))
        if per == 0:
            return
        parts = [R["ws"][o0 + r * per: o0 + (r + 1) * per].clone() for r, R in enumerate(ranks)]
        for R in ranks:
            for r in range(world):
                R["ws"][o0 + r * per: o0 + (r + 1) * per] = parts[r]

    stage(_lib.SPAVA_SHARD_SELECT)
    allgather("pass_k_offset", "pass_bytes_per_rank")
    allgather("pass_v_offset", "pass_bytes_per_rank")
    src = ranks[owner[0]]
    for R in ranks:
        R["k"][:A] = src["k"][:A]
        R["v"][:A] = src["v"][:A]
    if flow == "two_stage":
        stage(_lib.SPAVA_SHARD_LOCAL)
        allgather("text_o_offset", "text_o_bytes_per_rank")
        allgather("text_lse_offset", "text_lse_bytes_per_rank")
        stage(_lib.SPAVA_SHARD_REMOTE)
    else:
        stage(_lib.SPAVA_SHARD_ATTEND)
        allgather("text_o_offset", "text_o_bytes_per_rank")
        allgather("text_lse_offset", "text_lse_bytes_per_rank")
    stage(_lib.SPAVA_SHARD_MERGE)
    for R in ranks:
        sab.check_device_error(R["plan"], R["ws"])
    torch.cuda.synchronize()
    return cfg, f64, dev, sizes, off, owner, ranks


@pytest.mark.parametrize("flow", ["two_stage", "one_pass"])
@pytest.mark.parametrize("name", list(CASES))
def test_sharded_stages_match_oracle(name, flow):
    cfg, f64, dev, sizes, off, owner, ranks = _run_emulated(name, flow)
    H, N, NT = cfg.n_hosts, cfg.n_visual, cfg.n_total
    plan0 = ranks[0]["plan"]
    rows = plan0.score_rows
    O = torch.empty_like(dev["q"])
    lse = torch.empty((cfg.hq, NT), device="cuda")
    sel = np.zeros((max(H - 1, 0), rows, cfg.passing), dtype=np.int64)
    scores = np.zeros((rows, N), dtype=np.float32)
    for h in range(H):
        R = ranks[owner[h]]
        O[off[h]:off[h + 1]] = R["o"][off[h]:off[h + 1]]
        lse[:, off[h]:off[h + 1]] = R["lse"][:, off[h]:off[h + 1]]
        if h < H - 1 and cfg.passing > 0 and H > 1:
            L = R["L"]
            ws = R["ws"]
            idx = ws[int(L.idx_offset): int(L.idx_offset) + (H - 1) * rows * cfg.passing * 4].view(torch.int32)
            sel[h] = idx.view(H - 1, rows, cfg.passing)[h].cpu().numpy()
            sc = ws[int(L.scores_offset): int(L.scores_offset) + rows * N * 4].view(torch.float32).view(rows, N)
            scores[:, off[h]:off[h + 1]] = sc[:, off[h]:off[h + 1]].cpu().numpy()
    if NT > N:
        O[N:] = ranks[0]["o"][N:]
        lse[:, N:] = ranks[0]["lse"][:, N:]
        for R in ranks[1:]:   # every rank merged the same gathered slots
            assert torch.equal(R["o"][N:].view(torch.int16), ranks[0]["o"][N:].view(torch.int16)), name
            assert torch.equal(R["lse"][:, N:], ranks[0]["lse"][:, N:]), name
    scale = 1.0 / math.sqrt(cfg.head_dim)
    if H > 1 and cfg.passing > 0:
        # the same selection as one GPU running every host
        ref_plan = make_plan(sab, cfg, sizes)
        ref_plan.set_score_reduce(plan0.score_reduce)
        ref_plan.set_score_kind(plan0.score_kind)
        sc1, idx1 = sab.score_select(ref_plan, dev["q"], dev["k"])
        torch.cuda.synchronize()
        np.testing.assert_array_equal(sel, idx1.cpu().numpy())
        ref_plan.close()
        if plan0.score_kind == "logit":
            reduce = "none" if plan0.score_reduce == "per_query_head" else plan0.score_reduce
            ref = orc.probe_scores(f64["q"], f64["k"], off, cfg.probe_r, scale, head_reduce=reduce)
            G = cfg.hq // cfg.hkv
            tol = score_tolerance(f64["q"], f64["k"], off, cfg.probe_r, scale)
            if reduce == "none":
                tol = np.repeat(tol, G, axis=0)
            n_sc = int(off[H - 1])
            assert (np.abs(scores[:, :n_sc] - ref[:, :n_sc]) <= tol[:, :n_sc]).all(), name
    O_ref, L_ref = orc.approx_attention(f64["q"], f64["k"], f64["v"], off, cfg.anchor,
                                        sel if H > 1 else None, scale)
    compare_attention(O, lse, O_ref, L_ref, name)
    for R in ranks:
        R["plan"].close()


def test_stage_needs_a_shard():
    cfg = BASE
    plan = make_plan(sab, cfg, [256] * 4)
    ws = torch.zeros(1 << 20, dtype=torch.uint8, device="cuda")
    assert plan.lib.spava_shard_stage(plan.handle, 0, None, None, None, None, None,
                                      ws.data_ptr(), None) == _lib.SPAVA_ERR_INVALID_ARG
    with pytest.raises(sab.SpavaError):
        plan.set_shard(2, 2, [0, 1, 1, 0])
    with pytest.raises(sab.SpavaError):
        plan.set_shard(0, 2, [0, 1, 2, 0])
    plan.set_shard(0, 2, [0, 1, 1, 0])
    assert plan.lib.spava_shard_stage(plan.handle, 9, None, None, None, None, None,
                                      ws.data_ptr(), None) == _lib.SPAVA_ERR_INVALID_ARG
    assert plan.lib.spava_shard_stage(plan.handle, _lib.SPAVA_SHARD_LOCAL, None, None, None, None, None,
                                      ws.data_ptr(), None) == _lib.SPAVA_ERR_INVALID_ARG
    plan.close()


@pytest.mark.parametrize("world", [1, 2, 3, 5])
def test_plan_owners_match_oracle(world):
    """spava_plan_shard_owners: longest first from the plan's per-host costs (uneven
    blocks, text rows) equals the oracle's rule on its host_costs; the pairing policies
    equal spava_shard_owners'."""
    cfg = BASE.with_(n_hosts=8, head_dim=64, anchor=16, passing=48, n_text=70)
    sizes = [96, 160, 128, 112, 144, 128, 100, 156]
    plan = make_plan(sab, cfg, sizes)
    want = orc.longest_first_owners(orc.host_costs(sizes, cfg.anchor, cfg.passing, cfg.n_text), world)
    assert plan.shard_owners(world, "longest_first") == want.tolist()
    if 8 % (2 * world) == 0:
        assert plan.shard_owners(world, "zigzag") == orc.zigzag_owners(8, world).tolist()
    assert plan.shard_owners(world if 8 % world == 0 else 1, "contiguous") == \
        orc.contiguous_owners(8, world if 8 % world == 0 else 1).tolist()
    plan.close()


def test_stage_kernel_labels_for_a_rank_without_scored_hosts():
    """Rank 0 runs only the last host (nothing to score): SELECT launches nothing and
    the timing hook names ATTEND's kernels as the unpack and the attention (its empty
    work lists must not share an address with the one it runs)."""
    cfg = BASE
    plan = make_plan(sab, cfg, [256] * 4)
    plan.set_shard(0, 2, [1, 1, 1, 0])
    g, _, dev = inputs(cfg)
    ws = torch.zeros(plan.shard_workspace_bytes, dtype=torch.uint8, device="cuda")
    o = torch.zeros_like(dev["q"])
    lse = torch.zeros((cfg.hq, cfg.n_total), device="cuda")
    plan.profile_begin(64)
    for sid in (_lib.SPAVA_SHARD_SELECT, _lib.SPAVA_SHARD_ATTEND, _lib.SPAVA_SHARD_MERGE):
        sab.shard_stage(plan, sid, dev["q"], dev["k"], dev["v"], o, lse, ws)
    names = [n for n, _ in plan.profile_read()]
    plan.profile_end()
    assert names == ["text_slot_fill", "unpack_passing", "attention", "lse_merge"], names
    plan.close()
