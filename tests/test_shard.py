"""Host side of the sharded prefill, on CPU (no GPU needed).

* spava_shard_owners (the library's ZigZag and contiguous maps) against the oracle's,
  integer for integer, and its refusals;
* the orchestration of ShardedPrefill over two gloo ranks, with a stand-in plan whose
  stages write rank-tagged bytes and check, when they run, that the exchange before
  them delivered every rank's part: the passing parts all-gathered and the anchor rows
  broadcast before REMOTE, the text partials all-gathered before MERGE, the stages in
  order, and the same collectives on every rank.
"""

import ctypes
import os
import socket
import sys
from types import SimpleNamespace

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from oracle import spava_oracle as orc
from sequence_approximate_attention_b200 import _lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _owners(lib, H, W, policy):
    arr = (ctypes.c_int32 * H)()
    st = lib.spava_shard_owners(H, W, policy, arr)
    return st, [int(x) for x in arr]


@pytest.mark.parametrize("W", [1, 2, 3, 4, 8])
@pytest.mark.parametrize("rounds", [1, 2, 4])
def test_shard_owners_match_oracle(lib, W, rounds):
    H = 2 * W * rounds
    st, zz = _owners(lib, H, W, _lib.SPAVA_SHARD_ZIGZAG)
    assert st == _lib.SPAVA_OK
    assert zz == orc.zigzag_owners(H, W).tolist()
    st, ct = _owners(lib, H, W, _lib.SPAVA_SHARD_CONTIGUOUS)
    assert st == _lib.SPAVA_OK
    assert ct == orc.contiguous_owners(H, W).tolist()


@pytest.mark.parametrize("H,W,policy", [(6, 4, _lib.SPAVA_SHARD_ZIGZAG), (6, 4, _lib.SPAVA_SHARD_CONTIGUOUS),
                                        (8, 0, _lib.SPAVA_SHARD_ZIGZAG), (0, 2, _lib.SPAVA_SHARD_ZIGZAG),
                                        (8, 2, 7)])
def test_shard_owners_refuse_bad_sizes(lib, H, W, policy):
    arr = (ctypes.c_int32 * max(H, 1))(*([-5] * max(H, 1)))
    assert lib.spava_shard_owners(H, W, policy, arr) == _lib.SPAVA_ERR_INVALID_ARG
    assert list(arr) == [-5] * max(H, 1)   # nothing written
    assert lib.spava_shard_owners(8, 2, _lib.SPAVA_SHARD_ZIGZAG, None) == _lib.SPAVA_ERR_INVALID_ARG


def test_set_shard_refuses_null_plan(lib):
    arr = (ctypes.c_int32 * 2)(0, 0)
    assert lib.spava_plan_set_shard(None, 0, 1, arr) == _lib.SPAVA_ERR_INVALID_ARG
    assert lib.spava_plan_shard_owners(None, 2, _lib.SPAVA_SHARD_LONGEST_FIRST, arr) == _lib.SPAVA_ERR_INVALID_ARG
    assert lib.spava_shard_query(None, None) == _lib.SPAVA_ERR_INVALID_ARG
    assert lib.spava_shard_stage(None, 0, None, None, None, None, None, None, None) == _lib.SPAVA_ERR_INVALID_ARG


# ------------------------------------------------------------------ gloo orchestration
PASS_PART, TEXT_O_PART, TEXT_L_PART = 48, 32, 16


class StandInPlan:
    """Duck-typed plan for ShardedPrefill on CPU tensors.  Layout: the documented
    rank-major runs, with small made-up part sizes."""

    def __init__(self, n_hosts, anchor, n_visual, n_text, log):
        self.n_hosts, self.anchor, self.n_visual, self.n_text = n_hosts, anchor, n_visual, n_text
        self.n_total = n_visual + n_text
        self.hq = 2
        B = n_visual // n_hosts
        self.offsets = [h * B for h in range(n_hosts + 1)]
        self.device = torch.device("cpu")
        self.log = log

    def set_shard(self, rank, world, owner):
        self.rank, self.world, self.owner = rank, world, list(owner)
        o = 256
        lay = {}
        for name, part in (("pass_k", PASS_PART), ("pass_v", PASS_PART), ("text_o", TEXT_O_PART),
                           ("text_lse", TEXT_L_PART)):
            lay[name + "_offset"] = o
            o += world * part
        self.lay = SimpleNamespace(workspace_bytes=o, pass_bytes_per_rank=PASS_PART,
                                   text_o_bytes_per_rank=TEXT_O_PART, text_lse_bytes_per_rank=TEXT_L_PART, **lay)

    def shard_layout(self):
        return self.lay

    def _run(self, ws, name, per):
        off = getattr(self.lay, name + "_offset")
        return ws[off: off + self.world * per].view(self.world, per)

    def shard_stage(self, stage, q, k, v, o, lse, ws, stream=None):
        r = self.rank
        self.log.append(stage)
        pk, pv = self._run(ws, "pass_k", PASS_PART), self._run(ws, "pass_v", PASS_PART)
        to, tl = self._run(ws, "text_o", TEXT_O_PART), self._run(ws, "text_lse", TEXT_L_PART)
        if stage == _lib.SPAVA_SHARD_SELECT:
            pk[r] = 10 + r
            pv[r] = 20 + r
        elif stage == _lib.SPAVA_SHARD_LOCAL:
            to[r] = 30 + r
            tl[r] = 40 + r
        elif stage in (_lib.SPAVA_SHARD_REMOTE, _lib.SPAVA_SHARD_ATTEND):
            for rr in range(self.world):
                assert (pk[rr] == 10 + rr).all() and (pv[rr] == 20 + rr).all(), "passing exchange incomplete"
            assert (k[:self.anchor] == 7).all() and (v[:self.anchor] == 8).all(), "anchor rows missing"
            for h in range(self.n_hosts):
                if self.owner[h] == r:
                    o[self.offsets[h]:self.offsets[h + 1]] = r + 1
            if stage == _lib.SPAVA_SHARD_ATTEND:   # the one-pass form also fills the text slots
                to[r] = 30 + r
                tl[r] = 40 + r
        elif stage == _lib.SPAVA_SHARD_MERGE:
            for rr in range(self.world):
                assert (to[rr] == 30 + rr).all() and (tl[rr] == 40 + rr).all(), "text exchange incomplete"
            o[self.n_visual:] = 99


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, owner, overlap, out):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    from sequence_approximate_attention_b200.sharded import ShardedPrefill
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    log = []
    H, A, N, T = len(owner), 3, 64, 5
    plan = StandInPlan(H, A, N, T, log)
    sp = ShardedPrefill(plan, rank, world, owner, overlap=overlap)
    q = torch.zeros(N + T, 2, 4)
    k = torch.zeros(N + T, 1, 4)
    v = torch.zeros(N + T, 1, 4)
    if owner[0] == rank:   # the anchor's owner holds rows [0, A)
        k[:A], v[:A] = 7, 8
    o, _ = sp.forward(q, k, v)
    out[rank] = (log, o[:, 0, 0].tolist(), sp.owned_rows())
    dist.barrier()
    dist.destroy_process_group()


@pytest.mark.parametrize("overlap", [True, False])
@pytest.mark.parametrize("owner", [[0, 1, 1, 0], [1, 0, 0, 1], [0, 0, 1, 1]])
def test_sharded_orchestration_two_gloo_ranks(owner, overlap):
    world = 2
    with mp.get_context("spawn").Manager() as man:
        out = man.dict()
        mp.spawn(_rank_main, args=(world, _free_port(), owner, overlap, out), nprocs=world, join=True)
        res = dict(out)
    B = 64 // len(owner)
    stages = ([_lib.SPAVA_SHARD_SELECT, _lib.SPAVA_SHARD_LOCAL, _lib.SPAVA_SHARD_REMOTE, _lib.SPAVA_SHARD_MERGE]
              if overlap else [_lib.SPAVA_SHARD_SELECT, _lib.SPAVA_SHARD_ATTEND, _lib.SPAVA_SHARD_MERGE])
    for r in range(world):
        log, o, rows = res[r]
        assert log == stages
        o = np.array(o)
        for h, own in enumerate(owner):
            if own == r:
                assert (o[h * B:(h + 1) * B] == r + 1).all()
                assert (h * B, (h + 1) * B) in rows
        assert (o[64:] == 99).all()


@pytest.mark.parametrize("W", [1, 2, 3, 8])
@pytest.mark.parametrize("seed", [0, 1, 2])
def test_owners_by_cost_match_oracle(lib, W, seed):
    """spava_shard_owners_by_cost (longest first) against the oracle's, integer for
    integer, with many equal costs (ties go to the lower host, then the lower rank)."""
    rng = np.random.default_rng(seed)
    H = 16
    cost = rng.integers(0, 6, size=H).astype(np.int64) * 1000
    arr_c = (ctypes.c_int64 * H)(*[int(x) for x in cost])
    out = (ctypes.c_int32 * H)()
    assert lib.spava_shard_owners_by_cost(H, W, arr_c, out) == _lib.SPAVA_OK
    assert list(out) == orc.longest_first_owners(cost, W).tolist()
    arr_c[3] = -1
    assert lib.spava_shard_owners_by_cost(H, W, arr_c, out) == _lib.SPAVA_ERR_INVALID_ARG


# ------------------------------------------------------------------ a rank that fails
def _failing_rank_main(rank, world, port, out):
    import datetime

    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    from sequence_approximate_attention_b200.sharded import ShardedPrefill
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=5))
    log = []
    plan = StandInPlan(4, 3, 64, 5, log)
    sp = ShardedPrefill(plan, rank, world, [0, 1, 1, 0])
    q, k, v = torch.zeros(69, 2, 4), torch.zeros(69, 1, 4), torch.zeros(69, 1, 4)
    if rank == 1:
        out[rank] = "left before the exchange"
        os._exit(0)   # leaves between steps: none of its collectives is in flight
    try:
        sp.forward(q, k, v)
        out[rank] = "finished"
    except RuntimeError as e:
        out[rank] = "error: " + type(e).__name__
    os._exit(0)


def test_surviving_rank_gets_an_error_not_a_hang():
    """Failure on the host side: rank 1 leaves before the first exchange; rank 0's
    all-gather ends with an error within the process group's short timeout instead of
    waiting for ever."""
    world = 2
    ctx = mp.get_context("spawn")
    with ctx.Manager() as man:
        out = man.dict()
        port = _free_port()
        procs = [ctx.Process(target=_failing_rank_main, args=(r, world, port, out)) for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(timeout=120)
        alive = [p.is_alive() for p in procs]
        for p in procs:
            if p.is_alive():
                p.kill()
        res = dict(out)
    assert not any(alive), "a rank hung"
    assert res.get(1) == "left before the exchange"
    assert res.get(0, "").startswith("error"), res
