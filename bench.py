#!/usr/bin/env python
"""Benchmark of the approximate-attention prefill (one layer) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config 128k] [--impl b200|reference]

A step is one call of spava_attn_prefill over the whole hot path (probe scoring,
top-P selection, passing gather, the attention pass, the text lse merge) on one
seeded synthetic layer whose inputs already sit in HBM.  Q/K/V of the default
workload (2.1 GB + 2 x 0.27 GB) are far larger than the 126 MB L2, so no flush is
needed between steps.  With N GPUs (torchrun, NCCL) every rank runs its own replica
of the workload (weak scaling, no data-path collective); the time is the max over
ranks.  Rank 0 prints one JSON line.

--impl reference times the fp64 CPU oracle on the host cores instead (rank 0 only),
each step a bounded sample of the same workload.
"""

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from workloads import CONFIGS, generate  # noqa: E402

METRIC = "approx-attn prefill tokens/s and % of B200 BF16 tensor peak at 128K tokens"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# ---------------------------------------------------------------- workload arithmetic
def attended_pairs(cfg, sizes):
    """(query, key) pairs the approximate attention evaluates (per query head)."""
    N, T, A, P = cfg.n_visual, cfg.n_text, cfg.anchor, cfg.passing
    pairs = 0
    for h, B in enumerate(sizes):
        B = int(B)
        pairs += B * (B + 1) // 2
        if h >= 1:
            pairs += B * (A + h * P)
    pairs += T * N + T * (T + 1) // 2
    return pairs


def dense_pairs(cfg):
    n = cfg.n_visual + cfg.n_text
    return n * (n + 1) // 2


def score_flops(cfg, sizes):
    """Tensor-core work of the score kernel: every scored key meets the R probe rows of
    each of the G query heads of its group (2 d FLOP each); the N chunks are Rc G
    columns wide, so a short last chunk still costs its full width."""
    d, hq, hkv, H, R = cfg.head_dim, cfg.hq, cfg.hkv, cfg.n_hosts, cfg.probe_r
    G = hq // hkv
    n_scored = int(sum(int(b) for b in sizes[:H - 1]))
    rc = min(max(16, 16 * (256 // (16 * G))), R)
    cols = -(-R // rc) * rc * G
    return 2.0 * d * cols * n_scored * hkv


def select_gather_bytes(cfg, sizes):
    """Algorithmic HBM bytes of the score, select and gather kernels of one step."""
    d, hq, hkv, H, P, R, N = cfg.head_dim, cfg.hq, cfg.hkv, cfg.n_hosts, cfg.passing, cfg.probe_r, cfg.n_visual
    n_scored = int(sum(int(b) for b in sizes[:H - 1]))
    score = n_scored * hkv * d * 2 + (H - 1) * R * hq * d * 2 + n_scored * hkv * 4
    select = n_scored * hkv * 4 + (H - 1) * hkv * P * 4
    gather = 2 * 2 * (H - 1) * hkv * P * d * 2 + (H - 1) * hkv * P * 4
    return {"score": score, "select": select, "gather": gather, "select_gather": select + gather,
            "score_select_gather": score + select + gather}


def attn_algorithmic_bytes(cfg):
    """DRAM bytes the attention kernel must move once: Q, K, V and the passing K/V
    read, O (bf16, visual rows) and the text partials (fp32, one per host block plus
    the causal piece) written, lse written."""
    NT, N, T, H = cfg.n_visual + cfg.n_text, cfg.n_visual, cfg.n_text, cfg.n_hosts
    d, hq, hkv, P = cfg.head_dim, cfg.hq, cfg.hkv, cfg.passing
    rd = NT * hq * d * 2 + 2 * NT * hkv * d * 2 + 2 * hkv * max(H - 1, 0) * P * d * 2
    wr = N * hq * d * 2 + hq * N * 4 + (H + 1) * T * hq * (d + 1) * 4
    return rd + wr


# The ncu traffic of the attention kernel is recorded in profiles/ together with a
# digest of the sources it was measured on (kernel and plan ordering); the bench
# reports it only while that digest still matches, else null.
TRAFFIC_NOTE = os.path.join(ROOT, "profiles", "attn_fwd_128k_traffic.md")
TRAFFIC_SOURCES = [os.path.join("sequence_approximate_attention_b200", "csrc", f)
                   for f in ("attn_kernel.cuh", "common.cuh", "tmem_ops.inc", "exp2_poly.inc", "spava.cu")]


def attn_source_digest():
    import hashlib
    h = hashlib.sha256()
    for rel in TRAFFIC_SOURCES:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def recorded_traffic(workload):
    import re
    try:
        text = open(TRAFFIC_NOTE).read()
    except OSError:
        return None
    w = re.search(r"workload:\s*(\S+)", text)
    b = re.search(r"traffic_bytes_per_launch:\s*(\d+)", text)
    dg = re.search(r"source_sha256:\s*([0-9a-f]{64})", text)
    if not (w and b and dg) or w.group(1) != workload or dg.group(1) != attn_source_digest():
        return None
    return int(b.group(1))


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in ("hbm_gbs", "bf16_tflops", "bf16_tflops_sustained")}, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


# ---------------------------------------------------------------- ranks
def max_over_ranks(value, device=None):
    """Max of a per-rank float over all ranks of the default process group (the
    value itself when no group is initialised).  NCCL needs a CUDA device tensor,
    gloo a CPU one."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(world, tokens_per_step, steps, ms_max):
    """Whole-job tokens/s: every rank runs its own replica of the workload (weak
    scaling), so the job processes world * tokens_per_step * steps tokens in the
    slowest rank's time."""
    return world * tokens_per_step * steps / (ms_max / 1e3)


# ---------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi clock/throttle samples of this process's GPU during the timed region."""

    FIELDS = ("uuid,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, uuid: str):
        self.uuid = uuid.lower().replace("gpu-", "")
        self.proc = None
        self.lines = []
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "--query-gpu=" + self.FIELDS, "--format=csv,noheader,nounits",
                                          "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        if self.thread:
            self.thread.join(timeout=2)
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [x.strip() for x in ln.split(",")]
            if len(parts) < 9 or self.uuid not in parts[0].lower():
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for nm, val in zip(names, parts[5:9]):
                if val.lower() == "active":
                    reasons.add(nm)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------- CPU oracle (baseline arm)
class LazyF64:
    """bf16 bit array viewed as float64, converted only where indexed (keeps the
    oracle's memory to what it touches)."""

    def __init__(self, bits):
        self.bits = bits
        self.shape = bits.shape

    def __getitem__(self, key):
        b = np.ascontiguousarray(self.bits[key], dtype=np.uint16)
        return (b.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


def oracle_sample(cfg, g, seed, rows=64):
    """One bounded oracle run on a fixed stratified sample of the layer: probe scoring
    and top-P selection of every host in full, then the attention of one `rows`-row
    slice of every host block and of the text rows (all heads), each slice at a
    seeded position inside its stratum.  Each stratum is extrapolated by its own
    attended key pairs (remote-heavy late hosts and the dense text rows cost
    differently per row).  Returns (seconds for the whole layer; description;
    seconds actually spent; fraction of the layer's attended pairs computed)."""
    from oracle import spava_oracle as orc
    q, k, v = LazyF64(g["q"]), LazyF64(g["k"]), LazyF64(g["v"])
    sizes = [int(x) for x in g["host_sizes"]]
    off = orc.host_offsets(sizes)
    scale = 1.0 / math.sqrt(cfg.head_dim)
    N, T, A, P = cfg.n_visual, cfg.n_text, cfg.anchor, cfg.passing
    t0 = time.perf_counter()
    sel = None
    if cfg.n_hosts > 1:
        scores = orc.probe_scores(q, k, off, cfg.probe_r, scale)
        sel = orc.select_passing(scores, off, A, P)
    t_sel = time.perf_counter() - t0
    rng = np.random.default_rng(seed)
    # strata: (first row, end row, keys before the stratum's causal part per row)
    strata = [(int(off[h]), int(off[h + 1]), (A + h * P) if h >= 1 else 0) for h in range(cfg.n_hosts)]
    if T > 0:
        strata.append((N, N + T, N))
    t_att, t_total, pairs_done = 0.0, t_sel, 0
    for a, e, remote in strata:
        n = min(rows, e - a)
        r0 = a + int(rng.integers(0, e - a - n + 1))
        r1 = r0 + n
        # pairs of a row i: the remote keys plus its causal part; text rows see [0, i]
        pairs_of = (lambda i: i + 1) if a == N else (lambda i: remote + (i - a + 1))
        sample = sum(pairs_of(i) for i in range(r0, r1))
        stratum = sum(pairs_of(i) for i in range(a, e))
        t1 = time.perf_counter()
        orc.approx_attention(q, k, v, off, A, sel, scale, row_range=(r0, r1), compact=True)
        dt = time.perf_counter() - t1
        t_att += dt
        t_total += dt * stratum / sample
        pairs_done += sample
    frac = pairs_done / attended_pairs(cfg, sizes)
    desc = (f"fp64 numpy oracle: probe scoring + top-P selection of all {cfg.n_hosts} hosts in full "
            f"({t_sel:.2f} s), then one {rows}-row slice (all {cfg.hq} heads, seeded position) of every host "
            f"block{' and of the text rows' if T > 0 else ''} ({t_att:.2f} s, {100 * frac:.2f} % of the layer's "
            f"attended pairs), each slice extrapolated by its own stratum's attended pairs")
    return t_total, desc, t_sel + t_att, frac


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        info = threadpool_info()
        return max((int(x.get("num_threads", 1)) for x in info), default=os.cpu_count())
    except Exception:
        return os.cpu_count()


def run_reference(args, cfg):
    g = generate(cfg)
    NT = cfg.n_visual + cfg.n_text
    for w in range(args.warmup):
        oracle_sample(cfg, g, 100 + w, rows=args.ref_rows)
    times = []
    wall = 0.0
    desc, frac = "", 0.0
    for s in range(args.steps):
        t, desc, w, frac = oracle_sample(cfg, g, 1000 + s, rows=args.ref_rows)
        times.append(t)
        wall += w
    t_step = statistics.median(times)
    value = NT / t_step
    cores = blas_threads()
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": t_step * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
        "ms_per_step_kind": "extrapolated: each step computes a stratified sample of the layer and scales it by "
                            "attended pairs; not a wall time per step",
        "sampled_wall_s_per_step": wall / max(1, args.steps), "sampled_fraction_of_layer": frac,
        "config": workload_config(cfg),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                         "sample": desc + f"; median of {args.steps} samples (seeds 1000..), {wall:.1f} s of CPU work"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }
    print(json.dumps(line), flush=True)


def workload_config(cfg):
    return {"workload": cfg.name, "n_visual": cfg.n_visual, "n_text": cfg.n_text, "hosts": cfg.n_hosts,
            "anchor": cfg.anchor, "passing": cfg.passing, "probe_r": cfg.probe_r, "hq": cfg.hq,
            "hkv": cfg.hkv, "head_dim": cfg.head_dim, "kv": cfg.kv_kind, "seed": cfg.seed,
            "l2": "inputs larger than L2 (no flush)", "parallelism": "replicas"}


def init_nccl(dev, world):
    """NCCL process group bound to `dev`.  The communicator comes up eagerly here, with
    file descriptor 1 pointed at stderr meanwhile: the library prints a version banner
    on rank 0 from C, and stdout must carry only the one JSON line."""
    import contextlib
    import datetime

    import torch.distributed as dist

    @contextlib.contextmanager
    def stdout_to_stderr():
        sys.stdout.flush()
        saved = os.dup(1)
        os.dup2(2, 1)
        try:
            yield
        finally:
            sys.stdout.flush()
            import ctypes
            ctypes.CDLL(None).fflush(None)   # C stdio buffers written while fd 1 was stderr
            os.dup2(saved, 1)
            os.close(saved)

    with stdout_to_stderr():
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
        dist.barrier()


# ---------------------------------------------------------------- sharded prefill
def run_sharded(args, cfg, rank, world, local):
    """--sharded POLICY: the layer's hosts spread over the N ranks (ShardedPrefill, NCCL
    exchange), total work fixed (strong scaling).  Every rank generates the same
    seeded workload and uses its own host rows and the text rows; the anchor rows
    arrive by broadcast.  value = the layer's N+T tokens per step over the max-over-ranks
    time."""
    import torch
    import torch.distributed as dist

    import sequence_approximate_attention_b200 as sab
    from sequence_approximate_attention_b200.sharded import ShardedPrefill

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world == 1 and "MASTER_ADDR" not in os.environ:
        import socket
        with socket.socket() as sk:
            sk.bind(("127.0.0.1", 0))
            port = sk.getsockname()[1]
        os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK="0", WORLD_SIZE="1")
    init_nccl(dev, world)
    g = generate(cfg)
    sizes = [int(x) for x in g["host_sizes"]]
    NT = cfg.n_visual + cfg.n_text
    d_in = {x: torch.from_numpy(g[x].view(np.int16)).view(torch.bfloat16).to(dev) for x in ("q", "k", "v")}
    plan = sab.Plan(cfg.n_visual, cfg.n_text, cfg.n_hosts, sizes, cfg.anchor, cfg.passing, cfg.probe_r,
                    cfg.hq, cfg.hkv, cfg.head_dim, device=dev)
    owner = plan.shard_owners(world, args.sharded)
    sp = ShardedPrefill(plan, rank, world, owner, overlap=args.sharded_form == "overlap")
    o = torch.empty_like(d_in["q"])
    lse = torch.empty((cfg.hq, NT), dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)
    for _ in range(max(args.warmup, 3)):
        sp.forward(d_in["q"], d_in["k"], d_in["v"], o, lse)
    sab.check_device_error(plan, sp.ws)
    clocks = ClockSampler(str(torch.cuda.get_device_properties(dev).uuid))
    clocks.start()
    time.sleep(0.3)
    dist.barrier()
    torch.cuda.synchronize(dev)
    launches0 = sp.launches
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev0.record(stream)
    for _ in range(args.steps):
        sp.forward(d_in["q"], d_in["k"], d_in["v"], o, lse)
    ev1.record(stream)
    torch.cuda.synchronize(dev)
    dist.barrier()
    clk = clocks.stop()
    sab.check_device_error(plan, sp.ws)
    ms_total = max_over_ranks(ev0.elapsed_time(ev1), dev)
    if rank == 0:
        conf = workload_config(cfg)
        conf.update({"parallelism": f"sharded-{args.sharded}-{args.sharded_form}", "owner": owner,
                     "l2": "inputs larger than L2 (no flush)"})
        line = {"metric": METRIC, "value": NT * args.steps / (ms_total / 1e3), "unit": "tokens/s", "n_gpus": world,
                "steps": args.steps, "warmup": max(args.warmup, 3), "ms_per_step": ms_total / args.steps,
                "higher_is_better": True, "scaling": "strong", "vs_baseline": None, "dtype": "bf16",
                "data": "synthetic", "impl": "b200", "config": conf, "roofline": None, "cpu_baseline": None,
                "e2e": None, "gpu_launches": sp.launches - launches0, "clocks": clk,
                "note": "one layer's hosts spread over the ranks; inputs resident on every rank; the exchange "
                        "(NCCL all-gathers and broadcast) inside the timed region"}
        print(json.dumps(line), flush=True)
    del sp
    dist.barrier()
    dist.destroy_process_group()
    plan.close()


# ---------------------------------------------------------------- sharded prefill, ranks emulated
# the part of a layer each kernel of the timing hook belongs to
KERNEL_PART = {"probe_lse": "select", "score": "select", "select_gather": "select", "score_keys": "attention",
               "attention_local": "attention", "unpack_passing": "attention", "attention_remote": "attention",
               "attention": "attention", "text_slot_fill": "attention", "lse_merge": "merge"}
PARTS = ("select", "attention", "merge")


def shard_emulate(cfg, sizes, q, k, v, world, policy, steps, warmup, flow):
    """Per-rank compute of the sharded prefill with the W ranks emulated on one GPU:
    every rank's plan runs its stages in the order a W-GPU job would (every SELECT,
    the exchange, every LOCAL (or ATTEND), the text exchange, every REMOTE, every
    MERGE), the exchanged bytes moved by device copies between the stages, every
    kernel of each rank timed by the library's timing hook (CUDA events on the
    launching stream).  A rank's compute is the sum of its kernel times: what its own
    GPU would spend.  The collectives are not timed (one GPU)."""
    import torch

    import sequence_approximate_attention_b200 as sab
    from sequence_approximate_attention_b200 import _lib
    flows = {"two_stage": (_lib.SPAVA_SHARD_SELECT, _lib.SPAVA_SHARD_LOCAL, _lib.SPAVA_SHARD_REMOTE,
                           _lib.SPAVA_SHARD_MERGE),
             "one_pass": (_lib.SPAVA_SHARD_SELECT, _lib.SPAVA_SHARD_ATTEND, _lib.SPAVA_SHARD_MERGE)}
    dev = q.device

    def new_plan():
        return sab.Plan(cfg.n_visual, cfg.n_text, cfg.n_hosts, sizes, cfg.anchor, cfg.passing, cfg.probe_r,
                        cfg.hq, cfg.hkv, cfg.head_dim, device=dev)

    probe = new_plan()
    owner = probe.shard_owners(world, policy)
    probe.close()
    ranks = []
    for r in range(world):
        p = new_plan()
        p.set_shard(r, world, owner)
        L = p.shard_layout()
        ranks.append({"plan": p, "L": L, "ws": torch.zeros(int(L.workspace_bytes), dtype=torch.uint8, device=dev)})
    o = torch.zeros_like(q)
    lse = torch.zeros((cfg.hq, cfg.n_visual + cfg.n_text), dtype=torch.float32, device=dev)
    L0 = ranks[0]["L"]

    def exchange(off, per):
        off, per = int(off), int(per)
        for r, R in enumerate(ranks):
            part = R["ws"][off + r * per: off + (r + 1) * per]
            for S in ranks:
                if S is not R:
                    S["ws"][off + r * per: off + (r + 1) * per].copy_(part)

    def layer():
        for sid in flows[flow]:
            for R in ranks:
                sab.shard_stage(R["plan"], sid, q, k, v, o, lse, R["ws"])
            if sid == _lib.SPAVA_SHARD_SELECT:
                exchange(L0.pass_k_offset, L0.pass_bytes_per_rank)
                exchange(L0.pass_v_offset, L0.pass_bytes_per_rank)
            elif sid in (_lib.SPAVA_SHARD_LOCAL, _lib.SPAVA_SHARD_ATTEND):
                exchange(L0.text_o_offset, L0.text_o_bytes_per_rank)
                exchange(L0.text_lse_offset, L0.text_lse_bytes_per_rank)

    for _ in range(warmup):
        layer()
    torch.cuda.synchronize(dev)
    for R in ranks:
        R["plan"].profile_begin(steps * 16 + 16)
    for _ in range(steps):
        layer()
    torch.cuda.synchronize(dev)
    per_stage = np.zeros((world, len(PARTS)))   # [rank][part] ms per layer
    for r, R in enumerate(ranks):
        for name, ms in R["plan"].profile_read():
            per_stage[r, PARTS.index(KERNEL_PART[name])] += ms / steps
        R["plan"].profile_end()
        R["plan"].close()
    per_rank = per_stage.sum(axis=1)
    anchor_bytes = 2 * cfg.anchor * cfg.hkv * cfg.head_dim * 2
    return {
        "owner": owner,
        "rank_ms": [round(float(x), 4) for x in per_rank],
        "part_ms": {n: [round(float(x), 4) for x in per_stage[:, i]] for i, n in enumerate(PARTS)},
        "max_ms": float(per_rank.max()), "mean_ms": float(per_rank.mean()),
        "balance": float(per_rank.max() / per_rank.mean()),
        "exchange_bytes_per_rank": {"passing_kv": 2 * int(L0.pass_bytes_per_rank),
                                    "text_partials": int(L0.text_o_bytes_per_rank + L0.text_lse_bytes_per_rank),
                                    "anchor_broadcast": anchor_bytes},
    }


def run_shard_emulate(args, cfg):
    """--shard-emulate: one JSON line per (world W, ownership policy, form): per-rank
    compute (select, attention and merge parts), its max and mean, the balance
    (max / mean), the one-GPU spava_attn_prefill time on the same inputs and the
    compute-only speed-up the slowest rank allows.  Not the bench contract's line."""
    import torch

    import sequence_approximate_attention_b200 as sab
    g = generate(cfg)
    sizes = [int(x) for x in g["host_sizes"]]
    dev = torch.device("cuda", torch.cuda.current_device())
    q, k, v = (torch.from_numpy(g[x].view(np.int16)).view(torch.bfloat16).to(dev) for x in ("q", "k", "v"))
    p = sab.Plan(cfg.n_visual, cfg.n_text, cfg.n_hosts, sizes, cfg.anchor, cfg.passing, cfg.probe_r,
                 cfg.hq, cfg.hkv, cfg.head_dim, device=dev)
    ws = p.new_workspace()
    o = torch.empty_like(q)
    lse = torch.empty((cfg.hq, cfg.n_visual + cfg.n_text), dtype=torch.float32, device=dev)
    for _ in range(max(args.warmup, 3)):
        sab.attn_prefill(p, q, k, v, o=o, lse=lse, workspace=ws)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.steps):
        sab.attn_prefill(p, q, k, v, o=o, lse=lse, workspace=ws)
    e1.record()
    torch.cuda.synchronize()
    base = e0.elapsed_time(e1) / args.steps
    p.close()
    del ws
    combos = [(int(w), pol, f) for w in args.worlds.split(",") for pol in args.policies.split(",")
              for f in args.flows.split(",")]
    for world, policy, flow in combos:
        try:
            res = shard_emulate(cfg, sizes, q, k, v, world, policy, args.steps, max(args.warmup, 3), flow)
        except (ValueError, sab.SpavaError) as e:
            print(json.dumps({"config": cfg.name, "world": world, "policy": policy, "skipped": str(e)}))
            continue
        res.update({"metric": "sharded prefill: per-rank compute, ranks emulated on one GPU",
                    "unit": "ms", "config": cfg.name, "world": world, "policy": policy, "flow": flow,
                    "one_gpu_prefill_ms": round(base, 4),
                    "compute_speedup_vs_one_gpu": round(base / res["max_ms"], 3),
                    "ideal_speedup": world})
        print(json.dumps(res), flush=True)


# ---------------------------------------------------------------- GPU arm
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--config", default="128k", choices=sorted(CONFIGS))
    ap.add_argument("--impl", default="b200", choices=["b200", "reference"])
    ap.add_argument("--fused-select", type=int, default=0,
                    help="0: score kernel, then select+gather (default); 1: scoring, selection and gather in "
                         "one persistent launch")
    ap.add_argument("--flow", default="single", choices=["single", "two_stage"],
                    help="single: one attention pass per host (default); two_stage: local pass with fused "
                         "probe scores, then the remote pass merged through the lse")
    # one streamed step per layer of a 28-layer model of the workloads' shape
    # (Qwen2-VL-7B class): the copy pipeline fills and drains once per prefill
    ap.add_argument("--e2e-steps", type=int, default=28)
    ap.add_argument("--ttft-layers", type=int, default=0,
                    help="also time a synthetic prefill of this many attention blocks (projections + attention), "
                         "approximate vs dense")
    ap.add_argument("--dense", type=int, default=1, help="also time the dense causal kernel (0/1)")
    ap.add_argument("--cpu-baseline", type=int, default=1)
    # rows per stratum (host block, text rows) of the oracle's sample; the same for both
    # arms so their figures are comparable
    ap.add_argument("--cpu-rows", type=int, default=64)
    ap.add_argument("--ref-rows", type=int, default=64)
    ap.add_argument("--sharded", default=None, choices=["zigzag", "contiguous", "longest_first"],
                    help="instead of replicas: one layer's hosts spread over the N ranks with this ownership "
                         "(strong scaling)")
    ap.add_argument("--sharded-form", default="overlap", choices=["overlap", "one_pass"])
    ap.add_argument("--shard-emulate", action="store_true",
                    help="instead of the bench line: the sharded prefill's per-rank compute with the ranks "
                         "emulated on this one GPU, one JSON line per (world, policy, form)")
    ap.add_argument("--worlds", default="2,4,8")
    ap.add_argument("--policies", default="zigzag,contiguous,longest_first")
    ap.add_argument("--flows", default="two_stage,one_pass")
    args = ap.parse_args()
    cfg = CONFIGS[args.config]

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        if rank == 0:
            run_reference(args, cfg)
        return
    if args.sharded:
        run_sharded(args, cfg, rank, world, local)
        return
    if args.shard_emulate:
        if rank == 0:
            run_shard_emulate(args, cfg)
        return

    import torch
    import torch.distributed as dist

    import sequence_approximate_attention_b200 as sab

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        init_nccl(dev, world)

    def barrier():
        if world > 1:
            dist.barrier()

    g = generate(cfg)
    sizes = [int(x) for x in g["host_sizes"]]
    NT = cfg.n_visual + cfg.n_text
    host = {x: torch.from_numpy(g[x].view(np.int16)).view(torch.bfloat16) for x in ("q", "k", "v")}
    d_in = {x: host[x].to(dev) for x in host}
    plan = sab.Plan(cfg.n_visual, cfg.n_text, cfg.n_hosts, sizes, cfg.anchor, cfg.passing, cfg.probe_r,
                    cfg.hq, cfg.hkv, cfg.head_dim, device=dev)
    two_stage = args.flow == "two_stage"
    plan.set_fused_select(bool(args.fused_select))
    ws = plan.new_workspace(two_stage)
    o = torch.empty_like(d_in["q"])
    prefill = sab.attn_prefill_two_stage if two_stage else sab.attn_prefill
    lse = torch.empty((cfg.hq, NT), dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        prefill(plan, d_in["q"], d_in["k"], d_in["v"], o=o, lse=lse, workspace=ws)
        return sab.last_launch_count()

    for _ in range(max(args.warmup, 3)):
        step()
    sab.check_device_error(plan, ws)

    clocks = ClockSampler(str(torch.cuda.get_device_properties(dev).uuid))
    plan.profile_begin(args.steps * 8 + 16)
    launches = 0
    clocks.start()
    time.sleep(0.3)
    barrier()
    torch.cuda.synchronize(dev)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev0.record(stream)
    for _ in range(args.steps):
        launches += step()
    ev1.record(stream)
    torch.cuda.synchronize(dev)
    barrier()
    clk = clocks.stop()
    ms_total = ev0.elapsed_time(ev1)
    prof = plan.profile_read()
    plan.profile_end()
    sab.check_device_error(plan, ws)
    ms_total = max_over_ranks(ms_total, dev)
    ms_step = ms_total / args.steps
    value = job_throughput(world, NT, args.steps, ms_total)

    # per-kernel averages over the timed steps
    per = {}
    for name, ms in prof:
        per.setdefault(name, []).append(ms)
    avg = {k: sum(v) / len(v) for k, v in per.items()}
    peaks, peak_src = load_peaks()
    if two_stage:
        avg["attention"] = avg.get("attention_local", 0.0) + avg.get("attention_remote", 0.0)
    pairs = attended_pairs(cfg, sizes)
    flops = 4.0 * cfg.head_dim * cfg.hq * pairs
    achieved = flops / (avg.get("attention", float("nan")) / 1e3) / 1e12
    sgb = select_gather_bytes(cfg, sizes)
    hbm = {}
    for name in ("score", "select", "gather", "select_gather", "score_select_gather"):
        if name in avg:
            gbs = sgb[name] / (avg[name] / 1e3) / 1e9
            hbm[name] = {"ms": avg[name], "bytes": sgb[name], "GB/s": gbs, "frac": gbs / peaks["hbm_gbs"]}
    if "score" in hbm:
        # the score kernel also does 64 GFLOP of MMAs at 128k: report its tensor side too
        sf = score_flops(cfg, sizes)
        hbm["score"]["flops"] = sf
        hbm["score"]["TFLOP/s"] = sf / (avg["score"] / 1e3) / 1e12
        hbm["score"]["frac_of_tensor_peak"] = hbm["score"]["TFLOP/s"] / peaks["bf16_tflops"]
    ssg_names = [n for n in ("score", "select", "gather", "select_gather", "score_select_gather") if n in avg]
    ssg_ms = sum(avg[n] for n in ssg_names)
    ssg_bytes = sum(sgb[n] for n in ssg_names)
    roofline = {
        "bound": "tensor", "kernel": "attn_fwd_kernel", "achieved": achieved, "peak": peaks["bf16_tflops"],
        "unit": "TFLOP/s", "frac": achieved / peaks["bf16_tflops"], "traffic": recorded_traffic(cfg.name),
        "algorithmic_bytes": attn_algorithmic_bytes(cfg),
        "peak_source": f"{peak_src} bf16 burst (MEASURED_PEAKS.json)",
        "frac_of_sustained": achieved / peaks["bf16_tflops_sustained"],
        "frac_of_datasheet_2250": achieved / 2250.0,
        "flops_per_launch": flops, "attended_pairs_per_head": pairs,
        "launch_ms": avg.get("attention"),
        "score_select_gather": {"ms": ssg_ms, "bytes": ssg_bytes,
                                "GB/s": ssg_bytes / (ssg_ms / 1e3) / 1e9 if ssg_ms > 0 else None,
                                "frac_of_hbm": (ssg_bytes / (ssg_ms / 1e3) / 1e9) / peaks["hbm_gbs"] if ssg_ms > 0 else None,
                                "per_kernel": hbm},
        "kernel_ms": avg,
    }
    step_tflops = flops / (ms_step / 1e3) / 1e12

    # dense causal comparison on the same inputs
    dense = None
    if args.dense:
        for _ in range(2):
            sab.dense_causal(plan, d_in["q"], d_in["k"], d_in["v"], o=o, lse=lse, workspace=ws)
        torch.cuda.synchronize(dev)
        reps = 3
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(reps):
            sab.dense_causal(plan, d_in["q"], d_in["k"], d_in["v"], o=o, lse=lse, workspace=ws)
        e1.record(stream)
        torch.cuda.synchronize(dev)
        sab.check_device_error(plan, ws)
        dms = e0.elapsed_time(e1) / reps
        dfl = 4.0 * cfg.head_dim * cfg.hq * dense_pairs(cfg)
        dense = {"ms": dms, "tokens/s": NT / (dms / 1e3), "TFLOP/s": dfl / (dms / 1e3) / 1e12,
                 "frac": dfl / (dms / 1e3) / 1e12 / peaks["bf16_tflops"], "speedup_of_approx": dms / ms_step}

    # end to end through the public API with host buffers: the streaming prefill
    # (HostPrefillPipeline: copies of neighbouring layers overlap the compute), and
    # for reference the same call with its copies serialised on one stream
    e2e = None
    if args.e2e_steps > 0:
        from sequence_approximate_attention_b200.pipeline import HostPrefillPipeline
        pin = {x: host[x].pin_memory() for x in host}
        o_h = torch.empty(o.shape, dtype=o.dtype).pin_memory()
        l_h = torch.empty(lse.shape, dtype=lse.dtype).pin_memory()
        pipe = HostPrefillPipeline(plan, two_stage)

        def timed(run, k):
            run()
            torch.cuda.synchronize(dev)
            barrier()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            for _ in range(k):
                run()
            pipe.wait(stream)
            e1.record(stream)
            torch.cuda.synchronize(dev)
            barrier()
            return max_over_ranks(e0.elapsed_time(e1), dev)

        def pipelined_step():
            pipe.submit(pin["q"], pin["k"], pin["v"], o_h, l_h)

        def serial_step():
            for x in ("q", "k", "v"):
                d_in[x].copy_(pin[x], non_blocking=True)
            prefill(plan, d_in["q"], d_in["k"], d_in["v"], o=o, lse=lse, workspace=ws)
            o_h.copy_(o, non_blocking=True)
            l_h.copy_(lse, non_blocking=True)

        te = timed(pipelined_step, args.e2e_steps)
        n_serial = max(2, min(6, args.e2e_steps // 2))
        ts = timed(serial_step, n_serial)
        e2e = {"value": job_throughput(world, NT, args.e2e_steps, te), "unit": "tokens/s",
               "h2d_bytes_per_step": pipe.h2d_bytes, "d2h_bytes_per_step": pipe.d2h_bytes, "steps": args.e2e_steps,
               "api": "HostPrefillPipeline.submit (double-buffered; H2D of step n+1 and D2H of step n-1 overlap step n); "
                      "one step per layer of a 28-layer prefill, pipeline fill and drain included",
               "serial_value": job_throughput(world, NT, n_serial, ts)}
        del pipe

    # time-to-first-token style: L attention blocks (random weights, plain GEMM
    # projections around the library's attention), approximate vs dense attention
    ttft = None
    if args.ttft_layers > 0:
        from sequence_approximate_attention_b200.layer_stack import LayerStack
        hidden = cfg.hq * cfg.head_dim
        stack = LayerStack(plan, hidden, args.ttft_layers, seed=cfg.seed, two_stage=two_stage)
        x0 = (torch.randn(NT, hidden, generator=torch.Generator().manual_seed(cfg.seed)) * 0.5).to(torch.bfloat16).to(dev)
        times = {}
        for dense_mode in (False, True):
            stack.forward(x0, dense=dense_mode)
            torch.cuda.synchronize(dev)
            t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            t0.record(stream)
            for _ in range(2):
                stack.forward(x0, dense=dense_mode)
            t1.record(stream)
            torch.cuda.synchronize(dev)
            times["dense" if dense_mode else "approx"] = max_over_ranks(t0.elapsed_time(t1), dev) / 2
        stack.check_errors()
        # the projection kernels alone: one layer's QKV projection (RMSNorm fused) and
        # output projection + residual, timed on the stack's own buffers
        L0 = stack.layers[0]
        sab.qkv_projection(stack._x, L0["w_qkv"], cfg.hq, cfg.hkv, cfg.head_dim, stack._q, stack._k, stack._v,
                           stack.ws_layer)
        reps = 5
        t0, t1, t2 = (torch.cuda.Event(enable_timing=True) for _ in range(3))
        t0.record(stream)
        for _ in range(reps):
            sab.qkv_projection(stack._x, L0["w_qkv"], cfg.hq, cfg.hkv, cfg.head_dim, stack._q, stack._k, stack._v,
                               stack.ws_layer)
        t1.record(stream)
        for _ in range(reps):
            sab.out_projection(stack._o, L0["w_o"], stack._x, stack.ws_layer)
        t2.record(stream)
        torch.cuda.synchronize(dev)
        stack.check_errors()
        fl = stack.flops()
        qkv_ms, out_ms = t0.elapsed_time(t1) / reps, t1.elapsed_time(t2) / reps
        ttft = {"layers": args.ttft_layers, "hidden": hidden, "tokens": NT, "approx_ms": times["approx"],
                "dense_ms": times["dense"], "speedup": times["dense"] / times["approx"],
                "projection_tflop_per_layer": fl["projections"] / 1e12,
                "qkv_projection": {"ms": qkv_ms, "TFLOP/s": fl["qkv"] / (qkv_ms / 1e3) / 1e12,
                                   "frac": fl["qkv"] / (qkv_ms / 1e3) / 1e12 / peaks["bf16_tflops"]},
                "out_projection": {"ms": out_ms, "TFLOP/s": fl["out"] / (out_ms / 1e3) / 1e12,
                                   "frac": fl["out"] / (out_ms / 1e3) / 1e12 / peaks["bf16_tflops"]},
                "note": "attention blocks only: RMSNorm + QKV projection (tcgen05 GEMM, norm and q/k/v split "
                        "in its epilogue), attention, output projection + residual (tcgen05 GEMM); random "
                        "weights, no rotary embedding, no MLP"}
        del stack

    cpu = None
    if args.cpu_baseline and rank == 0 and world == 1:
        t_full, desc, work, frac = oracle_sample(cfg, g, 7, rows=args.cpu_rows)
        cpu = {"value": NT / t_full, "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle",
               "sample": desc + f"; seed 7, {work:.1f} s of CPU work", "host_cpus": os.cpu_count(),
               "sampled_fraction_of_layer": frac}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": max(args.warmup, 3), "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic", "impl": "b200", "flow": args.flow, "fused_select": bool(args.fused_select),
            "config": workload_config(cfg),
            "tflops_step": step_tflops, "tflops_step_frac": step_tflops / peaks["bf16_tflops"],
            "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": launches, "ttft": ttft,
            "clocks": clk, "dense_causal": dense,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    plan.close()


if __name__ == "__main__":
    main()
