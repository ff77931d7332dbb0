"""Per-rank compute of the sharded prefill, measured on one GPU.

    python -m sequence_approximate_attention_b200.shard_emulate --config 128k \\
        --worlds 2,4,8 --policies zigzag,contiguous,longest_first

For each (world W, ownership policy, form: LOCAL + REMOTE or the one-pass ATTEND)
it builds the W ranks' plans on this GPU, runs
their stages in the order a W-GPU job would (every rank's SELECT, the exchange, every
LOCAL, the text exchange, every REMOTE, every MERGE), moving the exchanged bytes with
device copies between the stages, and times every kernel of each rank with the
library's timing hook (CUDA events on the launching stream).  A rank's compute is the
sum of its kernel times: what its own GPU would spend.  The
stages of different ranks alternate on the GPU, so each stage starts with another
rank's data in L2 (no L2 reuse between a rank's stages is assumed).  The collectives
themselves are not timed (one GPU); the bytes each rank contributes are reported.

One JSON line per (W, policy, form): per-rank compute (its select, attention and merge
parts), its max and mean, the balance
(max / mean), the one-GPU spava_attn_prefill time on the same inputs, and the
compute-only speed-up that the slowest rank allows.
"""

import argparse
import json
import os
import sys

import numpy as np
import torch

from . import Plan, _lib, attn_prefill, shard_stage

FLOWS = {
    "two_stage": (_lib.SPAVA_SHARD_SELECT, _lib.SPAVA_SHARD_LOCAL, _lib.SPAVA_SHARD_REMOTE, _lib.SPAVA_SHARD_MERGE),
    "one_pass": (_lib.SPAVA_SHARD_SELECT, _lib.SPAVA_SHARD_ATTEND, _lib.SPAVA_SHARD_MERGE),
}
# the part of a layer each kernel of the timing hook belongs to
KERNEL_PART = {"probe_lse": "select", "score": "select", "select_gather": "select", "score_keys": "attention",
               "attention_local": "attention", "unpack_passing": "attention", "attention_remote": "attention",
               "attention": "attention", "text_slot_fill": "attention", "lse_merge": "merge"}
PARTS = ("select", "attention", "merge")


def _workloads():
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    if root not in sys.path:
        sys.path.insert(0, root)
    from workloads import CONFIGS, generate
    return CONFIGS, generate


def _plan(cfg, sizes, dev):
    return Plan(cfg.n_visual, cfg.n_text, cfg.n_hosts, sizes, cfg.anchor, cfg.passing, cfg.probe_r, cfg.hq, cfg.hkv,
                cfg.head_dim, device=dev)


def emulate(cfg, sizes, q, k, v, world, policy, steps, warmup, flow="two_stage"):
    dev = q.device
    probe = _plan(cfg, sizes, dev)
    owner = probe.shard_owners(world, policy)
    probe.close()
    ranks = []
    for r in range(world):
        p = _plan(cfg, sizes, dev)
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
        for sid in FLOWS[flow]:
            for R in ranks:
                shard_stage(R["plan"], sid, q, k, v, o, lse, R["ws"])
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


def one_gpu_ms(cfg, sizes, q, k, v, steps, warmup):
    p = _plan(cfg, sizes, q.device)
    ws = p.new_workspace()
    o = torch.empty_like(q)
    lse = torch.empty((cfg.hq, cfg.n_visual + cfg.n_text), dtype=torch.float32, device=q.device)
    for _ in range(warmup):
        attn_prefill(p, q, k, v, o=o, lse=lse, workspace=ws)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(steps):
        attn_prefill(p, q, k, v, o=o, lse=lse, workspace=ws)
    e1.record()
    torch.cuda.synchronize()
    p.close()
    return e0.elapsed_time(e1) / steps


def main(argv=None):
    CONFIGS, generate = _workloads()
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--config", default="128k", choices=sorted(CONFIGS))
    ap.add_argument("--worlds", default="2,4,8")
    ap.add_argument("--policies", default="zigzag,contiguous,longest_first")
    ap.add_argument("--flows", default="two_stage,one_pass")
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    args = ap.parse_args(argv)
    cfg = CONFIGS[args.config]
    g = generate(cfg)
    sizes = [int(x) for x in g["host_sizes"]]
    dev = torch.device("cuda", torch.cuda.current_device())
    q, k, v = (torch.from_numpy(g[x].view(np.int16)).view(torch.bfloat16).to(dev) for x in ("q", "k", "v"))
    base = one_gpu_ms(cfg, sizes, q, k, v, args.steps, args.warmup)
    combos = [(int(w), p, f) for w in args.worlds.split(",") for p in args.policies.split(",")
              for f in args.flows.split(",")]
    for world, policy, flow in combos:
        try:
            res = emulate(cfg, sizes, q, k, v, world, policy, args.steps, args.warmup, flow)
        except (ValueError, _lib.SpavaError) as e:
            print(json.dumps({"config": cfg.name, "world": world, "policy": policy, "skipped": str(e)}))
            continue
        res.update({"metric": "sharded prefill: per-rank compute, ranks emulated on one GPU",
                    "unit": "ms", "config": cfg.name, "world": world, "policy": policy, "flow": flow,
                    "one_gpu_prefill_ms": round(base, 4),
                    "compute_speedup_vs_one_gpu": round(base / res["max_ms"], 3),
                    "ideal_speedup": world})
        print(json.dumps(res), flush=True)

if __name__ == "__main__":
    main()
