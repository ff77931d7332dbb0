"""Seeded input generator: Q/K/V as bf16 bit patterns plus host block sizes.

Recipe (one numpy ``default_rng(seed)`` stream, drawn in this order):
  1. host block sizes (uneven workloads only);
  2. Q ~ N(0,1), shape [N+T, hq, d];
  3. K, then V: "iid" draws N(0,1) for every token; "frame" draws, for every
     256-token frame and KV head, a mean mu ~ N(0,1)^d and sets each token of the
     frame to mu + 0.3 * N(0,1); text tokens are always iid N(0,1);
  4. salient tokens (if any): a uniform sample without replacement of
     round(frac * N) visual tokens whose keys are scaled by 3 in every KV head.
All draws are float32 and are rounded to bf16 (round-to-nearest-even) at the end,
so the GPU and the oracle see the same bytes.  Nothing here scores, selects or
attends.
"""

from typing import Dict, Optional

import numpy as np

from .configs import Workload

_CHUNK = 1 << 24


def bf16_round_bits(x: np.ndarray) -> np.ndarray:
    """float32 array -> uint16 bf16 bit patterns, round to nearest even."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    flat = x.reshape(-1)
    out = np.empty(flat.shape, dtype=np.uint16)
    for s in range(0, flat.size, _CHUNK):
        u = flat[s:s + _CHUNK].view(np.uint32)
        bias = ((u >> np.uint32(16)) & np.uint32(1)) + np.uint32(0x7FFF)
        out[s:s + _CHUNK] = ((u + bias) >> np.uint32(16)).astype(np.uint16)
    return out.reshape(x.shape)


def host_sizes_for(cfg: Workload, rng: Optional[np.random.Generator] = None) -> np.ndarray:
    """Block sizes B_h (int32 [H]).  Equal split unless ``cfg.uneven`` is set.

    Uneven recipe: every host starts at the minimum size; the remaining tokens are
    shared out in units of ``multiple`` proportionally to U[0,1) weights, capped at
    the maximum size, with the leftover units given to the hosts with the largest
    fractional share that still have room.
    """
    N, H = cfg.n_visual, cfg.n_hosts
    if cfg.uneven is None:
        if N % H:
            raise ValueError("equal split needs N % H == 0")
        return np.full(H, N // H, dtype=np.int32)
    lo, hi, mult = cfg.uneven
    if rng is None:
        rng = np.random.default_rng(cfg.seed)
    units_total = (N - H * lo) // mult
    if (N - H * lo) % mult or units_total < 0:
        raise ValueError("uneven split does not fit")
    cap = (hi - lo) // mult
    w = rng.uniform(0.0, 1.0, size=H)
    share = w / w.sum() * units_total
    units = np.minimum(np.floor(share).astype(np.int64), cap)
    frac = share - np.floor(share)
    left = units_total - int(units.sum())
    while left > 0:
        room = np.where(units < cap)[0]
        order = room[np.argsort(-frac[room], kind="stable")]
        for h in order[:left]:
            units[h] += 1
        left = units_total - int(units.sum())
        frac[:] = 0.0
    sizes = (lo + units * mult).astype(np.int32)
    assert int(sizes.sum()) == N and sizes.min() >= lo and sizes.max() <= hi
    return sizes


def _normal(rng: np.random.Generator, shape) -> np.ndarray:
    return rng.standard_normal(size=shape, dtype=np.float32)


def _kv(cfg: Workload, rng: np.random.Generator) -> np.ndarray:
    N, T, hkv, d = cfg.n_visual, cfg.n_text, cfg.hkv, cfg.head_dim
    out = np.empty((N + T, hkv, d), dtype=np.float32)
    if cfg.kv_kind == "iid":
        out[:] = _normal(rng, (N + T, hkv, d))
        return out
    if cfg.kv_kind != "frame":
        raise ValueError(f"unknown kv_kind {cfg.kv_kind!r}")
    F = cfg.frame
    n_frames = (N + F - 1) // F
    mu = _normal(rng, (n_frames, hkv, d))
    for f in range(n_frames):
        a, b = f * F, min(N, (f + 1) * F)
        out[a:b] = mu[f][None] + np.float32(cfg.frame_noise) * _normal(rng, (b - a, hkv, d))
    if T:
        out[N:] = _normal(rng, (T, hkv, d))
    return out


def generate(cfg: Workload, seed: Optional[int] = None) -> Dict[str, np.ndarray]:
    """Return {"q","k","v": uint16 bf16 bits [tokens, heads, d], "host_sizes": int32 [H],
    "salient": int64 indices}."""
    rng = np.random.default_rng(cfg.seed if seed is None else seed)
    sizes = host_sizes_for(cfg, rng) if cfg.uneven is not None else host_sizes_for(cfg)
    q = _normal(rng, (cfg.n_total, cfg.hq, cfg.head_dim))
    qb = bf16_round_bits(q)
    del q
    k = _kv(cfg, rng)
    v = _kv(cfg, rng)
    sal = np.zeros(0, dtype=np.int64)
    if cfg.salient_frac > 0:
        n_sal = int(round(cfg.salient_frac * cfg.n_visual))
        sal = np.sort(rng.choice(cfg.n_visual, size=n_sal, replace=False))
        k[sal] *= np.float32(cfg.salient_scale)
    return {"q": qb, "k": bf16_round_bits(k), "v": bf16_round_bits(v),
            "host_sizes": sizes, "salient": sal}
