"""fp64 CPU oracle of the Spava / APB-V approximate-attention prefill.

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, ``__graft_entry__.smoke()`` and
the CPU-baseline leg of ``bench.py``, never by the library.  Slow and plain on
purpose: every step is numpy fp64 in the order the method states it, with
``np.matmul`` as the only library primitive.

Source pages: "Spava: Accelerating Long-Video Understanding via
Sequence-Parallelism-aware Approximate Attention", also titled "APB-V: ..."
(arXiv 2601.21444).  The most detailed are the gist.science technical summaries
(German and Portuguese twins):
  * "Methodology", 1. Framework design -- "Context splitting & ZigZag
    arrangement": the input embeddings are split into an anchor block B_a, a query
    block B_qr and context blocks B^(h), one per host;
  * same section, "Approximate attention mechanism": the anchor block is a fixed
    initial segment; for each host the most essential key-value pairs are picked
    by query-to-context attention scores and aggregated into passing blocks that
    later hosts receive; attention runs over the anchor, the local context, the
    aggregated passing blocks and the query;
  * 2. System optimisations -- "Fused context and query forward": partial query
    results are merged through FlashAttention's lse outputs;
  * "Limitations": on a single GPU the method degenerates to standard
    FlashAttention (dense causal attention).

The pages give no formula for the score, no constants and no worked example.
Readings taken where they are silent (each is a parameter of this oracle):
  R1  score of key j of host h, KV head g: the max, over the last R query rows i
      of host h with i >= j and over the query heads c of group g, of
      s_c(i, j) = (q_{i,c} . k_{j,g}) * scale, scale = d^-1/2.  (max over heads:
      parity unpinned -- no page value fixes sum vs max.)  Switchable
      (``head_reduce``): with "sum" or "mean" each head first takes its own max
      over the probe rows, m_c(j), and the group's score is sum_c m_c(j) or its
      mean; "max" is max_c m_c(j), the default above.  With "none" every query
      head keeps its own row m_c(j) and selects its own passing keys (per-query-head
      selection); query head c then attends to its own passing set, drawn from KV
      head c // G.  ``score_kind`` "prob" replaces each logit by the probe row's
      attention probability over its own host block, p_c(i, j) = exp(s_c(i, j) -
      lse_c(i)) with lse_c(i) = log sum over keys j' of the block, j' <= i, of
      exp s_c(i, j'); m_c(j) is then the max of p_c over the probe rows (the pages'
      scores may be read as the attention weights rather than the logits).
  R2  causal inside the probe: probe row i never scores a key j > i.
  R3  host 0's anchor positions [0, A) are not passing candidates, so no key is
      attended twice by a later host (parity unpinned -- a plan-level reading).
  R4  the last host selects nothing (nothing reads its passing blocks).
  R5  each earlier host contributes its own P keys per KV head; later hosts see
      h * P passing keys (not re-compressed).
  R6  the trailing text (query) segment attends densely and causally to every
      token before it and contributes no scores.
  R7  ties in selection: larger score first; equal scores -> lower token index;
      -0.0 equals +0.0.  The P chosen indices are stored in ascending order.
  R8  GQA: query head c uses KV head c // (hq / hkv) (parity unpinned).
  R11 ZigZag arrangement with more than 2W virtual hosts on W ranks: the pairing of
      rank r with virtual hosts r and 2W-1-r repeats over consecutive rounds of 2W
      hosts (the pages only describe one round).
"""

from typing import Dict, Optional, Sequence

import numpy as np


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """uint16 bf16 bit patterns -> exact float64 values."""
    b = np.ascontiguousarray(bits, dtype=np.uint16)
    return (b.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


def host_offsets(host_sizes: Sequence[int]) -> np.ndarray:
    """Context splitting: off[0] = 0, off[h+1] = off[h] + B_h (context blocks B^(h))."""
    sizes = np.asarray(host_sizes, dtype=np.int64)
    if sizes.ndim != 1 or sizes.size == 0 or (sizes <= 0).any():
        raise ValueError("host sizes must be a non-empty list of positive ints")
    off = np.zeros(sizes.size + 1, dtype=np.int64)
    off[1:] = np.cumsum(sizes)
    return off


def host_of_row(off: np.ndarray, i: int) -> int:
    """Host whose context block holds visual token i."""
    return int(np.searchsorted(off, i, side="right") - 1)


def _groups(hq: int, hkv: int) -> int:
    if hq % hkv:
        raise ValueError("hq must be a multiple of hkv")
    return hq // hkv


HEAD_REDUCE = ("max", "sum", "mean", "none")
SCORE_KIND = ("logit", "prob")


def probe_scores(q: np.ndarray, k: np.ndarray, off: np.ndarray, probe_r: int,
                 scale: float, head_reduce: str = "max", score_kind: str = "logit") -> np.ndarray:
    """Query-to-context scores of every visual key (readings R1, R2).

    q [tokens, hq, d], k [tokens, hkv, d] float64; returns float64 [hkv, N], or
    [hq, N] (one row per query head, row c = m_c) with head_reduce="none".
    ``head_reduce`` combines the per-head probe maxima of a KV group (R1).
    """
    if head_reduce not in HEAD_REDUCE:
        raise ValueError(f"head_reduce must be one of {HEAD_REDUCE}")
    if score_kind not in SCORE_KIND:
        raise ValueError(f"score_kind must be one of {SCORE_KIND}")
    hq, hkv = q.shape[1], k.shape[1]
    G = _groups(hq, hkv)
    H = len(off) - 1
    N = int(off[-1])
    scores = np.empty((hq if head_reduce == "none" else hkv, N), dtype=np.float64)
    for h in range(H):
        a, e = int(off[h]), int(off[h + 1])
        if probe_r > e - a:
            raise ValueError("probe_r exceeds a host block")
        probe_rows = np.arange(e - probe_r, e)
        keys = np.arange(a, e)
        visible = probe_rows[:, None] >= keys[None, :]             # [R, B]  (R2)
        for g in range(hkv):
            qg = q[e - probe_r:e, g * G:(g + 1) * G, :]              # [R, G, d]
            s = np.matmul(qg.transpose(1, 0, 2), k[a:e, g, :].T)     # [G, R, B]
            s = np.where(visible[None], s * scale, -np.inf)
            if score_kind == "prob":
                # each probe row's softmax over the keys of its block it can see
                mrow = s.max(axis=2, keepdims=True)
                lse = mrow + np.log(np.exp(s - mrow).sum(axis=2, keepdims=True))
                s = np.exp(s - lse)                                  # 0 where not visible
            per_head = s.max(axis=1)                                 # [G, B]: m_c(j)
            if head_reduce == "none":
                scores[g * G:(g + 1) * G, a:e] = per_head
            elif head_reduce == "max":
                scores[g, a:e] = per_head.max(axis=0)
            elif head_reduce == "sum":
                scores[g, a:e] = per_head.sum(axis=0)
            else:
                scores[g, a:e] = per_head.sum(axis=0) / G
    return scores


def select_passing(scores: np.ndarray, off: np.ndarray, anchor: int, passing: int) -> np.ndarray:
    """Top-P passing keys of each host h < H-1 and KV head (readings R3, R4, R7).

    ``scores`` may be float64 (oracle) or float32 (the GPU's tensor): comparisons run
    in the array's own precision.  Returns int64 [H-1, hkv, P], ascending per row.
    """
    H = len(off) - 1
    hkv = scores.shape[0]
    out = np.empty((max(H - 1, 0), hkv, passing), dtype=np.int64)
    for h in range(H - 1):
        lo = int(off[h]) + (anchor if h == 0 else 0)
        hi = int(off[h + 1])
        if hi - lo < passing:
            raise ValueError("fewer candidates than passing keys")
        cand = np.arange(lo, hi)
        for g in range(hkv):
            s = scores[g, lo:hi]
            if np.isnan(s).any():
                raise ValueError("NaN score")
            # np.lexsort: last key is primary.  -s ascending == s descending; equal
            # values (including -0.0 vs +0.0, which compare equal) fall back to the
            # token index ascending.
            order = np.lexsort((cand, -s))
            out[h, g] = np.sort(cand[order[:passing]])
    return out


def sel_row(sel: Optional[np.ndarray], c: int, hq: int, hkv: int) -> int:
    """Row of the selection that query head c attends through: its KV head c // G when
    ``sel`` has one row per KV head, c itself when it has one per query head (R1)."""
    if sel is None or sel.shape[1] == hkv:
        return c // _groups(hq, hkv)
    if sel.shape[1] != hq:
        raise ValueError("selection must have hkv or hq rows")
    return c


def key_set(off: np.ndarray, anchor: int, sel: Optional[np.ndarray], g: int, i: int,
            n_visual: int) -> np.ndarray:
    """Keys attended by row i through selection row g (``sel_row``): anchor | passing
    of earlier hosts | own block up to i (causal).  Host 0 and text rows: [0, i]
    (readings R5, R6)."""
    if i >= n_visual:
        return np.arange(0, i + 1)
    h = host_of_row(off, i)
    if h == 0:
        return np.arange(0, i + 1)
    parts = [np.arange(0, anchor)]
    parts += [np.asarray(sel[hp, g], dtype=np.int64) for hp in range(h)]
    parts.append(np.arange(int(off[h]), i + 1))
    return np.concatenate(parts)


def _masked_softmax_attend(logits: np.ndarray, visible: np.ndarray, vals: np.ndarray):
    """Stable softmax over the visible entries of each row; returns (O, lse)."""
    z = np.where(visible, logits, -np.inf)
    m = z.max(axis=1, keepdims=True)
    p = np.where(visible, np.exp(z - m), 0.0)
    l = p.sum(axis=1, keepdims=True)
    o = np.matmul(p, vals) / l
    return o, (m + np.log(l))[:, 0]


def approx_attention(q: np.ndarray, k: np.ndarray, v: np.ndarray, off: np.ndarray,
                     anchor: int, sel: Optional[np.ndarray], scale: float,
                     row_chunk: int = 512, row_range=None, compact: bool = False):
    """Approximate attention of every row (host blocks + trailing text rows).

    Host h >= 1 attends to [anchor | passing of hosts < h | own block, causal];
    host 0 and text rows attend densely and causally.  Returns O float64
    [tokens, hq, d] and lse float64 [hq, tokens] (natural log).  With
    ``row_range=(r0, r1)`` only rows r0..r1-1 are computed (the rest stay NaN);
    with ``compact`` as well, only those rows are stored: O [r1-r0, hq, d] and lse
    [hq, r1-r0] (a storage choice, the arithmetic is the same).
    """
    NT, hq, d = q.shape
    hkv = k.shape[1]
    G = _groups(hq, hkv)
    H = len(off) - 1
    N = int(off[-1])
    lo_row, hi_row = (0, NT) if row_range is None else (int(row_range[0]), int(row_range[1]))
    compact = compact and row_range is not None
    base = lo_row if compact else 0
    n_out = hi_row - lo_row if compact else NT
    O = np.full((n_out, hq, d), np.nan, dtype=np.float64)
    lse = np.full((hq, n_out), np.nan, dtype=np.float64)
    for h in range(H):
        a, e = int(off[h]), int(off[h + 1])
        if e <= lo_row or a >= hi_row:
            continue
        for c in range(hq):
            g = c // G
            if h == 0:
                remote = np.zeros(0, dtype=np.int64)
            else:
                sr = sel_row(sel, c, hq, hkv)
                remote = np.concatenate([np.arange(0, anchor)] +
                                        [np.asarray(sel[hp, sr], dtype=np.int64) for hp in range(h)])
            for r0 in range(max(a, lo_row), min(e, hi_row), row_chunk):
                r1 = min(e, hi_row, r0 + row_chunk)
                keys = np.concatenate([remote, np.arange(a, r1)])
                visible = np.ones((r1 - r0, keys.size), dtype=bool)
                visible[:, remote.size:] = np.arange(a, r1)[None, :] <= np.arange(r0, r1)[:, None]
                kk, vv = k[keys, g, :], v[keys, g, :]
                logits = np.matmul(q[r0:r1, c, :], kk.T) * scale
                O[r0 - base:r1 - base, c], lse[c, r0 - base:r1 - base] = _masked_softmax_attend(logits, visible, vv)
    for r0 in range(max(N, lo_row), min(NT, hi_row), row_chunk):
        r1 = min(NT, hi_row, r0 + row_chunk)
        keys = np.arange(0, r1)
        visible = keys[None, :] <= np.arange(r0, r1)[:, None]
        for g in range(hkv):
            kk, vv = k[:r1, g, :], v[:r1, g, :]
            for c in range(g * G, (g + 1) * G):
                logits = np.matmul(q[r0:r1, c, :], kk.T) * scale
                O[r0 - base:r1 - base, c], lse[c, r0 - base:r1 - base] = _masked_softmax_attend(logits, visible, vv)
    return O, lse


def attention_rows(q: np.ndarray, k: np.ndarray, v: np.ndarray, off: np.ndarray,
                   anchor: int, sel: Optional[np.ndarray], scale: float,
                   rows: Sequence[int], heads: Sequence[int]):
    """The same attention for chosen (row, head) pairs only, one at a time through
    ``key_set``.  Used to check full-size runs on a sample of outputs."""
    hq, hkv = q.shape[1], k.shape[1]
    G = _groups(hq, hkv)
    N = int(off[-1])
    O = np.empty((len(rows), q.shape[2]), dtype=np.float64)
    L = np.empty(len(rows), dtype=np.float64)
    for n, (i, c) in enumerate(zip(rows, heads)):
        g = int(c) // G
        keys = key_set(off, anchor, sel, sel_row(sel, int(c), hq, hkv), int(i), N)
        s = np.matmul(k[keys, g, :], q[int(i), int(c), :]) * scale
        m = s.max()
        p = np.exp(s - m)
        l = p.sum()
        O[n] = np.matmul(p, v[keys, g, :]) / l
        L[n] = m + np.log(l)
    return O, L


def dense_causal(q: np.ndarray, k: np.ndarray, v: np.ndarray, scale: float,
                 row_chunk: int = 512):
    """Standard dense causal attention (what one host degenerates to)."""
    NT, hq, d = q.shape
    hkv = k.shape[1]
    G = _groups(hq, hkv)
    O = np.empty((NT, hq, d), dtype=np.float64)
    lse = np.empty((hq, NT), dtype=np.float64)
    for r0 in range(0, NT, row_chunk):
        r1 = min(NT, r0 + row_chunk)
        visible = np.arange(r1)[None, :] <= np.arange(r0, r1)[:, None]
        for c in range(hq):
            g = c // G
            logits = np.matmul(q[r0:r1, c, :], k[:r1, g, :].T) * scale
            O[r0:r1, c], lse[c, r0:r1] = _masked_softmax_attend(logits, visible, v[:r1, g, :])
    return O, lse


def lse_merge(o1: np.ndarray, l1: np.ndarray, o2: np.ndarray, l2: np.ndarray):
    """Merge two partial attention results over disjoint key sets through their lse
    (the fused context + query forward): l = log(e^l1 + e^l2),
    O = e^(l1-l) O1 + e^(l2-l) O2.  o*: [..., d], l*: [...]."""
    m = np.maximum(l1, l2)
    l = m + np.log(np.exp(l1 - m) + np.exp(l2 - m))
    return np.exp(l1 - l)[..., None] * o1 + np.exp(l2 - l)[..., None] * o2, l


def prefill(q: np.ndarray, k: np.ndarray, v: np.ndarray, host_sizes: Sequence[int],
            anchor: int, passing: int, probe_r: int, scale: Optional[float] = None,
            sel: Optional[np.ndarray] = None, rows=None, head_reduce: str = "max",
            score_kind: str = "logit") -> Dict[str, np.ndarray]:
    """Whole prefill: split -> score -> select -> approximate attention.

    q/k/v are float64 (see ``bf16_bits_to_f64``).  If ``sel`` is given it replaces
    the oracle's own selection (to re-run attention with another selection).
    With ``rows=(rows, heads)`` only those outputs are computed.
    """
    d = q.shape[2]
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    off = host_offsets(host_sizes)
    out: Dict[str, np.ndarray] = {"offsets": off}
    out["scores"] = probe_scores(q, k, off, probe_r, scale, head_reduce, score_kind)
    out["sel"] = select_passing(out["scores"], off, anchor, passing) if sel is None else sel
    if rows is None:
        out["O"], out["lse"] = approx_attention(q, k, v, off, anchor, out["sel"], scale)
    else:
        out["O"], out["lse"] = attention_rows(q, k, v, off, anchor, out["sel"], scale, *rows)
    return out


def zigzag_owners(n_hosts: int, world: int) -> np.ndarray:
    """ZigZag arrangement (APB-V technical summary, 1. Framework design, "Context
    splitting & ZigZag arrangement": a physical host runs the pair of virtual hosts h
    and 2H-1-h; the German explainer, "Lastverteilung": the first worker takes the
    first and the last block, the second the second and the one before last, and so
    on).  Rank of each of n_hosts virtual hosts on ``world`` ranks; reading R11 for
    n_hosts > 2 * world."""
    if world < 1 or n_hosts % (2 * world):
        raise ValueError("zigzag needs n_hosts to be a multiple of 2 * world")
    owner = np.empty(n_hosts, dtype=np.int64)
    for h in range(n_hosts):
        t = h % (2 * world)          # position inside its round of 2W hosts
        owner[h] = t if t < world else 2 * world - 1 - t
    return owner


def contiguous_owners(n_hosts: int, world: int) -> np.ndarray:
    """Plain split: rank r runs the n_hosts / world consecutive hosts starting at
    r * n_hosts / world."""
    if world < 1 or n_hosts % world:
        raise ValueError("contiguous split needs n_hosts to be a multiple of world")
    per = n_hosts // world
    return np.array([h // per for h in range(n_hosts)], dtype=np.int64)


def sharded_attention(q: np.ndarray, k: np.ndarray, v: np.ndarray, off: np.ndarray, anchor: int,
                      sel: np.ndarray, scale: float, owner: Sequence[int]):
    """The multi-host form of ``approx_attention`` (2. System optimisations, "Fused
    context and query forward" and the two-stage attention of "Main contributions"):
    every rank computes, for its own hosts, the rows' attention over the own block
    (causal) and, separately, over [anchor | passing of earlier hosts], and merges the
    two through the lse; the text rows get one partial per host block (from the
    rank owning that host) plus their own causal part (from the owner of the last
    host), merged through the lse.  Returns (O, lse) like approx_attention; equal to it
    up to rounding, which pins the decomposition."""
    NT, hq, d = q.shape
    hkv = k.shape[1]
    H = len(off) - 1
    N = int(off[H])
    O = np.zeros((NT, hq, d))
    lse = np.zeros((hq, NT))
    for c in range(hq):
        g = sel_row(sel, c, hq, hkv)
        kv = c // _groups(hq, hkv)
        for h in range(H):
            a, e = int(off[h]), int(off[h + 1])
            rows = np.arange(a, e)
            logits = np.matmul(q[a:e, c, :], k[a:e, kv, :].T) * scale
            o_loc, l_loc = _masked_softmax_attend(logits, rows[None, :] <= rows[:, None], v[a:e, kv, :])
            remote = []
            if h >= 1:
                remote = list(range(anchor)) + [int(x) for hh in range(h) for x in sel[hh, g]]
            if remote:
                ridx = np.array(remote)
                logits = np.matmul(q[a:e, c, :], k[ridx, kv, :].T) * scale
                o_rem, l_rem = _masked_softmax_attend(logits, np.ones(logits.shape, bool), v[ridx, kv, :])
                o_loc, l_loc = lse_merge(o_loc, l_loc, o_rem, l_rem)
            O[a:e, c], lse[c, a:e] = o_loc, l_loc
        if NT > N:
            rows = np.arange(N, NT)
            parts = []
            for h in range(H):
                a, e = int(off[h]), int(off[h + 1])
                logits = np.matmul(q[N:NT, c, :], k[a:e, kv, :].T) * scale
                parts.append((owner[h], _masked_softmax_attend(logits, np.ones(logits.shape, bool), v[a:e, kv, :])))
            logits = np.matmul(q[N:NT, c, :], k[N:NT, kv, :].T) * scale
            parts.append((owner[H - 1], _masked_softmax_attend(logits, rows[None, :] <= rows[:, None],
                                                               v[N:NT, kv, :])))
            # all ranks' pieces meet after the exchange: merged in rank order
            parts.sort(key=lambda x: x[0])
            o_t, l_t = parts[0][1]
            for _, (op, lp) in parts[1:]:
                o_t, l_t = lse_merge(o_t, l_t, op, lp)
            O[N:NT, c], lse[c, N:NT] = o_t, l_t
    return O, lse


def host_costs(host_sizes: Sequence[int], anchor: int, passing: int, n_text: int) -> np.ndarray:
    """Work of each host in (query, key) pairs: its rows over its own block (causal),
    over the anchor and the passing rows of the earlier hosts (h >= 1), and the text
    rows over its block; the last host also carries the text rows' causal part (the
    piece that sharding puts on its rank).  Summed over the hosts this is the number
    of pairs the whole approximate attention evaluates per query head."""
    H = len(host_sizes)
    cost = np.zeros(H, dtype=np.int64)
    for h, B in enumerate(int(b) for b in host_sizes):
        cost[h] = B * (B + 1) // 2 + n_text * B
        if h >= 1:
            cost[h] += B * (anchor + h * passing)
        if h == H - 1:
            cost[h] += n_text * (n_text + 1) // 2
    return cost


def longest_first_owners(cost: Sequence[int], world: int) -> np.ndarray:
    """Longest-processing-time list scheduling: hosts taken by decreasing cost (equal
    costs in host order), each given to the rank with the least cost so far (the
    lowest such rank).  The one-GPU scheduler's longest-first rule applied to whole
    hosts across ranks."""
    order = sorted(range(len(cost)), key=lambda h: (-int(cost[h]), h))
    load = [0] * world
    owner = np.empty(len(cost), dtype=np.int64)
    for h in order:
        r = min(range(world), key=lambda x: (load[x], x))
        owner[h] = r
        load[r] += int(cost[h])
    return owner
