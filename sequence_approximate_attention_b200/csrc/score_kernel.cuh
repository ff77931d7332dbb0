// Query-to-context scoring on the tensor cores (APB-V technical summary,
// 1. Framework design, "Approximate attention mechanism": every host ranks its
// local keys by query-to-context attention scores).
//
//   m_c(j)   = max over probe rows i in [e-R, e), i >= j, of (q_{i,c} . k_{j,g})
//              (probability scores: of exp(scale q.k - lse_c(i)), lse_c(i) the probe
//              row's log-sum-exp over the keys of its block it sees)
//   score(g, j) = scale * reduce over the query heads c of group g of m_c(j),
//   e = end of j's host block; reduce = max (default), sum or mean (the pages leave
//   the combination open; max over heads and rows is the plainest reading), or none:
//   one score row m_c per query head (per-query-head selection).
//
// The product is computed transposed, S^T = K_tile * Qprobe^T, so that each TMEM
// lane holds one key and the max over (probe row, head) is a per-thread reduction
// along the lane's columns (no cross-thread reduction).  The probe queries of one
// (host, KV group) form the MMA's N dimension, ordered (head, token): one TMA box
// (64 x 1 x Rc) per query head, so head c owns columns [c Rc, c Rc + Rc) of a chunk
// of Rc probe tokens (Rc G <= 256).  Work item = one 128-key tile of one (host, KV
// head).
//
// CTA = 256 threads: warp 0 TMA (one thread), warps 1 and 3 the two MMA issuers (one
// thread each, one accumulator each), warp 2 TMEM allocator, warps 4-7 epilogue
// (lane = key).  TMEM holds the two 256-column accumulators, so the epilogue of one
// chunk overlaps the MMAs of the next.
#pragma once

#include "common.cuh"

namespace spava {

struct ScoreParams {
  const int4* items;  // (host, kv head, first key of the tile, block end e)
  int n_items;
  int probe_r;       // R
  int group;         // G = hq / hkv
  int chunk_tokens;  // Rc probe tokens per N chunk (Rc * G <= 256, multiple of 16)
  int n_chunks;      // ceil(R / Rc)
  int head_reduce;   // 0 max, 1 sum, 2 mean over the group's query heads; 3 none (one
                     // score row per query head: scores is [hq][N])
  // Probability scores: lse of every probe row over the keys of its block it sees,
  // probe_lse[c * lse_stride + row] (query head c); nullptr for logit scores.
  const float* probe_lse;
  int lse_stride;
  int n_visual;      // N (row stride of scores)
  float scale;
  float* scores;     // [hkv][N]
  unsigned int* err_word;
  uint64_t wait_limit_ns;
  // shared-memory pipeline, sized on the host: probe-query buffers (1 when every
  // (host, group) fits one chunk, else 2) and K-tile stages filling the rest
  int q_bufs;
  int q_buf_bytes;
  int k_stages;
};

template <int D>
struct ScoreShape {
  static constexpr int kHalves = D / 64;
  static constexpr int kKTileBytes = kHalves * 128 * 128;  // 128 keys
  static constexpr int kMaxStages = 8;
  static constexpr int kBarBytes = 256;
  static constexpr int kMaxLocalItems = 512;  // item metadata cached in shared memory
  static constexpr int kItemBytes = kMaxLocalItems * 16;
  static constexpr int kSmemMax = 232448;  // opt-in limit per CTA on sm_100
  static constexpr uint32_t kTmemCols = 512;
  static constexpr int kMaxGroup = 16;  // query heads per KV head
  // Bytes of dynamic shared memory for a given pipeline (plus alignment slack).
  static constexpr int smem_bytes(int q_bufs, int q_buf_bytes, int k_stages) {
    return q_bufs * q_buf_bytes + k_stages * kKTileBytes + kBarBytes + kItemBytes + 1024;
  }
};

// Chunk-use (li, c) of this CTA -- item li, probe chunk c, use u = li*n_chunks + c --
// needs a fresh load of probe queries iff the buffer it maps to (u % q_bufs) last
// held a different (host, group, chunk).  `items` is the CTA's item range in shared
// memory.  Written without integer division (q_bufs <= 2): this runs on the MMA
// thread's critical path once per chunk.
__device__ __forceinline__ bool chunk_needs_load(int q_bufs, int n_chunks, const int4* items, int li, int c) {
  int cb = c - q_bufs, lb = li;
  while (cb < 0) {
    cb += n_chunks;
    --lb;
  }
  if (lb < 0) return true;  // first uses of each buffer
  if (cb != c) return true;   // the buffer held another chunk of the probe
  const int4 x = items[li], y = items[lb];
  return x.x != y.x || x.y != y.y;
}

// The use that comes q_bufs uses after (li, c), as (item, chunk).
__device__ __forceinline__ void chunk_next_use(int q_bufs, int n_chunks, int li, int c, int* ln, int* cn) {
  int cc = c + q_bufs, l = li;
  while (cc >= n_chunks) {
    cc -= n_chunks;
    ++l;
  }
  *ln = l;
  *cn = cc;
}

// ---------------------------------------------------------------- the scoring pipeline
// Shared by score_kernel and the fused ssg_kernel: one TMA thread loads 128-key K
// tiles (a ring of n_stages) and the probe queries; two MMA threads issue the
// products, issuer X taking the chunk-uses u with u % 2 == X into TMEM accumulator X
// (columns 256 X ..), so one thread's waits and bookkeeping overlap the other's MMAs
// on the tensor core; the epilogue drains accumulator u % 2 for use u.
//
// Probe-query buffers.  q_bufs == 2 (several chunks per item): buffer X belongs to
// issuer X (use u reads buffer u % 2) and is reloaded whenever it last held another
// (host, group, chunk).  q_bufs == 1 (one chunk): the single buffer holds the probe of
// one (host, group) -- a "generation" of consecutive items -- and is reloaded when the
// group changes, after every issuer that used it released it (q_empty[X]: one commit
// per generation the issuer took part in).
// K stages: released by the issuers that read them (one issuer per item with one
// chunk, both with more), so k_empty counts 1 or 2 arrivals.
struct ScorePipe {
  uint8_t* sQ;
  uint8_t* sK;
  int q_bufs, q_buf_bytes, n_stages;
  uint64_t* k_full;     // [kMaxStages]
  uint64_t* k_empty;    // [kMaxStages]
  uint64_t* q_full;     // [2]
  uint64_t* q_empty;    // [2] per issuer
  uint64_t* acc_full;   // [2]
  uint64_t* acc_empty;  // [2], 4 epilogue-warp arrivals
  uint64_t* drain;      // [2] per issuer
};

struct ScoreGeom {
  int probe_r, group, chunk_tokens, n_chunks;
};

constexpr int kScorePipeStages = 8;  // most K stages any pipeline uses
constexpr int kScorePipeBarBytes = (2 * kScorePipeStages + 10) * 8;

// Barriers laid out from `bars` (kScorePipeBarBytes); initialised by one thread.
__device__ __forceinline__ ScorePipe score_pipe_at(uint8_t* sQ, uint8_t* sK, int q_bufs, int q_buf_bytes,
                                                   int n_stages, uint64_t* bars) {
  ScorePipe sp;
  sp.sQ = sQ;
  sp.sK = sK;
  sp.q_bufs = q_bufs;
  sp.q_buf_bytes = q_buf_bytes;
  sp.n_stages = n_stages;
  sp.k_full = bars;
  sp.k_empty = bars + kScorePipeStages;
  sp.q_full = bars + 2 * kScorePipeStages;
  sp.q_empty = sp.q_full + 2;
  sp.acc_full = sp.q_empty + 2;
  sp.acc_empty = sp.acc_full + 2;
  sp.drain = sp.acc_empty + 2;
  return sp;
}

__device__ __forceinline__ void score_pipe_init(const ScorePipe& sp, int n_chunks) {
  for (int b = 0; b < sp.n_stages; ++b) {
    mbar_init(sp.k_full + b, 1);
    mbar_init(sp.k_empty + b, n_chunks == 1 ? 1 : 2);
  }
  for (int b = 0; b < 2; ++b) {
    mbar_init(sp.q_full + b, 1);
    mbar_init(sp.q_empty + b, 1);
    mbar_init(sp.acc_full + b, 1);
    mbar_init(sp.acc_empty + b, 4);  // one arrival per epilogue warp
    mbar_init(sp.drain + b, 1);
  }
}

__device__ __forceinline__ bool same_group(int4 a, int4 b) { return a.x == b.x && a.y == b.y; }

// TMA producer (one thread): K tile of every item, probe queries when needed.
template <int D>
__device__ __forceinline__ void score_produce(const ScorePipe& sp, const ScoreGeom& g, const int4* items,
                                              int n_local, const CUtensorMap* tmK, const CUtensorMap* tmQp,
                                              const WaitCtx& wc) {
  constexpr int kHalves = D / 64, kKTileBytes = kHalves * 128 * 128;
  const int G = g.group;
  const uint32_t q_bytes = static_cast<uint32_t>(kHalves * g.chunk_tokens * G * 128);
  int qloads[2] = {0, 0};       // loads issued into each probe buffer
  int rel[2] = {0, 0};          // one buffer: releases of each issuer consumed
  bool part[2] = {false, false};  // one buffer: issuers that used the resident probe
  int slot = 0, use = 0;        // K stage and how often it was filled before
  bool ok = true;
  auto load_q = [&](int b, int4 it, int c) {
    mbar_arrive_expect_tx(sp.q_full + b, q_bytes);
    for (int hh = 0; hh < kHalves; ++hh)
      for (int h = 0; h < G; ++h)
        tma_load_3d(sp.sQ + b * sp.q_buf_bytes + hh * (g.chunk_tokens * G * 128) + h * (g.chunk_tokens * 128), tmQp,
                    sp.q_full + b, hh * 64, it.y * G + h, it.w - g.probe_r + c * g.chunk_tokens);
    ++qloads[b];
  };
  for (int li = 0; li < n_local && ok; ++li) {
    const int4 it = items[li];
    if (use > 0 && !(ok = mbar_wait(sp.k_empty + slot, (use - 1) & 1, wc, kErrWaitRelease))) break;
    mbar_arrive_expect_tx(sp.k_full + slot, kKTileBytes);
    for (int hh = 0; hh < kHalves; ++hh)
      tma_load_3d(sp.sK + slot * kKTileBytes + hh * 128 * 128, tmK, sp.k_full + slot, hh * 64, it.y, it.z);
    if (++slot == sp.n_stages) {
      slot = 0;
      ++use;
    }
    if (sp.q_bufs == 1) {
      if (li == 0 || !same_group(it, items[li - 1])) {
        for (int x = 0; x < 2 && ok; ++x)
          if (part[x]) {
            ok = mbar_wait(sp.q_empty + x, rel[x] & 1, wc, kErrWaitRelease);
            ++rel[x];
          }
        if (!ok) break;
        part[0] = part[1] = false;
        load_q(0, it, 0);
      }
      part[li & 1] = true;
    } else {
      for (int c = 0; c < g.n_chunks; ++c) {
        const int b = (li * g.n_chunks + c) & 1;
        if (!chunk_needs_load(2, g.n_chunks, items, li, c)) continue;
        if (qloads[b] > 0 && !(ok = mbar_wait(sp.q_empty + b, (qloads[b] - 1) & 1, wc, kErrWaitRelease))) break;
        load_q(b, it, c);
      }
    }
  }
  if (!ok) {
    // Abort: let every copy this thread issued land before the CTA exits.
    for (int b = 0; b < sp.n_stages; ++b) {
      const int uses = use + (b < slot ? 1 : 0);
      if (uses > 0) mbar_wait_drain(sp.k_full + b, (uses - 1) & 1, wc);
    }
    for (int b = 0; b < 2; ++b)
      if (qloads[b] > 0) mbar_wait_drain(sp.q_full + b, (qloads[b] - 1) & 1, wc);
  }
}

// MMA issuer X (one thread): S^T = K_tile Qprobe^T for the uses u = X, X + 2, ...
// into accumulator X.  Never waits on the other issuer.
template <int D>
__device__ __forceinline__ void score_issue(const ScorePipe& sp, const ScoreGeom& g, const int4* items, int n_local,
                                            int X, uint32_t tmem, const WaitCtx& wc) {
  constexpr int kKTileBytes = (D / 64) * 128 * 128;
  const int n_uses = n_local * g.n_chunks;
  const int nc = g.chunk_tokens * g.group;
  const uint32_t idesc = idesc_bf16_f32(128, nc, 0, 0);
  const uint32_t qhalf = static_cast<uint32_t>(nc * 128);
  const uint32_t qa = smem_u32(sp.sQ + (sp.q_bufs == 1 ? 0 : X) * sp.q_buf_bytes);
  int qwaits = 0;            // two buffers: loads of buffer X waited for
  int gen = 0, gen_li = 0;   // one buffer: generation (probe load) of item gen_li
  int my_gen = -1;           // one buffer: the generation this issuer holds
  bool ok = true, issued_any = false;
  int li_prev = -1;
  for (int u = X; u < n_uses && ok; u += 2) {
    const int li = u / g.n_chunks, c = u - li * g.n_chunks;
    const int slot = li % sp.n_stages;
    if (li != li_prev) {
      if (!(ok = mbar_wait(sp.k_full + slot, (li / sp.n_stages) & 1, wc, kErrWaitLoad))) break;
      if (sp.q_bufs == 1) {
        // one buffer: generation k of the probe (its k-th load, phase k of q_full)
        // starts at the k-th change of group along the items
        for (; gen_li < li; ++gen_li)
          if (!same_group(items[gen_li + 1], items[gen_li])) ++gen;
        if (gen != my_gen) {
          if (!(ok = mbar_wait(sp.q_full, gen & 1, wc, kErrWaitLoad))) break;
          my_gen = gen;
        }
      }
      li_prev = li;
    }
    if (sp.q_bufs == 2 && chunk_needs_load(2, g.n_chunks, items, li, c)) {
      if (!(ok = mbar_wait(sp.q_full + X, qwaits & 1, wc, kErrWaitLoad))) break;
      ++qwaits;
    }
    if (u >= 2 && !(ok = mbar_wait(sp.acc_empty + X, ((u >> 1) - 1) & 1, wc, kErrWaitMma))) break;
    tc_fence_after();
    const uint32_t ka = smem_u32(sp.sK + slot * kKTileBytes);
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      const uint32_t koff = (kk >> 2) * (128 * 128) + (kk & 3) * 32;
      const uint32_t qoff = (kk >> 2) * qhalf + (kk & 3) * 32;
      mma_ss(tmem + X * 256, sdesc_sw128(ka + koff, 16, 1024), sdesc_sw128(qa + qoff, 16, 1024), idesc,
             kk > 0 ? 1u : 0u);
    }
    mma_commit(sp.acc_full + X);
    issued_any = true;
    const int un = u + 2;
    const int ln = un < n_uses ? un / g.n_chunks : -1;
    if (sp.q_bufs == 1) {
      if (ln < 0 || !same_group(items[ln], items[li])) mma_commit(sp.q_empty + X);
    } else if (ln >= 0 && chunk_needs_load(2, g.n_chunks, items, ln, un - ln * g.n_chunks)) {
      mma_commit(sp.q_empty + X);
    }
    if (ln != li) mma_commit(sp.k_empty + slot);  // this issuer's last use of the K tile
  }
  if (issued_any) {
    mma_commit(sp.drain + X);
    mbar_wait_drain(sp.drain + X, 0, wc);
  }
}

template <int D>
__global__ void __launch_bounds__(256, 1)
    score_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmQp,
                 const ScoreParams p) {
  using S = ScoreShape<D>;
  constexpr uint32_t FULL = 0xffffffffu;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int n_stages = p.k_stages;
  uint8_t* sK = smem + p.q_bufs * p.q_buf_bytes;  // q_buf_bytes is a multiple of 1024
  uint8_t* bar_base = sK + n_stages * S::kKTileBytes;
  const ScorePipe sp = score_pipe_at(smem, sK, p.q_bufs, p.q_buf_bytes, n_stages, reinterpret_cast<uint64_t*>(bar_base));
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar_base + kScorePipeBarBytes);
  int* abort_flag = reinterpret_cast<int*>(tmem_slot + 1);
  int4* s_items = reinterpret_cast<int4*>(bar_base + S::kBarBytes);
  const ScoreGeom geom{p.probe_r, p.group, p.chunk_tokens, p.n_chunks};

  const int warp = warp_id(), lane = lane_id();
  if (threadIdx.x == 0) {
    score_pipe_init(sp, p.n_chunks);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 2) tmem_alloc(tmem_slot, S::kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const WaitCtx wc{abort_flag, p.err_word, p.wait_limit_ns};

  // Contiguous range of items for this CTA.
  const int first = static_cast<int>((static_cast<long long>(p.n_items) * blockIdx.x) / gridDim.x);
  const int last = static_cast<int>((static_cast<long long>(p.n_items) * (blockIdx.x + 1)) / gridDim.x);
  const int n_local = last - first;
  const int G = p.group;
  // The host sizes the grid so that every CTA's range fits the shared-memory cache.
  for (int t = threadIdx.x; t < n_local; t += blockDim.x) s_items[t] = __ldg(p.items + first + t);
  __syncthreads();

  if (warp == 0) {
    if (lane == 0) score_produce<D>(sp, geom, s_items, n_local, &tmK, &tmQp, wc);
    __syncwarp();
  } else if (warp == 1 || warp == 3) {
    if (lane == 0) score_issue<D>(sp, geom, s_items, n_local, warp == 1 ? 0 : 1, tmem, wc);
    __syncwarp();
  } else if (warp >= 4) {
    // ------------------------------------------------------------ epilogue: one key per thread
    const int qd = warp & 3;
    const int row = qd * 32 + lane;
    const uint32_t tl = tmem + (static_cast<uint32_t>(qd * 32) << 16);
    const int Rc = p.chunk_tokens;
    bool ok = true;
    for (int li = 0; li < n_local && ok; ++li) {
      const int4 it = s_items[li];
      const int j = it.z + row;  // key position
      const int e = it.w;
      const bool prob = p.probe_lse != nullptr;
      const bool by_head = p.head_reduce != 0;
      float mx_all = -INFINITY;   // max over heads and rows
      float mh[S::kMaxGroup];     // sum / mean: m_c(j) of each query head (indexed at run time)
      if (by_head) {
#pragma unroll 1
        for (int h = 0; h < G; ++h) mh[h] = -INFINITY;
      }
      for (int c = 0; c < p.n_chunks; ++c) {
        const int u = li * p.n_chunks + c, b = u & 1;
        ok = __all_sync(FULL, mbar_wait(sp.acc_full + b, (u >> 1) & 1, wc, kErrWaitMma));
        if (!ok) break;
        tc_fence_after();
        const int row0 = e - p.probe_r + c * Rc;         // first probe row of the chunk
        const int rc = min(Rc, p.probe_r - c * Rc);      // probe rows in it (a multiple of 16)
        const uint32_t ta = tl + b * 256;
        if (!by_head && !prob && rc == Rc && it.z + 127 < row0) {
          // Max over heads and rows with every column visible to every key of the
          // tile: order-free, whole 128-column TMEM loads and a three-input max tree.
          const int nc = Rc * G;
          int n0 = 0;
#pragma unroll 1  // one 128-register block live at a time
          for (; n0 + 128 <= nc; n0 += 128) {
            uint32_t v[128];
            tmem_ld_x128(ta + n0, v);
            float m8[8];
#pragma unroll
            for (int k = 0; k < 8; ++k) m8[k] = fmaxf(__uint_as_float(v[k]), __uint_as_float(v[k + 8]));
#pragma unroll
            for (int t = 16; t < 128; t += 16)
#pragma unroll
              for (int k = 0; k < 8; ++k) m8[k] = fmax3(m8[k], __uint_as_float(v[t + k]), __uint_as_float(v[t + 8 + k]));
            mx_all = fmax3(mx_all, fmax3(fmax3(m8[0], m8[1], m8[2]), fmax3(m8[3], m8[4], m8[5]), fmaxf(m8[6], m8[7])),
                           -INFINITY);
          }
          for (; n0 < nc; n0 += 16) {
            uint32_t v[16];
            tmem_ld_x16(ta + n0, v);
#pragma unroll
            for (int t = 0; t < 16; ++t) mx_all = fmaxf(mx_all, __uint_as_float(v[t]));
          }
        } else {
          // Per head h: columns [h Rc, h Rc + rc); probe row row0 + t scores key j iff
          // row0 + t >= j.
          const int t_min = j - row0;
#pragma unroll 1
          for (int h = 0; h < G; ++h) {
            float m = -INFINITY;
            const float* lse_h = prob ? p.probe_lse + static_cast<size_t>(it.y * G + h) * p.lse_stride + row0 : nullptr;
            for (int t0 = 0; t0 < rc; t0 += 16) {
              uint32_t v[16];
              tmem_ld_x16(ta + h * Rc + t0, v);
              if (prob) {
                // log probability scale * s - lse_c(row); lane t of each half-warp holds
                // the lse of probe row row0 + t0 + t
                const float lse_lane = __ldg(lse_h + t0 + (lane & 15));
#pragma unroll
                for (int t = 0; t < 16; ++t) {
                  const float lp = fmaf(__uint_as_float(v[t]), p.scale, -__shfl_sync(FULL, lse_lane, t));
                  if (t0 + t >= t_min) m = fmaxf(m, lp);
                }
              } else {
#pragma unroll
                for (int t = 0; t < 16; ++t)
                  if (t0 + t >= t_min) m = fmaxf(m, __uint_as_float(v[t]));
              }
            }
            if (prob) m = expf(m);
            if (by_head)
              mh[h] = fmaxf(mh[h], m);
            else
              mx_all = fmaxf(mx_all, m);
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(sp.acc_empty + b);
      }
      if (!ok) break;
      const float out_scale = prob ? 1.0f : p.scale;  // probabilities carry the scale already
      if (p.head_reduce == 3) {
        if (j < e) {
#pragma unroll 1
          for (int h = 0; h < G; ++h)
            p.scores[(static_cast<size_t>(it.y) * G + h) * p.n_visual + j] = mh[h] * out_scale;
        }
        continue;
      }
      float r = mx_all;
      if (by_head) {
        r = 0.f;
#pragma unroll 1
        for (int h = 0; h < G; ++h) r += mh[h];
        if (p.head_reduce == 2) r = r / static_cast<float>(G);
      }
      if (j < e) p.scores[static_cast<size_t>(it.y) * p.n_visual + j] = r * out_scale;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tmem, S::kTmemCols);
  }
}

}  // namespace spava
