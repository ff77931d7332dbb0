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
// CTA = 256 threads: warp 0 TMA (one thread), warp 1 MMA (one thread), warp 2 TMEM
// allocator, warps 4-7 epilogue (lane = key).  TMEM holds two 256-column accumulators so the
// epilogue of one chunk overlaps the MMA of the next.
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
__device__ __forceinline__ bool score_needs_load(const ScoreParams& p, const int4* items, int li, int c) {
  int cb = c - p.q_bufs, lb = li;
  while (cb < 0) {
    cb += p.n_chunks;
    --lb;
  }
  if (lb < 0) return true;  // first uses of each buffer
  if (cb != c) return true;   // the buffer held another chunk of the probe
  const int4 x = items[li], y = items[lb];
  return x.x != y.x || x.y != y.y;
}

// The use that comes q_bufs uses after (li, c), as (item, chunk).
__device__ __forceinline__ void score_next_use(const ScoreParams& p, int li, int c, int* ln, int* cn) {
  int cc = c + p.q_bufs, l = li;
  while (cc >= p.n_chunks) {
    cc -= p.n_chunks;
    ++l;
  }
  *ln = l;
  *cn = cc;
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
  uint8_t* sQ = smem;
  uint8_t* sK = smem + p.q_bufs * p.q_buf_bytes;   // q_buf_bytes is a multiple of 1024
  uint64_t* bars = reinterpret_cast<uint64_t*>(sK + n_stages * S::kKTileBytes);
  uint64_t* k_full = bars + 0;                   // [kMaxStages]
  uint64_t* k_empty = k_full + S::kMaxStages;    // [kMaxStages]
  uint64_t* q_full = k_empty + S::kMaxStages;    // [2]
  uint64_t* q_empty = q_full + 2;                // [2]
  uint64_t* acc_full = q_empty + 2;              // [2]
  uint64_t* acc_empty = acc_full + 2;            // [2]
  uint64_t* drain = acc_empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  int4* s_items = reinterpret_cast<int4*>(reinterpret_cast<uint8_t*>(bars) + S::kBarBytes);
  int* abort_flag = reinterpret_cast<int*>(tmem_slot + 1);

  const int warp = warp_id(), lane = lane_id();
  if (threadIdx.x == 0) {
    for (int b = 0; b < n_stages; ++b) {
      mbar_init(k_full + b, 1);
      mbar_init(k_empty + b, 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(q_full + b, 1);
      mbar_init(q_empty + b, 1);
      mbar_init(acc_full + b, 1);
      mbar_init(acc_empty + b, 4);  // one arrival per epilogue warp
    }
    mbar_init(drain, 1);
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
    // ------------------------------------------------------------ TMA producer (lane 0)
    if (lane == 0) {
      int qloads[2] = {0, 0};
      int slot = 0, use = 0;  // K stage and how often it was filled before (no division)
      bool ok = true;
      for (int li = 0; li < n_local && ok; ++li) {
        const int4 it = s_items[li];
        if (use > 0 && !(ok = mbar_wait(k_empty + slot, (use - 1) & 1, wc, kErrWaitRelease))) break;
        mbar_arrive_expect_tx(k_full + slot, S::kKTileBytes);
        for (int hh = 0; hh < S::kHalves; ++hh)
          tma_load_3d(sK + slot * S::kKTileBytes + hh * 128 * 128, &tmK, k_full + slot, hh * 64, it.y, it.z);
        if (++slot == n_stages) {
          slot = 0;
          ++use;
        }
        for (int c = 0; c < p.n_chunks; ++c) {
          const int u = li * p.n_chunks + c, b = u & (p.q_bufs - 1);
          if (!score_needs_load(p, s_items, li, c)) continue;
          if (qloads[b] > 0 && !(ok = mbar_wait(q_empty + b, (qloads[b] - 1) & 1, wc, kErrWaitRelease))) break;
          mbar_arrive_expect_tx(q_full + b, static_cast<uint32_t>(S::kHalves * p.chunk_tokens * G * 128));
          for (int hh = 0; hh < S::kHalves; ++hh)
            for (int h = 0; h < G; ++h)
              tma_load_3d(sQ + b * p.q_buf_bytes + hh * (p.chunk_tokens * G * 128) + h * (p.chunk_tokens * 128), &tmQp,
                          q_full + b, hh * 64, it.y * G + h, it.w - p.probe_r + c * p.chunk_tokens);
          ++qloads[b];
        }
      }
      if (!ok) {
        // Abort: let every copy this thread issued land before the CTA exits.
        for (int b = 0; b < n_stages; ++b) {
          const int uses = use + (b < slot ? 1 : 0);  // loads issued into stage b
          if (uses > 0) mbar_wait_drain(k_full + b, (uses - 1) & 1, wc);
        }
        for (int b = 0; b < 2; ++b)
          if (qloads[b] > 0) mbar_wait_drain(q_full + b, (qloads[b] - 1) & 1, wc);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (lane 0)
    // One thread issues every MMA (tcgen05.mma returns once the tensor core has taken
    // the instruction), with no warp-wide votes between them.
    if (lane == 0) {
      int qloads[2] = {0, 0};
      bool ok = true, issued_any = false;
      int slot = 0, kphase = 0;
      for (int li = 0; li < n_local && ok; ++li) {
        if (!(ok = mbar_wait(k_full + slot, kphase, wc, kErrWaitLoad))) break;
        for (int c = 0; c < p.n_chunks; ++c) {
          const int u = li * p.n_chunks + c;
          const int qb = u & (p.q_bufs - 1);  // probe-query buffer (q_bufs is 1 or 2)
          const int ab = u & 1;               // TMEM accumulator
          if (score_needs_load(p, s_items, li, c)) {
            ok = mbar_wait(q_full + qb, qloads[qb] & 1, wc, kErrWaitLoad);
            ++qloads[qb];
            if (!ok) break;
          }
          if (u >= 2 && !(ok = mbar_wait(acc_empty + ab, ((u >> 1) - 1) & 1, wc, kErrWaitMma))) break;
          tc_fence_after();
          // All Rc G columns: with (head, token) order a short last chunk's probe rows
          // are not a prefix; the epilogue masks the rest.
          const int nc = p.chunk_tokens * G;
          const uint32_t idesc = idesc_bf16_f32(128, nc, 0, 0);
          const uint32_t ka = smem_u32(sK + slot * S::kKTileBytes);
          const uint32_t qa = smem_u32(sQ + qb * p.q_buf_bytes);
          const uint32_t qhalf = static_cast<uint32_t>(p.chunk_tokens * G * 128);
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t koff = (kk >> 2) * (128 * 128) + (kk & 3) * 32;
            const uint32_t qoff = (kk >> 2) * qhalf + (kk & 3) * 32;
            mma_ss(tmem + ab * 256, sdesc_sw128(ka + koff, 16, 1024), sdesc_sw128(qa + qoff, 16, 1024), idesc,
                   kk > 0 ? 1u : 0u);
          }
          mma_commit(acc_full + ab);
          int ln, cn;
          score_next_use(p, li, c, &ln, &cn);
          if (ln < n_local && score_needs_load(p, s_items, ln, cn)) mma_commit(q_empty + qb);
          issued_any = true;
        }
        if (!ok) break;
        mma_commit(k_empty + slot);
        if (++slot == n_stages) {
          slot = 0;
          kphase ^= 1;
        }
      }
      if (issued_any) {
        mma_commit(drain);
        mbar_wait_drain(drain, 0, wc);
      }
    }
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
        ok = __all_sync(FULL, mbar_wait(acc_full + b, (u >> 1) & 1, wc, kErrWaitMma));
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
        if (lane == 0) mbar_arrive(acc_empty + b);
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
