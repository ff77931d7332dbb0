// Query-to-context scoring on the tensor cores (APB-V technical summary,
// 1. Framework design, "Approximate attention mechanism": every host ranks its
// local keys by query-to-context attention scores).
//
//   score(g, j) = scale * max over probe rows i in [e-R, e), i >= j, and query heads
//                 c of group g of (q_{i,c} . k_{j,g}),   e = end of j's host block.
//
// The product is computed transposed, S^T = K_tile * Qprobe^T, so that each TMEM
// lane holds one key and the max over (probe row, head) is a per-thread reduction
// along the lane's columns (no cross-thread reduction).  The probe queries of one
// (host, KV group) form the MMA's N dimension: rows ordered (token, head) exactly as
// a TMA box (64 x G x Rc) of q lands in shared memory, cut into chunks of at most
// 256 columns.  Work item = one 128-key tile of one (host, KV head).
//
// CTA = 256 threads: warp 0 TMA, warp 1 MMA, warp 2 TMEM allocator,
// warps 4-7 epilogue (lane = key).  TMEM holds two 256-column accumulators so the
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
  int n_visual;      // N (row stride of scores)
  float scale;
  float* scores;     // [hkv][N]
  unsigned int* err_word;
  uint64_t wait_limit_ns;
};

template <int D>
struct ScoreShape {
  static constexpr int kHalves = D / 64;
  static constexpr int kKTileBytes = kHalves * 128 * 128;  // 128 keys
  static constexpr int kQBufBytes = kHalves * 256 * 128;   // up to 256 probe rows
  static constexpr int kKOff = 0;
  static constexpr int kQOff = 2 * kKTileBytes;
  static constexpr int kBarOff = kQOff + 2 * kQBufBytes;
  static constexpr int kSmemBytes = kBarOff + 256 + 1024;
  static constexpr uint32_t kTmemCols = 512;
};

// Chunk-use u of this CTA needs a fresh load of probe queries iff the buffer it
// maps to (u & 1) last held a different (host, group, chunk).
__device__ __forceinline__ bool score_needs_load(const ScoreParams& p, int first, int u) {
  if (u < 2) return true;
  const int a = u, b = u - 2;
  const int ia = first + a / p.n_chunks, ib = first + b / p.n_chunks;
  if (a % p.n_chunks != b % p.n_chunks) return true;
  const int4 x = __ldg(p.items + ia), y = __ldg(p.items + ib);
  return x.x != y.x || x.y != y.y;
}

template <int D>
__global__ void __launch_bounds__(256, 1)
    score_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmQp,
                 const ScoreParams p) {
  using S = ScoreShape<D>;
  constexpr uint32_t FULL = 0xffffffffu;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sK = smem + S::kKOff;
  uint8_t* sQ = smem + S::kQOff;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S::kBarOff);
  uint64_t* k_full = bars + 0;      // [2]
  uint64_t* k_empty = bars + 2;     // [2]
  uint64_t* q_full = bars + 4;      // [2]
  uint64_t* q_empty = bars + 6;     // [2]
  uint64_t* acc_full = bars + 8;    // [2]
  uint64_t* acc_empty = bars + 10;  // [2]
  uint64_t* drain = bars + 12;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 13);
  int* abort_flag = reinterpret_cast<int*>(tmem_slot + 1);

  const int warp = warp_id(), lane = lane_id();
  if (threadIdx.x == 0) {
    for (int b = 0; b < 2; ++b) {
      mbar_init(k_full + b, 1);
      mbar_init(k_empty + b, 1);
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
  const int total_uses = n_local * p.n_chunks;
  const int G = p.group;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    int qloads[2] = {0, 0}, kloads[2] = {0, 0};
    bool ok = true;
    for (int li = 0; li < n_local && ok; ++li) {
      const int4 it = __ldg(p.items + first + li);
      const int slot = li & 1;
      if (li >= 2) {
        ok = __all_sync(FULL, mbar_wait(k_empty + slot, ((li >> 1) - 1) & 1, wc, kErrWaitRelease));
        if (!ok) break;
      }
      if (lane == 0) {
        mbar_arrive_expect_tx(k_full + slot, S::kKTileBytes);
        for (int hh = 0; hh < S::kHalves; ++hh)
          tma_load_3d(sK + slot * S::kKTileBytes + hh * 128 * 128, &tmK, k_full + slot, hh * 64, it.y, it.z);
      }
      __syncwarp();
      ++kloads[slot];
      for (int c = 0; c < p.n_chunks; ++c) {
        const int u = li * p.n_chunks + c, b = u & 1;
        if (!score_needs_load(p, first, u)) continue;
        if (qloads[b] > 0) {
          ok = __all_sync(FULL, mbar_wait(q_empty + b, (qloads[b] - 1) & 1, wc, kErrWaitRelease));
          if (!ok) break;
        }
        if (lane == 0) {
          mbar_arrive_expect_tx(q_full + b, static_cast<uint32_t>(S::kHalves * p.chunk_tokens * G * 128));
          for (int hh = 0; hh < S::kHalves; ++hh)
            tma_load_3d(sQ + b * S::kQBufBytes + hh * (p.chunk_tokens * G * 128), &tmQp, q_full + b, hh * 64,
                        it.y * G, it.w - p.probe_r + c * p.chunk_tokens);
        }
        __syncwarp();
        ++qloads[b];
      }
    }
    if (!ok) {
      // Abort: let every copy this warp issued land before the CTA exits.
      if (lane == 0) {
        for (int b = 0; b < 2; ++b) {
          if (kloads[b] > 0) mbar_wait_drain(k_full + b, (kloads[b] - 1) & 1, wc);
          if (qloads[b] > 0) mbar_wait_drain(q_full + b, (qloads[b] - 1) & 1, wc);
        }
      }
      __syncwarp();
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    int qloads[2] = {0, 0};
    bool ok = true, issued_any = false;
    for (int li = 0; li < n_local && ok; ++li) {
      const int slot = li & 1;
      ok = __all_sync(FULL, mbar_wait(k_full + slot, (li >> 1) & 1, wc, kErrWaitLoad));
      if (!ok) break;
      for (int c = 0; c < p.n_chunks; ++c) {
        const int u = li * p.n_chunks + c, b = u & 1;
        if (score_needs_load(p, first, u)) {
          ok = __all_sync(FULL, mbar_wait(q_full + b, qloads[b] & 1, wc, kErrWaitLoad));
          ++qloads[b];
          if (!ok) break;
        }
        if (u >= 2) {
          ok = __all_sync(FULL, mbar_wait(acc_empty + b, ((u >> 1) - 1) & 1, wc, kErrWaitMma));
          if (!ok) break;
        }
        tc_fence_after();
        const int rc = min(p.chunk_tokens, p.probe_r - c * p.chunk_tokens);
        const int nc = rc * G;
        if (lane == 0) {
          const uint32_t idesc = idesc_bf16_f32(128, nc, 0, 0);
          const uint32_t ka = smem_u32(sK + slot * S::kKTileBytes);
          const uint32_t qa = smem_u32(sQ + b * S::kQBufBytes);
          const uint32_t qhalf = static_cast<uint32_t>(p.chunk_tokens * G * 128);
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t koff = (kk >> 2) * (128 * 128) + (kk & 3) * 32;
            const uint32_t qoff = (kk >> 2) * qhalf + (kk & 3) * 32;
            mma_ss(tmem + b * 256, sdesc_sw128(ka + koff, 16, 1024), sdesc_sw128(qa + qoff, 16, 1024), idesc,
                   kk > 0 ? 1u : 0u);
          }
          mma_commit(acc_full + b);
          if (u + 2 < total_uses && score_needs_load(p, first, u + 2)) mma_commit(q_empty + b);
        }
        issued_any = true;
        __syncwarp();
      }
      if (!ok) break;
      if (lane == 0) mma_commit(k_empty + slot);
      __syncwarp();
    }
    if (issued_any) {
      if (lane == 0) {
        mma_commit(drain);
        mbar_wait_drain(drain, 0, wc);
      }
      __syncwarp();
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------ epilogue: one key per thread
    const int qd = warp & 3;
    const int row = qd * 32 + lane;
    const uint32_t tl = tmem + (static_cast<uint32_t>(qd * 32) << 16);
    bool ok = true;
    for (int li = 0; li < n_local && ok; ++li) {
      const int4 it = __ldg(p.items + first + li);
      const int j = it.z + row;  // key position
      const int e = it.w;
      float mx = -INFINITY;
      for (int c = 0; c < p.n_chunks; ++c) {
        const int u = li * p.n_chunks + c, b = u & 1;
        ok = __all_sync(FULL, mbar_wait(acc_full + b, (u >> 1) & 1, wc, kErrWaitMma));
        if (!ok) break;
        tc_fence_after();
        const int rc = min(p.chunk_tokens, p.probe_r - c * p.chunk_tokens);
        const int nc = rc * G;
        // Column n is probe token c*Rc + n/G, i.e. row e - R + c*Rc + n/G; it may score
        // key j iff that row >= j, i.e. n >= G * (j - (e - R + c*Rc)).
        const int col_min = G * (j - (e - p.probe_r + c * p.chunk_tokens));
        for (int n0 = 0; n0 < nc; n0 += 16) {
          uint32_t v[16];
          tmem_ld_x16(tl + b * 256 + n0, v);
          if (col_min <= n0) {
#pragma unroll
            for (int t = 0; t < 16; ++t) mx = fmaxf(mx, __uint_as_float(v[t]));
          } else {
#pragma unroll
            for (int t = 0; t < 16; ++t)
              if (n0 + t >= col_min) mx = fmaxf(mx, __uint_as_float(v[t]));
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(acc_empty + b);
      }
      if (!ok) break;
      if (j < e) p.scores[static_cast<size_t>(it.y) * p.n_visual + j] = mx * p.scale;
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
