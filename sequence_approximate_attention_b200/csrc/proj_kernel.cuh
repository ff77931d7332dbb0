// The linear maps around the attention of one decoder layer, on the tensor cores
// (tcgen05 MMA, TMEM accumulators, TMA loads), for the multi-layer prefill whose
// time to first token the pages report (APB-V technical summary, "Experimental
// results"; the query segment's forward is fused with the context's, 2. System
// optimisations, "Fused context and query forward").
//
//   QKV mode:       y = diag(inv_rms) (x W_qkv^T); columns [0, hq d) of y are q,
//                   [hq d, (hq + hkv) d) k and the rest v, each written straight into
//                   its [tokens, heads, d] tensor.  The RMSNorm of x is the row scale
//                   inv_rms applied to the fp32 accumulator (rms_rows_kernel computes
//                   it), so the normalised activations are never stored.
//   residual mode:  out = residual + x W_o^T (out may be the residual itself).
//
// x [M, K] and W [N, K] are bf16 with K contiguous (both operands K-major).  Tile
// 128 x 256 x 64: one CTA per SM, persistent over the (m, n) tiles in m-major
// order, so the CTAs running at one time share a few rows of x and all of W in L2.
//   warp 0      TMA producer (one thread): A (x rows) and B (W rows) into a 4-stage ring
//   warp 1      MMA issuer (one thread): M = 128, N = 256, K = 16 per instruction
//   warp 2      TMEM allocator: two 256-column accumulators, so the epilogue of one
//               tile runs under the MMAs of the next
//   warps 4-7   epilogue: one output row per thread, 32 columns per TMEM load
#pragma once

#include "common.cuh"

namespace spava {

enum : int { kProjQKV = 0, kProjResidual = 1 };

struct ProjParams {
  int M, K, N;       // rows (tokens), inputs, outputs
  int n_tiles_n;     // N / 256
  int n_tiles;       // ceil(M / 128) * n_tiles_n
  int mode;          // kProjQKV or kProjResidual
  int nq, nk;        // QKV mode: hq d and hkv d (multiples of 256)
  __nv_bfloat16* q;  // [M][nq]
  __nv_bfloat16* k;  // [M][nk]
  __nv_bfloat16* v;  // [M][nk]
  const float* inv_rms;          // [M]
  const __nv_bfloat16* residual;  // residual mode: [M][N]
  __nv_bfloat16* out;             // residual mode: [M][N]
  unsigned int* err_word;
  uint64_t wait_limit_ns;
};

struct ProjShape {
  static constexpr int kBM = 128, kBN = 256, kBK = 64;
  static constexpr int kABytes = kBM * 128;  // 128 rows x 64 bf16
  static constexpr int kBBytes = kBN * 128;  // 256 rows x 64 bf16
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kStages = 4;
  static constexpr int kBarOff = kStages * kStageBytes;
  static constexpr int kSmemBytes = kBarOff + 256 + 1024;
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t kIdesc = idesc_bf16_f32(kBM, kBN, 0, 0);
  static constexpr int kThreads = 256;
};

// inv_rms[m] = 1 / sqrt(mean_k x[m][k]^2 + eps), one warp per row, fp32 sums of the
// bf16 inputs (16-byte loads; K a multiple of 256).
__global__ void __launch_bounds__(256) rms_rows_kernel(const __nv_bfloat16* __restrict__ x, int M, int K, float eps,
                                                        float* __restrict__ inv_rms) {
  const int row = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
  if (row >= M) return;
  const uint4* src = reinterpret_cast<const uint4*>(x + static_cast<size_t>(row) * K);
  float ss = 0.f;
  for (int c = lane; c < K / 8; c += 32) {
    const uint4 w = __ldg(src + c);
    const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      const float lo = __uint_as_float(u[t] << 16), hi = __uint_as_float(u[t] & 0xffff0000u);
      ss = fmaf(lo, lo, ss);
      ss = fmaf(hi, hi, ss);
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  if (lane == 0) inv_rms[row] = rsqrtf(ss / static_cast<float>(K) + eps);
}

__global__ void __launch_bounds__(256, 1)
    proj_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                     const ProjParams p) {
  using S = ProjShape;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S::kBarOff);
  uint64_t* full = bars;                    // [kStages]
  uint64_t* empty = full + S::kStages;      // [kStages]
  uint64_t* acc_full = empty + S::kStages;  // [2]
  uint64_t* acc_empty = acc_full + 2;       // [2]
  uint64_t* drain = acc_empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  int* abort_flag = reinterpret_cast<int*>(tmem_slot + 1);

  const int warp = warp_id(), lane = lane_id();
  if (threadIdx.x == 0) {
    for (int s = 0; s < S::kStages; ++s) {
      mbar_init(full + s, 1);
      mbar_init(empty + s, 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(acc_full + b, 1);
      mbar_init(acc_empty + b, 4);  // one arrival per epilogue warp
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 2) tmem_alloc(tmem_slot, S::kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const WaitCtx wc{abort_flag, p.err_word, p.wait_limit_ns};
  const int kb_n = p.K / S::kBK;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer (lane 0)
    if (lane == 0) {
      int ring = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < p.n_tiles && ok; t += gridDim.x) {
        const int m0 = (t / p.n_tiles_n) * S::kBM, n0 = (t % p.n_tiles_n) * S::kBN;
        for (int kb = 0; kb < kb_n; ++kb) {
          const int slot = ring % S::kStages, use = ring / S::kStages;
          if (use > 0 && !(ok = mbar_wait(empty + slot, (use - 1) & 1, wc, kErrWaitRelease))) break;
          uint8_t* st = smem + slot * S::kStageBytes;
          mbar_arrive_expect_tx(full + slot, S::kStageBytes);
          tma_load_2d(st, &tmA, full + slot, kb * S::kBK, m0);                 // rows past M read as zero
          tma_load_2d(st + S::kABytes, &tmB, full + slot, kb * S::kBK, n0);
          ++ring;
        }
      }
      if (!ok) {
        // Abort: let every copy this thread issued land before the CTA exits.
        for (int s = 0; s < S::kStages; ++s) {
          const int uses = ring / S::kStages + (s < ring % S::kStages ? 1 : 0);
          if (uses > 0) mbar_wait_drain(full + s, (uses - 1) & 1, wc);
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (lane 0)
    if (lane == 0) {
      int ring = 0, n_done = 0;
      bool ok = true, issued_any = false;
      const uint64_t a_desc0 = sdesc_sw128(smem_u32(smem), 16, 1024);
      const uint64_t b_desc0 = sdesc_sw128(smem_u32(smem + S::kABytes), 16, 1024);
      for (int t = blockIdx.x; t < p.n_tiles && ok; t += gridDim.x, ++n_done) {
        const int acc = n_done & 1;
        if (n_done >= 2 && !(ok = mbar_wait(acc_empty + acc, ((n_done >> 1) - 1) & 1, wc, kErrWaitMma))) break;
        tc_fence_after();
        for (int kb = 0; kb < kb_n; ++kb) {
          const int slot = ring % S::kStages;
          if (!(ok = mbar_wait(full + slot, (ring / S::kStages) & 1, wc, kErrWaitLoad))) break;
          tc_fence_after();
          const uint32_t so = static_cast<uint32_t>(slot * S::kStageBytes) >> 4;
#pragma unroll
          for (int kk = 0; kk < S::kBK / 16; ++kk)
            mma_ss(tmem + acc * S::kBN, a_desc0 + so + ((kk * 32) >> 4), b_desc0 + so + ((kk * 32) >> 4), S::kIdesc,
                   (kb > 0 || kk > 0) ? 1u : 0u);
          mma_commit(empty + slot);
          issued_any = true;
          ++ring;
        }
        if (!ok) break;
        mma_commit(acc_full + acc);
      }
      if (issued_any) {
        mma_commit(drain);
        mbar_wait_drain(drain, 0, wc);
      }
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ------------------------------------------------------------ epilogue: one row per thread
    const int qd = warp & 3;
    const int row = qd * 32 + lane;
    const uint32_t tl = tmem + (static_cast<uint32_t>(qd * 32) << 16);
    int n_done = 0;
    for (int t = blockIdx.x; t < p.n_tiles; t += gridDim.x, ++n_done) {
      const int acc = n_done & 1;
      if (!__all_sync(0xffffffffu, mbar_wait(acc_full + acc, (n_done >> 1) & 1, wc, kErrWaitMma))) break;
      tc_fence_after();
      const int m = (t / p.n_tiles_n) * S::kBM + row, n0 = (t % p.n_tiles_n) * S::kBN;
      const bool live = m < p.M;
      __nv_bfloat16* dst = nullptr;
      const __nv_bfloat16* res = nullptr;
      float scale = 1.0f;
      if (p.mode == kProjQKV) {
        if (live) scale = __ldg(p.inv_rms + m);
        if (n0 < p.nq)
          dst = p.q + static_cast<size_t>(m) * p.nq + n0;
        else if (n0 < p.nq + p.nk)
          dst = p.k + static_cast<size_t>(m) * p.nk + (n0 - p.nq);
        else
          dst = p.v + static_cast<size_t>(m) * p.nk + (n0 - p.nq - p.nk);
      } else {
        dst = p.out + static_cast<size_t>(m) * p.N + n0;
        res = p.residual + static_cast<size_t>(m) * p.N + n0;
      }
#pragma unroll 1
      for (int c0 = 0; c0 < S::kBN; c0 += 32) {
        uint32_t a[32];
        tmem_ld_x32(tl + acc * S::kBN + c0, a);
        if (!live) continue;
        float f[32];
#pragma unroll
        for (int c = 0; c < 32; ++c) f[c] = __uint_as_float(a[c]) * scale;
        if (p.mode == kProjResidual) {
          const uint4* r4 = reinterpret_cast<const uint4*>(res + c0);
#pragma unroll
          for (int v4 = 0; v4 < 4; ++v4) {
            const uint4 w = r4[v4];
            const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
            for (int t2 = 0; t2 < 4; ++t2) {
              f[8 * v4 + 2 * t2] += __uint_as_float(u[t2] << 16);
              f[8 * v4 + 2 * t2 + 1] += __uint_as_float(u[t2] & 0xffff0000u);
            }
          }
        }
        uint4* d4 = reinterpret_cast<uint4*>(dst + c0);
#pragma unroll
        for (int v4 = 0; v4 < 4; ++v4)
          d4[v4] = make_uint4(pack_bf16x2(f[8 * v4 + 0], f[8 * v4 + 1]), pack_bf16x2(f[8 * v4 + 2], f[8 * v4 + 3]),
                              pack_bf16x2(f[8 * v4 + 4], f[8 * v4 + 5]), pack_bf16x2(f[8 * v4 + 6], f[8 * v4 + 7]));
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(acc_empty + acc);
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
