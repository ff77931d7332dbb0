// Passing-block selection (top-P per host and KV head), the on-device "pass" of the
// passing blocks (a gather), and the lse merge of split-KV partials.
#pragma once

#include "common.cuh"

namespace spava {


// Exclusive prefix sum over the block (blockDim.x a multiple of 32, <= 1024).
// `scratch` holds 33 uint32.  Also returns the block total through *total.
__device__ __forceinline__ uint32_t block_exclusive_scan(uint32_t v, uint32_t* scratch, uint32_t* total) {
  const int lane = lane_id(), warp = warp_id(), nw = blockDim.x >> 5;
  uint32_t incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) scratch[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    uint32_t w = lane < nw ? scratch[lane] : 0u;
    uint32_t wi = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, wi, o);
      if (lane >= o) wi += y;
    }
    scratch[lane] = wi - w;  // exclusive warp offsets
    if (lane == 31) scratch[32] = wi;
  }
  __syncthreads();
  const uint32_t res = scratch[warp] + incl - v;
  *total = scratch[32];
  __syncthreads();
  return res;
}

// One CTA per (host h < H-1, selection row g: a KV head, or a query head with
// per-query-head selection); with a host list, CTA (s, g) takes host hosts[s]
// (the sharded prefill: a rank's own hosts), else host s.  Candidates: [off[h] + (h == 0 ? A : 0),
// off[h+1]).  Radix select (four 8-bit digits, most significant first) finds the
// P-th largest key T and how many keys equal to T are taken; a stable compaction in
// index order then writes the P winners ascending: keys > T, and the lowest-index
// keys == T.  Result is bit-exact and independent of thread timing.
// Thread t owns the contiguous keys [t*per, (t+1)*per).  With kPer > 0 they are read
// once into registers (segments up to kPer * blockDim.x keys); kPer == 0 re-reads
// them from global memory on every pass (any segment length).
// With kGather the CTA then copies its P passing rows of K and V into host slot s
// of the destination (16 bytes per thread), so the prefill needs no separate gather.
constexpr int kGatherUnroll = 4;

struct GatherArgs {
  const uint4* k;
  const uint4* v;
  uint4* kp;
  uint4* vp;
  int chunks_per_row;  // 16-byte chunks per K/V row (d * 2 / 16)
  int kv_heads;        // hkv (row stride of k and v)
  int group_div;       // selection row r reads KV head r / group_div (1, or G per query head)
  // Destination of passing row j of selection row g in host slot s, in 16-byte
  // chunks: kp + g * dst_g + s * dst_h + j * dst_j.  k_pass/v_pass[g][h][j] has
  // dst_j = chunks_per_row, dst_h = P * dst_j, dst_g = (H-1) * dst_h; the rank-major
  // exchange buffer of the sharded prefill, [slot][j][g], has dst_g = chunks_per_row,
  // dst_j = rows * chunks_per_row, dst_h = P * dst_j.
  size_t dst_g, dst_h, dst_j;
};

template <int kPer, bool kGather>
__global__ void __launch_bounds__(1024) select_topp_kernel(const float* __restrict__ scores, int n_visual,
                                                            const int* __restrict__ off, int anchor, int passing,
                                                            int rows, const int* __restrict__ hosts,
                                                            int32_t* __restrict__ idx, GatherArgs ga) {
  __shared__ uint32_t hist[256];
  __shared__ uint32_t scan_scratch[33];
  __shared__ uint32_t sh_prefix, sh_k;
  const int slot = blockIdx.x / rows, g = blockIdx.x % rows;
  const int h = hosts ? hosts[slot] : slot;
  const int lo = off[h] + (h == 0 ? anchor : 0), hi = off[h + 1];
  const int n = hi - lo;
  const float* s = scores + static_cast<size_t>(g) * n_visual + lo;
  int32_t* out = idx + (static_cast<size_t>(h) * rows + g) * passing;
  const int tid = threadIdx.x, nt = blockDim.x;
  if (passing <= 0) return;
  const int per = (n + nt - 1) / nt;
  const int j0 = min(n, tid * per), cnt = min(n, j0 + per) - j0;

  constexpr int kRegs = kPer > 0 ? kPer : 1;
  uint32_t u[kRegs];
  if (kPer > 0) {
#pragma unroll
    for (int i = 0; i < kRegs; ++i) u[i] = i < cnt ? ordered_key(__ldg(s + j0 + i)) : 0u;
  }
  auto key = [&](int i) -> uint32_t { return kPer > 0 ? u[i] : ordered_key(__ldg(s + j0 + i)); };
  const int n_loop = kPer > 0 ? kRegs : per;

  uint32_t prefix = 0u, pmask = 0u, k = static_cast<uint32_t>(passing);
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int t = tid; t < 256; t += nt) hist[t] = 0u;
    __syncthreads();
#pragma unroll
    for (int i = 0; i < n_loop; ++i) {
      if (i < cnt) {
        const uint32_t x = key(i);
        if ((x & pmask) == prefix) atomicAdd(&hist[(x >> shift) & 0xFFu], 1u);
      }
    }
    __syncthreads();
    if (tid < 32) {
      // lane l owns bins 255-8l .. 248-8l (descending); find the bin holding rank k.
      uint32_t c[8], sum = 0u;
#pragma unroll
      for (int t = 0; t < 8; ++t) {
        c[t] = hist[255 - 8 * tid - t];
        sum += c[t];
      }
      uint32_t incl = sum;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
        if (tid >= o) incl += y;
      }
      const uint32_t excl = incl - sum;
      if (excl < k && k <= incl) {
        uint32_t acc = excl;
#pragma unroll
        for (int t = 0; t < 8; ++t) {
          if (acc + c[t] >= k) {
            sh_prefix = prefix | (static_cast<uint32_t>(255 - 8 * tid - t) << shift);
            sh_k = k - acc;
            break;
          }
          acc += c[t];
        }
      }
    }
    __syncthreads();
    prefix = sh_prefix;
    k = sh_k;
    pmask |= 0xFFu << shift;
  }
  const uint32_t T = prefix;   // key of the P-th largest score
  const uint32_t take_eq = k;  // keys equal to T that are selected (lowest index first)

  uint32_t cgt = 0u, ceq = 0u;
#pragma unroll
  for (int i = 0; i < n_loop; ++i) {
    if (i < cnt) {
      const uint32_t x = key(i);
      cgt += x > T;
      ceq += x == T;
    }
  }
  uint32_t tot;
  const uint32_t eq_before = block_exclusive_scan(ceq, scan_scratch, &tot);
  const uint32_t eq_take = eq_before >= take_eq ? 0u : min(ceq, take_eq - eq_before);
  uint32_t pos = block_exclusive_scan(cgt + eq_take, scan_scratch, &tot);
  uint32_t eq_seen = eq_before;
#pragma unroll
  for (int i = 0; i < n_loop; ++i) {
    if (i < cnt) {
      const uint32_t x = key(i);
      if (x > T) {
        out[pos++] = lo + j0 + i;
      } else if (x == T) {
        if (eq_seen < take_eq) out[pos++] = lo + j0 + i;
        ++eq_seen;
      }
    }
  }
  if (kGather) {
    __syncthreads();  // the block's index writes are visible to the block after this
    // kGatherUnroll rows' chunks per thread are loaded before any is stored, so each
    // SM keeps kGatherUnroll * 2 * 16 B * blockDim.x of K/V reads in flight.
    const int cpr = ga.chunks_per_row;  // a power of two (8 or 16)
    const int cpr_shift = __ffs(cpr) - 1;
    const int total = passing * cpr;
    const size_t dst0 = static_cast<size_t>(g) * ga.dst_g + static_cast<size_t>(slot) * ga.dst_h;
    const int kvh = g / ga.group_div;
    for (int t0 = tid; t0 < total; t0 += kGatherUnroll * nt) {
      uint4 kv[kGatherUnroll], vv[kGatherUnroll];
#pragma unroll
      for (int u = 0; u < kGatherUnroll; ++u) {
        const int t = t0 + u * nt;
        if (t < total) {
          const int r = t >> cpr_shift, ch = t & (cpr - 1);
          const size_t src = (static_cast<size_t>(out[r]) * ga.kv_heads + kvh) * cpr + ch;
          kv[u] = __ldg(ga.k + src);
          vv[u] = __ldg(ga.v + src);
        }
      }
#pragma unroll
      for (int u = 0; u < kGatherUnroll; ++u) {
        const int t = t0 + u * nt;
        if (t < total) {
          const size_t dst = dst0 + static_cast<size_t>(t >> cpr_shift) * ga.dst_j + (t & (cpr - 1));
          ga.kp[dst] = kv[u];
          ga.vp[dst] = vv[u];
        }
      }
    }
  }
}

// Score keys of the two-stage flow: fill with ordered(-inf) before the local pass
// max-reduces into them, and turn them back into fp32 scores afterwards (in place).
__global__ void __launch_bounds__(256) fill_u32_kernel(uint32_t* __restrict__ p, size_t n, uint32_t v) {
  for (size_t t = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x; t < n;
       t += static_cast<size_t>(gridDim.x) * blockDim.x)
    p[t] = v;
}
__global__ void __launch_bounds__(256) keys_to_scores_kernel(uint32_t* __restrict__ p, size_t n) {
  for (size_t t = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x; t < n;
       t += static_cast<size_t>(gridDim.x) * blockDim.x)
    p[t] = __float_as_uint(key_to_float(p[t]));
}

// Two-stage flow with a sum or mean head reduction: keys hold each query head's max
// over its probe rows, [hq][N]; scores[g][j] = sum (or mean) over the G heads of
// group g.  mode 1 sum, 2 mean.
__global__ void __launch_bounds__(256) combine_head_keys_kernel(const uint32_t* __restrict__ keys,
                                                                 float* __restrict__ scores, int hkv, int group,
                                                                 size_t n, int mode) {
  const size_t total = static_cast<size_t>(hkv) * n;
  for (size_t t = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x; t < total;
       t += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const size_t g = t / n, j = t - g * n;
    float r = 0.f;
    for (int c = 0; c < group; ++c) r += key_to_float(__ldg(keys + (g * group + c) * n + j));
    scores[t] = mode == 2 ? r / static_cast<float>(group) : r;
  }
}

// k_pass[g][h][j][:] = k[idx[h][g][j]][g / group_div][:] (same for v), 16 bytes per
// thread; g runs over the selection rows (KV heads, or query heads).
__global__ void __launch_bounds__(256) gather_passing_kernel(const uint4* __restrict__ k, const uint4* __restrict__ v,
                                                              const int32_t* __restrict__ idx, uint4* __restrict__ kp,
                                                              uint4* __restrict__ vp, int rows, int kv_heads,
                                                              int group_div, int hosts_m1, int passing,
                                                              int chunks_per_row) {
  const size_t rows_per_g = static_cast<size_t>(hosts_m1) * passing;
  const size_t total = static_cast<size_t>(rows) * rows_per_g * chunks_per_row;
  for (size_t t = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x; t < total;
       t += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const size_t r = t / chunks_per_row;
    const int ch = static_cast<int>(t - r * chunks_per_row);
    const int g = static_cast<int>(r / rows_per_g);
    const size_t rem = r - static_cast<size_t>(g) * rows_per_g;
    const int h = static_cast<int>(rem / passing);
    const int j = static_cast<int>(rem - static_cast<size_t>(h) * passing);
    const int tok = __ldg(idx + (static_cast<size_t>(h) * rows + g) * passing + j);
    const size_t src = (static_cast<size_t>(tok) * kv_heads + g / group_div) * chunks_per_row + ch;
    kp[t] = __ldg(k + src);
    vp[t] = __ldg(v + src);
  }
}

// Sharded prefill: the passing rows of every host, from the rank-major exchange
// buffer that the ranks' selections filled (row j of host h's slot, selection row g,
// at x[(xrow0[h] + j) * rows + g]), into k_pass/v_pass[g][h][j][:].
__global__ void __launch_bounds__(256) unpack_passing_kernel(const uint4* __restrict__ xk,
                                                              const uint4* __restrict__ xv,
                                                              const int* __restrict__ xrow0, uint4* __restrict__ kp,
                                                              uint4* __restrict__ vp, int rows, int hosts_m1,
                                                              int passing, int chunks_per_row) {
  const size_t rows_per_g = static_cast<size_t>(hosts_m1) * passing;
  const size_t total = static_cast<size_t>(rows) * rows_per_g * chunks_per_row;
  for (size_t t = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x; t < total;
       t += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const size_t r = t / chunks_per_row;
    const int ch = static_cast<int>(t - r * chunks_per_row);
    const int g = static_cast<int>(r / rows_per_g);
    const size_t rem = r - static_cast<size_t>(g) * rows_per_g;
    const int h = static_cast<int>(rem / passing);
    const int j = static_cast<int>(rem - static_cast<size_t>(h) * passing);
    const size_t src = ((static_cast<size_t>(__ldg(xrow0 + h)) + j) * rows + g) * chunks_per_row + ch;
    kp[t] = __ldg(xk + src);
    vp[t] = __ldg(xv + src);
  }
}

// Merge of split-KV partials through their lse (APB-V technical summary,
// 2. System optimisations, "Fused context and query forward"):
//   lse = log sum_k exp(lse_k),  O = sum_k exp(lse_k - lse) O_k.
// One warp per (text row, head); slots with lse = -inf contribute nothing.  Lane k
// reads slot k's lse (so the slots' loads go out together), the maximum and the
// weights are formed with shuffles, and the O partials are read kMergeUnroll slots
// at a time.
constexpr int kMergeUnroll = 4;

__global__ void __launch_bounds__(256) lse_merge_kernel(const float* __restrict__ o_part,
                                                         const float* __restrict__ lse_part, int n_slots,
                                                         int part_rows, int hq, int d, int row0, int n_rows_out,
                                                         __nv_bfloat16* __restrict__ o, float* __restrict__ lse) {
  const int gw = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = lane_id();
  if (gw >= part_rows * hq) return;
  const int t = gw / hq, c = gw % hq;
  // slot lse values, 32 per pass of the warp
  float m = -INFINITY;
  for (int k0 = 0; k0 < n_slots; k0 += 32) {
    const int k = k0 + lane;
    const float l = k < n_slots ? __ldg(lse_part + (static_cast<size_t>(k) * hq + c) * part_rows + t) : -INFINITY;
    m = fmaxf(m, l);
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
  float wsum = 0.f;
  float acc[4] = {0.f, 0.f, 0.f, 0.f};  // d <= 128: lane owns d/32 <= 4 columns
  const int per = d / 32;
  for (int k0 = 0; k0 < n_slots; k0 += 32) {
    const int kl = k0 + lane;
    const float l = kl < n_slots ? __ldg(lse_part + (static_cast<size_t>(kl) * hq + c) * part_rows + t) : -INFINITY;
    const float w_lane = (l == -INFINITY) ? 0.f : expf(l - m);
    const int kn = min(32, n_slots - k0);
    for (int kb = 0; kb < kn; kb += kMergeUnroll) {
      float x[kMergeUnroll][4];
#pragma unroll
      for (int u = 0; u < kMergeUnroll; ++u) {
        const int k = k0 + kb + u;
        const float* src = o_part + ((static_cast<size_t>(min(k, n_slots - 1)) * part_rows + t) * hq + c) * d;
#pragma unroll
        for (int e = 0; e < 4; ++e) x[u][e] = (e < per && kb + u < kn) ? __ldg(src + lane + 32 * e) : 0.f;
      }
#pragma unroll
      for (int u = 0; u < kMergeUnroll; ++u) {
        const float w = __shfl_sync(0xffffffffu, w_lane, (kb + u) & 31);
        if (kb + u < kn) {
          wsum += w;
#pragma unroll
          for (int e = 0; e < 4; ++e) acc[e] = fmaf(w, x[u][e], acc[e]);
        }
      }
    }
  }
  const float inv = 1.0f / wsum;
  __nv_bfloat16* dst = o + (static_cast<size_t>(row0 + t) * hq + c) * d;
  for (int e = 0; e < per; ++e) dst[lane + 32 * e] = __float2bfloat16_rn(acc[e] * inv);
  if (lane == 0) lse[static_cast<size_t>(c) * n_rows_out + row0 + t] = m + logf(wsum);
}

}  // namespace spava
