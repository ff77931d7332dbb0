// Top-P selection of one (host, selection row) by a group of NT threads: the P
// largest of n fp32 scores, ties to the lower index, indices written ascending
// (APB-V technical summary, 1. Framework design, "Approximate attention mechanism":
// each host passes its most essential keys, ranked by query-to-context scores).
// The worker group of the fused score/select/gather launch (8 warps, its own named
// barrier passed as a functor) selects with it.  select_topp_kernel applies the same
// rule with contiguous key ownership and 8-bit digits, which measured faster for a
// whole 1024-thread CTA.
#pragma once

#include "common.cuh"

namespace spava {

// Scratch of one selecting group in shared memory.
struct ToppShared {
  uint32_t hist[2048];  // digit histogram; reused as the (row, warp) count grid (32 (NT/32 + 1) words)
  uint32_t s[200];      // scan and min/max scratch
  uint32_t sel_prefix, sel_k;
};

// Exclusive prefix sum of v over the group's threads (thread t, warp-major order);
// the group total is left in s[2 NW].
template <int NT, class Bar>
__device__ __forceinline__ uint32_t group_exclusive_scan(uint32_t v, uint32_t* s, int t, const Bar& bar) {
  constexpr int NW = NT / 32;
  const int lane = t & 31, w = t >> 5;
  uint32_t incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) s[w] = incl;
  bar();
  if (w == 0) {
    const uint32_t x = lane < NW ? s[lane] : 0u;
    uint32_t xi = x;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, xi, o);
      if (lane >= o) xi += y;
    }
    if (lane < NW) s[NW + lane] = xi - x;  // exclusive warp offsets
    if (lane == 31) s[2 * NW] = xi;
  }
  bar();
  const uint32_t res = s[NW + w] + incl - v;
  bar();
  return res;
}

// Exclusive prefix of per-(row, warp) counts in index order over one block of 32
// rows of NT keys: lane i of warp w passes the count of row i; returns in lane i the
// number of counted keys before (row i, warp w), and the block total in *total.
template <int NT, class Bar>
__device__ __forceinline__ uint32_t row_warp_scan(uint32_t cnt, ToppShared* c, int t, const Bar& bar,
                                                  uint32_t* total) {
  constexpr int NW = NT / 32;
  constexpr int NP = NW + 1;  // padded row: a warp's 32 lanes (rows) fall in 32 banks
  const int lane = t & 31, w = t >> 5;
  uint32_t* grid = c->hist;  // 32 rows of NP words
  grid[lane * NP + w] = cnt;
  bar();
  const int row = t / NW, wv = t - row * NW;  // entry t in index order
  const uint32_t v = grid[row * NP + wv];
  const uint32_t ex = group_exclusive_scan<NT>(v, c->s, t, bar);
  grid[row * NP + wv] = ex;
  bar();
  const uint32_t r = grid[lane * NP + w];
  *total = c->s[2 * NW];
  bar();
  return r;
}

// Top-P of the n candidate scores s[0..n) (token lo + i), written ascending to
// out[0..P).  Thread t owns keys i NT + t (rows of NT keys, read coalesced); with
// kPer > 0 (n <= NT kPer, kPer <= 32) they stay in registers, else every pass reads
// them again from L2.  Radix select of the P-th largest ordered key T: the leading
// bits all keys share (from the group's min and max) are known at once, the rest is
// resolved in digits of up to 11 bits, most significant first.  Then a stable
// compaction in index order (row, warp, lane): keys > T, and the keys == T of lowest
// index, P in all.  A position past P (impossible when the scores are unchanged
// during the call) is not written; it sets kErrBadIndex in *err_word if given.
template <int NT, int kPer, class Bar>
__device__ __forceinline__ void topp_select(const float* s, int n, int lo, int passing, int32_t* out, ToppShared* c,
                                            int t, const Bar& bar, unsigned int* err_word) {
  constexpr int NW = NT / 32;
  constexpr uint32_t FULL = 0xffffffffu;
  const int lane = t & 31, w = t >> 5;
  const int rows = (n + NT - 1) / NT;
  constexpr int kRegs = kPer > 0 ? kPer : 1;
  uint32_t u[kRegs];
  if (kPer > 0) {
#pragma unroll
    for (int i = 0; i < kRegs; ++i) u[i] = i * NT + t < n ? ordered_key(__ldcg(s + i * NT + t)) : 0u;
  }
  auto key = [&](int i) -> uint32_t { return kPer > 0 ? u[i] : ordered_key(__ldcg(s + i * NT + t)); };
  const int n_loop = kPer > 0 ? kRegs : rows;

  // min and max key: the leading bits every key shares
  uint32_t kmin = 0xffffffffu, kmax = 0u;
#pragma unroll
  for (int i = 0; i < n_loop; ++i) {
    if (i * NT + t < n) {
      const uint32_t x = key(i);
      kmin = min(kmin, x);
      kmax = max(kmax, x);
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    kmin = min(kmin, __shfl_xor_sync(FULL, kmin, o));
    kmax = max(kmax, __shfl_xor_sync(FULL, kmax, o));
  }
  uint32_t* smin = c->s + 3 * NW;
  uint32_t* smax = c->s + 4 * NW;
  if (lane == 0) {
    smin[w] = kmin;
    smax[w] = kmax;
  }
  bar();
  kmin = smin[0];
  kmax = smax[0];
  for (int x = 1; x < NW; ++x) {
    kmin = min(kmin, smin[x]);
    kmax = max(kmax, smax[x]);
  }
  bar();
  const int cp = kmin == kmax ? 32 : __clz(kmin ^ kmax);
  uint32_t pmask = cp == 32 ? 0xffffffffu : ~(0xffffffffu >> cp);
  uint32_t prefix = kmax & pmask, k = static_cast<uint32_t>(passing);
  int shift = 32 - cp;
#pragma unroll 1
  while (shift > 0) {
    const int wd = min(11, shift);
    shift -= wd;
    const int nb = 1 << wd;  // bins of this digit
    const uint32_t dmask = static_cast<uint32_t>(nb - 1);
    for (int b = t; b < nb; b += NT) c->hist[b] = 0u;
    bar();
#pragma unroll
    for (int i = 0; i < n_loop; ++i) {
      if (i * NT + t < n) {
        const uint32_t x = key(i);
        if ((x & pmask) == prefix) atomicAdd(&c->hist[(x >> shift) & dmask], 1u);
      }
    }
    bar();
    // thread t owns bins top .. top-bpt+1 (descending order of keys)
    const int bpt = nb >= NT ? nb / NT : 1;
    const int top = nb - 1 - t * bpt;
    uint32_t sum = 0u;
    for (int q = 0; q < bpt && top - q >= 0; ++q) sum += c->hist[top - q];
    const uint32_t excl = group_exclusive_scan<NT>(sum, c->s, t, bar);
    if (excl < k && k <= excl + sum) {
      uint32_t acc = excl;
      for (int q = 0; q < bpt; ++q) {
        const uint32_t cb = c->hist[top - q];
        if (acc + cb >= k) {
          c->sel_prefix = prefix | (static_cast<uint32_t>(top - q) << shift);
          c->sel_k = k - acc;
          break;
        }
        acc += cb;
      }
    }
    bar();
    prefix = c->sel_prefix;
    k = c->sel_k;
    pmask |= dmask << shift;
  }
  const uint32_t T = prefix;   // key of the P-th largest score
  const uint32_t take_eq = k;  // keys equal to T that are taken (lowest index first)

  // compaction over blocks of 32 rows; with the keys in registers there is one block
  // and the row loops unroll (static register indices)
  const uint32_t below = (1u << lane) - 1u;
  constexpr int kRowsPerBlock = kPer > 0 ? kRegs : 32;
  uint32_t eq_base = 0u, win_base = 0u;
#pragma unroll 1
  for (int r0 = 0; r0 < rows; r0 += 32) {
    const int rb = min(32, rows - r0);
    uint32_t eq_cnt = 0u;
#pragma unroll
    for (int i = 0; i < kRowsPerBlock; ++i) {
      if (i < rb) {
        const int ii = r0 + i;
        const bool e = ii * NT + t < n && key(kPer > 0 ? i : ii) == T;
        const uint32_t m = __popc(__ballot_sync(FULL, e));
        if (lane == i) eq_cnt = m;
      }
    }
    uint32_t tot_eq;
    const uint32_t eq_before = row_warp_scan<NT>(eq_cnt, c, t, bar, &tot_eq);  // lane i: row r0 + i
    uint32_t win_cnt = 0u;
#pragma unroll
    for (int i = 0; i < kRowsPerBlock; ++i) {
      if (i < rb) {
        const int ii = r0 + i;
        const bool valid = ii * NT + t < n;
        const uint32_t x = valid ? key(kPer > 0 ? i : ii) : 0u;
        const uint32_t eb = __ballot_sync(FULL, valid && x == T);
        const uint32_t rank = eq_base + __shfl_sync(FULL, eq_before, i) + __popc(eb & below);
        const bool win = valid && (x > T || (x == T && rank < take_eq));
        const uint32_t m = __popc(__ballot_sync(FULL, win));
        if (lane == i) win_cnt = m;
      }
    }
    uint32_t tot_win;
    const uint32_t win_before = row_warp_scan<NT>(win_cnt, c, t, bar, &tot_win);
#pragma unroll
    for (int i = 0; i < kRowsPerBlock; ++i) {
      if (i < rb) {
        const int ii = r0 + i;
        const bool valid = ii * NT + t < n;
        const uint32_t x = valid ? key(kPer > 0 ? i : ii) : 0u;
        const uint32_t eb = __ballot_sync(FULL, valid && x == T);
        const uint32_t rank = eq_base + __shfl_sync(FULL, eq_before, i) + __popc(eb & below);
        const bool win = valid && (x > T || (x == T && rank < take_eq));
        const uint32_t wb = __ballot_sync(FULL, win);
        const uint32_t pos = win_base + __shfl_sync(FULL, win_before, i) + __popc(wb & below);
        if (win) {
          if (pos < static_cast<uint32_t>(passing))
            out[pos] = lo + ii * NT + t;
          else if (err_word)
            atomicOr(err_word, kErrBadIndex);
        }
      }
    }
    eq_base += tot_eq;
    win_base += tot_win;
  }
}

}  // namespace spava
