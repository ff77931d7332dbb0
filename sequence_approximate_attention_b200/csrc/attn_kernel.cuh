// Variable-length, multi-segment flash-attention forward for sm_100a
// (tcgen05 MMA with TMEM accumulators, TMA loads, warp specialisation).
//
// One work item = up to 256 query rows (two 128-row Q tiles) of one query head,
// attending to the concatenation of up to three KV segments.  A segment is a
// run of rows of K/V (token positions) or of the gathered passing K/V, optionally
// causal (key position <= query position).  For a host h >= 1 of the
// approximate-attention prefill the segments are
//     [anchor rows 0..A) | passing rows of hosts 0..h-1 | own block, causal]
// (APB-V technical summary, 1. Framework design, "Approximate attention
// mechanism"); host 0, dense causal attention and text rows use one causal
// segment, and text rows split over host blocks write fp32 partials with their
// lse for a later merge (2. System optimisations, "Fused context and query
// forward").
//
// CTA = 384 threads, one per SM, persistent over a cost-sorted item list:
//   warp 0      TMA producer (one thread): Q tiles, then K_j, V_j into a ring of smem stages
//   warp 1      MMA issuer (one thread): S_i = Q_i K_j^T (SS), O_i += P_i V_j (P from TMEM)
//   warp 2      TMEM allocator
//   warps 4-7   softmax of Q tile 0 (TMEM lanes 0..127, one row per thread)
//   warps 8-11  softmax of Q tile 1
// TMEM (512 columns): S_0 | S_1 | O_0 | O_1; P_i (bf16) overwrites the first
// half of S_i after the row has been read.  The MMA order
//     S0(0) S1(0) | PV0(j) S0(j+1) PV1(j) S1(j+1) ...
// lets one softmax warpgroup work while the tensor core runs the other tile.
// Online softmax in the exp2 domain with a lazily updated row max: O is only
// rescaled when the max grows by more than 2^8, which is exact after the final
// division by the row sum.
#pragma once

#include "common.cuh"

namespace spava {

enum : int { kSegCausal = 1, kSegPassing = 2 };

struct AttnSeg {
  int row0;   // first row (token position, or row of the passing buffer)
  int len;    // rows in the segment (0 = unused)
  int flags;  // kSegCausal | kSegPassing
  int aux;    // causal segment of a scoring item: end of the host block
};

// What an item does with its result (bits 24..27 of AttnItem::out), plus a flag that
// makes it also contribute probe scores (two-stage flow) and a partial slot.
enum : int {
  kOutFinal = 0,        // bf16 O and lse of these rows
  kOutTextPartial = 1,  // fp32 partial O and lse into text slot (out & 0xFFFF)
  kOutRowPartial = 2,   // fp32 partial O and lse of visual rows (local pass)
  kOutMerge = 3,        // lse-merge with the rows' partial, then bf16 O and lse
  kOutLseOnly = 4,      // the rows' lse alone, into row_lse (probe rows of probability scores)
};
constexpr int kOutScore = 1 << 20;
__host__ __device__ constexpr int make_out(int mode, int slot = 0, bool score = false) {
  return (mode << 24) | (score ? kOutScore : 0) | slot;
}

struct AttnItem {
  int q_row0;  // first query row (token position)
  int q_rows;  // 1..256 valid query rows
  int q_head;  // query head
  int out;     // make_out(mode, slot, score)
  AttnSeg seg[3];
};
static_assert(sizeof(AttnItem) == 64, "AttnItem layout");

struct AttnParams {
  const AttnItem* items;
  int n_items;
  int group;       // hq / hkv
  int pass_per_qhead;  // passing buffers have one row per query head (per-query-head selection)
  int hq;
  int n_rows_out;  // rows of o and lse (N + T)
  __nv_bfloat16* o;
  float* lse;
  float* o_part;    // [slots][part_rows][hq][D]
  float* lse_part;  // [slots][hq][part_rows]
  int part_row0;
  int part_rows;
  float scale_log2;  // softmax scale * log2(e)
  unsigned int* err_word;
  uint64_t wait_limit_ns;
  int stall_producer;
  // two-stage flow
  float* row_o;               // [N][hq][D] fp32 partials of visual rows
  float* row_lse;             // [hq][N]
  unsigned int* score_keys;   // ordered probe-score keys, max-reduced: [hkv][N], or
                              // [hq][N] (one row per query head) when score_per_qhead
  int score_per_qhead;        // the heads are combined later (sum / mean reductions)
  int n_visual;
  int probe_r;
  float scale;                // softmax scale (scores are max(q.k) * scale)
};

// Pairs (out of every 8) whose exp2 runs on the FMA/ALU pipes (exp2_poly2) instead
// of MUFU.  Measured on B200 at this tile shape (two 128-row tiles, 128-key KV
// tiles, one softmax warp per 32 rows), every share above 0 was slower: each
// warp's softmax is bound by its own issue and latency chain, not by MUFU
// throughput, so the extra instructions cost more than the MUFU time they free.
#ifndef SPAVA_POLY_PAIRS_OF_8
#define SPAVA_POLY_PAIRS_OF_8 0
#endif
constexpr int kPolyPairsOf8 = SPAVA_POLY_PAIRS_OF_8;

template <int D>
struct AttnShape {
  static_assert(D == 64 || D == 128, "head_dim");
  static constexpr int kHalves = D / 64;            // 128-byte column blocks per row
  static constexpr int kHalfBytes = 128 * 128;      // 128 rows x 128 bytes
  static constexpr int kTileBytes = kHalves * kHalfBytes;
#ifndef SPAVA_KV_STAGES_D128
#define SPAVA_KV_STAGES_D128 5
#endif
  // K/V ring stages (K and V tiles alternate); Q, the ring and the barriers fill the
  // 227 KB a CTA may use at D = 128.
  static constexpr int kStages = (D == 128) ? SPAVA_KV_STAGES_D128 : 8;
  static constexpr int kQOff = 0;
  static constexpr int kKVOff = 2 * kTileBytes;
  static constexpr int kBarOff = kKVOff + kStages * kTileBytes;
  static constexpr int kSmemBytes = kBarOff + 512 + 1024;
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t kIdescS = idesc_bf16_f32(128, 128, 0, 0);
  static constexpr uint32_t kIdescO = idesc_bf16_f32(128, D, 0, 1);
  static constexpr int kThreads = 384;

  __device__ static constexpr uint32_t tmem_s(int i) { return static_cast<uint32_t>(i * 128); }
  __device__ static constexpr uint32_t tmem_o(int i) { return static_cast<uint32_t>(256 + i * D); }
};

__device__ __forceinline__ int attn_num_tiles(const AttnItem& it) {
  return (it.seg[0].len + 127) / 128 + (it.seg[1].len + 127) / 128 + (it.seg[2].len + 127) / 128;
}

// Segment s of an item, picked with selects so the item stays in registers
// (dynamic indexing of the array would put it in local memory).
__device__ __forceinline__ AttnSeg seg_at(const AttnItem& it, int s) {
  AttnSeg r;
  r.row0 = s == 0 ? it.seg[0].row0 : (s == 1 ? it.seg[1].row0 : it.seg[2].row0);
  r.len = s == 0 ? it.seg[0].len : (s == 1 ? it.seg[1].len : it.seg[2].len);
  r.flags = s == 0 ? it.seg[0].flags : (s == 1 ? it.seg[1].flags : it.seg[2].flags);
  r.aux = s == 0 ? it.seg[0].aux : (s == 1 ? it.seg[1].aux : it.seg[2].aux);
  return r;
}

// Walks the KV tiles of an item in order: segment s, tile t inside it.
struct TileCursor {
  int s, t;
  __device__ __forceinline__ void start(const AttnItem& it) {
    s = 0;
    t = 0;
    settle(it);
  }
  __device__ __forceinline__ void settle(const AttnItem& it) {
    while (s < 3 && seg_at(it, s).len <= t * 128) {
      ++s;
      t = 0;
    }
  }
  __device__ __forceinline__ void next(const AttnItem& it) {
    ++t;
    settle(it);
  }
  __device__ __forceinline__ bool done() const { return s >= 3; }
};

// Column maxima of a warp's 32 rows x 32 columns (v: this lane's row) by recursive
// halving: at each step a lane keeps one half of its columns and sends the other to
// the partner lane (xor 16, 8, 4, 2, 1); 31 shuffles.  On return lane l holds the
// maximum of column l in v[0].
__device__ __forceinline__ void warp_column_max32(float (&v)[32], int lane) {
#pragma unroll
  for (int s = 0; s < 5; ++s) {
    const int half = 16 >> s, mask = 16 >> s;
    const bool upper = (lane & mask) != 0;
#pragma unroll
    for (int k = 0; k < half; ++k) {
      const float keep = upper ? v[k + half] : v[k];
      const float send = upper ? v[k] : v[k + half];
      v[k] = fmaxf(keep, __shfl_xor_sync(0xffffffffu, send, mask));
    }
  }
}

// Static longest-first schedule: items are sorted by cost (descending); CTA b takes
// item r*G + b in even rounds and r*G + G-1-b in odd rounds (snake order).
__device__ __forceinline__ int attn_sched(int r, int b, int G) { return r * G + ((r & 1) ? (G - 1 - b) : b); }

__device__ __forceinline__ AttnItem load_item(const AttnItem* items, int idx) {
  const int4* src = reinterpret_cast<const int4*>(items + idx);
  AttnItem it;
  int4* dst = reinterpret_cast<int4*>(&it);
#pragma unroll
  for (int k = 0; k < 4; ++k) dst[k] = __ldg(src + k);
  return it;
}

template <int D>
__global__ void __launch_bounds__(384, 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmKp,
                    const __grid_constant__ CUtensorMap tmVp, const AttnParams p) {
  using S = AttnShape<D>;
  constexpr uint32_t FULL = 0xffffffffu;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem + S::kQOff;
  uint8_t* sKV = smem + S::kKVOff;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S::kBarOff);
  uint64_t* q_full = bars + 0;
  uint64_t* q_empty = bars + 1;
  uint64_t* kv_full = bars + 2;
  uint64_t* kv_empty = kv_full + S::kStages;
  uint64_t* s_full = kv_empty + S::kStages;  // [2]
  uint64_t* p_full = s_full + 2;             // [2]
  uint64_t* o_full = p_full + 2;             // [2]
  uint64_t* drain = o_full + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  int* abort_flag = reinterpret_cast<int*>(tmem_slot + 1);

  const int warp = warp_id(), lane = lane_id();
  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    for (int s = 0; s < S::kStages; ++s) {
      mbar_init(kv_full + s, 1);
      mbar_init(kv_empty + s, 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(s_full + i, 1);
      mbar_init(p_full + i, 4);  // one arrival per softmax warp
      mbar_init(o_full + i, 1);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
  }
  if (warp == 2) tmem_alloc(tmem_slot, S::kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const WaitCtx wc{abort_flag, p.err_word, p.wait_limit_ns};
  const int G = gridDim.x, cta = blockIdx.x;
  if (warp < 4) {
  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer (lane 0)
    if (lane == 0) {
    int ring = 0, m = 0, q_issued = 0;
    bool ok = true;
#ifndef SPAVA_NO_L2_HINTS
    // Q tiles are read by one item only; K/V rows (own block, anchor, passing) by the
    // items of every query head of the group and every later row block.
    const uint64_t pol_q = l2_policy_evict_first(), pol_kv = l2_policy_evict_last();
#endif
    if (!p.stall_producer) {
      for (int r = 0; ok; ++r) {
        const int idx = attn_sched(r, cta, G);
        if (idx >= p.n_items) break;
        const AttnItem it = load_item(p.items, idx);
        const int kvh = it.q_head / p.group;
        const bool act1 = it.q_rows > 128;
        if (m > 0) {
          ok = mbar_wait(q_empty, (m - 1) & 1, wc, kErrWaitRelease);
          if (!ok) break;
        }
        mbar_arrive_expect_tx(q_full, (act1 ? 2 : 1) * S::kTileBytes);
        for (int i = 0; i < (act1 ? 2 : 1); ++i)
          for (int hh = 0; hh < S::kHalves; ++hh) {
#ifndef SPAVA_NO_L2_HINTS
            tma_load_3d_hint(sQ + i * S::kTileBytes + hh * S::kHalfBytes, &tmQ, q_full, hh * 64, it.q_head,
                             it.q_row0 + i * 128, pol_q);
#else
            tma_load_3d(sQ + i * S::kTileBytes + hh * S::kHalfBytes, &tmQ, q_full, hh * 64, it.q_head,
                        it.q_row0 + i * 128);
#endif
          }
        q_issued = m + 1;
        TileCursor cur;
        for (cur.start(it); !cur.done() && ok; cur.next(it)) {
          const AttnSeg sg = seg_at(it, cur.s);
          const int row = sg.row0 + cur.t * 128;
          const bool passing = (sg.flags & kSegPassing) != 0;
          for (int kv = 0; kv < 2; ++kv) {
            const int slot = ring % S::kStages, use = ring / S::kStages;
            if (use > 0) {
              ok = mbar_wait(kv_empty + slot, (use - 1) & 1, wc, kErrWaitRelease);
              if (!ok) break;
            }
            uint8_t* dst = sKV + slot * S::kTileBytes;
            mbar_arrive_expect_tx(kv_full + slot, S::kTileBytes);
            const CUtensorMap* map = passing ? (kv ? &tmVp : &tmKp) : (kv ? &tmV : &tmK);
            for (int hh = 0; hh < S::kHalves; ++hh) {
#ifndef SPAVA_NO_L2_HINTS
              if (passing)
                tma_load_3d_hint(dst + hh * S::kHalfBytes, map, kv_full + slot, hh * 64, row,
                                 p.pass_per_qhead ? it.q_head : kvh, pol_kv);
              else
                tma_load_3d_hint(dst + hh * S::kHalfBytes, map, kv_full + slot, hh * 64, kvh, row, pol_kv);
#else
              if (passing)
                tma_load_3d(dst + hh * S::kHalfBytes, map, kv_full + slot, hh * 64, row,
                            p.pass_per_qhead ? it.q_head : kvh);
              else
                tma_load_3d(dst + hh * S::kHalfBytes, map, kv_full + slot, hh * 64, kvh, row);
#endif
            }
            ++ring;
          }
        }
        ++m;
      }
    }
    if (!ok) {
      // Abort: let every copy this thread issued land before the CTA exits.
      for (int s = 0; s < S::kStages; ++s) {
        const int uses = ring / S::kStages + (s < ring % S::kStages ? 1 : 0);
        if (uses > 0) mbar_wait_drain(kv_full + s, (uses - 1) & 1, wc);
      }
      if (q_issued > 0) mbar_wait_drain(q_full, (q_issued - 1) & 1, wc);
    }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (lane 0)
    // One thread issues every MMA: tcgen05.mma returns only once the tensor core has
    // taken the instruction, so this thread's issue stream is the tensor core's
    // schedule and any warp-wide vote or reconvergence in it is idle tensor time.
    if (lane == 0) {
    int ring = 0, m = 0;
    uint32_t pc0 = 0, pc1 = 0;
    bool ok = true, issued_any = false;
    // Descriptor bases built once; per MMA only the start-address field moves (it is
    // the low 14 bits of the descriptor, in 16-byte units, and never carries:
    // shared memory addresses stay below 256 KB).  Keeping the issue path down to
    // a handful of integer adds per MMA matters: this one thread feeds the tensor
    // core 32 MMAs per KV tile.
    const uint64_t q_desc0 = sdesc_sw128(smem_u32(sQ), 16, 1024);
    const uint64_t kv_desc0 = sdesc_sw128(smem_u32(sKV), 16, 1024);
    const uint64_t v_desc0 = sdesc_sw128(smem_u32(sKV), S::kHalfBytes, 1024);
    constexpr uint32_t kTileStep = S::kTileBytes >> 4;
    auto issue_s = [&](int i, int slot) {
      const uint64_t qd = q_desc0 + static_cast<uint32_t>(i) * kTileStep;
      const uint64_t kd = kv_desc0 + static_cast<uint32_t>(slot) * kTileStep;
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint32_t off = ((kk >> 2) * S::kHalfBytes + (kk & 3) * 32) >> 4;
        mma_ss(tmem + S::tmem_s(i), qd + off, kd + off, S::kIdescS, kk > 0 ? 1u : 0u);
      }
    };
    auto issue_pv = [&](int i, int slot, bool acc) {
      const uint64_t vd = v_desc0 + static_cast<uint32_t>(slot) * kTileStep;
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        mma_ts(tmem + S::tmem_o(i), tmem + S::tmem_s(i) + kk * 8, vd + ((kk * 2048) >> 4), S::kIdescO,
               (acc || kk > 0) ? 1u : 0u);
      }
    };
    for (int r = 0; ok; ++r) {
      const int idx = attn_sched(r, cta, G);
      if (idx >= p.n_items) break;
      const AttnItem it = load_item(p.items, idx);
      const int nt = attn_num_tiles(it);
      const bool act1 = it.q_rows > 128;
      ok = mbar_wait(q_full, m & 1, wc, kErrWaitLoad);
      if (!ok) break;
      int slotK = ring % S::kStages;
      ok = mbar_wait(kv_full + slotK, (ring / S::kStages) & 1, wc, kErrWaitLoad);
      if (!ok) break;
      ++ring;
      tc_fence_after();
      issue_s(0, slotK);
      mma_commit(s_full + 0);
      if (act1) {
        issue_s(1, slotK);
        mma_commit(s_full + 1);
      }
      mma_commit(kv_empty + slotK);
      if (nt == 1) mma_commit(q_empty);
      issued_any = true;
      for (int j = 0; j < nt; ++j) {
        const int slotV = ring % S::kStages;
        ok = mbar_wait(kv_full + slotV, (ring / S::kStages) & 1, wc, kErrWaitLoad);
        if (!ok) break;
        ++ring;
        // K_{j+1} is waited for before P_0(j): the loads run ahead, and this keeps the
        // wait off the path from the softmax's hand-over to S_0(j+1).
        int slotK2 = -1;
        if (j + 1 < nt) {
          slotK2 = ring % S::kStages;
          ok = mbar_wait(kv_full + slotK2, (ring / S::kStages) & 1, wc, kErrWaitLoad);
          if (!ok) break;
          ++ring;
        }
        ok = mbar_wait(p_full + 0, pc0 & 1, wc, kErrWaitSoftmax);
        ++pc0;
        if (!ok) break;
        tc_fence_after();
        issue_pv(0, slotV, j > 0);
        if (j == nt - 1) mma_commit(o_full + 0);
        if (j + 1 < nt) {
          issue_s(0, slotK2);
          mma_commit(s_full + 0);
        }
        if (act1) {
          ok = mbar_wait(p_full + 1, pc1 & 1, wc, kErrWaitSoftmax);
          ++pc1;
          if (!ok) break;
          tc_fence_after();
          issue_pv(1, slotV, j > 0);
          if (j == nt - 1) mma_commit(o_full + 1);
          if (j + 1 < nt) {
            issue_s(1, slotK2);
            mma_commit(s_full + 1);
          }
        }
        mma_commit(kv_empty + slotV);
        if (j + 1 < nt) {
          mma_commit(kv_empty + slotK2);
          if (j + 1 == nt - 1) mma_commit(q_empty);
        }
      }
      if (!ok) break;
      ++m;
    }
    if (issued_any) {
      // Every MMA issued so far must finish before TMEM is released (on the normal
      // path the softmax warps have already seen them finish; after an abort they
      // may still be running).
      mma_commit(drain);
      mbar_wait_drain(drain, 0, wc);
    }
    }
    __syncwarp();
  }
  } else {
    // ------------------------------------------------------------ softmax / epilogue
    const int i = (warp - 4) >> 2;  // Q tile of this warpgroup
    const int qd = warp & 3;        // TMEM lane quarter
    const int row = qd * 32 + lane;
    const uint32_t tl = tmem + (static_cast<uint32_t>(qd * 32) << 16);
    const float sl2 = p.scale_log2;
    uint32_t sc = 0, oc = 0;
    bool ok = true;
    for (int r = 0; ok; ++r) {
      const int idx = attn_sched(r, cta, G);
      if (idx >= p.n_items) break;
      const AttnItem it = load_item(p.items, idx);
      if (i == 1 && it.q_rows <= 128) continue;
      const int qrow0 = it.q_row0 + i * 128;
      const int qpos = qrow0 + row;
      const int out_mode = (it.out >> 24) & 0xF;
      const bool score_item = (it.out & kOutScore) != 0;
      float m_run = -INFINITY, l_run = 0.f;
      int j = 0;
      TileCursor cur;
      for (cur.start(it); !cur.done(); cur.next(it), ++j) {
        ok = __all_sync(FULL, mbar_wait(s_full + i, sc & 1, wc, kErrWaitMma));
        ++sc;
        if (!ok) break;
        tc_fence_after();
        const AttnSeg sg = seg_at(it, cur.s);
        const int kpos0 = sg.row0 + cur.t * 128;
        const int valid = min(128, sg.len - cur.t * 128);
        const bool causal = (sg.flags & kSegCausal) != 0;
        uint32_t sr[128];
        tmem_ld_x128(tl + S::tmem_s(i), sr);
        if (valid < 128 || (causal && kpos0 + 127 > qrow0)) {
          int lim = valid;
          if (causal) lim = min(lim, qpos - kpos0 + 1);
#pragma unroll
          for (int c = 0; c < 128; ++c)
            if (c >= lim) sr[c] = 0xff800000u;  // -inf
        }
        // Row max: eight independent chains of three-input maxes, then a tree.
        float mx[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) mx[k] = fmaxf(__uint_as_float(sr[k]), __uint_as_float(sr[k + 8]));
#pragma unroll
        for (int c = 16; c < 128; c += 16)
#pragma unroll
          for (int k = 0; k < 8; ++k) mx[k] = fmax3(mx[k], __uint_as_float(sr[c + k]), __uint_as_float(sr[c + 8 + k]));
        const float tmax = fmax3(fmax3(mx[0], mx[1], mx[2]), fmax3(mx[3], mx[4], mx[5]), fmaxf(mx[6], mx[7]));
        const float m_tile = tmax * sl2;
        float alpha = 1.0f;
        bool rescale = false;
        if (j == 0) {
          m_run = m_tile;
        } else {
          const bool need = m_tile > m_run + 8.0f;
          rescale = __any_sync(FULL, need);
          if (need) {
            alpha = fast_exp2(m_run - m_tile);
            m_run = m_tile;
          }
        }
        const float m_use = (m_run == -INFINITY) ? 0.0f : m_run;
        // P = exp2(s * scale_log2 - m) on the MUFU unit, packed to bf16 pairs in place
        // (pair c lands in sr[c] after sr[2c], sr[2c+1] have been read); the scale-
        // subtract and the row sum run as packed fp32 pairs in four chains.
        const float2 sl2x2 = make_float2(sl2, sl2), negm = make_float2(-m_use, -m_use);
        float2 rs[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
        for (int c = 0; c < 64; ++c) {
          const float2 x = ffma2(make_float2(__uint_as_float(sr[2 * c]), __uint_as_float(sr[2 * c + 1])), sl2x2, negm);
          const float2 pp = ((c & 7) < kPolyPairsOf8) ? exp2_poly2(x) : make_float2(fast_exp2(x.x), fast_exp2(x.y));
          rs[c & 3] = fadd2(rs[c & 3], pp);
          sr[c] = pack_bf16x2(pp.x, pp.y);
        }
        const float2 r01 = fadd2(rs[0], rs[1]), r23 = fadd2(rs[2], rs[3]), r = fadd2(r01, r23);
        l_run = l_run * alpha + (r.x + r.y);
        if (score_item && causal && p.score_keys != nullptr) {
          // Two-stage flow: this item holds probe rows [aux - R, aux) of its host; fold
          // their raw q.k into the per-key scores (max over probe rows here, over the
          // group's query heads through the atomic max).  S is still intact in TMEM
          // (P has not been stored yet) and is re-read 32 columns at a time.
          const bool probe_row = qpos >= sg.aux - p.probe_r && qpos < sg.aux && (i * 128 + row) < it.q_rows;
          if (__any_sync(FULL, probe_row)) {
            unsigned int* keys =
                p.score_keys + static_cast<size_t>(p.score_per_qhead ? it.q_head : it.q_head / p.group) * p.n_visual +
                kpos0;
            int lim = valid;
            if (causal) lim = min(lim, qpos - kpos0 + 1);
#pragma unroll 1
            for (int h0 = 0; h0 < 128; h0 += 32) {
              uint32_t raw[32];
              tmem_ld_x32(tl + S::tmem_s(i) + h0, raw);
              float cv[32];
#pragma unroll
              for (int c = 0; c < 32; ++c) cv[c] = (probe_row && h0 + c < lim) ? __uint_as_float(raw[c]) : -INFINITY;
              warp_column_max32(cv, lane);
              const int c = h0 + lane;
              if (c < valid && cv[0] != -INFINITY) atomicMax(keys + c, ordered_key(cv[0] * p.scale));
            }
          }
        }
        tmem_st_x64(tl + S::tmem_s(i), *reinterpret_cast<uint32_t(*)[64]>(sr));
        if (rescale) {
          // O_i holds the sum up to tile j-1 (its MMA finished before S_i(j) did).
#pragma unroll
          for (int c0 = 0; c0 < D; c0 += 32) {
            uint32_t ov[32];
            tmem_ld_x32(tl + S::tmem_o(i) + c0, ov);
#pragma unroll
            for (int c = 0; c < 32; ++c) ov[c] = __float_as_uint(__uint_as_float(ov[c]) * alpha);
            tmem_st_x32(tl + S::tmem_o(i) + c0, ov);
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(p_full + i);
      }
      if (!ok) break;
      ok = __all_sync(FULL, mbar_wait(o_full + i, oc & 1, wc, kErrWaitMma));
      ++oc;
      if (!ok) break;
      tc_fence_after();
      const float m_use = (m_run == -INFINITY) ? 0.0f : m_run;
      const float inv_l = l_run > 0.f ? 1.0f / l_run : 0.0f;
      const bool store = (i * 128 + row) < it.q_rows;
      const int grow = qpos;
      const float lse_own = (m_use + log2f(l_run)) * 0.69314718055994531f;
      if (out_mode == kOutFinal || out_mode == kOutMerge) {
        // kOutMerge: combine with the rows' local partial through the lse.
        float w_own = inv_l, w_loc = 0.f, lse_out = lse_own;
        const float* lrow = nullptr;
        if (out_mode == kOutMerge) {
          const float lse_loc = p.row_lse[static_cast<size_t>(it.q_head) * p.n_visual + grow];
          const float mm = fmaxf(lse_loc, lse_own);
          const float e_loc = expf(lse_loc - mm), e_own = expf(lse_own - mm);
          lse_out = mm + logf(e_loc + e_own);
          const float inv = 1.0f / (e_loc + e_own);
          w_own = inv_l * e_own * inv;
          w_loc = e_loc * inv;
          lrow = p.row_o + (static_cast<size_t>(grow) * p.hq + it.q_head) * D;
        }
        __nv_bfloat16* orow = p.o + (static_cast<size_t>(grow) * p.hq + it.q_head) * D;
#pragma unroll
        for (int c0 = 0; c0 < D; c0 += 32) {
          uint32_t ov[32];
          tmem_ld_x32(tl + S::tmem_o(i) + c0, ov);
          if (store) {
            float f[32];
#pragma unroll
            for (int c = 0; c < 32; ++c) f[c] = __uint_as_float(ov[c]) * w_own;
            if (out_mode == kOutMerge) {
              const float4* src = reinterpret_cast<const float4*>(lrow + c0);
#pragma unroll
              for (int v4 = 0; v4 < 8; ++v4) {
                const float4 x = src[v4];
                f[4 * v4 + 0] = fmaf(x.x, w_loc, f[4 * v4 + 0]);
                f[4 * v4 + 1] = fmaf(x.y, w_loc, f[4 * v4 + 1]);
                f[4 * v4 + 2] = fmaf(x.z, w_loc, f[4 * v4 + 2]);
                f[4 * v4 + 3] = fmaf(x.w, w_loc, f[4 * v4 + 3]);
              }
            }
            uint4* dst = reinterpret_cast<uint4*>(orow + c0);
#pragma unroll
            for (int v4 = 0; v4 < 4; ++v4) {
              uint4 w;
              w.x = pack_bf16x2(f[8 * v4 + 0], f[8 * v4 + 1]);
              w.y = pack_bf16x2(f[8 * v4 + 2], f[8 * v4 + 3]);
              w.z = pack_bf16x2(f[8 * v4 + 4], f[8 * v4 + 5]);
              w.w = pack_bf16x2(f[8 * v4 + 6], f[8 * v4 + 7]);
              dst[v4] = w;
            }
          }
        }
        if (store) p.lse[static_cast<size_t>(it.q_head) * p.n_rows_out + grow] = lse_out;
      } else {
        // fp32 partials: a text slot, or the visual rows of the local pass
        float* orow;
        float* lse_dst;
        if (out_mode == kOutLseOnly) {
          if (store) p.row_lse[static_cast<size_t>(it.q_head) * p.n_visual + grow] = lse_own;
          continue;
        }
        if (out_mode == kOutTextPartial) {
          const int slot = it.out & 0xFFFF, prow = grow - p.part_row0;
          orow = p.o_part + ((static_cast<size_t>(slot) * p.part_rows + prow) * p.hq + it.q_head) * D;
          lse_dst = p.lse_part + (static_cast<size_t>(slot) * p.hq + it.q_head) * p.part_rows + prow;
        } else {
          orow = p.row_o + (static_cast<size_t>(grow) * p.hq + it.q_head) * D;
          lse_dst = p.row_lse + static_cast<size_t>(it.q_head) * p.n_visual + grow;
        }
#pragma unroll
        for (int c0 = 0; c0 < D; c0 += 32) {
          uint32_t ov[32];
          tmem_ld_x32(tl + S::tmem_o(i) + c0, ov);
          if (store) {
            float4* dst = reinterpret_cast<float4*>(orow + c0);
#pragma unroll
            for (int v4 = 0; v4 < 8; ++v4)
              dst[v4] = make_float4(__uint_as_float(ov[4 * v4 + 0]) * inv_l, __uint_as_float(ov[4 * v4 + 1]) * inv_l,
                                    __uint_as_float(ov[4 * v4 + 2]) * inv_l, __uint_as_float(ov[4 * v4 + 3]) * inv_l);
          }
        }
        if (store) *lse_dst = lse_own;
      }
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
