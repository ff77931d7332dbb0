// Host side of the C ABI declared in include/spava.h: plan (context splitting and
// the cost-sorted work lists), argument checks, TMA descriptors and launches.
//
// Call graph of spava_attn_prefill, all on the caller's stream:
//   score_kernel      probe scores of hosts 0..H-2 (tensor cores)
//   select_topp       top-P passing keys per (host, KV head), each CTA then
//                     gathering its passing K/V rows into one contiguous buffer
//                     per KV head (spava_gather_passing runs that gather alone)
//   attn_fwd_kernel   one flash-attention pass per host item, text rows as
//                     split-KV partials over the host blocks
//   lse_merge         text partials -> final rows
#include "spava.h"

#include <cudaTypedefs.h>

#include <algorithm>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>
#include <vector>

#include "attn_kernel.cuh"
#include "common.cuh"
#include "proj_kernel.cuh"
#include "score_kernel.cuh"
#include "ssg_kernel.cuh"
#include "select_gather.cuh"

using spava::AttnItem;
using spava::AttnParams;
using spava::AttnSeg;
using spava::ScoreParams;

namespace {

thread_local std::string g_last_error;
thread_local int g_last_launches = 0;

spava_status fail(spava_status st, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return st;
}

spava_status ok() {
  g_last_error.clear();
  return SPAVA_OK;
}

#define SPAVA_CUDA(call)                                                                            \
  do {                                                                                             \
    cudaError_t e_ = (call);                                                                       \
    if (e_ != cudaSuccess) return fail(SPAVA_ERR_CUDA, "%s: %s", #call, cudaGetErrorString(e_)); \
  } while (0)

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// 3-D bf16 tensor map with 128-byte swizzle over a row-major [d2][d1][d0] tensor;
// d0 is contiguous.  The box is (64, b1, b2); out-of-range rows read as zero.
spava_status make_map(CUtensorMap* map, const void* base, uint64_t d0, uint64_t d1, uint64_t d2, uint32_t b1,
                      uint32_t b2) {
  auto fn = encode_fn();
  if (!fn) return fail(SPAVA_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
  const cuuint64_t dims[3] = {d0, d1, d2};
  const cuuint64_t strides[2] = {d0 * 2, d0 * d1 * 2};
  const cuuint32_t box[3] = {64, b1, b2};
  const cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(SPAVA_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", static_cast<int>(r));
  return SPAVA_OK;
}

// 2-D bf16 tensor map with 128-byte swizzle over a row-major [outer][inner] matrix
// (inner contiguous); box (64, box_outer); rows past `outer` read as zero.
spava_status make_map_2d(CUtensorMap* map, const void* base, uint64_t inner, uint64_t outer, uint32_t box_outer) {
  auto fn = encode_fn();
  if (!fn) return fail(SPAVA_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {inner * 2};
  const cuuint32_t box[2] = {64, box_outer};
  const cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(SPAVA_ERR_CUDA, "cuTensorMapEncodeTiled (2-D) failed (%d)", static_cast<int>(r));
  return SPAVA_OK;
}

}  // namespace

struct spava_plan {
  int N = 0, T = 0, H = 0, A = 0, P = 0, R = 0, hq = 0, hkv = 0, d = 0;
  float scale = 0.f;
  std::vector<int> off;
  int device = 0, num_sms = 0;
  // score chunking: Rc probe tokens per MMA N chunk
  int rc = 0, n_chunks = 0;
  int score_reduce = SPAVA_SCORE_MAX;  // spava_plan_set_score_reduce
  int score_kind = SPAVA_SCORE_LOGIT;  // spava_plan_set_score_kind
  int fused_select = 0;                // spava_plan_set_fused_select
  // device table (owned)
  void* dtab = nullptr;
  int* d_off = nullptr;
  AttnItem* d_items_pre = nullptr;
  int n_items_pre = 0;
  AttnItem* d_items_dense = nullptr;
  int n_items_dense = 0;
  AttnItem* d_items_local = nullptr;   // two-stage flow, first launch
  int n_items_local = 0;
  AttnItem* d_items_remote = nullptr;  // two-stage flow, second launch
  int n_items_remote = 0;
  AttnItem* d_items_probe = nullptr;   // probability scores: lse of every host's probe rows
  int n_items_probe = 0;
  int4* d_score_pre = nullptr;  // hosts 0..H-2
  int n_score_pre = 0;
  int4* d_score_all = nullptr;  // all hosts
  int n_score_all = 0;
  // fused score/select/gather: hosts 0..H-2's score tiles dealt to ssg_grid CTAs in
  // rounds; CTA b takes d_ssg_items[d_ssg_first[b] .. d_ssg_first[b+1])
  int4* d_ssg_items = nullptr;
  int* d_ssg_first = nullptr;
  int ssg_grid = 0, ssg_max_local = 0;
  // sharded prefill (spava_plan_set_shard): this rank's work lists in their own
  // device table; the exchange buffers' slots per rank
  int shard_rank = 0, shard_world = 0;  // world 0: not sharded
  std::vector<int> owner;               // rank of each host
  int pass_slots = 0, text_slots = 0;   // per rank
  int text_slots_used = 0;              // this rank's text pieces
  void* dtab_shard = nullptr;
  int* d_shard_hosts = nullptr;  // own hosts < H-1, ascending: the select grid's host list
  int n_shard_hosts = 0;
  int* d_xrow0 = nullptr;        // [H-1] first exchange row of each host's passing rows
  int4* d_score_shard = nullptr;
  int n_score_shard = 0;
  AttnItem* d_items_shard_local = nullptr;
  int n_items_shard_local = 0;
  AttnItem* d_items_shard_remote = nullptr;
  int n_items_shard_remote = 0;
  AttnItem* d_items_shard_probe = nullptr;
  int n_items_shard_probe = 0;
  AttnItem* d_items_shard_pre = nullptr;  // one-pass form (SPAVA_SHARD_ATTEND)
  int n_items_shard_pre = 0;
  // workspace layout
  size_t ws_err = 0, ws_sync = 0, ws_scores = 0, ws_idx = 0, ws_kp = 0, ws_vp = 0, ws_opart = 0, ws_lpart = 0, ws_total = 0;
  size_t ws_row_o = 0, ws_row_lse = 0, ws_qkeys = 0, ws_total_two_stage = 0;  // two-stage flow only
  size_t ws_probe_lse = 0;  // probability scores: [hq][N] lse (probe rows only)
  size_t ws_xk = 0, ws_xv = 0, ws_to = 0, ws_tl = 0, ws_total_shard = 0;  // sharded prefill
  // debug knobs
  uint64_t wait_limit_ns = spava::kDefaultWaitLimitNs;
  int stall_producer = 0;
  // kernel timing hook: one event per mark, the label of the kernel that follows
  // it (-1 = end of call) and the call it belongs to
  mutable std::vector<cudaEvent_t> prof_ev;
  mutable std::vector<int> prof_label, prof_call;
  mutable int prof_used = 0, prof_call_id = 0;
};

namespace {

int ceil_div(int a, int b) { return (a + b - 1) / b; }

enum KernelLabel {
  kLabScore = 0, kLabSelect = 1, kLabGather = 2, kLabAttn = 3, kLabMerge = 4, kLabDense = 5, kLabSelectGather = 6,
  kLabFill = 7, kLabAttnLocal = 8, kLabAttnRemote = 9, kLabProbeLse = 10, kLabUnpack = 11, kLabTextFill = 12,
  kLabScoreSelectGather = 13
};

void mark(const spava_plan* p, int label, cudaStream_t st) {
  if (p->prof_used >= static_cast<int>(p->prof_ev.size())) return;
  if (cudaEventRecord(p->prof_ev[p->prof_used], st) != cudaSuccess) return;
  p->prof_label[p->prof_used] = label;
  p->prof_call[p->prof_used] = p->prof_call_id;
  ++p->prof_used;
}

int item_cost(const AttnItem& it) {
  int tiles = 0;
  for (int s = 0; s < 3; ++s) tiles += ceil_div(it.seg[s].len, 128);
  return tiles * (it.q_rows > 128 ? 2 : 1);
}

void sort_by_cost(std::vector<AttnItem>& v) {
  std::stable_sort(v.begin(), v.end(), [](const AttnItem& a, const AttnItem& b) { return item_cost(a) > item_cost(b); });
}

// Prefill order: KV groups in order; inside a group, hosts from the longest KV list to
// the shortest; longest items first inside a (group, host).  Consecutive items (which
// run at the same time on the 148 CTAs) then share one host's block of one KV head,
// and every host of a group reads the same anchor and passing rows of that KV head,
// which therefore stay in L2 from the first host of the group to the last (ordering
// hosts outermost re-read them from DRAM once per host); every round of CTAs still
// gets a spread of item costs for balance.
// `group` gives each item its host (text pieces are grouped with the host block
// they read, their own causal piece with the last host).
void sort_host_major(std::vector<AttnItem>& v, const std::vector<int>& group, int heads_per_group) {
  auto kv_group_of = [&](const AttnItem& it) { return it.q_head / heads_per_group; };
  std::vector<int> order(v.size());
  for (size_t i = 0; i < v.size(); ++i) order[i] = static_cast<int>(i);
  std::stable_sort(order.begin(), order.end(), [&](int a, int b) {
    if (kv_group_of(v[a]) != kv_group_of(v[b])) return kv_group_of(v[a]) < kv_group_of(v[b]);
    if (group[a] != group[b]) return group[a] > group[b];
    return item_cost(v[a]) > item_cost(v[b]);
  });
  std::vector<AttnItem> out;
  out.reserve(v.size());
  for (int i : order) out.push_back(v[i]);
  v.swap(out);
}

AttnItem blank_item(int q_row0, int q_rows, int q_head, int out) {
  AttnItem it;
  std::memset(&it, 0, sizeof(it));
  it.q_row0 = q_row0;
  it.q_rows = q_rows;
  it.q_head = q_head;
  it.out = out;
  return it;
}

// Which hosts a work list covers: every host (nullptr), or one rank's hosts in the
// sharded prefill.
using HostMask = std::vector<char>;
bool runs(const HostMask* mine, int h) { return !mine || (*mine)[h] != 0; }

// Text-query pieces of the prefill (shared by all flows): T rows in 256-row items,
// split over the host blocks (piece k < H) plus their own causal part (piece H),
// each an fp32 partial into slot k, or into slot[k] when a slot map is given
// (pieces with slot -1 belong to other ranks).
void add_text_items(const spava_plan& p, std::vector<AttnItem>& v, std::vector<int>& group,
                    const std::vector<int>* slot = nullptr) {
  for (int r0 = p.N; r0 < p.N + p.T; r0 += 256) {
    const int rows = std::min(256, p.N + p.T - r0);
    for (int c = 0; c < p.hq; ++c) {
      for (int k = 0; k <= p.H; ++k) {
        const int sl = slot ? (*slot)[k] : k;
        if (sl < 0) continue;
        AttnItem it = blank_item(r0, rows, c, spava::make_out(spava::kOutTextPartial, sl));
        if (k < p.H)
          it.seg[0] = AttnSeg{p.off[k], p.off[k + 1] - p.off[k], 0, 0};
        else
          it.seg[0] = AttnSeg{p.N, r0 + rows - p.N, spava::kSegCausal, 0};
        v.push_back(it);
        group.push_back(k < p.H ? k : p.H - 1);
      }
    }
  }
}

// Work list of the prefill.  Host h's rows go in 256-row items per query head with
// the KV list [anchor | passing of hosts < h | own block, causal]; text rows (the
// query block) are split over the host blocks plus their own causal part, each
// piece writing an fp32 partial with its lse.  With a host mask (sharded prefill)
// only those hosts' rows and text pieces, into the given text slots.
std::vector<AttnItem> build_prefill_items(const spava_plan& p, const HostMask* mine = nullptr,
                                          const std::vector<int>* text_slot = nullptr) {
  std::vector<AttnItem> v;
  std::vector<int> group;
  for (int h = 0; h < p.H; ++h) {
    if (!runs(mine, h)) continue;
    const int a = p.off[h], e = p.off[h + 1];
    for (int r0 = a; r0 < e; r0 += 256) {
      const int rows = std::min(256, e - r0);
      for (int c = 0; c < p.hq; ++c) {
        AttnItem it = blank_item(r0, rows, c, spava::make_out(spava::kOutFinal));
        int ns = 0;
        if (h >= 1 && p.A > 0) it.seg[ns++] = AttnSeg{0, p.A, 0, 0};
        if (h >= 1 && p.P > 0) it.seg[ns++] = AttnSeg{0, h * p.P, spava::kSegPassing, 0};
        it.seg[ns++] = AttnSeg{a, r0 + rows - a, spava::kSegCausal, 0};
        v.push_back(it);
        group.push_back(h);
      }
    }
  }
  add_text_items(p, v, group, text_slot);
  sort_host_major(v, group, p.hq / p.hkv);
  return v;
}

bool has_remote(const spava_plan& p, int h) { return h >= 1 && (p.A > 0 || p.P > 0); }
bool scores_needed(const spava_plan& p) { return p.H >= 2 && p.P > 0; }

// Two-stage flow, first launch: every host's queries over its own block (causal).
// Hosts with a remote part write fp32 partials of their rows; items holding probe
// rows of hosts < H-1 also fold their logits into the probe scores (one GPU; the
// sharded prefill scores with the score kernel first).  Text pieces run here too.
std::vector<AttnItem> build_local_items(const spava_plan& p, const HostMask* mine = nullptr,
                                        const std::vector<int>* text_slot = nullptr) {
  std::vector<AttnItem> v;
  std::vector<int> group;
  for (int h = 0; h < p.H; ++h) {
    if (!runs(mine, h)) continue;
    const int a = p.off[h], e = p.off[h + 1];
    for (int r0 = a; r0 < e; r0 += 256) {
      const int rows = std::min(256, e - r0);
      const bool probe = !mine && scores_needed(p) && h < p.H - 1 && r0 + rows > e - p.R;
      const int mode = has_remote(p, h) ? spava::kOutRowPartial : spava::kOutFinal;
      for (int c = 0; c < p.hq; ++c) {
        AttnItem it = blank_item(r0, rows, c, spava::make_out(mode, 0, probe));
        it.seg[0] = AttnSeg{a, r0 + rows - a, spava::kSegCausal, e};
        v.push_back(it);
        group.push_back(h);
      }
    }
  }
  add_text_items(p, v, group, text_slot);
  sort_host_major(v, group, p.hq / p.hkv);
  return v;
}

// Two-stage flow, second launch: host h >= 1 over [anchor | passing of hosts < h],
// lse-merged with its local partial into the final output.
std::vector<AttnItem> build_remote_items(const spava_plan& p, const HostMask* mine = nullptr) {
  std::vector<AttnItem> v;
  std::vector<int> group;
  for (int h = 1; h < p.H; ++h) {
    if (!has_remote(p, h) || !runs(mine, h)) continue;
    const int a = p.off[h], e = p.off[h + 1];
    for (int r0 = a; r0 < e; r0 += 256) {
      const int rows = std::min(256, e - r0);
      for (int c = 0; c < p.hq; ++c) {
        AttnItem it = blank_item(r0, rows, c, spava::make_out(spava::kOutMerge));
        int ns = 0;
        if (p.A > 0) it.seg[ns++] = AttnSeg{0, p.A, 0, 0};
        if (p.P > 0) it.seg[ns++] = AttnSeg{0, h * p.P, spava::kSegPassing, 0};
        v.push_back(it);
        group.push_back(h);
      }
    }
  }
  sort_host_major(v, group, p.hq / p.hkv);
  return v;
}

// Probability scores: the last R rows of every host h < h_end over its own block
// (causal), lse only -- each probe row's log-sum-exp over the keys of its block it sees.
std::vector<AttnItem> build_probe_items(const spava_plan& p, int h_end, const HostMask* mine = nullptr) {
  std::vector<AttnItem> v;
  std::vector<int> group;
  if (p.R == 0) return v;
  for (int h = 0; h < h_end; ++h) {
    if (!runs(mine, h)) continue;
    const int a = p.off[h], e = p.off[h + 1];
    for (int r0 = e - p.R; r0 < e; r0 += 256) {
      const int rows = std::min(256, e - r0);
      for (int c = 0; c < p.hq; ++c) {
        AttnItem it = blank_item(r0, rows, c, spava::make_out(spava::kOutLseOnly));
        it.seg[0] = AttnSeg{a, r0 + rows - a, spava::kSegCausal, 0};
        v.push_back(it);
        group.push_back(h);
      }
    }
  }
  sort_host_major(v, group, p.hq / p.hkv);
  return v;
}

std::vector<AttnItem> build_dense_items(const spava_plan& p) {
  std::vector<AttnItem> v;
  const int NT = p.N + p.T;
  for (int r0 = 0; r0 < NT; r0 += 256) {
    const int rows = std::min(256, NT - r0);
    for (int c = 0; c < p.hq; ++c) {
      AttnItem it = blank_item(r0, rows, c, spava::make_out(spava::kOutFinal));
      it.seg[0] = AttnSeg{0, r0 + rows, spava::kSegCausal, 0};
      v.push_back(it);
    }
  }
  sort_by_cost(v);
  return v;
}

std::vector<int4> build_score_items(const spava_plan& p, int h_end, const HostMask* mine = nullptr) {
  std::vector<int4> v;
  for (int h = 0; h < h_end; ++h)
    if (runs(mine, h))
      for (int g = 0; g < p.hkv; ++g)
        for (int k0 = p.off[h]; k0 < p.off[h + 1]; k0 += 128) v.push_back(make_int4(h, g, k0, p.off[h + 1]));
  return v;
}

// Score tiles `v` (unit order) dealt to `grid` CTAs in rounds, for the fused
// score/select/gather launch: CTA b takes n / grid tiles (+-1) in `rounds` near-equal
// chunks, and round r hands every CTA, in CTA order, its r-th chunk from the next
// stretch of the list.  A unit is then complete once the round holding its last tile
// is scored everywhere, so units complete round after round instead of all at the
// end.  Rounds: about one per ten tiles of a CTA (a new chunk usually reloads the
// probe queries), at most 8.
void deal_rounds(const std::vector<int4>& v, int grid, std::vector<int4>* out, std::vector<int>* first) {
  const int n = static_cast<int>(v.size());
  const int per = ceil_div(n, grid);
  const int rounds = std::max(1, std::min(8, (per + 5) / 10));
  std::vector<int> tot(grid);
  first->assign(grid + 1, 0);
  for (int b = 0; b < grid; ++b) {
    tot[b] = static_cast<int>(static_cast<long long>(n) * (b + 1) / grid - static_cast<long long>(n) * b / grid);
    (*first)[b + 1] = (*first)[b] + tot[b];
  }
  out->assign(v.size(), make_int4(0, 0, 0, 0));
  std::vector<int> placed(grid, 0);
  int pos = 0;
  for (int r = 0; r < rounds; ++r)
    for (int b = 0; b < grid; ++b) {
      const int sz = tot[b] * (r + 1) / rounds - tot[b] * r / rounds;
      for (int k = 0; k < sz; ++k) (*out)[(*first)[b] + placed[b]++] = v[pos++];
    }
}

template <class K>
spava_status ensure_smem(K kernel, int bytes) {
  SPAVA_CUDA(cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes));
  return SPAVA_OK;
}

unsigned int* err_word(const spava_plan* p, void* ws) {
  return reinterpret_cast<unsigned int*>(static_cast<uint8_t*>(ws) + p->ws_err);
}

// Rows of scores, selections and passing buffers: one per KV head, or one per query
// head with per-query-head selection.
int score_rows(const spava_plan& p) { return p.score_reduce == SPAVA_SCORE_PER_QUERY_HEAD ? p.hq : p.hkv; }

// Byte offsets of the workspace (sized by the plan and by the selection rows).
void layout_workspace(spava_plan* p) {
  const size_t n_visual = static_cast<size_t>(p->N), n_text = static_cast<size_t>(p->T);
  const size_t hq = static_cast<size_t>(p->hq), d = static_cast<size_t>(p->d), P = static_cast<size_t>(p->P);
  const size_t rows = static_cast<size_t>(score_rows(*p));
  const size_t hm1 = p->H > 1 ? static_cast<size_t>(p->H - 1) : 0;
  size_t o = 0;
  p->ws_err = o;
  o += 256;
  p->ws_sync = o;  // fused score/select/gather: unit counters and ready flags
  o = align_up(o + 2 * hm1 * rows * 4, 256);
  p->ws_scores = o;
  o = align_up(o + rows * n_visual * 4, 256);
  p->ws_idx = o;
  o = align_up(o + hm1 * rows * P * 4, 256);
  p->ws_kp = o;
  o = align_up(o + hm1 * rows * P * d * 2, 256);
  p->ws_vp = o;
  o = align_up(o + hm1 * rows * P * d * 2, 256);
  p->ws_probe_lse = o;
  if (p->score_kind == SPAVA_SCORE_PROB) o = align_up(o + hq * n_visual * 4, 256);
  p->ws_opart = o;
  o = align_up(o + static_cast<size_t>(p->H + 1) * n_text * hq * d * 4, 256);
  p->ws_lpart = o;
  o = align_up(o + static_cast<size_t>(p->H + 1) * hq * n_text * 4, 256);
  p->ws_total = o;
  p->ws_row_o = o;
  o = align_up(o + n_visual * hq * d * 4, 256);
  p->ws_row_lse = o;
  o = align_up(o + hq * n_visual * 4, 256);
  p->ws_qkeys = o;  // per-query-head score keys (all but the max head reduction)
  o = align_up(o + hq * n_visual * 4, 256);
  p->ws_total_two_stage = o;
  // Sharded prefill: rank-major exchange buffers, each rank's part one contiguous run.
  const size_t world = static_cast<size_t>(p->shard_world);
  p->ws_xk = o;
  o = align_up(o + world * p->pass_slots * P * rows * d * 2, 256);
  p->ws_xv = o;
  o = align_up(o + world * p->pass_slots * P * rows * d * 2, 256);
  p->ws_to = o;
  o = align_up(o + world * p->text_slots * n_text * hq * d * 4, 256);
  p->ws_tl = o;
  o = align_up(o + world * p->text_slots * hq * n_text * 4, 256);
  p->ws_total_shard = o;
}

spava_status check_plan_ws(const spava_plan* p, void* ws) {
  if (!p) return fail(SPAVA_ERR_INVALID_ARG, "plan is NULL");
  if (!ws) return fail(SPAVA_ERR_INVALID_ARG, "workspace is NULL");
  if (reinterpret_cast<uintptr_t>(ws) & 255u) return fail(SPAVA_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
  return SPAVA_OK;
}

// ------------------------------------------------------------------ launches
template <int D>
spava_status launch_score(const spava_plan* p, const void* q, const void* k, float* scores, const int4* items,
                          int n_items, void* ws, cudaStream_t st) {
  if (n_items == 0) return SPAVA_OK;
  CUtensorMap tmK, tmQp;
  spava_status s;
  if ((s = make_map(&tmK, k, D, p->hkv, p->N + p->T, 1, 128)) != SPAVA_OK) return s;
  const int G = p->hq / p->hkv;
  if ((s = make_map(&tmQp, q, D, p->hq, p->N + p->T, 1, p->rc)) != SPAVA_OK) return s;
  ScoreParams sp;
  sp.items = items;
  sp.n_items = n_items;
  sp.probe_r = p->R;
  sp.group = G;
  sp.chunk_tokens = p->rc;
  sp.n_chunks = p->n_chunks;
  sp.head_reduce = p->score_reduce;
  sp.probe_lse = p->score_kind == SPAVA_SCORE_PROB
                     ? reinterpret_cast<const float*>(static_cast<const uint8_t*>(ws) + p->ws_probe_lse)
                     : nullptr;
  sp.lse_stride = p->N;
  sp.n_visual = p->N;
  sp.scale = p->scale;
  sp.scores = scores;
  sp.err_word = err_word(p, ws);
  sp.wait_limit_ns = p->wait_limit_ns;
  using S = spava::ScoreShape<D>;
  // Probe-query buffers: one when every (host, group) is a single chunk (it stays
  // resident across that group's key tiles), two otherwise; the rest of shared
  // memory holds K-tile stages.
  sp.q_bufs = p->n_chunks == 1 ? 1 : 2;
  sp.q_buf_bytes = (D / 64) * p->rc * G * 128;
  sp.k_stages = std::min<int>(S::kMaxStages, (S::kSmemMax - S::smem_bytes(sp.q_bufs, sp.q_buf_bytes, 0)) / S::kKTileBytes);
  if (sp.k_stages < 2) return fail(SPAVA_ERR_UNSUPPORTED, "probe queries too large for shared memory");
  const int smem = S::smem_bytes(sp.q_bufs, sp.q_buf_bytes, sp.k_stages);
  if ((s = ensure_smem(spava::score_kernel<D>, S::kSmemMax)) != SPAVA_OK) return s;
  int grid = std::min(n_items, p->num_sms);
  // every CTA's item range must fit the kernel's shared-memory item cache
  grid = std::max(grid, (n_items + S::kMaxLocalItems - 1) / S::kMaxLocalItems);
  mark(p, kLabScore, st);
  spava::score_kernel<D><<<grid, 256, smem, st>>>(tmK, tmQp, sp);
  SPAVA_CUDA(cudaGetLastError());
  ++g_last_launches;
  return SPAVA_OK;
}

// Where a fused selection writes its passing rows: k_pass/v_pass[g][h][j] (one GPU),
// or this rank's part of the rank-major exchange buffers [slot][j][g] (sharded).
struct PassDest {
  void* kp = nullptr;
  void* vp = nullptr;
  bool exchange = false;
};

// Top-P selection of hosts 0..H-2, or of the hosts in `hosts` (device list of
// n_hosts); with k/v and a destination given, each selection CTA also gathers its
// passing rows (the prefill's fused select + gather).
spava_status launch_select(const spava_plan* p, const float* scores, int32_t* idx, cudaStream_t st,
                           const void* k = nullptr, const void* v = nullptr, PassDest dst = PassDest(),
                           const int* hosts = nullptr, int n_hosts = -1) {
  if (p->H < 2 || p->P == 0) return SPAVA_OK;
  if (n_hosts < 0) n_hosts = p->H - 1;
  if (n_hosts == 0) return SPAVA_OK;
  int max_seg = 0;
  for (int h = 0; h + 1 < p->H; ++h) max_seg = std::max(max_seg, p->off[h + 1] - p->off[h]);
  const int rows = score_rows(*p);
  const size_t cpr = static_cast<size_t>(p->d) * 2 / 16;
  spava::GatherArgs ga{static_cast<const uint4*>(k), static_cast<const uint4*>(v), static_cast<uint4*>(dst.kp),
                       static_cast<uint4*>(dst.vp), static_cast<int>(cpr), p->hkv, rows / p->hkv, 0, 0, 0};
  if (dst.exchange) {
    ga.dst_g = cpr;
    ga.dst_j = rows * cpr;
    ga.dst_h = static_cast<size_t>(p->P) * ga.dst_j;
  } else {
    ga.dst_j = cpr;
    ga.dst_h = static_cast<size_t>(p->P) * cpr;
    ga.dst_g = static_cast<size_t>(p->H - 1) * ga.dst_h;
  }
  const bool fused = k != nullptr;
  const int grid = n_hosts * rows;
  mark(p, fused ? kLabSelectGather : kLabSelect, st);
  if (max_seg <= 16 * 1024) {
    if (fused)
      spava::select_topp_kernel<16, true><<<grid, 1024, 0, st>>>(scores, p->N, p->d_off, p->A, p->P, rows, hosts,
                                                                  idx, ga);
    else
      spava::select_topp_kernel<16, false><<<grid, 1024, 0, st>>>(scores, p->N, p->d_off, p->A, p->P, rows, hosts,
                                                                   idx, ga);
  } else {
    if (fused)
      spava::select_topp_kernel<0, true><<<grid, 1024, 0, st>>>(scores, p->N, p->d_off, p->A, p->P, rows, hosts,
                                                                 idx, ga);
    else
      spava::select_topp_kernel<0, false><<<grid, 1024, 0, st>>>(scores, p->N, p->d_off, p->A, p->P, rows, hosts,
                                                                  idx, ga);
  }
  SPAVA_CUDA(cudaGetLastError());
  ++g_last_launches;
  return SPAVA_OK;
}

// Grid of the fused score/select/gather launch (ssg_kernel.cuh) for this plan, or 0
// when the plan is outside what that kernel covers (another head reduction or score
// kind, the fused path switched off, more score tiles per CTA than it caches, or a
// grid that cannot be resident at once); the prefill then takes the score kernel and
// the select+gather kernel.  Sets *smem_out and *task_rows_out.
template <int D>
int ssg_grid(const spava_plan* p, int* smem_out, int* k_stages_out, int* task_rows_out) {
  using S = spava::SsgShape<D>;
  if (!p->fused_select || p->score_reduce != SPAVA_SCORE_MAX || p->score_kind != SPAVA_SCORE_LOGIT) return 0;
  if (p->H < 2 || p->P == 0 || p->n_score_pre == 0) return 0;
  const int grid = p->ssg_grid;
  if (grid <= 0 || p->ssg_max_local > S::kMaxLocalItems) return 0;
  const int G = p->hq / p->hkv;
  const int q_bufs = p->n_chunks == 1 ? 1 : 2, q_buf_bytes = (D / 64) * p->rc * G * 128;
  const int k_stages =
      std::min<int>(S::kMaxStages, (S::kSmemMax - S::smem_bytes(q_bufs, q_buf_bytes, 0)) / S::kKTileBytes);
  if (k_stages < 2) return 0;
  const int smem = S::smem_bytes(q_bufs, q_buf_bytes, k_stages);
  if (ensure_smem(spava::ssg_kernel<D>, S::kSmemMax) != SPAVA_OK) return 0;
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, spava::ssg_kernel<D>, S::kThreads, smem) != cudaSuccess)
    return 0;
  if (per_sm < 1 || grid > per_sm * p->num_sms) return 0;
  // gather tasks: at most kMaxOwnTasks per CTA (one unit per task the coarsest split)
  const int n_units = (p->H - 1) * p->hkv;
  int task_rows = 128;
  while (static_cast<long long>(n_units) * ceil_div(p->P, task_rows) > static_cast<long long>(S::kMaxOwnTasks) * grid) {
    if (task_rows >= p->P) return 0;
    task_rows *= 2;
  }
  *smem_out = smem;
  *k_stages_out = k_stages;
  *task_rows_out = task_rows;
  return grid;
}

// Scores, selection and passing K/V of hosts 0..H-2 in one cooperative launch.  The
// unit counters and ready flags (workspace, ws_sync) must be zero: begin_call clears
// them.  `grid`, `smem`, `k_stages` and `task_rows` come from ssg_grid.
template <int D>
spava_status launch_ssg(const spava_plan* p, int grid, int smem, int k_stages, int task_rows, const void* q,
                        const void* k, const void* v, float* scores, int32_t* idx, void* kp, void* vp, void* ws,
                        cudaStream_t st) {
  using S = spava::SsgShape<D>;
  CUtensorMap tmK, tmQp;
  spava_status s;
  if ((s = make_map(&tmK, k, D, p->hkv, p->N + p->T, 1, 128)) != SPAVA_OK) return s;
  if ((s = make_map(&tmQp, q, D, p->hq, p->N + p->T, 1, p->rc)) != SPAVA_OK) return s;
  const int G = p->hq / p->hkv;
  const int n_units = (p->H - 1) * p->hkv;
  const size_t cpr = static_cast<size_t>(D) * 2 / 16;
  spava::SsgParams sp{};
  sp.items = p->d_ssg_items;
  sp.cta_first = p->d_ssg_first;
  sp.probe_r = p->R;
  sp.group = G;
  sp.chunk_tokens = p->rc;
  sp.n_chunks = p->n_chunks;
  sp.n_visual = p->N;
  sp.scale = p->scale;
  sp.scores = scores;
  sp.q_bufs = p->n_chunks == 1 ? 1 : 2;
  sp.q_buf_bytes = (D / 64) * p->rc * G * 128;
  sp.k_stages = k_stages;
  sp.off = p->d_off;
  sp.hkv = p->hkv;
  sp.anchor = p->A;
  sp.passing = p->P;
  sp.unit_cnt = reinterpret_cast<int*>(static_cast<uint8_t*>(ws) + p->ws_sync);
  sp.unit_ready = sp.unit_cnt + n_units;
  sp.idx = idx;
  sp.k = static_cast<const uint4*>(k);
  sp.v = static_cast<const uint4*>(v);
  sp.kp = static_cast<uint4*>(kp);
  sp.vp = static_cast<uint4*>(vp);
  sp.chunks_per_row = static_cast<int>(cpr);
  sp.dst_h = static_cast<size_t>(p->P) * cpr;
  sp.dst_g = static_cast<size_t>(p->H - 1) * sp.dst_h;
  sp.task_rows = task_rows;
  sp.tasks_per_unit = ceil_div(p->P, task_rows);
  sp.n_tasks = n_units * sp.tasks_per_unit;
  sp.err_word = err_word(p, ws);
  sp.wait_limit_ns = p->wait_limit_ns;
  sp.stall_producer = p->stall_producer;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(S::kThreads);
  cfg.dynamicSmemBytes = static_cast<size_t>(smem);
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  mark(p, kLabScoreSelectGather, st);
  SPAVA_CUDA(cudaLaunchKernelEx(&cfg, spava::ssg_kernel<D>, tmK, tmQp, sp));
  ++g_last_launches;
  return SPAVA_OK;
}

spava_status launch_gather(const spava_plan* p, const void* k, const void* v, const int32_t* idx, void* kp, void* vp,
                           cudaStream_t st) {
  if (p->H < 2 || p->P == 0) return SPAVA_OK;
  const int chunks = p->d * 2 / 16;
  const int rows = score_rows(*p);
  const size_t total = static_cast<size_t>(rows) * (p->H - 1) * p->P * chunks;
  const int grid = static_cast<int>(std::min<size_t>((total + 255) / 256, static_cast<size_t>(p->num_sms) * 8));
  mark(p, kLabGather, st);
  spava::gather_passing_kernel<<<grid, 256, 0, st>>>(static_cast<const uint4*>(k), static_cast<const uint4*>(v), idx,
                                                      static_cast<uint4*>(kp), static_cast<uint4*>(vp), rows, p->hkv,
                                                      rows / p->hkv, p->H - 1, p->P, chunks);
  SPAVA_CUDA(cudaGetLastError());
  ++g_last_launches;
  return SPAVA_OK;
}

// Buffers only the two-stage flow uses (row partials and probe-score keys).
struct TwoStageBufs {
  float* row_o = nullptr;
  float* row_lse = nullptr;
  unsigned int* score_keys = nullptr;
  int per_qhead = 0;  // score_keys has one row per query head
  float* text_o = nullptr;    // text partial slots elsewhere than the workspace's
  float* text_lse = nullptr;  // (the sharded prefill's exchange buffers)
};

template <int D>
spava_status launch_attn(const spava_plan* p, const AttnItem* items, int n_items, const void* q, const void* k,
                         const void* v, const void* kp, const void* vp, void* o, float* lse, void* ws,
                         cudaStream_t st, const TwoStageBufs& ts = TwoStageBufs()) {
  if (n_items == 0) return SPAVA_OK;
  CUtensorMap tmQ, tmK, tmV, tmKp, tmVp;
  spava_status s;
  const uint64_t NT = static_cast<uint64_t>(p->N) + p->T;
  if ((s = make_map(&tmQ, q, D, p->hq, NT, 1, 128)) != SPAVA_OK) return s;
  if ((s = make_map(&tmK, k, D, p->hkv, NT, 1, 128)) != SPAVA_OK) return s;
  if ((s = make_map(&tmV, v, D, p->hkv, NT, 1, 128)) != SPAVA_OK) return s;
  if (p->H >= 2 && p->P > 0 && kp && vp) {
    const uint64_t rows = static_cast<uint64_t>(p->H - 1) * p->P;
    if ((s = make_map(&tmKp, kp, D, rows, score_rows(*p), 128, 1)) != SPAVA_OK) return s;
    if ((s = make_map(&tmVp, vp, D, rows, score_rows(*p), 128, 1)) != SPAVA_OK) return s;
  } else {
    tmKp = tmK;  // never read: no item has a passing segment
    tmVp = tmV;
  }
  AttnParams ap;
  ap.items = items;
  ap.n_items = n_items;
  ap.group = p->hq / p->hkv;
  ap.pass_per_qhead = p->score_reduce == SPAVA_SCORE_PER_QUERY_HEAD;
  ap.hq = p->hq;
  ap.n_rows_out = p->N + p->T;
  ap.o = static_cast<__nv_bfloat16*>(o);
  ap.lse = lse;
  uint8_t* w = static_cast<uint8_t*>(ws);
  ap.o_part = ts.text_o ? ts.text_o : reinterpret_cast<float*>(w + p->ws_opart);
  ap.lse_part = ts.text_lse ? ts.text_lse : reinterpret_cast<float*>(w + p->ws_lpart);
  ap.part_row0 = p->N;
  ap.part_rows = p->T;
  ap.scale_log2 = p->scale * 1.4426950408889634f;
  ap.err_word = err_word(p, ws);
  ap.wait_limit_ns = p->wait_limit_ns;
  ap.stall_producer = p->stall_producer;
  ap.row_o = ts.row_o;
  ap.row_lse = ts.row_lse;
  ap.score_keys = ts.score_keys;
  ap.score_per_qhead = ts.per_qhead;
  ap.n_visual = p->N;
  ap.probe_r = p->R;
  ap.scale = p->scale;
  using S = spava::AttnShape<D>;
  if ((s = ensure_smem(spava::attn_fwd_kernel<D>, S::kSmemBytes)) != SPAVA_OK) return s;
  const int grid = std::min(n_items, p->num_sms);
  mark(p, items == p->d_items_dense ? kLabDense
             : (items == p->d_items_local || items == p->d_items_shard_local) ? kLabAttnLocal
             : (items == p->d_items_remote || items == p->d_items_shard_remote) ? kLabAttnRemote
             : (items == p->d_items_probe || items == p->d_items_shard_probe) ? kLabProbeLse : kLabAttn, st);
  spava::attn_fwd_kernel<D><<<grid, S::kThreads, S::kSmemBytes, st>>>(tmQ, tmK, tmV, tmKp, tmVp, ap);
  SPAVA_CUDA(cudaGetLastError());
  ++g_last_launches;
  return SPAVA_OK;
}

// Probability scores: the lse of every host's probe rows over its block, into the
// workspace (the items' O is not stored; V only has to be a readable K/V tensor).
spava_status launch_probe_lse(const spava_plan* p, const void* q, const void* k, const void* v, void* ws,
                              cudaStream_t st, const AttnItem* items = nullptr, int n_items = -1) {
  if (p->score_kind != SPAVA_SCORE_PROB) return SPAVA_OK;
  if (!items) {
    items = p->d_items_probe;
    n_items = p->n_items_probe;
  }
  TwoStageBufs t;
  t.row_lse = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + p->ws_probe_lse);
  return p->d == 128 ? launch_attn<128>(p, items, n_items, q, k, v, nullptr, nullptr, nullptr, nullptr, ws, st, t)
                     : launch_attn<64>(p, items, n_items, q, k, v, nullptr, nullptr, nullptr, nullptr, ws, st, t);
}

// Text rows from n_slots partial slots (the workspace's H+1, or the sharded prefill's
// gathered world * slots-per-rank).
spava_status launch_merge(const spava_plan* p, void* o, float* lse, void* ws, cudaStream_t st,
                          const float* o_part = nullptr, const float* lse_part = nullptr, int n_slots = -1) {
  if (p->T == 0) return SPAVA_OK;
  uint8_t* w = static_cast<uint8_t*>(ws);
  if (!o_part) {
    o_part = reinterpret_cast<const float*>(w + p->ws_opart);
    lse_part = reinterpret_cast<const float*>(w + p->ws_lpart);
    n_slots = p->H + 1;
  }
  const int warps = p->T * p->hq;
  const int grid = (warps * 32 + 255) / 256;
  mark(p, kLabMerge, st);
  spava::lse_merge_kernel<<<grid, 256, 0, st>>>(o_part, lse_part, n_slots, p->T, p->hq, p->d, p->N, p->N + p->T,
                                                 static_cast<__nv_bfloat16*>(o), lse);
  SPAVA_CUDA(cudaGetLastError());
  ++g_last_launches;
  return SPAVA_OK;
}

spava_status begin_call(const spava_plan* p, void* ws, cudaStream_t st, bool clear_error = true) {
  g_last_launches = 0;
  ++p->prof_call_id;
  int dev = -1;
  SPAVA_CUDA(cudaGetDevice(&dev));
  if (dev != p->device) return fail(SPAVA_ERR_INVALID_ARG, "current device %d differs from the plan's device %d", dev, p->device);
  // the error word and the fused launch's counters, which must start at zero
  if (clear_error) SPAVA_CUDA(cudaMemsetAsync(err_word(p, ws), 0, p->ws_scores - p->ws_err, st));
  return SPAVA_OK;
}

// Upload `host` (built with the same put() packing as the plan table) to a fresh
// device allocation.
spava_status upload_table(const std::vector<uint8_t>& host, void** out) {
  *out = nullptr;
  if (host.empty()) return SPAVA_OK;
  cudaError_t e = cudaMalloc(out, host.size());
  if (e != cudaSuccess) return fail(SPAVA_ERR_CUDA, "cudaMalloc(plan table): %s", cudaGetErrorString(e));
  e = cudaMemcpy(*out, host.data(), host.size(), cudaMemcpyHostToDevice);
  if (e != cudaSuccess) {
    cudaFree(*out);
    *out = nullptr;
    return fail(SPAVA_ERR_CUDA, "cudaMemcpy(plan table): %s", cudaGetErrorString(e));
  }
  return SPAVA_OK;
}

// Packs arrays into one host image for upload_table, each 256-byte aligned.  An
// empty array still takes a slot, so no two arrays share an address (the kernel
// timing labels tell work lists apart by address).
struct TablePacker {
  std::vector<uint8_t> host;
  size_t put(const void* src, size_t bytes) {
    const size_t at = host.size();
    const uint8_t* b = static_cast<const uint8_t*>(src);
    if (bytes) host.insert(host.end(), b, b + bytes);
    host.resize(align_up(at + std::max<size_t>(bytes, 1), 256), 0);
    return at;
  }
};

}  // namespace

// =================================================================== C ABI
extern "C" {

const char* spava_status_string(spava_status s) {
  switch (s) {
    case SPAVA_OK: return "SPAVA_OK";
    case SPAVA_ERR_INVALID_ARG: return "SPAVA_ERR_INVALID_ARG";
    case SPAVA_ERR_UNSUPPORTED: return "SPAVA_ERR_UNSUPPORTED";
    case SPAVA_ERR_CUDA: return "SPAVA_ERR_CUDA";
    case SPAVA_ERR_TIMEOUT: return "SPAVA_ERR_TIMEOUT";
    case SPAVA_ERR_DEVICE_CHECK: return "SPAVA_ERR_DEVICE_CHECK";
  }
  return "SPAVA_ERR_UNKNOWN";
}

const char* spava_last_error(void) { return g_last_error.c_str(); }

int32_t spava_last_launch_count(void) { return g_last_launches; }

spava_status spava_plan_create(spava_plan** out, int32_t n_visual, int32_t n_text, int32_t n_hosts,
                               const int32_t* host_sizes, int32_t anchor, int32_t passing, int32_t probe_r,
                               int32_t hq, int32_t hkv, int32_t head_dim, float softmax_scale) {
  if (!out) return fail(SPAVA_ERR_INVALID_ARG, "out is NULL");
  *out = nullptr;
  if (n_visual < 1 || n_text < 0 || n_hosts < 1) return fail(SPAVA_ERR_INVALID_ARG, "need N >= 1, T >= 0, H >= 1");
  if (n_hosts > n_visual) return fail(SPAVA_ERR_INVALID_ARG, "more hosts than visual tokens");
  if (hq < 1 || hkv < 1 || hq % hkv) return fail(SPAVA_ERR_INVALID_ARG, "hq must be a positive multiple of hkv");
  if (hq / hkv > 16) return fail(SPAVA_ERR_UNSUPPORTED, "query heads per KV head must be <= 16");
  if (head_dim != 64 && head_dim != 128) return fail(SPAVA_ERR_UNSUPPORTED, "head_dim must be 64 or 128");
  if (anchor < 0 || passing < 0 || probe_r < 0) return fail(SPAVA_ERR_INVALID_ARG, "negative A, P or R");
  if (static_cast<int64_t>(n_visual) + n_text > (1ll << 30))
    return fail(SPAVA_ERR_UNSUPPORTED, "more than 2^30 tokens");
  std::vector<int> off(n_hosts + 1, 0);
  if (host_sizes) {
    int64_t sum = 0;
    for (int h = 0; h < n_hosts; ++h) {
      if (host_sizes[h] < 1) return fail(SPAVA_ERR_INVALID_ARG, "host %d has size %d", h, host_sizes[h]);
      sum += host_sizes[h];
      off[h + 1] = static_cast<int>(sum);
    }
    if (sum != n_visual) return fail(SPAVA_ERR_INVALID_ARG, "host sizes sum to %lld, not N=%d", (long long)sum, n_visual);
  } else {
    if (n_visual % n_hosts) return fail(SPAVA_ERR_INVALID_ARG, "equal split needs N %% H == 0");
    for (int h = 0; h < n_hosts; ++h) off[h + 1] = off[h] + n_visual / n_hosts;
  }
  int min_b = n_visual;
  for (int h = 0; h < n_hosts; ++h) min_b = std::min(min_b, off[h + 1] - off[h]);
  if (n_hosts > 1) {
    if (probe_r < 1 || probe_r > min_b) return fail(SPAVA_ERR_INVALID_ARG, "need 1 <= R <= min block size (%d)", min_b);
    if (probe_r % 16) return fail(SPAVA_ERR_UNSUPPORTED, "R must be a multiple of 16");
    if (anchor + passing > off[1]) return fail(SPAVA_ERR_INVALID_ARG, "host 0 needs A + P <= B_0");
    for (int h = 1; h < n_hosts - 1; ++h)
      if (passing > off[h + 1] - off[h]) return fail(SPAVA_ERR_INVALID_ARG, "P exceeds block %d", h);
  }
  if (anchor > n_visual) return fail(SPAVA_ERR_INVALID_ARG, "A > N");

  spava_plan* p = new spava_plan();
  p->N = n_visual;
  p->T = n_text;
  p->H = n_hosts;
  p->A = anchor;
  p->P = passing;
  p->R = probe_r;
  p->hq = hq;
  p->hkv = hkv;
  p->d = head_dim;
  p->scale = softmax_scale > 0.f ? softmax_scale : 1.0f / std::sqrt(static_cast<float>(head_dim));
  p->off = off;
  const int G = hq / hkv;
  p->rc = std::max(16, 16 * (256 / (16 * G)));
  if (probe_r > 0) p->rc = std::min(p->rc, probe_r);
  p->n_chunks = probe_r > 0 ? ceil_div(probe_r, p->rc) : 0;

  layout_workspace(p);

  // device
  auto bail = [&](spava_status s) {
    if (p->dtab) cudaFree(p->dtab);
    delete p;
    return s;
  };
  cudaError_t e = cudaGetDevice(&p->device);
  if (e != cudaSuccess) return bail(fail(SPAVA_ERR_CUDA, "no CUDA device: %s", cudaGetErrorString(e)));
  cudaDeviceProp prop;
  e = cudaGetDeviceProperties(&prop, p->device);
  if (e != cudaSuccess) return bail(fail(SPAVA_ERR_CUDA, "cudaGetDeviceProperties: %s", cudaGetErrorString(e)));
  if (prop.major != 10 || prop.minor != 0)
    return bail(fail(SPAVA_ERR_UNSUPPORTED, "needs an sm_100 (B200) device, found sm_%d%d", prop.major, prop.minor));
  p->num_sms = prop.multiProcessorCount;

  const auto pre = build_prefill_items(*p);
  const auto dense = build_dense_items(*p);
  const auto local = build_local_items(*p);
  const auto remote = build_remote_items(*p);
  const auto probe = build_probe_items(*p, n_hosts);
  const auto sc_pre = build_score_items(*p, n_hosts - 1);
  const auto sc_all = build_score_items(*p, n_hosts);
  p->n_items_pre = static_cast<int>(pre.size());
  p->n_items_dense = static_cast<int>(dense.size());
  p->n_items_local = static_cast<int>(local.size());
  p->n_items_remote = static_cast<int>(remote.size());
  p->n_items_probe = static_cast<int>(probe.size());
  p->n_score_pre = static_cast<int>(sc_pre.size());
  p->n_score_all = static_cast<int>(sc_all.size());
  std::vector<int4> ssg_items;
  std::vector<int> ssg_first;
  p->ssg_grid = std::min(p->n_score_pre, p->num_sms);
  if (p->ssg_grid > 0) {
    deal_rounds(sc_pre, p->ssg_grid, &ssg_items, &ssg_first);
    for (int b = 0; b < p->ssg_grid; ++b) p->ssg_max_local = std::max(p->ssg_max_local, ssg_first[b + 1] - ssg_first[b]);
  }
  // One device table, each array 256-byte aligned.
  TablePacker tab;
  const size_t o_off = tab.put(off.data(), off.size() * 4);
  const size_t o_pre = tab.put(pre.data(), pre.size() * sizeof(AttnItem));
  const size_t o_dense = tab.put(dense.data(), dense.size() * sizeof(AttnItem));
  const size_t o_spre = tab.put(sc_pre.data(), sc_pre.size() * sizeof(int4));
  const size_t o_sall = tab.put(sc_all.data(), sc_all.size() * sizeof(int4));
  const size_t o_local = tab.put(local.data(), local.size() * sizeof(AttnItem));
  const size_t o_remote = tab.put(remote.data(), remote.size() * sizeof(AttnItem));
  const size_t o_probe = tab.put(probe.data(), probe.size() * sizeof(AttnItem));
  const size_t o_ssg_items = tab.put(ssg_items.data(), ssg_items.size() * sizeof(int4));
  const size_t o_ssg_first = tab.put(ssg_first.data(), ssg_first.size() * 4);
  spava_status ust = upload_table(tab.host, &p->dtab);
  if (ust != SPAVA_OK) return bail(ust);
  uint8_t* base = static_cast<uint8_t*>(p->dtab);
  p->d_off = reinterpret_cast<int*>(base + o_off);
  p->d_items_pre = reinterpret_cast<AttnItem*>(base + o_pre);
  p->d_items_dense = reinterpret_cast<AttnItem*>(base + o_dense);
  p->d_score_pre = reinterpret_cast<int4*>(base + o_spre);
  p->d_score_all = reinterpret_cast<int4*>(base + o_sall);
  p->d_items_local = reinterpret_cast<AttnItem*>(base + o_local);
  p->d_items_remote = reinterpret_cast<AttnItem*>(base + o_remote);
  p->d_items_probe = reinterpret_cast<AttnItem*>(base + o_probe);
  p->d_ssg_items = reinterpret_cast<int4*>(base + o_ssg_items);
  p->d_ssg_first = reinterpret_cast<int*>(base + o_ssg_first);
  *out = p;
  return ok();
}

spava_status spava_plan_destroy(spava_plan* p) {
  if (!p) return ok();
  spava_status s = SPAVA_OK;
  for (cudaEvent_t e : p->prof_ev) cudaEventDestroy(e);
  if (p->dtab || p->dtab_shard) {
    cudaError_t e = cudaDeviceSynchronize();
    if (e == cudaSuccess && p->dtab) e = cudaFree(p->dtab);
    if (e == cudaSuccess && p->dtab_shard) e = cudaFree(p->dtab_shard);
    if (e != cudaSuccess) s = fail(SPAVA_ERR_CUDA, "plan destroy: %s", cudaGetErrorString(e));
  }
  delete p;
  return s == SPAVA_OK ? ok() : s;
}

size_t spava_workspace_bytes(const spava_plan* p) { return p ? p->ws_total : 0; }

int32_t spava_plan_offsets(const spava_plan* p, int32_t* offsets_out) {
  if (!p) return -1;
  if (offsets_out)
    for (int h = 0; h <= p->H; ++h) offsets_out[h] = p->off[h];
  return p->H;
}

spava_status spava_plan_set_score_reduce(spava_plan* p, int32_t mode) {
  if (!p) return fail(SPAVA_ERR_INVALID_ARG, "plan is NULL");
  if (mode != SPAVA_SCORE_MAX && mode != SPAVA_SCORE_SUM && mode != SPAVA_SCORE_MEAN &&
      mode != SPAVA_SCORE_PER_QUERY_HEAD)
    return fail(SPAVA_ERR_INVALID_ARG, "unknown score reduction %d", mode);
  p->score_reduce = mode;
  layout_workspace(p);  // selection rows decide the sizes of scores, indices, passing K/V
  return ok();
}

spava_status spava_plan_set_score_kind(spava_plan* p, int32_t kind) {
  if (!p) return fail(SPAVA_ERR_INVALID_ARG, "plan is NULL");
  if (kind != SPAVA_SCORE_LOGIT && kind != SPAVA_SCORE_PROB)
    return fail(SPAVA_ERR_INVALID_ARG, "unknown score kind %d", kind);
  p->score_kind = kind;
  layout_workspace(p);  // probability scores keep the probe rows' lse in the workspace
  return ok();
}

spava_status spava_plan_set_fused_select(spava_plan* p, int32_t enable) {
  if (!p) return fail(SPAVA_ERR_INVALID_ARG, "plan is NULL");
  p->fused_select = enable ? 1 : 0;
  return ok();
}

spava_status spava_plan_set_debug(spava_plan* p, uint64_t wait_limit_ns, int32_t stall_producer) {
  if (!p) return fail(SPAVA_ERR_INVALID_ARG, "plan is NULL");
  p->wait_limit_ns = wait_limit_ns ? wait_limit_ns : spava::kDefaultWaitLimitNs;
  p->stall_producer = stall_producer ? 1 : 0;
  return ok();
}

spava_status spava_score_select(const spava_plan* p, const void* q, const void* k, float* scores, int32_t* idx,
                                uint32_t flags, void* ws, void* stream) {
  spava_status s;
  if ((s = check_plan_ws(p, ws)) != SPAVA_OK) return s;
  if (!scores || !idx) return fail(SPAVA_ERR_INVALID_ARG, "scores and idx must not be NULL");
  if (!(flags & SPAVA_SCORES_GIVEN) && (!q || !k)) return fail(SPAVA_ERR_INVALID_ARG, "q and k must not be NULL");
  if (!(flags & SPAVA_SCORES_GIVEN) && (!aligned16(q) || !aligned16(k)))
    return fail(SPAVA_ERR_INVALID_ARG, "q and k must be 16-byte aligned");
  if (flags & ~SPAVA_SCORES_GIVEN) return fail(SPAVA_ERR_INVALID_ARG, "unknown flags 0x%x", flags);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if ((s = begin_call(p, ws, st)) != SPAVA_OK) return s;
  if (!(flags & SPAVA_SCORES_GIVEN) && p->H >= 1) {
    if (p->R == 0) return fail(SPAVA_ERR_INVALID_ARG, "plan has R = 0: nothing to score");
    if ((s = launch_probe_lse(p, q, k, k, ws, st)) != SPAVA_OK) return s;
    s = p->d == 128 ? launch_score<128>(p, q, k, scores, p->d_score_all, p->n_score_all, ws, st)
                    : launch_score<64>(p, q, k, scores, p->d_score_all, p->n_score_all, ws, st);
    if (s != SPAVA_OK) return s;
  }
  if ((s = launch_select(p, scores, idx, st)) != SPAVA_OK) return s;
  mark(p, -1, st);
  return ok();
}

spava_status spava_gather_passing(const spava_plan* p, const void* k, const void* v, const int32_t* idx, void* k_pass,
                                  void* v_pass, void* stream) {
  if (!p) return fail(SPAVA_ERR_INVALID_ARG, "plan is NULL");
  if (!k || !v || !idx || !k_pass || !v_pass) return fail(SPAVA_ERR_INVALID_ARG, "NULL pointer");
  if (!aligned16(k) || !aligned16(v) || !aligned16(k_pass) || !aligned16(v_pass))
    return fail(SPAVA_ERR_INVALID_ARG, "k, v, k_pass, v_pass must be 16-byte aligned");
  g_last_launches = 0;
  ++p->prof_call_id;
  spava_status s = launch_gather(p, k, v, idx, k_pass, v_pass, static_cast<cudaStream_t>(stream));
  if (s != SPAVA_OK) return s;
  mark(p, -1, static_cast<cudaStream_t>(stream));
  return ok();
}

spava_status spava_attn_prefill(const spava_plan* p, const void* q, const void* k, const void* v, void* o, float* lse,
                                float* scores_out, int32_t* idx_out, void* ws, void* stream) {
  spava_status s;
  if ((s = check_plan_ws(p, ws)) != SPAVA_OK) return s;
  if (!q || !k || !v || !o || !lse) return fail(SPAVA_ERR_INVALID_ARG, "NULL tensor pointer");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o))
    return fail(SPAVA_ERR_INVALID_ARG, "q, k, v, o must be 16-byte aligned");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if ((s = begin_call(p, ws, st)) != SPAVA_OK) return s;
  uint8_t* w = static_cast<uint8_t*>(ws);
  float* scores = scores_out ? scores_out : reinterpret_cast<float*>(w + p->ws_scores);
  int32_t* idx = idx_out ? idx_out : reinterpret_cast<int32_t*>(w + p->ws_idx);
  void* kp = w + p->ws_kp;
  void* vp = w + p->ws_vp;
  if (p->H >= 2 && p->P > 0) {
    int smem = 0, k_stages = 0, task_rows = 0;
    const int grid = p->d == 128 ? ssg_grid<128>(p, &smem, &k_stages, &task_rows)
                                 : ssg_grid<64>(p, &smem, &k_stages, &task_rows);
    if (grid > 0) {
      s = p->d == 128 ? launch_ssg<128>(p, grid, smem, k_stages, task_rows, q, k, v, scores, idx, kp, vp, ws, st)
                      : launch_ssg<64>(p, grid, smem, k_stages, task_rows, q, k, v, scores, idx, kp, vp, ws, st);
      if (s != SPAVA_OK) return s;
    } else {
      if ((s = launch_probe_lse(p, q, k, v, ws, st)) != SPAVA_OK) return s;
      s = p->d == 128 ? launch_score<128>(p, q, k, scores, p->d_score_pre, p->n_score_pre, ws, st)
                      : launch_score<64>(p, q, k, scores, p->d_score_pre, p->n_score_pre, ws, st);
      if (s != SPAVA_OK) return s;
      if ((s = launch_select(p, scores, idx, st, k, v, PassDest{kp, vp, false})) != SPAVA_OK) return s;
    }
  }
  s = p->d == 128 ? launch_attn<128>(p, p->d_items_pre, p->n_items_pre, q, k, v, kp, vp, o, lse, ws, st)
                  : launch_attn<64>(p, p->d_items_pre, p->n_items_pre, q, k, v, kp, vp, o, lse, ws, st);
  if (s != SPAVA_OK) return s;
  if ((s = launch_merge(p, o, lse, ws, st)) != SPAVA_OK) return s;
  mark(p, -1, st);
  return ok();
}

}  // extern "C"

// Scratch of spava_attn_prefill_noalloc: one array per device holding the
// library's kernels, shared by every call on that device.
static __device__ __align__(256) unsigned char g_noalloc_scratch[SPAVA_NOALLOC_SCRATCH_BYTES];

namespace {

// Device address of g_noalloc_scratch on the current device.  In host code the
// symbol is only a host-side stand-in, so the address is looked up on every call:
// the lookup enqueues nothing, and a cached address would go stale if the device's
// context were torn down and re-created (cudaDeviceReset reloads the module, and the
// array may then sit elsewhere).
spava_status noalloc_scratch_address(void** out) {
  void* addr = nullptr;
  cudaError_t e = cudaGetSymbolAddress(&addr, g_noalloc_scratch);
  if (e != cudaSuccess || !addr)
    return fail(SPAVA_ERR_CUDA, "cudaGetSymbolAddress(static scratch): %s", cudaGetErrorString(e));
  *out = addr;
  return SPAVA_OK;
}

}  // namespace

extern "C" {

spava_status spava_attn_prefill_noalloc(const spava_plan* p, const void* q, const void* k, const void* v, void* o,
                                        float* lse, void* stream) {
  if (!p) return fail(SPAVA_ERR_INVALID_ARG, "plan is NULL");
  if (p->ws_total > SPAVA_NOALLOC_SCRATCH_BYTES)
    return fail(SPAVA_ERR_UNSUPPORTED,
                "this plan needs %zu bytes of scratch, the static scratch holds %u; "
                "use spava_attn_prefill with a workspace",
                p->ws_total, SPAVA_NOALLOC_SCRATCH_BYTES);
  int dev = -1;
  SPAVA_CUDA(cudaGetDevice(&dev));
  if (dev != p->device) return fail(SPAVA_ERR_INVALID_ARG, "current device %d differs from the plan's device %d", dev, p->device);
  void* ws = nullptr;
  spava_status s = noalloc_scratch_address(&ws);
  if (s != SPAVA_OK) return s;
  return spava_attn_prefill(p, q, k, v, o, lse, nullptr, nullptr, ws, stream);
}

size_t spava_two_stage_workspace_bytes(const spava_plan* p) { return p ? p->ws_total_two_stage : 0; }

spava_status spava_attn_prefill_two_stage(const spava_plan* p, const void* q, const void* k, const void* v, void* o,
                                          float* lse, float* scores_out, int32_t* idx_out, void* ws, void* stream) {
  spava_status s;
  if ((s = check_plan_ws(p, ws)) != SPAVA_OK) return s;
  if (!q || !k || !v || !o || !lse) return fail(SPAVA_ERR_INVALID_ARG, "NULL tensor pointer");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o))
    return fail(SPAVA_ERR_INVALID_ARG, "q, k, v, o must be 16-byte aligned");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if ((s = begin_call(p, ws, st)) != SPAVA_OK) return s;
  uint8_t* w = static_cast<uint8_t*>(ws);
  float* scores = scores_out ? scores_out : reinterpret_cast<float*>(w + p->ws_scores);
  int32_t* idx = idx_out ? idx_out : reinterpret_cast<int32_t*>(w + p->ws_idx);
  void* kp = w + p->ws_kp;
  void* vp = w + p->ws_vp;
  TwoStageBufs ts;
  ts.row_o = reinterpret_cast<float*>(w + p->ws_row_o);
  ts.row_lse = reinterpret_cast<float*>(w + p->ws_row_lse);
  // Max over heads: one key row per KV head, turned into scores in place.  Sum / mean:
  // one key row per query head, combined into the scores after the local pass.
  // Probability scores need each probe row's final lse: scored by the score kernel
  // instead of being folded into the local pass.
  const bool prob = p->score_kind == SPAVA_SCORE_PROB;
  ts.per_qhead = p->score_reduce != SPAVA_SCORE_MAX;
  ts.score_keys = prob ? nullptr
                  : ts.per_qhead ? reinterpret_cast<unsigned int*>(w + p->ws_qkeys)
                                 : reinterpret_cast<unsigned int*>(scores);
  const size_t n_keys = static_cast<size_t>(ts.per_qhead ? p->hq : p->hkv) * p->N;
  const int grid_small = std::max(1, std::min(p->num_sms * 4, static_cast<int>((n_keys + 255) / 256)));
  if (scores_needed(*p) && prob) {
    if ((s = launch_probe_lse(p, q, k, v, ws, st)) != SPAVA_OK) return s;
    s = p->d == 128 ? launch_score<128>(p, q, k, scores, p->d_score_pre, p->n_score_pre, ws, st)
                    : launch_score<64>(p, q, k, scores, p->d_score_pre, p->n_score_pre, ws, st);
    if (s != SPAVA_OK) return s;
  } else if (scores_needed(*p)) {
    mark(p, kLabFill, st);
    spava::fill_u32_kernel<<<grid_small, 256, 0, st>>>(ts.score_keys, n_keys, spava::kOrderedNegInf);
    SPAVA_CUDA(cudaGetLastError());
    ++g_last_launches;
  }
  // stage 1: local causal pass (+ fused probe scores, + text pieces)
  s = p->d == 128 ? launch_attn<128>(p, p->d_items_local, p->n_items_local, q, k, v, nullptr, nullptr, o, lse, ws, st, ts)
                  : launch_attn<64>(p, p->d_items_local, p->n_items_local, q, k, v, nullptr, nullptr, o, lse, ws, st, ts);
  if (s != SPAVA_OK) return s;
  if (scores_needed(*p)) {
    if (!prob) {
      mark(p, kLabFill, st);
      if (p->score_reduce == SPAVA_SCORE_PER_QUERY_HEAD)  // one score row per query head: convert
        spava::combine_head_keys_kernel<<<grid_small, 256, 0, st>>>(ts.score_keys, scores, p->hq, 1,
                                                                     static_cast<size_t>(p->N), SPAVA_SCORE_SUM);
      else if (ts.per_qhead)
        spava::combine_head_keys_kernel<<<grid_small, 256, 0, st>>>(ts.score_keys, scores, p->hkv, p->hq / p->hkv,
                                                                     static_cast<size_t>(p->N), p->score_reduce);
      else
        spava::keys_to_scores_kernel<<<grid_small, 256, 0, st>>>(ts.score_keys, n_keys);
      SPAVA_CUDA(cudaGetLastError());
      ++g_last_launches;
    }
    if ((s = launch_select(p, scores, idx, st, k, v, PassDest{kp, vp, false})) != SPAVA_OK) return s;
  }
  // stage 2: remote pass over [anchor | passing], lse-merged with the local partials
  s = p->d == 128 ? launch_attn<128>(p, p->d_items_remote, p->n_items_remote, q, k, v, kp, vp, o, lse, ws, st, ts)
                  : launch_attn<64>(p, p->d_items_remote, p->n_items_remote, q, k, v, kp, vp, o, lse, ws, st, ts);
  if (s != SPAVA_OK) return s;
  if ((s = launch_merge(p, o, lse, ws, st)) != SPAVA_OK) return s;
  mark(p, -1, st);
  return ok();
}

spava_status spava_dense_causal(const spava_plan* p, const void* q, const void* k, const void* v, void* o, float* lse,
                                void* ws, void* stream) {
  spava_status s;
  if ((s = check_plan_ws(p, ws)) != SPAVA_OK) return s;
  if (!q || !k || !v || !o || !lse) return fail(SPAVA_ERR_INVALID_ARG, "NULL tensor pointer");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o))
    return fail(SPAVA_ERR_INVALID_ARG, "q, k, v, o must be 16-byte aligned");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if ((s = begin_call(p, ws, st)) != SPAVA_OK) return s;
  s = p->d == 128 ? launch_attn<128>(p, p->d_items_dense, p->n_items_dense, q, k, v, nullptr, nullptr, o, lse, ws, st)
                  : launch_attn<64>(p, p->d_items_dense, p->n_items_dense, q, k, v, nullptr, nullptr, o, lse, ws, st);
  if (s != SPAVA_OK) return s;
  mark(p, -1, st);
  return ok();
}

spava_status spava_shard_owners(int32_t n_hosts, int32_t world, int32_t policy, int32_t* owner_out) {
  if (!owner_out || n_hosts < 1 || world < 1) return fail(SPAVA_ERR_INVALID_ARG, "need H >= 1, world >= 1, an array");
  if (policy == SPAVA_SHARD_CONTIGUOUS) {
    if (n_hosts % world) return fail(SPAVA_ERR_INVALID_ARG, "contiguous split needs H %% world == 0");
    const int per = n_hosts / world;
    for (int h = 0; h < n_hosts; ++h) owner_out[h] = h / per;
    return ok();
  }
  if (policy == SPAVA_SHARD_ZIGZAG) {
    if (n_hosts % (2 * world)) return fail(SPAVA_ERR_INVALID_ARG, "zigzag needs H %% (2 * world) == 0");
    for (int h = 0; h < n_hosts; ++h) {
      const int t = h % (2 * world);
      owner_out[h] = t < world ? t : 2 * world - 1 - t;
    }
    return ok();
  }
  return fail(SPAVA_ERR_INVALID_ARG, "unknown shard policy %d", policy);
}

spava_status spava_plan_shard_owners(const spava_plan* p, int32_t world, int32_t policy, int32_t* owner_out) {
  if (!p || !owner_out || world < 1) return fail(SPAVA_ERR_INVALID_ARG, "need a plan, world >= 1 and an array");
  if (policy != SPAVA_SHARD_LONGEST_FIRST) return spava_shard_owners(p->H, world, policy, owner_out);
  const int H = p->H;
  std::vector<int64_t> cost(H);
  for (int h = 0; h < H; ++h) {
    const int64_t B = p->off[h + 1] - p->off[h];
    cost[h] = B * (B + 1) / 2 + static_cast<int64_t>(p->T) * B;
    if (h >= 1) cost[h] += B * (p->A + static_cast<int64_t>(h) * p->P);
    if (h == H - 1) cost[h] += static_cast<int64_t>(p->T) * (p->T + 1) / 2;
  }
  return spava_shard_owners_by_cost(H, world, cost.data(), owner_out);
}

spava_status spava_shard_owners_by_cost(int32_t n_hosts, int32_t world, const int64_t* cost, int32_t* owner_out) {
  if (!cost || !owner_out || n_hosts < 1 || world < 1)
    return fail(SPAVA_ERR_INVALID_ARG, "need H >= 1, world >= 1 and two arrays");
  for (int h = 0; h < n_hosts; ++h)
    if (cost[h] < 0) return fail(SPAVA_ERR_INVALID_ARG, "host %d has a negative cost", h);
  std::vector<int> order(n_hosts);
  for (int h = 0; h < n_hosts; ++h) order[h] = h;
  std::stable_sort(order.begin(), order.end(), [&](int a, int b) { return cost[a] > cost[b]; });
  std::vector<int64_t> load(world, 0);
  for (int h : order) {
    int best = 0;
    for (int r = 1; r < world; ++r)
      if (load[r] < load[best]) best = r;
    owner_out[h] = best;
    load[best] += cost[h];
  }
  return ok();
}

spava_status spava_plan_set_shard(spava_plan* p, int32_t rank, int32_t world, const int32_t* owner) {
  if (!p || !owner) return fail(SPAVA_ERR_INVALID_ARG, "plan and owner must not be NULL");
  if (world < 1 || rank < 0 || rank >= world) return fail(SPAVA_ERR_INVALID_ARG, "need 0 <= rank < world");
  for (int h = 0; h < p->H; ++h)
    if (owner[h] < 0 || owner[h] >= world) return fail(SPAVA_ERR_INVALID_ARG, "host %d has owner %d", h, owner[h]);
  const int H = p->H;
  const bool passing = scores_needed(*p);
  // slots: passing rows of each rank's hosts < H-1, text pieces of each rank
  std::vector<int> n_pass(world, 0), n_text(world, 0), pslot(H, -1);
  for (int h = 0; h < H; ++h) {
    if (passing && h < H - 1) pslot[h] = n_pass[owner[h]]++;
    if (p->T > 0) ++n_text[owner[h]];
  }
  if (p->T > 0) ++n_text[owner[H - 1]];  // the text rows' own causal piece
  const int pass_slots = *std::max_element(n_pass.begin(), n_pass.end());
  const int text_slots = *std::max_element(n_text.begin(), n_text.end());
  HostMask mine(H, 0);
  for (int h = 0; h < H; ++h) mine[h] = owner[h] == rank;
  std::vector<int> tslot(H + 1, -1);
  int used = 0;
  if (p->T > 0) {
    for (int h = 0; h < H; ++h)
      if (mine[h]) tslot[h] = rank * text_slots + used++;
    if (mine[H - 1]) tslot[H] = rank * text_slots + used++;
  }
  std::vector<int> own_scored, xrow0(std::max(H - 1, 1), 0);
  for (int h = 0; h + 1 < H; ++h) {
    if (!passing) break;
    xrow0[h] = (owner[h] * pass_slots + pslot[h]) * p->P;
    if (mine[h]) own_scored.push_back(h);
  }
  const auto local = build_local_items(*p, &mine, &tslot);
  const auto remote = build_remote_items(*p, &mine);
  const auto pre = build_prefill_items(*p, &mine, &tslot);
  const auto probe = build_probe_items(*p, H - 1, &mine);
  const auto score = passing ? build_score_items(*p, H - 1, &mine) : std::vector<int4>();
  TablePacker tab;
  const size_t o_hosts = tab.put(own_scored.data(), own_scored.size() * 4);
  const size_t o_xrow = tab.put(xrow0.data(), xrow0.size() * 4);
  const size_t o_score = tab.put(score.data(), score.size() * sizeof(int4));
  const size_t o_local = tab.put(local.data(), local.size() * sizeof(AttnItem));
  const size_t o_remote = tab.put(remote.data(), remote.size() * sizeof(AttnItem));
  const size_t o_probe = tab.put(probe.data(), probe.size() * sizeof(AttnItem));
  const size_t o_pre = tab.put(pre.data(), pre.size() * sizeof(AttnItem));
  if (p->dtab_shard) {
    SPAVA_CUDA(cudaDeviceSynchronize());
    SPAVA_CUDA(cudaFree(p->dtab_shard));
    p->dtab_shard = nullptr;
    p->shard_world = 0;
  }
  void* d = nullptr;
  spava_status st = upload_table(tab.host, &d);
  if (st != SPAVA_OK) return st;
  uint8_t* base = static_cast<uint8_t*>(d);
  p->dtab_shard = d;
  p->shard_rank = rank;
  p->shard_world = world;
  p->owner.assign(owner, owner + H);
  p->pass_slots = pass_slots;
  p->text_slots = text_slots;
  p->text_slots_used = used;
  p->d_shard_hosts = reinterpret_cast<int*>(base + o_hosts);
  p->n_shard_hosts = static_cast<int>(own_scored.size());
  p->d_xrow0 = reinterpret_cast<int*>(base + o_xrow);
  p->d_score_shard = reinterpret_cast<int4*>(base + o_score);
  p->n_score_shard = static_cast<int>(score.size());
  p->d_items_shard_local = reinterpret_cast<AttnItem*>(base + o_local);
  p->n_items_shard_local = static_cast<int>(local.size());
  p->d_items_shard_remote = reinterpret_cast<AttnItem*>(base + o_remote);
  p->n_items_shard_remote = static_cast<int>(remote.size());
  p->d_items_shard_probe = reinterpret_cast<AttnItem*>(base + o_probe);
  p->n_items_shard_probe = static_cast<int>(probe.size());
  p->d_items_shard_pre = reinterpret_cast<AttnItem*>(base + o_pre);
  p->n_items_shard_pre = static_cast<int>(pre.size());
  layout_workspace(p);
  return ok();
}

spava_status spava_shard_query(const spava_plan* p, spava_shard_layout* out) {
  if (!p || !out) return fail(SPAVA_ERR_INVALID_ARG, "plan and out must not be NULL");
  if (p->shard_world == 0) return fail(SPAVA_ERR_INVALID_ARG, "plan is not sharded (spava_plan_set_shard)");
  spava_shard_layout l;
  std::memset(&l, 0, sizeof(l));
  l.workspace_bytes = p->ws_total_shard;
  l.pass_k_offset = p->ws_xk;
  l.pass_v_offset = p->ws_xv;
  l.pass_bytes_per_rank = static_cast<uint64_t>(p->pass_slots) * p->P * score_rows(*p) * p->d * 2;
  l.text_o_offset = p->ws_to;
  l.text_o_bytes_per_rank = static_cast<uint64_t>(p->text_slots) * p->T * p->hq * p->d * 4;
  l.text_lse_offset = p->ws_tl;
  l.text_lse_bytes_per_rank = static_cast<uint64_t>(p->text_slots) * p->hq * p->T * 4;
  l.scores_offset = p->ws_scores;
  l.idx_offset = p->ws_idx;
  l.pass_slots = p->pass_slots;
  l.text_slots = p->text_slots;
  *out = l;
  return ok();
}

spava_status spava_shard_stage(const spava_plan* p, int32_t stage, const void* q, const void* k, const void* v,
                               void* o, float* lse, void* ws, void* stream) {
  spava_status s;
  if ((s = check_plan_ws(p, ws)) != SPAVA_OK) return s;
  if (p->shard_world == 0) return fail(SPAVA_ERR_INVALID_ARG, "plan is not sharded (spava_plan_set_shard)");
  if (stage < SPAVA_SHARD_SELECT || stage > SPAVA_SHARD_ATTEND) return fail(SPAVA_ERR_INVALID_ARG, "unknown stage %d", stage);
  const bool need_qkv = stage != SPAVA_SHARD_MERGE, need_o = stage != SPAVA_SHARD_SELECT;
  if (need_qkv && (!q || !k || !v)) return fail(SPAVA_ERR_INVALID_ARG, "NULL q, k or v");
  if (need_o && (!o || !lse)) return fail(SPAVA_ERR_INVALID_ARG, "NULL o or lse");
  if ((need_qkv && (!aligned16(q) || !aligned16(k) || !aligned16(v))) || (need_o && !aligned16(o)))
    return fail(SPAVA_ERR_INVALID_ARG, "q, k, v, o must be 16-byte aligned");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if ((s = begin_call(p, ws, st, stage == SPAVA_SHARD_SELECT)) != SPAVA_OK) return s;
  uint8_t* w = static_cast<uint8_t*>(ws);
  TwoStageBufs ts;
  ts.row_o = reinterpret_cast<float*>(w + p->ws_row_o);
  ts.row_lse = reinterpret_cast<float*>(w + p->ws_row_lse);
  ts.text_o = reinterpret_cast<float*>(w + p->ws_to);
  ts.text_lse = reinterpret_cast<float*>(w + p->ws_tl);
  const size_t pass_part = static_cast<size_t>(p->pass_slots) * p->P * score_rows(*p) * p->d * 2;
  // this rank's unused text slots: O = 0, lse = -inf
  auto fill_spare_text = [&]() -> spava_status {
    const int spare = p->text_slots - p->text_slots_used;
    if (p->T == 0 || spare <= 0) return SPAVA_OK;
    const size_t slot0 = static_cast<size_t>(p->shard_rank) * p->text_slots + p->text_slots_used;
    const size_t n_o = static_cast<size_t>(spare) * p->T * p->hq * p->d, n_l = static_cast<size_t>(spare) * p->hq * p->T;
    uint32_t* fo = reinterpret_cast<uint32_t*>(ts.text_o) + slot0 * p->T * p->hq * p->d;
    uint32_t* fl = reinterpret_cast<uint32_t*>(ts.text_lse) + slot0 * p->hq * p->T;
    const int grid = std::max(1, std::min(p->num_sms * 4, static_cast<int>((n_o + 255) / 256)));
    mark(p, kLabTextFill, st);
    spava::fill_u32_kernel<<<grid, 256, 0, st>>>(fo, n_o, 0u);
    spava::fill_u32_kernel<<<grid, 256, 0, st>>>(fl, n_l, 0xFF800000u);
    SPAVA_CUDA(cudaGetLastError());
    g_last_launches += 2;
    return SPAVA_OK;
  };
  // every host's passing rows from the gathered exchange buffers into k_pass / v_pass
  auto unpack = [&]() -> spava_status {
    if (!scores_needed(*p)) return SPAVA_OK;
    const int rows = score_rows(*p), cpr = p->d * 2 / 16;
    const size_t total = static_cast<size_t>(rows) * (p->H - 1) * p->P * cpr;
    const int grid = static_cast<int>(std::min<size_t>((total + 255) / 256, static_cast<size_t>(p->num_sms) * 8));
    mark(p, kLabUnpack, st);
    spava::unpack_passing_kernel<<<grid, 256, 0, st>>>(
        reinterpret_cast<const uint4*>(w + p->ws_xk), reinterpret_cast<const uint4*>(w + p->ws_xv), p->d_xrow0,
        reinterpret_cast<uint4*>(w + p->ws_kp), reinterpret_cast<uint4*>(w + p->ws_vp), rows, p->H - 1, p->P, cpr);
    SPAVA_CUDA(cudaGetLastError());
    ++g_last_launches;
    return SPAVA_OK;
  };
  switch (stage) {
    case SPAVA_SHARD_SELECT: {
      if (!scores_needed(*p) || p->n_shard_hosts == 0) break;
      float* scores = reinterpret_cast<float*>(w + p->ws_scores);
      int32_t* idx = reinterpret_cast<int32_t*>(w + p->ws_idx);
      if ((s = launch_probe_lse(p, q, k, k, ws, st, p->d_items_shard_probe, p->n_items_shard_probe)) != SPAVA_OK)
        return s;
      s = p->d == 128 ? launch_score<128>(p, q, k, scores, p->d_score_shard, p->n_score_shard, ws, st)
                      : launch_score<64>(p, q, k, scores, p->d_score_shard, p->n_score_shard, ws, st);
      if (s != SPAVA_OK) return s;
      PassDest dst{w + p->ws_xk + p->shard_rank * pass_part, w + p->ws_xv + p->shard_rank * pass_part, true};
      if ((s = launch_select(p, scores, idx, st, k, v, dst, p->d_shard_hosts, p->n_shard_hosts)) != SPAVA_OK) return s;
      break;
    }
    case SPAVA_SHARD_LOCAL: {
      if ((s = fill_spare_text()) != SPAVA_OK) return s;
      s = p->d == 128 ? launch_attn<128>(p, p->d_items_shard_local, p->n_items_shard_local, q, k, v, nullptr, nullptr,
                                         o, lse, ws, st, ts)
                      : launch_attn<64>(p, p->d_items_shard_local, p->n_items_shard_local, q, k, v, nullptr, nullptr,
                                        o, lse, ws, st, ts);
      if (s != SPAVA_OK) return s;
      break;
    }
    case SPAVA_SHARD_REMOTE: {
      if (p->n_items_shard_remote == 0) break;
      void* kp = w + p->ws_kp;
      void* vp = w + p->ws_vp;
      if ((s = unpack()) != SPAVA_OK) return s;
      s = p->d == 128 ? launch_attn<128>(p, p->d_items_shard_remote, p->n_items_shard_remote, q, k, v, kp, vp, o, lse,
                                         ws, st, ts)
                      : launch_attn<64>(p, p->d_items_shard_remote, p->n_items_shard_remote, q, k, v, kp, vp, o, lse,
                                        ws, st, ts);
      if (s != SPAVA_OK) return s;
      break;
    }
    case SPAVA_SHARD_ATTEND: {
      if ((s = fill_spare_text()) != SPAVA_OK) return s;
      void* kp = w + p->ws_kp;
      void* vp = w + p->ws_vp;
      if (p->n_items_shard_remote > 0 && (s = unpack()) != SPAVA_OK) return s;
      s = p->d == 128 ? launch_attn<128>(p, p->d_items_shard_pre, p->n_items_shard_pre, q, k, v, kp, vp, o, lse, ws,
                                         st, ts)
                      : launch_attn<64>(p, p->d_items_shard_pre, p->n_items_shard_pre, q, k, v, kp, vp, o, lse, ws,
                                        st, ts);
      if (s != SPAVA_OK) return s;
      break;
    }
    case SPAVA_SHARD_MERGE: {
      if ((s = launch_merge(p, o, lse, ws, st, ts.text_o, ts.text_lse, p->shard_world * p->text_slots)) != SPAVA_OK)
        return s;
      break;
    }
  }
  mark(p, -1, st);
  return ok();
}

spava_status spava_profile_begin(spava_plan* p, int32_t max_marks) {
  if (!p || max_marks < 2) return fail(SPAVA_ERR_INVALID_ARG, "need a plan and max_marks >= 2");
  spava_profile_end(p);
  p->prof_ev.assign(max_marks, nullptr);
  for (auto& e : p->prof_ev) SPAVA_CUDA(cudaEventCreate(&e));
  p->prof_label.assign(max_marks, -1);
  p->prof_call.assign(max_marks, -1);
  p->prof_used = 0;
  return ok();
}

int32_t spava_profile_read(spava_plan* p, int32_t* labels, float* ms, int32_t max) {
  if (!p) return -1;
  if (p->prof_used > 0 && cudaEventSynchronize(p->prof_ev[p->prof_used - 1]) != cudaSuccess) return -1;
  int n = 0;
  for (int k = 0; k + 1 < p->prof_used && n < max; ++k) {
    if (p->prof_label[k] < 0 || p->prof_call[k] != p->prof_call[k + 1]) continue;
    float t = 0.f;
    if (cudaEventElapsedTime(&t, p->prof_ev[k], p->prof_ev[k + 1]) != cudaSuccess) return -1;
    if (labels) labels[n] = p->prof_label[k];
    if (ms) ms[n] = t;
    ++n;
  }
  p->prof_used = 0;
  return n;
}

spava_status spava_profile_end(spava_plan* p) {
  if (!p) return fail(SPAVA_ERR_INVALID_ARG, "plan is NULL");
  if (!p->prof_ev.empty()) cudaDeviceSynchronize();
  for (cudaEvent_t e : p->prof_ev)
    if (e) cudaEventDestroy(e);
  p->prof_ev.clear();
  p->prof_label.clear();
  p->prof_call.clear();
  p->prof_used = 0;
  return ok();
}

const char* spava_kernel_name(int32_t label) {
  switch (label) {
    case kLabScore: return "score";
    case kLabSelect: return "select";
    case kLabGather: return "gather";
    case kLabAttn: return "attention";
    case kLabMerge: return "lse_merge";
    case kLabDense: return "attention_dense";
    case kLabSelectGather: return "select_gather";
    case kLabFill: return "score_keys";
    case kLabAttnLocal: return "attention_local";
    case kLabAttnRemote: return "attention_remote";
    case kLabProbeLse: return "probe_lse";
    case kLabUnpack: return "unpack_passing";
    case kLabTextFill: return "text_slot_fill";
    case kLabScoreSelectGather: return "score_select_gather";
  }
  return "unknown";
}

spava_status spava_check_device_error(const spava_plan* p, void* ws, void* stream) {
  spava_status s;
  if ((s = check_plan_ws(p, ws)) != SPAVA_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  SPAVA_CUDA(cudaStreamSynchronize(st));
  unsigned int word = 0;
  SPAVA_CUDA(cudaMemcpy(&word, err_word(p, ws), sizeof(word), cudaMemcpyDeviceToHost));
  if (word) {
    SPAVA_CUDA(cudaMemsetAsync(err_word(p, ws), 0, 256, st));
    SPAVA_CUDA(cudaStreamSynchronize(st));
    if (word == spava::kErrBadIndex)
      return fail(SPAVA_ERR_DEVICE_CHECK, "an index fell outside its range; the access was skipped (error bits 0x%x)",
                  word);
    return fail(SPAVA_ERR_TIMEOUT, "a bounded device wait ran out (error bits 0x%x)", word);
  }
  return ok();
}

}  // extern "C"

// =================================================================== layer projections
namespace {

constexpr size_t kLayerErrBytes = 256;

// Current device, checked to be an sm_100 part; its SM count.
spava_status layer_device(int* num_sms) {
  int dev = -1, major = 0, minor = 0;
  SPAVA_CUDA(cudaGetDevice(&dev));
  SPAVA_CUDA(cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev));
  SPAVA_CUDA(cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev));
  if (major != 10 || minor != 0)
    return fail(SPAVA_ERR_UNSUPPORTED, "needs an sm_100 (B200) device, found sm_%d%d", major, minor);
  SPAVA_CUDA(cudaDeviceGetAttribute(num_sms, cudaDevAttrMultiProcessorCount, dev));
  return SPAVA_OK;
}

spava_status launch_proj(const void* a, int M, int K, const void* w, int N, spava::ProjParams pp, int num_sms,
                         cudaStream_t st) {
  using S = spava::ProjShape;
  CUtensorMap tmA, tmB;
  spava_status s;
  if ((s = make_map_2d(&tmA, a, K, M, S::kBM)) != SPAVA_OK) return s;
  if ((s = make_map_2d(&tmB, w, K, N, S::kBN)) != SPAVA_OK) return s;
  pp.M = M;
  pp.K = K;
  pp.N = N;
  pp.n_tiles_n = N / S::kBN;
  pp.n_tiles = ceil_div(M, S::kBM) * pp.n_tiles_n;
  pp.wait_limit_ns = spava::kDefaultWaitLimitNs;
  if ((s = ensure_smem(spava::proj_gemm_kernel, S::kSmemBytes)) != SPAVA_OK) return s;
  spava::proj_gemm_kernel<<<std::min(pp.n_tiles, num_sms), S::kThreads, S::kSmemBytes, st>>>(tmA, tmB, pp);
  SPAVA_CUDA(cudaGetLastError());
  ++g_last_launches;
  return SPAVA_OK;
}

}  // namespace

extern "C" {

size_t spava_layer_workspace_bytes(int32_t n_tokens) {
  return n_tokens < 0 ? 0 : kLayerErrBytes + align_up(static_cast<size_t>(n_tokens) * 4, 256);
}

spava_status spava_qkv_projection(const void* x, int32_t n_tokens, int32_t hidden, const void* w_qkv, int32_t hq,
                                  int32_t hkv, int32_t head_dim, float rms_eps, void* q, void* k, void* v, void* ws,
                                  void* stream) {
  g_last_launches = 0;
  if (!x || !w_qkv || !q || !k || !v || !ws) return fail(SPAVA_ERR_INVALID_ARG, "NULL pointer");
  if (n_tokens < 1 || hidden < 1 || hq < 1 || hkv < 1 || head_dim < 1 || hq % hkv)
    return fail(SPAVA_ERR_INVALID_ARG, "need n_tokens, hidden, hq, hkv, head_dim >= 1 and hq %% hkv == 0");
  if (!(rms_eps > 0.f)) return fail(SPAVA_ERR_INVALID_ARG, "rms_eps must be positive");
  const int nq = hq * head_dim, nk = hkv * head_dim;
  if (hidden % 256 || nq % 256 || nk % 256)
    return fail(SPAVA_ERR_UNSUPPORTED, "hidden, hq * head_dim and hkv * head_dim must be multiples of 256");
  if (!aligned16(x) || !aligned16(w_qkv) || !aligned16(q) || !aligned16(k) || !aligned16(v))
    return fail(SPAVA_ERR_INVALID_ARG, "x, w_qkv, q, k, v must be 16-byte aligned");
  if (reinterpret_cast<uintptr_t>(ws) & 255u) return fail(SPAVA_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
  int num_sms = 0;
  spava_status s;
  if ((s = layer_device(&num_sms)) != SPAVA_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* w8 = static_cast<uint8_t*>(ws);
  float* inv_rms = reinterpret_cast<float*>(w8 + kLayerErrBytes);
  SPAVA_CUDA(cudaMemsetAsync(w8, 0, kLayerErrBytes, st));
  spava::rms_rows_kernel<<<ceil_div(n_tokens, 8), 256, 0, st>>>(static_cast<const __nv_bfloat16*>(x), n_tokens,
                                                                 hidden, rms_eps, inv_rms);
  SPAVA_CUDA(cudaGetLastError());
  ++g_last_launches;
  spava::ProjParams pp;
  std::memset(&pp, 0, sizeof(pp));
  pp.mode = spava::kProjQKV;
  pp.nq = nq;
  pp.nk = nk;
  pp.q = static_cast<__nv_bfloat16*>(q);
  pp.k = static_cast<__nv_bfloat16*>(k);
  pp.v = static_cast<__nv_bfloat16*>(v);
  pp.inv_rms = inv_rms;
  pp.err_word = reinterpret_cast<unsigned int*>(w8);
  if ((s = launch_proj(x, n_tokens, hidden, w_qkv, nq + 2 * nk, pp, num_sms, st)) != SPAVA_OK) return s;
  return ok();
}

spava_status spava_out_projection(const void* o, int32_t n_tokens, int32_t in_features, const void* w_o,
                                  int32_t hidden, void* x, void* ws, void* stream) {
  g_last_launches = 0;
  if (!o || !w_o || !x || !ws) return fail(SPAVA_ERR_INVALID_ARG, "NULL pointer");
  if (n_tokens < 1 || in_features < 1 || hidden < 1) return fail(SPAVA_ERR_INVALID_ARG, "sizes must be positive");
  if (in_features % 256 || hidden % 256)
    return fail(SPAVA_ERR_UNSUPPORTED, "in_features and hidden must be multiples of 256");
  if (!aligned16(o) || !aligned16(w_o) || !aligned16(x))
    return fail(SPAVA_ERR_INVALID_ARG, "o, w_o, x must be 16-byte aligned");
  if (reinterpret_cast<uintptr_t>(ws) & 255u) return fail(SPAVA_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
  int num_sms = 0;
  spava_status s;
  if ((s = layer_device(&num_sms)) != SPAVA_OK) return s;
  spava::ProjParams pp;
  std::memset(&pp, 0, sizeof(pp));
  pp.mode = spava::kProjResidual;
  pp.residual = static_cast<const __nv_bfloat16*>(x);
  pp.out = static_cast<__nv_bfloat16*>(x);
  pp.err_word = static_cast<unsigned int*>(ws);
  if ((s = launch_proj(o, n_tokens, in_features, w_o, hidden, pp, num_sms, static_cast<cudaStream_t>(stream))) !=
      SPAVA_OK)
    return s;
  return ok();
}

spava_status spava_layer_check_error(void* ws, void* stream) {
  if (!ws) return fail(SPAVA_ERR_INVALID_ARG, "workspace is NULL");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  SPAVA_CUDA(cudaStreamSynchronize(st));
  unsigned int word = 0;
  SPAVA_CUDA(cudaMemcpy(&word, ws, sizeof(word), cudaMemcpyDeviceToHost));
  if (word) {
    SPAVA_CUDA(cudaMemsetAsync(ws, 0, kLayerErrBytes, st));
    SPAVA_CUDA(cudaStreamSynchronize(st));
    return fail(SPAVA_ERR_TIMEOUT, "a bounded device wait ran out in a projection (error bits 0x%x)", word);
  }
  return ok();
}

}  // extern "C"
