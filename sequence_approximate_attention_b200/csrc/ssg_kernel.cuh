// Probe scoring, top-P selection and the passing-KV gather of hosts 0..H-2 in one
// persistent launch (APB-V technical summary, 1. Framework design, "Approximate
// attention mechanism": every host ranks its local keys by query-to-context
// attention scores and passes the top P of them, with their values, to the hosts
// after it).
//
// A unit is one (host h <= H-2, KV head g).  Its 128-key score tiles are the work
// items, listed in unit order and dealt to the CTAs in rounds: round r gives every CTA
// the next contiguous chunk of the list, so the units of round r are complete once
// round r is scored everywhere, and their selection and copies overlap the scoring of
// the rounds after it.  The scores are those of score_kernel with the max over probe
// rows and the group's query heads (logit scores), from the same pipeline (one TMA
// thread, two MMA issuers, S^T = K_tile Qprobe^T with one key per TMEM lane).
//
// Hand-offs go through global memory.  The epilogue warps count their stored tiles
// in shared memory; a publisher thread adds each finished run of a unit's tiles to the
// unit's global counter (gpu-scope fence, then atomic) and hands a unit whose count
// it completes to its own CTA's worker group.  The worker group selects the unit's
// top P -- radix select on the unit's scores, read back from L2, with
// select_topp_kernel's rule: keys above the P-th largest, then the keys equal to it
// lowest index first, written in index order -- and raises the unit's ready flag.
// The gather of a unit is split into tasks of `task_rows` passing rows; task t
// belongs to CTA t % gridDim.x, so the copies of the units that complete last still
// spread over every SM.  A worker group with nothing to do polls the ready flags of
// its tasks' units.
//
// CTAs wait on one another's progress, so the launch is cooperative (every CTA is
// resident); every wait has a time limit, after which the waiting thread records an
// error bit and its CTA winds down.
//
// CTA = 512 threads: warp 0 TMA (one thread), warps 1 and 3 the MMA issuers (one
// thread each), warp 2 TMEM allocator and publisher (one thread), warps 4-7 score
// epilogue (lane = key), warps 8-15 the worker group (named barrier 1).
#pragma once

#include "common.cuh"
#include "score_kernel.cuh"
#include "topp_select.cuh"

namespace spava {

struct SsgParams {
  // scoring
  const int4* items;      // (host, kv head, first key of the tile, block end e), dealt in rounds
  const int* cta_first;   // [gridDim.x + 1]: CTA b scores items [cta_first[b], cta_first[b+1])
  int probe_r;            // R
  int group;              // G = hq / hkv
  int chunk_tokens;       // Rc probe tokens per N chunk (Rc * G <= 256, multiple of 16)
  int n_chunks;           // ceil(R / Rc)
  int n_visual;           // N (row stride of scores)
  float scale;
  float* scores;          // [hkv][N]
  int q_bufs;             // probe-query buffers (1 when every (host, group) is one chunk, else 2)
  int q_buf_bytes;
  int k_stages;
  // units and selection
  const int* off;         // host offsets [H + 1]
  int hkv, anchor, passing;
  int* unit_cnt;          // [(H-1) hkv], zero at launch: score tiles of the unit stored so far
  int* unit_ready;        // [(H-1) hkv], zero at launch: 1 once the unit's indices are written
  int32_t* idx;           // [H-1][hkv][P]
  // gather: k/v [tokens][hkv][d] and k_pass/v_pass [hkv][H-1][P][d], in 16-byte chunks
  const uint4* k;
  const uint4* v;
  uint4* kp;
  uint4* vp;
  int chunks_per_row;     // d * 2 / 16 (8 or 16)
  size_t dst_g, dst_h;    // chunks between KV heads / hosts of k_pass
  int task_rows, tasks_per_unit, n_tasks;
  unsigned int* err_word;
  uint64_t wait_limit_ns;
  int stall_producer;     // testing aid: the load thread issues nothing
};

// Shared state of the worker group, the publisher and the hand-off ring.
struct SsgCtl {
  ToppShared sel;  // the worker group's selection scratch
  int ring[32];    // units this CTA completed, + 1 (0 = empty slot)
  int ring_tail;   // slots the publisher filled
  int stored;      // epilogue-warp arrivals: 4 per score tile stored
  int pub_done;    // 1 once the publisher handed over every unit it will
  int cmd, arg;    // the worker leader's decision
  int abort_flag;
};
constexpr int kSsgRing = 32;
constexpr int kSsgBar = 1;  // named barrier of the worker group

template <int D>
struct SsgShape {
  static constexpr int kThreads = 512;
  static constexpr int kHalves = D / 64;
  static constexpr int kKTileBytes = kHalves * 128 * 128;  // 128 keys
  static constexpr int kMaxStages = kScorePipeStages;
  static constexpr int kBarBytes = 256;
  static constexpr int kMaxLocalItems = 256;  // item metadata cached in shared memory
  static constexpr int kItemBytes = kMaxLocalItems * 16;
  static constexpr int kCtlBytes = (static_cast<int>(sizeof(SsgCtl)) + 255) / 256 * 256;
  static constexpr int kSmemMax = 232448;  // opt-in limit per CTA on sm_100
  static constexpr uint32_t kTmemCols = 512;
  static constexpr int kMaxOwnTasks = 64;  // gather tasks per CTA (one bit each)
  static constexpr int kSelPer = 32;       // rows of 256 candidates held in registers (one key per worker thread per row)
  static constexpr int smem_bytes(int q_bufs, int q_buf_bytes, int k_stages) {
    return q_bufs * q_buf_bytes + k_stages * kKTileBytes + kBarBytes + kItemBytes + kCtlBytes + 1024;
  }
};

// Named barrier of the worker group.  The compiler does not see an inline barrier, so
// nothing else reconverges a warp whose lanes took different branches just before it
// (the leader warp's lane-0 work): __syncwarp does, and the non-aligned form of the
// barrier is the one defined for a warp that arrives in parts.
__device__ __forceinline__ void worker_bar() {
  __syncwarp();
  asm volatile("barrier.sync %0, %1;" ::"n"(kSsgBar), "n"(256) : "memory");
}
struct WorkerBar {
  __device__ __forceinline__ void operator()() const { worker_bar(); }
};

__device__ __forceinline__ int ld_acquire_gpu(const int* p) {
  int v;
  asm volatile("ld.acquire.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void st_release_gpu(int* p, int v) {
  asm volatile("st.release.gpu.global.s32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ int ld_acquire_cta_shared(const int* p) {
  int v;
  asm volatile("ld.acquire.cta.shared::cta.s32 %0, [%1];" : "=r"(v) : "r"(smem_u32(p)) : "memory");
  return v;
}
__device__ __forceinline__ void red_release_cta_shared_add(int* p, int v) {
  asm volatile("red.release.cta.shared::cta.add.s32 [%0], %1;" ::"r"(smem_u32(p)), "r"(v) : "memory");
}

__device__ __forceinline__ void fence_acq_rel_gpu() { asm volatile("fence.acq_rel.gpu;" ::: "memory"); }

// Gather task: passing rows [c task_rows, ...) of unit u (host h, KV head g), K and V,
// 16 bytes per thread; each thread first reads its rows' indices, then keeps eight
// rows' K and V chunks in flight before storing any.
__device__ __forceinline__ void ssg_gather(const SsgParams& p, int u, int c, int wt) {
  constexpr int NT = 256, kUnroll = 8;
  const int h = u / p.hkv, g = u - h * p.hkv;
  const int r0 = c * p.task_rows, nr = min(p.task_rows, p.passing - r0);
  const int32_t* ix = p.idx + (static_cast<size_t>(h) * p.hkv + g) * p.passing + r0;
  const int cpr = p.chunks_per_row, cs = __ffs(cpr) - 1;
  const int total = nr * cpr;
  const size_t dst0 = static_cast<size_t>(g) * p.dst_g + static_cast<size_t>(h) * p.dst_h + static_cast<size_t>(r0) * cpr;
  for (int t0 = wt; t0 < total; t0 += kUnroll * NT) {
    int tok[kUnroll];
#pragma unroll
    for (int i = 0; i < kUnroll; ++i) {
      const int t = t0 + i * NT;
      tok[i] = t < total ? __ldcg(ix + (t >> cs)) : 0;
    }
    uint4 kv[kUnroll], vv[kUnroll];
#pragma unroll
    for (int i = 0; i < kUnroll; ++i) {
      const int t = t0 + i * NT;
      if (t < total && static_cast<unsigned>(tok[i]) < static_cast<unsigned>(p.n_visual)) {
        const size_t src = (static_cast<size_t>(tok[i]) * p.hkv + g) * cpr + (t & (cpr - 1));
        kv[i] = __ldg(p.k + src);
        vv[i] = __ldg(p.v + src);
      } else if (t < total) {
        atomicOr(p.err_word, kErrBadIndex);
      }
    }
#pragma unroll
    for (int i = 0; i < kUnroll; ++i) {
      const int t = t0 + i * NT;
      if (t < total && static_cast<unsigned>(tok[i]) < static_cast<unsigned>(p.n_visual)) {
        p.kp[dst0 + t] = kv[i];
        p.vp[dst0 + t] = vv[i];
      }
    }
  }
}

enum : int { kSsgCmdExit = 0, kSsgCmdSelect = 1, kSsgCmdGather = 2 };

// Poll wait for `*flag >= target` by one thread, bounded; false on abort or timeout.
__device__ __forceinline__ bool ssg_wait_count(const int* flag, int target, const SsgParams& p, SsgCtl* ctl) {
  if (ld_acquire_cta_shared(flag) >= target) return true;
  const uint64_t t0 = global_timer_ns();
  for (;;) {
    __nanosleep(64);
    if (ld_acquire_cta_shared(flag) >= target) return true;
    if (*reinterpret_cast<volatile int*>(&ctl->abort_flag)) return false;
    if (global_timer_ns() - t0 > p.wait_limit_ns) {
      atomicOr(p.err_word, kErrWaitUnit);
      *reinterpret_cast<volatile int*>(&ctl->abort_flag) = 1;
      return false;
    }
  }
}

template <int D>
__global__ void __launch_bounds__(512, 1)
    ssg_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmQp,
               const SsgParams p) {
  using S = SsgShape<D>;
  constexpr uint32_t FULL = 0xffffffffu;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sK = smem + p.q_bufs * p.q_buf_bytes;  // q_buf_bytes is a multiple of 1024
  uint8_t* bar_base = sK + p.k_stages * S::kKTileBytes;
  const ScorePipe sp = score_pipe_at(smem, sK, p.q_bufs, p.q_buf_bytes, p.k_stages, reinterpret_cast<uint64_t*>(bar_base));
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar_base + kScorePipeBarBytes);
  int4* s_items = reinterpret_cast<int4*>(bar_base + S::kBarBytes);
  SsgCtl* ctl = reinterpret_cast<SsgCtl*>(reinterpret_cast<uint8_t*>(s_items) + S::kItemBytes);
  const ScoreGeom geom{p.probe_r, p.group, p.chunk_tokens, p.n_chunks};

  const int warp = warp_id(), lane = lane_id();
  if (threadIdx.x == 0) {
    score_pipe_init(sp, p.n_chunks);
    fence_mbar_init();
    ctl->ring_tail = 0;
    ctl->stored = 0;
    ctl->pub_done = 0;
    ctl->abort_flag = 0;
  }
  if (threadIdx.x < kSsgRing) ctl->ring[threadIdx.x] = 0;
  if (warp == 2) tmem_alloc(tmem_slot, S::kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const WaitCtx wc{&ctl->abort_flag, p.err_word, p.wait_limit_ns};

  // This CTA's score tiles (the host keeps every range within the cache).
  const int first = __ldg(p.cta_first + blockIdx.x);
  const int n_local = __ldg(p.cta_first + blockIdx.x + 1) - first;
  for (int t = threadIdx.x; t < n_local; t += blockDim.x) s_items[t] = __ldg(p.items + first + t);
  __syncthreads();

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer (lane 0)
    if (lane == 0 && !p.stall_producer) score_produce<D>(sp, geom, s_items, n_local, &tmK, &tmQp, wc);
    __syncwarp();
  } else if (warp == 1 || warp == 3) {
    // ------------------------------------------------------------ MMA issuers (lane 0)
    if (lane == 0) score_issue<D>(sp, geom, s_items, n_local, warp == 1 ? 0 : 1, tmem, wc);
    __syncwarp();
  } else if (warp == 2) {
    // ------------------------------------------------------------ publisher (lane 0)
    // Once all four epilogue warps stored tile li (their release increments of
    // `stored`, observed by this thread's acquire), a run of the unit's tiles that ends
    // at li is added to the unit's global counter after a gpu-scope fence; the
    // addition that completes the unit queues it for this CTA's worker group.
    if (lane == 0) {
      volatile int* vring = ctl->ring;
      int run = 0, tail = 0;
      bool ok = true;
      for (int li = 0; li < n_local && ok; ++li) {
        const int4 it = s_items[li];
        ++run;
        if (li + 1 < n_local && same_group(s_items[li + 1], it)) continue;  // the run goes on
        if (!(ok = ssg_wait_count(&ctl->stored, 4 * (li + 1), p, ctl))) break;
        fence_acq_rel_gpu();
        const int unit = it.x * p.hkv + it.y;
        const int need = (it.w - __ldg(p.off + it.x) + 127) >> 7;  // tiles of the unit
        const int before = atomicAdd(p.unit_cnt + unit, run);
        const bool completes = before + run == need;
        run = 0;
        if (!completes) continue;
        fence_acq_rel_gpu();
        // hand the unit to the worker group; a full ring waits (bounded) for a free slot
        volatile int* rs = vring + (tail & (kSsgRing - 1));
        const uint64_t t0 = global_timer_ns();
        while (*rs != 0) {
          if (*reinterpret_cast<volatile int*>(&ctl->abort_flag)) {
            ok = false;
            break;
          }
          if (global_timer_ns() - t0 > p.wait_limit_ns) {
            atomicOr(p.err_word, kErrWaitUnit);
            *reinterpret_cast<volatile int*>(&ctl->abort_flag) = 1;
            ok = false;
            break;
          }
          __nanosleep(128);
        }
        if (!ok) break;
        *rs = unit + 1;
        ++tail;
        __threadfence_block();
        *reinterpret_cast<volatile int*>(&ctl->ring_tail) = tail;
      }
      __threadfence_block();
      *reinterpret_cast<volatile int*>(&ctl->pub_done) = 1;
    }
    __syncwarp();
  } else if (warp < 8) {
    // ------------------------------------------------------------ score epilogue: one key per thread
    const int qd = warp & 3;
    const int row = qd * 32 + lane;
    const uint32_t tl = tmem + (static_cast<uint32_t>(qd * 32) << 16);
    const int Rc = p.chunk_tokens, G = p.group;
    bool ok = true;
    for (int li = 0; li < n_local && ok; ++li) {
      const int4 it = s_items[li];
      const int j = it.z + row;  // key position
      float mx = -INFINITY;      // max over the group's heads and the probe rows that see key j
      for (int c = 0; c < p.n_chunks; ++c) {
        const int u = li * p.n_chunks + c, b = u & 1;
        ok = __all_sync(FULL, mbar_wait(sp.acc_full + b, (u >> 1) & 1, wc, kErrWaitMma));
        if (!ok) break;
        tc_fence_after();
        const int row0 = it.w - p.probe_r + c * Rc;  // first probe row of the chunk
        const int rc = min(Rc, p.probe_r - c * Rc);  // probe rows in it (a multiple of 16)
        const uint32_t ta = tl + b * 256;
        if (rc == Rc && it.z + 127 < row0) {
          // every column visible to every key of the tile: order-free max over 64-column loads
          const int ncols = Rc * G;
          int n0 = 0;
#pragma unroll 1
          for (; n0 + 64 <= ncols; n0 += 64) {
            uint32_t v[64];
            tmem_ld_x64(ta + n0, v);
            float m8[8];
#pragma unroll
            for (int q = 0; q < 8; ++q) m8[q] = fmaxf(__uint_as_float(v[q]), __uint_as_float(v[q + 8]));
#pragma unroll
            for (int t = 16; t < 64; t += 16)
#pragma unroll
              for (int q = 0; q < 8; ++q) m8[q] = fmax3(m8[q], __uint_as_float(v[t + q]), __uint_as_float(v[t + 8 + q]));
            mx = fmax3(mx, fmax3(fmax3(m8[0], m8[1], m8[2]), fmax3(m8[3], m8[4], m8[5]), fmaxf(m8[6], m8[7])),
                       -INFINITY);
          }
          for (; n0 < ncols; n0 += 16) {
            uint32_t v[16];
            tmem_ld_x16(ta + n0, v);
#pragma unroll
            for (int t = 0; t < 16; ++t) mx = fmaxf(mx, __uint_as_float(v[t]));
          }
        } else {
          // head h: columns [h Rc, h Rc + rc); probe row row0 + t sees key j iff row0 + t >= j
          const int t_min = j - row0;
#pragma unroll 1
          for (int h = 0; h < G; ++h) {
            for (int t0 = 0; t0 < rc; t0 += 16) {
              uint32_t v[16];
              tmem_ld_x16(ta + h * Rc + t0, v);
#pragma unroll
              for (int t = 0; t < 16; ++t)
                if (t0 + t >= t_min) mx = fmaxf(mx, __uint_as_float(v[t]));
            }
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(sp.acc_empty + b);
      }
      if (!ok) break;
      if (j < it.w) p.scores[static_cast<size_t>(it.y) * p.n_visual + j] = mx * p.scale;
      // the warp's 32 scores of tile li are stored (ordered before the release by the warp sync)
      __syncwarp();
      if (lane == 0) red_release_cta_shared_add(&ctl->stored, 1);
    }
  } else {
    // ------------------------------------------------------------ worker group: selection and gather
    const int wt = threadIdx.x - 256;
    const bool leader = warp == 8;
    const int grid = static_cast<int>(gridDim.x), cta = static_cast<int>(blockIdx.x);
    const int n_own = p.n_tasks > cta ? (p.n_tasks - cta + grid - 1) / grid : 0;  // <= kMaxOwnTasks
    uint64_t pending = n_own >= 64 ? ~0ull : ((1ull << n_own) - 1ull);  // own tasks not yet copied
    int head = 0;  // next ring slot to read
    volatile int* vring = ctl->ring;
    volatile int* vtail = &ctl->ring_tail;
    volatile int* vdone = &ctl->pub_done;
    volatile int* vabort = &ctl->abort_flag;
    volatile unsigned int* verr = p.err_word;
    for (;;) {
      if (leader) {
        int cmd = -1, arg = 0;
        const uint64_t t0 = global_timer_ns();
        while (cmd < 0) {
          // 1. a unit this CTA completed: select it first (it unlocks gather tasks everywhere)
          const int e = __shfl_sync(FULL, lane == 0 ? vring[head & (kSsgRing - 1)] : 0, 0);
          if (e > 0) {
            if (lane == 0) vring[head & (kSsgRing - 1)] = 0;
            ++head;
            fence_acq_rel_gpu();
            cmd = kSsgCmdSelect;
            arg = e - 1;
            break;
          }
          // 2. a gather task of this CTA whose unit is selected
          if (pending) {
            bool r0 = false, r1 = false;
            if ((pending >> lane) & 1ull)
              r0 = ld_acquire_gpu(p.unit_ready + (cta + lane * grid) / p.tasks_per_unit) != 0;
            if ((pending >> (lane + 32)) & 1ull)
              r1 = ld_acquire_gpu(p.unit_ready + (cta + (lane + 32) * grid) / p.tasks_per_unit) != 0;
            const uint32_t b0 = __ballot_sync(FULL, r0), b1 = __ballot_sync(FULL, r1);
            if (b0 | b1) {
              const int i = b0 ? __ffs(b0) - 1 : 32 + __ffs(b1) - 1;
              pending &= ~(1ull << i);
              cmd = kSsgCmdGather;
              arg = cta + i * grid;
              break;
            }
          }
          // 3. finished: no own task left, and the publisher is done with every unit it queued taken
          const bool pub_done = *vdone != 0;
          if (!pending && pub_done) {
            __threadfence_block();
            if (*vtail == head) {
              cmd = kSsgCmdExit;
              break;
            }
          }
          // 4. errors and the time limit
          if (*vabort || *verr) {
            cmd = kSsgCmdExit;
            break;
          }
          if (global_timer_ns() - t0 > p.wait_limit_ns) {
            if (lane == 0) {
              atomicOr(p.err_word, kErrWaitUnit);
              *vabort = 1;
            }
            cmd = kSsgCmdExit;
            break;
          }
          // poll slowly while this CTA still scores, quickly once it is done
          __nanosleep(pub_done ? 128 : 1000);
        }
        if (lane == 0) {
          ctl->cmd = cmd;
          ctl->arg = arg;
        }
      }
      worker_bar();
      const int cmd = ctl->cmd, arg = ctl->arg;
      worker_bar();
      if (cmd == kSsgCmdExit) break;
      if (cmd == kSsgCmdSelect) {
        const int h = arg / p.hkv, g = arg - h * p.hkv;
        const int b0 = __ldg(p.off + h), lo = b0 + (h == 0 ? p.anchor : 0), n = __ldg(p.off + h + 1) - lo;
        const float* sc = p.scores + static_cast<size_t>(g) * p.n_visual + lo;
        int32_t* out = p.idx + static_cast<size_t>(arg) * p.passing;
        const WorkerBar bar;
        if (n <= 256 * S::kSelPer)
          topp_select<256, S::kSelPer>(sc, n, lo, p.passing, out, &ctl->sel, wt, bar, p.err_word);
        else
          topp_select<256, 0>(sc, n, lo, p.passing, out, &ctl->sel, wt, bar, p.err_word);
        worker_bar();  // every index of the unit is written (ordered before the release)
        if (wt == 0) st_release_gpu(p.unit_ready + arg, 1);
      } else {
        ssg_gather(p, arg / p.tasks_per_unit, arg % p.tasks_per_unit, wt);
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
