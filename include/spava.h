/*
 * spava.h -- C ABI of the B200 (sm_100a) approximate-attention prefill of
 * Spava / APB-V ("Accelerating Long-Video Understanding via
 * Sequence-Parallelism-aware Approximate Attention", arXiv 2601.21444), with all
 * hosts virtual on one GPU.
 *
 * The method (APB-V technical summary, "Methodology", 1. Framework design):
 * N visual tokens are split into H contiguous context blocks, one per host;
 * the first A tokens form the anchor block; every host scores its local keys
 * with query-to-context attention scores and keeps the best P per KV head as
 * its passing block; host h's queries attend to
 *     [anchor | passing blocks of hosts 0..h-1 | own block, causal];
 * a trailing text (query) segment of T tokens attends densely and causally, and
 * its partial results over the host blocks are merged through their lse
 * (2. System optimisations, "Fused context and query forward").  One host is
 * plain dense causal attention ("Limitations").
 *
 * Readings where the pages give no formula (plan-level constants):
 *   score(g, j) = max over the last R query rows i >= j of the host of key j and
 *                 over the query heads c of KV group g of (q_{i,c} . k_{j,g}) * scale;
 *   host 0's anchor tokens are not passing candidates;
 *   selection ties go to the lower token index, -0.0 == +0.0, indices ascending;
 *   GQA: query head c uses KV head c / (hq / hkv).
 *
 * Conventions for every entry point below.
 *   Layouts   q [N+T][hq][d], k and v [N+T][hkv][d], o [N+T][hq][d]: bf16,
 *             d contiguous, visual tokens first, then the T text tokens.
 *             lse [hq][N+T] fp32, natural log.  scores [hkv][N] fp32.
 *             idx [H-1][hkv][P] int32, token ids ascending per (host, KV head).
 *             k_pass, v_pass [hkv][H-1][P][d] bf16 (host-major inside a KV head,
 *             so hosts 0..h-1 of one KV head are one contiguous run).
 *             With SPAVA_SCORE_PER_QUERY_HEAD (spava_plan_set_score_reduce) the
 *             hkv of scores, idx and k_pass / v_pass becomes hq: one selection
 *             row per query head.
 *   Pointers  all tensor pointers are DEVICE pointers owned by the caller, 16-byte
 *             aligned; the workspace is 256-byte aligned and at least
 *             spava_workspace_bytes(plan) bytes.  Outputs must not alias inputs.
 *   Streams   `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *             stream).  Every call only enqueues work: it never synchronises and
 *             never allocates device memory.  Calls that share one workspace must
 *             not overlap in time.
 *   Errors    argument errors are detected on the host before anything is
 *             enqueued and return SPAVA_ERR_INVALID_ARG / SPAVA_ERR_UNSUPPORTED;
 *             spava_last_error() gives a one-line reason (thread-local).  Device
 *             waits inside the kernels are bounded: a wait that runs out sets an
 *             error word in the workspace and the kernel returns;
 *             spava_check_device_error() synchronises the stream, reads that word
 *             and returns SPAVA_ERR_TIMEOUT (or SPAVA_ERR_DEVICE_CHECK for a failed
 *             range check) if it is set, then clears it.
 */
#ifndef SPAVA_H_
#define SPAVA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  SPAVA_OK = 0,
  SPAVA_ERR_INVALID_ARG = 1,  /* bad size, pointer, alignment or combination */
  SPAVA_ERR_UNSUPPORTED = 2,  /* valid but outside what the kernels handle    */
  SPAVA_ERR_CUDA = 3,         /* a CUDA runtime/driver call failed            */
  SPAVA_ERR_TIMEOUT = 4,      /* a bounded device wait ran out                */
  SPAVA_ERR_DEVICE_CHECK = 5  /* a device-side range check failed; the access
                                 it guarded was skipped (none faulted)         */
} spava_status;

/* Flags of spava_score_select. */
#define SPAVA_SCORES_GIVEN 1u /* skip scoring: select from the caller's scores */

/* Opaque host-side plan: sizes, host block offsets and the cost-sorted work lists
 * of the attention kernel (uploaded once to a small device table owned by the
 * plan). */
typedef struct spava_plan spava_plan;

/*
 * Build a plan (context splitting: APB-V technical summary, 1. Framework design).
 *   n_visual     N >= 1 visual tokens; n_text T >= 0 trailing text tokens.
 *   n_hosts      H >= 1 virtual hosts.
 *   host_sizes   HOST pointer to H block sizes summing to N, or NULL for an equal
 *                split (then N % H must be 0).  Copied; the caller keeps ownership.
 *   anchor       A: tokens [0, A) form the anchor block (0 <= A; H > 1 needs
 *                A + P <= B_0).
 *   passing      P: passing keys per host and KV head (P <= B_h for h < H-1).
 *   probe_r      R: probe queries per host, 16 <= R <= min B_h, R % 16 == 0.
 *   hq, hkv      query / KV heads, hq % hkv == 0, hq / hkv <= 16.
 *   head_dim     d in {64, 128}.
 *   softmax_scale  <= 0 selects 1/sqrt(d).
 * Needs a current CUDA device (it uploads the plan's device table there).
 * Returns SPAVA_ERR_INVALID_ARG / _UNSUPPORTED before touching the device when the
 * sizes are not acceptable.  Release with spava_plan_destroy.
 */
spava_status spava_plan_create(spava_plan** out, int32_t n_visual, int32_t n_text,
                               int32_t n_hosts, const int32_t* host_sizes,
                               int32_t anchor, int32_t passing, int32_t probe_r,
                               int32_t hq, int32_t hkv, int32_t head_dim,
                               float softmax_scale);

/* Free a plan and its device table (synchronises the device first).  NULL is OK. */
spava_status spava_plan_destroy(spava_plan* plan);

/* How the query heads of a KV group combine into one score per key.  The pages say
 * only that hosts pick their passing keys by query-to-context attention scores (APB-V
 * technical summary, 1. Framework design, "Approximate attention mechanism"); with
 * m_c(j) = max over the probe rows i >= j of q_{i,c} . k_j (query head c):
 *   SPAVA_SCORE_MAX   score(g, j) = scale * max_c m_c(j)          (default)
 *   SPAVA_SCORE_SUM   score(g, j) = scale * sum_c m_c(j)
 *   SPAVA_SCORE_MEAN  score(g, j) = scale * sum_c m_c(j) / G
 * over the G query heads c of KV head g, or
 *   SPAVA_SCORE_PER_QUERY_HEAD  no reduction: score(c, j) = scale * m_c(j) for every
 *                     query head c, each query head selects its own P passing keys
 *                     (from KV head c / G) and attends through them.
 * "Selection rows" below are the hkv KV heads, or the hq query heads in the last mode:
 * scores [rows, N], indices [H-1, rows, P], passing K/V [rows, H-1, P, d]. */
typedef enum {
  SPAVA_SCORE_MAX = 0,
  SPAVA_SCORE_SUM = 1,
  SPAVA_SCORE_MEAN = 2,
  SPAVA_SCORE_PER_QUERY_HEAD = 3
} spava_score_reduce;

/* Select the head reduction (spava_score_reduce) for this plan's later calls
 * (spava_score_select, spava_gather_passing, spava_attn_prefill and its variants).
 * Host-side only.  It sets the number of selection rows, so query
 * spava_workspace_bytes / spava_two_stage_workspace_bytes after it.  Returns
 * SPAVA_ERR_INVALID_ARG for a NULL plan or an unknown mode. */
spava_status spava_plan_set_score_reduce(spava_plan* plan, int32_t mode);

/* What a probe row contributes to a key's score (the same passage leaves it open
 * whether the attention scores are the logits or the attention weights):
 *   SPAVA_SCORE_LOGIT  q_{i,c} . k_j (scaled), as above               (default)
 *   SPAVA_SCORE_PROB   exp(scale * q_{i,c} . k_j - lse_c(i)): the probe row's
 *                      attention probability over the keys of its own host block
 *                      it sees (lse_c(i) = log sum over keys j' <= i of the block of
 *                      exp(scale * q_{i,c} . k_j'), computed by the attention kernel
 *                      over the probe rows first); m_c(j) is the max of these over
 *                      the probe rows, then the head reduction applies as above.
 * The two-stage flow scores with the score kernel in this mode (the final lse of a
 * probe row is not known inside the local pass). */
typedef enum { SPAVA_SCORE_LOGIT = 0, SPAVA_SCORE_PROB = 1 } spava_score_kind;

/* Select the score kind (spava_score_kind) for this plan's later calls.  Host-side
 * only; probability scores add an [hq][N] fp32 buffer to both workspaces, so query
 * the workspace sizes after it.  Returns SPAVA_ERR_INVALID_ARG for a NULL plan or an
 * unknown kind. */
spava_status spava_plan_set_score_kind(spava_plan* plan, int32_t kind);

/* How spava_attn_prefill (and spava_attn_prefill_noalloc) produce the passing K/V.
 * enable == 0 (default): the score kernel, then the select + gather kernel.
 * enable != 0: with the max head reduction over logit scores, scoring, selection and
 * gather run as one persistent cooperative launch -- score tiles dealt to the SMs in
 * rounds, each (host, KV head)'s selection started as soon as its last score tile is
 * stored, its gather shared out over all SMs while later units are still scored.
 * Plans outside that case run the two kernels either way.  Both give the same scores,
 * indices and passing K/V (bit for bit); on B200 the two-kernel form is the faster
 * one at the workloads measured, hence the default.  Host-side only;
 * SPAVA_ERR_INVALID_ARG for a NULL plan. */
spava_status spava_plan_set_fused_select(spava_plan* plan, int32_t enable);

/* Bytes of scratch the calls below need (scores, indices, passing K/V, text
 * partials, scheduler counters, error word).  0 if plan is NULL. */
size_t spava_workspace_bytes(const spava_plan* plan);

/* Host block offsets (HOST array of H+1 ints) and work-list statistics, for
 * callers that want the plan's view of the split.  Returns H, or -1. */
int32_t spava_plan_offsets(const spava_plan* plan, int32_t* offsets_out /* H+1 or NULL */);

/*
 * Query-to-context scoring and passing-block selection (APB-V technical summary,
 * 1. Framework design, "Approximate attention mechanism": passing blocks hold the
 * most essential key-value pairs, picked by query-to-context attention scores).
 *   q, k        device bf16, layouts above.
 *   scores      device fp32 [hkv][N]: written (every host's keys), or read when
 *               flags & SPAVA_SCORES_GIVEN.
 *   idx         device int32 [H-1][hkv][P]: the P best candidates of each host
 *               h < H-1 and KV head, ties to the lower index, ascending.
 *   flags       0 or SPAVA_SCORES_GIVEN.
 *   ws          device workspace.
 */
spava_status spava_score_select(const spava_plan* plan, const void* q, const void* k,
                                float* scores, int32_t* idx, uint32_t flags,
                                void* ws, void* stream);

/*
 * Passing ("sending passing blocks to later hosts", 2. System optimisations,
 * "Overlapped communication"): on one GPU every pass is an on-device gather
 *   k_pass[g][h][j][:] = k[idx[h][g][j]][g][:], and the same for v.
 *   k, v     device bf16 [N+T][hkv][d];  idx device int32 [H-1][hkv][P].
 *   k_pass, v_pass  device bf16 [hkv][H-1][P][d].
 * Indices outside [0, N) are not checked on the device: callers pass the output of
 * spava_score_select.
 */
spava_status spava_gather_passing(const spava_plan* plan, const void* k, const void* v,
                                  const int32_t* idx, void* k_pass, void* v_pass,
                                  void* stream);

/*
 * The whole approximate-attention prefill of one layer: scoring -> selection ->
 * gather (see spava_plan_set_fused_select) -> one flash-attention pass per host over
 * [anchor | passing of hosts < h | own block, causal] (tcgen05/TMEM, bf16 in, fp32
 * accumulation, online softmax) -> text rows as split-KV partials over the host
 * blocks merged through their lse.
 *   q, k, v    device bf16 inputs.
 *   o          device bf16 [N+T][hq][d] output.
 *   lse        device fp32 [hq][N+T] output (natural log).
 *   scores_out, idx_out  optional device buffers ([hkv][N] fp32, [H-1][hkv][P]
 *              int32): when not NULL the run uses them instead of the workspace,
 *              so the caller can read the scores and the selection back.
 */
spava_status spava_attn_prefill(const spava_plan* plan, const void* q, const void* k,
                                const void* v, void* o, float* lse, float* scores_out,
                                int32_t* idx_out, void* ws, void* stream);

/*
 * spava_attn_prefill without a workspace, for callers that cannot allocate device
 * memory at call time: frameworks whose device memory belongs to their own pooling
 * allocator and that forbid a library to call cudaMalloc (an allocation outside the
 * pool breaks its accounting, or fails outright under a hard memory cap), loops that
 * cannot absorb the device-wide synchronisation cudaMalloc/cudaFree may cause, and
 * interfaces that have no way to hand a scratch buffer to the library.  The paper
 * has no counterpart of this entry point; it only changes where the scratch lives.
 *
 * The scratch is one static device array of SPAVA_NOALLOC_SCRATCH_BYTES (32 MiB)
 * inside this library: every GPU on which the library's kernels are loaded holds it
 * until the process exits.  This call allocates nothing (no cudaMalloc, cudaFree or
 * allocating library routine); the inputs and outputs are the caller's, with the
 * layouts of spava_attn_prefill.  The plan must have been created beforehand
 * (spava_plan_create allocates its table once, at set-up).
 *   Address: every call looks up the array's device address on the current device
 *   (cudaGetSymbolAddress, a host-side lookup that enqueues nothing) and caches
 *   nothing, so a context torn down and re-created in the same process
 *   (cudaDeviceReset) gets the array's new address.  With lazy module loading the
 *   first lookup on a device loads the library's kernels there: make that first call
 *   before any stream capture.
 *   Sizes: returns SPAVA_ERR_UNSUPPORTED, before enqueueing anything, when
 *   spava_workspace_bytes(plan) exceeds SPAVA_NOALLOC_SCRATCH_BYTES.
 *   Sharing: every call on a device uses the same array, which keeps the previous
 *   call's contents (the call clears the part that must start at zero itself).  Calls
 *   that overlap on the GPU (other streams, threads or plans) race on it: serialise
 *   them.  The scores, selection and error word stay in the array; a bounded-wait
 *   timeout inside this call is therefore not reported (use spava_attn_prefill with a
 *   workspace and spava_check_device_error when that check is needed).
 */
#define SPAVA_NOALLOC_SCRATCH_BYTES (32u * 1024u * 1024u)
spava_status spava_attn_prefill_noalloc(const spava_plan* plan, const void* q, const void* k,
                                        const void* v, void* o, float* lse, void* stream);

/*
 * The same prefill in the two stages the pages describe (APB-V technical summary,
 * "Main contributions": two-stage attention; 1. Framework design: passing blocks
 * picked by query-to-context scores; 2. System optimisations: partial results merged
 * through FlashAttention's lse):
 *   stage 1  every host's queries over its own block, causal, on the attention
 *            kernel; the items that hold a host's last R query rows fold their raw
 *            q.k logits into the probe scores as they go (fused scoring: column
 *            maxima per warp, max over the group's query heads by atomic max on
 *            order-preserving integer keys); hosts with a remote part keep fp32
 *            partial O and lse of their rows;
 *   select + gather of the passing rows;
 *   stage 2  host h >= 1 over [anchor | passing of hosts < h], merged with its
 *            stage-1 partial through the lse into the final O and lse;
 *   text rows as in spava_attn_prefill.
 * Arguments and layouts as spava_attn_prefill; `ws` must hold
 * spava_two_stage_workspace_bytes(plan) bytes (it adds the fp32 row partials,
 * N * hq * d * 4 bytes).  Results equal spava_attn_prefill's up to fp32 rounding
 * order (the scores come from a different MMA, so selections may differ at exact
 * ties within rounding).  spava_attn_prefill is the faster flow on one GPU: it needs
 * no partials of the visual rows.
 */
spava_status spava_attn_prefill_two_stage(const spava_plan* plan, const void* q, const void* k,
                                          const void* v, void* o, float* lse, float* scores_out,
                                          int32_t* idx_out, void* ws, void* stream);

/* Workspace bytes of spava_attn_prefill_two_stage (0 if plan is NULL). */
size_t spava_two_stage_workspace_bytes(const spava_plan* plan);

/*
 * Dense causal attention over all N+T tokens on the same kernel (the standard
 * FlashAttention the method degenerates to on one host; the comparison kernel).
 * Layouts as above.
 */
spava_status spava_dense_causal(const spava_plan* plan, const void* q, const void* k,
                                const void* v, void* o, float* lse, void* ws, void* stream);

/*
 * Sharded prefill: the host blocks spread over `world` ranks, one process per GPU,
 * each rank running the work of its own hosts (APB-V technical summary, 1. Framework
 * design, "Context splitting & ZigZag arrangement": a physical host runs a pair of
 * virtual hosts; 2. System optimisations, "Overlapped communication": passing blocks
 * and partial query results travel while attention runs).  The library computes; the
 * caller moves bytes between the ranks between the stages (an all-gather of each
 * exchange buffer, a broadcast of the anchor rows), on a stream of its own so that
 * the transfers overlap the next stage.
 *
 * Ownership policies (spava_shard_owners):
 *   SPAVA_SHARD_CONTIGUOUS  rank r runs hosts [r*H/world, (r+1)*H/world).
 *   SPAVA_SHARD_ZIGZAG      the hosts form rounds of 2*world; in each round rank r runs
 *                           hosts r and 2*world-1-r (a later host attends to more
 *                           passing rows, so the pairs carry equal passing lengths).
 *   SPAVA_SHARD_LONGEST_FIRST  (spava_plan_shard_owners only) hosts by decreasing
 *                           cost, each to the rank with the least cost so far (ties to
 *                           the lower host, then the lower rank); a host's cost is the
 *                           (query, key) pairs its rows and its text piece attend:
 *                           B(B+1)/2 + B(A + hP) for h >= 1, + T B, and T(T+1)/2 more
 *                           for the last host (the text rows' causal part).  The one-GPU
 *                           scheduler's longest-first rule applied to whole hosts; it
 *                           balances uneven blocks, which the pairing does not.
 */
typedef enum {
  SPAVA_SHARD_CONTIGUOUS = 0,
  SPAVA_SHARD_ZIGZAG = 1,
  SPAVA_SHARD_LONGEST_FIRST = 2
} spava_shard_policy;

/* Host-side only (no device needed): owner_out[h] = the rank that runs host h, for a
 * HOST array of n_hosts ints.  CONTIGUOUS needs n_hosts % world == 0, ZIGZAG
 * n_hosts % (2 * world) == 0; otherwise, or for a NULL array or world < 1, returns
 * SPAVA_ERR_INVALID_ARG and writes nothing. */
spava_status spava_shard_owners(int32_t n_hosts, int32_t world, int32_t policy, int32_t* owner_out);

/* Longest-first assignment of n_hosts hosts with the given costs (HOST array of
 * n_hosts int64 >= 0) to `world` ranks, into owner_out (HOST array).  Host-side only.
 * SPAVA_ERR_INVALID_ARG for NULL arrays, n_hosts < 1, world < 1 or a negative cost. */
spava_status spava_shard_owners_by_cost(int32_t n_hosts, int32_t world, const int64_t* cost,
                                        int32_t* owner_out);

/* Ownership for this plan's host sizes: CONTIGUOUS and ZIGZAG as spava_shard_owners,
 * LONGEST_FIRST from the plan's per-host costs above (any H >= 1, world >= 1).
 * Host-side only; owner_out is a HOST array of H ints.  SPAVA_ERR_INVALID_ARG as
 * above. */
spava_status spava_plan_shard_owners(const spava_plan* plan, int32_t world, int32_t policy, int32_t* owner_out);

/* Make `plan` run rank `rank` of `world`, host h on rank owner[h] (HOST array of H
 * ints in [0, world), copied; every rank of a job passes the same array).  Builds this
 * rank's work lists into a device table owned by the plan (synchronises the device
 * when it replaces an earlier one) and sizes the sharded workspace; query the layout
 * afterwards, and again after spava_plan_set_score_reduce / _kind.  Returns
 * SPAVA_ERR_INVALID_ARG for a bad rank, world or owner entry. */
spava_status spava_plan_set_shard(spava_plan* plan, int32_t rank, int32_t world, const int32_t* owner);

/* Workspace layout of the sharded prefill (byte offsets into the workspace).
 *   pass_k / pass_v   passing exchange buffers, bf16 [world][pass_slots][P][rows][d]
 *                     (rows = selection rows): slot s of rank r holds the passing rows
 *                     of rank r's s-th own host < H-1 (ascending), row j of selection
 *                     row g at [r][s][j][g].  Rank r's part is the contiguous run
 *                     [r * pass_bytes_per_rank, (r+1) * pass_bytes_per_rank).
 *   text_o / text_lse text partial exchange buffers, fp32 [world][text_slots][T][hq][d]
 *                     and [world][text_slots][hq][T]: slot s of rank r is its s-th text
 *                     piece (the text rows over each own host's block, ascending, then
 *                     on the owner of host H-1 the text rows' own causal part); unused
 *                     slots hold O = 0, lse = -inf.  Parts per rank as above.
 *   scores, idx       this rank's scores [rows][N] and selection [H-1][rows][P] (the
 *                     entries of its own hosts < H-1 are written).
 */
typedef struct {
  uint64_t workspace_bytes;
  uint64_t pass_k_offset, pass_v_offset, pass_bytes_per_rank;
  uint64_t text_o_offset, text_o_bytes_per_rank;
  uint64_t text_lse_offset, text_lse_bytes_per_rank;
  uint64_t scores_offset, idx_offset;
  int32_t pass_slots, text_slots;
} spava_shard_layout;

/* Fill *out for a plan after spava_plan_set_shard; SPAVA_ERR_INVALID_ARG otherwise. */
spava_status spava_shard_query(const spava_plan* plan, spava_shard_layout* out);

/* Stages of the sharded prefill, run in this order on every rank:
 *   SPAVA_SHARD_SELECT  score the own hosts < H-1 (score kernel), select their top P
 *                       and write the passing rows into this rank's part of pass_k /
 *                       pass_v.  Reads the probe rows of q and the own blocks of k, v.
 *                       Clears the workspace error word.
 *     caller: all-gather pass_k and pass_v; broadcast k, v rows [0, A) from the owner
 *     of host 0 into every rank's k, v (both may overlap LOCAL).
 *   SPAVA_SHARD_LOCAL   own hosts' rows over their own block (causal): final O/lse for
 *                       hosts without a remote part (host 0), fp32 row partials for the
 *                       others; the text rows over each own block into this rank's
 *                       text slots.  Reads own rows of q, k, v and the text rows of q
 *                       (and of k, v on the owner of host H-1).
 *     caller: all-gather text_o and text_lse (may overlap REMOTE).
 *   SPAVA_SHARD_REMOTE  own hosts h >= 1 over [anchor | passing of hosts < h], merged
 *                       with their row partials into the final O/lse of their rows.
 *                       Needs the gathered pass_k / pass_v and the anchor rows.
 *   SPAVA_SHARD_MERGE   text rows from all ranks' text slots (needs the gathered
 *                       text_o / text_lse): final O/lse of rows [N, N+T).
 * One-pass form: SELECT, the passing exchange and the anchor broadcast (waited for),
 * then SPAVA_SHARD_ATTEND in place of LOCAL + REMOTE -- own hosts' rows in one pass
 * over [anchor | passing of hosts < h | own block, causal] (final O/lse, no row
 * partials) and the text pieces into this rank's slots -- then the text exchange and
 * MERGE.  It gives up overlapping the passing exchange with the local pass and saves
 * the fp32 row partials and the second online softmax.
 * q, k, v, o [N+T][heads][d] bf16 and lse [hq][N+T] are full-size device buffers with
 * the layouts above.  Rows a rank does not own are not written and do not change the
 * result, but they must hold finite values (zeros will do): a 128-row tile can load
 * rows past the end of a block, which then take part with weight exactly 0.  `ws`
 * holds spava_shard_layout.workspace_bytes.  Together the four stages over all
 * ranks compute spava_attn_prefill_two_stage's result with the score kernel's
 * scores (spava_attn_prefill's selection). */
typedef enum {
  SPAVA_SHARD_SELECT = 0,
  SPAVA_SHARD_LOCAL = 1,
  SPAVA_SHARD_REMOTE = 2,
  SPAVA_SHARD_MERGE = 3,
  SPAVA_SHARD_ATTEND = 4
} spava_shard_stage_id;

spava_status spava_shard_stage(const spava_plan* plan, int32_t stage, const void* q, const void* k,
                               const void* v, void* o, float* lse, void* ws, void* stream);

/* Synchronise `stream`, read the workspace error word, clear it.  Returns SPAVA_OK,
 * SPAVA_ERR_TIMEOUT (a bounded device wait ran out), SPAVA_ERR_DEVICE_CHECK (a
 * selection position or gather index of the one-launch score/select/gather form fell
 * outside its range and was skipped; the passing K/V are then incomplete) or
 * SPAVA_ERR_CUDA; spava_last_error() names the error bits. */
spava_status spava_check_device_error(const spava_plan* plan, void* ws, void* stream);

/* Testing aid: the next kernel launches of this plan use a device wait limit of
 * `ns` nanoseconds (0 restores the default of 2 s), and with `stall_producer` != 0
 * the attention kernel's load warp issues nothing, so every consumer wait runs out
 * and the kernel returns with SPAVA_ERR_TIMEOUT recorded.  Never faults or hangs. */
spava_status spava_plan_set_debug(spava_plan* plan, uint64_t wait_limit_ns, int32_t stall_producer);

/*
 * Kernel timing hook (for benchmarks).  After spava_profile_begin(plan, max_marks)
 * every entry point of this plan records a CUDA event on its stream before each
 * kernel it launches and one after the last; spava_profile_read synchronises the
 * plan's device, writes for each recorded kernel its label (see
 * spava_kernel_name) and its duration in ms, returns how many it wrote (at most
 * `max`, -1 on error) and starts a new recording.  Recording stops silently once
 * max_marks events are used.  spava_profile_end releases the events.
 */
spava_status spava_profile_begin(spava_plan* plan, int32_t max_marks);
int32_t spava_profile_read(spava_plan* plan, int32_t* labels, float* ms, int32_t max);
spava_status spava_profile_end(spava_plan* plan);

/* Name of a kernel label: 0 score, 1 select, 2 gather, 3 attention (prefill),
 * 4 lse merge, 5 attention (dense causal), 6 select + gather (fused, prefill),
 * 7 score-key fill/convert (two-stage), 8 attention stage 1, 9 attention stage 2,
 * 10 probe-row lse (probability scores), 11 passing unpack (sharded prefill),
 * 12 spare text-slot fill (sharded prefill), 13 score + select + gather (one launch,
 * prefill). */
const char* spava_kernel_name(int32_t label);

/*
 * The linear maps around the attention of one decoder layer, for a multi-layer
 * prefill (the pages report time to first token: APB-V technical summary,
 * "Experimental results"; their fused forward of context and query runs every token
 * of the layer through the same projections, 2. System optimisations, "Fused context
 * and query forward").  Both run a tcgen05 GEMM (TMA-fed, TMEM accumulators, 128 x
 * 256 output tiles, persistent over the SMs) with a fused epilogue.  Pointers are
 * device pointers owned by the caller; bf16 tensors are row-major with the last
 * dimension contiguous; all must be 16-byte aligned.  Calls are asynchronous on
 * `stream` and allocate nothing.
 *
 * spava_layer_workspace_bytes(n_tokens): bytes of the caller's workspace `ws`
 * (256-byte aligned) that both calls of a layer use: a device error word and the
 * rows' RMS factors.  Returns 0 for n_tokens < 0.
 *
 * spava_qkv_projection: RMSNorm + QKV projection.
 *   x      [n_tokens][hidden] bf16, the layer's input hidden states;
 *   w_qkv  [(hq + 2 hkv) head_dim][hidden] bf16: the query, key and value weights
 *          stacked row-wise (row j of the stack produces output feature j);
 *   q      [n_tokens][hq][head_dim], k and v [n_tokens][hkv][head_dim] bf16 (the
 *          layouts spava_attn_prefill reads), written:
 *            y = (x / rms(x)) W_qkv^T,  rms(x_m) = sqrt(mean_j x_mj^2 + rms_eps),
 *          columns [0, hq d) of y into q, [hq d, (hq + hkv) d) into k, the rest into v.
 *   The row scale 1 / rms is applied to the fp32 accumulator (the normalised x is
 *   never stored); outputs are rounded to bf16 (RNE).  Clears the workspace error word.
 *   Errors: SPAVA_ERR_INVALID_ARG for NULL or misaligned pointers, non-positive sizes,
 *   hq % hkv != 0 or rms_eps <= 0; SPAVA_ERR_UNSUPPORTED unless hidden, hq head_dim
 *   and hkv head_dim are multiples of 256 or when the device is not sm_100.
 *
 * spava_out_projection: output projection + residual, in place:
 *   x[m][:] += o[m][:] W_o^T,  o [n_tokens][in_features] bf16 (the attention output,
 *   [n_tokens][hq][head_dim] read as rows of hq head_dim), w_o [hidden][in_features]
 *   bf16, x [n_tokens][hidden] bf16 (read, then overwritten with the rounded sum).
 *   Errors as above; in_features and hidden must be multiples of 256.
 *
 * spava_layer_check_error: synchronise `stream`, read and clear the workspace error
 *   word; SPAVA_ERR_TIMEOUT if a bounded device wait of either call ran out.
 */
size_t spava_layer_workspace_bytes(int32_t n_tokens);
spava_status spava_qkv_projection(const void* x, int32_t n_tokens, int32_t hidden, const void* w_qkv, int32_t hq,
                                  int32_t hkv, int32_t head_dim, float rms_eps, void* q, void* k, void* v, void* ws,
                                  void* stream);
spava_status spava_out_projection(const void* o, int32_t n_tokens, int32_t in_features, const void* w_o,
                                  int32_t hidden, void* x, void* ws, void* stream);
spava_status spava_layer_check_error(void* ws, void* stream);

/* Static text of a status code. */
const char* spava_status_string(spava_status status);

/* One-line reason for the last non-OK status returned on this thread ("" if none). */
const char* spava_last_error(void);

/* Kernel launches enqueued by the last successful call on this thread (for
 * accounting of launches in benchmarks). */
int32_t spava_last_launch_count(void);

#ifdef __cplusplus
}
#endif

#endif /* SPAVA_H_ */
