/*
 * zb.h -- C ABI of libzb: load-balanced MoE token dispatch and combine on
 * B200 (sm_100a) across P expert-parallel ranks: virtual ranks whose buffers
 * partition one device memory (zb_plan, zb_dispatch, zb_combine), or one rank
 * per GPU, each holding its own tokens (zb_count, zb_plan_rank,
 * zb_dispatch_rank, zb_combine_rank).
 *
 * One invocation is five steps, in order:
 *   1. per-rank, per-expert histogram of the top-K routing ids        (zb_plan)
 *   2. greedy hot-expert replica planner down to the water level T    (zb_plan)
 *   3. locality-first assignment of every (token,k), cu_seqlens       (zb_plan)
 *   4. scatter of bf16 token rows into expert-grouped S*K buffers     (zb_dispatch)
 *   5. gate-weighted combine gather, fp32 accumulation in k order     (zb_combine)
 *
 * Conventions for every entry point:
 *  - Every pointer argument is DEVICE memory owned by the caller, except
 *    `cfg`, the `plan` and `merge` structs themselves, the host out-parameters
 *    of zb_plan_status and zb_recalibrate, the host arrays of zb_place_by_demand,
 *    and the host tables of per-rank device pointers taken by
 *    zb_dispatch_rank and zb_combine_rank.  The library allocates nothing and
 *    keeps no state between calls (zb_plan_noalloc's fixed scratch array is
 *    the one exception, described there).
 *  - `stream` is a cudaStream_t passed as void* (NULL = the legacy default
 *    stream).  Every call except zb_plan_status only enqueues work on it and
 *    returns without synchronising.
 *  - Layouts are dense row-major, C order, no padding.  bf16 arrays are passed
 *    as uint16_t bit patterns.  Rows and tensors must be 16-byte aligned
 *    (H % 8 == 0 and 16-byte aligned base pointers).
 *  - Return value: ZB_OK (0), a positive warning, or a negative error.  A call
 *    that returns an error has enqueued nothing.  Errors that only the device
 *    can see (bad ids, capacity) are recorded in plan->stats and reported by
 *    zb_plan_status; dispatch and combine launched on such a plan do nothing.
 *
 * Notation: i = source rank, j = destination rank, e = expert, Eh = E/P home
 * experts per rank (expert e lives on rank home(e) = e / Eh), f = s*K + k the
 * flat index of an entry inside its source rank, g = i*S*K + f the global
 * entry index, cap = cfg->cap_rows.
 */
#ifndef ZB_H
#define ZB_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define ZB_API __attribute__((visibility("default")))
#else
#define ZB_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* ------------------------------------------------------------ status codes */
#define ZB_OK 0
#define ZB_WARN_UNBALANCED 1 /* R slots did not permit T: some rank ends above T */
#define ZB_ERR_INVALID (-1)  /* bad configuration, pointer, size or alignment */
#define ZB_ERR_CAPACITY (-2) /* planned max rank load > cap_rows */
#define ZB_ERR_BAD_ID (-3)   /* a routing id outside [0, E) */
#define ZB_ERR_TIMEOUT (-4)  /* reserved: a bounded device wait gave up */
#define ZB_ERR_CUDA (-5)     /* a CUDA runtime call failed */

/* Problem shape.
 *   P   ranks, 1..32          E  experts, P..384, E % P == 0
 *   K   top-K, 1..16          S  tokens per rank, >= 0
 *   H   hidden width in bf16 elements, H >= 8, H % 8 == 0
 *   R   replica (helper) slots per rank, 0..P-1
 *   C   relaxation ratio of the routing constraint |sum_i M_ij - q_j| <= C q_j
 *       of eq. (1) (Zepp, 4.1 Expert Placement and Token Routing), 0 <= C < 1;
 *       used only when relax = 1
 *   gpus_per_node  1 = flat locality cost; g > 1 groups ranks into nodes of g
 *       consecutive ranks (P % g == 0)
 *   cap_rows  rows of each rank's receive buffer, >= S*K; P*cap_rows and
 *       P*S*K must fit in int32
 *   policy  receiver choice of the greedy planner:
 *       ZB_POLICY_ROOM (0): among eligible ranks, the one whose node does not
 *         yet hold the expert, then the lowest load, then the lowest rank;
 *       ZB_POLICY_LOCAL (1): balance first, locality among equal moves:
 *         after node coverage, the rank that takes the most rows m_r (the
 *         move's balance progress), then the rank whose own rows for the
 *         expert the copy would serve locally are most, min(cnt[r][e], m_r),
 *         then the lowest load, then the lowest rank (ISER-MoE, HALO-Q
 *         Objective 2: the most locally computed tokens among balanced
 *         routings).
 *   relax   0: every host of an expert receives exactly its quota q (the
 *         default; fixed S*K buffers leave no slack).  1: each host receives
 *         between q - dl and q + dl rows, dl = floor(q * floor(C * 2^20) / 2^20),
 *         so more rows are served on their own rank: own-rank rows up to
 *         q - dl, then more own-rank rows in ascending host rank while the band's
 *         total slack (sum of dl) lasts, then the other ranks by cost level.
 *         When the quota loads reach T, a rank receives at most
 *         T + floor(T * floor(C * 2^20) / 2^20) = floor((1+C) T) rows; size
 *         cap_rows for that (a plan needing more is ZB_ERR_CAPACITY).
 *   repair  1: after the greedy (or the kept placement's quotas), quota
 *         repair between rank pairs (ISER-MoE, HALO-Q stage 4).  Ranks i and
 *         j that both hold experts e and e' cancel opposite flows: where i's
 *         own rows of e exceed its quota (surplus) and j's quota of e exceeds
 *         j's own rows (spare), and the reverse holds for e', m rows of quota
 *         of e move from j to i and m of e' from i to j.  Both loads are
 *         unchanged; 2m more rows are served on their own rank.  Per pair,
 *         m = min(sum_e min(surplus_i, spare_j), sum_e min(surplus_j, spare_i)),
 *         consumed in ascending expert order.  Pairs come from the circle
 *         method over P rounded up to even (a bye for odd P), one round after
 *         another.  Filled slots may end with quota 0.  0: no repair. */
#define ZB_POLICY_ROOM 0
#define ZB_POLICY_LOCAL 1
typedef struct zb_config {
  int P, E, K, S, H, R;
  float C;
  int gpus_per_node;
  int cap_rows;
  int policy;
  int relax;
  int repair;
} zb_config;

/* Indices into plan->stats (int64). */
#define ZB_STAT_STATUS 0        /* final status of the plan (a ZB_* code) */
#define ZB_STAT_MAX_LOAD 1      /* max_j load_after[j] */
#define ZB_STAT_N_REPLICAS 2    /* filled helper slots */
#define ZB_STAT_N_ITERS 3       /* greedy iterations taken */
#define ZB_STAT_WATER_LEVEL 4   /* T = ceil(sum_r L_r / P) */
#define ZB_STAT_LOCALITY_COST 5 /* sum_{e,i,j} a_ij M^e_ij */
#define ZB_STAT_BAD_IDS 6       /* count of ids outside [0, E) */
#define ZB_STAT_REPAIRED 7      /* rows moved by quota repair, per direction */
#define ZB_STATS_LEN 8

/* The plan: caller-allocated device buffers that zb_plan fills and
 * zb_dispatch / zb_combine read.  Shapes (int32 unless stated):
 *   cnt         [P][E]        cnt[i][e] = #{(s,k): ids[i,s,k] = e}
 *   rep_expert  [P][R]        expert held by helper slot (j, r), -1 = empty
 *   rep_quota   [P][R]        rows that slot receives (0 if empty; with
 *                             repair, a filled slot may also have 0)
 *   home_quota  [E]           rows the home copy of e receives
 *   load_before [P]           L_j = rows homed on j before planning
 *   load_after  [P]           rows rank j receives after planning (its
 *                             quota load; with relax, within the band)
 *   cu_seqlens  [P][Eh+R+1]   exclusive prefix of the rows of rank j's groups:
 *                             groups 0..Eh-1 are its home experts j*Eh+g,
 *                             groups Eh..Eh+R-1 its helper slots 0..R-1
 *   dst_row     [P][S][K]     j*cap + row of each entry in the receive buffers
 *   row_src     [P][cap]      inverse of dst_row: g, or -1 for an unused row;
 *                             OPTIONAL, may be NULL (then not written)
 *   stats       int64 [ZB_STATS_LEN], see ZB_STAT_*
 *   trace       uint64 [ZB_TRACE_LEN]  device clock stamps of the plan's
 *                             kernels, see ZB_TRACE_*; OPTIONAL, may be NULL
 *                             (then not written) */
typedef struct zb_plan_t {
  int32_t *cnt;
  int32_t *rep_expert;
  int32_t *rep_quota;
  int32_t *home_quota;
  int32_t *load_before;
  int32_t *load_after;
  int32_t *cu_seqlens;
  int32_t *dst_row;
  int32_t *row_src;
  int64_t *stats;
  uint64_t *trace;
} zb_plan_t;

/* plan->trace, when not NULL: per kernel of the plan, three %globaltimer
 * stamps (ns): the first of its CTAs to start, the first released by its
 * wait on the kernel before it (k_zero has no wait: a second start stamp), and
 * the last to finish.  The plan call resets them first (one more small
 * launch on the stream); a kernel the call does not run (k_zero and k_hist
 * in zb_plan_rank) keeps UINT64_MAX, UINT64_MAX, 0.  Kernels overlap under
 * programmatic dependent launch, so a kernel may start before the one
 * before it ends; its release stamp is when it could read that kernel's
 * results. */
#define ZB_TRACE_ZERO 0    /* k_zero: zeroes the per-source totals */
#define ZB_TRACE_HIST 3    /* k_hist: histograms; waits on k_zero to add its totals */
#define ZB_TRACE_PLANNER 6 /* k_planner: waits on k_hist */
#define ZB_TRACE_ASSIGN 9  /* k_assign: waits on k_planner */
#define ZB_TRACE_LEN 12

/* Text of a status code (static storage; never NULL). */
ZB_API const char *zb_strerror(int status);

/* ZB_OK if `cfg` satisfies every bound listed at zb_config, else
 * ZB_ERR_INVALID.  Host only; touches no device. */
ZB_API int zb_validate(const zb_config *cfg);

/* Bytes of device scratch memory zb_plan needs for `cfg` (0 if `cfg` is
 * invalid).  Host only.  The workspace holds the per-chunk histograms, the
 * per-source totals, the first segment of each expert and the per-(source,
 * expert) segment table; its contents need not be initialised and are dead
 * after the plan's kernels complete. */
ZB_API size_t zb_workspace_bytes(const zb_config *cfg);

/* Steps 1-3: histogram, greedy replica plan, assignment.
 *
 * Steps, after the pages:
 *  - count routes per rank and expert (ISER-MoE, Methodology, HALO-Q
 *    Scheduler, stage 1, where ranks share these counts);
 *  - water level T = ceil(sum_r L_r / P) (ISER-MoE, HALO-Q Objective 1); since
 *    every entry routes exactly once, T = S*K, MoonEP's per-rank S x K
 *    invariant ("What MoonEP enforces and how");
 *  - greedy placement: while the busiest rank d (ties: lowest rank) is above T,
 *    it offers its heaviest home expert (largest remaining home quota, ties:
 *    lowest expert) for which an eligible receiver exists; eligible = another
 *    rank with a free slot, load below T and no copy of the expert; the
 *    receiver is chosen by cfg->policy (see zb_config): by default the one
 *    whose node does not yet hold the expert, then the lowest load, then the
 *    lowest rank (Zepp "4.1 Expert Placement and Token Routing": R extra
 *    slots per GPU, round-robin across nodes first); it takes
 *    m = min(load_d - T, T - load_r, quota_e) rows into its lowest free slot
 *    (HALO-Q stages 2-3).  A donor with no movable expert is marked stuck;
 *  - routing: expert e's rows are assigned to its hosts by eq. (1) of Zepp 4.1,
 *    minimising sum a_ij M^e_ij with each host receiving exactly its quota
 *    (a_ij = 0 same rank, 1 other rank; with nodes 1 same node, 4 other node):
 *    each host first serves its own rank, then per cost level, hosts in
 *    ascending rank take from sources in ascending rank (HALO-Q stage 5,
 *    the route rewrite that keeps rows local before moving them);
 *  - rows: source i walks its entries of expert e in flat order and fills its
 *    hosts in order of (a_ij, j); inside a group, rows are ordered by source
 *    rank, then flat index; cu_seqlens indexes the groups (MoonEP, section on
 *    what it enforces: the on-GPU planner hands kernels these offsets).
 *
 * topk_ids: device int32 [P][S][K].  plan: all required buffers as listed at
 * zb_plan_t.  workspace: device, zb_workspace_bytes(cfg) bytes (pass that
 * count as workspace_bytes), 256-byte aligned.
 * Returns ZB_OK once the work is enqueued, ZB_ERR_INVALID (bad cfg, NULL
 * buffer, short or misaligned workspace, a trace array not 8-byte aligned)
 * or ZB_ERR_CUDA.  The plan's own outcome (OK,
 * UNBALANCED, CAPACITY, BAD_ID) lands in plan->stats; read it with
 * zb_plan_status.  On CAPACITY or BAD_ID, dst_row and row_src are undefined. */
ZB_API int zb_plan(const zb_config *cfg, const int32_t *topk_ids, const zb_plan_t *plan,
            void *workspace, size_t workspace_bytes, void *stream);

/* Steps 1-3 with the replica placement given instead of chosen: the slots
 * of `placement` (device int32 [P][R], -1 = empty) are kept, and only their
 * quotas are planned, by the same greedy restricted to existing copies (a
 * receiver must already hold the expert; a move adds rows to that copy's
 * quota; receivers by most room, then lowest rank).  For plans that keep a
 * placement across invocations: Zepp "4.1 Expert Placement and Token
 * Routing" places replicas from historical demand, and ViBE re-places only
 * when the expert load has drifted.  `placement` may be the rep_expert of
 * the previous plan, and may alias plan->rep_expert.  A slot naming an
 * expert homed on its own rank, an id outside [0, E) or an expert twice on
 * one rank makes the plan's status ZB_ERR_INVALID (reported by
 * zb_plan_status; nothing else is written).  Other arguments, results and
 * errors as zb_plan; rep_expert receives the placement, rep_quota the
 * planned quotas (0 for copies that take no rows). */
ZB_API int zb_plan_placed(const zb_config *cfg, const int32_t *topk_ids, const int32_t *placement,
                          const zb_plan_t *plan, void *workspace, size_t workspace_bytes,
                          void *stream);

/* Synchronises `stream`, then returns the plan's status (ZB_OK,
 * ZB_WARN_UNBALANCED, ZB_ERR_CAPACITY, ZB_ERR_BAD_ID, or ZB_ERR_INVALID for
 * a bad placement given to zb_plan_placed), or ZB_ERR_CUDA.
 * If max_load is not NULL it receives the planned max rank load (host int). */
ZB_API int zb_plan_status(const zb_config *cfg, const zb_plan_t *plan, void *stream,
                   int32_t *max_load);

/* Size of the scratch array behind zb_plan_noalloc: 4 MiB.  A config is
 * accepted there only if zb_workspace_bytes(cfg) <= this. */
#define ZB_NOALLOC_SCRATCH_BYTES (4u << 20)

/* zb_plan without a caller-provided workspace, for callers that cannot
 * allocate device memory: for example a plugin enqueued by a host framework
 * that owns every allocation and offers it no scratch buffer, or a serving
 * loop that bans cudaMalloc/cudaFree on its hot path because they can
 * synchronise the device.  The pages have no counterpart; this is a
 * convenience of the library.
 *
 * Same arguments, results and errors as zb_plan, minus the workspace: the
 * scratch is a fixed 4 MiB device array inside libzb that every GPU loading
 * the library keeps until the process exits.  It allocates nothing and calls
 * no allocating routine.
 *  - Limit: returns ZB_ERR_INVALID, enqueueing nothing, when
 *    zb_workspace_bytes(cfg) > ZB_NOALLOC_SCRATCH_BYTES (besides every reason
 *    zb_plan gives).
 *  - The scratch belongs to the calling thread's current device, so `stream`
 *    must belong to that device too.  The first call on a device looks up the
 *    array's device address (once per device) and caches it for the life of
 *    the process; make that first call before any stream capture starts.  A
 *    process that resets a device (cudaDeviceReset) must not call
 *    zb_plan_noalloc on that device again: the library's module is loaded
 *    anew and the cached address no longer names the array.
 *  - Every call on a device shares the one array, which keeps what the last
 *    call left in it; each call clears what it needs zeroed.  Calls whose work
 *    overlaps on the GPU (two streams, or two host threads) race on the
 *    array: order them on one stream or serialise them. */
ZB_API int zb_plan_noalloc(const zb_config *cfg, const int32_t *topk_ids, const zb_plan_t *plan,
                           void *stream);

/* Step 4: buf[dst_row[i,s,k]][:] = hidden[i,s][:], bit for bit: each token row
 * is written into the fixed-shape, expert-grouped receive buffer of every rank
 * that serves one of its K experts (MoonEP, section on what it enforces: rows
 * go straight into static per-rank buffers with no staging copy; on one GPU
 * that remote write is a local scatter).  hidden: device bf16 [P][S][H]; buf: device bf16 [P][cap][H].
 * Rows of buf past load_after[j] are not written.  If plan->stats holds an
 * error status the kernel writes nothing.  Returns ZB_OK, ZB_ERR_INVALID or
 * ZB_ERR_CUDA. */
ZB_API int zb_dispatch(const zb_config *cfg, const zb_plan_t *plan, const uint16_t *hidden,
                uint16_t *buf, void *stream);

/* Step 5: for every token t = (i,s) and column h,
 *   acc = +0.0f;  for k = 0..K-1: acc = fmaf(w[t][k], float(y[dst_row[t][k]][h]), acc);
 *   out[t][h] = bf16(acc), rounded to nearest, ties to even,
 * the inverse of dispatch weighted by the gates (Zepp 4.2, merge for combine;
 * ISER-MoE, Key Formula, the combine half of the dispatch+combine traffic).  One
 * rounding per term, in this fixed order, so the result is reproducible bit
 * for bit.  y: device bf16 [P][cap][H] (expert outputs, same layout as buf);
 * topk_weights: device float32 [P][S][K]; out: device bf16 [P][S][H].  If
 * plan->stats holds an error status the kernel writes nothing.  Returns
 * ZB_OK, ZB_ERR_INVALID or ZB_ERR_CUDA. */
ZB_API int zb_combine(const zb_config *cfg, const zb_plan_t *plan, const uint16_t *y,
               const float *topk_weights, uint16_t *out, void *stream);

/* ------------------------------------------- the path on one of P GPUs */

/* The same five steps when the P ranks are P GPUs, one process (or thread)
 * per GPU, each holding only its own S tokens: ISER-MoE ("Methodology /
 * HALO-Q Scheduler", stage 1) has the ranks exchange their route counts and
 * then every rank plan alike; MoonEP ("What MoonEP enforces and how") has
 * each rank write its rows straight into the fixed-shape, expert-grouped
 * receive buffers of the other ranks.  On rank i:
 *   1. zb_count: the counts of its own ids (one row of E+1 ints);
 *   2. the caller all-gathers every rank's row, in rank order, into a
 *      [P][E+1] table (for example an NCCL all-gather of P*(E+1) int32);
 *   3. zb_plan_rank: the plan from that table, identical on every rank,
 *      and the destination rows of its own entries;
 *   4. zb_dispatch_rank: its rows written into every rank's receive buffer;
 *   5. after the expert computation, zb_combine_rank: its tokens' outputs
 *      gathered from every rank's expert output buffer.
 * Between 4 and the expert computation, and between the expert computation
 * and 5, the ranks must synchronise (for example a barrier on the stream):
 * these calls only move rows and never wait for another rank.
 *
 * For rank i, every table these calls produce equals zb_plan's over the whole
 * batch, and plan->dst_row [S][K] equals zb_plan's rows of source i (values
 * j*cap + row, as there).  On one GPU the P buffers may be P parts of one
 * allocation, which reproduces zb_dispatch and zb_combine bit for bit. */

/* Bytes of device scratch memory zb_count and zb_plan_rank need (0 if cfg
 * is invalid): the per-chunk histograms of this rank's ids and the segment
 * table. */
ZB_API size_t zb_rank_workspace_bytes(const zb_config *cfg);

/* Step 1 on one rank: counts[e] = #{(s,k) : ids[s][k] = e} for e < E and
 * counts[E] = the number of ids outside [0, E).  ids: device int32 [S][K],
 * this rank's entries; counts: device int32 [E+1]; workspace:
 * zb_rank_workspace_bytes(cfg) bytes, 256-byte aligned.  The workspace keeps
 * the per-chunk histograms that zb_plan_rank reads: pass the same workspace,
 * untouched, and the same ids to the zb_plan_rank that follows.  Returns
 * ZB_OK, ZB_ERR_INVALID or ZB_ERR_CUDA. */
ZB_API int zb_count(const zb_config *cfg, const int32_t *topk_ids, int32_t *counts,
                    void *workspace, size_t workspace_bytes, void *stream);

/* Steps 2-3 on rank `rank` (0 <= rank < P): counts is the all-gathered
 * device table int32 [P][E+1] (rank j's zb_count row at j), topk_ids this
 * rank's ids [S][K], placement NULL (the greedy places the replicas) or a
 * kept placement as for zb_plan_placed.  plan: as for zb_plan, except that
 * dst_row is [S][K] (this rank's entries) and row_src must be NULL.
 * workspace: the one zb_count filled for these ids.  The plan's status
 * (zb_plan_status) is ZB_ERR_INVALID when counts[rank] is not the count of
 * this rank's ids or a row of counts does not hold S*K non-negative counts,
 * and ZB_ERR_BAD_ID on every rank when any rank counted an id outside
 * [0, E); otherwise as zb_plan.  Returns ZB_OK once enqueued, ZB_ERR_INVALID
 * or ZB_ERR_CUDA. */
ZB_API int zb_plan_rank(const zb_config *cfg, int rank, const int32_t *counts,
                        const int32_t *topk_ids, const int32_t *placement, const zb_plan_t *plan,
                        void *workspace, size_t workspace_bytes, void *stream);

/* Step 4 on one rank: for each entry (s,k) of this rank with
 * d = plan->dst_row[s][k], bufs[d / cap][d % cap][:] = hidden[s][:], bit for
 * bit.  bufs is a HOST array of P device pointers, bufs[j] = rank j's receive
 * buffer bf16 [cap][H], 16-byte aligned: peer memory mapped into this process
 * (CUDA IPC or symmetric memory) for the other ranks, or P parts of one
 * buffer on one GPU.  Rows go out as plain stores.  hidden: device bf16
 * [S][H], this rank's rows.  If the plan's status is an error nothing is
 * written.  Returns ZB_OK, ZB_ERR_INVALID or ZB_ERR_CUDA. */
ZB_API int zb_dispatch_rank(const zb_config *cfg, const zb_plan_t *plan, const uint16_t *hidden,
                            uint16_t *const *bufs, void *stream);

/* Step 5 on one rank: for each token s of this rank,
 *   acc = +0.0f; acc = fmaf(w[s][k], float(ys[d/cap][d%cap][h]), acc) for
 *   k = 0..K-1, d = plan->dst_row[s][k]; out[s][h] = bf16(acc), nearest even,
 * the fold of zb_combine.  ys: HOST array of P device pointers, ys[j] = rank
 * j's expert outputs bf16 [cap][H] in its receive buffer's rows, 16-byte
 * aligned (read with plain loads); topk_weights: device float32 [S][K]; out:
 * device bf16 [S][H].  If the plan's status is an error nothing is written.
 * Returns ZB_OK, ZB_ERR_INVALID or ZB_ERR_CUDA. */
ZB_API int zb_combine_rank(const zb_config *cfg, const zb_plan_t *plan, const uint16_t *const *ys,
                           const float *topk_weights, uint16_t *out, void *stream);

/* ------------------------------------------------------- merged dispatch */

/* The merged dispatch layout (Zepp "4.2 Split and Merge": the experts one
 * token selects on the same destination share a single transfer).  Rank j
 * keeps one row per token that sends it at least one entry, in (source
 * rank, token) order, instead of one row per (token, k).  Caller-allocated
 * device buffers (int32):
 *   tok_row [P][S][K]  j*cap + u: the merged row of entry (i,s,k) on its
 *                      destination rank j
 *   grp_tok [P][cap]   for each expert-grouped row of the plan (the rows
 *                      dst_row points at), the merged row that holds its
 *                      data, -1 for unused rows: a grouped expert kernel
 *                      reads grouped row p of rank j from merged row
 *                      grp_tok[j][p]
 *   tok_cnt [P]        rows used in rank j's merged buffer (<= load_after[j]) */
typedef struct zb_merge_t {
  int32_t *tok_row;
  int32_t *grp_tok;
  int32_t *tok_cnt;
} zb_merge_t;

/* Bytes of device scratch memory zb_merge needs (0 if cfg is invalid). */
ZB_API size_t zb_merge_workspace_bytes(const zb_config *cfg);

/* The merged layout of a completed plan (enqueued after zb_plan on the same
 * stream).  workspace: zb_merge_workspace_bytes(cfg) bytes, 256-byte aligned.
 * If the plan's status is an error, the buffers are left undefined.  Returns
 * ZB_OK, ZB_ERR_INVALID or ZB_ERR_CUDA. */
ZB_API int zb_merge(const zb_config *cfg, const zb_plan_t *plan, const zb_merge_t *merge,
                    void *workspace, size_t workspace_bytes, void *stream);

/* tbuf[tok_row[i,s,k]][:] = hidden[i,s][:], each merged row written once:
 * hidden bf16 [P][S][H] -> tbuf bf16 [P][cap][H]; rows past tok_cnt[j] are
 * not written.  Writes a token's row once per destination rank instead of
 * once per selected expert.  Returns ZB_OK, ZB_ERR_INVALID or ZB_ERR_CUDA. */
ZB_API int zb_dispatch_merged(const zb_config *cfg, const zb_plan_t *plan,
                              const zb_merge_t *merge, const uint16_t *hidden, uint16_t *tbuf,
                              void *stream);

/* Combine with node-local pre-reduction (Zepp, 4.2 Split and Merge: a rank
 * sums the outputs of the experts a token selected on it into one partial
 * before sending it back), in two calls, the destination side and the source
 * side.  The merged layout `merge` must come from zb_merge of the same plan.
 *
 * zb_combine_reduce: y bf16 [P][cap][H] (expert outputs in the plan's
 * expert-grouped rows), topk_weights fp32 [P][S][K] -> part bf16 [P][cap][H]
 * (merged rows).  For each merged row r of token t:
 *   acc = +0.0f; acc = fmaf(w[t,k], y[dst_row[t,k]], acc) for k = 0..K-1
 *   with tok_row[t,k] = r; part[r] = bf16(acc), rounded to nearest even.
 * Rows past tok_cnt[j] are not written.
 *
 * zb_combine_merged: part -> out bf16 [P][S][H]:
 *   acc = +0.0f; acc = acc + part[r] for the token's merged rows r in the
 *   order of the first k naming each; out[t] = bf16(acc).
 * Where all of a token's experts sit on one rank, out equals zb_combine's
 * output bit for bit; otherwise each partial adds one bf16 rounding.
 * Both: y, part and out 16-byte aligned; ZB_OK, ZB_ERR_INVALID or
 * ZB_ERR_CUDA; nothing is written when the plan's status is an error. */
ZB_API int zb_combine_reduce(const zb_config *cfg, const zb_plan_t *plan, const zb_merge_t *merge,
                             const uint16_t *y, const float *topk_weights, uint16_t *part,
                             void *stream);
ZB_API int zb_combine_merged(const zb_config *cfg, const zb_plan_t *plan, const zb_merge_t *merge,
                             const uint16_t *part, uint16_t *out, void *stream);

/* A replica placement from historical demand (Zepp, 4.1 Expert Placement and
 * Token Routing: the R slots of each GPU go greedily to the experts with the
 * highest historical demand per replica, spread round-robin across nodes
 * first, then across a node's GPUs, for node-level coverage).  HOST memory:
 * demand int64 [E] >= 0 (e.g. rows routed to each expert over past
 * invocations), placement int32 [P][R] (written; -1 = empty), for use with
 * zb_plan_placed.  Each pick takes the expert with the largest demand per copy
 * D_e / n_e (n_e its copies so far, home included; exact comparison; ties to
 * the lowest id) among experts that still fit.  The copy goes to the first
 * node, from a round-robin cursor, that holds no copy of the expert and has a
 * GPU that can take it, else to the first node from the cursor with such a
 * GPU; within the node, the first such GPU from the node's own cursor; the
 * lowest free slot.  Both cursors then move past the choice.  An expert that
 * fits nowhere is not picked again; slots nothing fits stay empty.  Touches no
 * device.  ZB_OK, or ZB_ERR_INVALID for a bad argument or a demand outside
 * [0, 2^57] (demand times copies must fit in int64). */
ZB_API int zb_place_by_demand(const zb_config *cfg, const int64_t *demand, int32_t *placement);

/* Placement recalibration between invocations (not part of an invocation's
 * path).  From the replica placement `placement` (device int32 [P][R], -1 =
 * empty; changed in place) and the route counts `cnt` (device int32 [P][E],
 * e.g. plan->cnt of the invocation that showed drift), each step applies the
 * candidate whose kept-placement plan (zb_plan_placed's quotas) has the
 * lowest max rank load, the first in candidate order among equals, and only
 * if it lowers the max load.  The search stops once
 *   max load <= (1 + eps) * (sum of cnt) / P
 * (every rank within eps of the mean; ViBE's default eps is 0.03), when no
 * candidate lowers the max load, or after max_swaps steps.
 *   mode 0 (ViBE, Drift-Aware Recalibration, incremental placement update):
 *     a candidate puts expert e into helper slot x (one copy moved in over
 *     the network); order: x = j*R + slot ascending, then e ascending.
 *   mode 1 (Zepp, 4.3, eq. (4), intra-node swaps): a candidate exchanges the
 *     experts of slots x1 < x2 on two ranks of one node (one may be empty),
 *     keeping the node's set of experts; order: x1, then x2 ascending.
 * A candidate must leave a valid placement (see zb_plan_placed).  Every step
 * scores all candidates on the device, one warp each, and reads the scores
 * back: this call synchronises `stream`.  workspace:
 * zb_recalibrate_workspace_bytes(cfg, mode) bytes, 256-byte aligned.  On
 * ZB_OK, *swaps (steps taken) and *max_load (the final plan's max rank load)
 * are written when non-NULL.  ZB_ERR_INVALID for a bad argument, an invalid
 * placement or negative counts; ZB_ERR_CUDA if a CUDA call fails. */
ZB_API size_t zb_recalibrate_workspace_bytes(const zb_config *cfg, int mode);
ZB_API int zb_recalibrate(const zb_config *cfg, const int32_t *cnt, int32_t *placement, int mode,
                          float eps, int max_swaps, void *workspace, size_t workspace_bytes,
                          void *stream, int32_t *swaps, int32_t *max_load);

/* ------------------------------------------------------ bounds-checked build
 *
 * Built with -DZB_DEBUG (token_dispatch_top_b200/libzb_debug.so), every
 * kernel checks the accesses whose index comes from data -- a row number
 * from dst_row or from the segment table, an expert id, a slot -- against
 * the extent of what it indexes.  A failed check skips that access and is
 * recorded on the device: a count, and the site, index and bound of the
 * first failure.  This stands in for a memory checker: the GPU tests can run
 * against the debug library and require that nothing was recorded.
 *
 * The release library keeps the guards that protect memory (rows outside
 * [0, P*cap) are skipped) and compiles the rest of the checks away; there,
 * zb_debug_read returns ZB_ERR_INVALID and touches nothing. */
#define ZB_SITE_ASSIGN_EXPERT 1 /* k_assign: per-warp histogram indexed by an id */
#define ZB_SITE_ASSIGN_SEGMENT 2 /* k_assign: segment index from hoff */
#define ZB_SITE_ASSIGN_ROW 3    /* k_assign: the row an entry is given */
#define ZB_SITE_PLAN_SEGMENT 4  /* k_planner: segment-table write */
#define ZB_SITE_PLAN_SLOT 5     /* k_planner / k_eval_placements: helper slot or holder table */
#define ZB_SITE_DISPATCH_ROW 6  /* k_dispatch*: a destination row of dst_row */
#define ZB_SITE_COMBINE_ROW 7   /* k_combine*: a source row of dst_row */
#define ZB_SITE_MERGE_ROW 8     /* merge kernels: a row of dst_row or of the merged layout */
typedef struct zb_debug_record {
  uint64_t count; /* failed checks since the last reset, over all kernels */
  int32_t site;   /* ZB_SITE_* of the first failure recorded (0: none) */
  int32_t reserved;
  int64_t index;  /* its index */
  int64_t bound;  /* and the extent the index had to stay below */
} zb_debug_record;

/* Copies the record into *out (host) and, when reset != 0, clears it.
 * Synchronises the device.  ZB_ERR_INVALID in the release library or for a
 * NULL out; ZB_ERR_CUDA if a CUDA call fails.  The record is per process and
 * per device; calls from several threads at once are not ordered. */
ZB_API int zb_debug_read(zb_debug_record *out, int reset);

#ifdef __cplusplus
}
#endif

#endif /* ZB_H */
