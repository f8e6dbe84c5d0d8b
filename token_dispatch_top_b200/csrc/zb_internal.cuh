// zb_internal.cuh -- definitions shared by the device library's translation
// units: workspace layout, launch constants and the kernel declarations.
#pragma once

#include <cstddef>
#include <cstdint>
#include <utility>

#include <cuda_runtime.h>

#include "zb.h"

namespace zb {

// Entries of one source rank handled by one CTA of the histogram and the
// assignment kernels.
constexpr int kChunk = 2048;
constexpr int kChunkThreads = 512;
constexpr int kMaxE = 384;
constexpr int kMaxP = 32;
constexpr int kPlanThreads = 512;  // 16 warps
constexpr int kPlanWarps = kPlanThreads / 32;

// Widest row of the segment table: E + P*R entries.
constexpr int kMaxSegWidth = kMaxE + kMaxP * (kMaxP - 1);

inline int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }
inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// Layout of the scratch workspace (all offsets 256-byte aligned).  Nothing in
// it needs initialising: every word is written before it is read.
//   chunk_hist int32 [nsrc][nchunk][E+1]  per-chunk expert counts of the
//                                      sources histogrammed here (all P on one
//                                      GPU, or one rank's own); column E
//                                      counts the chunk's ids outside [0, E)
//   tot        int32 [nsrc][E+1]       the same summed over the chunks (zeroed
//                                      by k_zero, then added to by k_hist)
//   hoff       int32 [E+1]             first segment of expert e in a row of seg
//   seg        int2  [P][E + P*R]      per (source i, expert e): the hosts in
//                                      the order source i fills them, as
//                                      (cumulative end count, base row)
struct Workspace {
  int nchunk;
  int seg_width;
  size_t off_chunk_hist, off_tot, off_hoff, off_seg, bytes;
};

inline Workspace workspace_layout(const zb_config& c, int nsrc) {
  Workspace w{};
  const int64_t nk = int64_t(c.S) * c.K;
  w.nchunk = int(ceil_div(nk, kChunk));
  w.seg_width = c.E + c.P * c.R;
  size_t o = 0;
  w.off_chunk_hist = o;
  o = align256(o + sizeof(int32_t) * size_t(nsrc) * w.nchunk * (c.E + 1));
  w.off_tot = o;
  o = align256(o + sizeof(int32_t) * size_t(nsrc) * (c.E + 1));
  w.off_hoff = o;
  o = align256(o + sizeof(int32_t) * size_t(c.E + 1));
  w.off_seg = o;
  o = align256(o + sizeof(int2) * size_t(c.P) * w.seg_width);
  w.bytes = o;
  return w;
}

// Kernel parameter block shared by the plan kernels.
//
// The planner reads the route counts from plan_hist [P][E+1]: the
// per-source totals k_hist adds up (whole batch on one GPU), or the exchanged
// count rows of P ranks.  k_hist and k_assign handle the sources src0 ..
// src0 + gridDim.y - 1; ids, dst_row and chunk_hist are indexed from src0
// (local), seg and row_src by the global source.  own_hist, when set, holds
// the per-chunk histograms of source src0 alone, which the planner checks
// against its row of plan_hist.
struct PlanArgs {
  int P, E, K, S, R, Eh, gpn, cap, policy;
  int relax, cfix;  // eq. (1)'s band: C as floor(C * 2^20), 0 unless relax
  int repair;       // quota repair between rank pairs after the greedy
  int nchunk, seg_width;
  float inv_gpn, inv_eh;  // 1/gpn and 1/Eh, for div_small
  int src0;
  const int32_t* plan_hist;
  const int32_t* own_hist;
  const int32_t* ids;
  const int32_t* placement;  // [P][R] replica placement to keep, or nullptr
  int32_t* cnt;
  int32_t* rep_expert;
  int32_t* rep_quota;
  int32_t* home_quota;
  int32_t* load_before;
  int32_t* load_after;
  int32_t* cu_seqlens;
  int32_t* dst_row;
  int32_t* row_src;
  int64_t* stats;
  int32_t* chunk_hist;
  int32_t* tot;  // [nsrc][E+1] per-source totals k_hist adds into, or nullptr
  int32_t* hoff;
  int2* seg;
  unsigned long long* trace;  // plan->trace, or nullptr
  int assign_sub;             // chunks per k_assign CTA (set by launch_assign)
};

// k_assign stages each of its chunks' experts and ranks in shared memory.
constexpr int kMaxAssignSub = 4;
inline size_t assign_smem_bytes(int sub) { return size_t(sub) * 2 * kChunk * sizeof(int32_t); }

// Candidate placements scored by the kept-placement greedy (recalibration).
constexpr int kEvalThreads = 256;
constexpr int kEvalWarps = kEvalThreads / 32;

struct EvalArgs {
  int P, E, R, gpn, mode;
  int64_t ncand;           // candidate 0 is the base placement
  const int32_t* Te;       // [E] rows per expert
  const int32_t* base;     // [P*R] the placement candidates change
  int32_t* out;            // [ncand] max rank load, INT32_MAX when invalid
};

// Tokens per CTA of the merged-dispatch layout kernels.
constexpr int kMergeChunk = 256;

struct MergeArgs {
  int P, K, cap;
  int64_t ntok;
  const int32_t* dst_row;
  const int32_t* load_after;
  const int64_t* stats;
  int32_t* tok_row;
  int32_t* grp_tok;
  int32_t* tok_cnt;
  int32_t* chunk_cnt;  // workspace [nchunk][P]
};

// Bounds checks.  ZB_IN(site, i, n) is 0 <= i < n for an access whose index
// comes from data, and ZB_FAIL(site, i, n) marks a guard that has just
// refused one.  In the release build ZB_IN is the constant true and ZB_FAIL
// nothing, so both compile away (the guards that protect memory stay).  In
// the debug build (ZB_DEBUG) a failure is counted, the first one's site,
// index and bound are kept in the translation unit's device record, and the
// access is skipped; zb_debug_read collects the records.  ZB_DEBUG_TU(name)
// defines a translation unit's record and its host reader `name`.
struct DebugRecord {
  unsigned long long count;
  long long index, bound;
  int site, reserved;
};

#ifdef ZB_DEBUG
#define ZB_DEBUG_TU(NAME)                                                          \
  namespace {                                                                      \
  __device__ DebugRecord g_debug;                                                  \
  __device__ __noinline__ bool debug_fail(int site, long long i, long long n) {    \
    if (atomicAdd(&g_debug.count, 1ull) == 0ull) {                                 \
      g_debug.site = site;                                                         \
      g_debug.index = i;                                                           \
      g_debug.bound = n;                                                           \
    }                                                                              \
    return false;                                                                  \
  }                                                                                \
  }                                                                                \
  cudaError_t NAME(DebugRecord* out, bool reset) {                                 \
    cudaError_t e = cudaMemcpyFromSymbol(out, g_debug, sizeof(DebugRecord));       \
    if (e == cudaSuccess && reset) {                                               \
      const DebugRecord zero{};                                                    \
      e = cudaMemcpyToSymbol(g_debug, &zero, sizeof(DebugRecord));                 \
    }                                                                              \
    return e;                                                                      \
  }
#define ZB_IN(site, i, n)                                                   \
  (((long long)(i) >= 0 && (long long)(i) < (long long)(n)) ||              \
   debug_fail((site), (long long)(i), (long long)(n)))
#define ZB_FAIL(site, i, n) ((void)debug_fail((site), (long long)(i), (long long)(n)))
cudaError_t debug_read_plan(DebugRecord* out, bool reset);
cudaError_t debug_read_move(DebugRecord* out, bool reset);
cudaError_t debug_read_merge(DebugRecord* out, bool reset);
#else
#define ZB_DEBUG_TU(NAME)
#define ZB_IN(site, i, n) true
#define ZB_FAIL(site, i, n) ((void)0)
#endif

// Programmatic dependent launch.  A kernel launched with launch_pdl may start
// while the kernel before it on the stream is still running, once every CTA
// of that kernel has called griddep_launch_dependents (or exited).  Before
// it touches anything its predecessor writes, it calls griddep_wait, which
// returns once the predecessor has completed and its writes are visible.
// Without a pending dependency (a plain launch) griddep_wait returns at once.
__device__ __forceinline__ void griddep_wait() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}
__device__ __forceinline__ void griddep_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t s, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

size_t planner_smem_bytes(const zb_config& c);

cudaError_t launch_trace_reset(unsigned long long* trace, cudaStream_t s);

cudaError_t launch_hist(const PlanArgs& a, int nsrc, cudaStream_t s);
cudaError_t launch_hist_totals(const PlanArgs& a, int nsrc, cudaStream_t s);
cudaError_t launch_count_row(const PlanArgs& a, int32_t* counts, cudaStream_t s);
cudaError_t launch_planner(const PlanArgs& a, size_t smem, cudaStream_t s);
cudaError_t launch_assign(const PlanArgs& a, int nsrc, cudaStream_t s);
size_t eval_smem_bytes(int P, int E, int R);
cudaError_t launch_eval_placements(const EvalArgs& ea, cudaStream_t s);

// Receive buffers of the P ranks: one per rank (base pointers; for one
// buffer holding every rank's rows, rank j's base is buf + j*cap*H).
struct RankBufs {
  uint16_t* p[kMaxP];
};

cudaError_t launch_dispatch(int P, int S, int K, int H, int cap, const int32_t* dst_row,
                            const int64_t* stats, const uint16_t* hidden, uint16_t* buf,
                            cudaStream_t s);
cudaError_t launch_dispatch_ranks(int P, int ntok, int K, int H, int cap,
                                  const int32_t* dst_row, const int64_t* stats,
                                  const uint16_t* hidden, const RankBufs& bufs, cudaStream_t s);
cudaError_t launch_combine_ranks(int P, int ntok, int K, int H, int cap, const int32_t* dst_row,
                                 const int64_t* stats, const RankBufs& ys, const float* w,
                                 uint16_t* out, bool wide_ok, cudaStream_t s);
cudaError_t launch_merge(const MergeArgs& a, cudaStream_t s);
cudaError_t launch_dispatch_merged(int P, int S, int K, int H, int cap, const int32_t* tok_row,
                                   const int64_t* stats, const uint16_t* hidden, uint16_t* tbuf,
                                   cudaStream_t s);
cudaError_t launch_combine_reduce(int P, int S, int K, int H, int cap, const int32_t* dst_row,
                                  const int32_t* tok_row, const int64_t* stats,
                                  const uint16_t* y, const float* w, uint16_t* part,
                                  cudaStream_t s);
cudaError_t launch_combine_merged(int P, int S, int K, int H, int cap, const int32_t* tok_row,
                                  const int64_t* stats, const uint16_t* part, uint16_t* out,
                                  cudaStream_t s);
cudaError_t launch_combine(int P, int S, int K, int H, int cap, const int32_t* dst_row,
                           const int64_t* stats, const uint16_t* y, const float* w,
                           uint16_t* out, cudaStream_t s);

}  // namespace zb
