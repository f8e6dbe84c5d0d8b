// zb_api.cu -- the C ABI declared in include/zb.h: validation, workspace
// sizing, status codes and the launch sequence of each call.  No allocation
// and no synchronisation happen here, except the documented stream
// synchronisation of zb_plan_status.
#include <cstring>

#include <cmath>

#include "zb_internal.cuh"

using zb::Workspace;

namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }

int plan_buffers_ok(const zb_config& c, const zb_plan_t* p) {
  if (!p) return 0;
  if (!p->cnt || !p->home_quota || !p->load_before || !p->load_after || !p->cu_seqlens ||
      !p->stats)
    return 0;
  if (c.R > 0 && (!p->rep_expert || !p->rep_quota)) return 0;
  if (c.S > 0 && !p->dst_row) return 0;
  if (reinterpret_cast<uintptr_t>(p->trace) & 7u) return 0;  // 64-bit atomics
  return 1;
}

}  // namespace

extern "C" {

const char* zb_strerror(int status) {
  switch (status) {
    case ZB_OK: return "ok";
    case ZB_WARN_UNBALANCED: return "unbalanced: the replica slots do not permit the water level";
    case ZB_ERR_INVALID: return "invalid configuration, pointer, size or alignment";
    case ZB_ERR_CAPACITY: return "planned rank load exceeds cap_rows";
    case ZB_ERR_BAD_ID: return "routing id outside [0, E)";
    case ZB_ERR_TIMEOUT: return "a bounded device wait gave up";
    case ZB_ERR_CUDA: return "CUDA runtime error";
    default: return "unknown status";
  }
}

int zb_validate(const zb_config* c) {
  if (!c) return ZB_ERR_INVALID;
  if (c->P < 1 || c->P > zb::kMaxP) return ZB_ERR_INVALID;
  if (c->E < c->P || c->E > zb::kMaxE || c->E % c->P != 0) return ZB_ERR_INVALID;
  if (c->K < 1 || c->K > 16) return ZB_ERR_INVALID;
  if (c->S < 0) return ZB_ERR_INVALID;
  if (c->H < 8 || c->H % 8 != 0) return ZB_ERR_INVALID;
  if (c->R < 0 || c->R > c->P - 1) return ZB_ERR_INVALID;
  if (!(c->C >= 0.0f && c->C < 1.0f)) return ZB_ERR_INVALID;
  if (c->gpus_per_node < 1 || c->P % c->gpus_per_node != 0) return ZB_ERR_INVALID;
  const int64_t sk = int64_t(c->S) * c->K;
  if (sk > INT32_MAX) return ZB_ERR_INVALID;
  if (int64_t(c->cap_rows) < sk) return ZB_ERR_INVALID;
  if (int64_t(c->P) * sk > INT32_MAX) return ZB_ERR_INVALID;
  if (int64_t(c->P) * c->cap_rows > INT32_MAX) return ZB_ERR_INVALID;
  if (c->policy != ZB_POLICY_ROOM && c->policy != ZB_POLICY_LOCAL) return ZB_ERR_INVALID;
  if (c->relax != 0 && c->relax != 1) return ZB_ERR_INVALID;
  if (c->repair != 0 && c->repair != 1) return ZB_ERR_INVALID;
  return ZB_OK;
}

size_t zb_workspace_bytes(const zb_config* c) {
  if (zb_validate(c) != ZB_OK) return 0;
  return zb::workspace_layout(*c, c->P).bytes;
}

}  // extern "C"

namespace {

// The kernel arguments of a plan over the sources [src0, src0 + nsrc) whose
// ids, per-chunk histograms and dst_row are laid out from src0.
zb::PlanArgs plan_args(const zb_config* c, const zb::Workspace& w, const int32_t* ids,
                       const int32_t* placement, const zb_plan_t* plan, void* ws) {
  char* base = static_cast<char*>(ws);
  zb::PlanArgs a{};
  a.P = c->P; a.E = c->E; a.K = c->K; a.S = c->S; a.R = c->R; a.Eh = c->E / c->P;
  a.gpn = c->gpus_per_node; a.cap = c->cap_rows; a.policy = c->policy;
  a.relax = c->relax;
  a.repair = c->repair;
  a.cfix = c->relax ? int(std::floor(double(c->C) * 1048576.0)) : 0;
  a.nchunk = w.nchunk; a.seg_width = w.seg_width;
  a.inv_gpn = 1.0f / float(c->gpus_per_node);
  a.inv_eh = 1.0f / float(a.Eh);
  a.ids = ids;
  a.placement = placement;
  if (plan) {
    a.cnt = plan->cnt; a.rep_expert = plan->rep_expert; a.rep_quota = plan->rep_quota;
    a.home_quota = plan->home_quota; a.load_before = plan->load_before;
    a.load_after = plan->load_after; a.cu_seqlens = plan->cu_seqlens;
    a.dst_row = plan->dst_row; a.row_src = plan->row_src; a.stats = plan->stats;
    a.trace = reinterpret_cast<unsigned long long*>(plan->trace);
  }
  a.chunk_hist = reinterpret_cast<int32_t*>(base + w.off_chunk_hist);
  a.tot = nullptr;
  a.hoff = reinterpret_cast<int32_t*>(base + w.off_hoff);
  a.seg = reinterpret_cast<int2*>(base + w.off_seg);
  a.src0 = 0;
  a.plan_hist = nullptr;  // set by the calls that plan
  a.own_hist = nullptr;
  return a;
}

bool workspace_ok(const void* ws, size_t ws_bytes, size_t need) {
  return ws && ws_bytes >= need && (reinterpret_cast<uintptr_t>(ws) & 255u) == 0;
}

int plan_impl(const zb_config* c, const int32_t* ids, const int32_t* placement,
              const zb_plan_t* plan, void* ws, size_t ws_bytes, void* stream) {
  if (zb_validate(c) != ZB_OK) return ZB_ERR_INVALID;
  if (!plan_buffers_ok(*c, plan)) return ZB_ERR_INVALID;
  const Workspace w = zb::workspace_layout(*c, c->P);
  if (!workspace_ok(ws, ws_bytes, w.bytes)) return ZB_ERR_INVALID;
  if (c->S > 0 && !ids) return ZB_ERR_INVALID;
  cudaStream_t s = as_stream(stream);
  zb::PlanArgs a = plan_args(c, w, ids, placement, plan, ws);
  // the planner reads the per-source totals that k_hist adds up
  a.tot = reinterpret_cast<int32_t*>(static_cast<char*>(ws) + w.off_tot);
  a.plan_hist = a.tot;

  if (a.trace && zb::launch_trace_reset(a.trace, s) != cudaSuccess) return ZB_ERR_CUDA;
  if (a.row_src &&
      cudaMemsetAsync(a.row_src, 0xff, sizeof(int32_t) * size_t(c->P) * c->cap_rows, s) !=
          cudaSuccess)
    return ZB_ERR_CUDA;
  if (zb::launch_hist_totals(a, c->P, s) != cudaSuccess) return ZB_ERR_CUDA;
  if (zb::launch_planner(a, zb::planner_smem_bytes(*c), s) != cudaSuccess) return ZB_ERR_CUDA;
  if (zb::launch_assign(a, c->P, s) != cudaSuccess) return ZB_ERR_CUDA;
  return ZB_OK;
}

}  // namespace

extern "C" {

int zb_plan(const zb_config* c, const int32_t* ids, const zb_plan_t* plan, void* ws,
            size_t ws_bytes, void* stream) {
  return plan_impl(c, ids, nullptr, plan, ws, ws_bytes, stream);
}

int zb_plan_placed(const zb_config* c, const int32_t* ids, const int32_t* placement,
                   const zb_plan_t* plan, void* ws, size_t ws_bytes, void* stream) {
  if (c && c->R > 0 && !placement) return ZB_ERR_INVALID;
  return plan_impl(c, ids, c && c->R > 0 ? placement : nullptr, plan, ws, ws_bytes, stream);
}

size_t zb_rank_workspace_bytes(const zb_config* c) {
  if (zb_validate(c) != ZB_OK) return 0;
  return zb::workspace_layout(*c, 1).bytes;
}

int zb_count(const zb_config* c, const int32_t* ids, int32_t* counts, void* ws,
             size_t ws_bytes, void* stream) {
  if (zb_validate(c) != ZB_OK || !counts) return ZB_ERR_INVALID;
  const Workspace w = zb::workspace_layout(*c, 1);
  if (!workspace_ok(ws, ws_bytes, w.bytes)) return ZB_ERR_INVALID;
  if (c->S > 0 && !ids) return ZB_ERR_INVALID;
  cudaStream_t s = as_stream(stream);
  const zb::PlanArgs a = plan_args(c, w, ids, nullptr, nullptr, ws);
  if (zb::launch_hist(a, 1, s) != cudaSuccess) return ZB_ERR_CUDA;
  if (zb::launch_count_row(a, counts, s) != cudaSuccess) return ZB_ERR_CUDA;
  return ZB_OK;
}

int zb_plan_rank(const zb_config* c, int rank, const int32_t* counts, const int32_t* ids,
                 const int32_t* placement, const zb_plan_t* plan, void* ws, size_t ws_bytes,
                 void* stream) {
  if (zb_validate(c) != ZB_OK || rank < 0 || rank >= c->P || !counts) return ZB_ERR_INVALID;
  if (!plan_buffers_ok(*c, plan) || plan->row_src) return ZB_ERR_INVALID;
  const Workspace w = zb::workspace_layout(*c, 1);
  if (!workspace_ok(ws, ws_bytes, w.bytes)) return ZB_ERR_INVALID;
  if (c->S > 0 && !ids) return ZB_ERR_INVALID;
  cudaStream_t s = as_stream(stream);
  zb::PlanArgs a = plan_args(c, w, ids, c->R > 0 ? placement : nullptr, plan, ws);
  a.src0 = rank;
  a.plan_hist = counts;
  a.own_hist = a.chunk_hist;
  if (a.trace && zb::launch_trace_reset(a.trace, s) != cudaSuccess) return ZB_ERR_CUDA;
  if (zb::launch_planner(a, zb::planner_smem_bytes(*c), s) != cudaSuccess) return ZB_ERR_CUDA;
  if (zb::launch_assign(a, 1, s) != cudaSuccess) return ZB_ERR_CUDA;
  return ZB_OK;
}

int zb_plan_status(const zb_config* c, const zb_plan_t* plan, void* stream, int32_t* max_load) {
  if (zb_validate(c) != ZB_OK || !plan || !plan->stats) return ZB_ERR_INVALID;
  int64_t st[ZB_STATS_LEN];
  cudaStream_t s = as_stream(stream);
  if (cudaMemcpyAsync(st, plan->stats, sizeof(st), cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return ZB_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return ZB_ERR_CUDA;
  if (max_load) *max_load = int32_t(st[ZB_STAT_MAX_LOAD]);
  return int(st[ZB_STAT_STATUS]);
}

int zb_dispatch(const zb_config* c, const zb_plan_t* plan, const uint16_t* hidden,
                uint16_t* buf, void* stream) {
  if (zb_validate(c) != ZB_OK || !plan || !plan->stats) return ZB_ERR_INVALID;
  if (c->S > 0 && (!plan->dst_row || !hidden || !buf)) return ZB_ERR_INVALID;
  if ((hidden && !aligned16(hidden)) || (buf && !aligned16(buf))) return ZB_ERR_INVALID;
  if (zb::launch_dispatch(c->P, c->S, c->K, c->H, c->cap_rows, plan->dst_row, plan->stats,
                          hidden, buf, as_stream(stream)) != cudaSuccess)
    return ZB_ERR_CUDA;
  return ZB_OK;
}

size_t zb_merge_workspace_bytes(const zb_config* c) {
  if (zb_validate(c) != ZB_OK) return 0;
  const int64_t nchunk = zb::ceil_div(int64_t(c->P) * c->S, zb::kMergeChunk);
  return zb::align256(size_t(sizeof(int32_t)) * size_t(nchunk) * c->P + 1);
}

int zb_merge(const zb_config* c, const zb_plan_t* plan, const zb_merge_t* m, void* ws,
             size_t ws_bytes, void* stream) {
  if (zb_validate(c) != ZB_OK || !plan || !plan->stats || !m) return ZB_ERR_INVALID;
  if (!m->tok_cnt || !m->grp_tok) return ZB_ERR_INVALID;
  if (c->S > 0 && (!plan->dst_row || !m->tok_row)) return ZB_ERR_INVALID;
  if (!ws || ws_bytes < zb_merge_workspace_bytes(c) || (reinterpret_cast<uintptr_t>(ws) & 255u))
    return ZB_ERR_INVALID;
  if (!plan->load_after) return ZB_ERR_INVALID;
  cudaStream_t s = as_stream(stream);
  zb::MergeArgs a{};
  a.P = c->P; a.K = c->K; a.cap = c->cap_rows; a.ntok = int64_t(c->P) * c->S;
  if (a.ntok == 0) {  // no tokens: no kernel runs, every row is unused
    if (cudaMemsetAsync(m->grp_tok, 0xff, sizeof(int32_t) * size_t(c->P) * c->cap_rows, s) !=
            cudaSuccess ||
        cudaMemsetAsync(m->tok_cnt, 0, sizeof(int32_t) * size_t(c->P), s) != cudaSuccess)
      return ZB_ERR_CUDA;
    return ZB_OK;
  }
  a.dst_row = plan->dst_row; a.load_after = plan->load_after; a.stats = plan->stats;
  a.tok_row = m->tok_row; a.grp_tok = m->grp_tok; a.tok_cnt = m->tok_cnt;
  a.chunk_cnt = static_cast<int32_t*>(ws);
  if (zb::launch_merge(a, s) != cudaSuccess) return ZB_ERR_CUDA;
  return ZB_OK;
}

int zb_dispatch_merged(const zb_config* c, const zb_plan_t* plan, const zb_merge_t* m,
                       const uint16_t* hidden, uint16_t* tbuf, void* stream) {
  if (zb_validate(c) != ZB_OK || !plan || !plan->stats || !m) return ZB_ERR_INVALID;
  if (c->S > 0 && (!m->tok_row || !hidden || !tbuf)) return ZB_ERR_INVALID;
  if ((hidden && !aligned16(hidden)) || (tbuf && !aligned16(tbuf))) return ZB_ERR_INVALID;
  if (zb::launch_dispatch_merged(c->P, c->S, c->K, c->H, c->cap_rows, m->tok_row, plan->stats,
                                 hidden, tbuf, as_stream(stream)) != cudaSuccess)
    return ZB_ERR_CUDA;
  return ZB_OK;
}

int zb_combine_reduce(const zb_config* c, const zb_plan_t* plan, const zb_merge_t* m,
                      const uint16_t* y, const float* w, uint16_t* part, void* stream) {
  if (zb_validate(c) != ZB_OK || !plan || !plan->stats || !m) return ZB_ERR_INVALID;
  if (c->S > 0 && (!plan->dst_row || !m->tok_row || !y || !w || !part)) return ZB_ERR_INVALID;
  if ((y && !aligned16(y)) || (part && !aligned16(part))) return ZB_ERR_INVALID;
  if (zb::launch_combine_reduce(c->P, c->S, c->K, c->H, c->cap_rows, plan->dst_row, m->tok_row,
                                plan->stats, y, w, part, as_stream(stream)) != cudaSuccess)
    return ZB_ERR_CUDA;
  return ZB_OK;
}

int zb_combine_merged(const zb_config* c, const zb_plan_t* plan, const zb_merge_t* m,
                      const uint16_t* part, uint16_t* out, void* stream) {
  if (zb_validate(c) != ZB_OK || !plan || !plan->stats || !m) return ZB_ERR_INVALID;
  if (c->S > 0 && (!m->tok_row || !part || !out)) return ZB_ERR_INVALID;
  if ((part && !aligned16(part)) || (out && !aligned16(out))) return ZB_ERR_INVALID;
  if (zb::launch_combine_merged(c->P, c->S, c->K, c->H, c->cap_rows, m->tok_row, plan->stats,
                                part, out, as_stream(stream)) != cudaSuccess)
    return ZB_ERR_CUDA;
  return ZB_OK;
}

int zb_dispatch_rank(const zb_config* c, const zb_plan_t* plan, const uint16_t* hidden,
                     uint16_t* const* bufs, void* stream) {
  if (zb_validate(c) != ZB_OK || !plan || !plan->stats || !bufs) return ZB_ERR_INVALID;
  if (c->S > 0 && (!plan->dst_row || !hidden)) return ZB_ERR_INVALID;
  if (hidden && !aligned16(hidden)) return ZB_ERR_INVALID;
  zb::RankBufs t{};
  for (int j = 0; j < c->P; ++j) {
    if (!bufs[j] || !aligned16(bufs[j])) return ZB_ERR_INVALID;
    t.p[j] = bufs[j];
  }
  if (zb::launch_dispatch_ranks(c->P, c->S, c->K, c->H, c->cap_rows, plan->dst_row, plan->stats,
                                hidden, t, as_stream(stream)) != cudaSuccess)
    return ZB_ERR_CUDA;
  return ZB_OK;
}

int zb_combine_rank(const zb_config* c, const zb_plan_t* plan, const uint16_t* const* ys,
                    const float* w, uint16_t* out, void* stream) {
  if (zb_validate(c) != ZB_OK || !plan || !plan->stats || !ys) return ZB_ERR_INVALID;
  if (c->S > 0 && (!plan->dst_row || !w || !out)) return ZB_ERR_INVALID;
  if (out && !aligned16(out)) return ZB_ERR_INVALID;
  zb::RankBufs t{};
  bool wide_ok = (reinterpret_cast<uintptr_t>(out) & 31u) == 0;
  for (int j = 0; j < c->P; ++j) {
    if (!ys[j] || !aligned16(ys[j])) return ZB_ERR_INVALID;
    t.p[j] = const_cast<uint16_t*>(ys[j]);
    wide_ok = wide_ok && (reinterpret_cast<uintptr_t>(ys[j]) & 31u) == 0;
  }
  if (zb::launch_combine_ranks(c->P, c->S, c->K, c->H, c->cap_rows, plan->dst_row, plan->stats,
                               t, w, out, wide_ok, as_stream(stream)) != cudaSuccess)
    return ZB_ERR_CUDA;
  return ZB_OK;
}

int zb_combine(const zb_config* c, const zb_plan_t* plan, const uint16_t* y, const float* w,
               uint16_t* out, void* stream) {
  if (zb_validate(c) != ZB_OK || !plan || !plan->stats) return ZB_ERR_INVALID;
  if (c->S > 0 && (!plan->dst_row || !y || !w || !out)) return ZB_ERR_INVALID;
  if ((y && !aligned16(y)) || (out && !aligned16(out))) return ZB_ERR_INVALID;
  if (zb::launch_combine(c->P, c->S, c->K, c->H, c->cap_rows, plan->dst_row, plan->stats, y, w,
                         out, as_stream(stream)) != cudaSuccess)
    return ZB_ERR_CUDA;
  return ZB_OK;
}

int zb_debug_read(zb_debug_record* out, int reset) {
#ifdef ZB_DEBUG
  if (!out) return ZB_ERR_INVALID;
  if (cudaDeviceSynchronize() != cudaSuccess) return ZB_ERR_CUDA;
  // the first failure reported is the first one recorded by the plan
  // kernels, else by the data kernels, else by the merge kernels
  cudaError_t (*const readers[])(zb::DebugRecord*, bool) = {
      zb::debug_read_plan, zb::debug_read_move, zb::debug_read_merge};
  *out = zb_debug_record{};
  for (auto read : readers) {
    zb::DebugRecord r{};
    if (read(&r, reset != 0) != cudaSuccess) return ZB_ERR_CUDA;
    if (r.count > 0 && out->count == 0) {
      out->site = r.site;
      out->index = r.index;
      out->bound = r.bound;
    }
    out->count += r.count;
  }
  return ZB_OK;
#else
  (void)out;
  (void)reset;
  return ZB_ERR_INVALID;
#endif
}

}  // extern "C"
