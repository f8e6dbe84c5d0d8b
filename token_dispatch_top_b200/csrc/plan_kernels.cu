// plan_kernels.cu -- steps 1-3 of an invocation on one GPU:
//   k_zero     zeroes the per-source totals (one GPU, the plan's first kernel)
//   k_hist     per-(source rank, chunk) expert histogram in shared memory,
//              added into the source's totals when there are totals
//   k_planner  one CTA: route counts, water level, greedy replica placement
//              (one warp, lanes = ranks; or the quotas over a kept
//              placement), optional quota repair between rank pairs, quotas,
//              cu_seqlens, locality-first transport (exact quotas or eq. (1)'s
//              band) and the per-(source, expert) segment table; one instance
//              per greedy mode x repair x band
//   k_assign   per-(source rank, chunk): stable rank of every entry among the
//              source's entries of the same expert, then its destination row
// and, between invocations,
//   k_eval_placements  one warp per candidate placement: the kept-placement
//              greedy's max rank load (scores for zb_recalibrate)
//
// No kernel waits on another CTA: the chunk prefix each assignment CTA needs
// is summed directly from the per-chunk histograms.  The three kernels of a
// plan are chained by programmatic dependent launch: k_planner and k_assign
// start while their predecessor finishes, and wait for it (griddepcontrol)
// only where they read what it writes, so each launch's start-up overlaps the
// kernel before it.
//
// Sources: ISER-MoE "Methodology / HALO-Q Scheduler" (Objectives 1 and 2,
// stages 1-5); Zepp "4.1 Expert Placement and Token Routing" (R slots per GPU,
// node-first placement, eq. (1) and its relaxation C), "4.3 Three-Stream
// Scheduling" (eq. (4)); ViBE "Drift-Aware Recalibration"; MoonEP "What MoonEP
// enforces and how" (S x K per rank, cu_seqlens, expert-grouped fixed
// buffers).
#include <atomic>
#include <mutex>

#include "zb_internal.cuh"

namespace zb {
ZB_DEBUG_TU(debug_read_plan)
namespace {

constexpr unsigned kFull = 0xffffffffu;
constexpr int kPerThread = kChunk / kChunkThreads;  // entries per thread

__device__ __forceinline__ int warp_incl_scan(int v, int lane) {
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int u = __shfl_up_sync(kFull, v, o);
    if (lane >= o) v += u;
  }
  return v;
}

__device__ __forceinline__ long long warp_sum64(long long v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(kFull, v, o);
  return v;
}

// Sum of col[0], col[stride], ..., col[(n-1)*stride], kInFlight loads in
// flight.
template <int kInFlight = 8>
__device__ __forceinline__ int strided_sum(const int32_t* col, int n, int64_t stride) {
  int v = 0;
  for (int c = 0; c < n; c += kInFlight) {
    int x[kInFlight];
#pragma unroll
    for (int u = 0; u < kInFlight; ++u) x[u] = c + u < n ? __ldcg(col + int64_t(c + u) * stride) : 0;
#pragma unroll
    for (int u = 0; u < kInFlight; ++u) v += x[u];
  }
  return v;
}

// r / g for the planner's small non-negative integers (ranks, experts), from
// inv = float(1/g): (r + 1/2) / g lies at least 1/(2g) from an integer, and
// for r < 2^22 the float product (r + 1/2) * inv is within (r + 1/2) / g *
// 2^-23 < 1/(2g) of it, so truncating it gives r / g exactly.  Two float
// instructions instead of an integer division by a runtime value.
__device__ __forceinline__ int div_small(int r, float inv) {
  return int((float(r) + 0.5f) * inv);
}

// a_ij of eq. (1): 0 same rank; 1 other rank (flat) or same node; 4 other node.
__device__ __forceinline__ int cost_a(int i, int j, int gpn, float inv_gpn) {
  if (i == j) return 0;
  if (gpn > 1 && div_small(i, inv_gpn) != div_small(j, inv_gpn)) return 4;
  return 1;
}

// Trace stamps (plan->trace): %globaltimer nanoseconds, the minimum over a
// grid's CTAs for a start or a release from the dependency wait, the maximum
// for an end.  Every stamp is skipped when the plan has no trace.
__device__ __forceinline__ unsigned long long global_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
__device__ __forceinline__ void trace_first(const PlanArgs& a, int slot) {
  if (a.trace != nullptr && threadIdx.x == 0) atomicMin(a.trace + slot, global_ns());
}
// Called by every thread of the CTA at the same point.
__device__ __forceinline__ void trace_last(const PlanArgs& a, int slot) {
  if (a.trace != nullptr) {
    __syncthreads();
    if (threadIdx.x == 0) atomicMax(a.trace + slot, global_ns());
  }
}

__global__ void k_trace_reset(unsigned long long* trace) {
  const int x = threadIdx.x;
  if (x < ZB_TRACE_LEN) trace[x] = x % 3 == 2 ? 0ull : ~0ull;
}

// ------------------------------------------------------------------ step 1

// One CTA per (chunk c, source rank i).  Thread t handles entries
// t + kChunkThreads*u, u < kPerThread, all loaded before the first is counted.
// Column E of the chunk's row counts ids outside [0, E).  Each entry is one
// shared-memory atomic; merging equal ids first with a match-any vote measured
// slower, most of all on skewed batches (2.4 against 6.0 us on the hot one).
__global__ void __launch_bounds__(kChunkThreads) k_hist(PlanArgs a) {
  __shared__ int32_t sh[kMaxE + 1];
  trace_first(a, ZB_TRACE_HIST);
  griddep_launch_dependents();  // the planner may launch now and wait for us
  const int c = blockIdx.x, i = blockIdx.y, tid = threadIdx.x, lane = tid & 31;
  const int E = a.E;
  for (int e = tid; e <= E; e += kChunkThreads) sh[e] = 0;
  const int64_t nk = int64_t(a.S) * a.K;
  const int64_t start = int64_t(c) * kChunk;
  const int n = (nk - start) < kChunk ? int(nk - start) : kChunk;
  const int32_t* src = a.ids + int64_t(i) * nk + start;
  int ids[kPerThread];
#pragma unroll
  for (int u = 0; u < kPerThread; ++u) {
    const int t = tid + u * kChunkThreads;
    ids[u] = t < n ? __ldg(src + t) : -1;
  }
  __syncthreads();
  int bad = 0;
#pragma unroll
  for (int u = 0; u < kPerThread; ++u) {
    const int t = tid + u * kChunkThreads;
    const int e = ids[u];
    const bool ok = t < n && e >= 0 && e < E;
    bad += (t < n && !ok);
    if (ok) atomicAdd(&sh[e], 1);
  }
  bad = int(__reduce_add_sync(kFull, unsigned(bad)));
  if (lane == 0 && bad) atomicAdd(&sh[E], bad);
  __syncthreads();
  int32_t* out = a.chunk_hist + (int64_t(i) * a.nchunk + c) * (E + 1);
  for (int e = tid; e <= E; e += kChunkThreads) out[e] = sh[e];
  if (a.tot) {
    // the source's totals: zeroed by k_zero, this kernel's predecessor
    griddep_wait();
    trace_first(a, ZB_TRACE_HIST + 1);
    int32_t* tot = a.tot + int64_t(i) * (E + 1);
    for (int e = tid; e <= E; e += kChunkThreads)
      if (sh[e]) atomicAdd(tot + e, sh[e]);
  }
  trace_last(a, ZB_TRACE_HIST + 2);
}

// Zeroes the per-source totals k_hist adds into (the first kernel of a plan
// on one GPU; k_hist, launched as its programmatic dependent, histograms its
// chunk before waiting for it).
__global__ void __launch_bounds__(kChunkThreads) k_zero(PlanArgs a, int n) {
  trace_first(a, ZB_TRACE_ZERO);
  trace_first(a, ZB_TRACE_ZERO + 1);
  griddep_launch_dependents();
  const int x = blockIdx.x * kChunkThreads + threadIdx.x;
  if (x < n) a.tot[x] = 0;
  trace_last(a, ZB_TRACE_ZERO + 2);
}

// The count row of one source, counts[e] = sum over its chunks of
// chunk_hist[c][e] (column E: ids outside [0, E)), one thread per column.
__global__ void __launch_bounds__(kPlanThreads) k_count_row(PlanArgs a, int32_t* counts) {
  griddep_wait();
  const int e = blockIdx.x * kPlanThreads + threadIdx.x;
  if (e <= a.E) counts[e] = strided_sum<16>(a.chunk_hist + e, a.nchunk, a.E + 1);
}

// ------------------------------------------------------------------ step 2+3

struct PlannerSmem {
  int32_t* cnt;    // [P*E]
  int32_t* hq;     // [E]   remaining home quota
  uint32_t* hold;  // [E]   ranks holding a replica of e (bit r)
  int32_t* repe;   // [P*R]
  int32_t* repq;   // [P*R]
  int32_t* cu;     // [P*(Eh+R+1)]
  int32_t* hoff;   // [E+1]
  int32_t* order;  // [E]   experts with replicas first, then the rest
  int32_t* q;      // [warps][32 hosts] remaining quota in transport
  int32_t* misc;   // [16]
  int32_t* M;      // [warps][32 hosts][32 sources]
  int16_t* qidx;   // [P*E] quota repair only: where rank r keeps its quota of
                   // e (e: hq[e]; E + x: repq[x]; -1: no copy)
};

__device__ PlannerSmem carve(char* base, const PlanArgs& a) {
  PlannerSmem s;
  int32_t* p = reinterpret_cast<int32_t*>(base);
  s.cnt = p; p += a.P * a.E;
  s.hq = p; p += a.E;
  s.hold = reinterpret_cast<uint32_t*>(p); p += a.E;
  s.repe = p; p += a.P * a.R;
  s.repq = p; p += a.P * a.R;
  s.cu = p; p += a.P * (a.Eh + a.R + 1);
  s.hoff = p; p += a.E + 1;
  s.order = p; p += a.E;
  s.q = p; p += kPlanWarps * 32;
  s.misc = p; p += 16;
  s.M = p; p += kPlanWarps * 32 * 32;
  s.qidx = reinterpret_cast<int16_t*>(p);
  return s;
}

enum {
  kMiscT = 0, kMiscMax = 1, kMiscNrep = 2, kMiscIters = 3, kMiscBad = 4, kMiscErr = 5,
  kMiscRecv = 6,      // banded plans: the most rows any rank receives
  kMiscRepaired = 7,  // rows moved by quota repair, per direction
  kMiscNRepExp = 8,   // experts with at least one replica (first in order)
  kMiscNextRep = 9    // next replicated expert a transport warp takes
};

// Greedy replica placement, run by one warp; lane r holds rank r's load,
// filled-slot count and stuck flag, and every decision is one or two warp
// reductions.  (ISER-MoE HALO-Q Objective 1 and stages 2-3; Zepp 4.1 R slots
// per GPU and node-first hierarchical placement.)
template <int kPolicy>
__device__ void greedy_warp(const PlanArgs& a, PlannerSmem& s, int T, int load, int lane) {
  const int P = a.P, R = a.R, Eh = a.Eh, gpn = a.gpn;
  int nfill = 0;
  bool stuck = lane >= P;
  int iters = 0;
  const int max_iters = P * R + P + 1;
  // mask of the ranks on lane's node
  const unsigned node_mask =
      gpn >= 32 ? kFull : (((1u << gpn) - 1u) << ((lane / gpn) * gpn));
  const int my_node = lane / gpn;
  for (int guard = 0; guard <= max_iters; ++guard) {
    // donor: the busiest non-stuck rank, ties to the lowest rank
    const unsigned dl = stuck ? 0u : unsigned(load) + 1u;
    const unsigned dmax = __reduce_max_sync(kFull, dl);
    if (dmax == 0u) break;
    const int d = __ffs(__ballot_sync(kFull, dl == dmax)) - 1;
    const int dload = int(dmax - 1u);
    if (dload <= T) break;
    ++iters;
    // receivers with room: not the donor, a free slot, load below T
    const unsigned base = __ballot_sync(kFull, lane < P && lane != d && nfill < R && load < T);
    // d's heaviest home expert (largest remaining quota, ties: lowest id)
    // that some rank in base can take (it holds no copy yet)
    unsigned bq = 0u, bx = 0xffffffffu, bh = 0u;
    for (int x = lane; x < Eh; x += 32) {
      const int e = d * Eh + x;
      const unsigned q = unsigned(s.hq[e]);
      const unsigned h = s.hold[e];
      if (q > 0u && (base & ~h) != 0u && q > bq) {
        bq = q;
        bx = unsigned(x);
        bh = h;
      }
    }
    const unsigned qmax = __reduce_max_sync(kFull, bq);
    if (qmax == 0u) {
      if (lane == d) stuck = true;
      continue;
    }
    const unsigned xmin = __reduce_min_sync(kFull, bq == qmax ? bx : 0xffffffffu);
    const int e = d * Eh + int(xmin);
    const int q = int(qmax);
    // the holders of e, from the lane that examined it (x = xmin there)
    const unsigned hold = __shfl_sync(kFull, bh, int(xmin & 31u));
    // receiver: a node without the expert first, then the lowest load, then
    // the lowest rank (e is homed on the donor d)
    const bool elig = ((base >> lane) & 1u) && !((hold >> lane) & 1u);
    const bool cov = (__shfl_sync(kFull, my_node, d) == my_node) || ((hold & node_mask) != 0u);
    int r, rload;
    if (kPolicy == ZB_POLICY_LOCAL) {
      // balance first, locality among equal moves (HALO-Q Objective 2): after
      // node coverage, the largest move m_r, then the most own rows the copy
      // would serve locally, min(cnt[r][e], m_r), then load and rank
      const int mr = min(min(dload - T, T - load), q);
      const int own = lane < P ? s.cnt[lane * a.E + e] : 0;
      const int gain = min(own, mr);
      const unsigned k1 =
          elig ? ((cov ? 0x80000000u : 0u) | unsigned(0x7fffffff - mr)) : 0xffffffffu;
      const unsigned k1min = __reduce_min_sync(kFull, k1);
      const bool c1 = elig && k1 == k1min;
      const unsigned k2 = c1 ? unsigned(0x7fffffff - gain) : 0xffffffffu;
      const unsigned k2min = __reduce_min_sync(kFull, k2);
      const bool c2 = c1 && k2 == k2min;
      const unsigned lmin = __reduce_min_sync(kFull, c2 ? unsigned(load) : 0xffffffffu);
      r = __ffs(__ballot_sync(kFull, c2 && unsigned(load) == lmin)) - 1;
      rload = int(lmin);
    } else {
      const unsigned rk = elig ? (unsigned(load) | (cov ? 0x80000000u : 0u)) : 0xffffffffu;
      const unsigned rmin = __reduce_min_sync(kFull, rk);
      r = __ffs(__ballot_sync(kFull, elig && rk == rmin)) - 1;
      rload = int(rmin & 0x7fffffffu);
    }
    int m = dload - T;
    m = min(m, T - rload);
    m = min(m, q);
    if (lane == r && ZB_IN(ZB_SITE_PLAN_SLOT, nfill, R)) {
      s.repe[r * R + nfill] = e;
      s.repq[r * R + nfill] = m;
      ++nfill;
      load += m;
    }
    if (lane == d) load -= m;
    if (lane == 0) {
      s.hq[e] = q - m;
      s.hold[e] = hold | (1u << r);
    }
    __syncwarp();
  }
  if (lane < P) a.load_after[lane] = load;
  const int mx = int(__reduce_max_sync(kFull, lane < P ? unsigned(load) : 0u));
  const int nrep = int(__reduce_add_sync(kFull, lane < P ? unsigned(nfill) : 0u));
  if (lane == 0) {
    s.misc[kMiscMax] = mx;
    s.misc[kMiscNrep] = nrep;
    s.misc[kMiscIters] = iters;
  }
}

// Quotas for a given replica placement, run by one warp: the greedy of
// greedy_warp restricted to copies that already exist (a receiver must hold
// the expert, and the move adds to that copy's quota), receivers by most room
// then lowest rank.  Each move brings the donor to T, fills the receiver to T
// or exhausts the expert's home quota: at most 3P + E iterations with the
// stuck marks.  (Zepp 4.1: replicas placed from historical demand; ViBE:
// placement recalibrated only on drift.)
// Returns this lane's rank load after the moves (lanes >= P: 0).
__device__ int greedy_placed_warp(const PlanArgs& a, PlannerSmem& s, int T, int load,
                                  int lane) {
  const int P = a.P, R = a.R, Eh = a.Eh;
  bool stuck = lane >= P;
  int iters = 0;
  const int max_iters = 3 * P + a.E + 1;
  for (int guard = 0; guard <= max_iters; ++guard) {
    const unsigned dl = stuck ? 0u : unsigned(load) + 1u;
    const unsigned dmax = __reduce_max_sync(kFull, dl);
    if (dmax == 0u) break;
    const int d = __ffs(__ballot_sync(kFull, dl == dmax)) - 1;
    const int dload = int(dmax - 1u);
    if (dload <= T) break;
    ++iters;
    const unsigned base = __ballot_sync(kFull, lane < P && lane != d && load < T);
    // d's heaviest home expert with a copy on some rank in base
    unsigned bq = 0u, bx = 0xffffffffu, bh = 0u;
    const int e0 = d * Eh;
    for (int x = lane; x < Eh; x += 32) {
      const unsigned q = unsigned(s.hq[e0 + x]);
      const unsigned h = s.hold[e0 + x];
      if (q > bq && (base & h) != 0u) {
        bq = q;
        bx = unsigned(x);
        bh = h;
      }
    }
    const unsigned qmax = __reduce_max_sync(kFull, bq);
    if (qmax == 0u) {
      if (lane == d) stuck = true;
      continue;
    }
    const unsigned xmin = __reduce_min_sync(kFull, bq == qmax ? bx : 0xffffffffu);
    const unsigned held = __shfl_sync(kFull, bh, int(xmin & 31u));
    const int e = e0 + int(xmin);
    const int q = int(qmax);
    const bool elig = ((base >> lane) & 1u) && ((held >> lane) & 1u);
    const unsigned rk = elig ? unsigned(load) : 0xffffffffu;
    const unsigned rmin = __reduce_min_sync(kFull, rk);
    const int r = __ffs(__ballot_sync(kFull, elig && rk == rmin)) - 1;
    const int m = min(min(dload - T, T - int(rmin)), q);
    if (lane == r) {
      for (int sl = 0; sl < R; ++sl)
        if (s.repe[r * R + sl] == e) s.repq[r * R + sl] += m;
      load += m;
    }
    if (lane == d) load -= m;
    if (lane == 0) s.hq[e] = q - m;
    __syncwarp();
  }
  int nrep = 0;
  if (lane < P)
    for (int sl = 0; sl < R; ++sl) nrep += s.repe[lane * R + sl] >= 0;
  const int mx = int(__reduce_max_sync(kFull, lane < P ? unsigned(load) : 0u));
  nrep = int(__reduce_add_sync(kFull, unsigned(nrep)));
  if (lane == 0) {
    s.misc[kMiscMax] = mx;
    s.misc[kMiscNrep] = nrep;
    s.misc[kMiscIters] = iters;
  }
  return lane < P ? load : 0;
}

// Quota of the copy at quota index x (x < E: home quota of x; else helper
// slot x - E).
__device__ __forceinline__ int32_t& quota_at(const PlanArgs& a, PlannerSmem& s, int x) {
  return x < a.E ? s.hq[x] : s.repq[x - a.E];
}

// Quota repair of one rank pair (i < j), run by one warp (ISER-MoE, HALO-Q
// stage 4).  The experts both ranks hold are i's helper copies of experts j
// holds, plus j's helper copies of experts homed on i: lane c < R takes i's
// slot c, lane R + c takes j's slot c (two rounds of lanes when 2R > 32).
// For each, a = min(surplus_i, spare_j) and b = min(surplus_j, spare_i);
// m = min(sum a, sum b) rows of quota move each way.  The side whose sum
// exceeds m is consumed in ascending expert order, the other in full.
// Both loads are unchanged.
__device__ void repair_pair_warp(const PlanArgs& a, PlannerSmem& s, int i, int j, int lane) {
  const int R = a.R, E = a.E, Eh = a.Eh, nc = 2 * R;
  const int nu = nc > 32 ? 2 : 1;
  int ce[2], ca[2], cb[2], xi[2], xj[2];
#pragma unroll
  for (int u = 0; u < 2; ++u) {
    ce[u] = -1;
    ca[u] = cb[u] = 0;
    xi[u] = xj[u] = 0;
    const int c = lane + 32 * u;
    if (u >= nu || c >= nc) continue;
    int e = c < R ? s.repe[i * R + c] : s.repe[j * R + (c - R)];
    if (e < 0) continue;
    if (c < R ? s.qidx[j * E + e] < 0 : e / Eh != i) continue;
    ce[u] = e;
    xi[u] = s.qidx[i * E + e];
    xj[u] = s.qidx[j * E + e];
    const int qi = quota_at(a, s, xi[u]), qj = quota_at(a, s, xj[u]);
    const int di = s.cnt[i * E + e], dj = s.cnt[j * E + e];
    ca[u] = min(max(di - qi, 0), max(qj - dj, 0));
    cb[u] = min(max(dj - qj, 0), max(qi - di, 0));
  }
  const int sa = int(__reduce_add_sync(kFull, unsigned(ca[0] + ca[1])));
  const int sb = int(__reduce_add_sync(kFull, unsigned(cb[0] + cb[1])));
  const int m = min(sa, sb);
  if (m == 0) return;
  int ta[2] = {ca[0], ca[1]}, tb[2] = {cb[0], cb[1]};
  if (sa != sb) {  // cut the larger side at m, in ascending expert order
    const bool cut_a = sa > m;
    int v[2] = {cut_a ? ca[0] : cb[0], cut_a ? ca[1] : cb[1]};
    int before[2] = {0, 0};
    for (int t = 0; t < nc; ++t) {
      const int et = __shfl_sync(kFull, t < 32 ? ce[0] : ce[1], t & 31);
      const int vt = __shfl_sync(kFull, t < 32 ? v[0] : v[1], t & 31);
#pragma unroll
      for (int u = 0; u < 2; ++u)
        if (et >= 0 && et < ce[u]) before[u] += vt;
    }
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int take = max(0, min(v[u], m - before[u]));
      if (cut_a)
        ta[u] = take;
      else
        tb[u] = take;
    }
  }
#pragma unroll
  for (int u = 0; u < 2; ++u)
    if (ce[u] >= 0 && (ta[u] | tb[u])) {
      quota_at(a, s, xi[u]) += ta[u] - tb[u];
      quota_at(a, s, xj[u]) += tb[u] - ta[u];
    }
  if (lane == 0) atomicAdd(&s.misc[kMiscRepaired], m);
}

// Host j's quota for expert e and the group that receives it on j.
__device__ __forceinline__ void host_quota(const PlanArgs& a, const PlannerSmem& s, int e,
                                           int h0, int j, int& q, int& grp) {
  if (j == h0) {
    q = s.hq[e];
    grp = e - h0 * a.Eh;
    return;
  }
  q = 0;
  grp = a.Eh;
  for (int r = 0; r < a.R; ++r)
    if (s.repe[j * a.R + r] == e) {
      q = s.repq[j * a.R + r];
      grp = a.Eh + r;
    }
}

// Flows of eq. (1) with exact quotas: every host receives exactly its quota.
// Own rank first (a = 0), then each cost level, hosts in ascending rank taking
// from sources in ascending rank.  Leaves this lane's column of Mw.
__device__ void flows_exact(const PlanArgs& a, PlannerSmem& s, int e, int h0,
                            unsigned hostmask, int nh, int d, int lane, int32_t* Mw,
                            int32_t* qw) {
  const int P = a.P, gpn = a.gpn;
  int dres = d;
  if (lane < P && ((hostmask >> lane) & 1u)) {
    int q, grp;
    host_quota(a, s, e, h0, lane, q, grp);
    const int my_t = __popc(hostmask & ((1u << lane) - 1u));
    const int take = min(dres, q);  // the host's own rank, a = 0
    Mw[my_t * 32 + lane] = take;
    dres -= take;
    qw[my_t] = q - take;
  }
  __syncwarp();
  const int nlev = gpn > 1 ? 2 : 1;
  for (int l = 0; l < nlev; ++l) {
    const int lev = l == 0 ? 1 : 4;
    unsigned hm = hostmask;
    for (int t = 0; t < nh; ++t) {
      const int j = __ffs(hm) - 1;
      hm &= hm - 1u;
      const int rem = qw[t];
      const int v = (lane < P && cost_a(lane, j, gpn, a.inv_gpn) == lev) ? dres : 0;
      const int inc = warp_incl_scan(v, lane);
      const int take = max(0, min(v, rem - (inc - v)));
      const int tot = int(__reduce_add_sync(kFull, unsigned(take)));
      Mw[t * 32 + lane] += take;
      dres -= take;
      __syncwarp();
      if (lane == 0) qw[t] = rem - tot;
      __syncwarp();
    }
  }
  if (__any_sync(kFull, dres != 0) && lane == 0) atomicExch(&s.misc[kMiscErr], 1);
}

// Flows of eq. (1) within its band: host j of quota q receives lo..hi rows,
// lo/hi = q -/+ floor(q * cfix / 2^20).  The slack sum(q) - sum(lo) is what
// may go above the lower bounds in total.  1: own rank up to lo; 2: hosts in
// ascending rank take more own rows, up to hi, while slack lasts; 3: each cost
// level, hosts in ascending rank, sources in ascending rank: up to lo, then up
// to hi while slack lasts.  Lane j keeps host j's bounds and receipt; returns
// the receipt (0 on other lanes) and its group in *grp_out.
__device__ int flows_band(const PlanArgs& a, PlannerSmem& s, int e, int h0, unsigned hostmask,
                          int nh, int d, int lane, int32_t* Mw, int* grp_out) {
  const int P = a.P, gpn = a.gpn;
  const bool host = lane < P && ((hostmask >> lane) & 1u);
  const int my_t = __popc(hostmask & ((1u << lane) - 1u));
  int dres = d, lo = 0, hi = 0, recv = 0, dl = 0, grp = -1;
  if (host) {
    int q;
    host_quota(a, s, e, h0, lane, q, grp);
    dl = int((long long)q * a.cfix >> 20);
    lo = q - dl;
    hi = q + dl;
    recv = min(dres, lo);  // 1: own rank up to the lower bound
    dres -= recv;
  }
  int slack = int(__reduce_add_sync(kFull, unsigned(dl)));
  {  // 2: own rank into the band, hosts in ascending rank
    const int want = host ? min(dres, hi - recv) : 0;
    const int inc = warp_incl_scan(want, lane);
    const int take = max(0, min(want, slack - (inc - want)));
    dres -= take;
    recv += take;
    slack -= int(__reduce_add_sync(kFull, unsigned(take)));
  }
  if (host) Mw[my_t * 32 + lane] = recv;
  __syncwarp();
  const int nlev = gpn > 1 ? 2 : 1;
  for (int l = 0; l < nlev; ++l) {  // 3: the other ranks, by cost level
    const int lev = l == 0 ? 1 : 4;
    unsigned hm = hostmask;
    for (int t = 0; t < nh; ++t) {
      const int j = __ffs(hm) - 1;
      hm &= hm - 1u;
      const int rj = __shfl_sync(kFull, recv, j);
      const int loj = __shfl_sync(kFull, lo, j);
      const int hij = __shfl_sync(kFull, hi, j);
      const int need = max(loj - rj, 0);
      const int avail = need + min(hij - max(rj, loj), slack);
      const int v = (lane < P && cost_a(lane, j, gpn, a.inv_gpn) == lev) ? dres : 0;
      const int inc = warp_incl_scan(v, lane);
      const int take = max(0, min(v, avail - (inc - v)));
      const int tot = int(__reduce_add_sync(kFull, unsigned(take)));
      Mw[t * 32 + lane] += take;
      dres -= take;
      if (lane == j) recv += tot;
      slack -= max(tot - need, 0);
    }
  }
  __syncwarp();
  const bool bad = dres != 0 || (host && (recv < lo || recv > hi));
  if (__any_sync(kFull, bad) && lane == 0) atomicExch(&s.misc[kMiscErr], 1);
  *grp_out = grp;
  return host ? recv : 0;
}

// From the flows in Mw: the locality cost of this source lane, and its
// segments of expert e in host order (a ascending, then rank), each (end
// position among the source's entries of e, first destination row).
__device__ long long emit_segments(const PlanArgs& a, const PlannerSmem& s, int e, int h0,
                                   unsigned hostmask, int nh, int lane, int32_t* Mw,
                                   int2* seg) {
  const int P = a.P, R = a.R, Eh = a.Eh, G = Eh + R, gpn = a.gpn;
  long long cost = 0;
  {
    unsigned hm = hostmask;
    for (int t = 0; t < nh; ++t) {
      const int j = __ffs(hm) - 1;
      hm &= hm - 1u;
      const int m = Mw[t * 32 + lane];
      cost += (long long)cost_a(lane, j, gpn, a.inv_gpn) * m;
      const int inc = warp_incl_scan(m, lane);
      __syncwarp();
      Mw[t * 32 + lane] = inc;  // inclusive prefix over sources
    }
    __syncwarp();
  }
  if (lane < P) {
    int idx = 0, cum = 0;
    for (int lv = 0; lv < 3; ++lv) {
      const int want = lv == 0 ? 0 : (lv == 1 ? 1 : 4);
      unsigned hm = hostmask;
      for (int t = 0; t < nh; ++t) {
        const int j = __ffs(hm) - 1;
        hm &= hm - 1u;
        if (cost_a(lane, j, gpn, a.inv_gpn) != want) continue;
        const int inc = Mw[t * 32 + lane];
        const int prev = lane > 0 ? Mw[t * 32 + lane - 1] : 0;
        int grp;
        if (j == h0) {
          grp = e - h0 * Eh;
        } else {
          grp = Eh;
          for (int r = 0; r < R; ++r)
            if (s.repe[j * R + r] == e) grp = Eh + r;
        }
        cum += inc - prev;
        if (ZB_IN(ZB_SITE_PLAN_SEGMENT, s.hoff[e] + idx, s.hoff[e + 1]))
          seg[idx] = make_int2(cum, j * a.cap + s.cu[j * (G + 1) + grp] + prev);
        ++idx;
      }
    }
  }
  __syncwarp();
  return cost;
}

// Transport of eq. (1) for expert e, run by one warp, lane = source rank.
// kEmit: write the source lane's segments of e into the segment table and
// return the lane's share of the locality cost.  Otherwise (banded plans
// only) record each host's receipt in s.cu[j][grp + 1]; the group offsets
// are known only once every expert's receipts are.
template <bool kBand, bool kEmit>
__device__ long long transport_warp(const PlanArgs& a, PlannerSmem& s, int e, int lane,
                                    int32_t* Mw, int32_t* qw) {
  const int P = a.P, Eh = a.Eh, G = Eh + a.R, gpn = a.gpn;
  const int h0 = div_small(e, a.inv_eh);
  const unsigned hold = s.hold[e];
  const int d = lane < P ? s.cnt[lane * a.E + e] : 0;
  int2* seg = a.seg + int64_t(lane) * a.seg_width + s.hoff[e];
  if (hold == 0u) {
    // the home rank is the only host: every source sends it all its rows
    if (!kEmit) {
      if (lane == 0) s.cu[h0 * (G + 1) + (e - h0 * Eh) + 1] = s.hq[e];
      return 0;
    }
    const int inc = warp_incl_scan(d, lane);
    if (lane < P && ZB_IN(ZB_SITE_PLAN_SEGMENT, s.hoff[e], s.hoff[e + 1]))
      seg[0] = make_int2(d, h0 * a.cap + s.cu[h0 * (G + 1) + (e - h0 * Eh)] + inc - d);
    return (long long)cost_a(lane, h0, gpn, a.inv_gpn) * d;
  }
  const unsigned hostmask = hold | (1u << h0);
  const int nh = __popc(hostmask);
  for (int t = 0; t < nh; ++t) Mw[t * 32 + lane] = 0;
  __syncwarp();
  if (kBand) {
    int grp;
    const int recv = flows_band(a, s, e, h0, hostmask, nh, d, lane, Mw, &grp);
    if (!kEmit) {
      if (lane < P && ((hostmask >> lane) & 1u)) s.cu[lane * (G + 1) + grp + 1] = recv;
      __syncwarp();
      return 0;
    }
  } else {
    flows_exact(a, s, e, h0, hostmask, nh, d, lane, Mw, qw);
  }
  return emit_segments(a, s, e, h0, hostmask, nh, lane, Mw, seg);
}

// One instance per greedy mode (kMode: 0 room, 1 local, 2 kept placement),
// quota repair (kRepair) and transport (kBand: quotas exact, or within eq.
// (1)'s band), so that each instance carries only the code it runs.
template <int kMode, bool kRepair, bool kBand>
__global__ void __launch_bounds__(kPlanThreads, 1) k_planner(PlanArgs a) {
  extern __shared__ __align__(16) char smem_raw[];
  __shared__ unsigned long long s_cost;
  __shared__ int s_wsum[3][kPlanWarps];  // per warp of experts: hosts, replicated, home-only
  PlannerSmem s = carve(smem_raw, a);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int P = a.P, E = a.E, R = a.R, Eh = a.Eh, G = Eh + R;
  // the chunk histograms are read once k_hist has completed; from then on
  // the assignment CTAs may launch (they read their ids and the chunk
  // histograms before waiting for this plan)
  trace_first(a, ZB_TRACE_PLANNER);
  griddep_wait();
  trace_first(a, ZB_TRACE_PLANNER + 1);
  griddep_launch_dependents();

  // route counts cnt[i][e] and ids outside [0, E), one row per source
  if (tid == 0) {
    s.misc[kMiscBad] = 0;
    s.misc[kMiscErr] = 0;
    s.misc[kMiscRepaired] = 0;
    s.misc[kMiscNextRep] = 0;
    s_cost = 0ull;
  }
  __syncthreads();
  const float inv_e1 = 1.0f / float(E + 1);  // for div_small: x < 32 * 385 < 2^22
  for (int x0 = tid; x0 < P * (E + 1); x0 += 8 * kPlanThreads) {
    int v[8];  // eight columns of the table per thread in flight
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int x = x0 + u * kPlanThreads;
      v[u] = x < P * (E + 1) ? __ldcg(a.plan_hist + x) : 0;
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int x = x0 + u * kPlanThreads;
      if (x >= P * (E + 1)) break;
      const int i = div_small(x, inv_e1), e = x - i * (E + 1);
      if (e < E) {
        s.cnt[i * E + e] = v[u];
        a.cnt[i * E + e] = v[u];
      } else if (v[u]) {
        atomicAdd(&s.misc[kMiscBad], v[u]);
      }
    }
  }
  if (a.own_hist) {
    // exchanged count rows (one rank of P GPUs): this rank's row must be the
    // count of its own ids, and every row must be S*K non-negative counts
    for (int e = tid; e <= E; e += kPlanThreads) {
      const int own = strided_sum<16>(a.own_hist + e, a.nchunk, E + 1);
      if (own != a.plan_hist[int64_t(a.src0) * (E + 1) + e]) atomicExch(&s.misc[kMiscErr], 1);
    }
    for (int i = warp; i < P; i += kPlanWarps) {
      long long sum = 0;
      bool neg = false;
      for (int e = lane; e <= E; e += 32) {
        const int v = a.plan_hist[int64_t(i) * (E + 1) + e];
        neg = neg || v < 0;
        sum += v;
      }
      sum = warp_sum64(sum);
      if ((__any_sync(kFull, neg) || sum != (long long)a.S * a.K) && lane == 0)
        atomicExch(&s.misc[kMiscErr], 1);
    }
  }
  // the replica table: empty, or the placement to keep (checked: each slot
  // empty or an expert homed elsewhere, no expert twice on a rank)
  for (int x = tid; x < P * R; x += kPlanThreads) {
    int e = -1;
    if (kMode == 2) {
      e = a.placement[x];
      const int j = x / R, sl = x - j * R;
      bool ok = e == -1 || (e >= 0 && e < E && e / Eh != j);
      for (int t = 0; t < sl && ok; ++t) ok = a.placement[j * R + t] != e || e == -1;
      if (!ok) atomicExch(&s.misc[kMiscErr], 1);
    }
    s.repe[x] = e;
    s.repq[x] = 0;
  }
  __syncthreads();
  if (s.misc[kMiscErr]) {
    if (tid == 0) {
      for (int k = 0; k < ZB_STATS_LEN; ++k) a.stats[k] = 0;
      a.stats[ZB_STAT_STATUS] = ZB_ERR_INVALID;
    }
    trace_last(a, ZB_TRACE_PLANNER + 2);
    return;
  }
  const int bad = s.misc[kMiscBad];
  if (bad) {
    if (tid == 0) {
      for (int k = 0; k < ZB_STATS_LEN; ++k) a.stats[k] = 0;
      a.stats[ZB_STAT_STATUS] = ZB_ERR_BAD_ID;
      a.stats[ZB_STAT_BAD_IDS] = bad;
    }
    trace_last(a, ZB_TRACE_PLANNER + 2);
    return;
  }
  // T_e, the initial home quotas, and the holders of each placed copy
  for (int e = tid; e < E; e += kPlanThreads) {
    int t = 0;
    for (int i = 0; i < P; ++i) t += s.cnt[i * E + e];
    s.hq[e] = t;
    s.hold[e] = 0u;
  }
  __syncthreads();
  if (kMode == 2)
    for (int x = tid; x < P * R; x += kPlanThreads)
      if (s.repe[x] >= 0 && ZB_IN(ZB_SITE_PLAN_SLOT, s.repe[x], E))
        atomicOr(&s.hold[s.repe[x]], 1u << (x / R));
  __syncthreads();

  if (warp == 0) {
    // L_j and the water level T = ceil(sum_r L_r / P)
    int L = 0;
    if (lane < P)
      for (int e = lane * Eh; e < (lane + 1) * Eh; ++e) L += s.hq[e];
    if (lane < P) a.load_before[lane] = L;
    // sum_r L_r = P*S*K (or the exchanged rows' total), which the validation
    // keeps below 2^31: 32-bit arithmetic suffices
    const int total = int(__reduce_add_sync(kFull, lane < P ? unsigned(L) : 0u));
    const int T = (total + P - 1) / P;
    if (lane == 0) s.misc[kMiscT] = T;
    if (kMode == 2) {
      const int load = greedy_placed_warp(a, s, T, L, lane);
      if (lane < P) a.load_after[lane] = load;
    } else
      greedy_warp<kMode>(a, s, T, L, lane);
  }
  __syncthreads();

  if (kRepair) {
    for (int x = tid; x < P * E; x += kPlanThreads) s.qidx[x] = -1;
    __syncthreads();
    for (int e = tid; e < E; e += kPlanThreads) s.qidx[(e / Eh) * E + e] = int16_t(e);
    for (int x = tid; x < P * R; x += kPlanThreads)
      if (s.repe[x] >= 0) s.qidx[(x / R) * E + s.repe[x]] = int16_t(E + x);
    __syncthreads();
    // circle method: ranks 0..Pp-1 (rank P is a bye when P is odd); round r
    // pairs Pp-1 with r and (r+k) mod (Pp-1) with (r-k) mod (Pp-1); the pairs
    // of a round are disjoint, one warp each
    const int Pp = P + (P & 1);
    for (int r = 0; r < Pp - 1; ++r) {
      for (int k = warp; k < Pp / 2; k += kPlanWarps) {
        const int x = k == 0 ? Pp - 1 : (r + k) % (Pp - 1);
        const int y = k == 0 ? r : (r - k + (Pp - 1)) % (Pp - 1);
        if (x < P && y < P) repair_pair_warp(a, s, min(x, y), max(x, y), lane);
      }
      __syncthreads();
    }
  }

  const int T = s.misc[kMiscT];
  const int max_load = s.misc[kMiscMax];
  for (int e = tid; e < E; e += kPlanThreads) a.home_quota[e] = s.hq[e];
  for (int x = tid; x < P * R; x += kPlanThreads) {
    a.rep_expert[x] = s.repe[x];
    a.rep_quota[x] = s.repq[x];
  }
  // hosts per expert and their first segment index, and the transport
  // order: experts with replicas (the long case) first, so that they land on
  // different warps, then the experts served by home alone, each by expert
  // id.  Warp w scans experts [32w, 32w + 32) (E <= kMaxE = 12 warps of
  // them), then adds the totals of the warps before it.
  static_assert(kMaxE <= 32 * kPlanWarps, "one warp per 32 experts");
  const int nwe = (E + 31) / 32;
  const int e_mine = warp * 32 + lane;
  const bool e_in = warp < nwe && e_mine < E;
  const int nh = e_in ? 1 + __popc(s.hold[e_mine]) : 0;
  const bool rep = nh > 1;
  int nh_inc = 0;
  unsigned m_rep = 0u, m_home = 0u;
  if (warp < nwe) {
    nh_inc = warp_incl_scan(nh, lane);
    m_rep = __ballot_sync(kFull, rep);
    m_home = __ballot_sync(kFull, e_in && !rep);
    if (lane == 31) s_wsum[0][warp] = nh_inc;
    if (lane == 0) {
      s_wsum[1][warp] = __popc(m_rep);
      s_wsum[2][warp] = __popc(m_home);
    }
  }
  __syncthreads();
  if (warp < nwe) {
    int off_h = 0, off_r = 0, off_o = 0, nrx = 0;
    for (int w = 0; w < nwe; ++w) {
      if (w < warp) {
        off_h += s_wsum[0][w];
        off_r += s_wsum[1][w];
        off_o += s_wsum[2][w];
      }
      nrx += s_wsum[1][w];
    }
    if (e_in) s.hoff[e_mine] = off_h + nh_inc - nh;
    if (warp == nwe - 1 && lane == 31) s.hoff[E] = off_h + nh_inc;
    const unsigned below = (1u << lane) - 1u;
    if (rep) s.order[off_r + __popc(m_rep & below)] = e_mine;
    if (e_in && !rep) s.order[nrx + off_o + __popc(m_home & below)] = e_mine;
    if (warp == 0 && lane == 0) s.misc[kMiscNRepExp] = nrx;
  }
  int32_t* Mw = s.M + warp * 32 * 32;
  int32_t* qw = s.q + warp * 32;
  // cu_seqlens: exclusive prefix of each rank's group receipts.  Exact quotas
  // are the receipts; in a band they are known after a first transport pass.
  if (kBand)
    for (int x = tid; x < P * (G + 1); x += kPlanThreads) s.cu[x] = 0;
  __syncthreads();
  if (kBand)
    for (int k = warp; k < E; k += kPlanWarps)
      transport_warp<true, false>(a, s, s.order[k], lane, Mw, qw);
  __syncthreads();
  for (int j = warp; j < P; j += kPlanWarps) {
    int carry = 0;
    int32_t* cu = s.cu + j * (G + 1);
    for (int g0 = 0; g0 < G; g0 += 32) {
      const int g = g0 + lane;
      int v = 0;
      if (g < G) {
        if (kBand)
          v = cu[g + 1];
        else
          v = g < Eh ? s.hq[j * Eh + g] : s.repq[j * R + (g - Eh)];
      }
      const int inc = warp_incl_scan(v, lane);
      __syncwarp();
      if (g < G) cu[g + 1] = carry + inc;
      carry += __shfl_sync(kFull, inc, 31);
    }
    if (lane == 0) cu[0] = 0;
  }
  __syncthreads();
  if (kBand && warp == 0) {
    const int v = lane < P ? s.cu[lane * (G + 1) + G] : 0;
    if (lane < P) a.load_after[lane] = v;
    const int mx = int(__reduce_max_sync(kFull, unsigned(v)));
    if (lane == 0) s.misc[kMiscRecv] = mx;
  }
  for (int x = tid; x < P * (G + 1); x += kPlanThreads) a.cu_seqlens[x] = s.cu[x];
  for (int e = tid; e <= E; e += kPlanThreads) a.hoff[e] = s.hoff[e];
  __syncthreads();

  const int rows_max = kBand ? s.misc[kMiscRecv] : max_load;
  const bool capacity = rows_max > a.cap;
  long long cost_part = 0;
  if (!capacity) {
    // experts with replicas: the transport of eq. (1), one warp each; a warp
    // takes the next expert when it is done with one, so that experts with
    // many sources or hosts do not leave the other warps idle
    const int nrx = s.misc[kMiscNRepExp];
    for (;;) {
      int k = 0;
      if (lane == 0) k = atomicAdd(&s.misc[kMiscNextRep], 1);
      k = __shfl_sync(kFull, k, 0);
      if (k >= nrx) break;
      cost_part += transport_warp<kBand, true>(a, s, s.order[k], lane, Mw, qw);
    }
    // experts served by their home rank alone: every source sends it all its
    // rows, one segment per source; a thread per expert walks the sources
    // in rank order (the same segments transport_warp's home-only case
    // writes, without a warp scan per expert).  Threads take them from the
    // top of the block down: the replicated experts above tend to go to the
    // warps that reach the counter first, most often the low ones.
    for (int k = nrx + (kPlanThreads - 1 - tid); k < E; k += kPlanThreads) {
      const int e = s.order[k];
      const int h0 = div_small(e, a.inv_eh);
      const int base = h0 * a.cap + s.cu[h0 * (G + 1) + (e - h0 * Eh)];
      const int h = s.hoff[e];
      const bool in = ZB_IN(ZB_SITE_PLAN_SEGMENT, h, s.hoff[e + 1]);
      int run = 0;
      for (int i = 0; i < P; ++i) {
        const int d = s.cnt[i * E + e];
        if (in) a.seg[int64_t(i) * a.seg_width + h] = make_int2(d, base + run);
        cost_part += (long long)cost_a(i, h0, a.gpn, a.inv_gpn) * d;
        run += d;
      }
    }
  }
  cost_part = warp_sum64(cost_part);
  if (lane == 0) atomicAdd(&s_cost, (unsigned long long)cost_part);
  __syncthreads();
  if (tid == 0) {
    int status = ZB_OK;
    if (capacity)
      status = ZB_ERR_CAPACITY;
    else if (s.misc[kMiscErr])
      status = ZB_ERR_INVALID;  // unreachable: the transport always closes
    else if (max_load > T)
      status = ZB_WARN_UNBALANCED;
    a.stats[ZB_STAT_STATUS] = status;
    a.stats[ZB_STAT_MAX_LOAD] = rows_max;
    a.stats[ZB_STAT_N_REPLICAS] = s.misc[kMiscNrep];
    a.stats[ZB_STAT_N_ITERS] = s.misc[kMiscIters];
    a.stats[ZB_STAT_WATER_LEVEL] = T;
    a.stats[ZB_STAT_LOCALITY_COST] = capacity ? 0 : (long long)s_cost;
    a.stats[ZB_STAT_BAD_IDS] = 0;
    a.stats[ZB_STAT_REPAIRED] = s.misc[kMiscRepaired];
  }
  trace_last(a, ZB_TRACE_PLANNER + 2);
}

// ------------------------------------------------------------------ step 3

constexpr int kAssignWarps = kChunkThreads / 32;
constexpr int kPerWarp = kChunk / kAssignWarps;  // kPerThread steps of 32

// One CTA per (a.assign_sub consecutive chunks, source rank i).  The host
// gives a CTA several chunks when one per CTA would not fit on the device at
// once, so that every CTA does its share of the work below while the planner
// runs.  Within a chunk, warp w owns entries [kPerWarp*w, kPerWarp*(w+1)) and
// walks them 32 at a time in flat order, so ranks among equal experts come
// out in flat-index order.  Each entry's rank within the source's entries of
// its expert (earlier chunks, earlier warps, the warp's earlier slices,
// lower lanes) depends on nothing the planner writes, so it is complete
// before the wait, and staged in shared memory with the entry's expert;
// after the wait only the segment lookup and the stores remain.
__global__ void __launch_bounds__(kChunkThreads, 2) k_assign(PlanArgs a) {
  __shared__ int32_t wh[kAssignWarps][kMaxE];  // per-warp counts, then bases
  __shared__ int32_t s_run[kMaxE];             // prefix of the chunks before
  __shared__ int32_t s_hoff[kMaxE + 1];
  __shared__ int2 s_seg[kMaxSegWidth];
  extern __shared__ int32_t s_ent[];  // per chunk: kChunk experts, kChunk ranks
  trace_first(a, ZB_TRACE_ASSIGN);
  const int nsub = a.assign_sub, c0 = blockIdx.x * nsub, il = blockIdx.y, i = a.src0 + il,
            tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int E = a.E;
  const int64_t nk = int64_t(a.S) * a.K;
  const int w0 = warp * kPerWarp;
  const int32_t* hist = a.chunk_hist + int64_t(il) * a.nchunk * (E + 1);

  for (int sub = 0; sub < nsub && c0 + sub < a.nchunk; ++sub) {
    const int c = c0 + sub;
    const int64_t start = int64_t(c) * kChunk;
    const int n = (nk - start) < kChunk ? int(nk - start) : kChunk;
    const int32_t* src = a.ids + int64_t(il) * nk + start;
    // ids outside [0, E) become -1 here: they are counted by k_hist and stop
    // the plan (ZB_ERR_BAD_ID) before any row is written, and no table below
    // is indexed by them
    int ids[kPerThread];
#pragma unroll
    for (int u = 0; u < kPerThread; ++u) {
      const int t = w0 + 32 * u + lane;
      const int v = t < n ? __ldg(src + t) : -1;
      ids[u] = unsigned(v) < unsigned(E) && ZB_IN(ZB_SITE_ASSIGN_EXPERT, v, kMaxE) ? v : -1;
    }
    for (int x = tid; x < kAssignWarps * kMaxE; x += kChunkThreads) (&wh[0][0])[x] = 0;
    __syncthreads();

    // pass 1: each entry's rank among the warp's entries of its expert so
    // far, and the per-warp histogram
    int pos[kPerThread];
#pragma unroll
    for (int u = 0; u < kPerThread; ++u) {
      const int e = ids[u];
      const unsigned peers = __match_any_sync(kFull, e);
      pos[u] = e >= 0 ? wh[warp][e] + __popc(peers & ((1u << lane) - 1u)) : 0;
      __syncwarp();
      if (e >= 0 && lane == __ffs(peers) - 1) wh[warp][e] += __popc(peers);
      __syncwarp();
    }
    __syncthreads();
    // exclusive prefix: earlier chunks of this source, then earlier warps.
    // The chunk histograms are complete: the planner launches this kernel
    // only after its own wait on k_hist has returned.  The first chunk of
    // the CTA sums the chunk histograms before it; each next one adds the
    // chunk just done.
    for (int e = tid; e < E; e += kChunkThreads) {
      int run = sub == 0 ? strided_sum<16>(hist + e, c, E + 1) : s_run[e];
#pragma unroll
      for (int w = 0; w < kAssignWarps; ++w) {
        const int v = wh[w][e];
        wh[w][e] = run;
        run += v;
      }
      s_run[e] = run;
    }
    __syncthreads();
    int32_t* ent = s_ent + sub * 2 * kChunk;
#pragma unroll
    for (int u = 0; u < kPerThread; ++u) {
      const int t = w0 + 32 * u + lane;
      ent[t] = ids[u];
      ent[kChunk + t] = ids[u] >= 0 ? pos[u] + wh[warp][ids[u]] : 0;
    }
    __syncthreads();  // wh is zeroed again for the next chunk
  }

  griddep_wait();  // the planner has completed: its tables are visible
  trace_first(a, ZB_TRACE_ASSIGN + 1);
  // the plan's status and the tables this CTA reads, fetched together
  const int64_t status = a.stats[ZB_STAT_STATUS];
  for (int e = tid; e <= E; e += kChunkThreads) s_hoff[e] = a.hoff[e];
  const int2* segrow = a.seg + int64_t(i) * a.seg_width;
  for (int x = tid; x < a.seg_width; x += kChunkThreads) s_seg[x] = segrow[x];
  __syncthreads();
  if (status < 0) {  // bad ids or capacity: no rows
    trace_last(a, ZB_TRACE_ASSIGN + 2);
    return;
  }
  // pass 2: each entry's segment (the host its rank falls in) and row
  const int64_t nrows = int64_t(a.P) * a.cap;
  for (int sub = 0; sub < nsub && c0 + sub < a.nchunk; ++sub) {
    const int64_t start = int64_t(c0 + sub) * kChunk;
    const int32_t* ent = s_ent + sub * 2 * kChunk;
#pragma unroll
    for (int u = 0; u < kPerThread; ++u) {
      const int t = w0 + 32 * u + lane;
      const int e = ent[t];
      if (e < 0) continue;
      const int p = ent[kChunk + t];
      const int h_end = s_hoff[e + 1];
      int prev = 0, row = -1;
      for (int h = s_hoff[e]; h < h_end; ++h) {
        if (!ZB_IN(ZB_SITE_ASSIGN_SEGMENT, h, a.seg_width)) break;
        const int2 sg = s_seg[h];
        if (p < sg.x) {
          row = sg.y + (p - prev);
          break;
        }
        prev = sg.x;
      }
      if (!ZB_IN(ZB_SITE_ASSIGN_ROW, row, nrows)) row = -1;
      const int64_t f = start + t;
      a.dst_row[int64_t(il) * nk + f] = row;
      if (a.row_src && row >= 0 && int64_t(row) < nrows)
        a.row_src[row] = int32_t(int64_t(i) * nk + f);
    }
  }
  trace_last(a, ZB_TRACE_ASSIGN + 2);
}

// ------------------------------------------------ placement recalibration

// Candidate placements scored by the kept-placement greedy, one warp each:
// candidate 0 is the base placement; in mode 0 candidate 1 + x*E + e puts
// expert e into helper slot x; in mode 1 candidate 1 + x1*(P*R) + x2 (x1 <
// x2, ranks of one node) exchanges the experts of slots x1 and x2.  An
// invalid candidate scores INT32_MAX.  The score is the plan's max rank load
// (ViBE, Drift-Aware Recalibration; Zepp 4.3, eq. (4)).
__global__ void __launch_bounds__(kEvalThreads) k_eval_placements(EvalArgs ea) {
  extern __shared__ __align__(16) char smem_raw[];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t c = int64_t(blockIdx.x) * kEvalWarps + warp;
  if (c >= ea.ncand) return;
  const int P = ea.P, E = ea.E, R = ea.R, Eh = E / P, n = P * R, gpn = ea.gpn;
  const int words = 2 * E + 2 * n + 16;
  int32_t* base = reinterpret_cast<int32_t*>(smem_raw) + warp * words;
  PlannerSmem s{};
  s.hq = base;
  s.hold = reinterpret_cast<uint32_t*>(base + E);
  s.repe = base + 2 * E;
  s.repq = base + 2 * E + n;
  s.misc = base + 2 * E + 2 * n;
  // the candidate's change: slot xa gets ea_e (and slot xb gets eb_e)
  int xa = -1, xb = -1, ea_e = -1, eb_e = -1;
  bool ok = true;
  if (c > 0) {
    const int64_t k = c - 1;
    if (ea.mode == 0) {
      xa = int(k / E);
      ea_e = int(k - int64_t(xa) * E);
      ok = ea_e != ea.base[xa];
    } else {
      xa = int(k / n);
      xb = int(k - int64_t(xa) * n);
      ea_e = ea.base[xb];
      eb_e = ea.base[xa];
      const int ra = xa / R, rb = xb / R;
      ok = xa < xb && ra != rb && ra / gpn == rb / gpn && ea_e != eb_e;
    }
  }
  for (int x = lane; x < n; x += 32) {
    s.repe[x] = x == xa ? ea_e : (x == xb ? eb_e : ea.base[x]);
    s.repq[x] = 0;
  }
  __syncwarp();
  // a changed slot may hold its expert only if the expert is homed elsewhere
  // and no other slot of that rank holds it
  auto takes = [&](int x) {
    const int e = s.repe[x];
    if (e < 0) return true;
    const int r = x / R;
    if (e / Eh == r) return false;
    for (int t = r * R; t < r * R + R; ++t)
      if (t != x && s.repe[t] == e) return false;
    return true;
  };
  if (ok && c > 0) ok = takes(xa) && (xb < 0 || takes(xb));
  if (!ok) {
    if (lane == 0) ea.out[c] = INT32_MAX;
    return;
  }
  for (int e = lane; e < E; e += 32) {
    s.hq[e] = ea.Te[e];
    s.hold[e] = 0u;
  }
  __syncwarp();
  for (int x = lane; x < n; x += 32)
    if (s.repe[x] >= 0 && ZB_IN(ZB_SITE_PLAN_SLOT, s.repe[x], E))
      atomicOr(&s.hold[s.repe[x]], 1u << (x / R));
  __syncwarp();
  int L = 0;
  if (lane < P)
    for (int e = lane * Eh; e < (lane + 1) * Eh; ++e) L += s.hq[e];
  const long long total = warp_sum64(lane < P ? (long long)L : 0ll);
  const int T = int((total + P - 1) / P);
  PlanArgs a{};
  a.P = P; a.E = E; a.R = R; a.Eh = Eh;
  greedy_placed_warp(a, s, T, L, lane);
  if (lane == 0) ea.out[c] = s.misc[kMiscMax];
}

}  // namespace

size_t planner_smem_bytes(const zb_config& c) {
  const int Eh = c.E / c.P;
  size_t words = size_t(c.P) * c.E + 2 * size_t(c.E) + 2 * size_t(c.P) * c.R +
                 size_t(c.P) * (Eh + c.R + 1) + size_t(c.E + 1) + size_t(c.E) +
                 kPlanWarps * 32 + 16;
  words += size_t(kPlanWarps) * 32 * 32;
  size_t bytes = words * sizeof(int32_t);
  if (c.repair) bytes += sizeof(int16_t) * size_t(c.P) * c.E;  // qidx
  return bytes;
}

cudaError_t launch_hist(const PlanArgs& a, int nsrc, cudaStream_t s) {
  if (a.nchunk == 0 || nsrc == 0) return cudaSuccess;
  k_hist<<<dim3(a.nchunk, nsrc), kChunkThreads, 0, s>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_trace_reset(unsigned long long* trace, cudaStream_t s) {
  k_trace_reset<<<1, 32, 0, s>>>(trace);
  return cudaGetLastError();
}

cudaError_t launch_hist_totals(const PlanArgs& a, int nsrc, cudaStream_t s) {
  const int n = nsrc * (a.E + 1);
  k_zero<<<(n + kChunkThreads - 1) / kChunkThreads, kChunkThreads, 0, s>>>(a, n);
  cudaError_t err = cudaGetLastError();
  if (err != cudaSuccess || a.nchunk == 0 || nsrc == 0) return err;
  return launch_pdl(k_hist, dim3(a.nchunk, nsrc), dim3(kChunkThreads), 0, s, a);
}

cudaError_t launch_count_row(const PlanArgs& a, int32_t* counts, cudaStream_t s) {
  const int blocks = (a.E + 1 + kPlanThreads - 1) / kPlanThreads;
  return launch_pdl(k_count_row, dim3(blocks), dim3(kPlanThreads), 0, s, a, counts);
}

template <int kMode, bool kRepair, bool kBand>
cudaError_t launch_planner_mode(const PlanArgs& a, size_t smem, cudaStream_t s) {
  static std::atomic<bool> configured[64];
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!configured[dev].load(std::memory_order_acquire)) {
    err = cudaFuncSetAttribute(k_planner<kMode, kRepair, kBand>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024);
    if (err != cudaSuccess) return err;
    configured[dev].store(true, std::memory_order_release);
  }
  return launch_pdl(k_planner<kMode, kRepair, kBand>, dim3(1), dim3(kPlanThreads), smem, s, a);
}

template <bool kRepair, bool kBand>
cudaError_t launch_planner_variant(const PlanArgs& a, size_t smem, cudaStream_t s) {
  if (a.placement) return launch_planner_mode<2, kRepair, kBand>(a, smem, s);
  if (a.policy == ZB_POLICY_LOCAL)
    return launch_planner_mode<ZB_POLICY_LOCAL, kRepair, kBand>(a, smem, s);
  return launch_planner_mode<ZB_POLICY_ROOM, kRepair, kBand>(a, smem, s);
}

cudaError_t launch_planner(const PlanArgs& a, size_t smem, cudaStream_t s) {
  if (a.repair)
    return a.relax ? launch_planner_variant<true, true>(a, smem, s)
                   : launch_planner_variant<true, false>(a, smem, s);
  return a.relax ? launch_planner_variant<false, true>(a, smem, s)
                 : launch_planner_variant<false, false>(a, smem, s);
}

size_t eval_smem_bytes(int P, int E, int R) {
  return size_t(kEvalWarps) * size_t(2 * E + 2 * P * R + 16) * sizeof(int32_t);
}

cudaError_t launch_eval_placements(const EvalArgs& ea, cudaStream_t s) {
  if (ea.ncand == 0) return cudaSuccess;
  const size_t smem = eval_smem_bytes(ea.P, ea.E, ea.R);
  static std::atomic<bool> configured[64];
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!configured[dev].load(std::memory_order_acquire)) {
    err = cudaFuncSetAttribute(k_eval_placements, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               200 * 1024);
    if (err != cudaSuccess) return err;
    configured[dev].store(true, std::memory_order_release);
  }
  const int64_t blocks = (ea.ncand + kEvalWarps - 1) / kEvalWarps;
  k_eval_placements<<<unsigned(blocks), kEvalThreads, smem, s>>>(ea);
  return cudaGetLastError();
}

// Chunks per assignment CTA: the fewest (at most kMaxAssignSub) with which
// every CTA of the grid fits on the device at once, beside the planner's CTA,
// from the occupancy of k_assign at each staging size (computed once per
// device).
int assign_sub(int nchunk, int nsrc) {
  constexpr int kMaxDevices = 64;
  static std::mutex mu;
  static int resident[kMaxDevices][kMaxAssignSub + 1];
  static bool known[kMaxDevices];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 1;
  int local[kMaxAssignSub + 1] = {};
  int* res = dev < kMaxDevices ? resident[dev] : local;
  {
    std::lock_guard<std::mutex> lock(mu);
    if (dev >= kMaxDevices || !known[dev]) {
      int sms = 0;
      if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
          cudaFuncSetAttribute(k_assign, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               int(assign_smem_bytes(kMaxAssignSub))) != cudaSuccess)
        return 1;
      for (int sub = 1; sub <= kMaxAssignSub; ++sub) {
        int per_sm = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k_assign, kChunkThreads,
                                                          assign_smem_bytes(sub)) !=
            cudaSuccess)
          return 1;
        res[sub] = per_sm * (sms - 1);  // the planner's CTA holds one SM meanwhile
      }
      if (dev < kMaxDevices) known[dev] = true;
    }
  }
  for (int sub = 1; sub <= kMaxAssignSub; ++sub)
    if (ceil_div(nchunk, sub) * nsrc <= res[sub]) return sub;
  return kMaxAssignSub;
}

cudaError_t launch_assign(const PlanArgs& a, int nsrc, cudaStream_t s) {
  if (a.nchunk == 0 || nsrc == 0) return cudaSuccess;
  PlanArgs b = a;
  b.assign_sub = assign_sub(a.nchunk, nsrc);
  return launch_pdl(k_assign, dim3(unsigned(ceil_div(a.nchunk, b.assign_sub)), nsrc),
                    dim3(kChunkThreads), assign_smem_bytes(b.assign_sub), s, b);
}

}  // namespace zb
