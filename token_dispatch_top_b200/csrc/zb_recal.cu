// zb_recal.cu -- replica placement between invocations.
//   zb_place_by_demand  a placement from historical per-expert demand (host
//                       only: a few hundred picks over at most 384 experts)
//   zb_recalibrate      recalibration of a kept placement; with
//                       zb_plan_status the only calls that synchronise their
//                       stream: every step reads the scores of all candidates
//                       back to the host to pick one, and the host keeps the
//                       placement being changed (in host memory it allocates)
//
// Sources: Zepp, "4.1 Expert Placement and Token Routing" (R slots per GPU
// given to the experts of highest historical demand per replica, spread
// round-robin over nodes, then over a node's GPUs); ViBE, "Drift-Aware
// Recalibration" (incremental placement update:
// from the current placement, minimal cross-GPU expert swaps until every GPU
// is within eps of the mean); Zepp, "4.3 Three-Stream Scheduling", eq. (4)
// (intra-node swaps of expert replicas that keep node-level coverage).
#include <algorithm>
#include <climits>
#include <cstring>
#include <vector>

#include "zb_internal.cuh"

namespace {

int64_t candidates(const zb_config& c, int mode) {
  const int64_t n = int64_t(c.P) * c.R;
  return 1 + (mode == 0 ? n * c.E : n * n);
}

// The rules of a replica placement: each slot empty or an expert homed on
// another rank, no expert twice on one rank.
bool placement_ok(const zb_config& c, const std::vector<int32_t>& pl) {
  const int Eh = c.E / c.P;
  for (int j = 0; j < c.P; ++j)
    for (int s = 0; s < c.R; ++s) {
      const int e = pl[j * c.R + s];
      if (e == -1) continue;
      if (e < 0 || e >= c.E || e / Eh == j) return false;
      for (int t = 0; t < s; ++t)
        if (pl[j * c.R + t] == e) return false;
    }
  return true;
}

struct RecalLayout {
  size_t off_te, off_base, off_out, bytes;
};

RecalLayout recal_layout(const zb_config& c, int mode) {
  RecalLayout w{};
  size_t o = 0;
  w.off_te = o;
  o = zb::align256(o + sizeof(int32_t) * size_t(c.E));
  w.off_base = o;
  o = zb::align256(o + sizeof(int32_t) * size_t(c.P) * size_t(c.R) + 1);
  w.off_out = o;
  o = zb::align256(o + sizeof(int32_t) * size_t(candidates(c, mode)));
  w.bytes = o;
  return w;
}

// Demand-per-copy placement state: copies so far per expert, and the
// round-robin cursors over nodes and over each node's GPUs.
class DemandPlacer {
 public:
  DemandPlacer(const zb_config& c, const int64_t* demand, int32_t* pl)
      : c_(c), d_(demand), pl_(pl), copies_(size_t(c.E), 1), skip_(size_t(c.E), false),
        gcur_(size_t(c.P / c.gpus_per_node), 0) {}

  void run() {
    const int slots = c_.P * c_.R;
    std::fill(pl_, pl_ + slots, -1);
    int filled = 0;
    while (filled < slots) {
      const int e = most_deserving();
      if (e < 0) return;  // no expert fits anywhere: the rest stays empty
      if (place(e))
        ++filled;
      else
        skip_[size_t(e)] = true;
    }
  }

 private:
  // The expert with the largest demand per copy D_e / n_e (exact: compare
  // D_a * n_b with D_b * n_a), the lowest id among equals.
  int most_deserving() const {
    int best = -1;
    for (int e = 0; e < c_.E; ++e) {
      if (skip_[size_t(e)]) continue;
      if (best < 0 || d_[e] * copies_[size_t(best)] > d_[best] * copies_[size_t(e)]) best = e;
    }
    return best;
  }

  bool holds(int r, int e) const {
    if (e / (c_.E / c_.P) == r) return true;
    for (int s = 0; s < c_.R; ++s)
      if (pl_[r * c_.R + s] == e) return true;
    return false;
  }

  bool has_free_slot(int r) const {
    for (int s = 0; s < c_.R; ++s)
      if (pl_[r * c_.R + s] < 0) return true;
    return false;
  }

  // First GPU of node nd, from that node's cursor, that can take e.
  int rank_in_node(int nd, int e) const {
    const int g = c_.gpus_per_node;
    for (int t = 0; t < g; ++t) {
      const int r = nd * g + (gcur_[size_t(nd)] + t) % g;
      if (!holds(r, e) && has_free_slot(r)) return r;
    }
    return -1;
  }

  bool node_covers(int nd, int e) const {
    const int g = c_.gpus_per_node;
    for (int r = nd * g; r < nd * g + g; ++r)
      if (holds(r, e)) return true;
    return false;
  }

  // Nodes from the cursor: one without a copy of e first, then any; within
  // the node, its GPUs from its own cursor; the lowest free slot.
  bool place(int e) {
    const int g = c_.gpus_per_node, nodes = c_.P / g;
    int nd = -1, r = -1;
    for (int pass = 0; pass < 2 && r < 0; ++pass)
      for (int t = 0; t < nodes && r < 0; ++t) {
        const int cand = (ncur_ + t) % nodes;
        if (pass == 0 && node_covers(cand, e)) continue;
        const int rr = rank_in_node(cand, e);
        if (rr >= 0) {
          nd = cand;
          r = rr;
        }
      }
    if (r < 0) return false;
    int s = 0;
    while (pl_[r * c_.R + s] >= 0) ++s;
    pl_[r * c_.R + s] = e;
    ++copies_[size_t(e)];
    ncur_ = (nd + 1) % nodes;
    gcur_[size_t(nd)] = (r - nd * g + 1) % g;
    return true;
  }

  const zb_config& c_;
  const int64_t* d_;
  int32_t* pl_;
  std::vector<int64_t> copies_;
  std::vector<bool> skip_;
  std::vector<int> gcur_;
  int ncur_ = 0;
};

}  // namespace

extern "C" {

int zb_place_by_demand(const zb_config* c, const int64_t* demand, int32_t* placement) {
  if (zb_validate(c) != ZB_OK || !demand || (c->R > 0 && !placement)) return ZB_ERR_INVALID;
  for (int e = 0; e < c->E; ++e)  // D * copies (copies <= 32) must fit in int64
    if (demand[e] < 0 || demand[e] > (int64_t(1) << 57)) return ZB_ERR_INVALID;
  if (c->R == 0) return ZB_OK;
  DemandPlacer(*c, demand, placement).run();
  return ZB_OK;
}

size_t zb_recalibrate_workspace_bytes(const zb_config* c, int mode) {
  if (zb_validate(c) != ZB_OK || (mode != 0 && mode != 1)) return 0;
  return recal_layout(*c, mode).bytes;
}

int zb_recalibrate(const zb_config* c, const int32_t* cnt, int32_t* placement, int mode,
                   float eps, int max_swaps, void* ws, size_t ws_bytes, void* stream,
                   int32_t* swaps_out, int32_t* max_load_out) {
  if (zb_validate(c) != ZB_OK || (mode != 0 && mode != 1)) return ZB_ERR_INVALID;
  if (!cnt || (c->R > 0 && !placement) || max_swaps < 0 || !(eps >= 0.0f)) return ZB_ERR_INVALID;
  const RecalLayout w = recal_layout(*c, mode);
  if (!ws || ws_bytes < w.bytes || (reinterpret_cast<uintptr_t>(ws) & 255u)) return ZB_ERR_INVALID;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int P = c->P, E = c->E, n = P * c->R;
  std::vector<int32_t> h_cnt(static_cast<size_t>(P) * E);
  std::vector<int32_t> pl(static_cast<size_t>(n));
  std::vector<int32_t> te(static_cast<size_t>(E), 0);
  if (cudaMemcpyAsync(h_cnt.data(), cnt, sizeof(int32_t) * h_cnt.size(), cudaMemcpyDeviceToHost,
                      s) != cudaSuccess)
    return ZB_ERR_CUDA;
  if (n > 0 && cudaMemcpyAsync(pl.data(), placement, sizeof(int32_t) * size_t(n),
                               cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return ZB_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return ZB_ERR_CUDA;
  if (!placement_ok(*c, pl)) return ZB_ERR_INVALID;
  long long sum = 0;
  for (int i = 0; i < P; ++i)
    for (int e = 0; e < E; ++e) {
      if (h_cnt[size_t(i) * E + e] < 0) return ZB_ERR_INVALID;
      te[e] += h_cnt[size_t(i) * E + e];
      sum += h_cnt[size_t(i) * E + e];
    }
  char* base = static_cast<char*>(ws);
  zb::EvalArgs ea{};
  ea.P = P; ea.E = E; ea.R = c->R; ea.gpn = c->gpus_per_node; ea.mode = mode;
  ea.ncand = candidates(*c, mode);
  ea.Te = reinterpret_cast<int32_t*>(base + w.off_te);
  ea.base = reinterpret_cast<int32_t*>(base + w.off_base);
  ea.out = reinterpret_cast<int32_t*>(base + w.off_out);
  std::vector<int32_t> res(static_cast<size_t>(ea.ncand));
  if (cudaMemcpyAsync(const_cast<int32_t*>(ea.Te), te.data(), sizeof(int32_t) * size_t(E),
                      cudaMemcpyHostToDevice, s) != cudaSuccess)
    return ZB_ERR_CUDA;
  // score every candidate of the current placement (index 0 = as it is)
  auto score = [&]() -> bool {
    if (n > 0 && cudaMemcpyAsync(const_cast<int32_t*>(ea.base), pl.data(),
                                 sizeof(int32_t) * size_t(n), cudaMemcpyHostToDevice,
                                 s) != cudaSuccess)
      return false;
    if (zb::launch_eval_placements(ea, s) != cudaSuccess) return false;
    if (cudaMemcpyAsync(res.data(), ea.out, sizeof(int32_t) * res.size(),
                        cudaMemcpyDeviceToHost, s) != cudaSuccess)
      return false;
    return cudaStreamSynchronize(s) == cudaSuccess;
  };
  if (!score()) return ZB_ERR_CUDA;
  const double bound = (1.0 + double(eps)) * double(sum) / double(P);
  int32_t cur = res[0];
  int swaps = 0;
  while (swaps < max_swaps && double(cur) > bound) {
    int32_t best = cur;
    int64_t pick = -1;
    for (int64_t k = 1; k < ea.ncand; ++k)
      if (res[size_t(k)] < best) {
        best = res[size_t(k)];
        pick = k;
      }
    if (pick < 0) break;
    const int64_t k = pick - 1;
    if (mode == 0) {
      pl[size_t(k / E)] = int32_t(k % E);
    } else {
      const int x1 = int(k / n), x2 = int(k % n);
      std::swap(pl[size_t(x1)], pl[size_t(x2)]);
    }
    cur = best;
    ++swaps;
    if (swaps < max_swaps && double(cur) > bound && !score()) return ZB_ERR_CUDA;
  }
  if (n > 0) {
    if (cudaMemcpyAsync(placement, pl.data(), sizeof(int32_t) * size_t(n),
                        cudaMemcpyHostToDevice, s) != cudaSuccess ||
        cudaStreamSynchronize(s) != cudaSuccess)
      return ZB_ERR_CUDA;
  }
  if (swaps_out) *swaps_out = swaps;
  if (max_load_out) *max_load_out = cur;
  return ZB_OK;
}

}  // extern "C"
