// zb_recal.cu -- zb_recalibrate: placement recalibration between invocations.
// The only call besides zb_plan_status that synchronises its stream: every
// step reads the scores of all candidates back to the host to pick one, and
// the host keeps the placement being changed (in host memory it allocates).
//
// Sources: ViBE, "Drift-Aware Recalibration" (incremental placement update:
// from the current placement, minimal cross-GPU expert swaps until every GPU
// is within eps of the mean); Zepp, "4.3 Three-Stream Scheduling", eq. (4)
// (intra-node swaps of expert replicas that keep node-level coverage).
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

}  // namespace

extern "C" {

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
