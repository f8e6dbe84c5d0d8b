// move_kernels.cu -- steps 4 and 5: the row scatter (dispatch) and the
// gate-weighted gather (combine).  Both are pure data movement bound by HBM
// bandwidth: one warp per token row, 16-byte vectors, several vectors in
// flight per lane, and K specialised at compile time so the K destination (or
// source) rows are all addressed before the first access.
//
// The combine for K = 7 and 8 on wide rows (H >= 4096) loads 32-byte vectors
// when the buffers are 32-byte aligned (k_combine_wide).
//
// Sources: MoonEP "What MoonEP enforces and how" (zero-copy writes into
// fixed-shape expert-grouped buffers); Zepp "4.2 Split and Merge" (combine);
// ISER-MoE "Key Formula" (dispatch + combine traffic term).
#include "zb_internal.cuh"
#include "zb_rows.cuh"

namespace zb {
namespace {

constexpr int kMoveThreads = 256;
constexpr int kMoveWarps = kMoveThreads / 32;

// One warp per token t = i*S + s: read the row once, write it to its K rows.
template <int K, int U>
__global__ void __launch_bounds__(kMoveThreads) k_dispatch(int ntok, int H, int64_t nrows,
                                                           const int32_t* __restrict__ dst_row,
                                                           const int64_t* __restrict__ stats,
                                                           const uint4* __restrict__ hidden,
                                                           uint4* __restrict__ buf) {
  if (stats[ZB_STAT_STATUS] < 0) return;
  const int lane = threadIdx.x & 31;
  const int64_t t = int64_t(blockIdx.x) * kMoveWarps + (threadIdx.x >> 5);
  if (t >= ntok) return;
  const int nv = H >> 3;  // 16-byte vectors per row
  int my_row = lane < K ? __ldg(dst_row + t * K + lane) : -1;
  int64_t rows[K];
#pragma unroll
  for (int k = 0; k < K; ++k) {
    const int r = __shfl_sync(0xffffffffu, my_row, k);
    rows[k] = (r >= 0 && r < nrows) ? int64_t(r) * nv : -1;  // out of range: skip
  }
  const uint4* src = hidden + t * nv;
  for (int v0 = lane; v0 < nv; v0 += 32 * U) {
    uint4 x[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int v = v0 + 32 * u;
      if (v < nv) x[u] = ld_nc(src + v);
    }
#pragma unroll
    for (int k = 0; k < K; ++k) {
      if (rows[k] < 0) continue;
      uint4* dst = buf + rows[k];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int v = v0 + 32 * u;
        if (v < nv) st_v4(dst + v, x[u]);
      }
    }
  }
}

// One warp per token: gather its K rows, fold them with one fused
// multiply-add per term in k order from +0.0f, round once to bf16.
template <int K, int U>
__global__ void __launch_bounds__(kMoveThreads) k_combine(int ntok, int H, int64_t nrows,
                                                          const int32_t* __restrict__ dst_row,
                                                          const int64_t* __restrict__ stats,
                                                          const uint4* __restrict__ y,
                                                          const float* __restrict__ w,
                                                          uint4* __restrict__ out) {
  if (stats[ZB_STAT_STATUS] < 0) return;
  const int lane = threadIdx.x & 31;
  const int64_t t = int64_t(blockIdx.x) * kMoveWarps + (threadIdx.x >> 5);
  if (t >= ntok) return;
  const int nv = H >> 3;
  const int my_row = lane < K ? __ldg(dst_row + t * K + lane) : 0;
  const float my_w = lane < K ? __ldg(w + t * K + lane) : 0.f;
  int64_t rows[K];
  float wk[K];
  bool ok = true;
#pragma unroll
  for (int k = 0; k < K; ++k) {
    const int r = __shfl_sync(0xffffffffu, my_row, k);
    wk[k] = __shfl_sync(0xffffffffu, my_w, k);
    ok = ok && r >= 0 && r < nrows;
    rows[k] = int64_t(r) * nv;
  }
  if (!ok) return;  // a corrupt plan row: leave the output row untouched
  for (int v0 = lane; v0 < nv; v0 += 32 * U) {
    uint4 x[U][K];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int v = v0 + 32 * u;
      if (v < nv) {
#pragma unroll
        for (int k = 0; k < K; ++k) x[u][k] = ld_nc(y + rows[k] + v);
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int v = v0 + 32 * u;
      if (v < nv) {
        float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int k = 0; k < K; ++k) fma8(acc, wk[k], x[u][k]);
        st_v4(out + t * nv + v, pack_bf16x8(acc));
      }
    }
  }
}

// k_combine with 32-byte vectors, for K = 7 and 8 on rows of H >= 4096 (H % 16
// == 0, y and out 32-byte aligned): the same fold, half as many load
// instructions per row.
template <int K>
__global__ void __launch_bounds__(kMoveThreads) k_combine_wide(int ntok, int H, int64_t nrows,
                                                               const int32_t* __restrict__ dst_row,
                                                               const int64_t* __restrict__ stats,
                                                               const V8* __restrict__ y,
                                                               const float* __restrict__ w,
                                                               V8* __restrict__ out) {
  if (stats[ZB_STAT_STATUS] < 0) return;
  const int lane = threadIdx.x & 31;
  const int64_t t = int64_t(blockIdx.x) * kMoveWarps + (threadIdx.x >> 5);
  if (t >= ntok) return;
  const int nv = H >> 4;  // 32-byte vectors per row
  const int my_row = lane < K ? __ldg(dst_row + t * K + lane) : 0;
  const float my_w = lane < K ? __ldg(w + t * K + lane) : 0.f;
  int64_t rows[K];
  float wk[K];
  bool ok = true;
#pragma unroll
  for (int k = 0; k < K; ++k) {
    const int r = __shfl_sync(0xffffffffu, my_row, k);
    wk[k] = __shfl_sync(0xffffffffu, my_w, k);
    ok = ok && r >= 0 && r < nrows;
    rows[k] = int64_t(r) * nv;
  }
  if (!ok) return;  // a corrupt plan row: leave the output row untouched
  for (int v = lane; v < nv; v += 32) {
    V8 x[K];
#pragma unroll
    for (int k = 0; k < K; ++k) x[k] = ld_nc8(y + rows[k] + v);
    float acc[16];
#pragma unroll
    for (int q = 0; q < 16; ++q) acc[q] = 0.f;
#pragma unroll
    for (int k = 0; k < K; ++k)
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        acc[2 * q] = __fmaf_rn(wk[k], bf_lo(x[k].v[q]), acc[2 * q]);
        acc[2 * q + 1] = __fmaf_rn(wk[k], bf_hi(x[k].v[q]), acc[2 * q + 1]);
      }
    V8 o;
#pragma unroll
    for (int q = 0; q < 8; ++q) o.v[q] = pack_bf16x2(acc[2 * q], acc[2 * q + 1]);
    st_v8(out + t * nv + v, o);
  }
}

template <int K>
cudaError_t dispatch_k(int ntok, int H, int64_t nrows, const int32_t* dst_row,
                       const int64_t* stats, const uint16_t* hidden, uint16_t* buf,
                       cudaStream_t s) {
  const int blocks = (ntok + kMoveWarps - 1) / kMoveWarps;
  k_dispatch<K, 8><<<blocks, kMoveThreads, 0, s>>>(ntok, H, nrows, dst_row, stats,
                                                   reinterpret_cast<const uint4*>(hidden),
                                                   reinterpret_cast<uint4*>(buf));
  return cudaGetLastError();
}

template <int K>
cudaError_t combine_k(int ntok, int H, int64_t nrows, const int32_t* dst_row,
                      const int64_t* stats, const uint16_t* y, const float* w, uint16_t* out,
                      cudaStream_t s) {
  constexpr int U = K <= 6 ? 4 : (K <= 16 ? 2 : 1);
  const int blocks = (ntok + kMoveWarps - 1) / kMoveWarps;
  // Measured: at K = 8 the 32-byte kernel is 4% faster for H = 7168 and 3%
  // slower for H = 2048; at K = 6, and at K >= 12 for H = 2048, it is slower.
  if constexpr (K == 7 || K == 8) {
    const bool wide_ok = H >= 4096 && (H % 16) == 0 &&
                         (reinterpret_cast<uintptr_t>(y) & 31u) == 0 &&
                         (reinterpret_cast<uintptr_t>(out) & 31u) == 0;
    if (wide_ok) {
      k_combine_wide<K><<<blocks, kMoveThreads, 0, s>>>(ntok, H, nrows, dst_row, stats,
                                                        reinterpret_cast<const V8*>(y), w,
                                                        reinterpret_cast<V8*>(out));
      return cudaGetLastError();
    }
  }
  k_combine<K, U><<<blocks, kMoveThreads, 0, s>>>(ntok, H, nrows, dst_row, stats,
                                                  reinterpret_cast<const uint4*>(y), w,
                                                  reinterpret_cast<uint4*>(out));
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_dispatch(int P, int S, int K, int H, int cap, const int32_t* dst_row,
                            const int64_t* stats, const uint16_t* hidden, uint16_t* buf,
                            cudaStream_t s) {
  const int ntok = P * S;
  if (ntok == 0) return cudaSuccess;
  const int64_t nrows = int64_t(P) * cap;
  switch (K) {
#define X(k) \
  case k:    \
    return dispatch_k<k>(ntok, H, nrows, dst_row, stats, hidden, buf, s);
    ZB_K_CASES(X)
#undef X
    default:
      return cudaErrorInvalidValue;
  }
}

cudaError_t launch_combine(int P, int S, int K, int H, int cap, const int32_t* dst_row,
                           const int64_t* stats, const uint16_t* y, const float* w,
                           uint16_t* out, cudaStream_t s) {
  const int ntok = P * S;
  if (ntok == 0) return cudaSuccess;
  const int64_t nrows = int64_t(P) * cap;
  switch (K) {
#define X(k) \
  case k:    \
    return combine_k<k>(ntok, H, nrows, dst_row, stats, y, w, out, s);
    ZB_K_CASES(X)
#undef X
    default:
      return cudaErrorInvalidValue;
  }
}

}  // namespace zb
