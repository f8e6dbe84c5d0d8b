// move_kernels.cu -- steps 4 and 5: the row scatter (dispatch) and the
// gate-weighted gather (combine).  Both are pure data movement bound by HBM
// bandwidth: one warp per token row, 16-byte vectors, several vectors in
// flight per lane, and K specialised at compile time so the K destination (or
// source) rows are all addressed before the first access.
//
// Sources: MoonEP "What MoonEP enforces and how" (zero-copy writes into
// fixed-shape expert-grouped buffers); Zepp "4.2 Split and Merge" (combine);
// ISER-MoE "Key Formula" (dispatch + combine traffic term).
#include <cuda_bf16.h>

#include "zb_internal.cuh"

namespace zb {
namespace {

constexpr int kMoveThreads = 256;
constexpr int kMoveWarps = kMoveThreads / 32;

// Every row is read once and written once per destination: streaming
// (evict-first) loads and stores keep the 126 MB L2 for the small plan tables.
__device__ __forceinline__ uint4 ld_nc(const uint4* p) { return __ldcs(p); }
__device__ __forceinline__ void st_v4(uint4* p, const uint4& v) { __stcs(p, v); }

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

__device__ __forceinline__ float bf_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  const uint32_t l = __bfloat16_as_ushort(__float2bfloat16_rn(lo));
  const uint32_t h = __bfloat16_as_ushort(__float2bfloat16_rn(hi));
  return l | (h << 16);
}

// acc = fmaf(w, y, acc) on the 8 bf16 lanes of one 16-byte vector.
__device__ __forceinline__ void fma8(float (&acc)[8], float w, const uint4& y) {
  acc[0] = __fmaf_rn(w, bf_lo(y.x), acc[0]);
  acc[1] = __fmaf_rn(w, bf_hi(y.x), acc[1]);
  acc[2] = __fmaf_rn(w, bf_lo(y.y), acc[2]);
  acc[3] = __fmaf_rn(w, bf_hi(y.y), acc[3]);
  acc[4] = __fmaf_rn(w, bf_lo(y.z), acc[4]);
  acc[5] = __fmaf_rn(w, bf_hi(y.z), acc[5]);
  acc[6] = __fmaf_rn(w, bf_lo(y.w), acc[6]);
  acc[7] = __fmaf_rn(w, bf_hi(y.w), acc[7]);
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
        uint4 o;
        o.x = pack_bf16x2(acc[0], acc[1]);
        o.y = pack_bf16x2(acc[2], acc[3]);
        o.z = pack_bf16x2(acc[4], acc[5]);
        o.w = pack_bf16x2(acc[6], acc[7]);
        st_v4(out + t * nv + v, o);
      }
    }
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
  constexpr int U = K <= 6 ? 4 : (K <= 8 ? 2 : 1);
  const int blocks = (ntok + kMoveWarps - 1) / kMoveWarps;
  k_combine<K, U><<<blocks, kMoveThreads, 0, s>>>(ntok, H, nrows, dst_row, stats,
                                                  reinterpret_cast<const uint4*>(y), w,
                                                  reinterpret_cast<uint4*>(out));
  return cudaGetLastError();
}

}  // namespace

#define ZB_K_CASES(X) \
  X(1) X(2) X(3) X(4) X(5) X(6) X(7) X(8) X(9) X(10) X(11) X(12) X(13) X(14) X(15) X(16)

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
