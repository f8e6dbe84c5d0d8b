// move_kernels.cu -- steps 4 and 5: the row scatter (dispatch) and the
// gate-weighted gather (combine).  Both are pure data movement bound by HBM
// bandwidth: one warp per token row, 16-byte vectors, several vectors in
// flight per lane, and K specialised at compile time so the K destination (or
// source) rows are all addressed before the first access.
//
// The combine for K = 7 and 8 on wide rows (H >= 4096) loads 32-byte vectors
// when the buffers are 32-byte aligned (k_combine_wide).
//
// Rows are addressed one of two ways.  FlatRows: one buffer holds every
// rank's rows, rank j's from row j*cap (the path on one GPU).  RankRows: each
// rank's rows live in a buffer of its own, found through a table of P base
// pointers, row d - j*cap of rank j = d / cap (the path on one of P GPUs,
// where the other ranks' buffers are peer memory mapped into this process).
// Both use plain per-thread loads and stores only.
//
// Sources: MoonEP "What MoonEP enforces and how" (zero-copy writes into
// fixed-shape expert-grouped buffers on remote ranks); Zepp "4.2 Split and
// Merge" (combine); ISER-MoE "Key Formula" (dispatch + combine traffic term).
#include "zb_internal.cuh"
#include "zb_rows.cuh"

namespace zb {
ZB_DEBUG_TU(debug_read_move)
namespace {

constexpr int kMoveThreads = 256;
constexpr int kMoveWarps = kMoveThreads / 32;

// A row outside [0, P*cap) -- which a plan with a non-negative status never
// holds -- gives nullptr, and the access is skipped (recorded at `site` in the
// bounds-checked build).
struct FlatRows {
  char* base;
  int64_t nrows;  // P * cap
  __device__ __forceinline__ char* row(int d, int64_t row_bytes, int site) const {
    if (d >= 0 && d < nrows) return base + int64_t(d) * row_bytes;
    ZB_FAIL(site, d, nrows);
    return nullptr;
  }
};

struct RankRows {
  RankBufs t;
  int P, cap;
  __device__ __forceinline__ char* row(int d, int64_t row_bytes, int site) const {
    const int j = d >= 0 ? d / cap : 0;
    if (d < 0 || j >= P) {
      ZB_FAIL(site, d, int64_t(P) * cap);
      return nullptr;
    }
    return reinterpret_cast<char*>(t.p[j]) + int64_t(d - j * cap) * row_bytes;
  }
};

// Row d of the plan's entry held by lane k < K of the warp, broadcast: the K
// row addresses of token t (nullptr where d is out of range).
template <int K, class T, class Rows>
__device__ __forceinline__ void entry_rows(const Rows& rows, const int32_t* dst_row, int64_t t,
                                           int64_t row_bytes, int lane, int site,
                                           T* (&out)[K]) {
  char* mine =
      lane < K ? rows.row(__ldg(dst_row + t * K + lane), row_bytes, site) : nullptr;
#pragma unroll
  for (int k = 0; k < K; ++k)
    out[k] = reinterpret_cast<T*>(
        __shfl_sync(0xffffffffu, reinterpret_cast<unsigned long long>(mine), k));
}

// One warp per token t: read the row once, write it to its K rows.
template <int K, int U, class Rows>
__global__ void __launch_bounds__(kMoveThreads) k_dispatch(int ntok, int H, Rows rows,
                                                           const int32_t* __restrict__ dst_row,
                                                           const int64_t* __restrict__ stats,
                                                           const uint4* __restrict__ hidden) {
  if (stats[ZB_STAT_STATUS] < 0) return;
  const int lane = threadIdx.x & 31;
  const int64_t t = int64_t(blockIdx.x) * kMoveWarps + (threadIdx.x >> 5);
  if (t >= ntok) return;
  const int nv = H >> 3;  // 16-byte vectors per row
  uint4* dst[K];
  entry_rows<K>(rows, dst_row, t, int64_t(nv) * 16, lane, ZB_SITE_DISPATCH_ROW, dst);
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
      if (dst[k] == nullptr) continue;
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int v = v0 + 32 * u;
        if (v < nv) st_v4(dst[k] + v, x[u]);
      }
    }
  }
}

// One warp per token: gather its K rows, fold them with one fused
// multiply-add per term in k order from +0.0f, round once to bf16.
template <int K, int U, class Rows>
__global__ void __launch_bounds__(kMoveThreads) k_combine(int ntok, int H, Rows rows,
                                                          const int32_t* __restrict__ dst_row,
                                                          const int64_t* __restrict__ stats,
                                                          const float* __restrict__ w,
                                                          uint4* __restrict__ out) {
  if (stats[ZB_STAT_STATUS] < 0) return;
  const int lane = threadIdx.x & 31;
  const int64_t t = int64_t(blockIdx.x) * kMoveWarps + (threadIdx.x >> 5);
  if (t >= ntok) return;
  const int nv = H >> 3;
  const uint4* src[K];
  entry_rows<K>(rows, dst_row, t, int64_t(nv) * 16, lane, ZB_SITE_COMBINE_ROW, src);
  const float my_w = lane < K ? __ldg(w + t * K + lane) : 0.f;
  float wk[K];
  bool ok = true;
#pragma unroll
  for (int k = 0; k < K; ++k) {
    wk[k] = __shfl_sync(0xffffffffu, my_w, k);
    ok = ok && src[k] != nullptr;
  }
  if (!ok) return;  // a corrupt plan row: leave the output row untouched
  for (int v0 = lane; v0 < nv; v0 += 32 * U) {
    uint4 x[U][K];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int v = v0 + 32 * u;
      if (v < nv) {
#pragma unroll
        for (int k = 0; k < K; ++k) x[u][k] = ld_nc(src[k] + v);
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
// == 0, rows and out 32-byte aligned): the same fold, half as many load
// instructions per row.
template <int K, class Rows>
__global__ void __launch_bounds__(kMoveThreads) k_combine_wide(int ntok, int H, Rows rows,
                                                               const int32_t* __restrict__ dst_row,
                                                               const int64_t* __restrict__ stats,
                                                               const float* __restrict__ w,
                                                               V8* __restrict__ out) {
  if (stats[ZB_STAT_STATUS] < 0) return;
  const int lane = threadIdx.x & 31;
  const int64_t t = int64_t(blockIdx.x) * kMoveWarps + (threadIdx.x >> 5);
  if (t >= ntok) return;
  const int nv = H >> 4;  // 32-byte vectors per row
  const V8* src[K];
  entry_rows<K>(rows, dst_row, t, int64_t(nv) * 32, lane, ZB_SITE_COMBINE_ROW, src);
  const float my_w = lane < K ? __ldg(w + t * K + lane) : 0.f;
  float wk[K];
  bool ok = true;
#pragma unroll
  for (int k = 0; k < K; ++k) {
    wk[k] = __shfl_sync(0xffffffffu, my_w, k);
    ok = ok && src[k] != nullptr;
  }
  if (!ok) return;  // a corrupt plan row: leave the output row untouched
  for (int v = lane; v < nv; v += 32) {
    V8 x[K];
#pragma unroll
    for (int k = 0; k < K; ++k) x[k] = ld_nc8(src[k] + v);
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

template <int K, class Rows>
cudaError_t dispatch_k(int ntok, int H, const Rows& rows, const int32_t* dst_row,
                       const int64_t* stats, const uint16_t* hidden, cudaStream_t s) {
  const int blocks = (ntok + kMoveWarps - 1) / kMoveWarps;
  k_dispatch<K, 8, Rows><<<blocks, kMoveThreads, 0, s>>>(
      ntok, H, rows, dst_row, stats, reinterpret_cast<const uint4*>(hidden));
  return cudaGetLastError();
}

// wide_ok: rows and out are 32-byte aligned.
template <int K, class Rows>
cudaError_t combine_k(int ntok, int H, const Rows& rows, bool wide_ok, const int32_t* dst_row,
                      const int64_t* stats, const float* w, uint16_t* out, cudaStream_t s) {
  constexpr int U = K <= 6 ? 4 : (K <= 16 ? 2 : 1);
  const int blocks = (ntok + kMoveWarps - 1) / kMoveWarps;
  // Measured: at K = 8 the 32-byte kernel is 4% faster for H = 7168 and 3%
  // slower for H = 2048; at K = 6, and at K >= 12 for H = 2048, it is slower.
  if constexpr (K == 7 || K == 8) {
    if (wide_ok && H >= 4096 && (H % 16) == 0) {
      k_combine_wide<K, Rows><<<blocks, kMoveThreads, 0, s>>>(ntok, H, rows, dst_row, stats, w,
                                                              reinterpret_cast<V8*>(out));
      return cudaGetLastError();
    }
  }
  k_combine<K, U, Rows><<<blocks, kMoveThreads, 0, s>>>(ntok, H, rows, dst_row, stats, w,
                                                        reinterpret_cast<uint4*>(out));
  return cudaGetLastError();
}

bool aligned32(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 31u) == 0; }

}  // namespace

cudaError_t launch_dispatch(int P, int S, int K, int H, int cap, const int32_t* dst_row,
                            const int64_t* stats, const uint16_t* hidden, uint16_t* buf,
                            cudaStream_t s) {
  const int ntok = P * S;
  if (ntok == 0) return cudaSuccess;
  const FlatRows rows{reinterpret_cast<char*>(buf), int64_t(P) * cap};
  switch (K) {
#define X(k) \
  case k:    \
    return dispatch_k<k>(ntok, H, rows, dst_row, stats, hidden, s);
    ZB_K_CASES(X)
#undef X
    default:
      return cudaErrorInvalidValue;
  }
}

cudaError_t launch_dispatch_ranks(int P, int ntok, int K, int H, int cap,
                                  const int32_t* dst_row, const int64_t* stats,
                                  const uint16_t* hidden, const RankBufs& bufs, cudaStream_t s) {
  if (ntok == 0) return cudaSuccess;
  const RankRows rows{bufs, P, cap};
  switch (K) {
#define X(k) \
  case k:    \
    return dispatch_k<k>(ntok, H, rows, dst_row, stats, hidden, s);
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
  const FlatRows rows{reinterpret_cast<char*>(const_cast<uint16_t*>(y)), int64_t(P) * cap};
  const bool wide_ok = aligned32(y) && aligned32(out);
  switch (K) {
#define X(k) \
  case k:    \
    return combine_k<k>(ntok, H, rows, wide_ok, dst_row, stats, w, out, s);
    ZB_K_CASES(X)
#undef X
    default:
      return cudaErrorInvalidValue;
  }
}

cudaError_t launch_combine_ranks(int P, int ntok, int K, int H, int cap, const int32_t* dst_row,
                                 const int64_t* stats, const RankBufs& ys, const float* w,
                                 uint16_t* out, bool wide_ok, cudaStream_t s) {
  if (ntok == 0) return cudaSuccess;
  const RankRows rows{ys, P, cap};
  switch (K) {
#define X(k) \
  case k:    \
    return combine_k<k>(ntok, H, rows, wide_ok, dst_row, stats, w, out, s);
    ZB_K_CASES(X)
#undef X
    default:
      return cudaErrorInvalidValue;
  }
}

}  // namespace zb
