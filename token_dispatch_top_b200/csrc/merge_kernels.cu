// merge_kernels.cu -- the merged dispatch layout and scatter: one row per
// (token, destination rank) instead of one per (token, k).  When several of
// a token's K experts are served by the same rank, they share one copy of its
// row there (Zepp, "4.2 Split and Merge": the experts a token selects on one
// remote node share a single transfer).
//   k_merge_count   per 256-token chunk: tokens sending to each rank
//   k_merge_assign  per chunk: each token's position among the tokens of its
//                   destination ranks (prefix of earlier chunks + in-order
//                   ballots), giving tok_row, grp_tok and tok_cnt
//   k_dispatch_merged  one warp per token: read the row once, write it once
//                   per distinct destination row
//   k_combine_reduce   destination side of the merged combine: one warp per
//                   token folds the gated outputs each rank served into one
//                   bf16 partial per merged row (Zepp 4.2: node-local
//                   pre-reduction into partial sums before transfer)
//   k_combine_merged   source side: one warp per token adds its partials
#include "zb_internal.cuh"
#include "zb_rows.cuh"

namespace zb {
ZB_DEBUG_TU(debug_read_merge)
namespace {

constexpr unsigned kFull = 0xffffffffu;
constexpr int kMergeThreads = 256;  // one token per thread
constexpr int kMergeWarps = kMergeThreads / 32;
constexpr int kTokPerThread = kMergeChunk / kMergeThreads;  // 1

// Bit j set when one of token t's entries goes to rank j (rows outside
// [0, nrows), which a plan with a non-negative status never holds, count
// nowhere).
__device__ __forceinline__ unsigned rank_mask(const int32_t* dst_row, int64_t t, int K,
                                              int cap, int64_t nrows) {
  unsigned m = 0u;
  for (int k = 0; k < K; ++k) {
    const int d = __ldg(dst_row + t * K + k);
    if (ZB_IN(ZB_SITE_MERGE_ROW, d, nrows) && d >= 0 && d < nrows) m |= 1u << (d / cap);
  }
  return m;
}

__global__ void __launch_bounds__(kMergeThreads) k_merge_count(MergeArgs a) {
  if (a.stats[ZB_STAT_STATUS] < 0) return;
  __shared__ int32_t cnt[kMaxP];
  const int c = blockIdx.x, tid = threadIdx.x;
  if (tid < kMaxP) cnt[tid] = 0;
  __syncthreads();
  for (int u = 0; u < kTokPerThread; ++u) {
    const int64_t t = int64_t(c) * kMergeChunk + u * kMergeThreads + tid;
    if (t < a.ntok) {
      unsigned m = rank_mask(a.dst_row, t, a.K, a.cap, int64_t(a.P) * a.cap);
      while (m) {
        const int j = __ffs(m) - 1;
        m &= m - 1u;
        atomicAdd(&cnt[j], 1);
      }
    }
  }
  __syncthreads();
  if (tid < a.P) a.chunk_cnt[int64_t(c) * a.P + tid] = cnt[tid];
  // grouped rows past each rank's load are unused: grp_tok -1 there (the
  // used rows are all written by k_merge_assign)
  const int64_t nrows = int64_t(a.P) * a.cap;
  for (int64_t x = int64_t(c) * kMergeThreads + tid; x < nrows;
       x += int64_t(gridDim.x) * kMergeThreads) {
    const int j = int(x / a.cap);
    if (x - int64_t(j) * a.cap >= a.load_after[j]) a.grp_tok[x] = -1;
  }
}

__global__ void __launch_bounds__(kMergeThreads) k_merge_assign(MergeArgs a) {
  if (a.stats[ZB_STAT_STATUS] < 0) return;
  __shared__ int32_t wc[kMergeWarps][kMaxP];  // per-warp start position per rank
  const int c = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int P = a.P, K = a.K, cap = a.cap;
  const int64_t nrows = int64_t(P) * cap;
  const int64_t t = int64_t(c) * kMergeChunk + tid;  // this thread's token
  int d[16];
  unsigned m = 0u;
#pragma unroll
  for (int k = 0; k < 16; ++k) {
    d[k] = (k < K && t < a.ntok) ? __ldg(a.dst_row + t * K + k) : -1;
    if (d[k] >= 0 && d[k] < nrows) m |= 1u << (d[k] / cap);
  }
  // tokens per rank in this warp
  for (int j = 0; j < P; ++j) {
    const int n = __popc(__ballot_sync(kFull, (m >> j) & 1u));
    if (lane == 0) wc[warp][j] = n;
  }
  __syncthreads();
  // exclusive prefix: earlier chunks, then earlier warps of this chunk
  if (tid < P) {
    const int j = tid;
    int run = 0;
    for (int c0 = 0; c0 < c; c0 += 8) {  // eight loads in flight
      int x[8];
#pragma unroll
      for (int q = 0; q < 8; ++q) x[q] = c0 + q < c ? a.chunk_cnt[int64_t(c0 + q) * P + j] : 0;
#pragma unroll
      for (int q = 0; q < 8; ++q) run += x[q];
    }
    for (int w = 0; w < kMergeWarps; ++w) {
      const int v = wc[w][j];
      wc[w][j] = run;
      run += v;
    }
    if (c == gridDim.x - 1) a.tok_cnt[j] = run;
  }
  __syncthreads();
  // position of this token among the tokens of each of its ranks, in token order
  int pos[kMaxP];
#pragma unroll
  for (int j = 0; j < kMaxP; ++j) {
    if (j >= P) break;
    const unsigned b = __ballot_sync(kFull, (m >> j) & 1u);
    pos[j] = wc[warp][j] + __popc(b & ((1u << lane) - 1u));
  }
  if (t < a.ntok) {
#pragma unroll
    for (int k = 0; k < 16; ++k) {
      if (k >= K) break;
      if (d[k] < 0 || d[k] >= nrows) {  // only a valid plan has rows
        ZB_FAIL(ZB_SITE_MERGE_ROW, d[k], nrows);
        continue;
      }
      const int j = d[k] / cap;
      int pj = 0;
#pragma unroll
      for (int q = 0; q < kMaxP; ++q)
        if (q == j) pj = pos[q];
      const int row = j * cap + pj;
      a.tok_row[t * K + k] = row;
      a.grp_tok[d[k]] = row;
    }
  }
}

// One warp per token: lanes < K hold the token's merged rows; a row is
// written only by the lowest k that names it.
template <int K, int U>
__global__ void __launch_bounds__(256) k_dispatch_merged(int ntok, int H, int64_t nrows,
                                                         const int32_t* __restrict__ tok_row,
                                                         const int64_t* __restrict__ stats,
                                                         const uint4* __restrict__ hidden,
                                                         uint4* __restrict__ tbuf) {
  if (stats[ZB_STAT_STATUS] < 0) return;
  const int lane = threadIdx.x & 31;
  const int64_t t = int64_t(blockIdx.x) * 8 + (threadIdx.x >> 5);
  if (t >= ntok) return;
  const int nv = H >> 3;
  const int my = lane < K ? __ldg(tok_row + t * K + lane) : -2 - lane;
  const unsigned peers = __match_any_sync(kFull, my);
  const bool in = lane >= K || ZB_IN(ZB_SITE_MERGE_ROW, my, nrows);
  const bool first = in && lane < K && (__ffs(peers) - 1) == lane && my >= 0 && my < nrows;
  const unsigned firsts = __ballot_sync(kFull, first);
  int64_t rows[K];
#pragma unroll
  for (int k = 0; k < K; ++k) {
    const int r = __shfl_sync(kFull, my, k);
    rows[k] = ((firsts >> k) & 1u) ? int64_t(r) * nv : -1;
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
      uint4* dst = tbuf + rows[k];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int v = v0 + 32 * u;
        if (v < nv) st_v4(dst + v, x[u]);
      }
    }
  }
}

// Destination side of the merged combine, one warp per token.  Lanes < K hold
// the token's grouped rows, gates and merged rows.  For each merged row, led
// by the lowest k that names it, the gated outputs of the k naming it are
// folded in k order, acc = fmaf(w_k, y_k, acc) from +0.0f, and rounded once
// to bf16 into that merged row.
template <int K, int U>
__global__ void __launch_bounds__(256) k_combine_reduce(int ntok, int H, int64_t nrows,
                                                        const int32_t* __restrict__ dst_row,
                                                        const int32_t* __restrict__ tok_row,
                                                        const int64_t* __restrict__ stats,
                                                        const uint4* __restrict__ y,
                                                        const float* __restrict__ w,
                                                        uint4* __restrict__ part) {
  if (stats[ZB_STAT_STATUS] < 0) return;
  const int lane = threadIdx.x & 31;
  const int64_t t = int64_t(blockIdx.x) * 8 + (threadIdx.x >> 5);
  if (t >= ntok) return;
  const int nv = H >> 3;
  const int my_d = lane < K ? __ldg(dst_row + t * K + lane) : 0;
  const int my_m = lane < K ? __ldg(tok_row + t * K + lane) : -2 - lane;
  const float my_w = lane < K ? __ldg(w + t * K + lane) : 0.f;
  const unsigned peers = __match_any_sync(kFull, my_m);
  const unsigned leads = __ballot_sync(kFull, lane < K && (__ffs(peers) - 1) == lane);
  int64_t rows[K];
  int mrow[K];
  float wk[K];
  bool ok = true;
#pragma unroll
  for (int k = 0; k < K; ++k) {
    const int r = __shfl_sync(kFull, my_d, k);
    mrow[k] = __shfl_sync(kFull, my_m, k);
    wk[k] = __shfl_sync(kFull, my_w, k);
    ok = ok && r >= 0 && r < nrows && mrow[k] >= 0 && mrow[k] < nrows;
    if (!(r >= 0 && r < nrows)) ZB_FAIL(ZB_SITE_MERGE_ROW, r, nrows);
    if (!(mrow[k] >= 0 && mrow[k] < nrows)) ZB_FAIL(ZB_SITE_MERGE_ROW, mrow[k], nrows);
    rows[k] = int64_t(r) * nv;
  }
  if (!ok) return;  // a corrupt plan or layout: write nothing for this token
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
    for (int k0 = 0; k0 < K; ++k0) {
      if (!((leads >> k0) & 1u)) continue;
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int v = v0 + 32 * u;
        if (v >= nv) continue;
        float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int k = k0; k < K; ++k)
          if (mrow[k] == mrow[k0]) fma8(acc, wk[k], x[u][k]);
        st_v4(part + int64_t(mrow[k0]) * nv + v, pack_bf16x8(acc));
      }
    }
  }
}

// Source side of the merged combine, one warp per token: out = bf16 of the
// float sum of the token's partials, acc = acc + part from +0.0f, in the
// order of the first k naming each merged row.
template <int K, int U>
__global__ void __launch_bounds__(256) k_combine_merged(int ntok, int H, int64_t nrows,
                                                        const int32_t* __restrict__ tok_row,
                                                        const int64_t* __restrict__ stats,
                                                        const uint4* __restrict__ part,
                                                        uint4* __restrict__ out) {
  if (stats[ZB_STAT_STATUS] < 0) return;
  const int lane = threadIdx.x & 31;
  const int64_t t = int64_t(blockIdx.x) * 8 + (threadIdx.x >> 5);
  if (t >= ntok) return;
  const int nv = H >> 3;
  const int my_m = lane < K ? __ldg(tok_row + t * K + lane) : -2 - lane;
  const unsigned peers = __match_any_sync(kFull, my_m);
  const unsigned leads = __ballot_sync(kFull, lane < K && (__ffs(peers) - 1) == lane);
  int64_t rows[K];
  bool ok = true;
#pragma unroll
  for (int k = 0; k < K; ++k) {
    const int m = __shfl_sync(kFull, my_m, k);
    ok = ok && m >= 0 && m < nrows;
    if (!(m >= 0 && m < nrows)) ZB_FAIL(ZB_SITE_MERGE_ROW, m, nrows);
    rows[k] = int64_t(m) * nv;
  }
  if (!ok) return;
  for (int v0 = lane; v0 < nv; v0 += 32 * U) {
    uint4 x[U][K];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int v = v0 + 32 * u;
      if (v < nv) {
#pragma unroll
        for (int k = 0; k < K; ++k)
          if ((leads >> k) & 1u) x[u][k] = ld_nc(part + rows[k] + v);
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int v = v0 + 32 * u;
      if (v >= nv) continue;
      float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int k = 0; k < K; ++k)
        if ((leads >> k) & 1u) add8(acc, x[u][k]);
      st_v4(out + t * nv + v, pack_bf16x8(acc));
    }
  }
}

template <int K>
cudaError_t dispatch_merged_k(int ntok, int H, int64_t nrows, const int32_t* tok_row,
                              const int64_t* stats, const uint16_t* hidden, uint16_t* tbuf,
                              cudaStream_t s) {
  const int blocks = (ntok + 7) / 8;
  k_dispatch_merged<K, 8><<<blocks, 256, 0, s>>>(ntok, H, nrows, tok_row, stats,
                                                  reinterpret_cast<const uint4*>(hidden),
                                                  reinterpret_cast<uint4*>(tbuf));
  return cudaGetLastError();
}

template <int K>
cudaError_t combine_reduce_k(int ntok, int H, int64_t nrows, const int32_t* dst_row,
                             const int32_t* tok_row, const int64_t* stats, const uint16_t* y,
                             const float* w, uint16_t* part, cudaStream_t s) {
  constexpr int U = K <= 6 ? 4 : (K <= 8 ? 2 : 1);
  k_combine_reduce<K, U><<<(ntok + 7) / 8, 256, 0, s>>>(
      ntok, H, nrows, dst_row, tok_row, stats, reinterpret_cast<const uint4*>(y), w,
      reinterpret_cast<uint4*>(part));
  return cudaGetLastError();
}

template <int K>
cudaError_t combine_merged_k(int ntok, int H, int64_t nrows, const int32_t* tok_row,
                             const int64_t* stats, const uint16_t* part, uint16_t* out,
                             cudaStream_t s) {
  constexpr int U = K <= 6 ? 4 : (K <= 8 ? 2 : 1);
  k_combine_merged<K, U><<<(ntok + 7) / 8, 256, 0, s>>>(
      ntok, H, nrows, tok_row, stats, reinterpret_cast<const uint4*>(part),
      reinterpret_cast<uint4*>(out));
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_merge(const MergeArgs& a, cudaStream_t s) {
  const int nchunk = int(ceil_div(a.ntok, kMergeChunk));
  if (nchunk == 0) return cudaSuccess;
  k_merge_count<<<nchunk, kMergeThreads, 0, s>>>(a);
  cudaError_t err = cudaGetLastError();
  if (err != cudaSuccess) return err;
  k_merge_assign<<<nchunk, kMergeThreads, 0, s>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_dispatch_merged(int P, int S, int K, int H, int cap, const int32_t* tok_row,
                                   const int64_t* stats, const uint16_t* hidden, uint16_t* tbuf,
                                   cudaStream_t s) {
  const int ntok = P * S;
  if (ntok == 0) return cudaSuccess;
  const int64_t nrows = int64_t(P) * cap;
  switch (K) {
#define X(k) \
  case k:    \
    return dispatch_merged_k<k>(ntok, H, nrows, tok_row, stats, hidden, tbuf, s);
    ZB_K_CASES(X)
#undef X
    default:
      return cudaErrorInvalidValue;
  }
}

cudaError_t launch_combine_reduce(int P, int S, int K, int H, int cap, const int32_t* dst_row,
                                  const int32_t* tok_row, const int64_t* stats,
                                  const uint16_t* y, const float* w, uint16_t* part,
                                  cudaStream_t s) {
  const int ntok = P * S;
  if (ntok == 0) return cudaSuccess;
  const int64_t nrows = int64_t(P) * cap;
  switch (K) {
#define X(k) \
  case k:    \
    return combine_reduce_k<k>(ntok, H, nrows, dst_row, tok_row, stats, y, w, part, s);
    ZB_K_CASES(X)
#undef X
    default:
      return cudaErrorInvalidValue;
  }
}

cudaError_t launch_combine_merged(int P, int S, int K, int H, int cap, const int32_t* tok_row,
                                  const int64_t* stats, const uint16_t* part, uint16_t* out,
                                  cudaStream_t s) {
  const int ntok = P * S;
  if (ntok == 0) return cudaSuccess;
  const int64_t nrows = int64_t(P) * cap;
  switch (K) {
#define X(k) \
  case k:    \
    return combine_merged_k<k>(ntok, H, nrows, tok_row, stats, part, out, s);
    ZB_K_CASES(X)
#undef X
    default:
      return cudaErrorInvalidValue;
  }
}

}  // namespace zb
