// zb_rows.cuh -- device helpers shared by the row-moving kernels: streaming
// 16-byte loads and stores, bf16 <-> float on the 8 lanes of a vector, and
// the K cases every row kernel is instantiated for.
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

namespace zb {

// Every row is read once and written once per destination: streaming
// (evict-first) loads and stores keep the 126 MB L2 for the small plan tables.
__device__ __forceinline__ uint4 ld_nc(const uint4* p) { return __ldcs(p); }
__device__ __forceinline__ void st_v4(uint4* p, const uint4& v) { __stcs(p, v); }

// 32-byte vectors (sm_100's 256-bit global accesses): 16 bf16 per lane.
struct alignas(32) V8 {
  uint32_t v[8];
};
__device__ __forceinline__ V8 ld_nc8(const V8* p) {
  V8 r;
  asm volatile("ld.global.cs.v8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
               : "=r"(r.v[0]), "=r"(r.v[1]), "=r"(r.v[2]), "=r"(r.v[3]), "=r"(r.v[4]),
                 "=r"(r.v[5]), "=r"(r.v[6]), "=r"(r.v[7])
               : "l"(p));
  return r;
}
__device__ __forceinline__ void st_v8(V8* p, const V8& r) {
  asm volatile("st.global.cs.v8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"l"(p), "r"(r.v[0]),
               "r"(r.v[1]), "r"(r.v[2]), "r"(r.v[3]), "r"(r.v[4]), "r"(r.v[5]), "r"(r.v[6]),
               "r"(r.v[7])
               : "memory");
}

// bf16 widens to float exactly: it is the upper half of a binary32.
__device__ __forceinline__ float bf_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// Two floats to a pair of bf16, each rounded to nearest, ties to even.
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  const uint32_t l = __bfloat16_as_ushort(__float2bfloat16_rn(lo));
  const uint32_t h = __bfloat16_as_ushort(__float2bfloat16_rn(hi));
  return l | (h << 16);
}

__device__ __forceinline__ uint4 pack_bf16x8(const float (&acc)[8]) {
  uint4 o;
  o.x = pack_bf16x2(acc[0], acc[1]);
  o.y = pack_bf16x2(acc[2], acc[3]);
  o.z = pack_bf16x2(acc[4], acc[5]);
  o.w = pack_bf16x2(acc[6], acc[7]);
  return o;
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

// acc = acc + y on the 8 bf16 lanes of one 16-byte vector (no contraction).
__device__ __forceinline__ void add8(float (&acc)[8], const uint4& y) {
  acc[0] = __fadd_rn(acc[0], bf_lo(y.x));
  acc[1] = __fadd_rn(acc[1], bf_hi(y.x));
  acc[2] = __fadd_rn(acc[2], bf_lo(y.y));
  acc[3] = __fadd_rn(acc[3], bf_hi(y.y));
  acc[4] = __fadd_rn(acc[4], bf_lo(y.z));
  acc[5] = __fadd_rn(acc[5], bf_hi(y.z));
  acc[6] = __fadd_rn(acc[6], bf_lo(y.w));
  acc[7] = __fadd_rn(acc[7], bf_hi(y.w));
}

}  // namespace zb

#define ZB_K_CASES(X) \
  X(1) X(2) X(3) X(4) X(5) X(6) X(7) X(8) X(9) X(10) X(11) X(12) X(13) X(14) X(15) X(16)
