// Device helpers shared by the kernels: RoPE angle factors from the two-level
// table, and 8-element vector loads/stores between bf16/fp32 storage and fp32
// registers.
#pragma once

#include <cuda_bf16.h>

#include "dbsa_internal.h"

namespace dbsa {

using bf16 = __nv_bfloat16;

// (cos, sin) of p * w_i for the 8 frequencies i0..i0+7, as hi[p >> 6] * lo[p & 63].
__device__ __forceinline__ void rope_cs8(const RopeTables &t, int64_t p, int i0, int half,
                                         float (&c)[8], float (&s)[8]) {
  const float4 *h4 = reinterpret_cast<const float4 *>(t.hi + (p >> 6) * half + i0);
  const float4 *l4 = reinterpret_cast<const float4 *>(t.lo + (p & 63) * half + i0);
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const float4 a = __ldg(h4 + e), b = __ldg(l4 + e);
    c[2 * e] = __fmaf_rn(a.x, b.x, __fmul_rn(-a.y, b.y));
    s[2 * e] = __fmaf_rn(a.x, b.y, __fmul_rn(a.y, b.x));
    c[2 * e + 1] = __fmaf_rn(a.z, b.z, __fmul_rn(-a.w, b.w));
    s[2 * e + 1] = __fmaf_rn(a.z, b.w, __fmul_rn(a.w, b.z));
  }
}

// 8 consecutive elements as fp32, from bf16 (16 B) or fp32 (32 B) storage.
__device__ __forceinline__ void load8(const bf16 *p, float (&f)[8]) {
  const uint4 r = *reinterpret_cast<const uint4 *>(p);
  const uint32_t w[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    f[2 * e] = __uint_as_float(w[e] << 16);
    f[2 * e + 1] = __uint_as_float(w[e] & 0xFFFF0000u);
  }
}
__device__ __forceinline__ void load8(const float *p, float (&f)[8]) {
  const float4 a = reinterpret_cast<const float4 *>(p)[0];
  const float4 b = reinterpret_cast<const float4 *>(p)[1];
  f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w;
  f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
}
__device__ __forceinline__ void store8_bf16(bf16 *p, const float (&f)[8]) {
  uint32_t w[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    __nv_bfloat162 h = __floats2bfloat162_rn(f[2 * e], f[2 * e + 1]);
    w[e] = *reinterpret_cast<uint32_t *>(&h);
  }
  *reinterpret_cast<uint4 *>(p) = make_uint4(w[0], w[1], w[2], w[3]);
}
// Raw copy of 8 elements (bit-identical).
__device__ __forceinline__ void copy8(const bf16 *src, bf16 *dst) {
  *reinterpret_cast<uint4 *>(dst) = *reinterpret_cast<const uint4 *>(src);
}
__device__ __forceinline__ void copy8(const float *src, float *dst) {
  reinterpret_cast<float4 *>(dst)[0] = reinterpret_cast<const float4 *>(src)[0];
  reinterpret_cast<float4 *>(dst)[1] = reinterpret_cast<const float4 *>(src)[1];
}

// y_i = x_i c - x_{i+h} s ; y_{i+h} = x_{i+h} c + x_i s  (rotate-half RoPE).
// The rounding sequence is pinned with explicit intrinsics so that every
// kernel rotating the same value at the same position produces the same bits.
__device__ __forceinline__ void rotate8(float (&lo)[8], float (&hi)[8], const float (&c)[8],
                                        const float (&s)[8]) {
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    const float a = lo[e], b = hi[e];
    lo[e] = __fmaf_rn(a, c[e], __fmul_rn(-b, s[e]));
    hi[e] = __fmaf_rn(b, c[e], __fmul_rn(a, s[e]));
  }
}


}  // namespace dbsa
