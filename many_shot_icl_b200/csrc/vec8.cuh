// Device helpers shared by the kernels: RoPE angle factors from the two-level
// table, and 8-element vector loads/stores between bf16/fp32 storage and fp32
// registers.
#pragma once

#include <cuda_bf16.h>

#include "dbsa_internal.h"

namespace dbsa {

using bf16 = __nv_bfloat16;

// (cos, sin) of p * w_i for the 8 frequencies i0..i0+7, as the complex
// product hi[p >> 4] * lo[p & 15] (rounding pinned as in cmul below).
__device__ __forceinline__ void rope_cs8(const RopeTables &t, int64_t p, int i0, int half,
                                         float (&c)[8], float (&s)[8]) {
  const int64_t hoff = (p >> kRopeShift) * half + i0, loff = (p & (kRopeLo - 1)) * half + i0;
#pragma unroll
  for (int e = 0; e < 2; ++e) {
    const float4 hc = __ldg(reinterpret_cast<const float4 *>(t.hc + hoff) + e);
    const float4 hs = __ldg(reinterpret_cast<const float4 *>(t.hs + hoff) + e);
    const float4 lc = __ldg(reinterpret_cast<const float4 *>(t.lc + loff) + e);
    const float4 ls = __ldg(reinterpret_cast<const float4 *>(t.ls + loff) + e);
    const float ac[4] = {hc.x, hc.y, hc.z, hc.w}, as[4] = {hs.x, hs.y, hs.z, hs.w};
    const float bc[4] = {lc.x, lc.y, lc.z, lc.w}, bs[4] = {ls.x, ls.y, ls.z, ls.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      c[4 * e + k] = __fmaf_rn(ac[k], bc[k], __fmul_rn(-as[k], bs[k]));
      s[4 * e + k] = __fmaf_rn(ac[k], bs[k], __fmul_rn(as[k], bc[k]));
    }
  }
}

// (cos, sin) of p * w_i for one frequency i, with the rounding of rope_cs8.
__device__ __forceinline__ void rope_cs1(const RopeTables &t, int64_t p, int i, int half, float &c,
                                         float &s) {
  const int64_t hoff = (p >> kRopeShift) * half + i, loff = (p & (kRopeLo - 1)) * half + i;
  const float ac = __ldg(t.hc + hoff), as = __ldg(t.hs + hoff);
  const float bc = __ldg(t.lc + loff), bs = __ldg(t.ls + loff);
  c = __fmaf_rn(ac, bc, __fmul_rn(-as, bs));
  s = __fmaf_rn(ac, bs, __fmul_rn(as, bc));
}

// One element between bf16 / fp32 storage and fp32 (output rounding RNE).
__device__ __forceinline__ float to_f32(bf16 x) { return __bfloat162float(x); }
__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ void from_f32(float x, bf16 &d) { d = __float2bfloat16_rn(x); }
__device__ __forceinline__ void from_f32(float x, float &d) { d = x; }

// 2 consecutive elements as fp32, from bf16 (4 B) or fp32 (8 B) storage, and
// back to bf16 (RNE).
__device__ __forceinline__ void load2(const bf16 *p, float (&f)[2]) {
  const uint32_t w = *reinterpret_cast<const uint32_t *>(p);
  f[0] = __uint_as_float(w << 16);
  f[1] = __uint_as_float(w & 0xFFFF0000u);
}
__device__ __forceinline__ void load2(const float *p, float (&f)[2]) {
  const float2 v = *reinterpret_cast<const float2 *>(p);
  f[0] = v.x;
  f[1] = v.y;
}
__device__ __forceinline__ void store2_bf16(bf16 *p, const float (&f)[2]) {
  __nv_bfloat162 h = __floats2bfloat162_rn(f[0], f[1]);
  *reinterpret_cast<__nv_bfloat162 *>(p) = h;
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

// Packed pairs of fp32 (sm_100 f32x2 arithmetic: two independent IEEE fp32
// operations per instruction, each rounded exactly like its scalar form).
using f32x2 = unsigned long long;
__device__ __forceinline__ f32x2 f2_pack(float a, float b) {
  f32x2 r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
  return r;
}
__device__ __forceinline__ void f2_unpack(f32x2 r, float &a, float &b) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(r));
}
__device__ __forceinline__ f32x2 f2_fma(f32x2 a, f32x2 b, f32x2 c) {
  f32x2 d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ f32x2 f2_mul(f32x2 a, f32x2 b) {
  f32x2 d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ f32x2 f2_neg(f32x2 a) { return a ^ 0x8000000080000000ull; }
// bf16 pair (low half = first element) <-> packed fp32 pair
__device__ __forceinline__ f32x2 f2_from_bf16x2(uint32_t w) {
  return f2_pack(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
}
__device__ __forceinline__ uint32_t f2_to_bf16x2(f32x2 v) {
  float a, b;
  f2_unpack(v, a, b);
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t *>(&h);
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
