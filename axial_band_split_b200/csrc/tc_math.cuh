// Elementwise epilogue math shared by the tensor-core kernels: packed f32x2 helpers and
// the GELU of the feed-forward layers.
#pragma once
#include <cuda_fp16.h>

namespace mrf {
namespace tcm {

// Packed pairs (one f32x2 instruction for two lanes of math).
__device__ __forceinline__ unsigned long long f2_pack(float a, float b) {
  return (static_cast<unsigned long long>(__float_as_uint(b)) << 32) | __float_as_uint(a);
}
__device__ __forceinline__ float2 f2_unpack(unsigned long long v) {
  return make_float2(__uint_as_float(static_cast<unsigned>(v)), __uint_as_float(static_cast<unsigned>(v >> 32)));
}
__device__ __forceinline__ unsigned long long fma2(unsigned long long a, unsigned long long b, unsigned long long c) {
  unsigned long long d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ unsigned long long mul2(unsigned long long a, unsigned long long b) {
  unsigned long long d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}

// GELU of y0 = v0 * rs + b0 and y1 = v1 * rs + b1, y * (1 + erf(y / sqrt 2)) / 2, with the
// erf of Abramowitz & Stegun 7.1.26 (|error| <= 1.5e-7), branch-free:
// erf(z) = 1 - t (a1 + t (a2 + t (a3 + t (a4 + t a5)))) exp(-z^2), t = 1 / (1 + p z), z >= 0;
// the polynomial and the scalings in packed pairs.
__device__ __forceinline__ float2 gelu2(float v0, float v1, float rs, float b0, float b1) {
  const unsigned long long y = fma2(f2_pack(v0, v1), f2_pack(rs, rs), f2_pack(b0, b1));
  const float2 yy = f2_unpack(y);
  const unsigned long long z = mul2(f2_pack(fabsf(yy.x), fabsf(yy.y)), f2_pack(0.70710678118654752f, 0.70710678118654752f));
  const unsigned long long den = fma2(z, f2_pack(0.3275911f, 0.3275911f), f2_pack(1.f, 1.f));
  const float2 dd = f2_unpack(den);
  float t0, t1;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(t0) : "f"(dd.x));
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(t1) : "f"(dd.y));
  const unsigned long long t = f2_pack(t0, t1);
  unsigned long long poly = fma2(t, f2_pack(1.061405429f, 1.061405429f), f2_pack(-1.453152027f, -1.453152027f));
  poly = fma2(t, poly, f2_pack(1.421413741f, 1.421413741f));
  poly = fma2(t, poly, f2_pack(-0.284496736f, -0.284496736f));
  poly = fma2(t, poly, f2_pack(0.254829592f, 0.254829592f));
  poly = mul2(poly, t);
  const float2 ez = f2_unpack(mul2(mul2(z, z), f2_pack(-1.4426950408889634f, -1.4426950408889634f)));
  float e0, e1;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(e0) : "f"(ez.x));
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(e1) : "f"(ez.y));
  const float2 er = f2_unpack(fma2(poly, f2_pack(-e0, -e1), f2_pack(1.f, 1.f)));   // erf(|y| / sqrt 2)
  const unsigned long long h = mul2(y, f2_pack(0.5f, 0.5f));
  const float2 g = f2_unpack(fma2(h, f2_pack(copysignf(er.x, yy.x), copysignf(er.y, yy.y)), h));
  return g;
}

}  // namespace tcm
}  // namespace mrf
