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

// GELU of y0 = v0 * rs + b0 and y1 = v1 * rs + b1, y * (1 + erf(y / sqrt 2)) / 2.  The
// complementary error function of z = |y| / sqrt 2 comes from Abramowitz & Stegun 7.1.28,
// erfc(z) = (1 + a1 z + ... + a6 z^6)^-16 (|error| <= 3e-7), one reciprocal per value (the
// power by four squarings; it overflows to inf for large z, whose reciprocal is 0).  Then
// 1 + erf(y / sqrt 2) = 2 - erfc for y >= 0 and erfc for y < 0, so no cancellation on the
// negative side.  The polynomial and the scalings run in packed pairs.
__device__ __forceinline__ float2 gelu2(float v0, float v1, float rs, float b0, float b1) {
  const unsigned long long y = fma2(f2_pack(v0, v1), f2_pack(rs, rs), f2_pack(b0, b1));
  const float2 yy = f2_unpack(y);
  const unsigned long long z = mul2(f2_pack(fabsf(yy.x), fabsf(yy.y)), f2_pack(0.70710678118654752f, 0.70710678118654752f));
  unsigned long long p = fma2(z, f2_pack(0.0000430638f, 0.0000430638f), f2_pack(0.0002765672f, 0.0002765672f));
  p = fma2(z, p, f2_pack(0.0001520143f, 0.0001520143f));
  p = fma2(z, p, f2_pack(0.0092705272f, 0.0092705272f));
  p = fma2(z, p, f2_pack(0.0422820123f, 0.0422820123f));
  p = fma2(z, p, f2_pack(0.0705230784f, 0.0705230784f));
  p = fma2(z, p, f2_pack(1.f, 1.f));
  p = mul2(p, p);
  p = mul2(p, p);
  p = mul2(p, p);
  p = mul2(p, p);
  const float2 pp = f2_unpack(p);
  float r0, r1;  // erfc(|y| / sqrt 2)
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r0) : "f"(pp.x));
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r1) : "f"(pp.y));
  const float2 two_minus = f2_unpack(fma2(f2_pack(r0, r1), f2_pack(-1.f, -1.f), f2_pack(2.f, 2.f)));
  const unsigned long long q = f2_pack(yy.x >= 0.f ? two_minus.x : r0, yy.y >= 0.f ? two_minus.y : r1);
  return f2_unpack(mul2(mul2(y, f2_pack(0.5f, 0.5f)), q));
}

}  // namespace tcm
}  // namespace mrf
