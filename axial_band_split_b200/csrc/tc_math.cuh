// Elementwise epilogue math shared by the tensor-core kernels: the GELU of the feed-forward
// layers (packed f32x2 pairs) and tanh and the sigmoid on the MUFU.
#pragma once
#include <cuda_fp16.h>

namespace mrf {
namespace tcm {

// GELU of y0 = v0 * rs + b0 and y1 = v1 * rs + b1, y * (1 + erf(y / sqrt 2)) / 2, written
// as max(y, 0) - |y| * erfc(|y| / sqrt 2) / 2 (both signs of y).  The complementary error
// function comes from Abramowitz & Stegun 7.1.28, erfc(z) = (1 + a1 z + ... + a6 z^6)^-16
// (|error| <= 3e-7): one reciprocal per value, the power by four squarings (it overflows to inf
// for large z, whose reciprocal is 0).  The polynomial is evaluated in w = -|y|: coefficient k
// is a_k 2^(-k/2) (z = |y| / sqrt 2) times (-1)^k (the sign of w^k) times 2^(1/16) (so the
// 16th power is doubled and its reciprocal is erfc / 2).  Packed pairs throughout.  (An
// infinite y gives NaN; finite inputs never reach inf.)
__device__ __forceinline__ float2 gelu2(float v0, float v1, float rs, float b0, float b1) {
  // packed pairs through the compiler's f32x2 builtins (one fma.rn.f32x2 / mul.rn.f32x2 each)
  const float2 y = __ffma2_rn(make_float2(v0, v1), make_float2(rs, rs), make_float2(b0, b1));
  const float2 w = make_float2(-fabsf(y.x), -fabsf(y.y));
  float2 q = __ffma2_rn(w, make_float2(5.62129980608006e-06f, 5.62129980608006e-06f),
                        make_float2(-5.105520904180594e-05f, -5.105520904180594e-05f));
  q = __ffma2_rn(w, q, make_float2(3.9686136005911976e-05f, 3.9686136005911976e-05f));
  q = __ffma2_rn(w, q, make_float2(-0.003422739217057824f, -0.003422739217057824f));
  q = __ffma2_rn(w, q, make_float2(0.02207699790596962f, 0.02207699790596962f));
  q = __ffma2_rn(w, q, make_float2(-0.052075162529945374f, -0.052075162529945374f));
  q = __ffma2_rn(w, q, make_float2(1.0442737340927124f, 1.0442737340927124f));
  q = __fmul2_rn(q, q);
  q = __fmul2_rn(q, q);
  q = __fmul2_rn(q, q);
  q = __fmul2_rn(q, q);
  float e0, e1;  // erfc(|y| / sqrt 2) / 2
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(e0) : "f"(q.x));
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(e1) : "f"(q.y));
  return __ffma2_rn(w, make_float2(e0, e1), make_float2(fmaxf(y.x, 0.f), fmaxf(y.y, 0.f)));
}

// tanh and the logistic sigmoid on the MUFU, from the identities tanh y = 1 - 2 / (1 + e^(2y))
// and sigmoid x = 1 / (1 + e^-x), with e^u = 2^(u log2 e) (ex2.approx: relative error about
// 2^-22) and the reciprocal by rcp.approx (relative error about 2^-23).  Absolute error of either
// below 2e-6 over all finite inputs, far under the fp16 resolution of the outputs they feed; the
// limits come out exactly: e^(2y) overflows to inf (tanh 1, rcp(inf) = 0) or underflows to 0
// (tanh -1).  Two MUFU operations a value, against the CUDA-core sequence of tanhf.
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float rcp_approx(float x) {
  float y;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
constexpr float kTwoLog2e = 2.8853900817779268f;   // 2 log2(e)
constexpr float kNegLog2e = -1.4426950408889634f;  // -log2(e)
__device__ __forceinline__ float tanh_mufu(float y) {
  return fmaf(-2.f, rcp_approx(1.f + ex2_approx(y * kTwoLog2e)), 1.f);
}
__device__ __forceinline__ float sigmoid_mufu(float x) { return rcp_approx(1.f + ex2_approx(x * kNegLog2e)); }

}  // namespace tcm
}  // namespace mrf
