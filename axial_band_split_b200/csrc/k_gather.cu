// Mel-band gather and BandSplit norm of the tensor-core schedule: per (band, frame) the band's
// features divided by their L2 norm, in the schedule's 16-bit type (fp16 or bf16), laid out as
// the A operand of the band-split GEMM.
//
// "Mel-Band RoFormer — architecture, inference hot path & RTX 3050 feasibility", section "The
// mel-band split, exactly": band k's features at frame t are the (re, im) pairs of the
// stft_repr rows f*C + s of its bins f (ascending) and channels s, i.e. the contiguous rows
// first_k*C .. (last_k + 1)*C - 1; the BandSplit RMSNorm is x / max(|x|_2, 1e-12) (its
// sqrt(d_in) * gamma is folded into the GEMM's weight).
//
// The gather is a transpose: stft_repr is [row][frame][re, im] (frames contiguous) and the
// GEMM wants [frame][feature] (features contiguous, feature 2 * (row - first row) + c).  A CTA
// takes one band and 32 frames of one window with 16 warps: warp w covers frames 4 (w % 8) ..
// 4 (w % 8) + 3 and every second 16-row step (from step w / 8), two lanes per row, each lane one
// 16-byte load of two frames' (re, im) (two 8-byte loads when T is odd, where a row's frame pairs
// are not 16-byte aligned): 32 contiguous bytes per row.
//   pass 1  loads (eight in flight per thread), per-frame sums of squares (shuffle-xor over the
//           lanes holding the same frames, then the two warps sharing the frames through shared
//           memory);
//   pass 2  the same loads again (the CTA's tile, at most 133 KB, is still in L2), scaled by
//           1 / max(|x|, 1e-12) and stored as fp16 pairs: each store instruction of a warp
//           writes 64 contiguous bytes of two frames' feature rows, so nothing is staged in
//           shared memory; rows up to the band's width rounded up to 64 features store zeros.
// Keeping the registers and shared memory small lets many CTAs share an SM, which hides the
// loads' latency; the widest bands (40 times the narrowest's data) are scheduled first.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "mrf_internal.h"

namespace mrf {

namespace {

constexpr int kFrames = 32;    // frames per CTA
constexpr int kThreads = 512;  // 16 warps: warp w covers frames 4 (w % 8) .. 4 (w % 8) + 3
constexpr float kNormEps = 1e-12f;

template <bool kEvenT>
__device__ __forceinline__ float4 load_pair(const float *p, int t, int T) {
  float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
  if (kEvenT) {
    if (t < T) v = __ldg(reinterpret_cast<const float4 *>(p));
  } else {
    if (t < T) {
      const float2 a = __ldg(reinterpret_cast<const float2 *>(p));
      v.x = a.x; v.y = a.y;
    }
    if (t + 1 < T) {
      const float2 c = __ldg(reinterpret_cast<const float2 *>(p + 2));
      v.z = c.x; v.w = c.y;
    }
  }
  return v;
}

// Two floats as one pair of the schedule's 16-bit type (fp16, or bf16 with kBF).
template <bool kBF>
__device__ __forceinline__ uint32_t pack2(float a, float b) {
  if constexpr (kBF) {
    __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t *>(&h);
  } else {
    __half2 h = __floats2half2_rn(a, b);
    return *reinterpret_cast<uint32_t *>(&h);
  }
}

template <bool kEvenT, bool kBF>
__global__ void __launch_bounds__(kThreads) band_gather_kernel(const float *__restrict__ in,
                                                                   const int32_t *__restrict__ feat_row,
                                                                   const BandDesc *__restrict__ bands, int nb,
                                                                   int B, int T, int R, int tiles,
                                                                   long long frame_stride, int k_stride,
                                                                   __half *__restrict__ A) {
  __shared__ float ss[2][kFrames];
  // programmatic dependent launch: the input may be an earlier kernel's output
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int per_band = B * tiles;
  const int k = nb - 1 - (int)(blockIdx.x / per_band);   // widest bands first
  const int rem = (int)(blockIdx.x % per_band);
  const int b = rem / tiles, t0 = (rem % tiles) * kFrames;
  const BandDesc bd = bands[k];
  const int nrows = bd.width >> 1, prow = ((bd.width + 63) & ~63) >> 1;  // rows, rows incl. zero padding
  const int row0 = feat_row[bd.feat_off];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int f0 = 4 * (warp & 7) + 2 * (lane & 1);  // this lane's two frames of the tile
  const int t = t0 + f0;
  const int rl = (warp >> 3) * 16 + (lane >> 1);   // first row; rows step by 32
  const float *base = in + (((long long)b * R + row0) * T + t) * 2;
  float s0 = 0.f, s1 = 0.f;
#pragma unroll 8
  for (int r = rl; r < nrows; r += 32) {
    const float4 v = load_pair<kEvenT>(base + (long long)r * T * 2, t, T);
    s0 = fmaf(v.x, v.x, fmaf(v.y, v.y, s0));
    s1 = fmaf(v.z, v.z, fmaf(v.w, v.w, s1));
  }
#pragma unroll
  for (int o = 2; o < 32; o <<= 1) {  // lanes of equal parity hold the same two frames
    s0 += __shfl_xor_sync(0xffffffffu, s0, o);
    s1 += __shfl_xor_sync(0xffffffffu, s1, o);
  }
  if (lane < 2) {  // every frame of the tile is written by exactly one lane of each row group
    ss[warp >> 3][f0] = s0;
    ss[warp >> 3][f0 + 1] = s1;
  }
  __syncthreads();
  const float sc0 = 1.f / fmaxf(sqrtf(ss[0][f0] + ss[1][f0]), kNormEps);
  const float sc1 = 1.f / fmaxf(sqrtf(ss[0][f0 + 1] + ss[1][f0 + 1]), kNormEps);
  const bool st0 = t < T, st1 = t + 1 < T;
  __half *out0 = A + ((long long)k * frame_stride + (long long)b * T + t) * k_stride;
  __half *out1 = out0 + k_stride;
#pragma unroll 4
  for (int r = rl; r < prow; r += 32) {
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    if (r < nrows) v = load_pair<kEvenT>(base + (long long)r * T * 2, t, T);
    if (st0) *reinterpret_cast<uint32_t *>(out0 + 2 * r) = pack2<kBF>(v.x * sc0, v.y * sc0);
    if (st1) *reinterpret_cast<uint32_t *>(out1 + 2 * r) = pack2<kBF>(v.z * sc1, v.w * sc1);
  }
}

}  // namespace

void launch_band_gather(const float *in, const int32_t *feat_row, const BandDesc *bands, int nb, int B, int T,
                        int rows, long long frame_stride, int k_stride, __half *A, bool bf16, bool pdl,
                        cudaStream_t st) {
  const int tiles = (T + kFrames - 1) / kFrames;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(nb * B * tiles), 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
#define MRF_GATHER(E, BF) \
  cudaLaunchKernelEx(&cfg, band_gather_kernel<E, BF>, in, feat_row, bands, nb, B, T, rows, tiles, frame_stride, k_stride, A)
  if (T % 2 == 0) {
    if (bf16) MRF_GATHER(true, true);
    else MRF_GATHER(true, false);
  } else {
    if (bf16) MRF_GATHER(false, true);
    else MRF_GATHER(false, false);
  }
#undef MRF_GATHER
}

}  // namespace mrf
