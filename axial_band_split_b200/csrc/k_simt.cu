// CUDA-core kernels: the band split, the overlap average, and the fp32 debug schedule
// (grouped SIMT GEMM, row norm, RoPE split, online-softmax attention).
//
// Passages: "Mel-Band RoFormer — architecture, inference hot path & RTX 3050
// feasibility", sections "The forward chain", "The mel-band split, exactly" (RMSNorm is
// x / max(|x|, 1e-12) * sqrt(d) * gamma) and "The two transformers are not the same
// shape"; "@audio/neural-separate 0.4.0 → 0.5.0", package/scripts/export-roformer.py,
// class Core (gamma*sqrt(d) folded into the next Linear; masks averaged from at most two
// sources with a per-row weight).
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <cmath>

#include "mrf_internal.h"

namespace mrf {

namespace {

constexpr float kNormEps = 1e-12f;

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

__device__ __forceinline__ float gelu_erf(float x) { return 0.5f * x * (1.f + erff(x * 0.70710678118654752f)); }
__device__ __forceinline__ float sigm(float x) { return 1.f / (1.f + expf(-x)); }

// ------------------------------------------------------------------ band split
// CTA: one band k, kFrames consecutive frames (b, t flattened).  Features are gathered
// into shared memory, normalised per frame, then multiplied by the band's weight stored
// transposed [width][dim] so that a warp reads 32 consecutive outputs' weights.
constexpr int kBsFrames = 16;
constexpr int kBsThreads = 128;

__global__ void __launch_bounds__(kBsThreads) band_split_kernel(
    const float *__restrict__ in, const int32_t *__restrict__ feat_row,
    const int32_t *__restrict__ feat_c, const BandDesc *__restrict__ bands, int nb,
    const float *__restrict__ wt, const float *__restrict__ bias, int dim, int B, int T, int R,
    float *__restrict__ X, __half *__restrict__ Xh, float *__restrict__ ss) {
  extern __shared__ float xs[];  // [kBsFrames][width]
  __shared__ float red[kBsThreads / 32][kBsFrames];
  const int k = blockIdx.y;
  const BandDesc bd = bands[k];
  const int W = bd.width;
  const long long frames = (long long)B * T;
  const long long f0 = (long long)blockIdx.x * kBsFrames;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  // gather
  for (int i = tid; i < kBsFrames * W; i += kBsThreads) {
    const int f = i / W, e = i % W;
    const long long bt = f0 + f;
    float v = 0.f;
    if (bt < frames) {
      const long long b = bt / T, t = bt % T;
      const int row = feat_row[bd.feat_off + e], c = feat_c[bd.feat_off + e];
      v = in[((b * R + row) * T + t) * 2 + c];
    }
    xs[i] = v;
  }
  __syncthreads();
  // per-frame L2 normalisation (gamma * sqrt(d_in) is folded into the weight)
  for (int f = warp; f < kBsFrames; f += kBsThreads / 32) {
    float s = 0.f;
    for (int e = lane; e < W; e += 32) s += xs[f * W + e] * xs[f * W + e];
    s = warp_sum(s);
    const float r = 1.f / fmaxf(sqrtf(s), kNormEps);
    for (int e = lane; e < W; e += 32) xs[f * W + e] *= r;
  }
  __syncthreads();
  float sq[kBsFrames];
#pragma unroll
  for (int f = 0; f < kBsFrames; ++f) sq[f] = 0.f;
  const float *wk = wt + bd.w_off;
  for (int d = tid; d < dim; d += kBsThreads) {
    float acc[kBsFrames];
#pragma unroll
    for (int f = 0; f < kBsFrames; ++f) acc[f] = 0.f;
    for (int e = 0; e < W; ++e) {
      const float w = wk[(long long)e * dim + d];
#pragma unroll
      for (int f = 0; f < kBsFrames; ++f) acc[f] = fmaf(w, xs[f * W + e], acc[f]);
    }
    const float bb = bias[(long long)k * dim + d];
#pragma unroll
    for (int f = 0; f < kBsFrames; ++f) {
      const long long bt = f0 + f;
      if (bt >= frames) continue;
      const float v = acc[f] + bb;
      const long long tok = bt * nb + k;
      X[tok * dim + d] = v;
      if (Xh) Xh[tok * dim + d] = __float2half_rn(v);
      sq[f] += v * v;
    }
  }
  if (ss) {
#pragma unroll
    for (int f = 0; f < kBsFrames; ++f) {
      const float s = warp_sum(sq[f]);
      if (lane == 0) red[warp][f] = s;
    }
    __syncthreads();
    if (tid < kBsFrames) {
      const long long bt = f0 + tid;
      float s = 0.f;
      for (int w = 0; w < kBsThreads / 32; ++w) s += red[w][tid];
      if (bt < frames) ss[bt * nb + k] = s;
    }
  }
}

// ------------------------------------------------------------------ grouped SIMT GEMM
constexpr int kGt = 64, kGk = 16;

__global__ void __launch_bounds__(256) gemm_f32_kernel(
    const float *__restrict__ A, const float *__restrict__ Wt, const float *__restrict__ bias,
    float *__restrict__ C, const SimtGroup *__restrict__ groups, int M, int K, int epi) {
  const SimtGroup g = groups[blockIdx.z];
  const int n0 = blockIdx.x * kGt, m0 = blockIdx.y * kGt;
  if (n0 >= g.N) return;
  __shared__ float As[kGk][kGt + 4];
  __shared__ float Ws[kGk][kGt + 4];
  const int tid = threadIdx.x, tx = tid % 16, ty = tid / 16;
  const float *a = A + g.a_off;
  const float *w = Wt + g.w_off;
  float acc[4][4] = {};
  for (int k0 = 0; k0 < K; k0 += kGk) {
    for (int i = tid; i < kGt * kGk; i += 256) {
      const int r = i / kGk, kk = i % kGk;
      const int m = m0 + r, n = n0 + r, kx = k0 + kk;
      As[kk][r] = (m < M && kx < K) ? a[(long long)m * g.lda + kx] : 0.f;
      Ws[kk][r] = (n < g.N && kx < K) ? w[(long long)n * K + kx] : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < kGk; ++kk) {
      float av[4], wv[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) { av[i] = As[kk][ty * 4 + i]; wv[i] = Ws[kk][tx * 4 + i]; }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(av[i], wv[j], acc[i][j]);
    }
    __syncthreads();
  }
  float *c = C + g.c_off;
  const float *bs = bias ? bias + g.bias_off : nullptr;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int m = m0 + ty * 4 + i;
    if (m >= M) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int n = n0 + tx * 4 + j;
      if (n >= g.N) continue;
      float v = acc[i][j] + (bs ? bs[n] : 0.f);
      float *dst = c + (long long)m * g.ldc;
      switch (epi) {
        case kEpiResidual: dst[n] += v; break;
        case kEpiGelu: dst[n] = gelu_erf(v); break;
        case kEpiTanh: dst[n] = tanhf(v); break;
        case kEpiSigmoid: dst[n] = sigm(v); break;
        case kEpiGlu:
          // columns interleaved (value e, gate e): j even holds the value, j+1 the gate
          if ((j & 1) == 0 && n + 1 < g.N) {
            const float gt = acc[i][j + 1] + (bs ? bs[n + 1] : 0.f);
            dst[n >> 1] = v * sigm(gt);
          }
          break;
        case kEpiGeglu:
          if ((j & 1) == 0 && n + 1 < g.N) {
            const float gt = acc[i][j + 1] + (bs ? bs[n + 1] : 0.f);
            dst[n >> 1] = v * gelu_erf(gt);
          }
          break;
        default: dst[n] = v; break;
      }
    }
  }
}

// ------------------------------------------------------------------ row norm
__global__ void rownorm_kernel(const float *__restrict__ x, const float *__restrict__ gain,
                               float *__restrict__ y, long long rows, int D) {
  const long long row = (long long)blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32;
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  const float *xr = x + row * D;
  float s = 0.f;
  for (int j = lane; j < D; j += 32) s += xr[j] * xr[j];
  s = warp_sum(s);
  const float r = 1.f / fmaxf(sqrtf(s), kNormEps);
  float *yr = y + row * D;
  for (int j = lane; j < D; j += 32) yr[j] = xr[j] * r * gain[j];
}

// ------------------------------------------------------------------ RoPE split
// One thread per (token, feature pair) of the projection row [q | k | v] (q and k heads x dqk,
// v heads x dv, each (head, d)); pairs of q and k are rotated by their position.
__global__ void rope_split_kernel(const float *__restrict__ qkv, const float2 *__restrict__ rope,
                                  float *__restrict__ q, float *__restrict__ k,
                                  float *__restrict__ v, int B, int T, int nb, int H, int dqk, int dv,
                                  int axis) {
  const long long ntok = (long long)B * T * nb;
  const int Aqk = H * dqk, W = 2 * Aqk + H * dv, halfw = W / 2;
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= ntok * halfw) return;
  const int c = 2 * (int)(i % halfw);           // feature of the pair's first value
  const long long tok = i / halfw;
  const int which = c < Aqk ? 0 : c < 2 * Aqk ? 1 : 2;
  const int width = which < 2 ? dqk : dv;
  const int rel = c - which * Aqk;
  const int head = rel / width, d = rel % width;
  const int band = tok % nb;
  const long long bt = tok / nb;
  const long long b = bt / T, t = bt % T;
  long long seq; int pos, n;
  if (axis == 0) { seq = b * nb + band; pos = (int)t; n = T; }
  else { seq = bt; pos = band; n = nb; }
  const float x0 = qkv[tok * W + c], x1 = qkv[tok * W + c + 1];
  float y0 = x0, y1 = x1;
  if (which < 2) {
    const float2 cs = rope[(long long)pos * (dqk / 2) + d / 2];
    y0 = x0 * cs.x - x1 * cs.y;
    y1 = x1 * cs.x + x0 * cs.y;
  }
  float *dst = which == 0 ? q : which == 1 ? k : v;
  const long long o = ((seq * H + head) * n + pos) * width + d;
  dst[o] = y0;
  dst[o + 1] = y1;
}

// ------------------------------------------------------------------ attention (CUDA cores)
// One warp per query row; keys in chunks of 32 (one per lane), online softmax.  q, k, v
// are [(seq*H + head)*n_pad + pos]*dh; o[tok, head*dh + d] = gate[tok, head] * result.
__device__ __forceinline__ float ld_f(const float *p) { return *p; }
__device__ __forceinline__ float ld_f(const __half *p) { return __half2float(*p); }
__device__ __forceinline__ void st_f(float *p, float v) { *p = v; }
__device__ __forceinline__ void st_f(__half *p, float v) { *p = __float2half_rn(v); }

template <class TI, class TO>
__global__ void attention_simt_kernel(const TI *__restrict__ q, const TI *__restrict__ k,
                                      const TI *__restrict__ v, const float *__restrict__ gate,
                                      TO *__restrict__ o, int B, int T, int nb, int H, int dh,
                                      int dv, int axis, int n_pad) {
  __shared__ float qs[8][128];
  const int warp = threadIdx.x / 32, lane = threadIdx.x & 31;
  const long long nseq = axis == 0 ? (long long)B * nb : (long long)B * T;
  const int n = axis == 0 ? T : nb;
  const long long qi = (long long)blockIdx.x * 8 + warp;
  if (qi >= nseq * H * n) return;
  const int pos = qi % n;
  const long long sh = qi / n;  // seq * H + head
  const int head = sh % H;
  const long long seq = sh / H;
  const TI *qr = q + (sh * n_pad + pos) * dh;
  const float scale = rsqrtf((float)dh);
  for (int d = lane; d < dh; d += 32) qs[warp][d] = ld_f(qr + d) * scale;
  __syncwarp();
  const TI *kb = k + sh * n_pad * dh;
  const TI *vb = v + sh * n_pad * dv;
  float m = -INFINITY, l = 0.f, o0 = 0.f, o1 = 0.f;
  for (int j0 = 0; j0 < n; j0 += 32) {
    const int j = j0 + lane;
    float s = -INFINITY;
    if (j < n) {
      s = 0.f;
      for (int d = 0; d < dh; ++d) s = fmaf(qs[warp][d], ld_f(kb + (long long)j * dh + d), s);
    }
    const float mn = fmaxf(m, warp_max(s));
    const float p = (j < n) ? expf(s - mn) : 0.f;
    const float corr = expf(m - mn);
    l = l * corr + warp_sum(p);
    o0 *= corr; o1 *= corr;
    const int cnt = min(32, n - j0);
    for (int jj = 0; jj < cnt; ++jj) {
      const float pj = __shfl_sync(0xffffffffu, p, jj);
      const TI *vr = vb + (long long)(j0 + jj) * dv;
      if (lane < dv) o0 = fmaf(pj, ld_f(vr + lane), o0);
      if (lane + 32 < dv) o1 = fmaf(pj, ld_f(vr + lane + 32), o1);
    }
    m = mn;
  }
  long long tok;
  if (axis == 0) { const long long b = seq / nb, band = seq % nb; tok = (b * T + pos) * nb + band; }
  else tok = seq * nb + pos;
  const float g = gate[tok * H + head] / l;
  TO *orow = o + tok * (long long)H * dv + head * dv;
  if (lane < dv) st_f(orow + lane, o0 * g);
  if (lane + 32 < dv) st_f(orow + lane + 32, o1 * g);
}

__device__ __forceinline__ float to_f(__half v) { return __half2float(v); }
__device__ __forceinline__ float to_f(__nv_bfloat16 v) { return __bfloat162float(v); }
template <class T16>
__device__ __forceinline__ T16 from_f(float v);
template <>
__device__ __forceinline__ __half from_f<__half>(float v) { return __float2half_rn(v); }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float v) { return __float2bfloat16_rn(v); }

// Same on the tensor-core schedule's token-major projection rows (fp16, or bf16) qkv[tok][ld] = [q | k | v | gates]
// (gates already squashed by the sigmoid), for head widths the tensor-core kernel does not take.
template <class T16>
__global__ void attention_tokmajor_kernel(const T16 *__restrict__ qkv, int ld, T16 *__restrict__ o, int B,
                                          int T, int nb, int H, int dh, int dv, int axis) {
  __shared__ float qs[8][128];
  const int warp = threadIdx.x / 32, lane = threadIdx.x & 31;
  const long long nseq = axis == 0 ? (long long)B * nb : (long long)B * T;
  const int n = axis == 0 ? T : nb;
  const long long qi = (long long)blockIdx.x * 8 + warp;
  if (qi >= nseq * H * n) return;
  const int A = H * dh, Av = H * dv;  // q (and k) width, v width
  const int pos = qi % n;
  const long long sh = qi / n;
  const int head = sh % H;
  const long long seq = sh / H;
  // token of position p of this sequence
  auto tok_of = [&](int p_) -> long long {
    if (axis == 0) { const long long b = seq / nb, band = seq % nb; return (b * T + p_) * nb + band; }
    return seq * nb + p_;
  };
  const long long tq = tok_of(pos);
  const float scale = rsqrtf((float)dh);
  for (int d = lane; d < dh; d += 32) qs[warp][d] = to_f(qkv[tq * ld + head * dh + d]) * scale;
  __syncwarp();
  float m = -INFINITY, l = 0.f, o0 = 0.f, o1 = 0.f;
  for (int j0 = 0; j0 < n; j0 += 32) {
    const int j = j0 + lane;
    float s = -INFINITY;
    if (j < n) {
      const T16 *kr = qkv + tok_of(j) * ld + A + head * dh;
      s = 0.f;
      for (int d = 0; d < dh; ++d) s = fmaf(qs[warp][d], to_f(kr[d]), s);
    }
    const float mn = fmaxf(m, warp_max(s));
    const float p = (j < n) ? expf(s - mn) : 0.f;
    const float corr = expf(m - mn);
    l = l * corr + warp_sum(p);
    o0 *= corr; o1 *= corr;
    const int cnt = min(32, n - j0);
    for (int jj = 0; jj < cnt; ++jj) {
      const float pj = __shfl_sync(0xffffffffu, p, jj);
      const T16 *vr = qkv + tok_of(j0 + jj) * ld + 2 * A + head * dv;
      if (lane < dv) o0 = fmaf(pj, to_f(vr[lane]), o0);
      if (lane + 32 < dv) o1 = fmaf(pj, to_f(vr[lane + 32]), o1);
    }
    m = mn;
  }
  const float g = to_f(qkv[tq * ld + 2 * A + Av + head]) / l;
  T16 *orow = o + tq * (long long)Av + head * dv;
  if (lane < dv) orow[lane] = from_f<T16>(o0 * g);
  if (lane + 32 < dv) orow[lane + 32] = from_f<T16>(o1 * g);
}

// ------------------------------------------------------------------ overlap average
// masks[b, r, t, c] = wrow[r] * (m[b, t, src0] + m[b, t, src1]) written at out + b * out_bstride
// + (r T + t) 2 + c; with `spec` (stft_repr [B, R, T, 2]) the complex product of the mask and
// spec at (b, r, t) is written instead (the separated spectrum).
__global__ void overlap_average_kernel(const float *__restrict__ m, int ldm,
                                       const int32_t *__restrict__ src0,
                                       const int32_t *__restrict__ src1,
                                       const float *__restrict__ wrow, float *__restrict__ out,
                                       long long out_bstride, const float *__restrict__ spec,
                                       int B, int T, int R) {
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const long long total = (long long)B * R * T * 2;
  if (i >= total) return;
  const int c = i & 1;
  const long long t = (i >> 1) % T;
  const long long r = ((i >> 1) / T) % R;
  const long long b = (i >> 1) / ((long long)T * R);
  const long long j = i - b * (long long)R * T * 2;  // (r T + t) 2 + c
  const float *mr = m + (b * T + t) * ldm;
  const float w = wrow[r];
  auto mask = [&](int cc) {
    const int o = (int)r * 2 + cc;
    const int s0 = src0[o], s1 = src1[o];
    float v = mr[s0];
    if (s1 >= 0) v += mr[s1];
    return v * w;
  };
  if (!spec) {
    out[b * out_bstride + j] = mask(c);
    return;
  }
  const float m_re = mask(0), m_im = mask(1);
  const float *x = spec + i - c;
  out[b * out_bstride + j] = c == 0 ? m_re * x[0] - m_im * x[1] : m_re * x[1] + m_im * x[0];
}

__global__ void fill_kernel(float *p, float v, long long n) {
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) p[i] = v;
}

unsigned grid1(long long n, int bs) { return (unsigned)((n + bs - 1) / bs); }

}  // namespace

void launch_band_split(const float *in, const int32_t *feat_row, const int32_t *feat_c,
                       const BandDesc *bands, int nb, const float *w, const float *bias, int dim,
                       int B, int T, int rows, float *X, __half *Xh, float *ss, cudaStream_t st,
                       int max_width) {
  const long long frames = (long long)B * T;
  dim3 grid(grid1(frames, kBsFrames), nb);
  const size_t smem = sizeof(float) * kBsFrames * max_width;
  band_split_kernel<<<grid, kBsThreads, smem, st>>>(in, feat_row, feat_c, bands, nb, w, bias, dim,
                                                   B, T, rows, X, Xh, ss);
}

void launch_gemm_f32(const float *A, const float *W, const float *bias, float *C,
                     const SimtGroup *groups_dev, int ngroups, int M, int K, int max_n, int epi,
                     cudaStream_t st) {
  dim3 grid(grid1(max_n, kGt), grid1(M, kGt), ngroups);
  gemm_f32_kernel<<<grid, 256, 0, st>>>(A, W, bias, C, groups_dev, M, K, epi);
}

void launch_rownorm_f32(const float *x, const float *gain, float *y, long long rows, int D,
                        cudaStream_t st) {
  rownorm_kernel<<<grid1(rows, 8), 256, 0, st>>>(x, gain, y, rows, D);
}

void launch_rope_split_f32(const float *qkv, const float2 *rope, float *q, float *k, float *v,
                           int B, int T, int nb, int heads, int dqk, int dv, int axis, cudaStream_t st) {
  const long long n = (long long)B * T * nb * heads * (2 * dqk + dv) / 2;
  rope_split_kernel<<<grid1(n, 256), 256, 0, st>>>(qkv, rope, q, k, v, B, T, nb, heads, dqk, dv, axis);
}

void launch_attention_f32(const float *q, const float *k, const float *v, const float *gate,
                          float *o, int B, int T, int nb, int heads, int dqk, int dv, int axis,
                          cudaStream_t st) {
  const long long rows = (long long)B * T * nb * heads;
  const int n = axis == 0 ? T : nb;
  attention_simt_kernel<float, float><<<grid1(rows, 8), 256, 0, st>>>(q, k, v, gate, o, B, T, nb, heads, dqk,
                                                                      dv, axis, n);
}

void launch_attention_simt_f16(const __half *qkv, int ld, __half *o, int B, int T, int nb, int heads, int dqk,
                               int dv, int axis, bool bf16, cudaStream_t st) {
  const long long rows = (long long)B * T * nb * heads;
  if (bf16)
    attention_tokmajor_kernel<__nv_bfloat16><<<grid1(rows, 8), 256, 0, st>>>(
        reinterpret_cast<const __nv_bfloat16 *>(qkv), ld, reinterpret_cast<__nv_bfloat16 *>(o), B, T, nb, heads, dqk,
        dv, axis);
  else
    attention_tokmajor_kernel<__half><<<grid1(rows, 8), 256, 0, st>>>(qkv, ld, o, B, T, nb, heads, dqk, dv, axis);
}


void launch_overlap_average(const float *m, int ldm, const int32_t *src0, const int32_t *src1,
                            const float *row_weight, float *masks, long long out_bstride, const float *spec,
                            int B, int T, int rows, cudaStream_t st) {
  const long long n = (long long)B * rows * T * 2;
  overlap_average_kernel<<<grid1(n, 256), 256, 0, st>>>(m, ldm, src0, src1, row_weight, masks, out_bstride,
                                                        spec, B, T, rows);
}

void launch_fill_f32(float *p, float v, long long n, cudaStream_t st) {
  fill_kernel<<<grid1(n, 256), 256, 0, st>>>(p, v, n);
}

}  // namespace mrf
