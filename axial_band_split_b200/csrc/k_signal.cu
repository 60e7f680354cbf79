// Spectral front and back end of the separation pipeline and the chunk loop's kernels:
// the STFT of the model's input, the iSTFT of its separated spectra, and the padding,
// chunk gathering, fading and normalisation of "Mel-Band RoFormer — architecture, inference
// hot path & RTX 3050 feasibility", sections "The forward chain" (torch.stft n_fft 2048, hop
// 441, Hann window, center=True; istft back to the waveform) and "Verified inference hot
// path" (8 s chunks, stride 0.9 chunk, reflect padding, linear fades, out / counter).
//
// FFT: one CTA per frame, a radix-2 Stockham transform of n (power of two, <= 4096) complex
// points in shared memory (two ping-pong buffers, natural order out), twiddles from a table
// computed on the host in double precision.  The real input of a frame is transformed as a
// complex sequence with zero imaginary part; the inverse uses ifft(X) = conj(fft(conj X)) / n.
#include <cuda_runtime.h>

#include "mrf_internal.h"

namespace mrf {

namespace {

constexpr int kFftThreads = 256;

// Stockham radix-2 FFT of n = 2^log2n complex values: stage (l, m) maps a[k + j m] and
// a[k + j m + l m] to b[k + 2 j m] = sum and b[k + 2 j m + m] = w^(j m) * difference, w =
// exp(-2 pi i / n).  Returns the buffer that holds the result.
__device__ float2 *fft_smem(float2 *a, float2 *b, const float2 *__restrict__ tw, int log2n) {
  const int n = 1 << log2n;
  for (int lm = 0; lm < log2n; ++lm) {  // m = 2^lm, l = n / (2 m)
    const int m = 1 << lm, lmask = m - 1, lm_l = (n >> 1) >> lm;
    for (int bi = threadIdx.x; bi < (n >> 1); bi += blockDim.x) {
      const int j = bi >> lm, k = bi & lmask;
      const float2 w = tw[j << lm];
      const float2 c0 = a[k + (j << lm)], c1 = a[k + (j << lm) + lm_l * m];
      b[k + (j << (lm + 1))] = make_float2(c0.x + c1.x, c0.y + c1.y);
      const float2 d = make_float2(c0.x - c1.x, c0.y - c1.y);
      b[k + (j << (lm + 1)) + m] = make_float2(w.x * d.x - w.y * d.y, w.x * d.y + w.y * d.x);
    }
    __syncthreads();
    float2 *t = a;
    a = b;
    b = t;
  }
  return a;
}

// stft_repr[b, f * C + c, t] = sum_i x_pad[b, c, t hop + i] win[i] exp(-2 pi i f i / n), f <= n/2;
// x_pad is x reflect-padded by n/2 on both sides (numpy / torch "reflect": the edge sample is
// not repeated).  Grid (T, C, B).
__global__ void stft_kernel(const float *__restrict__ x, float *__restrict__ out, const float2 *__restrict__ tw,
                            const float *__restrict__ win, int C, int L, int T, int log2n, int hop) {
  extern __shared__ float2 fbuf[];
  const int n = 1 << log2n, F = (n >> 1) + 1;
  const int t = blockIdx.x, c = blockIdx.y, b = blockIdx.z;
  const float *xr = x + ((long long)b * C + c) * L;
  for (int i = threadIdx.x; i < n; i += blockDim.x) {
    int p = t * hop + i - (n >> 1);
    if (p < 0) p = -p;
    if (p >= L) p = 2 * (L - 1) - p;
    fbuf[i] = make_float2(xr[p] * win[i], 0.f);
  }
  __syncthreads();
  const float2 *r = fft_smem(fbuf, fbuf + n, tw, log2n);
  float2 *o = reinterpret_cast<float2 *>(out);
  for (int f = threadIdx.x; f < F; f += blockDim.x)
    o[(((long long)b * F + f) * C + c) * T + t] = r[f];
}

// frames[s, c, t, i] = win[i] * irfft(spec[s, f * C + c, t])[i]: the full Hermitian spectrum
// of the n/2 + 1 bins, inverse-transformed as conj(fft(conj X)) / n (real part).  Grid (T, C, S).
__global__ void istft_frames_kernel(const float *__restrict__ spec, float *__restrict__ frames,
                                    const float2 *__restrict__ tw, const float *__restrict__ win, int C, int T,
                                    int log2n) {
  extern __shared__ float2 fbuf[];
  const int n = 1 << log2n, F = (n >> 1) + 1;
  const int t = blockIdx.x, c = blockIdx.y, s = blockIdx.z;
  const float2 *sp = reinterpret_cast<const float2 *>(spec);
  for (int f = threadIdx.x; f < F; f += blockDim.x) {
    const float2 X = sp[(((long long)s * F + f) * C + c) * T + t];
    fbuf[f] = make_float2(X.x, -X.y);                       // conj X[f]
    if (f > 0 && f < F - 1) fbuf[n - f] = X;                // conj(X[n - f]) = X[f]
  }
  __syncthreads();
  const float2 *r = fft_smem(fbuf, fbuf + n, tw, log2n);
  const float inv = 1.f / (float)n;
  float *fr = frames + (((long long)s * C + c) * T + t) * n;
  for (int i = threadIdx.x; i < n; i += blockDim.x) fr[i] = r[i].x * inv * win[i];
}

// out[s, c, j] = sum_t frames[s, c, t, p - t hop] / sum_t win[p - t hop]^2 at p = j + n/2,
// over the frames covering p (the division skipped where the envelope is below 1e-11).
__global__ void istft_ola_kernel(const float *__restrict__ frames, float *__restrict__ out,
                                 const float *__restrict__ win, int S, int C, int T, int n, int hop, int length) {
  const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const long long total = (long long)S * C * length;
  if (idx >= total) return;
  const int j = (int)(idx % length);
  const long long sc = idx / length;
  const int p = j + (n >> 1);
  const int t_hi = min(T - 1, p / hop);
  const int t_lo = p >= n ? (p - n) / hop + 1 : 0;
  const float *fr = frames + sc * T * n;
  float acc = 0.f, env = 0.f;
  for (int t = t_lo; t <= t_hi; ++t) {
    const int i = p - t * hop;
    acc += fr[(long long)t * n + i];
    env += win[i] * win[i];
  }
  out[idx] = env > 1e-11f ? acc / env : acc;
}

// xp[c, i] = mix[c, reflect(i - border)] for i < L + 2 border.
__global__ void pad_reflect_kernel(const float *__restrict__ mix, float *__restrict__ xp, int C, int L, int border) {
  const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const int Lp = L + 2 * border;
  if (idx >= (long long)C * Lp) return;
  const int c = (int)(idx / Lp), i = (int)(idx % Lp);
  int p = i - border;
  if (p < 0) p = -p;
  if (p >= L) p = 2 * (L - 1) - p;
  xp[idx] = mix[(long long)c * L + p];
}

// chunks[k, c, i] = xp[c, off_k + i] for i < n_k; past n_k the chunk's own reflection
// (mode 1) or zeros (mode 0).
__global__ void gather_chunks_kernel(const float *__restrict__ xp, float *__restrict__ chunks, ChunkBatch cb, int C,
                                     int Lp, int chunk) {
  const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= (long long)cb.count * C * chunk) return;
  const int i = (int)(idx % chunk);
  const int c = (int)((idx / chunk) % C);
  const int k = (int)(idx / ((long long)chunk * C));
  const int off = cb.off[k], n = cb.n[k];
  float v = 0.f;
  if (i < n) v = xp[(long long)c * Lp + off + i];
  else if (cb.reflect[k]) v = xp[(long long)c * Lp + off + 2 * (n - 1) - i];
  chunks[idx] = v;
}

// acc[s, c, off + i] += est[s, c, i] * w[i], counter[off + i] += w[i] for i < n, w the
// chunk's fade window: linspace(0, 1, fade) over its first fade samples (1 on the first
// chunk), linspace(1, 0, fade) over its last (1 on the last chunk), 1 elsewhere.
__global__ void accumulate_chunk_kernel(const float *__restrict__ est, float *__restrict__ acc,
                                        float *__restrict__ counter, int S, int C, int Lp, int chunk, int fade,
                                        int off, int n, int first, int last) {
  const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= (long long)S * C * n) return;
  const int i = (int)(idx % n);
  const long long sc = idx / n;
  float w = 1.f;
  if (!first && i < fade) w = (float)i / (float)(fade - 1);
  if (!last && i >= chunk - fade) w = 1.f - (float)(i - (chunk - fade)) / (float)(fade - 1);
  acc[sc * Lp + off + i] += est[sc * chunk + i] * w;
  if (sc == 0) counter[off + i] += w;
}

// out[s, c, j] = acc[s, c, j + border] / max(counter[j + border], 1e-8).
__global__ void finalize_kernel(const float *__restrict__ acc, const float *__restrict__ counter,
                                float *__restrict__ out, int S, int C, int Lp, int L, int border) {
  const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= (long long)S * C * L) return;
  const int j = (int)(idx % L);
  const long long sc = idx / L;
  out[idx] = acc[sc * Lp + j + border] / fmaxf(counter[j + border], 1e-8f);
}

unsigned blocks(long long n, int bs) { return (unsigned)((n + bs - 1) / bs); }

}  // namespace

bool signal_kernels_init() {
  return cudaFuncSetAttribute(stft_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 2 * 4096 * 8) ==
             cudaSuccess &&
         cudaFuncSetAttribute(istft_frames_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 2 * 4096 * 8) ==
             cudaSuccess;
}

void launch_stft(const float *x, float *out, const float2 *tw, const float *win, int B, int C, int L, int T,
                 int log2n, int hop, cudaStream_t st) {
  const size_t smem = 2 * (size_t(1) << log2n) * sizeof(float2);
  stft_kernel<<<dim3(T, C, B), kFftThreads, smem, st>>>(x, out, tw, win, C, L, T, log2n, hop);
}

void launch_istft(const float *spec, float *frames, float *out, const float2 *tw, const float *win, int S, int C,
                  int T, int log2n, int hop, int length, cudaStream_t st) {
  const size_t smem = 2 * (size_t(1) << log2n) * sizeof(float2);
  istft_frames_kernel<<<dim3(T, C, S), kFftThreads, smem, st>>>(spec, frames, tw, win, C, T, log2n);
  const long long n = (long long)S * C * length;
  istft_ola_kernel<<<blocks(n, 256), 256, 0, st>>>(frames, out, win, S, C, T, 1 << log2n, hop, length);
}

void launch_pad_reflect(const float *mix, float *xp, int C, int L, int border, cudaStream_t st) {
  pad_reflect_kernel<<<blocks((long long)C * (L + 2 * border), 256), 256, 0, st>>>(mix, xp, C, L, border);
}

void launch_gather_chunks(const float *xp, float *chunks, const ChunkBatch &cb, int C, int Lp, int chunk,
                          cudaStream_t st) {
  gather_chunks_kernel<<<blocks((long long)cb.count * C * chunk, 256), 256, 0, st>>>(xp, chunks, cb, C, Lp, chunk);
}

void launch_accumulate_chunk(const float *est, float *acc, float *counter, int S, int C, int Lp, int chunk, int fade,
                             int off, int n, bool first, bool last, cudaStream_t st) {
  accumulate_chunk_kernel<<<blocks((long long)S * C * n, 256), 256, 0, st>>>(est, acc, counter, S, C, Lp, chunk,
                                                                             fade, off, n, first, last);
}

void launch_finalize(const float *acc, const float *counter, float *out, int S, int C, int Lp, int L, int border,
                     cudaStream_t st) {
  finalize_kernel<<<blocks((long long)S * C * L, 256), 256, 0, st>>>(acc, counter, out, S, C, Lp, L, border);
}

}  // namespace mrf
