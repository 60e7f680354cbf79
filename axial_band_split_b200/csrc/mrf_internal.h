// Internal declarations shared by the library's translation units.
#pragma once
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <string>
#include <vector>

#include "../../include/mrf.h"
#include "tables.h"

namespace mrf {

// ------------------------------------------------------------------ attention widths
// v per head (dim_head_v, or dim_head when 0); the projection row [q | k | v] and the attention
// output (the output projection's input).
inline int head_v(const mrf_config &c) { return c.dim_head_v > 0 ? c.dim_head_v : c.dim_head; }
inline int qkv_width(const mrf_config &c) { return c.heads * (2 * c.dim_head + head_v(c)); }
inline int attn_out_width(const mrf_config &c) { return c.heads * head_v(c); }

// ------------------------------------------------------------------ device status word
// Kernels with bounded waits write a nonzero code here instead of hanging or trapping.
enum DeviceStatus : unsigned { kStatusOk = 0, kStatusTimeout = 1 };

// ------------------------------------------------------------------ SIMT kernels (k_simt.cu)
// Per-band descriptor of the band split and the mask head.
struct BandDesc {
  int width;      // d_in of the band
  int feat_off;   // first feature of the band in the concatenated feature axis
  int w_off;      // first element of the band's band-split weight [dim, width]
  int w3_off;     // first element of the band's last mask layer [2*width, hidden] (fp32 path)
};

// X[(b*T + t)*nb + k, :] = W_k (x_k / max(|x_k|, eps)) + bias_k, gamma*sqrt(d_in) folded
// into W_k.  Also writes an fp16 copy and the row sum of squares when given.
void launch_band_split(const float *in, const int32_t *feat_row, const int32_t *feat_c,
                       const BandDesc *bands, int nb, const float *w, const float *bias,
                       int dim, int B, int T, int rows, float *X, __half *Xh, float *ss,
                       cudaStream_t st, int max_width);

// tensor-core schedule (k_gather.cu): normalised band features, fp16 (bf16 with bf16; the buffer
// type is the 16-bit container of either), [band][frame_stride][k_stride],
// each band's row zero-padded to a multiple of 64 (the A operand of the band-split GEMM).
void launch_band_gather(const float *in, const int32_t *feat_row, const BandDesc *bands, int nb, int B, int T,
                        int rows, long long frame_stride, int k_stride, __half *A, bool bf16, bool pdl,
                        cudaStream_t st);

enum SimtEpi : int {
  kEpiStore = 0,      // C = acc (+ bias)
  kEpiResidual = 1,   // C += acc (+ bias)
  kEpiGelu = 2,       // C = gelu(acc + bias)
  kEpiTanh = 3,       // C = tanh(acc + bias)
  kEpiSigmoid = 4,    // C = sigmoid(acc + bias)
  kEpiGlu = 5,        // value/gate halves of N: C[:, e] = v_e * sigmoid(g_e), N/2 outputs
  kEpiGeglu = 6,      // columns interleaved (value e, gate e): C[:, e] = v_e * gelu(g_e), N/2 outputs
};

// One group of a grouped fp32 GEMM: C[m, n] = sum_k A[m, k] * W[n, k] for m < M, n < N.
struct SimtGroup {
  long long a_off, w_off, c_off, bias_off;
  int lda, ldc, N, pad;
};
void launch_gemm_f32(const float *A, const float *W, const float *bias, float *C,
                     const SimtGroup *groups_dev, int ngroups, int M, int K, int max_n,
                     int epi, cudaStream_t st);

// y = x / max(|x|, eps) * gain (per column), rows of width D; y may alias x.
void launch_rownorm_f32(const float *x, const float *gain, float *y, long long rows, int D,
                        cudaStream_t st);

// qkv [tok, heads*(2 dqk + dv)] fp32 (q, k, v blocks, each (head, d)) -> q, k [seq*heads, n, dqk],
// v [seq*heads, n, dv], with RoPE on q and k.
// axis 0: sequences over time (seq = b*nb + band, pos = t); axis 1: over bands.
void launch_rope_split_f32(const float *qkv, const float2 *rope, float *q, float *k, float *v,
                           int B, int T, int nb, int heads, int dqk, int dv, int axis, cudaStream_t st);

// o[tok, head*dv + d] = gate[tok, head] * softmax(q k^T / sqrt(dqk)) v  (dqk <= 128, dv <= 64)
void launch_attention_f32(const float *q, const float *k, const float *v, const float *gate,
                          float *o, int B, int T, int nb, int heads, int dqk, int dv, int axis,
                          cudaStream_t st);

// Same on the tensor-core schedule's token-major rows qkv[tok][ld] = [q | k | v | sigmoid gates];
// 16-bit input and output (fp16, or bf16 with bf16).
void launch_attention_simt_f16(const __half *qkv, int ld, __half *o, int B, int T, int nb, int heads, int dqk,
                               int dv, int axis, bool bf16, cudaStream_t st);


// masks[b, r, t, c] = row_weight[r] * sum of the (<= 2) source features of (r, c)
// ------------------------------------------------------------------ spectral front / back end (k_signal.cu)
// Up to 16 chunks of the chunk loop gathered at once: chunk k covers samples off[k] .. off[k]
// + n[k] of the padded mix; past n[k] its own reflection (reflect[k] != 0) or zeros.
struct ChunkBatch {
  int count;
  int off[16], n[16], reflect[16];
};
bool signal_kernels_init();
// x [B, C, L] -> out [B, (n/2+1) C, T, 2], n = 2^log2n <= 4096; tw[i] = exp(-2 pi i i / n), i < n/2;
// win: the analysis window (n values).
void launch_stft(const float *x, float *out, const float2 *tw, const float *win, int B, int C, int L, int T,
                 int log2n, int hop, cudaStream_t st);
// spec [S, (n/2+1) C, T, 2] -> out [S, C, length]; frames: scratch of S * C * T * n floats.
void launch_istft(const float *spec, float *frames, float *out, const float2 *tw, const float *win, int S, int C,
                  int T, int log2n, int hop, int length, cudaStream_t st);
void launch_pad_reflect(const float *mix, float *xp, int C, int L, int border, cudaStream_t st);
void launch_gather_chunks(const float *xp, float *chunks, const ChunkBatch &cb, int C, int Lp, int chunk,
                          cudaStream_t st);
void launch_accumulate_chunk(const float *est, float *acc, float *counter, int S, int C, int Lp, int chunk, int fade,
                             int off, int n, bool first, bool last, cudaStream_t st);
void launch_finalize(const float *acc, const float *counter, float *out, int S, int C, int Lp, int L, int border,
                     cudaStream_t st);

// out_bstride: elements between batch items of `masks` (stems x rows x T x 2 when the
// stems are interleaved); spec: null, or stft_repr to multiply the masks into.
void launch_overlap_average(const float *m, int ldm, const int32_t *src0, const int32_t *src1,
                            const float *row_weight, float *masks, long long out_bstride, const float *spec,
                            int B, int T, int rows, cudaStream_t st);

void launch_fill_f32(float *p, float v, long long n, cudaStream_t st);

}  // namespace mrf
