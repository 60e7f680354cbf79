// Declarations of the tcgen05 GEMM (k_gemm_tc.cu) used by the fp16 schedule.
#pragma once
#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

namespace mrf {

// One group (a band of the mask head, or the single group of a trunk GEMM):
// C[m, n] = sum_k A[m, k] W[n, k] for m < M, n < N.
struct GemmGroup {
  int N;             // output columns of the group
  int n_tiles;       // ceil(N / BN)
  int n_tile_start;  // prefix sum of n_tiles over the previous groups
  int a_off;         // A: first row of the group (mode 0) or the group's coordinate (mode 1)
  int b_row_off;     // first row of the group's weight in the stacked weight matrix
  int out_off;       // epilogue output offset of the group
  int bias_off;      // offset of the group's bias
  int kblocks;       // 64-wide K blocks of the group (0: K / 64 of the launch)
};

enum GemmEpi : int {
  kTcQkv = 0,     // row norm, RoPE on q and k, softmax scale on q, sigmoid gates; token-major fp16 rows
  kTcResid = 1,   // x += acc (+ bias) on the fp16 residual stream Xh; row sums of squares
  kTcGelu = 2,    // out = gelu(acc * rowscale + bias) fp16
  kTcTanh = 3,    // out = tanh(acc + bias) fp16 (group-strided)
  kTcGlu = 4,     // interleaved (value, gate) pairs -> value * sigmoid(gate), averaged into the masks
  kTcBandSplit = 5,  // x = acc + bias for token m*nb + group (band) into Xh; row sums of squares
  kTcGeglu = 6,   // interleaved (value, gate) pairs of acc * rowscale + bias -> value * gelu(gate), fp16
};

struct GemmParams {
  int M, K, BN, ngroups, total_n_tiles, a_mode, m_tiles;
  int stall_test;  // test hook: CTA 0's loads never arrive, so its bounded waits expire
  const GemmGroup *groups;
  unsigned *status;
  // epilogue
  // Row sums of squares are written as partial sums, one slot per (column tile, epilogue warp of
  // the row's lane quarter), ss_out_parts slots a row; a consumer adds its ss_in_parts slots in
  // order (deterministic: no atomics).
  const float *ss_in;       // row scale 1 / max(sqrt(sum of the row's slots), eps); null: 1
  int ss_in_parts;
  const float *bias;
  __half *Xh;               // the 16-bit residual stream [M, ld] (fp16: kTcResid reads and rewrites it)
  float *X;                 // bf16 schedule: the fp32 master copy of the residual stream (read and rewritten)
  float *ss_out;            // row sums of squares of the output (partial slots)
  int ss_out_parts;
  int ld;
  __half *out_h;            // fp16 output
  float *out_f;             // fp32 output
  int ldo;
  long long out_group_stride;
  // q, k, v, gates rows
  const float2 *rope;
  const float *gbias;
  int B, T, nb, H, dh, A, axis;
  int Av;                   // kTcQkv: v width (heads x dim_head_v); the row is [q (A) | k (A) | v (Av) | gates]
  float q_scale;            // q is multiplied by this after RoPE (the attention's softmax scale)
  // deferred output norm of the previous transformer (kTcResid): the residual input x is
  // scaled by res_gain[col] / max(sqrt(res_ss[row]), eps) before the add (null: no scaling);
  // res_ss has ss_in_parts slots a row
  const float *res_ss;
  const float *res_gain;
  // kTcResid: also the partial sums of (out_gain[j] * x_j)^2 into ssg_out (null: skip)
  float *ssg_out;
  const float *out_gain;
  // kTcGlu: the overlap average.  Feature e (global feature index) adds row_weight[feat_row[e]]
  // times its GLU output to masks[b * mask_bstride + (feat_row[e] * T + t) * 2 + (e & 1)] (zeroed
  // beforehand), multiplied by the complex spec[b, feat_row[e], t] when spec is not null.
  const int32_t *feat_row;
  const float *row_weight;
  float *masks;
  long long mask_bstride;
  const float *spec;
  int R;
};

enum TmapDtype : int { kTmF16 = 0, kTmF32 = 1 };

// Encode a tensor map of rank 1..5: dims and strides in elements (strides of dims 1..rank-1),
// box in elements, swizzle 0 / 32 / 64 / 128 bytes.
bool make_tmap(CUtensorMap *map, const void *base, int dtype, int rank, const unsigned long long *dims,
               const unsigned long long *strides_el, const unsigned *box, int swizzle_bytes);

// Encode a 3D fp16 tensor map with a 128-byte swizzle and a (64, box1, box2) box.
// dims/strides in elements; strides[0] is the stride of dim 1, strides[1] of dim 2.
bool make_tmap_f16(CUtensorMap *map, const void *base, unsigned long long d0, unsigned long long d1,
                   unsigned long long d2, unsigned long long s1, unsigned long long s2, unsigned box1,
                   unsigned box2);

// Resolve the tensor-map encoder and set the kernels' shared-memory limits (call once, outside capture).
bool gemm_tc_init();

// tmC / tmD: output tensor maps of the epilogues that store through bulk tensor stores
// (kTcQkv: [q | k | v | gates] fp16 [M, ld] box 32x32 swizzle 64; kTcResid: tmD = Xh fp16 [M, ld] box 32x32
//  swizzle 64; kTcBandSplit: tmD = the same as 3D (ld, nb, frames) boxes 32x1x32; kTcGelu: out fp16 [M, ldo]
//  box 32x32 swizzle 64; kTcTanh: out fp16 (ldo, frames, groups) box 32x32x1 swizzle 64;
//  kTcGlu: none (atomic adds into the masks); kTcGeglu: out fp16 [M, ldo] box 16x32,
//  no swizzle).  Unused maps may be any valid map.
// bf16: A, W and every 16-bit output in bf16 (MRF_BF16), the residual kinds also keeping the fp32
// master copy X (tmC: X fp32 box 32x32 swizzle 128, or the 3-D (ld, nb, frames) 32x1x32 box of the
// band split); otherwise fp16.  pair (for the kinds gemm_tc_pair_kind accepts): clusters of two
// CTAs, each cluster an M = 256 tile (p.m_tiles counted in 256-row tiles), grid even, and tmB's box
// BN / 2 rows; otherwise one CTA per M = 128 tile with tmB's box BN rows.
void launch_gemm_tc(int epi, bool bf16, bool pair, const CUtensorMap &tmA, const CUtensorMap &tmB,
                    const CUtensorMap &tmC, const CUtensorMap &tmD, const GemmParams &p, int grid, bool pdl,
                    cudaStream_t st);
bool gemm_tc_pair_kind(int epi);

// Fused feed-forward (k_ff_tc.cu): x <- x + W2 gelu(rs W1 x + b1) + b2 on the fp16 residual stream,
// rs the row scale of the ss_in partial slots; the new rows' sums of squares (and of out_gain * x)
// into ss_out / ssg_out, four slots a row.  tmX: Xh [M, D] fp16 box 64 x 128 (swizzle 128);
// tmW1: W1 [hidden, D] box 64 x 64; tmW2: W2 [D, hidden] box 64 x (D / 2, or D / 4 when D > 256);
// tmO: Xh box 32 x 32 (swizzle 64).  Runs as CTA pairs.
struct FfParams {
  int M, D, hidden, ld, ss_in_parts, ss_out_parts;
  unsigned *status;
  const float *ss_in;
  const float *b1, *b2, *out_gain;
  __half *Xh;
  float *ss_out, *ssg_out;
};
bool ff_tc_supported(int D, int hidden);
bool ff_tc_init();
void launch_ff_tc(const CUtensorMap &tmX, const CUtensorMap &tmW1, const CUtensorMap &tmW2, const CUtensorMap &tmO,
                  const FfParams &p, int sms, bool pdl, cudaStream_t st);

}  // namespace mrf
