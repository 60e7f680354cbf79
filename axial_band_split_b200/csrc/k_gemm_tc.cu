// Persistent tcgen05 GEMM with fused epilogues, for every dense contraction of the
// trunk and of the mask head: C = A W^T, A [M, K] and W [N, K] fp16, both K-major,
// accumulated in fp32 in tensor memory.
//
// The layers it serves are those of "Mel-Band RoFormer — architecture, inference hot path &
// RTX 3050 feasibility", section "The two transformers are not the same shape" (to_qkv,
// to_gates, to_out, feed-forward) and section "Parameter accounting" (the per-band mask
// MLP: Linear-Tanh-Linear-Tanh-Linear-GLU); the fusions restate the exact rewrites of
// "@audio/neural-separate 0.4.0 → 0.5.0", package/scripts/export-roformer.py, class Core
// (norm scale folded into the next weight, gates joined to q/k/v, bands batched).
//
// CTA layout (192 threads, one CTA per SM):
//   warps 0-3  epilogue: tcgen05.ld of the 128 x BN accumulator, fused epilogue, stores
//   warp 4     TMA producer (one lane) and TMEM allocator
//   warp 5     MMA issuer (one lane): 4 x tcgen05.mma (M=128, N<=256, K=16) per 64-wide K block
// Shared memory: kGemmStages stages of A (128 x 64) and B (256 x 64) tiles, 128-byte swizzle.
// Tensor memory: two 256-column fp32 accumulators, so the epilogue of tile i overlaps the
// main loop of tile i+1.
#include <cudaTypedefs.h>

#include <cmath>
#include <cstdio>

#include "gemm_tc.cuh"
#include "mrf_internal.h"
#include "tc_ptx.cuh"

namespace mrf {

namespace {

constexpr int BM = 128, BK = 64, BN_MAX = 256;
constexpr int A_STAGE = BM * BK * 2;        // 16 KB
constexpr int B_STAGE = BN_MAX * BK * 2;    // 32 KB
constexpr int TMEM_COLS = 512;
constexpr float kEps = 1e-12f;

struct SmemLayout {
  static constexpr int a_off = 0;
  static constexpr int b_off = kGemmStages * A_STAGE;
  static constexpr int bar_off = b_off + kGemmStages * B_STAGE;
  static constexpr int total = bar_off + 256;
};

__device__ __forceinline__ float sigmoidf_(float x) { return 1.f / (1.f + __expf(-x)); }
__device__ __forceinline__ float gelu_(float x) { return 0.5f * x * (1.f + erff(x * 0.70710678118654752f)); }

__device__ __forceinline__ uint32_t pack_h2(float a, float b) {
  __half2 h = __floats2half2_rn(a, b);
  return *reinterpret_cast<uint32_t *>(&h);
}

// Store 8 consecutive floats as fp16 (16 bytes).
__device__ __forceinline__ void st_h8(__half *dst, const float *v) {
  uint4 u;
  u.x = pack_h2(v[0], v[1]);
  u.y = pack_h2(v[2], v[3]);
  u.z = pack_h2(v[4], v[5]);
  u.w = pack_h2(v[6], v[7]);
  *reinterpret_cast<uint4 *>(dst) = u;
}

__device__ __forceinline__ int find_group(const GemmGroup *g, int n, int tile, int m_tiles) {
  int lo = 0, hi = n - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (g[mid].n_tile_start * m_tiles <= tile) lo = mid;
    else hi = mid - 1;
  }
  return lo;
}

struct TileInfo {
  int g, mb, nblk;
};

__device__ __forceinline__ TileInfo decode_tile(const GemmParams &p, int tile) {
  TileInfo ti;
  ti.g = p.ngroups == 1 ? 0 : find_group(p.groups, p.ngroups, tile, p.m_tiles);
  const GemmGroup &gr = p.groups[ti.g];
  const int r = tile - gr.n_tile_start * p.m_tiles;
  ti.mb = r / gr.n_tiles;
  ti.nblk = r % gr.n_tiles;
  return ti;
}

// ------------------------------------------------------------------ epilogues
// Each epilogue thread owns one row m of the tile and handles 32 consecutive columns
// [c0, c0 + 32) of the group's N per call.

__device__ __forceinline__ float row_scale(const GemmParams &p, long long row) {
  if (!p.ss_in) return 1.f;
  return 1.f / fmaxf(sqrtf(p.ss_in[row]), kEps);
}

// q, k, v scatter with RoPE (interleaved pairs) and sigmoid gates.
__device__ __forceinline__ void epi_qkv(const GemmParams &p, int m, int c0, float (&v)[32], float rs) {
  const long long tok = m;
  const int band = (int)(tok % p.nb);
  const long long bt = tok / p.nb;
  const int b = (int)(bt / p.T), t = (int)(bt % p.T);
  long long seq;
  int pos;
  if (p.axis == 0) { seq = (long long)b * p.nb + band; pos = t; }
  else { seq = bt; pos = band; }
  const int A3 = 3 * p.A;
  if (c0 >= A3) {  // gates
    for (int j = 0; j < 32; ++j) {
      const int h = c0 + j - A3;
      if (h < p.H) p.gates[tok * p.H + h] = sigmoidf_(v[j] * rs + p.gbias[h]);
    }
    return;
  }
  const int half = p.dh >> 1;
#pragma unroll
  for (int j8 = 0; j8 < 32; j8 += 8) {
    const int col = c0 + j8;
    const int which = col / p.A;
    const int rem = col - which * p.A;
    const int head = rem / p.dh;
    const int d = rem - head * p.dh;
    float o[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) o[j] = v[j8 + j] * rs;
    if (which < 2) {
#pragma unroll
      for (int j = 0; j < 8; j += 2) {
        const float2 cs = p.rope[(long long)pos * half + ((d + j) >> 1)];
        const float x0 = o[j], x1 = o[j + 1];
        o[j] = x0 * cs.x - x1 * cs.y;
        o[j + 1] = x1 * cs.x + x0 * cs.y;
      }
    }
    __half *dst = which == 0 ? p.q : which == 1 ? p.k : p.v;
    st_h8(dst + ((seq * p.H + head) * p.n_pad + pos) * p.dh + d, o);
  }
}

__device__ __forceinline__ float epi_resid(const GemmParams &p, int m, int c0, float (&v)[32], int N) {
  float *x = p.X + (long long)m * p.ld + c0;
  __half *xh = p.Xh + (long long)m * p.ld + c0;
  float sq = 0.f;
  if (c0 + 32 <= N) {
#pragma unroll
    for (int j = 0; j < 32; j += 4) {
      float4 r = *reinterpret_cast<const float4 *>(x + j);
      r.x += v[j] + (p.bias ? p.bias[c0 + j] : 0.f);
      r.y += v[j + 1] + (p.bias ? p.bias[c0 + j + 1] : 0.f);
      r.z += v[j + 2] + (p.bias ? p.bias[c0 + j + 2] : 0.f);
      r.w += v[j + 3] + (p.bias ? p.bias[c0 + j + 3] : 0.f);
      *reinterpret_cast<float4 *>(x + j) = r;
      v[j] = r.x; v[j + 1] = r.y; v[j + 2] = r.z; v[j + 3] = r.w;
      sq += r.x * r.x + r.y * r.y + r.z * r.z + r.w * r.w;
    }
#pragma unroll
    for (int j = 0; j < 32; j += 8) st_h8(xh + j, v + j);
  } else {
    for (int j = 0; j < 32 && c0 + j < N; ++j) {
      const float r = x[j] + v[j] + (p.bias ? p.bias[c0 + j] : 0.f);
      x[j] = r;
      xh[j] = __float2half_rn(r);
      sq += r * r;
    }
  }
  return sq;
}

__device__ __forceinline__ void epi_act(const GemmParams &p, int kind, int m, int c0, float (&v)[32], float rs,
                                        int N, const GemmGroup &gr) {
  __half *dst = p.out_h + gr.out_off * p.out_group_stride + (long long)m * p.ldo + c0;
  const float *bias = p.bias + gr.bias_off + c0;
  float o[32];
#pragma unroll
  for (int j = 0; j < 32; ++j) {
    const float y = v[j] * rs + (c0 + j < N ? bias[j] : 0.f);
    o[j] = kind == kTcGelu ? gelu_(y) : tanhf(y);
  }
  if (c0 + 32 <= N) {
#pragma unroll
    for (int j = 0; j < 32; j += 8) st_h8(dst + j, o + j);
  } else {
    for (int j = 0; j < 32 && c0 + j < N; ++j) dst[j] = __float2half_rn(o[j]);
  }
}

__device__ __forceinline__ void epi_glu(const GemmParams &p, int m, int c0, float (&v)[32], int N,
                                        const GemmGroup &gr) {
  float *dst = p.out_f + (long long)m * p.ldo + gr.out_off + (c0 >> 1);
  const float *bias = p.bias + gr.bias_off + c0;
  float o[16];
#pragma unroll
  for (int j = 0; j < 32; j += 2) {
    const bool ok = c0 + j + 1 < N;
    const float val = v[j] + (ok ? bias[j] : 0.f);
    const float gt = v[j + 1] + (ok ? bias[j + 1] : 0.f);
    o[j >> 1] = val * sigmoidf_(gt);
  }
  if (c0 + 32 <= N) {
#pragma unroll
    for (int j = 0; j < 16; ++j) dst[j] = o[j];
  } else {
    for (int j = 0; 2 * j + 1 < N - c0; ++j) dst[j] = o[j];
  }
}

// ------------------------------------------------------------------ the kernel
template <int EPI>
__global__ void __launch_bounds__(kGemmThreads, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                   const GemmParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *sA = smem + SmemLayout::a_off;
  uint8_t *sB = smem + SmemLayout::b_off;
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + SmemLayout::bar_off);
  uint64_t *full = bars;                       // [stages]
  uint64_t *empty = bars + kGemmStages;        // [stages]
  uint64_t *tfull = bars + 2 * kGemmStages;    // [2]
  uint64_t *tempty = tfull + 2;                // [2]
  uint64_t *done = tempty + 2;                 // [1]
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(done + 1);
  __shared__ int abort_flag;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    abort_flag = 0;
    for (int s = 0; s < kGemmStages; ++s) { tc::mbar_init(full + s, 1); tc::mbar_init(empty + s, 1); }
    for (int s = 0; s < 2; ++s) { tc::mbar_init(tfull + s, 1); tc::mbar_init(tempty + s, 4); }
    tc::mbar_init(done, 1);
    tc::fence_barrier_init();
  }
  if (warp == 4) {
    if (lane == 0) { tc::tma_prefetch(&tmA); tc::tma_prefetch(&tmB); }
    __syncwarp();
    tc::tmem_alloc(tmem_slot, TMEM_COLS);
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  volatile int *abort = &abort_flag;
  const int total = p.m_tiles * p.total_n_tiles;
  const int kblocks = p.K / BK;

  if (warp == 4) {
    // ---------------- TMA producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      const uint32_t bytes = A_STAGE + p.BN * BK * 2;
      for (int tile = blockIdx.x; tile < total; tile += gridDim.x) {
        const TileInfo ti = decode_tile(p, tile);
        const GemmGroup &gr = p.groups[ti.g];
        const int m0 = ti.mb * BM, n0 = gr.b_row_off + ti.nblk * p.BN;
        bool ok = true;
        for (int kb = 0; kb < kblocks; ++kb) {
          if (!tc::mbar_wait(empty + stage, phase ^ 1, p.status, 10, abort)) { ok = false; break; }
          tc::mbar_arrive_expect_tx(full + stage, bytes);
          if (p.a_mode == 0) tc::tma_load_3d(sA + stage * A_STAGE, &tmA, full + stage, kb * BK, gr.a_off + m0, 0);
          else tc::tma_load_3d(sA + stage * A_STAGE, &tmA, full + stage, kb * BK, gr.a_off, m0);
          tc::tma_load_3d(sB + stage * B_STAGE, &tmB, full + stage, kb * BK, n0, 0);
          if (++stage == kGemmStages) { stage = 0; phase ^= 1; }
        }
        if (!ok) break;
      }
    }
  } else if (warp == 5) {
    // ---------------- MMA issuer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int local = 0;
      for (int tile = blockIdx.x; tile < total; tile += gridDim.x, ++local) {
        const TileInfo ti = decode_tile(p, tile);
        const GemmGroup &gr = p.groups[ti.g];
        const int acc = local & 1;
        const uint32_t aphase = (local >> 1) & 1;
        int n_eff = min(p.BN, gr.N - ti.nblk * p.BN);
        n_eff = (n_eff + 15) & ~15;
        const uint32_t idesc = tc::idesc_f16(BM, n_eff);
        const uint32_t d_tmem = tmem_base + acc * 256;
        if (!tc::mbar_wait(tempty + acc, aphase ^ 1, p.status, 11, abort)) break;
        tc::tc_fence_after();
        bool ok = true;
        for (int kb = 0; kb < kblocks; ++kb) {
          if (!tc::mbar_wait(full + stage, phase, p.status, 12, abort)) { ok = false; break; }
          tc::tc_fence_after();
          const uint32_t a_addr = tc::smem_u32(sA + stage * A_STAGE);
          const uint32_t b_addr = tc::smem_u32(sB + stage * B_STAGE);
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            tc::mma_f16(d_tmem, tc::sw128_kmajor_desc(a_addr + kk * 32), tc::sw128_kmajor_desc(b_addr + kk * 32),
                        idesc, (kb | kk) != 0);
          }
          tc::mma_commit(empty + stage);
          if (++stage == kGemmStages) { stage = 0; phase ^= 1; }
        }
        if (!ok) break;
        tc::mma_commit(tfull + acc);
      }
      // all MMAs complete before tensor memory is released
      tc::mma_commit(done);
      tc::mbar_wait(done, 0, p.status, 13, abort);
    }
  } else {
    // ---------------- epilogue warps 0-3: TMEM lanes 32*warp .. 32*warp+31
    int local = 0;
    for (int tile = blockIdx.x; tile < total; tile += gridDim.x, ++local) {
      const TileInfo ti = decode_tile(p, tile);
      const GemmGroup &gr = p.groups[ti.g];
      const int acc = local & 1;
      const uint32_t aphase = (local >> 1) & 1;
      if (!tc::mbar_wait(tfull + acc, aphase, p.status, 14, abort)) break;
      tc::tc_fence_after();
      const int row = warp * 32 + lane;
      const int m = ti.mb * BM + row;
      const bool valid = m < p.M;
      const int nbase = ti.nblk * p.BN;
      const int n_eff = min(p.BN, gr.N - nbase);
      float rs = 1.f;
      if (valid && (EPI == kTcQkv || EPI == kTcGelu)) rs = row_scale(p, m);
      float sq = 0.f;
      for (int c = 0; c < n_eff; c += 32) {
        float v[32];
        tc::tmem_ld32(tmem_base + ((uint32_t)(warp * 32) << 16) + acc * 256 + c, v);
        if (!valid) continue;
        const int c0 = nbase + c;
        if (EPI == kTcQkv) epi_qkv(p, m, c0, v, rs);
        else if (EPI == kTcResid) sq += epi_resid(p, m, c0, v, gr.N);
        else if (EPI == kTcGelu || EPI == kTcTanh) epi_act(p, EPI, m, c0, v, rs, gr.N, gr);
        else epi_glu(p, m, c0, v, gr.N, gr);
      }
      if (EPI == kTcResid && valid && p.ss_out) atomicAdd(p.ss_out + m, sq);
      tc::tc_fence_before();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(tempty + acc);
    }
  }
  tc::tc_fence_before();
  __syncthreads();
  if (warp == 4) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    cudaDriverEntryPointQueryResult q;
    void *ptr = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  }
  return fn;
}

}  // namespace

size_t gemm_smem_bytes() { return SmemLayout::total + 1024; }

bool make_tmap_f16(CUtensorMap *map, const void *base, unsigned long long d0, unsigned long long d1,
                   unsigned long long d2, unsigned long long s1, unsigned long long s2, unsigned box1,
                   unsigned box2) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {d0, d1, d2};
  cuuint64_t strides[2] = {s1 * 2, s2 * 2};
  cuuint32_t box[3] = {64, box1, box2};
  cuuint32_t es[3] = {1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3, const_cast<void *>(base), dims, strides, box, es,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool gemm_tc_init() {
  const int smem = (int)gemm_smem_bytes();
  bool ok = encode_fn() != nullptr;
  ok = ok && cudaFuncSetAttribute(gemm_tc_kernel<kTcQkv>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) == cudaSuccess;
  ok = ok && cudaFuncSetAttribute(gemm_tc_kernel<kTcResid>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) == cudaSuccess;
  ok = ok && cudaFuncSetAttribute(gemm_tc_kernel<kTcGelu>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) == cudaSuccess;
  ok = ok && cudaFuncSetAttribute(gemm_tc_kernel<kTcTanh>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) == cudaSuccess;
  ok = ok && cudaFuncSetAttribute(gemm_tc_kernel<kTcGlu>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) == cudaSuccess;
  return ok;
}

void launch_gemm_tc(int epi, const CUtensorMap &tmA, const CUtensorMap &tmB, const GemmParams &p, int grid,
                    cudaStream_t st) {
  const size_t smem = gemm_smem_bytes();
  switch (epi) {
#define MRF_GEMM_CASE(E)                                                                         \
  case E:                                                                                        \
    gemm_tc_kernel<E><<<grid, kGemmThreads, smem, st>>>(tmA, tmB, p);                            \
    break;
    MRF_GEMM_CASE(kTcQkv)
    MRF_GEMM_CASE(kTcResid)
    MRF_GEMM_CASE(kTcGelu)
    MRF_GEMM_CASE(kTcTanh)
    MRF_GEMM_CASE(kTcGlu)
#undef MRF_GEMM_CASE
    default: break;
  }
}

}  // namespace mrf
