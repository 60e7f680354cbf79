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
// CTA layout (320 threads, one CTA per SM):
//   warps 0-7  epilogue: tcgen05.ld of the 128 x BN accumulator, fused epilogue, stores
//              (two warps per TMEM lane quarter, alternating 32-column chunks)
//   warp 8     TMA producer (one lane) and TMEM allocator
//   warp 9     MMA issuer (one lane): 4 x tcgen05.mma (M=128, N<=256, K=16) per 64-wide K block
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

constexpr int kEpiWarps = 8;

struct SmemLayout {
  static constexpr int a_off = 0;
  static constexpr int b_off = kGemmStages * A_STAGE;
  static constexpr int stg_off = b_off + kGemmStages * B_STAGE;
  static constexpr int bar_off = stg_off + kEpiWarps * 32 * 80;
  static constexpr int total = bar_off + 256;
};

__device__ __forceinline__ float sigmoidf_(float x) { return 1.f / (1.f + __expf(-x)); }

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
// Epilogue warp w owns TMEM lane quarter w % 4 (rows 32 (w % 4) .. +31 of the tile) and
// the 32-column chunks c = w / 4, w / 4 + 2, ... of the tile.  Global stores and the
// residual loads go through a per-warp staging buffer so that every warp instruction
// moves whole 64-byte row segments (4 lanes per row, 8 rows per instruction).

constexpr int kStageRow = 80;                   // 64 data bytes + 16 pad (conflict-free)
constexpr int kStageWarp = 32 * kStageRow;

__device__ __forceinline__ float row_scale(const GemmParams &p, long long row) {
  if (!p.ss_in) return 1.f;
  return 1.f / fmaxf(sqrtf(p.ss_in[row]), kEps);
}

// erf by Abramowitz & Stegun 7.1.26 (|error| <= 1.5e-7), branch-free:
// erf(z) = 1 - t (a1 + t (a2 + t (a3 + t (a4 + t a5)))) exp(-z^2), t = 1 / (1 + p z), z >= 0.
__device__ __forceinline__ float erf_as(float x) {
  const float z = fabsf(x);
  float t;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(t) : "f"(fmaf(0.3275911f, z, 1.f)));
  float poly = fmaf(t, 1.061405429f, -1.453152027f);
  poly = fmaf(t, poly, 1.421413741f);
  poly = fmaf(t, poly, -0.284496736f);
  poly = fmaf(t, poly, 0.254829592f);
  poly *= t;
  float e;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(e) : "f"(-z * z * 1.4426950408889634f));
  return copysignf(fmaf(-poly, e, 1.f), x);
}

__device__ __forceinline__ float gelu_(float x) { return 0.5f * x * (1.f + erf_as(x * 0.70710678118654752f)); }

// Each lane passes its row's destination (null: skip) and 64 bytes; written coalesced.
__device__ __forceinline__ void warp_store64(uint8_t *stg, int lane, uint8_t *dst, const uint4 (&d)[4]) {
  uint8_t *my = stg + lane * kStageRow;
#pragma unroll
  for (int q = 0; q < 4; ++q) *reinterpret_cast<uint4 *>(my + q * 16) = d[q];
  __syncwarp();
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int r = i * 8 + (lane >> 2), q = lane & 3;
    uint8_t *rd = reinterpret_cast<uint8_t *>(
        __shfl_sync(0xffffffffu, reinterpret_cast<unsigned long long>(dst), r));
    const uint4 v = *reinterpret_cast<const uint4 *>(stg + r * kStageRow + q * 16);
    if (rd) *reinterpret_cast<uint4 *>(rd + q * 16) = v;
  }
  __syncwarp();
}

// Coalesced 64-byte-per-row load, phase A: issue the global loads (lane holds pieces of rows
// i*8 + lane/4).  Phase B: redistribute through staging so each lane gets its own row.
__device__ __forceinline__ void warp_load64_issue(int lane, const uint8_t *src, uint4 (&pc)[4]) {
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int r = i * 8 + (lane >> 2), q = lane & 3;
    const uint8_t *rs = reinterpret_cast<const uint8_t *>(
        __shfl_sync(0xffffffffu, reinterpret_cast<unsigned long long>(src), r));
    pc[i] = rs ? *reinterpret_cast<const uint4 *>(rs + q * 16) : make_uint4(0, 0, 0, 0);
  }
}

__device__ __forceinline__ void warp_load64_finish(uint8_t *stg, int lane, const uint4 (&pc)[4], uint4 (&d)[4]) {
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int r = i * 8 + (lane >> 2), q = lane & 3;
    *reinterpret_cast<uint4 *>(stg + r * kStageRow + q * 16) = pc[i];
  }
  __syncwarp();
#pragma unroll
  for (int q = 0; q < 4; ++q) d[q] = *reinterpret_cast<const uint4 *>(stg + lane * kStageRow + q * 16);
  __syncwarp();
}

__device__ __forceinline__ void pack16(const float *v, uint4 (&d)[4]) {
  // 32 floats -> 32 fp16 (64 bytes)
#pragma unroll
  for (int q = 0; q < 4; ++q)
    d[q] = make_uint4(pack_h2(v[8 * q], v[8 * q + 1]), pack_h2(v[8 * q + 2], v[8 * q + 3]),
                      pack_h2(v[8 * q + 4], v[8 * q + 5]), pack_h2(v[8 * q + 6], v[8 * q + 7]));
}

__device__ __forceinline__ void as_u4(const float *v, uint4 (&d)[4]) {
  // 16 floats (64 bytes)
#pragma unroll
  for (int q = 0; q < 4; ++q)
    d[q] = make_uint4(__float_as_uint(v[4 * q]), __float_as_uint(v[4 * q + 1]), __float_as_uint(v[4 * q + 2]),
                      __float_as_uint(v[4 * q + 3]));
}

__device__ __forceinline__ void from_u4(const uint4 (&d)[4], float *v) {
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    v[4 * q] = __uint_as_float(d[q].x);
    v[4 * q + 1] = __uint_as_float(d[q].y);
    v[4 * q + 2] = __uint_as_float(d[q].z);
    v[4 * q + 3] = __uint_as_float(d[q].w);
  }
}

// Token of row m of group g: band-major rows (a_mode 1) are frame m of band g.
__device__ __forceinline__ long long token_of(const GemmParams &p, int m, int g) {
  return p.a_mode == 1 ? (long long)m * p.nb + g : (long long)m;
}

struct QkvRow {
  long long tok, seq;
  int pos;
};

__device__ __forceinline__ QkvRow qkv_row(const GemmParams &p, int m, int g) {
  QkvRow r;
  r.tok = token_of(p, m, g);
  const int band = (int)(r.tok % p.nb);
  const long long bt = r.tok / p.nb;
  if (p.axis == 0) {
    const int b = (int)(bt / p.T);
    r.pos = (int)(bt % p.T);
    r.seq = (long long)b * p.nb + band;
  } else {
    r.seq = bt;
    r.pos = band;
  }
  return r;
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
    for (int s = 0; s < 2; ++s) { tc::mbar_init(tfull + s, 1); tc::mbar_init(tempty + s, kEpiWarps); }
    tc::mbar_init(done, 1);
    tc::fence_barrier_init();
  }
  if (warp == kEpiWarps) {
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

  if (warp == kEpiWarps) {
    // ---------------- TMA producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      const uint32_t bytes = A_STAGE + p.BN * BK * 2;
      for (int tile = blockIdx.x; tile < total; tile += gridDim.x) {
        const TileInfo ti = decode_tile(p, tile);
        const GemmGroup &gr = p.groups[ti.g];
        const int m0 = ti.mb * BM, n0 = gr.b_row_off + ti.nblk * p.BN;
        const int kblocks = gr.kblocks ? gr.kblocks : p.K / BK;
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
  } else if (warp == kEpiWarps + 1) {
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
        const int kblocks = gr.kblocks ? gr.kblocks : p.K / BK;
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
      tc::mma_commit(done);
      tc::mbar_wait(done, 0, p.status, 13, abort);
    }
  } else {
    // ---------------- epilogue warps 0-7
    const int quarter = warp & 3, half = warp >> 2;
    uint8_t *stg = smem + SmemLayout::stg_off + warp * kStageWarp;
    int local = 0;
    for (int tile = blockIdx.x; tile < total; tile += gridDim.x, ++local) {
      const TileInfo ti = decode_tile(p, tile);
      const GemmGroup &gr = p.groups[ti.g];
      const int acc = local & 1;
      const uint32_t aphase = (local >> 1) & 1;
      const int row = quarter * 32 + lane;
      const int m = ti.mb * BM + row;
      const bool valid = m < p.M;
      const int nbase = ti.nblk * p.BN;
      const int n_eff = min(p.BN, gr.N - nbase);
      const int nchunks = (n_eff + 31) >> 5;
      const uint32_t tbase = tmem_base + ((uint32_t)(quarter * 32) << 16) + acc * 256;
      // ---- work that does not need the accumulator, before waiting for it
      float rs = 1.f;
      QkvRow qr{0, 0, 0};
      float2 cs[16];
      if (EPI == kTcQkv) {
        qr = qkv_row(p, valid ? m : 0, ti.g);
        if (valid) rs = row_scale(p, qr.tok);
        if (p.dh == 64) {
          const float2 *rp = p.rope + (long long)qr.pos * 32 + half * 16;
#pragma unroll
          for (int i = 0; i < 16; ++i) cs[i] = rp[i];
        }
      } else if (EPI == kTcGelu) {
        if (valid) rs = row_scale(p, m);
      }
      uint4 pre[8];
      int c = half;
      if (EPI == kTcResid && c < nchunks) {
        const float *xr = p.X + (long long)m * p.ld + nbase + 32 * c;
        warp_load64_issue(lane, valid ? reinterpret_cast<const uint8_t *>(xr) : nullptr,
                          *reinterpret_cast<uint4(*)[4]>(&pre[0]));
        warp_load64_issue(lane, valid ? reinterpret_cast<const uint8_t *>(xr + 16) : nullptr,
                          *reinterpret_cast<uint4(*)[4]>(&pre[4]));
      }
      if (!tc::mbar_wait(tfull + acc, aphase, p.status, 14, abort)) break;
      tc::tc_fence_after();
      float sq = 0.f;
      for (; c < nchunks; c += 2) {
        const int c0 = nbase + 32 * c;
        const bool full_chunk = c0 + 32 <= gr.N;
        float v[32];
        if (EPI == kTcBandSplit) {
          tc::tmem_ld32(tbase + 32 * c, v);
          const long long tok = (long long)m * p.nb + ti.g;
          const float *bias = p.bias + gr.bias_off + c0;
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            v[j] += bias[j];
            sq += v[j] * v[j];
          }
          float *xr = p.X + tok * p.ld + c0;
          __half *hr = p.Xh + tok * p.ld + c0;
          uint4 d[4];
          as_u4(v, d);
          warp_store64(stg, lane, valid ? reinterpret_cast<uint8_t *>(xr) : nullptr, d);
          as_u4(v + 16, d);
          warp_store64(stg, lane, valid ? reinterpret_cast<uint8_t *>(xr + 16) : nullptr, d);
          pack16(v, d);
          warp_store64(stg, lane, valid ? reinterpret_cast<uint8_t *>(hr) : nullptr, d);
          continue;
        }
        if (EPI == kTcResid) {
          // residual of this chunk (prefetched), then prefetch the next one
          uint4 r0[4], r1[4];
          warp_load64_finish(stg, lane, *reinterpret_cast<uint4(*)[4]>(&pre[0]), r0);
          warp_load64_finish(stg, lane, *reinterpret_cast<uint4(*)[4]>(&pre[4]), r1);
          if (c + 2 < nchunks) {
            const float *xr = p.X + (long long)m * p.ld + c0 + 64;
            warp_load64_issue(lane, valid ? reinterpret_cast<const uint8_t *>(xr) : nullptr,
                              *reinterpret_cast<uint4(*)[4]>(&pre[0]));
            warp_load64_issue(lane, valid ? reinterpret_cast<const uint8_t *>(xr + 16) : nullptr,
                              *reinterpret_cast<uint4(*)[4]>(&pre[4]));
          }
          float x[32];
          from_u4(r0, x);
          from_u4(r1, x + 16);
          tc::tmem_ld32(tbase + 32 * c, v);
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            x[j] += v[j] + (p.bias ? p.bias[c0 + j] : 0.f);
            sq += x[j] * x[j];
          }
          float *xr = p.X + (long long)m * p.ld + c0;
          __half *hr = p.Xh + (long long)m * p.ld + c0;
          uint4 d[4];
          as_u4(x, d);
          warp_store64(stg, lane, valid ? reinterpret_cast<uint8_t *>(xr) : nullptr, d);
          as_u4(x + 16, d);
          warp_store64(stg, lane, valid ? reinterpret_cast<uint8_t *>(xr + 16) : nullptr, d);
          pack16(x, d);
          warp_store64(stg, lane, valid ? reinterpret_cast<uint8_t *>(hr) : nullptr, d);
          continue;
        }
        tc::tmem_ld32(tbase + 32 * c, v);
        if (EPI == kTcQkv) {
          const int A3 = 3 * p.A;
          if (c0 >= A3) {  // sigmoid gates
            if (valid)
              for (int j = 0; j < 32; ++j) {
                const int h = c0 + j - A3;
                if (h < p.H) p.gates[qr.tok * p.H + h] = sigmoidf_(v[j] * rs + p.gbias[h]);
              }
            continue;
          }
#pragma unroll
          for (int j = 0; j < 32; ++j) v[j] *= rs;
          if (p.dh == 64) {
            const int which = c0 / p.A;
            const int head = (c0 - which * p.A) >> 6;
            const int d0 = c0 & 63;
            if (which < 2) {
              const float sc = which == 0 ? p.q_scale : 1.f;
#pragma unroll
              for (int i = 0; i < 16; ++i) {
                const float x0 = v[2 * i], x1 = v[2 * i + 1];
                v[2 * i] = (x0 * cs[i].x - x1 * cs[i].y) * sc;
                v[2 * i + 1] = (x1 * cs[i].x + x0 * cs[i].y) * sc;
              }
            }
            __half *dst = which == 0 ? p.q : which == 1 ? p.k : p.v;
            uint4 d[4];
            pack16(v, d);
            warp_store64(stg, lane,
                         valid ? reinterpret_cast<uint8_t *>(dst + ((qr.seq * p.H + head) * p.n_pad + qr.pos) * 64 + d0)
                               : nullptr,
                         d);
          } else if (valid) {
            const int half_dh = p.dh >> 1;
#pragma unroll
            for (int j8 = 0; j8 < 32; j8 += 8) {
              const int col = c0 + j8;
              const int which = col / p.A;
              const int rem = col - which * p.A;
              const int head = rem / p.dh;
              const int dd = rem - head * p.dh;
              float o[8];
#pragma unroll
              for (int j = 0; j < 8; ++j) o[j] = v[j8 + j];
              if (which < 2) {
                const float sc = which == 0 ? p.q_scale : 1.f;
#pragma unroll
                for (int j = 0; j < 8; j += 2) {
                  const float2 cc = p.rope[(long long)qr.pos * half_dh + ((dd + j) >> 1)];
                  const float x0 = o[j], x1 = o[j + 1];
                  o[j] = (x0 * cc.x - x1 * cc.y) * sc;
                  o[j + 1] = (x1 * cc.x + x0 * cc.y) * sc;
                }
              }
              __half *dst = which == 0 ? p.q : which == 1 ? p.k : p.v;
              st_h8(dst + ((qr.seq * p.H + head) * p.n_pad + qr.pos) * p.dh + dd, o);
            }
          }
        } else if (EPI == kTcGelu || EPI == kTcTanh) {
          const float *bias = p.bias + gr.bias_off + c0;
          __half *dst = p.out_h + gr.out_off * p.out_group_stride + (long long)m * p.ldo + c0;
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const float y = v[j] * rs + (c0 + j < gr.N ? bias[j] : 0.f);
            v[j] = EPI == kTcGelu ? gelu_(y) : tanhf(y);
          }
          if (full_chunk) {
            uint4 d[4];
            pack16(v, d);
            warp_store64(stg, lane, valid ? reinterpret_cast<uint8_t *>(dst) : nullptr, d);
          } else if (valid) {
            for (int j = 0; j < 32 && c0 + j < gr.N; ++j) dst[j] = __float2half_rn(v[j]);
          }
        } else {  // kTcGlu
          const float *bias = p.bias + gr.bias_off + c0;
          float *dst = p.out_f + (long long)m * p.ldo + gr.out_off + (c0 >> 1);
          float o[16];
#pragma unroll
          for (int j = 0; j < 32; j += 2) {
            const bool ok = c0 + j + 1 < gr.N;
            const float val = v[j] + (ok ? bias[j] : 0.f);
            const float gt = v[j + 1] + (ok ? bias[j + 1] : 0.f);
            o[j >> 1] = val * sigmoidf_(gt);
          }
          if (full_chunk) {
            uint4 d[4];
            as_u4(o, d);
            warp_store64(stg, lane, valid ? reinterpret_cast<uint8_t *>(dst) : nullptr, d);
          } else if (valid) {
            for (int j = 0; 2 * j + 1 < gr.N - c0; ++j) dst[j] = o[j];
          }
        }
      }
      if (EPI == kTcResid && valid && p.ss_out && half < nchunks) atomicAdd(p.ss_out + m, sq);
      if (EPI == kTcBandSplit && valid && half < nchunks) atomicAdd(p.ss_out + (long long)m * p.nb + ti.g, sq);
      tc::tc_fence_before();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(tempty + acc);
    }
  }
  tc::tc_fence_before();
  __syncthreads();
  if (warp == kEpiWarps) {
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
  ok = ok && cudaFuncSetAttribute(gemm_tc_kernel<kTcBandSplit>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) == cudaSuccess;
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
    MRF_GEMM_CASE(kTcBandSplit)
#undef MRF_GEMM_CASE
    default: break;
  }
}

}  // namespace mrf
