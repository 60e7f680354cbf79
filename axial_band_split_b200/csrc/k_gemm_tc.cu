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
// CTA layout (one CTA per SM; E = 8 or 16 epilogue warps by epilogue kind):
//   warps 0..E-1  epilogue: tcgen05.ld of the 128 x BN accumulator, fused epilogue, stores
//                 (E / 4 warps per TMEM lane quarter, taking turns over 32-column chunks)
//   warp E        TMA producer (one lane) and TMEM allocator
//   warp E+1      MMA issuer (one lane): 4 x tcgen05.mma (M=128, N<=256, K=16) per 64-wide K block
// Shared memory: gemm_stages(EPI) stages of A (128 x 64) and B (BN x 64) tiles, 128-byte swizzle,
// then per-epilogue-warp output boxes.  Tensor memory: two 256-column fp32 accumulators, so
// the epilogue of tile i overlaps the main loop of tile i+1.
//
// Epilogue stores: each warp writes its 32 rows x 32 columns into a shared-memory box in the
// tensor map's swizzled layout and one lane issues a bulk tensor store (cp.async.bulk.tensor),
// so global writes leave the SM as whole lines; rows past M are clipped by the tensor map.
#include <cudaTypedefs.h>
#include <cuda_bf16.h>

#include <cmath>
#include <cstdio>

#include "gemm_tc.cuh"
#include "tc_math.cuh"
#include "mrf_internal.h"
#include "tc_ptx.cuh"

namespace mrf {

namespace {

constexpr int BM = 128, BK = 64;
constexpr int A_STAGE = BM * BK * 2;        // 16 KB
constexpr int TMEM_COLS = 512;
constexpr float kEps = 1e-12f;
// Epilogue warps per kind: 16 (four per 32-lane quarter of the tile) where the epilogue's
// arithmetic is the bottleneck and fits 96 registers a thread (the register file of an SM
// sub-partition then holds five warps): GELU and the band split; 8 elsewhere, where the
// main loop wants four pipeline stages and the epilogue the 168 registers of a 10-warp
// CTA.  Pipeline stages fill what shared memory the epilogue staging leaves.
__host__ __device__ constexpr int epi_warps(int epi) { return (epi == kTcGelu || epi == kTcBandSplit) ? 16 : 8; }
__host__ __device__ constexpr int gemm_stages(int epi, bool pair = false) {
  return pair ? (epi_warps(epi) == 8 ? 6 : 5) : (epi_warps(epi) == 8 ? 4 : 3);
}
__host__ __device__ constexpr int gemm_threads(int epi) { return 32 * (epi_warps(epi) + 2); }

// Widest B tile of an epilogue kind, and the shared memory each epilogue warp needs.
__host__ __device__ constexpr int bn_max(int epi) { return (epi == kTcResid || epi == kTcBandSplit) ? 192 : 256; }
// Per epilogue warp: two 2 KB boxes; the bf16 schedule's residual kinds keep an fp32 master
// copy of the residual stream and stage a 4 KB fp32 box and a 2 KB bf16 box instead.
__host__ __device__ constexpr int warp_stage_bytes(int epi, bool bf) {
  return (bf && (epi == kTcResid || epi == kTcBandSplit)) ? 4096 + 2048 : 2 * 2048;
}

// The grouped epilogue kinds (one group per band; at most kMaxGroups groups) and the trunk's
// single-group kinds.
constexpr int kMaxGroups = 128;
__host__ __device__ constexpr bool grouped_kind(int epi) {
  return epi == kTcTanh || epi == kTcGlu || epi == kTcBandSplit;
}

// The residual kinds' per-column vectors (bias, the gain of the deferred norm applied to the
// residual, the gain of the output norm), copied to shared memory once per CTA: the epilogue
// streams the residual through L1, which would evict them from it.  Columns up to kMaxDim.
constexpr int kMaxDim = 1024;
__host__ __device__ constexpr int vec_bytes(int epi) { return epi == kTcResid ? 3 * kMaxDim * 4 : 0; }
constexpr int kSmemLimit = 232448;  // 227 KB per CTA

// kPair: a CTA of a pair holds half of the B tile's rows per stage (and has room for more stages).
// Grouped kinds end with the groups' (first tile, column blocks) table, residual kinds with the
// column vectors.  A configuration whose stages would not fit the limit drops one stage.
template <int EPI, bool kBF, bool kPair = false>
struct SmemLayout {
  static constexpr int b_stage = (kPair ? bn_max(EPI) / 2 : bn_max(EPI)) * BK * 2;
  static constexpr int fixed = epi_warps(EPI) * warp_stage_bytes(EPI, kBF) + 256 +
                               (grouped_kind(EPI) ? kMaxGroups * 8 : 0) + vec_bytes(EPI) + 1024;
  static constexpr int stages = gemm_stages(EPI, kPair) * (A_STAGE + b_stage) + fixed <= kSmemLimit
                                    ? gemm_stages(EPI, kPair) : gemm_stages(EPI, kPair) - 1;
  static constexpr int a_off = 0;
  static constexpr int b_off = stages * A_STAGE;
  static constexpr int stg_off = b_off + stages * b_stage;        // 1024-aligned
  static constexpr int bar_off = stg_off + epi_warps(EPI) * warp_stage_bytes(EPI, kBF);
  static constexpr int gtab_off = bar_off + 256;
  static constexpr int vec_off = gtab_off + (grouped_kind(EPI) ? kMaxGroups * 8 : 0);
  static constexpr int total = vec_off + vec_bytes(EPI);
};


// Two floats as one 32-bit pair of the schedule's 16-bit type (fp16, or bf16 with kBF), rounded
// to nearest even.
template <bool kBF>
__device__ __forceinline__ uint32_t pack_h2(float a, float b) {
  if constexpr (kBF) {
    __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t *>(&h);
  } else {
    __half2 h = __floats2half2_rn(a, b);
    return *reinterpret_cast<uint32_t *>(&h);
  }
}

// A tile's group g, its row block mb and column block nblk (tiles run group by group, and
// within a group row block by row block), and the group's record.  Nothing here waits on
// memory: the trunk GEMMs have one group, read into registers once per CTA; the grouped GEMMs
// (mask head, band split: one group per band) search a shared-memory table of the groups'
// (first tile, column blocks) and load the group's record from global memory, a load the
// callers issue one tile before they use it.
struct TileDec {
  int g, mb, nblk;
  GemmGroup gr;
};

template <bool kGrouped>
__device__ __forceinline__ TileDec tile_dec(const GemmParams &p, const GemmGroup &g0, const int2 *gtab, int tile) {
  TileDec d;
  if constexpr (!kGrouped) {
    d.g = 0;
    d.gr = g0;
    d.mb = tile / g0.n_tiles;
    d.nblk = tile - d.mb * g0.n_tiles;
  } else {
    int lo = 0, hi = p.ngroups - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (gtab[mid].x * p.m_tiles <= tile) lo = mid;
      else hi = mid - 1;
    }
    const int2 e = gtab[lo];
    const int r = tile - e.x * p.m_tiles;
    d.g = lo;
    d.mb = r / e.y;
    d.nblk = r - d.mb * e.y;
    d.gr = p.groups[lo];
  }
  return d;
}

// ------------------------------------------------------------------ epilogue helpers



template <bool kBF>
__device__ __forceinline__ void pack16(const float *v, uint4 (&d)[4]) {
  // 32 floats -> 32 16-bit values (64 bytes)
#pragma unroll
  for (int q = 0; q < 4; ++q)
    d[q] = make_uint4(pack_h2<kBF>(v[8 * q], v[8 * q + 1]), pack_h2<kBF>(v[8 * q + 2], v[8 * q + 3]),
                      pack_h2<kBF>(v[8 * q + 4], v[8 * q + 5]), pack_h2<kBF>(v[8 * q + 6], v[8 * q + 7]));
}

// Box rows in shared memory, in the layouts the tensor maps' swizzle modes define:
// 128-byte rows with SWIZZLE_128B (16-byte chunk index ^= row % 8) and 64-byte rows with
// SWIZZLE_64B (chunk index ^= (row / 2) % 4).  Both are conflict-free for row-per-lane access.
__device__ __forceinline__ void box128_put_row(uint8_t *box, int row, const float *v) {
#pragma unroll
  for (int q = 0; q < 8; ++q)
    *reinterpret_cast<float4 *>(box + row * 128 + ((q ^ (row & 7)) << 4)) =
        make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
}

__device__ __forceinline__ void box128_get_row(const uint8_t *box, int row, float *v) {
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    const float4 a = *reinterpret_cast<const float4 *>(box + row * 128 + ((q ^ (row & 7)) << 4));
    v[4 * q] = a.x; v[4 * q + 1] = a.y; v[4 * q + 2] = a.z; v[4 * q + 3] = a.w;
  }
}

__device__ __forceinline__ void box64_put_row(uint8_t *box, int row, const uint4 (&d)[4]) {
#pragma unroll
  for (int q = 0; q < 4; ++q) *reinterpret_cast<uint4 *>(box + row * 64 + ((q ^ ((row >> 1) & 3)) << 4)) = d[q];
}

__device__ __forceinline__ void box64_get_row(const uint8_t *box, int row, float *v) {
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const uint4 a = *reinterpret_cast<const uint4 *>(box + row * 64 + ((q ^ ((row >> 1) & 3)) << 4));
    const uint32_t w[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&w[i]));
      v[8 * q + 2 * i] = f.x;
      v[8 * q + 2 * i + 1] = f.y;
    }
  }
}

// Token of row m of group g: band-major rows (a_mode 1) are frame m of band g.
__device__ __forceinline__ long long token_of(const GemmParams &p, int m, int g) {
  return p.a_mode == 1 ? (long long)m * p.nb + g : (long long)m;
}

struct QkvRow {
  long long tok;
  int pos;
};

// A QKV row's token and its rotary position: the frame within the window (time axis) or
// the band (band axis).  Tokens fit 32 bits (the handle limits B * T * bands).
__device__ __forceinline__ QkvRow qkv_row(const GemmParams &p, int m, int g) {
  QkvRow r;
  r.tok = token_of(p, m, g);
  const unsigned tok = (unsigned)r.tok, bt = tok / (unsigned)p.nb;
  r.pos = p.axis == 0 ? (int)(bt % (unsigned)p.T) : (int)(tok - bt * (unsigned)p.nb);
  return r;
}

__device__ __forceinline__ void load_bias32(const float *b, float *bv) {
  const float4 *b4 = reinterpret_cast<const float4 *>(b);
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const float4 x = b4[j];
    bv[4 * j] = x.x; bv[4 * j + 1] = x.y; bv[4 * j + 2] = x.z; bv[4 * j + 3] = x.w;
  }
}

// A row's sum of squares from its `parts` partial sums (one per (column tile, epilogue warp)
// of the producing GEMM), added in a fixed order so every run gives the same value.  The first
// kPf slots are only loaded here (independent loads whose latency hides under the current tile,
// summed by row_ss_sum when the next tile needs them); slots beyond kPf (more than three column
// tiles of the producer) are added at once.
constexpr int kPf = 8;
struct RowSS {
  float v[kPf];
  float extra;
};
__device__ __forceinline__ void row_ss_fetch(RowSS &r, const float *s, long long row, int parts) {
  const float *q = s + row * parts;
#pragma unroll
  for (int i = 0; i < kPf; ++i) r.v[i] = i < parts ? q[i] : 0.f;
  r.extra = 0.f;
  for (int i = kPf; i < parts; ++i) r.extra += q[i];
}
__device__ __forceinline__ float row_ss_sum(const RowSS &r) {
  float a = 0.f;
#pragma unroll
  for (int i = 0; i < kPf; ++i) a += r.v[i];
  return a + r.extra;
}
__device__ __forceinline__ void row_ss_one(RowSS &r) {
#pragma unroll
  for (int i = 0; i < kPf; ++i) r.v[i] = 0.f;
  r.v[0] = 1.f;
  r.extra = 0.f;
}

// ------------------------------------------------------------------ the kernel
// kPair: the kernel runs as clusters of two CTAs on two SMs, each cluster one M = 256 tile at a
// time (cta_group::2 MMAs issued by the leader, rank 0): CTA r loads rows 128 r .. 128 r + 127 of
// the tile's A and rows n_mma r / 2 .. of its B (n_mma the tile's MMA width), both CTAs' loads
// complete on the leader's full barrier, the leader's commits arrive on both CTAs' empty and tfull
// barriers, and both CTAs' epilogue warps release the accumulator on the leader's tempty barrier.
// Each SM then streams half of every weight tile, halving the shared-memory traffic per MMA flop.
template <int EPI, bool kBF, bool kPair>
__global__ void __launch_bounds__(gemm_threads(EPI), 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                   const __grid_constant__ CUtensorMap tmC, const __grid_constant__ CUtensorMap tmD,
                   const GemmParams p) {
  using L = SmemLayout<EPI, kBF, kPair>;
  constexpr int kEpiWarps = epi_warps(EPI), kSplit = kEpiWarps / 4, kGemmStages = L::stages;
  constexpr int kTileM = kPair ? 2 * BM : BM;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *sA = smem + L::a_off;
  uint8_t *sB = smem + L::b_off;
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + L::bar_off);
  uint64_t *full = bars;                       // [stages]
  uint64_t *empty = bars + kGemmStages;        // [stages]
  uint64_t *tfull = bars + 2 * kGemmStages;    // [2]
  uint64_t *tempty = tfull + 2;                // [2]
  uint64_t *done = tempty + 2;                 // [1]
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(done + 1);
  int2 *gtab = reinterpret_cast<int2 *>(smem + L::gtab_off);
  constexpr bool kGrouped = grouped_kind(EPI);
  __shared__ int abort_flag;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = kPair ? tc::cluster_ctarank() : 0;       // rank within the CTA pair
  const int first_tile = kPair ? (int)(blockIdx.x >> 1) : (int)blockIdx.x;
  const int tile_step = kPair ? (int)(gridDim.x >> 1) : (int)gridDim.x;
  if (threadIdx.x == 0) {
    abort_flag = 0;
    for (int s = 0; s < kGemmStages; ++s) { tc::mbar_init(full + s, 1); tc::mbar_init(empty + s, 1); }
    for (int s = 0; s < 2; ++s) {
      tc::mbar_init(tfull + s, 1);
      tc::mbar_init(tempty + s, kPair ? 2 * kEpiWarps : kEpiWarps);  // pair: both CTAs' epilogue warps
    }
    tc::mbar_init(done, 1);
    tc::fence_barrier_init();
  }
  if (kGrouped)
    for (int i = threadIdx.x; i < p.ngroups; i += blockDim.x)
      gtab[i] = make_int2(p.groups[i].n_tile_start, p.groups[i].n_tiles);
  // [bias | res_gain | out_gain] of a residual GEMM (its N, the model dim, is at most kMaxDim)
  float *svec = reinterpret_cast<float *>(smem + L::vec_off);
  if (EPI == kTcResid)
    for (int i = threadIdx.x; i < min(p.groups[0].N, kMaxDim); i += blockDim.x) {
      if (p.bias) svec[i] = p.bias[i];
      if (p.res_gain) svec[kMaxDim + i] = p.res_gain[i];
      if (p.out_gain) svec[2 * kMaxDim + i] = p.out_gain[i];
    }
  if (warp == kEpiWarps) {
    if (lane == 0) { tc::tma_prefetch(&tmA); tc::tma_prefetch(&tmB); }
    __syncwarp();
    if (kPair) tc::tmem_alloc_pair(tmem_slot, TMEM_COLS);
    else tc::tmem_alloc(tmem_slot, TMEM_COLS);
  }
  tc::tc_fence_before();
  __syncthreads();
  if (kPair) tc::cluster_sync();  // the peer's barriers are initialised before any remote arrive
  tc::tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  volatile int *abort = &abort_flag;
  const int total = p.m_tiles * p.total_n_tiles;
  // the prologue above (barriers, TMEM, group table, column vectors: none of it produced by an
  // earlier kernel) overlaps the previous kernel's last tiles; its outputs are read from here on
  tc::griddep_wait();
  tc::griddep_launch_dependents();
  GemmGroup g0{};  // the single group of a trunk GEMM
  if (!kGrouped) g0 = p.groups[0];
  auto dec = [&](int tile_) { return tile_dec<kGrouped>(p, g0, gtab, tile_ < total ? tile_ : total - 1); };

  if (warp == kEpiWarps) {
    // ---------------- TMA producer
    // (stall test: CTA 0 loads nothing, a flag nobody sets; its MMA and epilogue waits expire
    // after their bounded limit, record the site and return)
    if (lane == 0 && !(p.stall_test && first_tile == 0)) {
      int stage = 0;
      uint32_t phase = 0;
      // bytes completing on this CTA's full barrier (pair: both CTAs' loads on the leader's)
      const uint32_t bytes = kPair ? 2 * (A_STAGE + (p.BN / 2) * BK * 2) : A_STAGE + p.BN * BK * 2;
      TileDec nx = dec(first_tile);
      for (int tile = first_tile; tile < total; tile += tile_step) {
        const TileDec ti = nx;
        nx = dec(tile + tile_step);
        const GemmGroup &gr = ti.gr;
        const int m0 = ti.mb * kTileM + (int)rank * BM;
        int n0 = gr.b_row_off + ti.nblk * p.BN;
        if (kPair) {  // this CTA's half of the tile's MMA width
          const int n_mma = (min(p.BN, gr.N - ti.nblk * p.BN) + 15) & ~15;
          n0 += (int)rank * (n_mma >> 1);
        }
        const int kblocks = gr.kblocks ? gr.kblocks : p.K / BK;
        bool ok = true;
        for (int kb = 0; kb < kblocks; ++kb) {
          if (!tc::mbar_wait(empty + stage, phase ^ 1, p.status, 10, abort)) { ok = false; break; }
          if (kPair) {
            if (rank == 0) tc::mbar_arrive_expect_tx(full + stage, bytes);
            const uint32_t lb = tc::leader_addr(full + stage);
            if (p.a_mode == 0) tc::tma_load_3d_pair(sA + stage * A_STAGE, &tmA, lb, kb * BK, gr.a_off + m0, 0);
            else tc::tma_load_3d_pair(sA + stage * A_STAGE, &tmA, lb, kb * BK, gr.a_off, m0);
            tc::tma_load_3d_pair(sB + stage * L::b_stage, &tmB, lb, kb * BK, n0, 0);
          } else {
            tc::mbar_arrive_expect_tx(full + stage, bytes);
            if (p.a_mode == 0) tc::tma_load_3d(sA + stage * A_STAGE, &tmA, full + stage, kb * BK, gr.a_off + m0, 0);
            else tc::tma_load_3d(sA + stage * A_STAGE, &tmA, full + stage, kb * BK, gr.a_off, m0);
            tc::tma_load_3d(sB + stage * L::b_stage, &tmB, full + stage, kb * BK, n0, 0);
          }
          if (++stage == kGemmStages) { stage = 0; phase ^= 1; }
        }
        if (!ok) break;
      }
    }
  } else if (warp == kEpiWarps + 1) {
    // ---------------- MMA issuer
    if (lane == 0 && rank == 0) {  // pair: the leader issues the pair's MMAs
      int stage = 0;
      uint32_t phase = 0;
      int local = 0;
      TileDec nx = dec(first_tile);
      for (int tile = first_tile; tile < total; tile += tile_step, ++local) {
        const TileDec ti = nx;
        nx = dec(tile + tile_step);
        const GemmGroup &gr = ti.gr;
        const int acc = local & 1;
        const uint32_t aphase = (local >> 1) & 1;
        int n_eff = min(p.BN, gr.N - ti.nblk * p.BN);
        n_eff = (n_eff + 15) & ~15;
        const uint32_t idesc = tc::idesc_f16(kTileM, n_eff, false, kBF);
        const uint32_t d_tmem = tmem_base + acc * 256;
        const int kblocks = gr.kblocks ? gr.kblocks : p.K / BK;
        if (!tc::mbar_wait(tempty + acc, aphase ^ 1, p.status, 11, abort)) break;
        tc::tc_fence_after();
        bool ok = true;
        for (int kb = 0; kb < kblocks; ++kb) {
          if (!tc::mbar_wait(full + stage, phase, p.status, 12, abort)) { ok = false; break; }
          tc::tc_fence_after();
          const uint32_t a_addr = tc::smem_u32(sA + stage * A_STAGE);
          const uint32_t b_addr = tc::smem_u32(sB + stage * L::b_stage);
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            if (kPair)
              tc::mma_f16_pair(d_tmem, tc::sw128_kmajor_desc(a_addr + kk * 32),
                               tc::sw128_kmajor_desc(b_addr + kk * 32), idesc, (kb | kk) != 0);
            else
              tc::mma_f16(d_tmem, tc::sw128_kmajor_desc(a_addr + kk * 32), tc::sw128_kmajor_desc(b_addr + kk * 32),
                          idesc, (kb | kk) != 0);
          }
          if (kPair) tc::mma_commit_pair(empty + stage, 0x3);
          else tc::mma_commit(empty + stage);
          if (++stage == kGemmStages) { stage = 0; phase ^= 1; }
        }
        if (!ok) break;
        if (kPair) tc::mma_commit_pair(tfull + acc, 0x3);
        else tc::mma_commit(tfull + acc);
      }
      if (kPair) tc::mma_commit_pair(done, 0x1);
      else tc::mma_commit(done);
      tc::mbar_wait(done, 0, p.status, 13, abort);
    }
  } else {
    // ---------------- epilogue warps 0-7
    const int quarter = warp & 3, sub = warp >> 2;  // rows 32 quarter.., chunks sub, sub + kSplit, ...
    uint8_t *stg = smem + L::stg_off + warp * warp_stage_bytes(EPI, kBF);
    int nstore = 0;  // boxes this warp has stored (double-buffer parity)
    int local = 0;
    // The row's deferred-norm sum of squares (and, for QKV, its rotary (cos, sin) pairs),
    // fetched one tile ahead so the loads' latency hides under the previous tile's
    // epilogue: nothing reads them before the next tile.
    RowSS ss_pf;
    row_ss_one(ss_pf);
    QkvRow qr_pf{0, 0};
    float2 cs_pf[16];
    auto row_fetch = [&](int tile_, const TileDec &t_) {
      if (tile_ >= total) return;
      const int m_ = t_.mb * kTileM + (int)rank * BM + quarter * 32 + lane;
      const bool v_ = m_ < p.M;
      if (EPI == kTcQkv) {
        qr_pf = qkv_row(p, v_ ? m_ : 0, t_.g);
        if (v_ && p.ss_in) row_ss_fetch(ss_pf, p.ss_in, qr_pf.tok, p.ss_in_parts);
        else row_ss_one(ss_pf);
        // rotary pairs only for q and k column blocks; 16-byte loads (a row's 16 pairs are
        // 128 contiguous bytes at a 128-byte offset of the table's 256-byte row)
        if (p.dh == 64 && t_.nblk * p.BN < 2 * p.A) {
          const float4 *rp = reinterpret_cast<const float4 *>(p.rope + (long long)qr_pf.pos * 32 + (sub & 1) * 16);
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const float4 w = rp[i];
            cs_pf[2 * i] = make_float2(w.x, w.y);
            cs_pf[2 * i + 1] = make_float2(w.z, w.w);
          }
        }
      } else if (EPI == kTcGelu || EPI == kTcGeglu) {
        if (v_ && p.ss_in) row_ss_fetch(ss_pf, p.ss_in, m_, p.ss_in_parts);
        else row_ss_one(ss_pf);
      } else if (EPI == kTcTanh) {
        if (v_ && p.ss_in) row_ss_fetch(ss_pf, p.ss_in, token_of(p, m_, t_.g), p.ss_in_parts);
        else row_ss_one(ss_pf);
      } else if (EPI == kTcResid) {
        if (v_ && p.res_ss) row_ss_fetch(ss_pf, p.res_ss, m_, p.ss_in_parts);
        else row_ss_one(ss_pf);
      }
    };
    TileDec nx = dec(first_tile);
    row_fetch(first_tile, nx);
    for (int tile = first_tile; tile < total; tile += tile_step, ++local) {
      const TileDec ti = nx;
      const GemmGroup &gr = ti.gr;
      const int acc = local & 1;
      const uint32_t aphase = (local >> 1) & 1;
      const int m0w = ti.mb * kTileM + (int)rank * BM + quarter * 32;  // first row of this warp's 32
      const int m = m0w + lane;
      const bool valid = m < p.M;
      const int nbase = ti.nblk * p.BN;
      const int n_eff = min(p.BN, gr.N - nbase);
      const int nchunks = (n_eff + 31) >> 5;
      const uint32_t tbase = tmem_base + ((uint32_t)(quarter * 32) << 16) + acc * 256;
      // ---- work that does not need the accumulator, before waiting for it
      float rs = 1.f;
      QkvRow qr{0, 0};
      float2 cs[16];
      // 1 / |x| of the row (deferred norm: of the GEMM input, or of the residual for kTcResid)
      const float rsq = 1.f / fmaxf(sqrtf(row_ss_sum(ss_pf)), kEps);
      if (EPI == kTcQkv) {
        qr = qr_pf;
#pragma unroll
        for (int i = 0; i < 16; ++i) cs[i] = cs_pf[i];
      }
      if (EPI == kTcQkv || EPI == kTcGelu || EPI == kTcGeglu || EPI == kTcTanh) rs = rsq;
      const float res_s = rsq;  // kTcResid
      // QKV: which of q (0), k (1), v or the gates (2) the tile's columns belong to, when all
      // of them belong to one; then the row's scale (1 / |x|, times the softmax scale for q) is
      // folded into the rotary (cos, sin) pairs once per tile
      int tile_which = -1;
      if (EPI == kTcQkv) {
        const int last = nbase + n_eff - 1;
        const int w0 = nbase < p.A ? 0 : (nbase < 2 * p.A ? 1 : 2), w1 = last < p.A ? 0 : (last < 2 * p.A ? 1 : 2);
        if (w0 == w1 && w0 < 2 && p.dh == 64) {
          tile_which = w0;
          const float k = w0 == 0 ? rs * p.q_scale : rs;
#pragma unroll
          for (int i = 0; i < 16; ++i) cs[i] = make_float2(cs[i].x * k, cs[i].y * k);
        }
      }
      nx = dec(tile + tile_step);
      row_fetch(tile + tile_step, nx);
      // residual prefetch (kTcResid): fp16 rows of 64 bytes, lane covering rows i*8 + lane/4 and
      // 16-byte piece lane%4; with kBF the fp32 master rows of 128 bytes, rows i*4 + lane/8, piece lane%8.
      // fp16 fetches two chunks ahead (pre: this warp's next chunk, pre2: the one after), which
      // hides a DRAM round trip; the bf16 pieces are twice as many and fetch one chunk ahead.
      constexpr int kPieces = kBF ? 8 : 4;
      uint4 pre[kPieces], pre2[kPieces];
      int c = sub;
      auto residual_fetch = [&](int col, uint4 (&dst)[kPieces]) {
#pragma unroll
        for (int i = 0; i < kPieces; ++i) {
          const int r = kBF ? i * 4 + (lane >> 3) : i * 8 + (lane >> 2);
          const bool ok = m0w + r < p.M;
          if constexpr (kBF)
            dst[i] = ok ? *reinterpret_cast<const uint4 *>(p.X + (long long)(m0w + r) * p.ld + col + (lane & 7) * 4)
                        : make_uint4(0, 0, 0, 0);
          else
            dst[i] = ok ? *reinterpret_cast<const uint4 *>(p.Xh + (long long)(m0w + r) * p.ld + col + (lane & 3) * 8)
                        : make_uint4(0, 0, 0, 0);
        }
      };
      if (EPI == kTcResid && c < nchunks) residual_fetch(nbase + 32 * c, pre);
      if (EPI == kTcResid && !kBF && c + kSplit < nchunks) residual_fetch(nbase + 32 * (c + kSplit), pre2);
      if (!tc::mbar_wait(tfull + acc, aphase, p.status, 14, abort)) break;
      tc::tc_fence_after();
      float sq = 0.f, sqg = 0.f;
      for (; c < nchunks; c += kSplit) {
        const int c0 = nbase + 32 * c;
        float v[32];
        if (EPI == kTcResid || EPI == kTcBandSplit) {
          // x (+ bias) + acc with its row statistics in fp32.  fp16: the residual stream is the
          // fp16 buffer itself.  bf16: an fp32 master copy X, and the bf16 copy the GEMMs read.
          uint8_t *hb = kBF ? stg + 4096 : stg + (nstore & 1) * 2048;
          uint8_t *xb = stg;  // kBF: the fp32 box
          // the boxes' previous stores must have read them (fp16: the store two chunks ago)
          if (lane == 0) {
            if (kBF) tc::bulk_wait_read<0>();
            else tc::bulk_wait_read<1>();
          }
          __syncwarp();
          float x[32];
          if (EPI == kTcResid) {
            // residual rows: coalesced pieces -> swizzled box -> own row
            if constexpr (kBF) {
#pragma unroll
              for (int i = 0; i < 8; ++i) {
                const int r = i * 4 + (lane >> 3), q = lane & 7;
                *reinterpret_cast<uint4 *>(xb + r * 128 + ((q ^ (r & 7)) << 4)) = pre[i];
              }
              __syncwarp();
              box128_get_row(xb, lane, x);
            } else {
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                const int r = i * 8 + (lane >> 2), q = lane & 3;
                *reinterpret_cast<uint4 *>(hb + r * 64 + ((q ^ ((r >> 1) & 3)) << 4)) = pre[i];
              }
              __syncwarp();
              box64_get_row(hb, lane, x);
            }
            if (p.res_ss) {
              float gv[32];
              load_bias32(svec + kMaxDim + c0, gv);
#pragma unroll
              for (int j = 0; j < 32; ++j) x[j] *= res_s * gv[j];
            }
            if constexpr (kBF) {
              if (c + kSplit < nchunks) residual_fetch(c0 + 32 * kSplit, pre);
            } else {
#pragma unroll
              for (int i = 0; i < kPieces; ++i) pre[i] = pre2[i];
              if (c + 2 * kSplit < nchunks) residual_fetch(c0 + 64 * kSplit, pre2);
            }
            if (p.bias) {
              float bv[32];
              load_bias32(svec + c0, bv);
#pragma unroll
              for (int j = 0; j < 32; ++j) x[j] += bv[j];
            }
            __syncwarp();  // every lane has read its row before the box is rewritten
          } else {
            load_bias32(p.bias + gr.bias_off + c0, x);
          }
          tc::tmem_ld32(tbase + 32 * c, v);
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            x[j] += v[j];
            sq += x[j] * x[j];
          }
          if (EPI == kTcResid && p.ssg_out) {
            float gv[32];
            load_bias32(svec + 2 * kMaxDim + c0, gv);
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              const float y = gv[j] * x[j];
              sqg += y * y;
            }
          }
          if (kBF) box128_put_row(xb, lane, x);
          uint4 d[4];
          pack16<kBF>(x, d);
          box64_put_row(hb, lane, d);
          tc::fence_proxy_async();
          __syncwarp();
          if (lane == 0) {
            if (EPI == kTcResid) {
              if (kBF) tc::tma_store_2d(&tmC, xb, c0, m0w);
              tc::tma_store_2d(&tmD, hb, c0, m0w);
            } else {
              if (kBF) tc::tma_store_3d(&tmC, xb, c0, ti.g, m0w);
              tc::tma_store_3d(&tmD, hb, c0, ti.g, m0w);
            }
            tc::bulk_commit();
          }
          ++nstore;
          continue;
        }
        tc::tmem_ld32(tbase + 32 * c, v);
        if (EPI == kTcQkv) {
          // one token-major row [q | k | v | gates]: scale by the row's norm, rotate q and k,
          // fold the softmax scale into q, squash the gates
          const int A3 = 2 * p.A + p.Av;  // the gates' first column
          if (c0 >= A3) {
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              const int h = c0 + j - A3;
              v[j] = h < p.H ? tcm::sigmoid_mufu(v[j] * rs + p.gbias[h]) : 0.f;
            }
          } else if (tile_which >= 0) {
            // q or k with the row scale in the (cos, sin) pairs: (x0 c - x1 s, x1 c + x0 s)
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              const float x0 = v[2 * i], x1 = v[2 * i + 1];
              v[2 * i] = fmaf(x0, cs[i].x, -x1 * cs[i].y);
              v[2 * i + 1] = fmaf(x1, cs[i].x, x0 * cs[i].y);
            }
          } else {
            const int which = c0 < p.A ? 0 : (c0 < 2 * p.A ? 1 : 2);
            const float k = which == 0 ? rs * p.q_scale : rs;
            if (which < 2) {
              if (p.dh == 64) {
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                  const float c = cs[i].x * k, sn = cs[i].y * k, x0 = v[2 * i], x1 = v[2 * i + 1];
                  v[2 * i] = fmaf(x0, c, -x1 * sn);
                  v[2 * i + 1] = fmaf(x1, c, x0 * sn);
                }
              } else {
                const int half_dh = p.dh >> 1;
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                  const int dd = (c0 - which * p.A + 2 * i) % p.dh;
                  const float2 cc = p.rope[(long long)qr.pos * half_dh + (dd >> 1)];
                  const float c = cc.x * k, sn = cc.y * k, x0 = v[2 * i], x1 = v[2 * i + 1];
                  v[2 * i] = fmaf(x0, c, -x1 * sn);
                  v[2 * i + 1] = fmaf(x1, c, x0 * sn);
                }
              }
            } else {
#pragma unroll
              for (int j = 0; j < 32; ++j) v[j] *= k;
            }
          }
          uint8_t *box = stg + (nstore & 1) * 2048;
          if (lane == 0) tc::bulk_wait_read<1>();
          __syncwarp();
          uint4 d[4];
          pack16<kBF>(v, d);
          box64_put_row(box, lane, d);
          tc::fence_proxy_async();
          __syncwarp();
          if (lane == 0) {
            tc::tma_store_2d(&tmC, box, c0, m0w);
            tc::bulk_commit();
          }
          ++nstore;
        } else if (EPI == kTcGelu || EPI == kTcTanh) {
          // N is a multiple of 32 for these layers: every chunk is full
          uint8_t *box = stg + (nstore & 1) * 2048;
          if (lane == 0) tc::bulk_wait_read<1>();
          __syncwarp();
          float bv[32];
          load_bias32(p.bias + gr.bias_off + c0, bv);
          if (EPI == kTcGelu) {
#pragma unroll
            for (int j = 0; j < 32; j += 2) {
              const float2 g = tcm::gelu2(v[j], v[j + 1], rs, bv[j], bv[j + 1]);
              v[j] = g.x;
              v[j + 1] = g.y;
            }
          } else {
#pragma unroll
            for (int j = 0; j < 32; ++j) v[j] = tcm::tanh_mufu(fmaf(v[j], rs, bv[j]));
          }
          uint4 d[4];
          pack16<kBF>(v, d);
          box64_put_row(box, lane, d);
          tc::fence_proxy_async();
          __syncwarp();
          if (lane == 0) {
            if (EPI == kTcGelu) tc::tma_store_2d(&tmC, box, c0, m0w);
            else tc::tma_store_3d(&tmC, box, c0, m0w, gr.out_off);
            tc::bulk_commit();
          }
          ++nstore;
        } else if (EPI == kTcGeglu) {
          // interleaved (value e, gate e) columns -> 16 fp16 outputs value * gelu(gate) per row,
          // stored through a 16 x 32 box (32-byte rows, no swizzle)
          uint8_t *box = stg + (nstore & 1) * 2048;
          if (lane == 0) tc::bulk_wait_read<1>();
          __syncwarp();
          float bv[32];
          load_bias32(p.bias + gr.bias_off + c0, bv);
          float o[16];
#pragma unroll
          for (int j = 0; j < 32; j += 4) {
            const float2 g = tcm::gelu2(v[j + 1], v[j + 3], rs, bv[j + 1], bv[j + 3]);
            o[j >> 1] = fmaf(v[j], rs, bv[j]) * g.x;
            o[(j >> 1) + 1] = fmaf(v[j + 2], rs, bv[j + 2]) * g.y;
          }
          *reinterpret_cast<uint4 *>(box + lane * 32) =
              make_uint4(pack_h2<kBF>(o[0], o[1]), pack_h2<kBF>(o[2], o[3]), pack_h2<kBF>(o[4], o[5]),
                         pack_h2<kBF>(o[6], o[7]));
          *reinterpret_cast<uint4 *>(box + lane * 32 + 16) =
              make_uint4(pack_h2<kBF>(o[8], o[9]), pack_h2<kBF>(o[10], o[11]), pack_h2<kBF>(o[12], o[13]),
                         pack_h2<kBF>(o[14], o[15]));
          tc::fence_proxy_async();
          __syncwarp();
          if (lane == 0) {
            tc::tma_store_2d(&tmC, box, c0 >> 1, m0w);
            tc::bulk_commit();
          }
          ++nstore;
        } else {  // kTcGlu: interleaved (value, gate) pairs -> up to 16 band features of frame m
          // The overlap average is fused here: feature e of the band adds
          // row_weight[r] * value * sigmoid(gate) to masks[b, r, t] (component e & 1) for its
          // stft_repr row r.  A row's (re, im) are features e, e + 1, so each pair is one
          // 8-byte add.  An element receives one add per band covering its bin, at most two,
          // onto the zeroed output: the sum is the same in either order (0 + a = a, a + b =
          // b + a), so the result does not depend on the order of the adds.
          const float *bias = p.bias + gr.bias_off + c0;
          const int nf = min(16, (gr.N - c0) >> 1);
          float o[16];
#pragma unroll
          for (int j = 0; j < 32; j += 2) {
            const bool ok = (j >> 1) < nf;
            const float val = v[j] + (ok ? bias[j] : 0.f);
            const float gt = v[j + 1] + (ok ? bias[j + 1] : 0.f);
            o[j >> 1] = val * tcm::sigmoid_mufu(gt);
          }
          if (valid) {
            const int fe0 = gr.out_off + (c0 >> 1);
            const int bb = m / p.T, t = m - bb * p.T;
            float *dst0 = p.masks + bb * p.mask_bstride + 2LL * t;
            const float *x0 = p.spec ? p.spec + ((long long)bb * p.R * p.T + t) * 2 : nullptr;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              if (2 * i < nf) {
                const int r = __ldg(p.feat_row + fe0 + 2 * i);
                const float w = __ldg(p.row_weight + r);
                if (w != 0.f) {
                  float2 add = make_float2(o[2 * i] * w, o[2 * i + 1] * w);
                  if (x0) {
                    const float2 x = *reinterpret_cast<const float2 *>(x0 + 2LL * r * p.T);
                    add = make_float2(add.x * x.x - add.y * x.y, add.x * x.y + add.y * x.x);
                  }
                  atomicAdd(reinterpret_cast<float2 *>(dst0 + 2LL * r * p.T), add);
                }
              }
            }
          }
        }
      }
      // this warp's partial row sums: one slot per (column tile, warp of the quarter), written
      // (zero when the warp had no chunk) so the consumer adds all slots in a fixed order
      const int slot = ti.nblk * kSplit + sub;
      if (EPI == kTcResid && valid && p.ss_out) p.ss_out[(long long)m * p.ss_out_parts + slot] = sq;
      if (EPI == kTcResid && valid && p.ssg_out) p.ssg_out[(long long)m * p.ss_out_parts + slot] = sqg;
      if (EPI == kTcBandSplit && valid) p.ss_out[((long long)m * p.nb + ti.g) * p.ss_out_parts + slot] = sq;
      tc::tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if (kPair && rank != 0) tc::mbar_arrive_cluster(tc::mapa_shared(tc::smem_u32(tempty + acc), 0));
        else tc::mbar_arrive(tempty + acc);
      }
    }
    // outstanding bulk stores must finish reading shared memory before the CTA exits
    if (lane == 0) tc::bulk_wait_all();
    __syncwarp();
  }
  tc::tc_fence_before();
  __syncthreads();
  if (kPair) tc::cluster_sync();  // no remote arrive or MMA of the pair is outstanding past here
  if (warp == kEpiWarps) {
    tc::tc_fence_after();
    if (kPair) tc::tmem_dealloc_pair(tmem_base, TMEM_COLS);
    else tc::tmem_dealloc(tmem_base, TMEM_COLS);
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

template <int EPI, bool kBF, bool kPair = false>
constexpr size_t smem_bytes() { return SmemLayout<EPI, kBF, kPair>::total + 1024; }
// The epilogue kinds that can run as CTA pairs (the trunk's four GEMMs and the mask MLP's tanh
// layers); the band split and the mask GLU layer run one CTA per tile.
__host__ __device__ constexpr bool pair_kind(int epi) {
  return epi == kTcQkv || epi == kTcResid || epi == kTcGelu || epi == kTcGeglu || epi == kTcTanh;
}
template <int EPI>
constexpr bool smem_fits() {
  return smem_bytes<EPI, false, false>() <= kSmemLimit && smem_bytes<EPI, true, false>() <= kSmemLimit &&
         (!pair_kind(EPI) || (smem_bytes<EPI, false, true>() <= kSmemLimit && smem_bytes<EPI, true, true>() <= kSmemLimit));
}
static_assert(smem_fits<kTcQkv>() && smem_fits<kTcResid>() && smem_fits<kTcGelu>() && smem_fits<kTcBandSplit>() &&
                  smem_fits<kTcGlu>() && smem_fits<kTcTanh>() && smem_fits<kTcGeglu>(),
              "shared memory per CTA over the 227 KB limit");

template <int EPI, bool kBF, bool kPair>
bool set_smem_attr() {
  return cudaFuncSetAttribute(gemm_tc_kernel<EPI, kBF, kPair>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              (int)smem_bytes<EPI, kBF, kPair>()) == cudaSuccess;
}

// pdl: launched with programmatic stream serialisation (the kernel waits for its inputs in
// griddep_wait after its prologue).
template <int EPI, bool kBF, bool kPair>
void launch_one(const CUtensorMap &tmA, const CUtensorMap &tmB, const CUtensorMap &tmC, const CUtensorMap &tmD,
                const GemmParams &p, int grid, bool pdl, cudaStream_t st) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid, 1, 1);
  cfg.blockDim = dim3(gemm_threads(EPI), 1, 1);
  cfg.dynamicSmemBytes = smem_bytes<EPI, kBF, kPair>();
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  int n = 0;
  if (kPair) {
    attr[n].id = cudaLaunchAttributeClusterDimension;
    attr[n].val.clusterDim.x = 2;
    attr[n].val.clusterDim.y = 1;
    attr[n].val.clusterDim.z = 1;
    ++n;
  }
  if (pdl) {
    attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[n].val.programmaticStreamSerializationAllowed = 1;
    ++n;
  }
  cfg.attrs = attr;
  cfg.numAttrs = n;
  cudaLaunchKernelEx(&cfg, gemm_tc_kernel<EPI, kBF, kPair>, tmA, tmB, tmC, tmD, p);
}

}  // namespace

bool make_tmap(CUtensorMap *map, const void *base, int dtype, int rank, const unsigned long long *dims,
               const unsigned long long *strides_el, const unsigned *box, int swizzle_bytes) {
  auto fn = encode_fn();
  if (!fn) return false;
  const int esz = dtype == kTmF32 ? 4 : 2;
  cuuint64_t d[5] = {1, 1, 1, 1, 1}, st[4] = {0, 0, 0, 0};
  cuuint32_t b[5] = {1, 1, 1, 1, 1}, es[5] = {1, 1, 1, 1, 1};
  if (rank < 1 || rank > 5) return false;
  for (int i = 0; i < rank; ++i) { d[i] = dims[i]; b[i] = box[i]; }
  for (int i = 0; i + 1 < rank; ++i) st[i] = strides_el[i] * esz;
  const CUtensorMapSwizzle sw = swizzle_bytes == 128 ? CU_TENSOR_MAP_SWIZZLE_128B
                                : swizzle_bytes == 64 ? CU_TENSOR_MAP_SWIZZLE_64B
                                : swizzle_bytes == 32 ? CU_TENSOR_MAP_SWIZZLE_32B
                                                      : CU_TENSOR_MAP_SWIZZLE_NONE;
  CUresult r = fn(map, dtype == kTmF32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, rank,
                  const_cast<void *>(base), d, st, b, es, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool make_tmap_f16(CUtensorMap *map, const void *base, unsigned long long d0, unsigned long long d1,
                   unsigned long long d2, unsigned long long s1, unsigned long long s2, unsigned box1,
                   unsigned box2) {
  const unsigned long long dims[3] = {d0, d1, d2}, st[2] = {s1, s2};
  const unsigned box[3] = {64, box1, box2};
  return make_tmap(map, base, kTmF16, 3, dims, st, box, 128);
}

bool gemm_tc_init() {
  bool ok = encode_fn() != nullptr;
#define MRF_GEMM_ATTR(E)                                                                      \
  ok = ok && set_smem_attr<E, false, false>() && set_smem_attr<E, true, false>();             \
  if (pair_kind(E)) ok = ok && set_smem_attr<E, false, pair_kind(E)>() && set_smem_attr<E, true, pair_kind(E)>();
  MRF_GEMM_ATTR(kTcQkv)
  MRF_GEMM_ATTR(kTcResid)
  MRF_GEMM_ATTR(kTcGelu)
  MRF_GEMM_ATTR(kTcTanh)
  MRF_GEMM_ATTR(kTcGlu)
  MRF_GEMM_ATTR(kTcGeglu)
  MRF_GEMM_ATTR(kTcBandSplit)
#undef MRF_GEMM_ATTR
  return ok;
}

bool gemm_tc_pair_kind(int epi) { return pair_kind(epi); }

void launch_gemm_tc(int epi, bool bf16, bool pair, const CUtensorMap &tmA, const CUtensorMap &tmB,
                    const CUtensorMap &tmC, const CUtensorMap &tmD, const GemmParams &p, int grid, bool pdl,
                    cudaStream_t st) {
  switch (epi) {
#define MRF_GEMM_CASE(E)                                                                          \
  case E:                                                                                         \
    if (pair && pair_kind(E)) {                                                                   \
      if (bf16) launch_one<E, true, pair_kind(E)>(tmA, tmB, tmC, tmD, p, grid, pdl, st);               \
      else launch_one<E, false, pair_kind(E)>(tmA, tmB, tmC, tmD, p, grid, pdl, st);                   \
    } else {                                                                                      \
      if (bf16) launch_one<E, true, false>(tmA, tmB, tmC, tmD, p, grid, pdl, st);                      \
      else launch_one<E, false, false>(tmA, tmB, tmC, tmD, p, grid, pdl, st);                          \
    }                                                                                             \
    break;
    MRF_GEMM_CASE(kTcQkv)
    MRF_GEMM_CASE(kTcResid)
    MRF_GEMM_CASE(kTcGelu)
    MRF_GEMM_CASE(kTcTanh)
    MRF_GEMM_CASE(kTcGlu)
    MRF_GEMM_CASE(kTcGeglu)
    MRF_GEMM_CASE(kTcBandSplit)
#undef MRF_GEMM_CASE
    default: break;
  }
}

}  // namespace mrf
