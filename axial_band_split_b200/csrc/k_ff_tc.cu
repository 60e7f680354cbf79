// Fused feed-forward of one transformer on CTA pairs (tcgen05, cta_group::2):
//   x <- x + W2 gelu(rs * (W1' x) + b1) + b2,   rs = 1 / max(|x|_2, eps) per row,
// with W1' = W1 gamma sqrt(D) (the pre-norm's gain folded into the weight), and the row sums of
// squares of the new x (and of g * x, the next output norm's input) written as partial slots.
//
// The layer is the FeedForward of "Mel-Band RoFormer — architecture, inference hot path & RTX 3050
// feasibility", section "The two transformers are not the same shape" (RMSNorm, Linear(D, 4D),
// GELU, Linear(4D, D), residual); the exact rewrites (gain folded into W1, the norm deferred to a
// row scale) are those of "@audio/neural-separate 0.4.0 → 0.5.0", package/scripts/export-roformer.py,
// class Core.  The hidden activations never leave the SM pair.
//
// A cluster of two CTAs on two SMs takes 256 rows of x at a time (CTA r: rows 128 r .. 128 r + 127):
//   x tile      the CTA's 128 rows x D in shared memory (D / 64 K-major 128-byte-swizzled blocks),
//               loaded once per tile;
//   chunk i     of the hidden units (128 each): MMA1 H_acc = x W1[128 i .. 128 i + 127]'
//               (M = 256 over the pair, N = 128, each CTA staging half of every W1 block); the
//               epilogue warps read H_acc, apply the row scale, bias and GELU, and write fp16 H in
//               the K-major swizzled layout of an MMA operand; MMA2 O_acc += H W2[:, chunk]'
//               (M = 256, N = D in pieces of at most 256, each CTA staging half of every W2 block);
//   epilogue    O_acc + b2 + x, written to the residual stream with its row statistics.
// The MMA issuer runs MMA1(i + 1) before MMA2(i), so the tensor core computes the next chunk while
// the epilogue turns the current one into H.
//
// Tensor memory: O_acc in columns 0 .. D - 1 (D <= 384), H_acc in columns 384 .. 511.
// Warps 0-15: epilogue (warp w: TMEM lane quarter w % 4, hidden columns 32 (w / 4) .. of a chunk;
// output columns 32 (w / 4 + 4 j) of the final epilogue); warp 16: TMA producer; warp 17: TMEM
// allocation and, in the leader CTA, the MMA issuer.  The epilogue warps release H_acc, hand over
// H and release O_acc on their own CTA's barriers; in the peer CTA, four lanes of warp 17 forward
// each completed phase to the leader's barrier with one cluster-scope arrive (an arrive with
// cluster release semantics from every epilogue warp cost each of them ~1,900 clk a chunk).  Every
// wait is bounded (the error path of tc::mbar_wait).
#include <cuda_fp16.h>

#include <algorithm>

#include "gemm_tc.cuh"
#include "mrf_internal.h"
#include "tc_math.cuh"
#include "tc_ptx.cuh"

namespace mrf {

namespace {

constexpr int kFfRows = 128;                 // rows per CTA (256 per pair)
constexpr int kChunk = 128;                  // hidden units per chunk
constexpr int kEpiWarps = 16;
constexpr int kThreadsFf = 32 * (kEpiWarps + 2);
constexpr int kW1Stages = 4, kW2Stages = 2;
constexpr int kMaxD = 384, kMaxHidden = 1536;
constexpr int kXBlock = kFfRows * 64 * 2;           // 16 KB: 128 rows x 64 fp16
constexpr int kW1Stage = (kChunk / 2) * 64 * 2;      // 8 KB: this CTA's half of a chunk's 64-wide K block
constexpr int kW2StageMax = (kMaxD / 2) * 64 * 2;    // 24 KB: this CTA's half of D rows x 64 hidden
constexpr float kEps = 1e-12f;

struct FfSmem {
  static constexpr int x = 0;                                   // [D / 64][128 rows x 128 B]
  static constexpr int w1 = x + (kMaxD / 64) * kXBlock;         // [kW1Stages]
  static constexpr int w2 = w1 + kW1Stages * kW1Stage;          // [kW2Stages]
  static constexpr int h = w2 + kW2Stages * kW2StageMax;        // [2][128 rows x 128 B]; the output staging later
  static constexpr int vec = h + 2 * kXBlock;                   // b1 [hidden], b2 [D], out_gain [D] floats
  static constexpr int bar = vec + (kMaxHidden + 2 * kMaxD) * 4;
  static constexpr int total = bar + 256;
};
static_assert(FfSmem::total + 1024 <= 232448, "fused feed-forward shared memory over the 227 KB limit");

__device__ __forceinline__ uint32_t pack_f16(float a, float b) {
  __half2 h = __floats2half2_rn(a, b);
  return *reinterpret_cast<uint32_t *>(&h);
}

// Arrive on the leader CTA's copy of a barrier from the peer (through the cluster address).
__device__ __forceinline__ void arrive_remote_leader(uint64_t *bar) {
  tc::mbar_arrive_cluster(tc::mapa_shared(tc::smem_u32(bar), 0));
}

__global__ void __launch_bounds__(kThreadsFf, 1)
    ff_tc_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW1,
                 const __grid_constant__ CUtensorMap tmW2, const __grid_constant__ CUtensorMap tmO,
                 const FfParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *sx = smem + FfSmem::x, *sw1 = smem + FfSmem::w1, *sw2 = smem + FfSmem::w2, *sh = smem + FfSmem::h;
  float *sb1 = reinterpret_cast<float *>(smem + FfSmem::vec), *sb2 = sb1 + kMaxHidden, *sg = sb2 + kMaxD;
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + FfSmem::bar);
  uint64_t *x_full = bars + 0, *x_empty = bars + 1;
  uint64_t *w1_full = bars + 2, *w1_empty = bars + 2 + kW1Stages;                     // [kW1Stages]
  uint64_t *w2_full = bars + 2 + 2 * kW1Stages, *w2_empty = w2_full + kW2Stages;     // [kW2Stages]
  uint64_t *hacc_full = w2_empty + kW2Stages, *hacc_empty = hacc_full + 1;
  uint64_t *hsm_full = hacc_full + 2, *hsm_empty = hacc_full + 4;  // [2]: per 64-wide K block of H
  uint64_t *o_full = hacc_full + 6, *o_empty = hacc_full + 7;
  uint64_t *stg_free = hacc_full + 8, *done = hacc_full + 9;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(done + 1);
  __shared__ int abort_flag;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = tc::cluster_ctarank();
  const int D = p.D, kbx = D / 64, nchunks = p.hidden / kChunk;
  const int n2 = D > 256 ? 2 : 1, np = D / n2;  // MMA2 pieces of np outputs (each CTA stages np / 2 rows)
  const uint32_t w2_stage = (uint32_t)(D / 2) * 128;
  const int tiles = (p.M + 2 * kFfRows - 1) / (2 * kFfRows);
  const int first_tile = (int)(blockIdx.x >> 1), tile_step = (int)(gridDim.x >> 1);

  if (threadIdx.x == 0) {
    abort_flag = 0;
    tc::mbar_init(x_full, 1);
    tc::mbar_init(x_empty, 1);
    for (int s = 0; s < kW1Stages; ++s) { tc::mbar_init(w1_full + s, 1); tc::mbar_init(w1_empty + s, 1); }
    for (int s = 0; s < kW2Stages; ++s) { tc::mbar_init(w2_full + s, 1); tc::mbar_init(w2_empty + s, 1); }
    // released by this CTA's epilogue warps, and in the leader also by the peer's forwarding lane
    const uint32_t fwd = rank == 0 ? 1 : 0;
    tc::mbar_init(hacc_full, 1);
    tc::mbar_init(hacc_empty, kEpiWarps + fwd);
    for (int kb = 0; kb < 2; ++kb) {
      tc::mbar_init(hsm_full + kb, kEpiWarps / 2 + fwd);  // the 8 warps that write the K block
      tc::mbar_init(hsm_empty + kb, 1);
    }
    tc::mbar_init(o_full, 1);
    tc::mbar_init(o_empty, kEpiWarps + fwd);
    tc::mbar_init(stg_free, kEpiWarps);        // this CTA's epilogue warps
    tc::mbar_init(done, 1);
    tc::fence_barrier_init();
  }
  // biases and the output gain (weights: not produced by an earlier kernel)
  for (int i = threadIdx.x; i < p.hidden; i += blockDim.x) sb1[i] = p.b1[i];
  for (int i = threadIdx.x; i < D; i += blockDim.x) {
    sb2[i] = p.b2[i];
    sg[i] = p.out_gain[i];
  }
  if (warp == kEpiWarps + 1) tc::tmem_alloc_pair(tmem_slot, 512);
  if (warp == kEpiWarps && lane == 0) {
    tc::tma_prefetch(&tmX);
    tc::tma_prefetch(&tmW1);
    tc::tma_prefetch(&tmW2);
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::cluster_sync();  // the peer's barriers are initialised before any remote arrive
  tc::tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  volatile int *abort = &abort_flag;
  tc::griddep_wait();
  tc::griddep_launch_dependents();

  if (warp == kEpiWarps) {
    // ---------------- TMA producer: x of a tile, then per chunk i its W1 blocks and W2(i - 1)'s
    // blocks, the order in which the MMA issuer consumes them
    if (lane == 0) {
      int s1 = 0, s2 = 0;
      uint32_t ph1 = 0, ph2 = 0;
      int lt = 0;
      bool ok = true;
      auto load_w2 = [&](int chunk) {
        for (int kb = 0; kb < kChunk / 64 && ok; ++kb) {
          if (!tc::mbar_wait(w2_empty + s2, ph2 ^ 1, p.status, 52, abort)) { ok = false; break; }
          if (rank == 0) tc::mbar_arrive_expect_tx(w2_full + s2, 2 * w2_stage);
          const uint32_t lb = tc::leader_addr(w2_full + s2);
          for (int pc = 0; pc < n2; ++pc)
            tc::tma_load_3d_pair(sw2 + s2 * kW2StageMax + pc * (np / 2) * 128, &tmW2, lb, chunk * kChunk + kb * 64,
                                 pc * np + (int)rank * (np / 2), 0);
          if (++s2 == kW2Stages) { s2 = 0; ph2 ^= 1; }
        }
      };
      for (int tile = first_tile; ok && tile < tiles; tile += tile_step, ++lt) {
        if (!tc::mbar_wait(x_empty, (lt & 1) ^ 1, p.status, 50, abort)) break;
        if (rank == 0) tc::mbar_arrive_expect_tx(x_full, 2 * kbx * kXBlock);
        const int m0 = tile * 2 * kFfRows + (int)rank * kFfRows;
        for (int kb = 0; kb < kbx; ++kb)
          tc::tma_load_3d_pair(sx + kb * kXBlock, &tmX, tc::leader_addr(x_full), kb * 64, m0, 0);
        for (int c = 0; c < nchunks && ok; ++c) {
          for (int kb = 0; kb < kbx; ++kb) {
            if (!tc::mbar_wait(w1_empty + s1, ph1 ^ 1, p.status, 51, abort)) { ok = false; break; }
            if (rank == 0) tc::mbar_arrive_expect_tx(w1_full + s1, 2 * kW1Stage);
            tc::tma_load_3d_pair(sw1 + s1 * kW1Stage, &tmW1, tc::leader_addr(w1_full + s1), kb * 64,
                                 c * kChunk + (int)rank * (kChunk / 2), 0);
            if (++s1 == kW1Stages) { s1 = 0; ph1 ^= 1; }
          }
          if (ok && c > 0) load_w2(c - 1);
        }
        if (ok) load_w2(nchunks - 1);
      }
    }
  } else if (warp == kEpiWarps + 1) {
    // ---------------- MMA issuer (the leader's thread): MMA1(i) into H_acc, then MMA2(i - 1)
    if (lane == 0 && rank == 0) {
      const uint32_t id1 = tc::idesc_f16(2 * kFfRows, kChunk), id2 = tc::idesc_f16(2 * kFfRows, np);
      const uint32_t t_h = tmem_base + kMaxD;  // H_acc columns
      int s1 = 0, s2 = 0;
      uint32_t ph1 = 0, ph2 = 0;
      int ch = 0;  // chunks issued so far (all tiles)
      int lt = 0;
      bool ok = true;
      auto mma2 = [&](int chunk, int gch) {
        // O_acc released by the previous tile's final epilogue before the tile's first accumulation
        if (chunk == 0 && !tc::mbar_wait(o_empty, (lt & 1) ^ 1, p.status, 56, abort)) { ok = false; return; }
        for (int kb = 0; kb < kChunk / 64; ++kb) {
          // K block kb of H(chunk) written by the epilogue (its gch-th H)
          if (!tc::mbar_wait<true>(hsm_full + kb, gch & 1, p.status, 55, abort)) { ok = false; return; }
          if (!tc::mbar_wait(w2_full + s2, ph2, p.status, 57, abort)) { ok = false; return; }
          tc::tc_fence_after();
          const uint32_t a = tc::smem_u32(sh + kb * kXBlock), b = tc::smem_u32(sw2 + s2 * kW2StageMax);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            for (int pc = 0; pc < n2; ++pc)
              tc::mma_f16_pair(tmem_base + pc * np, tc::sw128_kmajor_desc(a + kk * 32),
                               tc::sw128_kmajor_desc(b + pc * (np / 2) * 128 + kk * 32), id2,
                               (chunk | kb | kk) != 0);
          tc::mma_commit_pair(w2_empty + s2, 0x3);
          tc::mma_commit_pair(hsm_empty + kb, 0x3);  // this K block of H may be rewritten
          if (++s2 == kW2Stages) { s2 = 0; ph2 ^= 1; }
        }
      };
      for (int tile = first_tile; ok && tile < tiles; tile += tile_step, ++lt) {
        if (!tc::mbar_wait(x_full, lt & 1, p.status, 53, abort)) break;
        tc::tc_fence_after();
        for (int c = 0; c < nchunks && ok; ++c, ++ch) {
          // H_acc released by the epilogue of the previous chunk
          if (!tc::mbar_wait(hacc_empty, (ch & 1) ^ 1, p.status, 54, abort)) { ok = false; break; }
          tc::tc_fence_after();
          for (int kb = 0; kb < kbx; ++kb) {
            if (!tc::mbar_wait(w1_full + s1, ph1, p.status, 58, abort)) { ok = false; break; }
            tc::tc_fence_after();
            const uint32_t a = tc::smem_u32(sx + kb * kXBlock), b = tc::smem_u32(sw1 + s1 * kW1Stage);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              tc::mma_f16_pair(t_h, tc::sw128_kmajor_desc(a + kk * 32), tc::sw128_kmajor_desc(b + kk * 32), id1,
                               (kb | kk) != 0);
            tc::mma_commit_pair(w1_empty + s1, 0x3);
            if (++s1 == kW1Stages) { s1 = 0; ph1 ^= 1; }
          }
          if (!ok) break;
          if (c == nchunks - 1) tc::mma_commit_pair(x_empty, 0x3);  // x no longer read by the MMAs
          tc::mma_commit_pair(hacc_full, 0x3);
          if (c > 0) mma2(c - 1, ch - 1);
        }
        if (!ok) break;
        mma2(nchunks - 1, ch - 1);
        if (!ok) break;
        tc::mma_commit_pair(o_full, 0x3);
      }
      tc::mma_commit_pair(done, 0x1);
      tc::mbar_wait(done, 0, p.status, 59, abort);
    } else if (rank == 1 && lane < 4) {
      // the peer's forwarding lanes: lane 0 H_acc released, lanes 1 and 2 H's K blocks written,
      // lane 3 O_acc released; each waits for its local barrier's phases in order and arrives once
      // on the leader's copy (a local phase runs at most one ahead: the next needs the leader's
      // MMA, which needs this forward)
      uint64_t *bar = lane == 0 ? hacc_empty : (lane == 3 ? o_empty : hsm_full + (lane - 1));
      const int per_tile = lane == 3 ? 1 : nchunks;
      int n = 0;
      for (int tile = first_tile; tile < tiles; tile += tile_step)
        for (int i = 0; i < per_tile; ++i, ++n) {
          if (!tc::mbar_wait(bar, n & 1, p.status, 64, abort)) { tile = tiles; break; }
          arrive_remote_leader(bar);
        }
    }
  } else {
    // ---------------- epilogue warps 0-15
    const int quarter = warp & 3, sub = warp >> 2;
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const int r = quarter * 32 + lane;  // this thread's row of the CTA's 128
    uint8_t *stg = sh + warp * 2048;    // output staging box (the H buffer is free by then)
    int ch = 0, lt = 0;
    for (int tile = first_tile; tile < tiles; tile += tile_step, ++lt) {
      const int m0w = tile * 2 * kFfRows + (int)rank * kFfRows + quarter * 32;
      const int m = m0w + lane;
      const bool valid = m < p.M;
      // row scale of the pre-norm from the out-projection's partial sums of squares
      float ssum = 0.f;
      if (valid)
        for (int i = 0; i < p.ss_in_parts; ++i) ssum += p.ss_in[(long long)m * p.ss_in_parts + i];
      const float rs = 1.f / fmaxf(sqrtf(ssum), kEps);
      bool ok = true;
      for (int c = 0; c < nchunks; ++c, ++ch) {
        if (!tc::mbar_wait(hacc_full, ch & 1, p.status, 60, abort)) { ok = false; break; }
        tc::tc_fence_after();
        float v[32];
        tc::tmem_ld32(tmem_base + lane_off + kMaxD + 32 * sub, v);
        tc::tc_fence_before();
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(hacc_empty);  // MMA1 of the next chunk may overwrite H_acc
        const float *bv = sb1 + c * kChunk + 32 * sub;
        uint32_t hw[16];
#pragma unroll
        for (int j = 0; j < 32; j += 2) {
          const float2 g = tcm::gelu2(v[j], v[j + 1], rs, bv[j], bv[j + 1]);
          hw[j >> 1] = pack_f16(g.x, g.y);
        }
        // this warp's K block of H is free once the previous MMA2 has read it (and, for a tile's
        // first chunk, once the previous tile's output staging has been read by its bulk stores)
        if (!tc::mbar_wait(hsm_empty + (sub >> 1), (ch & 1) ^ 1, p.status, 61, abort)) { ok = false; break; }
        if (c == 0 && lt > 0 && !tc::mbar_wait(stg_free, (lt - 1) & 1, p.status, 62, abort)) { ok = false; break; }
        // row r's 32 hidden values at columns 32 sub .. of the chunk: K block sub / 2, 16-byte
        // pieces 4 (sub % 2) .. 4 (sub % 2) + 3 of the row's 128 bytes, 128-byte swizzle
        uint8_t *hrow = sh + (sub >> 1) * kXBlock + r * 128;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int piece = 4 * (sub & 1) + q;
          *reinterpret_cast<uint4 *>(hrow + ((piece ^ (r & 7)) << 4)) =
              make_uint4(hw[4 * q], hw[4 * q + 1], hw[4 * q + 2], hw[4 * q + 3]);
        }
        tc::fence_proxy_async_all();  // the pair's tensor core reads H through the async proxy
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(hsm_full + (sub >> 1));
      }
      if (!ok) break;
      // ---- final epilogue: x + O_acc + b2, row statistics, bulk stores through the staging box
      if (!tc::mbar_wait(o_full, lt & 1, p.status, 63, abort)) break;
      tc::tc_fence_after();
      float sq = 0.f, sqg = 0.f;
      for (int j = sub; j < D / 32; j += 4) {
        const int c0 = 32 * j;
        // residual rows: coalesced 16-byte pieces -> swizzled box -> own row
        uint4 pre[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int rr = i * 8 + (lane >> 2);
          pre[i] = m0w + rr < p.M
                       ? *reinterpret_cast<const uint4 *>(p.Xh + (long long)(m0w + rr) * p.ld + c0 + (lane & 3) * 8)
                       : make_uint4(0, 0, 0, 0);
        }
        if (lane == 0) tc::bulk_wait_read<0>();  // the box's previous store has read it
        __syncwarp();
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int rr = i * 8 + (lane >> 2), qq = lane & 3;
          *reinterpret_cast<uint4 *>(stg + rr * 64 + ((qq ^ ((rr >> 1) & 3)) << 4)) = pre[i];
        }
        __syncwarp();
        float x[32];
#pragma unroll
        for (int qq = 0; qq < 4; ++qq) {
          const uint4 a = *reinterpret_cast<const uint4 *>(stg + lane * 64 + ((qq ^ ((lane >> 1) & 3)) << 4));
          const uint32_t w[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&w[i]));
            x[8 * qq + 2 * i] = f.x;
            x[8 * qq + 2 * i + 1] = f.y;
          }
        }
        __syncwarp();  // every lane has read its row before the box is rewritten
        float o[32];
        tc::tmem_ld32(tmem_base + lane_off + c0, o);
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          x[i] += o[i] + sb2[c0 + i];
          sq += x[i] * x[i];
          const float y = sg[c0 + i] * x[i];
          sqg += y * y;
        }
#pragma unroll
        for (int qq = 0; qq < 4; ++qq)
          *reinterpret_cast<uint4 *>(stg + lane * 64 + ((qq ^ ((lane >> 1) & 3)) << 4)) =
              make_uint4(pack_f16(x[8 * qq], x[8 * qq + 1]), pack_f16(x[8 * qq + 2], x[8 * qq + 3]),
                         pack_f16(x[8 * qq + 4], x[8 * qq + 5]), pack_f16(x[8 * qq + 6], x[8 * qq + 7]));
        tc::fence_proxy_async();
        __syncwarp();
        if (lane == 0) {
          tc::tma_store_2d(&tmO, stg, c0, m0w);
          tc::bulk_commit();
        }
      }
      // O_acc read: the next tile's MMA2 may overwrite it
      tc::tc_fence_before();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(o_empty);
      if (valid) {
        p.ss_out[(long long)m * p.ss_out_parts + sub] = sq;
        p.ssg_out[(long long)m * p.ss_out_parts + sub] = sqg;
      }
      // the staging box (inside H) is free once this warp's bulk stores have read it
      if (lane == 0) {
        tc::bulk_wait_read<0>();
        tc::mbar_arrive(stg_free);
      }
      __syncwarp();
    }
    if (lane == 0) tc::bulk_wait_all();
    __syncwarp();
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::cluster_sync();  // no remote arrive or MMA of the pair is outstanding past here
  if (warp == kEpiWarps + 1) {
    tc::tc_fence_after();
    tc::tmem_dealloc_pair(tmem_base, 512);
  }
}

}  // namespace

bool ff_tc_supported(int D, int hidden) {
  return D % 64 == 0 && D >= 64 && D <= kMaxD && hidden % kChunk == 0 && hidden <= kMaxHidden;
}

bool ff_tc_init() {
  return cudaFuncSetAttribute(ff_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              (int)(FfSmem::total + 1024)) == cudaSuccess;
}

void launch_ff_tc(const CUtensorMap &tmX, const CUtensorMap &tmW1, const CUtensorMap &tmW2, const CUtensorMap &tmO,
                  const FfParams &p, int sms, bool pdl, cudaStream_t st) {
  const int tiles = (p.M + 2 * kFfRows - 1) / (2 * kFfRows);
  const int pairs = std::max(1, std::min(tiles, sms / 2));
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(2 * pairs), 1, 1);
  cfg.blockDim = dim3(kThreadsFf, 1, 1);
  cfg.dynamicSmemBytes = FfSmem::total + 1024;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 2 : 1;
  cudaLaunchKernelEx(&cfg, ff_tc_kernel, tmX, tmW1, tmW2, tmO, p);
}

}  // namespace mrf
