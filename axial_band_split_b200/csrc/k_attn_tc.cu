// Fused softmax attention on tcgen05 tensor cores, dim_head 64: o = softmax(q k^T /
// sqrt(dh)) v per (sequence, head), times the head's sigmoid gate, written token-major
// for the output projection.  The [n, n] scores never leave the SM.
//
// The layer is the gated attention of "Mel-Band RoFormer — architecture, inference hot
// path & RTX 3050 feasibility", sections "The two transformers are not the same shape"
// (per-head out * sigmoid(gates); the time transformer attends over T within each band,
// the band transformer over the bands within each frame) and "The flash-attn caveat" (the
// memory-efficient kernel tiles the scores rather than materialising them).  Splitting the
// queries into blocks is exact (model card "musetric/vocal-separation-roformer-onnx",
// section "How these graphs are written").
//
// Persistent CTAs; a work item is two 128-row query tiles t = 0, 1 processed in ping-pong:
//   time axis - two consecutive query tiles of one (band, head) sequence; the keys stream
//               in blocks of 128 and each K/V block serves both tiles;
//   band axis - each tile holds two 64-row problems (n <= 64) with their own single K/V
//               block, masked block-diagonally.
// Warps 0-3 and 4-7: softmax of tile 0 and tile 1 (one query row per thread); warp 8: TMA;
// warp 9: MMA issue.  Tensor memory (512 columns): S_t at 128 t, O_t at 256 + 64 t.
// O accumulates in tensor memory across key blocks; a row's running max is raised (and
// its O row rescaled in place) only when a block's max exceeds it by more than 2^8, so
// the unnormalised p stay below 256 and most blocks need no correction.
#include <cmath>

#include "mrf_internal.h"
#include "tc_ptx.cuh"

namespace mrf {

namespace {

constexpr int kDh = 64, kRows = 128, kKeys = 128, kStages = 2;
constexpr int kTile = kRows * kDh * 2;  // 16 KB: one 128 x 64 fp16 tile
constexpr int kThreads = 320;
constexpr float kRescaleLog2 = 8.f;

struct AttnSmem {
  static constexpr int q = 0;                              // [2 tiles]
  static constexpr int kv = q + 2 * kTile;                 // [stage][tile][K, V]
  static constexpr int p = kv + kStages * 4 * kTile;       // [2 tiles] 128 x 128 fp16 (two column blocks)
  static constexpr int bar = p + 2 * 2 * kTile;
  static constexpr int total = bar + 256;
};

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// 2^x on the FMA pipe: x = n + f with n = round(x) (magic-number rounding), 2^f by a
// degree-3 minimax polynomial on [-1/2, 1/2] (relative error 7.5e-5, coefficients from
// fit_exp2_poly.py), and 2^n added into the exponent bits.  x <= 8 here; below -126 the
// result is flushed to 0 like ex2.approx.ftz.
__device__ __forceinline__ float exp2_fma(float x) {
  x = fmaxf(x, -126.f);
  const float t = x + 12582912.f;          // 1.5 * 2^23: round to nearest integer
  const float n = t - 12582912.f;
  const float f = x - n;
  float p = fmaf(0.055171669f, f, 0.242611122f);
  p = fmaf(p, f, 0.693260985f);
  p = fmaf(p, f, 0.999928074f);
  return __int_as_float(__float_as_int(p) + (__float_as_int(t) << 23));
}

__device__ __forceinline__ uint32_t pack_h2(float a, float b) {
  __half2 h = __floats2half2_rn(a, b);
  return *reinterpret_cast<uint32_t *>(&h);
}

struct AttnArgs {
  const float *gate;
  __half *o;
  unsigned *status;
  int B, T, nb, H, axis, n_pad, n, q_tiles, pairs, items, n_blocks;
  long long problems;
};

// Rows of the item's query tiles and key blocks.
struct Item {
  long long q_row[2], k_row[2];
  long long sh;  // time axis: sequence * H + head; band axis: first problem of the item
  int qt0;       // time axis: index of tile 0 within the sequence
};

__device__ __forceinline__ Item item_rows(const AttnArgs &a, int item) {
  Item it;
  if (a.axis == 0) {
    it.sh = item / a.pairs;
    it.qt0 = 2 * (item % a.pairs);
    for (int t = 0; t < 2; ++t) {
      it.q_row[t] = it.sh * a.n_pad + (long long)(it.qt0 + t) * kRows;
      it.k_row[t] = it.sh * a.n_pad;
    }
  } else {
    it.sh = 4LL * item;
    it.qt0 = 0;
    for (int t = 0; t < 2; ++t) {
      it.q_row[t] = (it.sh + 2 * t) * a.n_pad;  // n_pad == 64
      it.k_row[t] = it.q_row[t];
    }
  }
  return it;
}

__global__ void __launch_bounds__(kThreads, 1)
    attn_tc_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                   const __grid_constant__ CUtensorMap tv, const AttnArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + AttnSmem::bar);
  uint64_t *q_full = bars + 0, *q_empty = bars + 1;
  uint64_t *kv_full = bars + 2;     // [kStages]
  uint64_t *kv_empty = bars + 4;    // [kStages]
  uint64_t *s_full = bars + 6;      // [2]
  uint64_t *p_full = bars + 8;      // [2]
  uint64_t *pv_done = bars + 10;    // [2]
  uint64_t *o_free = bars + 12;     // [2]
  uint64_t *done = bars + 14;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 15);
  __shared__ int abort_flag;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const bool shared_kv = a.axis == 0;
  if (threadIdx.x == 0) {
    abort_flag = 0;
    tc::mbar_init(q_full, 1);
    tc::mbar_init(q_empty, 1);
    for (int s = 0; s < kStages; ++s) { tc::mbar_init(kv_full + s, 1); tc::mbar_init(kv_empty + s, 1); }
    for (int t = 0; t < 2; ++t) {
      tc::mbar_init(s_full + t, 1);
      tc::mbar_init(p_full + t, 4);
      tc::mbar_init(pv_done + t, 1);
      tc::mbar_init(o_free + t, 4);
    }
    tc::mbar_init(done, 1);
    tc::fence_barrier_init();
  }
  if (warp == 8) tc::tmem_alloc(tmem_slot, 512);
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  volatile int *abort = &abort_flag;

  if (warp == 8) {
    // ---------------- TMA producer
    if (lane == 0) {
      const uint32_t kv_bytes = (shared_kv ? 2 : 4) * kTile;
      int g = 0;  // key blocks loaded so far
      int li = 0;
      bool ok = true;
      for (int item = blockIdx.x; ok && item < a.items; item += gridDim.x, ++li) {
        const Item it = item_rows(a, item);
        if (!tc::mbar_wait(q_empty, (li & 1) ^ 1, a.status, 30, abort)) break;
        tc::mbar_arrive_expect_tx(q_full, 2 * kTile);
        for (int t = 0; t < 2; ++t)
          tc::tma_load_3d(smem + AttnSmem::q + t * kTile, &tq, q_full, 0, (int)it.q_row[t], 0);
        for (int j = 0; j < a.n_blocks; ++j, ++g) {
          const int s = g % kStages;
          if (!tc::mbar_wait(kv_empty + s, ((g / kStages) & 1) ^ 1, a.status, 31, abort)) { ok = false; break; }
          tc::mbar_arrive_expect_tx(kv_full + s, kv_bytes);
          for (int t = 0; t < (shared_kv ? 1 : 2); ++t) {
            const int r = (int)(it.k_row[t] + (long long)j * kKeys);
            uint8_t *dst = smem + AttnSmem::kv + (s * 4 + 2 * t) * kTile;
            tc::tma_load_3d(dst, &tk, kv_full + s, 0, r, 0);
            tc::tma_load_3d(dst + kTile, &tv, kv_full + s, 0, r, 0);
          }
        }
      }
    }
  } else if (warp == 9) {
    // ---------------- MMA issuer
    if (lane == 0) {
      const uint32_t id_s = tc::idesc_f16(kRows, kKeys);
      const uint32_t id_pv = tc::idesc_f16(kRows, kDh, true);
      int g = 0;
      int li = 0;
      bool ok = true;
      auto issue_s = [&](int t, int s) {
        const uint32_t q_addr = tc::smem_u32(smem + AttnSmem::q + t * kTile);
        const uint32_t k_addr = tc::smem_u32(smem + AttnSmem::kv + (s * 4 + (shared_kv ? 0 : 2 * t)) * kTile);
#pragma unroll
        for (int kk = 0; kk < kDh / 16; ++kk)
          tc::mma_f16(tmem + 128 * t, tc::sw128_kmajor_desc(q_addr + kk * 32), tc::sw128_kmajor_desc(k_addr + kk * 32),
                      id_s, kk != 0);
        tc::mma_commit(s_full + t);
      };
      auto issue_pv = [&](int t, int s, bool acc) {
        const uint32_t p_addr = tc::smem_u32(smem + AttnSmem::p + t * 2 * kTile);
        const uint32_t v_addr = tc::smem_u32(smem + AttnSmem::kv + (s * 4 + (shared_kv ? 0 : 2 * t) + 1) * kTile);
#pragma unroll
        for (int kk = 0; kk < kKeys / 16; ++kk) {
          const uint32_t pa = p_addr + (kk >> 2) * kTile + (kk & 3) * 32;
          tc::mma_f16(tmem + 256 + 64 * t, tc::sw128_kmajor_desc(pa), tc::sw128_mnmajor_desc(v_addr + kk * 2048),
                      id_pv, acc || kk != 0);
        }
        tc::mma_commit(pv_done + t);
      };
      for (int item = blockIdx.x; ok && item < a.items; item += gridDim.x, ++li) {
        if (!tc::mbar_wait(q_full, li & 1, a.status, 32, abort)) break;
        int s = g % kStages;
        if (!tc::mbar_wait(kv_full + s, (g / kStages) & 1, a.status, 33, abort)) break;
        tc::tc_fence_after();
        issue_s(0, s);
        issue_s(1, s);
        for (int j = 0; j < a.n_blocks; ++j, ++g) {
          s = g % kStages;
          const bool last = j + 1 == a.n_blocks;
          const int s1 = (g + 1) % kStages;
          for (int t = 0; t < 2; ++t) {
            if (!tc::mbar_wait(p_full + t, g & 1, a.status, 34, abort)) { ok = false; break; }
            if (j == 0 && !tc::mbar_wait(o_free + t, (li & 1) ^ 1, a.status, 35, abort)) { ok = false; break; }
            tc::tc_fence_after();
            issue_pv(t, s, j != 0);
            if (t == 1) tc::mma_commit(kv_empty + s);
            if (!last) {
              if (t == 0 && !tc::mbar_wait(kv_full + s1, ((g + 1) / kStages) & 1, a.status, 36, abort)) { ok = false; break; }
              tc::tc_fence_after();
              issue_s(t, s1);
            }
          }
          if (!ok) break;
        }
        if (ok) tc::mma_commit(q_empty);
      }
      tc::mma_commit(done);
      tc::mbar_wait(done, 0, a.status, 37, abort);
    }
  } else {
    // ---------------- softmax warpgroups: tile t = warp / 4, query row r of the tile
    const int t = warp >> 2;
    const int r = (warp & 3) * 32 + lane;
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + 128 * t + lane_off, tO = tmem + 256 + 64 * t + lane_off;
    uint8_t *prow = smem + AttnSmem::p + t * 2 * kTile + r * 128;
    const int prob = r >> 6;  // band axis: which of the tile's two problems
    int g = 0;
    int li = 0;
    bool ok = true;
    for (int item = blockIdx.x; ok && item < a.items; item += gridDim.x, ++li) {
      float m_run = -INFINITY, l = 0.f;
      for (int j = 0; j < a.n_blocks; ++j, ++g) {
        if (!tc::mbar_wait(s_full + t, g & 1, a.status, 38, abort)) { ok = false; break; }
        tc::tc_fence_after();
        int lo, hi;
        if (a.axis == 0) { lo = 0; hi = min(kKeys, a.n - j * kKeys); }
        else { lo = prob * 64; hi = prob * 64 + a.n; }
        const bool full_blk = lo == 0 && hi == kKeys;  // no masking needed (warp-uniform on the time axis)
        float mx = -INFINITY;
        if (full_blk) {
#pragma unroll
          for (int c = 0; c < kKeys; c += 32) {
            float v[32];
            tc::tmem_ld32(tS + c, v);
#pragma unroll
            for (int i = 0; i < 32; ++i) mx = fmaxf(mx, v[i]);
          }
        } else {
#pragma unroll
          for (int c = 0; c < kKeys; c += 32) {
            float v[32];
            tc::tmem_ld32(tS + c, v);
#pragma unroll
            for (int i = 0; i < 32; ++i)
              if (c + i >= lo && c + i < hi) mx = fmaxf(mx, v[i]);
          }
        }
        // scores arrive in log2 units (q was scaled by log2(e) / sqrt(dh) in its projection)
        const float m_cand = fmaxf(m_run, mx);
        // P_t and O_t are free once the previous block's P*V has completed
        if (j > 0 && !tc::mbar_wait(pv_done + t, (g - 1) & 1, a.status, 39, abort)) { ok = false; break; }
        const bool need = m_cand > m_run + kRescaleLog2;
        if (__any_sync(0xffffffffu, need)) {
          const float alpha = need ? ex2(m_run - m_cand) : 1.f;
          if (need) { l *= alpha; m_run = m_cand; }
          if (j > 0) {
            tc::tc_fence_after();
#pragma unroll
            for (int c = 0; c < kDh; c += 32) {
              float v[32];
              tc::tmem_ld32(tO + c, v);
#pragma unroll
              for (int i = 0; i < 32; ++i) v[i] *= alpha;
              tc::tmem_st32(tO + c, v);
            }
          }
        }
        float sum = 0.f;
#pragma unroll
        for (int c = 0; c < kKeys; c += 32) {
          float v[32];
          tc::tmem_ld32(tS + c, v);
          uint32_t h[16];
#pragma unroll
          for (int i = 0; i < 32; i += 2) {
            float p0, p1;
            // one pair in four on the FMA pipe, the rest on MUFU
            if (((i >> 1) & 3) == 3) { p0 = exp2_fma(v[i] - m_run); p1 = exp2_fma(v[i + 1] - m_run); }
            else { p0 = ex2(v[i] - m_run); p1 = ex2(v[i + 1] - m_run); }
            if (!full_blk) {
              if (!(c + i >= lo && c + i < hi)) p0 = 0.f;
              if (!(c + i + 1 >= lo && c + i + 1 < hi)) p1 = 0.f;
            }
            sum += p0 + p1;
            h[i >> 1] = pack_h2(p0, p1);
          }
          // 128-byte swizzle: 16-byte chunk index XOR (row % 8); two column blocks of 64 keys
          uint8_t *blk = prow + (c >> 6) * kTile;
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const int chunk = ((c & 63) >> 3) + q;
            *reinterpret_cast<uint4 *>(blk + ((chunk ^ (r & 7)) << 4)) =
                make_uint4(h[4 * q], h[4 * q + 1], h[4 * q + 2], h[4 * q + 3]);
          }
        }
        l += sum;
        tc::tc_fence_before();
        tc::fence_proxy_async();
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(p_full + t);
      }
      if (!ok) break;
      // the item's output: O_t / l * gate once the last P*V has completed
      if (!tc::mbar_wait(pv_done + t, (g - 1) & 1, a.status, 40, abort)) break;
      tc::tc_fence_after();
      float o[kDh];
      {
        float v[32];
        tc::tmem_ld32(tO, v);
#pragma unroll
        for (int i = 0; i < 32; ++i) o[i] = v[i];
        tc::tmem_ld32(tO + 32, v);
#pragma unroll
        for (int i = 0; i < 32; ++i) o[32 + i] = v[i];
      }
      tc::tc_fence_before();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(o_free + t);
      const Item it = item_rows(a, item);
      long long tok = -1;
      int head = 0;
      if (a.axis == 0) {
        const int pos = (it.qt0 + t) * kRows + r;
        if (pos < a.n) {
          head = (int)(it.sh % a.H);
          const long long seq = it.sh / a.H;  // b * nb + band
          tok = ((seq / a.nb) * a.T + pos) * a.nb + (seq % a.nb);
        }
      } else {
        const long long shr = it.sh + 2 * t + prob;
        const int pos = r & 63;
        if (pos < a.n && shr < a.problems) {
          head = (int)(shr % a.H);
          tok = (shr / a.H) * a.nb + pos;
        }
      }
      if (tok >= 0) {
        const float gsc = a.gate[tok * a.H + head] / l;
        __half *dst = a.o + tok * (long long)a.H * kDh + head * kDh;
#pragma unroll
        for (int d = 0; d < kDh; d += 8) {
          *reinterpret_cast<uint4 *>(dst + d) =
              make_uint4(pack_h2(o[d] * gsc, o[d + 1] * gsc), pack_h2(o[d + 2] * gsc, o[d + 3] * gsc),
                         pack_h2(o[d + 4] * gsc, o[d + 5] * gsc), pack_h2(o[d + 6] * gsc, o[d + 7] * gsc));
        }
      }
    }
  }
  tc::tc_fence_before();
  __syncthreads();
  if (warp == 8) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, 512);
  }
}

int g_num_sms = 0;

}  // namespace

bool make_tmap_f16(CUtensorMap *map, const void *base, unsigned long long d0, unsigned long long d1,
                   unsigned long long d2, unsigned long long s1, unsigned long long s2, unsigned box1,
                   unsigned box2);

bool attention_tc_supported(int dh) { return dh == kDh; }

bool attention_tc_init() {
  int dev = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&g_num_sms, cudaDevAttrMultiProcessorCount, dev);
  return cudaFuncSetAttribute(attn_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              (int)(AttnSmem::total + 1024)) == cudaSuccess;
}

bool launch_attention_tc(const __half *q, const __half *k, const __half *v, const float *gate, __half *o, int B,
                         int T, int nb, int H, int axis, int n_pad, unsigned *status, cudaStream_t st) {
  AttnArgs a;
  a.gate = gate;
  a.o = o;
  a.status = status;
  a.B = B; a.T = T; a.nb = nb; a.H = H; a.axis = axis; a.n_pad = n_pad;
  a.n = axis == 0 ? T : nb;
  a.q_tiles = (a.n + kRows - 1) / kRows;
  long long rows;
  if (axis == 0) {
    a.problems = (long long)B * nb * H;
    a.pairs = (a.q_tiles + 1) / 2;
    a.items = (int)(a.problems * a.pairs);
    a.n_blocks = (a.n + kKeys - 1) / kKeys;
  } else {
    a.problems = (long long)B * T * H;
    a.pairs = 0;
    a.items = (int)((a.problems + 3) / 4);
    a.n_blocks = 1;
  }
  rows = a.problems * n_pad;
  CUtensorMap tq, tk, tv;
  if (!make_tmap_f16(&tq, q, kDh, rows, 1, kDh, rows * kDh, kRows, 1) ||
      !make_tmap_f16(&tk, k, kDh, rows, 1, kDh, rows * kDh, kKeys, 1) ||
      !make_tmap_f16(&tv, v, kDh, rows, 1, kDh, rows * kDh, kKeys, 1))
    return false;
  const size_t smem = AttnSmem::total + 1024;
  const int grid = (int)std::min<long long>(a.items, g_num_sms > 0 ? g_num_sms : 148);
  attn_tc_kernel<<<grid, kThreads, smem, st>>>(tq, tk, tv, a);
  return true;
}

}  // namespace mrf
