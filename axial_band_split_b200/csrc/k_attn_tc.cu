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
// One CTA = one tile of 128 query rows.  Time axis: the rows are 128 consecutive frames
// of one (band, head) sequence and the keys stream in blocks of 128.  Band axis (n <= 64):
// the tile holds two 64-row problems and a single 128-key block, masked block-diagonally.
//
// Warps 0-3: softmax (one query row per thread), warp 4: TMA, warp 5: MMA issue.
// Tensor memory: S (128 columns) and P*V of the current block (64 columns).
#include <cmath>

#include "mrf_internal.h"
#include "tc_ptx.cuh"

namespace mrf {

namespace {

constexpr int kDh = 64, kRows = 128, kKeys = 128, kKvStages = 2;
constexpr int kTile = kRows * kDh * 2;  // 16 KB: one 128 x 64 fp16 tile
constexpr int kThreads = 192;

struct AttnSmem {
  static constexpr int q = 0;
  static constexpr int k = q + kTile;
  static constexpr int v = k + kKvStages * kTile;
  static constexpr int p = v + kKvStages * kTile;   // 128 x 128 fp16 = two 16 KB column blocks
  static constexpr int bar = p + 2 * kTile;
  static constexpr int total = bar + 256;
};

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ void fence_proxy_async() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ uint32_t pack_h2(float a, float b) {
  __half2 h = __floats2half2_rn(a, b);
  return *reinterpret_cast<uint32_t *>(&h);
}

struct AttnArgs {
  const float *gate;
  __half *o;
  unsigned *status;
  int B, T, nb, H, axis, n_pad, n, q_tiles;
  long long problems;
};

__global__ void __launch_bounds__(kThreads, 1)
    attn_tc_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                   const __grid_constant__ CUtensorMap tv, const AttnArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + AttnSmem::bar);
  uint64_t *q_full = bars;
  uint64_t *kv_full = bars + 1;                 // [2]
  uint64_t *kv_empty = bars + 3;                // [2]
  uint64_t *s_full = bars + 5, *s_free = bars + 6;
  uint64_t *p_full = bars + 7;
  uint64_t *pv_full = bars + 8, *pv_free = bars + 9;
  uint64_t *done = bars + 10;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 11);
  __shared__ int abort_flag;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // tile -> rows of q and of the keys
  long long q_row0, k_row0;
  int n_blocks;
  long long sh;  // (sequence * H + head) of the first problem
  if (a.axis == 0) {
    sh = blockIdx.x / a.q_tiles;
    const int qt = blockIdx.x % a.q_tiles;
    q_row0 = sh * a.n_pad + (long long)qt * kRows;
    k_row0 = sh * a.n_pad;
    n_blocks = (a.n + kKeys - 1) / kKeys;
  } else {
    sh = 2LL * blockIdx.x;
    q_row0 = sh * a.n_pad;  // n_pad == 64
    k_row0 = q_row0;
    n_blocks = 1;
  }

  if (threadIdx.x == 0) {
    abort_flag = 0;
    tc::mbar_init(q_full, 1);
    for (int s = 0; s < kKvStages; ++s) { tc::mbar_init(kv_full + s, 1); tc::mbar_init(kv_empty + s, 1); }
    tc::mbar_init(s_full, 1);
    tc::mbar_init(s_free, 4);
    tc::mbar_init(p_full, 4);
    tc::mbar_init(pv_full, 1);
    tc::mbar_init(pv_free, 4);
    tc::mbar_init(done, 1);
    tc::fence_barrier_init();
  }
  if (warp == 4) {
    tc::tmem_alloc(tmem_slot, 256);
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tS = tmem, tPV = tmem + 128;
  volatile int *abort = &abort_flag;

  if (warp == 4) {
    if (lane == 0) {
      tc::mbar_arrive_expect_tx(q_full, kTile);
      tc::tma_load_3d(smem + AttnSmem::q, &tq, q_full, 0, (int)q_row0, 0);
      for (int j = 0; j < n_blocks; ++j) {
        const int s = j % kKvStages;
        const uint32_t ph = (j / kKvStages) & 1;
        if (!tc::mbar_wait(kv_empty + s, ph ^ 1, a.status, 20, abort)) break;
        tc::mbar_arrive_expect_tx(kv_full + s, 2 * kTile);
        const int r = (int)(k_row0 + (long long)j * kKeys);
        tc::tma_load_3d(smem + AttnSmem::k + s * kTile, &tk, kv_full + s, 0, r, 0);
        tc::tma_load_3d(smem + AttnSmem::v + s * kTile, &tv, kv_full + s, 0, r, 0);
      }
    }
  } else if (warp == 5) {
    if (lane == 0) {
      const uint32_t id_s = tc::idesc_f16(kRows, kKeys);
      const uint32_t id_pv = tc::idesc_f16(kRows, kDh, true);
      const uint32_t q_addr = tc::smem_u32(smem + AttnSmem::q);
      const uint32_t p_addr = tc::smem_u32(smem + AttnSmem::p);
      bool ok = tc::mbar_wait(q_full, 0, a.status, 21, abort);
      for (int j = 0; ok && j < n_blocks; ++j) {
        const int s = j % kKvStages;
        const uint32_t ph = (j / kKvStages) & 1;
        if (!tc::mbar_wait(kv_full + s, ph, a.status, 22, abort)) break;
        if (!tc::mbar_wait(s_free, (j & 1) ^ 1, a.status, 23, abort)) break;
        tc::tc_fence_after();
        const uint32_t k_addr = tc::smem_u32(smem + AttnSmem::k + s * kTile);
#pragma unroll
        for (int kk = 0; kk < kDh / 16; ++kk)
          tc::mma_f16(tS, tc::sw128_kmajor_desc(q_addr + kk * 32), tc::sw128_kmajor_desc(k_addr + kk * 32), id_s,
                      kk != 0);
        tc::mma_commit(s_full);
        if (!tc::mbar_wait(p_full, j & 1, a.status, 24, abort)) break;
        if (!tc::mbar_wait(pv_free, (j & 1) ^ 1, a.status, 25, abort)) break;
        tc::tc_fence_after();
        const uint32_t v_addr = tc::smem_u32(smem + AttnSmem::v + s * kTile);
#pragma unroll
        for (int kk = 0; kk < kKeys / 16; ++kk) {
          const uint32_t pa = p_addr + (kk >> 2) * kTile + (kk & 3) * 32;
          tc::mma_f16(tPV, tc::sw128_kmajor_desc(pa), tc::sw128_mnmajor_desc(v_addr + kk * 2048), id_pv, kk != 0);
        }
        tc::mma_commit(pv_full);
        tc::mma_commit(kv_empty + s);
      }
      tc::mma_commit(done);
      tc::mbar_wait(done, 0, a.status, 26, abort);
    }
  } else {
    // ---------------- softmax warps: thread = query row r of the tile
    const int r = warp * 32 + lane;
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
    const float sl2 = 1.4426950408889634f * rsqrtf((float)kDh);
    float m = -INFINITY, l = 0.f;
    float o[kDh];
#pragma unroll
    for (int d = 0; d < kDh; ++d) o[d] = 0.f;
    uint8_t *prow = smem + AttnSmem::p + r * 128;
    const int prob = r >> 6;  // band axis: which of the two problems
    bool ok = true;
    for (int j = 0; j < n_blocks; ++j) {
      if (!tc::mbar_wait(s_full, j & 1, a.status, 27, abort)) { ok = false; break; }
      tc::tc_fence_after();
      // valid keys of this block for this row: [lo, hi)
      int lo, hi;
      if (a.axis == 0) { lo = 0; hi = min(kKeys, a.n - j * kKeys); }
      else { lo = prob * 64; hi = prob * 64 + a.n; }
      // pass 1: row max
      float mx = -INFINITY;
#pragma unroll
      for (int c = 0; c < kKeys; c += 32) {
        float v[32];
        tc::tmem_ld32(tS + lane_off + c, v);
#pragma unroll
        for (int i = 0; i < 32; ++i)
          if (c + i >= lo && c + i < hi) mx = fmaxf(mx, v[i]);
      }
      const float m_new = fmaxf(m, mx * sl2);
      const float alpha = ex2(m - m_new);
      // pass 2: p = 2^(s*scale*log2e - m), row sum, P (fp16) into shared memory
      float sum = 0.f;
#pragma unroll
      for (int c = 0; c < kKeys; c += 32) {
        float v[32];
        tc::tmem_ld32(tS + lane_off + c, v);
        uint32_t h[16];
#pragma unroll
        for (int i = 0; i < 32; i += 2) {
          const float p0 = (c + i >= lo && c + i < hi) ? ex2(v[i] * sl2 - m_new) : 0.f;
          const float p1 = (c + i + 1 >= lo && c + i + 1 < hi) ? ex2(v[i + 1] * sl2 - m_new) : 0.f;
          sum += p0 + p1;
          h[i >> 1] = pack_h2(p0, p1);
        }
        // 128-byte swizzle: 16-byte chunk index XOR (row % 8), two column blocks of 64 keys
        uint8_t *blk = prow + (c >> 6) * kTile;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int chunk = ((c & 63) >> 3) + q;
          uint4 u = make_uint4(h[4 * q], h[4 * q + 1], h[4 * q + 2], h[4 * q + 3]);
          *reinterpret_cast<uint4 *>(blk + ((chunk ^ (r & 7)) << 4)) = u;
        }
      }
      tc::tc_fence_before();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(s_free);
      l = l * alpha + sum;
      m = m_new;
      fence_proxy_async();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(p_full);
      if (!tc::mbar_wait(pv_full, j & 1, a.status, 28, abort)) { ok = false; break; }
      tc::tc_fence_after();
#pragma unroll
      for (int c = 0; c < kDh; c += 32) {
        float v[32];
        tc::tmem_ld32(tPV + lane_off + c, v);
#pragma unroll
        for (int i = 0; i < 32; ++i) o[c + i] = o[c + i] * alpha + v[i];
      }
      tc::tc_fence_before();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(pv_free);
    }
    // epilogue: o / l * gate -> token-major fp16
    if (ok) {
      long long tok = -1;
      int head = 0;
      if (a.axis == 0) {
        const int pos = (blockIdx.x % a.q_tiles) * kRows + r;
        if (pos < a.n) {
          head = (int)(sh % a.H);
          const long long seq = sh / a.H;  // b * nb + band
          const long long b = seq / a.nb, band = seq % a.nb;
          tok = (b * a.T + pos) * a.nb + band;
        }
      } else {
        const long long shr = sh + prob;
        const int pos = r & 63;
        if (pos < a.n && shr < a.problems) {
          head = (int)(shr % a.H);
          const long long bt = shr / a.H;
          tok = bt * a.nb + pos;
        }
      }
      if (tok >= 0) {
        const float g = a.gate[tok * a.H + head] / l;
        __half *dst = a.o + tok * (long long)a.H * kDh + head * kDh;
#pragma unroll
        for (int d = 0; d < kDh; d += 8) {
          uint4 u = make_uint4(pack_h2(o[d] * g, o[d + 1] * g), pack_h2(o[d + 2] * g, o[d + 3] * g),
                               pack_h2(o[d + 4] * g, o[d + 5] * g), pack_h2(o[d + 6] * g, o[d + 7] * g));
          *reinterpret_cast<uint4 *>(dst + d) = u;
        }
      }
    }
  }
  tc::tc_fence_before();
  __syncthreads();
  if (warp == 4) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, 256);
  }
}

}  // namespace

bool make_tmap_f16(CUtensorMap *map, const void *base, unsigned long long d0, unsigned long long d1,
                   unsigned long long d2, unsigned long long s1, unsigned long long s2, unsigned box1,
                   unsigned box2);

bool attention_tc_supported(int dh) { return dh == kDh; }

bool launch_attention_tc(const __half *q, const __half *k, const __half *v, const float *gate, __half *o, int B,
                         int T, int nb, int H, int axis, int n_pad, unsigned *status, cudaStream_t st) {
  AttnArgs a;
  a.gate = gate;
  a.o = o;
  a.status = status;
  a.B = B; a.T = T; a.nb = nb; a.H = H; a.axis = axis; a.n_pad = n_pad;
  a.n = axis == 0 ? T : nb;
  a.q_tiles = (a.n + kRows - 1) / kRows;
  long long grid;
  long long rows;
  if (axis == 0) {
    a.problems = (long long)B * nb * H;
    grid = a.problems * a.q_tiles;
    rows = a.problems * n_pad;
  } else {
    a.problems = (long long)B * T * H;
    grid = (a.problems + 1) / 2;
    rows = a.problems * n_pad;
  }
  CUtensorMap tq, tk, tv;
  if (!make_tmap_f16(&tq, q, kDh, rows, 1, kDh, rows * kDh, kRows, 1) ||
      !make_tmap_f16(&tk, k, kDh, rows, 1, kDh, rows * kDh, kKeys, 1) ||
      !make_tmap_f16(&tv, v, kDh, rows, 1, kDh, rows * kDh, kKeys, 1))
    return false;
  const size_t smem = AttnSmem::total + 1024;
  attn_tc_kernel<<<(unsigned)grid, kThreads, smem, st>>>(tq, tk, tv, a);
  return true;
}

bool attention_tc_init() {
  return cudaFuncSetAttribute(attn_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              (int)(AttnSmem::total + 1024)) == cudaSuccess;
}

}  // namespace mrf
