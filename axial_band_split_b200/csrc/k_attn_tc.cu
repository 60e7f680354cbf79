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
// q, k, v are read from the token-major projection output [token][q | k | v | gates]
// through 4-D tensor maps (d, head, band, frame).
// Persistent CTAs; a work item is two 128-row query tiles t = 0, 1 processed in ping-pong:
//   time axis - two consecutive query tiles of one (band, head) sequence; the keys stream
//               in blocks of 128 and each K/V block serves both tiles;
//   band axis - each tile holds the band sequences of two frames for one head (64 rows
//               each, bands past n read as zeros) with their own single K/V block, masked
//               block-diagonally.
// Warps 0-3 and 4-7: softmax of tile 0 and tile 1 (one query row per thread, the row's
// live scores in registers: 128 on the time axis, the row's own 64-key half on the band
// axis); warp 8: TMA; warps 9 and 10: MMA issue for tile 0 and tile 1; warp 11 idle.  The third warpgroup gives
// registers up to the two softmax warpgroups (setmaxnreg).
// Tensor memory (512 columns): S_t at 128 t, O_t at 256 + 64 t, and P_t (the softmax's
// fp16 probabilities, two per 32-bit column) at 384 + 64 t, which the P*V MMA reads as its
// A operand straight from tensor memory.
// O accumulates in tensor memory across key blocks; a row's running max is raised (and
// its O row rescaled in place) only when a block's max exceeds it by more than 2^8, so
// the unnormalised p stay below 256 and most blocks need no correction.
#include <cuda_bf16.h>

#include <cmath>

#include "gemm_tc.cuh"
#include "mrf_internal.h"
#include "tc_ptx.cuh"

namespace mrf {

namespace {

constexpr int kDh = 64, kRows = 128, kKeys = 128;
// K/V ring: 8 tiles of 16 KB, filled block by block in order.  A key block takes one K and
// one V tile when both query tiles share the keys (two tiles of one time-axis sequence) and
// a K and a V tile per query tile otherwise (band axis; time-axis items that pair the odd
// last tiles of two sequences).  At most kMaxStages blocks are in flight, each with its own
// full/empty barrier pair.
constexpr int kMaxStages = 5;
static_assert(kKeys == 128, "the softmax reads a score row as two 64-column halves");
constexpr int kTile = kRows * kDh * 2;  // 16 KB: one 128 x 64 fp16 tile
constexpr int kThreads = 384;
// register split: launched at 168 per thread (384 threads, one CTA per SM); the TMA/MMA
// warpgroup drops to kRegsIo and the softmax warpgroups rise to kRegsSoftmax, within the
// launch's total: 2 * 128 * 208 + 128 * 72 = 62464 <= 384 * 168 = 64512.  (An increase
// beyond what the launch holds would wait forever; the init checks the launch count.)
constexpr int kRegsLaunch = 168, kRegsSoftmax = 208, kRegsIo = 72;
static_assert(2 * 128 * kRegsSoftmax + 128 * kRegsIo <= kThreads * kRegsLaunch, "register split over budget");
constexpr float kRescaleLog2 = 8.f;


// q and k are kQA 64-wide atoms deep (dim_head 64 or 128; v is 64 wide either way): each query
// tile takes kQA 16 KB tiles, a key block kQA K tiles and one V tile.  With 64-deep q there are
// two q buffers (items alternate between them, so the next item's queries load while this item
// runs: on the band axis an item is a single key block and would otherwise wait for them); with
// 128-deep q one, as the doubled tiles leave no room for a second.
template <int kQA>
struct AttnSmem {
  static constexpr int qbufs = kQA == 1 ? 2 : 1;           // q buffers
  static constexpr int ring = 8;                           // K/V ring tiles
  static constexpr int q = 0;                              // [qbufs][2 query tiles][kQA atoms]
  static constexpr int kv = q + qbufs * 2 * kQA * kTile;   // ring of 16 KB tiles
  static constexpr int ostage = kv + ring * kTile;         // [8 warps] 32 rows x 128 B of output
  static constexpr int bar = ostage + 8 * 4096;
  static constexpr int total = bar + 256;
};

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// max of three (one instruction on sm_100)
__device__ __forceinline__ float max3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// packed pair add (one f32x2 instruction)
__device__ __forceinline__ float2 add2(float2 a, float2 b) {
  float2 r;
  asm("{\n\t.reg .b64 ra, rb, rc;\n\t"
      "mov.b64 ra, {%2, %3};\n\t"
      "mov.b64 rb, {%4, %5};\n\t"
      "add.f32x2 rc, ra, rb;\n\t"
      "mov.b64 {%0, %1}, rc;\n\t}"
      : "=f"(r.x), "=f"(r.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return r;
}

// Consecutive fp32 columns of this thread's TMEM lane.  The wait takes the destination
// registers as operands so no use can be scheduled above it.
#define MRF_R8(b) "=r"(r[b]), "=r"(r[b + 1]), "=r"(r[b + 2]), "=r"(r[b + 3]), "=r"(r[b + 4]), "=r"(r[b + 5]), \
                  "=r"(r[b + 6]), "=r"(r[b + 7])
#define MRF_P8(b) "+r"(r[b]), "+r"(r[b + 1]), "+r"(r[b + 2]), "+r"(r[b + 3]), "+r"(r[b + 4]), "+r"(r[b + 5]), \
                  "+r"(r[b + 6]), "+r"(r[b + 7])
// N (64 or 128) consecutive fp32 columns: N / 32 loads, one wait.
template <int N>
__device__ __forceinline__ void tmem_ldn(uint32_t taddr, float (&v)[N]) {
  static_assert(N == 64 || N == 128, "64 or 128 columns");
  uint32_t r[128];
#pragma unroll
  for (int c = 0; c < N; c += 32) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
        "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
        : MRF_R8(c), MRF_R8(c + 8), MRF_R8(c + 16), MRF_R8(c + 24)
        : "r"(taddr + c));
  }
  asm volatile("tcgen05.wait::ld.sync.aligned;" : MRF_P8(0), MRF_P8(8), MRF_P8(16), MRF_P8(24) : : "memory");
  asm volatile("" : MRF_P8(32), MRF_P8(40), MRF_P8(48), MRF_P8(56));
  if (N == 128) {
    asm volatile("" : MRF_P8(64), MRF_P8(72), MRF_P8(80), MRF_P8(88));
    asm volatile("" : MRF_P8(96), MRF_P8(104), MRF_P8(112), MRF_P8(120));
  }
#pragma unroll
  for (int i = 0; i < N; ++i) v[i] = __uint_as_float(r[i]);
}
#undef MRF_R8
#undef MRF_P8


// 4 consecutive 32-bit TMEM columns of this thread's lane; no wait.  (Four-register
// pieces: a 16-register source group must sit in one aligned register block, which the
// allocator could only provide by spilling.)
__device__ __forceinline__ void tmem_st4(uint32_t taddr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x4.b32 [%0], {%1, %2, %3, %4};" ::"r"(taddr), "r"(a), "r"(b), "r"(c),
               "r"(d)
               : "memory");
}

// D (+)= A * B with A (M x K, fp16, two values per 32-bit column) in tensor memory.
__device__ __forceinline__ void mma_f16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                          bool accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate ? 1u : 0u));
}

// 5-D bulk tensor store from shared memory (one bulk group per call site commit).
__device__ __forceinline__ void tma_store_5d(const CUtensorMap *map, const void *src, int c0, int c1, int c2,
                                             int c3, int c4) {
  asm volatile("cp.async.bulk.tensor.5d.global.shared::cta.bulk_group [%0, {%2, %3, %4, %5, %6}], [%1];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(tc::smem_u32(src)), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(c4)
               : "memory");
}

// Two floats as one pair of the schedule's 16-bit type (fp16, or bf16 with kBF).
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

template <bool kBF>
__device__ __forceinline__ float to_float16b(unsigned short v) {
  if constexpr (kBF) return __uint_as_float((unsigned)v << 16);
  else return __half2float(__ushort_as_half(v));
}

struct AttnArgs {
  const __half *qkv;   // token-major [tok][ld]: q | k | v | sigmoid gates
  __half *o;
  unsigned *status;
  int B, T, nb, H, axis, ld, n, q_tiles, pairs, items, n_blocks, BT;
  int gate_col;  // column of head 0's gate in a projection row (after q, k and v)
  // odd last query tiles run alone (one per item, the item's second tile idle) instead of paired
  // across two sequences: with 128-deep q and k a block with separate keys would fill 6 of the
  // 8 ring tiles, and the MMA issuer needs the next block before it releases the current one
  int split_odd;
  int S;  // time axis: sequences (b, band, head)
};

// Query tile t of an item.  Tensor-map coordinates (d, head, band, frame): the tile's
// queries start at frame frame0 of (head, band) and its key block j at frame kv0 + j * 128.
// Time axis: a tile is 128 frames of one (band, head) sequence; an item holds either two
// consecutive tiles of one sequence (shared keys) or the odd last tiles of two sequences
// (mixed: separate keys; with an odd sequence count the last item's tile 1 is idle).
// Band axis: tile t covers frames frame0 and frame0 + 1, bands 0..63 of each (bands past
// nb read as zeros), with its own keys.
struct TileC {
  int head, band, b, qt, frame0, kv0;
  bool valid;
};

// Time-axis items come in groups of two sequences 2k, 2k + 1 (sequence index
// ((b * nb) + band) * H + head): the pairs of sequence 2k, those of 2k + 1, then (odd tile
// count) the item of their two last tiles, so all items reading a sequence's keys run close
// together and find them in L2.  With an odd sequence count the last group has one sequence.
struct ItemPos {
  int seq, pair;  // shared: sequence and pair index; mixed: first sequence, pair = -1;
                  // a lone odd last tile (split_odd): its sequence, pair = -2
};

__device__ __forceinline__ ItemPos item_pos(const AttnArgs &a, int item) {
  const int odd_items = (a.q_tiles & 1) ? (a.split_odd ? 2 : 1) : 0;
  const int gs = 2 * a.pairs + odd_items;
  const int grp = item / gs, r = item - grp * gs;
  const int n_seq = 2 * grp + 1 < a.S ? 2 : 1;
  ItemPos ip;
  if (r < n_seq * a.pairs) {
    ip.seq = 2 * grp + r / a.pairs;
    ip.pair = r % a.pairs;
  } else if (a.split_odd) {
    ip.seq = 2 * grp + (r - n_seq * a.pairs);
    ip.pair = -2;
  } else {
    ip.seq = 2 * grp;
    ip.pair = -1;
  }
  return ip;
}

__device__ __forceinline__ bool item_mixed(const AttnArgs &a, int item) {
  return a.axis != 0 || item_pos(a, item).pair == -1;
}

__device__ __forceinline__ TileC tile_coords(const AttnArgs &a, int item, int t) {
  TileC c;
  if (a.axis == 0) {
    const ItemPos ip = item_pos(a, item);
    int seq, qt;
    c.valid = true;
    if (ip.pair >= 0) {
      seq = ip.seq;
      qt = 2 * ip.pair + t;
    } else if (ip.pair == -2) {
      seq = ip.seq;  // a lone odd last tile: tile 1 repeats it on the same keys and stores nothing
      qt = a.q_tiles - 1;
      c.valid = t == 0;
    } else {
      seq = ip.seq + t;
      if (seq >= a.S) { seq = a.S - 1; c.valid = false; }
      qt = a.q_tiles - 1;
    }
    c.head = seq % a.H;
    const int bb = seq / a.H;
    c.band = bb % a.nb;
    c.b = bb / a.nb;
    c.qt = qt;
    c.kv0 = c.b * a.T;
    c.frame0 = c.kv0 + qt * kRows;
  } else {
    c.head = item % a.H;
    c.band = 0;
    c.b = 0;
    c.qt = 0;
    c.frame0 = c.kv0 = 4 * (item / a.H) + 2 * t;
    c.valid = true;
  }
  return c;
}

// Max of a score row: four independent max3 chains, joined at the end.
template <int NC>
__device__ __forceinline__ float row_max(const float (&sv)[NC]) {
  constexpr int Q = NC / 4;
  float ma = sv[0], mb = sv[Q], mc = sv[2 * Q], md = sv[3 * Q];
#pragma unroll
  for (int i = 1; i < Q; i += 2) {
    const int i2 = i + 1 < Q ? i + 1 : i;
    ma = max3(ma, sv[i], sv[i2]);
    mb = max3(mb, sv[Q + i], sv[Q + i2]);
    mc = max3(mc, sv[2 * Q + i], sv[2 * Q + i2]);
    md = max3(md, sv[3 * Q + i], sv[3 * Q + i2]);
  }
  return fmaxf(fmaxf(ma, mb), fmaxf(mc, md));
}

// One key block of one query row: scores from tensor memory (log2 units: q was scaled by
// log2(e) / sqrt(dh) in its projection), the running max and sum, p = 2^(s - m) into P as
// 16-bit pairs, and the O row rescaled in place when its max was raised.  NC live score columns
// at tS (columns >= hi are masked); P's matching NC / 2 columns at tP.  Returns false if a
// wait timed out.
//
template <int NC, bool kBF>
__device__ __forceinline__ bool softmax_block(uint32_t tS, uint32_t tP, uint32_t tO, int hi, float &m_run, float &l,
                                              bool wait_pv, uint64_t *pv_done, uint32_t pv_parity,
                                              uint64_t *s_free, uint64_t *p_full, int lane, unsigned *status,
                                              volatile int *abort) {
  float sv[NC];
  tmem_ldn<NC>(tS, sv);
  // S_t may now take the next block's scores
  tc::tc_fence_before();
  __syncwarp();
  if (lane == 0) tc::mbar_arrive(s_free);
  if (hi < NC) {
#pragma unroll
    for (int i = 0; i < NC; ++i)
      if (i >= hi) sv[i] = -INFINITY;
  }
  // the block's max; for the item's first block it is the running max (l is still 0)
  const bool first = !wait_pv;
  const float bm = row_max<NC>(sv);
  bool need = false;
  float alpha = 1.f;
  if (first) {
    m_run = bm;
  } else {
    need = bm > m_run + kRescaleLog2;
    if (need) {
      alpha = ex2(m_run - bm);
      l *= alpha;
      m_run = bm;
    }
  }
  // p = 2^(s - m): pairs through packed f32x2 subtract, exponentials on MUFU, packed to 16-bit
  // pairs (the P*V MMA's A operand), the row sum in four f32x2 chains.  This needs neither P_t
  // nor O_t, so it runs before the wait for the previous block's P*V, which then overlaps it.
  uint32_t pk[NC / 2];
  float2 sa = make_float2(0.f, 0.f), sb = sa, sc = sa, sd = sa;
  const float2 negm = make_float2(-m_run, -m_run);
#pragma unroll
  for (int i = 0; i < NC; i += 8) {
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const float2 d = add2(make_float2(sv[i + 2 * u], sv[i + 2 * u + 1]), negm);
      const float2 pp = make_float2(ex2(d.x), ex2(d.y));
      switch (u) {
        case 0: sa = add2(sa, pp); break;
        case 1: sb = add2(sb, pp); break;
        case 2: sc = add2(sc, pp); break;
        default: sd = add2(sd, pp); break;
      }
      pk[(i >> 1) + u] = pack_h2<kBF>(pp.x, pp.y);
    }
  }
  const float2 s4 = add2(add2(sa, sb), add2(sc, sd));
  // P_t and O_t are free once the previous block's P*V has completed
  if (wait_pv && !tc::mbar_wait(pv_done, pv_parity, status, 39, abort)) return false;
  tc::tc_fence_after();
  const bool any_need = __any_sync(0xffffffffu, need);
  // P into tensor memory, two 16-bit values per column, four columns (8 keys) per store
#pragma unroll
  for (int i = 0; i < NC / 2; i += 4) tmem_st4(tP + i, pk[i], pk[i + 1], pk[i + 2], pk[i + 3]);
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
  // O row rescaled in place when this row's max was raised
  if (any_need) {
#pragma unroll
    for (int c = 0; c < kDh; c += 32) {
      float v[32];
      tc::tmem_ld32(tO + c, v);
#pragma unroll
      for (int i = 0; i < 32; ++i) v[i] *= alpha;
      tc::tmem_st32(tO + c, v);
    }
  }
  l += s4.x + s4.y;
  tc::tc_fence_before();
  __syncwarp();
  if (lane == 0) tc::mbar_arrive(p_full);
  return true;
}

template <bool kBF, int kQA>
__global__ void __launch_bounds__(kThreads, 1)
    attn_tc_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                   const __grid_constant__ CUtensorMap tv, const __grid_constant__ CUtensorMap to,
                   const AttnArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + AttnSmem<kQA>::bar);
  uint64_t *q_full = bars + 26, *q_empty = bars + 28;  // [qbufs] each
  uint64_t *kv_full = bars + 2;     // [kMaxStages]
  uint64_t *kv_empty = bars + 8;    // [kMaxStages]
  uint64_t *s_full = bars + 14;     // [2]
  uint64_t *p_full = bars + 16;     // [2]
  uint64_t *pv_done = bars + 18;    // [2]
  uint64_t *o_free = bars + 20;     // [2]
  uint64_t *s_free = bars + 22;     // [2]
  uint64_t *done = bars + 24;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 30);
  constexpr int kQBufs = AttnSmem<kQA>::qbufs;
  __shared__ int abort_flag;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    abort_flag = 0;
    for (int b = 0; b < kQBufs; ++b) {
      tc::mbar_init(q_full + b, 1);
      tc::mbar_init(q_empty + b, 2);  // released by both tiles' MMA issuers
    }
    for (int s = 0; s < kMaxStages; ++s) { tc::mbar_init(kv_full + s, 1); tc::mbar_init(kv_empty + s, 2); }
    for (int t = 0; t < 2; ++t) {
      tc::mbar_init(s_full + t, 1);
      tc::mbar_init(s_free + t, 4);
      tc::mbar_init(p_full + t, 4);
      tc::mbar_init(pv_done + t, 1);
      tc::mbar_init(o_free + t, 4);
    }
    tc::mbar_init(done, 2);
    tc::fence_barrier_init();
  }
  if (warp == 8) tc::tmem_alloc(tmem_slot, 512);
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  volatile int *abort = &abort_flag;
  // the prologue overlaps the previous kernel's tail; q, k, v and the gates are its output
  tc::griddep_wait();
  tc::griddep_launch_dependents();
  if (warp >= 8) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsIo));
  if (warp == 8) {
    // ---------------- TMA producer
    if (lane == 0) {
      int g = 0;              // key blocks loaded so far
      int oldest = 0;         // oldest block whose ring tiles are not known to be free
      int used = 0;           // ring tiles held by blocks oldest .. g - 1
      int ptr = 0;            // next ring tile
      int held[kMaxStages];   // ring tiles of the block in each slot
      int li = 0;
      bool ok = true;
      for (int item = blockIdx.x; ok && item < a.items; item += gridDim.x, ++li) {
        const TileC c0 = tile_coords(a, item, 0), c1 = tile_coords(a, item, 1);
        const bool mixed = item_mixed(a, item);
        // item li's queries go to buffer li % kQBufs (its (li / kQBufs)-th use)
        const int qb = li % kQBufs;
        uint8_t *qbuf = smem + AttnSmem<kQA>::q + qb * 2 * kQA * kTile;
        if (!tc::mbar_wait(q_empty + qb, ((li / kQBufs) & 1) ^ 1, a.status, 30, abort)) break;
        tc::mbar_arrive_expect_tx(q_full + qb, 2 * kQA * kTile);
#pragma unroll
        for (int qa = 0; qa < kQA; ++qa) {
          tc::tma_load_4d(qbuf + qa * kTile, &tq, q_full + qb, 64 * qa, c0.head, c0.band, c0.frame0);
          tc::tma_load_4d(qbuf + (kQA + qa) * kTile, &tq, q_full + qb, 64 * qa, c1.head, c1.band,
                          c1.frame0);
        }
        const int need = (kQA + 1) * (mixed ? 2 : 1);
        for (int j = 0; j < a.n_blocks; ++j, ++g) {
          // a free slot and `need` free ring tiles: release the oldest blocks in order
          while (ok && (g - oldest >= kMaxStages || used + need > AttnSmem<kQA>::ring)) {
            const int so = oldest % kMaxStages;
            if (!tc::mbar_wait(kv_empty + so, (oldest / kMaxStages) & 1, a.status, 31, abort)) ok = false;
            used -= held[so];
            ++oldest;
          }
          if (!ok) break;
          const int s = g % kMaxStages;
          held[s] = need;
          tc::mbar_arrive_expect_tx(kv_full + s, need * kTile);
#pragma unroll
          for (int t = 0; t < 2; ++t) {
            if (t == 1 && !mixed) break;
            const TileC &c = t == 0 ? c0 : c1;
            const int f = c.kv0 + j * kKeys;
            const int b0 = ptr + (kQA + 1) * t;  // this tile's K atoms, then its V
#pragma unroll
            for (int qa = 0; qa < kQA; ++qa)
              tc::tma_load_4d(smem + AttnSmem<kQA>::kv + ((b0 + qa) % AttnSmem<kQA>::ring) * kTile, &tk, kv_full + s,
                              64 * qa, c.head, c.band, f);
            tc::tma_load_4d(smem + AttnSmem<kQA>::kv + ((b0 + kQA) % AttnSmem<kQA>::ring) * kTile, &tv, kv_full + s, 0,
                            c.head, c.band, f);
          }
          ptr = (ptr + need) % AttnSmem<kQA>::ring;
          used += need;
        }
      }
    }
  } else if (warp == 9 || warp == 10) {
    // ---------------- MMA issuers: warp 9 + t issues tile t's MMAs, so neither tile's S or
    // P*V waits behind the other tile's softmax (the tensor core queues both streams)
    const int t = warp - 9;
    if (lane == 0) {
      const uint32_t id_s = tc::idesc_f16(kRows, kKeys, false, kBF);
      const uint32_t id_pv = tc::idesc_f16(kRows, kDh, true, kBF);
      int g = 0;    // key blocks consumed so far
      int ptr = 0;  // ring tile of the next item's first block (the producer's order)
      int li = 0;
      bool ok = true;
      bool mixed = false;
      int qb = 0;  // the item's q buffer
      // block at ring tile `base`: tile t's K atoms at base (+ (kQA + 1) t when the tiles have
      // separate keys), its V after them
      auto kv_tile = [&](int base, int t, int which) {
        return smem + AttnSmem<kQA>::kv + ((base + (mixed ? (kQA + 1) * t : 0) + which) % AttnSmem<kQA>::ring) * kTile;
      };
      auto issue_s = [&](int t, int base) {
#pragma unroll
        for (int kk = 0; kk < 4 * kQA; ++kk) {
          const uint32_t q_addr =
              tc::smem_u32(smem + AttnSmem<kQA>::q + ((qb * 2 + t) * kQA + kk / 4) * kTile);
          const uint32_t k_addr = tc::smem_u32(kv_tile(base, t, kk / 4));
          tc::mma_f16(tmem + 128 * t, tc::sw128_kmajor_desc(q_addr + (kk % 4) * 32),
                      tc::sw128_kmajor_desc(k_addr + (kk % 4) * 32), id_s, kk != 0);
        }
        tc::mma_commit(s_full + t);
      };
      auto issue_pv = [&](int t, int base, bool acc) {
        const uint32_t v_addr = tc::smem_u32(kv_tile(base, t, kQA));
#pragma unroll
        for (int kk = 0; kk < kKeys / 16; ++kk)
          mma_f16_ts(tmem + 256 + 64 * t, tmem + 384 + 64 * t + 8 * kk, tc::sw128_mnmajor_desc(v_addr + kk * 2048),
                     id_pv, acc || kk != 0);
        tc::mma_commit(pv_done + t);
      };
      // S(t) of a block is issued once the softmax has read S(t) of the block before (its
      // registers then hold the scores), so the next scores compute under this block's
      // exponentials; P(t)*V follows once P(t) is in tensor memory.  A K/V block and the q
      // buffer are released when both issuers have committed their last read of them.
      for (int item = blockIdx.x; ok && item < a.items; item += gridDim.x, ++li) {
        mixed = item_mixed(a, item);
        const int need = (kQA + 1) * (mixed ? 2 : 1);
        qb = li % kQBufs;
        if (!tc::mbar_wait(q_full + qb, (li / kQBufs) & 1, a.status, 32, abort)) break;
        if (!tc::mbar_wait(kv_full + g % kMaxStages, (g / kMaxStages) & 1, a.status, 33, abort)) break;
        if (g > 0 && !tc::mbar_wait(s_free + t, (g - 1) & 1, a.status, 41, abort)) break;
        tc::tc_fence_after();
        issue_s(t, ptr);
        if (a.n_blocks == 1) tc::mma_commit(q_empty + qb);
        for (int j = 0; j < a.n_blocks; ++j, ++g) {
          const int base = (ptr + j * need) % AttnSmem<kQA>::ring;
          if (j + 1 < a.n_blocks) {
            if (!tc::mbar_wait(kv_full + (g + 1) % kMaxStages, ((g + 1) / kMaxStages) & 1, a.status, 36, abort) ||
                !tc::mbar_wait(s_free + t, g & 1, a.status, 41, abort)) {
              ok = false;
              break;
            }
            tc::tc_fence_after();
            issue_s(t, (base + need) % AttnSmem<kQA>::ring);
            if (j + 2 == a.n_blocks) tc::mma_commit(q_empty + qb);
          }
          if (!tc::mbar_wait(p_full + t, g & 1, a.status, 34, abort) ||
              (j == 0 && !tc::mbar_wait(o_free + t, (li & 1) ^ 1, a.status, 35, abort))) {
            ok = false;
            break;
          }
          tc::tc_fence_after();
          issue_pv(t, base, j != 0);
          tc::mma_commit(kv_empty + g % kMaxStages);
        }
        ptr = (ptr + a.n_blocks * need) % AttnSmem<kQA>::ring;
      }
      tc::mma_commit(done);
      tc::mbar_wait(done, 0, a.status, 37, abort);
    }
  }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegsSoftmax));
    // ---------------- softmax warpgroups: tile t = warp / 4, query row r of the tile
    const int t = warp >> 2;
    const int r = (warp & 3) * 32 + lane;
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + 128 * t + lane_off, tO = tmem + 256 + 64 * t + lane_off;
    const uint32_t tP = tmem + 384 + 64 * t + lane_off;  // P_t: 64 columns of packed fp16
    const int prob = r >> 6;  // band axis: which of the tile's two problems
    int g = 0;
    int li = 0;
    bool ok = true;
    if (a.axis == 1) {
      // band axis: a row's P over the other problem's 64 keys stays zero for the whole launch
#pragma unroll
      for (int c = 0; c < 32; c += 4) tmem_st4(tP + 32 * (1 - prob) + c, 0u, 0u, 0u, 0u);
      asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
    }
    for (int item = blockIdx.x; ok && item < a.items; item += gridDim.x, ++li) {
      float m_run = -INFINITY, l = 0.f;
      // this row's output token and its head's gate, fetched now so the load's latency is
      // hidden under the item's key blocks
      const TileC it = tile_coords(a, item, t);
      long long tok = -1;
      if (a.axis == 0) {
        const int pos = it.qt * kRows + r;
        if (it.valid && pos < a.n) tok = (long long)(it.frame0 + r) * a.nb + it.band;
      } else {
        const int f = it.frame0 + prob, k = r & 63;
        if (k < a.n && f < a.BT) tok = (long long)f * a.nb + k;
      }
      const unsigned short gate =
          tok >= 0 ? reinterpret_cast<const unsigned short *>(a.qkv)[tok * a.ld + a.gate_col + it.head] : 0;
      for (int j = 0; j < a.n_blocks; ++j, ++g) {
        if (!tc::mbar_wait(s_full + t, g & 1, a.status, 38, abort)) { ok = false; break; }
        tc::tc_fence_after();
        const bool go = a.axis == 0
                            ? softmax_block<kKeys, kBF>(tS, tP, tO, min(kKeys, a.n - j * kKeys), m_run, l, j > 0,
                                                   pv_done + t, (g - 1) & 1, s_free + t, p_full + t, lane, a.status,
                                                   abort)
                            : softmax_block<64, kBF>(tS + 64 * prob, tP + 32 * prob, tO, a.n, m_run, l, false,
                                                pv_done + t, 0, s_free + t, p_full + t, lane, a.status, abort);
        if (!go) { ok = false; break; }
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
      // staged in shared memory (128-byte swizzle: 16-byte chunk c of row i at c ^ (i % 8))
      // and written by one bulk tensor store per warp; rows outside the output tensor
      // (frames past T, bands past nb) are not written
      const float gsc = tok >= 0 ? to_float16b<kBF>(gate) / l : 0.f;
      uint8_t *stg = smem + AttnSmem<kQA>::ostage + warp * 4096;
      if (lane == 0) tc::bulk_wait_read<0>();
      __syncwarp();
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        const float *oc = o + 8 * c;
        *reinterpret_cast<uint4 *>(stg + lane * 128 + ((c ^ (lane & 7)) << 4)) =
            make_uint4(pack_h2<kBF>(oc[0] * gsc, oc[1] * gsc), pack_h2<kBF>(oc[2] * gsc, oc[3] * gsc),
                       pack_h2<kBF>(oc[4] * gsc, oc[5] * gsc), pack_h2<kBF>(oc[6] * gsc, oc[7] * gsc));
      }
      tc::fence_proxy_async();
      __syncwarp();
      if (lane == 0 && it.valid) {
        // output coordinates (d, head, band, frame within the window, batch)
        int c2, c3, c4;
        if (a.axis == 0) {
          c2 = it.band; c3 = it.qt * kRows + 32 * (warp & 3); c4 = it.b;
        } else {
          const int f = it.frame0 + ((warp & 3) >> 1);
          c2 = 32 * (warp & 1); c3 = f % a.T; c4 = f / a.T;
        }
        tma_store_5d(&to, stg, 0, it.head, c2, c3, c4);
        tc::bulk_commit();
      }
    }
    if (lane == 0) tc::bulk_wait_all();
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

// The tensor-core kernel takes q and k of 64 or 128 per head and v of 64.
bool attention_tc_supported(int dqk, int dv) { return dv == kDh && (dqk == 64 || dqk == 128); }

namespace {
template <bool kBF, int kQA>
bool attn_prepare() {
  cudaFuncAttributes fa;
  if (cudaFuncGetAttributes(&fa, attn_tc_kernel<kBF, kQA>) != cudaSuccess || fa.numRegs < kRegsLaunch) return false;
  return cudaFuncSetAttribute(attn_tc_kernel<kBF, kQA>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              (int)(AttnSmem<kQA>::total + 1024)) == cudaSuccess;
}
static_assert(AttnSmem<1>::total + 1024 <= 232448 && AttnSmem<2>::total + 1024 <= 232448,
              "attention shared memory over the 227 KB limit");
}  // namespace

bool attention_tc_init() {
  int dev = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&g_num_sms, cudaDevAttrMultiProcessorCount, dev);
  return attn_prepare<false, 1>() && attn_prepare<true, 1>() && attn_prepare<false, 2>() && attn_prepare<true, 2>();
}

bool launch_attention_tc(const __half *qkv, int ld, __half *o, int B, int T, int nb, int H, int dqk, int axis, bool pdl,
                         bool bf16, unsigned *status, cudaStream_t st) {
  AttnArgs a;
  a.qkv = qkv;
  a.o = o;
  a.status = status;
  a.B = B; a.T = T; a.nb = nb; a.H = H; a.axis = axis; a.ld = ld;
  a.BT = B * T;
  a.n = axis == 0 ? T : nb;
  a.q_tiles = (a.n + kRows - 1) / kRows;
  const size_t Aqk = (size_t)H * dqk, A = (size_t)H * kDh;  // q (and k) width, v width
  a.gate_col = (int)(2 * Aqk + A);
  unsigned box[4];
  if (axis == 0) {
    // pairs of consecutive tiles of one sequence; an odd last tile pairs with the next
    // sequence's (separate keys)
    a.S = B * nb * H;
    a.pairs = a.q_tiles / 2;
    a.split_odd = dqk == 128;
    a.items = a.S * a.pairs + ((a.q_tiles & 1) ? (a.split_odd ? a.S : (a.S + 1) / 2) : 0);
    a.n_blocks = (a.n + kKeys - 1) / kKeys;
    box[0] = 64; box[1] = 1; box[2] = 1; box[3] = kRows;       // 128 frames of one (band, head)
  } else {
    if (nb > 64) return false;
    a.split_odd = 0;
    a.pairs = 0;
    a.S = 0;
    a.items = H * ((a.BT + 3) / 4);
    a.n_blocks = 1;
    box[0] = 64; box[1] = 1; box[2] = 64; box[3] = 2;          // bands 0..63 of two frames
  }
  // (d, head, band, frame) over the token-major buffer; q, k, v differ by their column offset,
  // q and k by their depth (a 64-wide box of them per load)
  const unsigned long long dqk_dims[4] = {(unsigned long long)dqk, (unsigned long long)H, (unsigned long long)nb,
                                          (unsigned long long)a.BT};
  const unsigned long long dqk_str[3] = {(unsigned long long)dqk, (unsigned long long)ld, (unsigned long long)nb * ld};
  const unsigned long long dv_dims[4] = {(unsigned long long)kDh, (unsigned long long)H, (unsigned long long)nb,
                                         (unsigned long long)a.BT};
  const unsigned long long dv_str[3] = {(unsigned long long)kDh, (unsigned long long)ld, (unsigned long long)nb * ld};
  // output [token][head][d] as (d, head, band, frame within the window, batch); a warp
  // stores 32 rows: 32 frames of one band (time axis) or 32 bands of one frame (band axis)
  const unsigned long long odims[5] = {(unsigned long long)kDh, (unsigned long long)H, (unsigned long long)nb,
                                       (unsigned long long)T, (unsigned long long)B};
  const unsigned long long ostr[4] = {(unsigned long long)kDh, (unsigned long long)A, (unsigned long long)nb * A,
                                      (unsigned long long)T * nb * A};
  const unsigned obox[5] = {(unsigned)kDh, 1u, axis == 0 ? 1u : 32u, axis == 0 ? 32u : 1u, 1u};
  CUtensorMap tq, tk, tv, to;
  if (!make_tmap(&tq, qkv, kTmF16, 4, dqk_dims, dqk_str, box, 128) ||
      !make_tmap(&tk, qkv + Aqk, kTmF16, 4, dqk_dims, dqk_str, box, 128) ||
      !make_tmap(&tv, qkv + 2 * Aqk, kTmF16, 4, dv_dims, dv_str, box, 128) ||
      !make_tmap(&to, o, kTmF16, 5, odims, ostr, obox, 128))
    return false;
  const int grid = (int)std::min<long long>(a.items, g_num_sms > 0 ? g_num_sms : 148);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid, 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
#define MRF_ATTN(BF, QA)                                       \
  do {                                                         \
    cfg.dynamicSmemBytes = AttnSmem<QA>::total + 1024;         \
    cudaLaunchKernelEx(&cfg, attn_tc_kernel<BF, QA>, tq, tk, tv, to, a); \
  } while (0)
  if (dqk == 128) {
    if (bf16) MRF_ATTN(true, 2);
    else MRF_ATTN(false, 2);
  } else {
    if (bf16) MRF_ATTN(true, 1);
    else MRF_ATTN(false, 1);
  }
#undef MRF_ATTN
  return true;
}

}  // namespace mrf
