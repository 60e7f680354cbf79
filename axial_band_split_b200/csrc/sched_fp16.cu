// fp16 tensor-core schedule: weight packing, workspace and the per-forward launch list.
//
// Per forward (N_tok = B*T*bands tokens, token (b*T + t)*bands + k):
//   band split (gather + norm + Linear)        -> x (fp16 residual stream), |x|^2
//   per transformer (time axis, then band axis, depth times):
//     QKV+gates GEMM, RoPE epilogue            -> q, k, v fp16 in attention layout, gates
//     attention                                -> O fp16 (times the gate)
//     out-projection GEMM, residual epilogue   -> x, |x|^2
//     FF1 GEMM, GELU epilogue                  -> H fp16
//     FF2 GEMM, residual epilogue              -> x, |x|^2 and |g x|^2 (the output norm, deferred
//                                                 to the consumers' epilogues)
//   mask head: per-band GEMMs (tanh, tanh, GLU), the GLU epilogue adding each band feature
//   into its stft_repr row of the zeroed masks (the overlap average)  -> masks
//
// Exact rewrites (package/scripts/export-roformer.py of "@audio/neural-separate 0.4.0 →
// 0.5.0", class Core and its module docstring): each RMSNorm's sqrt(d)*gamma is folded
// into the weight of the Linear it feeds, leaving the per-row 1/max(|x|, 1e-12) as an
// epilogue scale; the gates' projection is appended to q, k, v; the mask head's bands
// are batched as groups of one GEMM; its last layer's value and gate rows are interleaved
// so that a GLU pair is two adjacent accumulator columns.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <algorithm>
#include <cmath>
#include <cstdlib>
#include <cstring>

#include "gemm_tc.cuh"
#include "mrf_handle.h"

namespace mrf {

bool launch_attention_tc(const __half *qkv, int ld, __half *o, int B, int T, int nb, int H, int dqk, int axis,
                         bool pdl, bool bf16, unsigned *status, cudaStream_t st);
bool attention_tc_supported(int dqk, int dv);
bool attention_tc_init();

struct TrF16 {
  __half *wqkvg = nullptr, *wo = nullptr, *w1 = nullptr, *w2 = nullptr;
  float *bg = nullptr, *b1 = nullptr, *b2 = nullptr, *gout = nullptr;
};

struct Fp16State {
  std::vector<TrF16> tr;
  __half *w_bs = nullptr;     // band split [nb*D, k_bs], gamma*sqrt(d_in) folded, zero-padded
  __half *A_bs = nullptr;     // normalised band features [nb][MBT][k_bs]
  int k_bs = 0;
  GemmGroup *g_bs = nullptr;
  // mask heads, one per stem: layers 0 .. mask_depth-1 stacked over bands [nb*MH, K] (mw[stem][layer]);
  // the last layer [sum 2*d_in, MH] with rows interleaved (value e, gate e)
  std::vector<std::vector<__half *>> mw;
  std::vector<std::vector<float *>> mb;
  std::vector<__half *> mw_last;
  std::vector<float *> mb_last;
  // group tables
  GemmGroup *g_qkv = nullptr, *g_out = nullptr, *g_ff1 = nullptr, *g_ff2 = nullptr;
  GemmGroup *g_m0 = nullptr, *g_mid = nullptr, *g_last = nullptr;
  int n_last_tiles = 0;
  // workspace
  // Row sums of squares as partial slots (parts_* a row, added in order by the consumer): |x|^2
  // of the out-projection output (ss), and the deferred output norm's |x|^2 and |g x|^2 of the
  // last FF2 output (ssx, ssg; g = sqrt(D) gamma_out; ssg holds the band split's |x|^2 first)
  float *ss = nullptr, *ssx = nullptr, *ssg = nullptr;
  int parts_res = 0, parts_bs = 0;
  __half *Xh = nullptr, *QKV = nullptr, *O = nullptr, *Hh = nullptr, *H1 = nullptr, *H2 = nullptr;
  int ldq = 0;  // row length of QKV: [q | k | v | gates], padded to a multiple of 8
  int sms = 148;
  bool tc_attention = true;
  // MRF_BF16: every 16-bit buffer and weight holds bf16 (the __half pointers are 16-bit
  // containers), and the residual stream also keeps an fp32 master copy X (rounding the residual
  // adds of twelve transformers to bf16's 8-bit significand would cost too much precision)
  bool bf16 = false;
  float *X = nullptr;
  // which GEMMs run as CTA pairs (cta_group::2), from MRF_GEMM_PAIR in the environment at
  // create: 0 none, 1 those with K >= kPairMinK (the default), 2 every pair-capable one (the four
  // trunk GEMMs and the mask MLP's tanh layers)
  int pair = 1;
  // the tensor-core kernels launched with programmatic stream serialisation (each waits for its
  // inputs after its prologue, which then overlaps the previous kernel's tail); MRF_PDL=0 in the
  // environment at create turns it off
  bool pdl = true;
  // the feed-forward as one kernel on CTA pairs (fp16, GELU, D <= 384, hidden <= 1536, four
  // row-statistic slots) when MRF_FF_FUSED=1 at create; by default the FF1 and FF2 GEMMs, which
  // measured faster (the fused kernel's 128-wide hidden chunks re-read x from shared memory for
  // every chunk: its MMAs run at about half the tensor rate)
  bool ff_fused = false;
};

namespace {

constexpr int kBnWide = 256, kBnNarrow = 192;

// Weights rounded once (to nearest even) to the schedule's 16-bit type, in 16-bit containers.
std::vector<__half> to16(const std::vector<float> &v, bool bf16) {
  std::vector<__half> o(v.size());
  if (bf16) {
    for (size_t i = 0; i < v.size(); ++i) {
      const __nv_bfloat16 b = __float2bfloat16_rn(v[i]);
      memcpy(&o[i], &b, 2);
    }
  } else {
    for (size_t i = 0; i < v.size(); ++i) o[i] = __float2half_rn(v[i]);
  }
  return o;
}

template <class T>
T *up(mrf_handle *h, const std::vector<T> &v) {
  T *p = h->alloc<T>(v.size());
  if (p && !h->upload(p, v.data(), v.size() * sizeof(T))) return nullptr;
  return p;
}

// W [N, K] with column j scaled by s[j] (an RMSNorm's sqrt(K)*gamma folded into the Linear after it).
std::vector<float> fold_cols(const std::vector<float> &w, const std::vector<float> &gamma, int N, int K) {
  std::vector<float> o(w.size());
  const double s = std::sqrt((double)K);
  for (int n = 0; n < N; ++n)
    for (int k = 0; k < K; ++k) o[(size_t)n * K + k] = (float)((double)w[(size_t)n * K + k] * gamma[k] * s);
  return o;
}

int cdiv(int a, int b) { return (a + b - 1) / b; }

GemmGroup *upload_groups(mrf_handle *h, const std::vector<GemmGroup> &g) { return up(h, g); }

}  // namespace

std::string fp16_supported(const mrf_config &c, const BandTables &t) {
  (void)t;
  const int Aqk = c.heads * c.dim_head, A = attn_out_width(c);
  if (c.dim % 64) return "fp16 schedule needs dim % 64 == 0";
  if (Aqk % 64 || A % 64) return "fp16 schedule needs heads*dim_head and heads*dim_head_v multiples of 64";
  if (c.dim_head % 16 || head_v(c) % 16) return "fp16 schedule needs dim_head and dim_head_v multiples of 16";
  if (c.mask_hidden % 64) return "fp16 schedule needs mask_hidden % 64 == 0";
  return "";
}

mrf_status pack_fp16(mrf_handle *h, WeightMap &W) {
  const mrf_config &c = h->cfg;
  const BandTables &t = h->tab;
  const int nb = c.num_bands, D = c.dim, H = c.heads, dh = c.dim_head, A = attn_out_width(c), QKVW = qkv_width(c),
            FF = c.ff_mult * D, MH = c.mask_hidden;
  const long long MBT = (long long)c.max_batch * c.max_frames, NT = MBT * nb;
  Fp16State *f = new (std::nothrow) Fp16State();
  if (!f) return MRF_ENOMEM;
  h->f16 = f;
  cudaDeviceGetAttribute(&f->sms, cudaDevAttrMultiProcessorCount, h->device);
  f->tc_attention = attention_tc_supported(dh, head_v(c));
  f->bf16 = c.compute == MRF_BF16;
  if (const char *e = getenv("MRF_GEMM_PAIR")) f->pair = std::min(std::max(atoi(e), 0), 2);
  if (const char *e = getenv("MRF_PDL")) f->pdl = atoi(e) != 0;
  const char *ffe = getenv("MRF_FF_FUSED");
  f->ff_fused = ffe && atoi(ffe) != 0 && !f->bf16 && c.ff_act == 0 && ff_tc_supported(c.dim, c.ff_mult * c.dim) &&
                cdiv(c.dim, kBnNarrow) * 2 == 4;
  if (f->ff_fused && !ff_tc_init()) {
    h->err = "fused feed-forward initialisation failed (shared-memory limit)";
    return MRF_ECUDA;
  }
  if (!gemm_tc_init() || (f->tc_attention && !attention_tc_init())) {
    h->err = "tcgen05 kernel initialisation failed (tensor-map encoder or shared-memory limit)";
    return MRF_ECUDA;
  }
  // band split: per band [D, d_in] with gamma*sqrt(d_in) folded, zero-padded to k_bs columns
  f->k_bs = cdiv(h->max_width, 64) * 64;
  {
    std::vector<float> wb((size_t)nb * D * f->k_bs, 0.f);
    for (int k = 0; k < nb; ++k) {
      const std::string p = "band_split.to_features." + std::to_string(k) + ".";
      const auto &g = W[p + "0.gamma"].v;
      const auto &w = W[p + "1.weight"].v;
      const int wd = t.width[k];
      const double sc = std::sqrt((double)wd);
      for (int n = 0; n < D; ++n)
        for (int e = 0; e < wd; ++e)
          wb[((size_t)k * D + n) * f->k_bs + e] = (float)((double)w[(size_t)n * wd + e] * g[e] * sc);
    }
    f->w_bs = up(h, to16(wb, f->bf16));
    std::vector<GemmGroup> gb(nb);
    for (int k = 0; k < nb; ++k)
      gb[k] = {D, cdiv(D, kBnNarrow), k * cdiv(D, kBnNarrow), (int)(k * MBT), k * D, k, k * D, cdiv(t.width[k], 64)};
    f->g_bs = upload_groups(h, gb);
    f->A_bs = h->alloc<__half>((size_t)nb * MBT * f->k_bs);
    if (!f->w_bs || !f->g_bs || !f->A_bs) return MRF_ENOMEM;
  }
  // transformers
  f->tr.resize(2 * c.depth);
  for (int l = 0; l < c.depth; ++l)
    for (int a = 0; a < 2; ++a) {
      const std::string p = "layers." + std::to_string(l) + "." + std::to_string(a) + ".";
      TrF16 &x = f->tr[2 * l + a];
      const auto &ga = W[p + "layers.0.0.norm.gamma"].v;
      std::vector<float> qkvg = fold_cols(W[p + "layers.0.0.to_qkv.weight"].v, ga, QKVW, D);
      std::vector<float> wg = fold_cols(W[p + "layers.0.0.to_gates.weight"].v, ga, H, D);
      qkvg.insert(qkvg.end(), wg.begin(), wg.end());
      if (2 * l + a > 0) {
        // the previous transformer's output norm is deferred: its sqrt(D) * gamma scales x
        // column-wise, folded here into every q, k, v and gate weight column
        const int pl = a == 1 ? l : l - 1, pa = a == 1 ? 0 : 1;
        const auto &gp = W["layers." + std::to_string(pl) + "." + std::to_string(pa) + ".norm.gamma"].v;
        const double sd = std::sqrt((double)D);
        for (int n = 0; n < QKVW + H; ++n)
          for (int k = 0; k < D; ++k) qkvg[(size_t)n * D + k] = (float)((double)qkvg[(size_t)n * D + k] * gp[k] * sd);
      }
      x.wqkvg = up(h, to16(qkvg, f->bf16));
      x.bg = up(h, W[p + "layers.0.0.to_gates.bias"].v);
      x.wo = up(h, to16(W[p + "layers.0.0.to_out.0.weight"].v, f->bf16));
      if (c.ff_act == 1) {  // GEGLU: (value, gate) rows paired for the epilogue
        x.w1 = up(h, to16(fold_cols(interleave_halves(W[p + "layers.0.1.net.1.weight"].v, FF, D),
                                       W[p + "layers.0.1.net.0.gamma"].v, 2 * FF, D), f->bf16));
        x.b1 = up(h, interleave_halves(W[p + "layers.0.1.net.1.bias"].v, FF, 1));
      } else {
        x.w1 = up(h, to16(fold_cols(W[p + "layers.0.1.net.1.weight"].v, W[p + "layers.0.1.net.0.gamma"].v, FF, D), f->bf16));
        x.b1 = up(h, W[p + "layers.0.1.net.1.bias"].v);
      }
      x.w2 = up(h, to16(W[p + "layers.0.1.net.4.weight"].v, f->bf16));
      x.b2 = up(h, W[p + "layers.0.1.net.4.bias"].v);
      std::vector<float> go(W[p + "norm.gamma"].v);
      for (auto &v : go) v = (float)(v * std::sqrt((double)D));
      x.gout = up(h, go);
      if (!x.wqkvg || !x.bg || !x.wo || !x.w1 || !x.b1 || !x.w2 || !x.b2 || !x.gout)
        return MRF_ENOMEM;
    }
  // mask heads
  for (int s = 0; s < c.num_stems; ++s) {
  std::vector<std::vector<float>> mw(c.mask_depth), mb(c.mask_depth);
  std::vector<float> wl, bl;
  for (int k = 0; k < nb; ++k) {
    const std::string p = "mask_estimators." + std::to_string(s) + ".to_freqs." + std::to_string(k) + ".0.";
    for (int i = 0; i < c.mask_depth; ++i) {
      const auto &w = W[p + std::to_string(2 * i) + ".weight"].v;
      const auto &b = W[p + std::to_string(2 * i) + ".bias"].v;
      mw[i].insert(mw[i].end(), w.begin(), w.end());
      mb[i].insert(mb[i].end(), b.begin(), b.end());
    }
    const std::string q = p + std::to_string(2 * c.mask_depth);
    const auto &w = W[q + ".weight"].v;
    const auto &b = W[q + ".bias"].v;
    const int wd = t.width[k];
    for (int e = 0; e < wd; ++e) {
      wl.insert(wl.end(), w.begin() + (size_t)e * MH, w.begin() + (size_t)(e + 1) * MH);
      wl.insert(wl.end(), w.begin() + (size_t)(wd + e) * MH, w.begin() + (size_t)(wd + e + 1) * MH);
      bl.push_back(b[e]);
      bl.push_back(b[wd + e]);
    }
  }
  if (c.depth > 0) {
    // the last transformer's output norm is deferred: fold its sqrt(D) * gamma into the
    // mask MLP's first layer (its 1 / |x| is a row scale in that layer's epilogue)
    const auto &gl = W["layers." + std::to_string(c.depth - 1) + ".1.norm.gamma"].v;
    const double sd = std::sqrt((double)D);
    for (size_t r = 0; r < mw[0].size() / D; ++r)
      for (int k = 0; k < D; ++k) mw[0][r * D + k] = (float)((double)mw[0][r * D + k] * gl[k] * sd);
  }
  f->mw.emplace_back();
  f->mb.emplace_back();
  for (int i = 0; i < c.mask_depth; ++i) {
    f->mw.back().push_back(up(h, to16(mw[i], f->bf16)));
    f->mb.back().push_back(up(h, mb[i]));
    if (!f->mw.back().back() || !f->mb.back().back()) return MRF_ENOMEM;
  }
  f->mw_last.push_back(up(h, to16(wl, f->bf16)));
  f->mb_last.push_back(up(h, bl));
  if (!f->mw_last.back() || !f->mb_last.back()) return MRF_ENOMEM;
  }
  // group tables
  auto single = [&](int N, int BN) {
    GemmGroup g{N, cdiv(N, BN), 0, 0, 0, 0, 0, 0};
    return upload_groups(h, {g});
  };
  f->g_qkv = single(QKVW + H, kBnWide);
  f->g_out = single(D, kBnNarrow);
  const int F1 = c.ff_act == 1 ? 2 * FF : FF;  // first feed-forward projection's outputs
  f->g_ff1 = single(F1, kBnWide);
  f->g_ff2 = single(D, kBnNarrow);
  std::vector<GemmGroup> g0(nb), g1(nb), g2(nb);
  int start = 0;
  for (int k = 0; k < nb; ++k) {
    g0[k] = {MH, cdiv(MH, kBnWide), k * cdiv(MH, kBnWide), k, k * MH, k, k * MH, 0};
    g1[k] = {MH, cdiv(MH, kBnWide), k * cdiv(MH, kBnWide), (int)(k * MBT), k * MH, k, k * MH, 0};
    const int N = 2 * t.width[k];
    g2[k] = {N, cdiv(N, kBnWide), start, (int)(k * MBT), 2 * t.feat_off[k], t.feat_off[k], 2 * t.feat_off[k], 0};
    start += g2[k].n_tiles;
  }
  f->n_last_tiles = start;
  f->g_m0 = upload_groups(h, g0);
  f->g_mid = upload_groups(h, g1);
  f->g_last = upload_groups(h, g2);
  if (!f->g_qkv || !f->g_out || !f->g_ff1 || !f->g_ff2 || !f->g_m0 || !f->g_mid || !f->g_last) return MRF_ENOMEM;
  // workspace
  f->ldq = cdiv(QKVW + H, 8) * 8;
  f->Xh = h->alloc<__half>(NT * D);
  f->parts_res = cdiv(D, kBnNarrow) * 2;  // residual GEMMs: 8 epilogue warps, 2 per lane quarter
  f->parts_bs = cdiv(D, kBnNarrow) * 4;   // band split: 16 epilogue warps, 4 per lane quarter
  const int parts = std::max(f->parts_res, f->parts_bs);
  f->ss = h->alloc<float>(NT * parts);
  f->ssx = h->alloc<float>(NT * parts);
  f->ssg = h->alloc<float>(NT * parts);
  f->QKV = h->alloc<__half>(NT * f->ldq);
  f->O = h->alloc<__half>(NT * A);
  f->Hh = h->alloc<__half>(NT * FF);
  f->H1 = h->alloc<__half>((long long)nb * MBT * MH);
  f->H2 = h->alloc<__half>((long long)nb * MBT * MH);
  if (f->bf16 && !(f->X = h->alloc<float>(NT * D))) return MRF_ENOMEM;
  if (!f->Xh || !f->ss || !f->ssx || !f->ssg || !f->QKV || !f->O || !f->Hh || !f->H1 || !f->H2)
    return MRF_ENOMEM;
  // rows past a forward's B*T are read by ragged tiles (and discarded): keep them finite
  if (cudaMemset(f->QKV, 0, NT * f->ldq * 2) != cudaSuccess || cudaMemset(f->H1, 0, (size_t)nb * MBT * MH * 2) != cudaSuccess ||
      cudaMemset(f->H2, 0, (size_t)nb * MBT * MH * 2) != cudaSuccess || cudaMemset(f->Xh, 0, NT * D * 2) != cudaSuccess)
    return MRF_ECUDA;
  return MRF_OK;
}

bool debug_buffer_fp16(mrf_handle *h, const std::string &name, const void **ptr, size_t *bytes) {
  Fp16State *f = h->f16;
  if (!f) return false;
  const long long BT = (long long)h->last_B * h->last_T;
  if (name == "X") {
    // the residual stream after the last transformer, with its deferred output norm applied
    const int D = h->cfg.dim;
    const long long rows = BT * h->cfg.num_bands;
    static thread_local std::vector<float> hx;
    hx.resize((size_t)rows * D);
    if (f->bf16) {
      if (cudaMemcpy(hx.data(), f->X, hx.size() * 4, cudaMemcpyDeviceToHost) != cudaSuccess) return false;
    } else {
      std::vector<__half> xh((size_t)rows * D);
      if (cudaMemcpy(xh.data(), f->Xh, xh.size() * 2, cudaMemcpyDeviceToHost) != cudaSuccess) return false;
      for (size_t i = 0; i < xh.size(); ++i) hx[i] = __half2float(xh[i]);
    }
    if (h->cfg.depth > 0) {
      std::vector<float> s2((size_t)rows * f->parts_res), g(D);
      if (cudaMemcpy(s2.data(), f->ssx, s2.size() * 4, cudaMemcpyDeviceToHost) != cudaSuccess ||
          cudaMemcpy(g.data(), f->tr.back().gout, D * 4, cudaMemcpyDeviceToHost) != cudaSuccess)
        return false;
      for (long long r = 0; r < rows; ++r) {
        float ssr = 0.f;
        for (int q = 0; q < f->parts_res; ++q) ssr += s2[(size_t)r * f->parts_res + q];
        const float inv = 1.f / std::max(std::sqrt(ssr), 1e-12f);
        for (int k = 0; k < D; ++k) hx[(size_t)r * D + k] *= inv * g[k];
      }
    }
    *ptr = hx.data();
    *bytes = hx.size() * 4;
    return true;
  }
  return false;  // the mask features ("M") are never stored: the GLU epilogue averages them into the masks
}

void destroy_fp16(mrf_handle *h) {
  delete h->f16;
  h->f16 = nullptr;
}

namespace {

GemmParams base_params(mrf_handle *h, int M, int K, int BN, const GemmGroup *groups, int ngroups,
                       int total_n_tiles) {
  GemmParams p;
  memset(&p, 0, sizeof p);
  p.M = M;
  p.K = K;
  p.BN = BN;
  p.groups = groups;
  p.ngroups = ngroups;
  p.total_n_tiles = total_n_tiles;
  p.m_tiles = cdiv(M, 128);
  p.status = h->status;
  return p;
}

// A trunk GEMM or a mask tanh layer may run as CTA pairs (M = 256 tiles, B maps with half-height
// boxes): each CTA then stages half of every B tile, which halves the shared-memory traffic of the
// main loop.  That pays where the main loop is long (FF2, K = 4 D: 1.14 -> 1.06 ms per forward)
// and costs where the epilogue dominates (the QKV, out-projection and FF1 GEMMs, K <= 512, run
// about 10 % slower as pairs on B200) or the rows are short (a band's T rows of the mask MLP fill
// 256-row tiles worse than 128-row ones: its K = 1536 layer ran 7 % slower), so by default only
// trunk GEMMs with K >= kPairMinK pair.  The band split and the GLU layer run one CTA per tile.
constexpr int kPairMinK = 1024;
// Per-kernel timing records an event pair around each launch, which a kernel started ahead of
// its predecessor's end would blur: timing runs launch without the programmatic attribute.
bool use_pdl(const mrf_handle *h) { return h->f16->pdl && !h->timing; }

bool use_pair(const mrf_handle *h, int epi, int K) {
  const int mode = h->f16->pair;
  return gemm_tc_pair_kind(epi) && (mode == 2 || (mode == 1 && epi != kTcTanh && K >= kPairMinK));
}

void gemm(mrf_handle *h, const char *name, int epi, const CUtensorMap &a, const CUtensorMap &b, const GemmParams &p0,
          const CUtensorMap *c = nullptr, const CUtensorMap *d = nullptr) {
  GemmParams p = p0;
  const bool pair = use_pair(h, epi, p.K);
  if (pair) p.m_tiles = cdiv(p.M, 256);
  const int tiles = p.m_tiles * p.total_n_tiles;
  const int grid = pair ? 2 * std::min(tiles, h->f16->sms / 2) : std::min(tiles, h->f16->sms);
  h->begin(name);
  launch_gemm_tc(epi, h->f16->bf16, pair, a, b, c ? *c : a, d ? *d : a, p, grid, use_pdl(h), h->cur_stream);
  h->end();
}

// Output maps of the bulk-store epilogues (extents exactly the rows of this forward).
bool map2(CUtensorMap *m, const void *base, int dtype, unsigned long long cols, unsigned long long rows,
          unsigned long long ld, unsigned box0, int swz) {
  const unsigned long long dims[2] = {cols, rows}, st[1] = {ld};
  const unsigned box[2] = {box0, 32};
  return make_tmap(m, base, dtype, 2, dims, st, box, swz);
}

}  // namespace

void schedule_fp16(mrf_handle *h, const float *in, float *out, int B, int T) {
  const mrf_config &c = h->cfg;
  Fp16State *f = h->f16;
  const int nb = c.num_bands, D = c.dim, H = c.heads, dh = c.dim_head, A = attn_out_width(c), QKVW = qkv_width(c),
            FF = c.ff_mult * D, MH = c.mask_hidden;
  const long long MBT = (long long)c.max_batch * c.max_frames, NT = MBT * nb;
  const int F1 = c.ff_act == 1 ? 2 * FF : FF;  // first feed-forward projection's outputs
  const int M = B * T * nb;
  const int R = h->tab.n_freqs * h->tab.channels;
  cudaStream_t st = h->cur_stream;

  // tensor maps of the activations (fixed buffers; extents cover the whole workspace)
  CUtensorMap mXh, mO, mHh, mXband, mH1, mH2;
  bool ok = make_tmap_f16(&mXh, f->Xh, D, NT, 1, D, NT * D, 128, 1) &&
            make_tmap_f16(&mO, f->O, A, NT, 1, A, NT * A, 128, 1) &&
            make_tmap_f16(&mHh, f->Hh, FF, NT, 1, FF, NT * FF, 128, 1) &&
            make_tmap_f16(&mXband, f->Xh, D, nb, MBT, D, (long long)nb * D, 1, 128) &&
            make_tmap_f16(&mH1, f->H1, MH, nb * MBT, 1, MH, nb * MBT * MH, 128, 1) &&
            make_tmap_f16(&mH2, f->H2, MH, nb * MBT, 1, MH, nb * MBT * MH, 128, 1);
  CUtensorMap mAbs, mWbs;
  ok = ok && make_tmap_f16(&mAbs, f->A_bs, f->k_bs, (long long)nb * MBT, 1, f->k_bs, (long long)nb * MBT * f->k_bs, 128, 1) &&
       make_tmap_f16(&mWbs, f->w_bs, f->k_bs, (long long)nb * D, 1, f->k_bs, (long long)nb * D * f->k_bs, kBnNarrow, 1);
  const int n_mask_maps = c.mask_depth + 1;  // per stem
  std::vector<CUtensorMap> wmaps(4 * 2 * c.depth + c.num_stems * n_mask_maps);
  // the fused feed-forward's weight maps: W1 in 64-row boxes (half of a 128-unit chunk), W2 in
  // boxes of half an MMA piece (D / 2 rows, D / 4 when D > 256)
  std::vector<CUtensorMap> ffmaps(f->ff_fused ? 2 * 2 * c.depth : 0);
  for (int i = 0; ok && f->ff_fused && i < 2 * c.depth; ++i) {
    const TrF16 &w = f->tr[i];
    const unsigned w2box = D > 256 ? D / 4 : D / 2;
    ok = make_tmap_f16(&ffmaps[2 * i], w.w1, D, FF, 1, D, (long long)FF * D, 64, 1) &&
         make_tmap_f16(&ffmaps[2 * i + 1], w.w2, FF, D, 1, FF, (long long)D * FF, w2box, 1);
  }
  for (int i = 0; ok && i < 2 * c.depth; ++i) {
    const TrF16 &w = f->tr[i];
    // weight boxes: BN rows, or BN / 2 for the CTA pairs (each CTA loads half of a B tile)
    const unsigned bq = use_pair(h, kTcQkv, D) ? kBnWide / 2 : kBnWide;
    const unsigned bo = use_pair(h, kTcResid, A) ? kBnNarrow / 2 : kBnNarrow;
    const unsigned b1 = use_pair(h, kTcGelu, D) ? kBnWide / 2 : kBnWide;
    const unsigned b2 = use_pair(h, kTcResid, FF) ? kBnNarrow / 2 : kBnNarrow;
    ok = make_tmap_f16(&wmaps[4 * i + 0], w.wqkvg, D, QKVW + H, 1, D, ((long long)QKVW + H) * D, bq, 1) &&
         make_tmap_f16(&wmaps[4 * i + 1], w.wo, A, D, 1, A, (long long)D * A, bo, 1) &&
         make_tmap_f16(&wmaps[4 * i + 2], w.w1, D, F1, 1, D, (long long)F1 * D, b1, 1) &&
         make_tmap_f16(&wmaps[4 * i + 3], w.w2, FF, D, 1, FF, (long long)D * FF, b2, 1);
  }
  const int wm0 = 8 * c.depth;
  const long long rows_last = 2LL * h->tab.n_feat();
  for (int s = 0; ok && s < c.num_stems; ++s) {
    const int w0 = wm0 + s * n_mask_maps;
    for (int i = 0; ok && i < c.mask_depth; ++i) {
      const int K = i == 0 ? D : MH;
      const unsigned bb = use_pair(h, kTcTanh, K) ? kBnWide / 2 : kBnWide;
      ok = make_tmap_f16(&wmaps[w0 + i], f->mw[s][i], K, (long long)nb * MH, 1, K, (long long)nb * MH * K, bb, 1);
    }
    ok = ok && make_tmap_f16(&wmaps[w0 + c.mask_depth], f->mw_last[s], MH, rows_last, 1, MH, rows_last * MH, kBnWide, 1);
  }
  // bulk-store output maps
  CUtensorMap mXho, mXhbs, mHo, mHo16, mH1o, mH2o, mQKVo;
  CUtensorMap mXo, mXbs;  // MRF_BF16: the fp32 master copy of the residual stream
  {
    const unsigned long long BT = (unsigned long long)B * T;
    const unsigned long long dx[3] = {(unsigned long long)D, (unsigned long long)nb, BT};
    const unsigned long long sx[2] = {(unsigned long long)D, (unsigned long long)nb * D};
    const unsigned bx[3] = {32, 1, 32};
    const unsigned long long dh3[3] = {(unsigned long long)MH, BT, (unsigned long long)nb};
    const unsigned long long sh3[2] = {(unsigned long long)MH, (unsigned long long)MBT * MH};
    const unsigned bh[3] = {32, 32, 1};
    ok = ok && map2(&mXho, f->Xh, kTmF16, D, M, D, 32, 64) && make_tmap(&mXhbs, f->Xh, kTmF16, 3, dx, sx, bx, 64) &&
         (!f->bf16 || (map2(&mXo, f->X, kTmF32, D, M, D, 32, 128) && make_tmap(&mXbs, f->X, kTmF32, 3, dx, sx, bx, 128))) &&
         map2(&mHo, f->Hh, kTmF16, FF, M, FF, 32, 64) && map2(&mHo16, f->Hh, kTmF16, FF, M, FF, 16, 0) &&
         make_tmap(&mH1o, f->H1, kTmF16, 3, dh3, sh3, bh, 64) &&
         make_tmap(&mH2o, f->H2, kTmF16, 3, dh3, sh3, bh, 64) &&
         map2(&mQKVo, f->QKV, kTmF16, QKVW + H, M, f->ldq, 32, 64);
  }
  if (!ok) {
    h->sched_error = "tensor-map encoding failed";
    return;
  }

  h->begin("band_gather");
  launch_band_gather(in, h->d_feat_row, h->d_bands, nb, B, T, R, MBT, f->k_bs, f->A_bs, f->bf16, use_pdl(h), st);
  h->end();
  {
    GemmParams p = base_params(h, B * T, f->k_bs, kBnNarrow, f->g_bs, nb, nb * cdiv(D, kBnNarrow));
    p.bias = h->b_bs; p.Xh = f->Xh; p.X = f->X; p.ss_out = f->ssg; p.ss_out_parts = f->parts_bs; p.ld = D; p.nb = nb;
    p.stall_test = h->stall_test ? 1 : 0;
    h->stall_test = false;
    gemm(h, "gemm_band_split", kTcBandSplit, mAbs, mWbs, p, f->bf16 ? &mXbs : &mXhbs, &mXhbs);
  }

  for (int i = 0; i < 2 * c.depth; ++i) {
    const TrF16 &w = f->tr[i];
    const int axis = i & 1;
    const CUtensorMap &mWqkv = wmaps[4 * i + 0], &mWo = wmaps[4 * i + 1], &mW1 = wmaps[4 * i + 2],
                      &mW2 = wmaps[4 * i + 3];
    // [q | k | v | gates] per token (RoPE positions along this transformer's axis)
    GemmParams p = base_params(h, M, D, kBnWide, f->g_qkv, 1, cdiv(QKVW + H, kBnWide));
    p.ss_in = f->ssg;  // |g x|^2 of the previous output (band split: |x|^2)
    p.ss_in_parts = i == 0 ? f->parts_bs : f->parts_res;
    p.rope = h->d_rope; p.gbias = w.bg;
    p.B = B; p.T = T; p.nb = nb; p.H = H; p.dh = dh; p.A = H * dh; p.Av = A; p.axis = axis;
    // the tensor-core attention takes scores in log2 units: fold log2(e) / sqrt(dh) into q
    p.q_scale = f->tc_attention ? (float)(1.4426950408889634 / std::sqrt((double)dh)) : 1.f;
    gemm(h, "gemm_qkv", kTcQkv, mXh, mWqkv, p, &mQKVo);

    h->begin(f->tc_attention ? (axis == 0 ? "attn_time_tc" : "attn_band_tc") : "attn_simt_f16");
    if (f->tc_attention) {
      if (!launch_attention_tc(f->QKV, f->ldq, f->O, B, T, nb, H, dh, axis, use_pdl(h), f->bf16, h->status, st)) {
        h->end();
        h->sched_error = "tensor-map encoding failed (attention)";
        return;
      }
    } else
      launch_attention_simt_f16(f->QKV, f->ldq, f->O, B, T, nb, H, dh, head_v(c), axis, f->bf16, st);
    h->end();

    p = base_params(h, M, A, kBnNarrow, f->g_out, 1, cdiv(D, kBnNarrow));
    p.Xh = f->Xh; p.X = f->X; p.ss_out = f->ss; p.ss_out_parts = f->parts_res; p.ld = D;
    if (i > 0) {  // the previous output norm
      p.res_ss = f->ssx; p.res_gain = f->tr[i - 1].gout; p.ss_in_parts = f->parts_res;
    }
    gemm(h, "gemm_out_resid", kTcResid, mO, mWo, p, f->bf16 ? &mXo : &mXho, &mXho);

    if (f->ff_fused) {
      FfParams q{};
      q.M = M; q.D = D; q.hidden = FF; q.ld = D; q.ss_in_parts = f->parts_res; q.ss_out_parts = f->parts_res;
      q.status = h->status; q.ss_in = f->ss; q.b1 = w.b1; q.b2 = w.b2; q.out_gain = w.gout; q.Xh = f->Xh;
      q.ss_out = f->ssx; q.ssg_out = f->ssg;
      h->begin("gemm_ff_fused");
      launch_ff_tc(mXh, ffmaps[2 * i], ffmaps[2 * i + 1], mXho, q, f->sms, use_pdl(h), st);
      h->end();
      continue;
    }
    p = base_params(h, M, D, kBnWide, f->g_ff1, 1, cdiv(F1, kBnWide));
    p.ss_in = f->ss; p.ss_in_parts = f->parts_res; p.bias = w.b1; p.out_h = f->Hh; p.ldo = FF;
    if (c.ff_act == 1) gemm(h, "gemm_ff1_geglu", kTcGeglu, mXh, mW1, p, &mHo16);
    else gemm(h, "gemm_ff1_gelu", kTcGelu, mXh, mW1, p, &mHo);

    p = base_params(h, M, FF, kBnNarrow, f->g_ff2, 1, cdiv(D, kBnNarrow));
    p.Xh = f->Xh; p.X = f->X; p.ss_out = f->ssx; p.ss_out_parts = f->parts_res; p.ld = D; p.bias = w.b2;
    p.ssg_out = f->ssg; p.out_gain = w.gout;  // the output norm is left to the consumers
    gemm(h, "gemm_ff2_resid", kTcResid, mHh, mW2, p, f->bf16 ? &mXo : &mXho, &mXho);
  }

  // mask heads, one per stem; each GLU epilogue adds its band features into the stem's slice
  // of the zeroed output (the overlap average; for mrf_forward_separate the features times
  // stft_repr, so the masks are never stored)
  const int BT = B * T;
  const long long per_stem = (long long)R * T * 2;  // one stem's masks of one window
  cudaMemsetAsync(out, 0, sizeof(float) * (size_t)B * c.num_stems * per_stem, st);
  for (int s = 0; s < c.num_stems; ++s) {
    const int w0 = wm0 + s * n_mask_maps;
    GemmParams p = base_params(h, BT, D, kBnWide, f->g_m0, nb, nb * cdiv(MH, kBnWide));
    p.a_mode = 1;
    p.ss_in = c.depth > 0 ? f->ssx : nullptr;  // 1 / |x| of the deferred last output norm
    p.ss_in_parts = f->parts_res;
    p.nb = nb;
    p.bias = f->mb[s][0]; p.out_h = f->H1; p.ldo = MH; p.out_group_stride = MBT * MH;
    gemm(h, "gemm_mask_tanh", kTcTanh, mXband, wmaps[w0], p, &mH1o);
    __half *cur = f->H1, *nxt = f->H2;
    const CUtensorMap *mcur = &mH1, *mnxt = &mH2;
    const CUtensorMap *ocur = &mH1o, *onxt = &mH2o;
    for (int i = 1; i < c.mask_depth; ++i) {
      p = base_params(h, BT, MH, kBnWide, f->g_mid, nb, nb * cdiv(MH, kBnWide));
      p.bias = f->mb[s][i]; p.out_h = nxt; p.ldo = MH; p.out_group_stride = MBT * MH;
      gemm(h, "gemm_mask_tanh", kTcTanh, *mcur, wmaps[w0 + i], p, onxt);
      std::swap(cur, nxt);
      std::swap(mcur, mnxt);
      std::swap(ocur, onxt);
    }
    p = base_params(h, BT, MH, kBnWide, f->g_last, nb, f->n_last_tiles);
    p.bias = f->mb_last[s];
    p.feat_row = h->d_feat_row; p.row_weight = h->d_row_weight;
    p.masks = out + s * per_stem; p.mask_bstride = c.num_stems * per_stem;
    p.spec = h->apply_masks ? in : nullptr;
    p.B = B; p.T = T; p.R = R;
    gemm(h, "gemm_mask_glu", kTcGlu, *mcur, wmaps[w0 + c.mask_depth], p);
  }
}

}  // namespace mrf

namespace mrf {

// ------------------------------------------------------------------ caller-provided workspace
// Lay the fp16 schedule's per-forward workspace out in one region of `bytes` at `base`
// (256-byte aligned pieces, the same sizes as the handle's own workspace) and, if `apply`,
// point the schedule at it; returns the bytes needed.  `saved` receives the handle's own
// pointers so that fp16_restore_workspace can put them back.
size_t fp16_workspace_layout(mrf_handle *h, void *base, bool apply, Fp16Workspace *saved,
                             size_t *qkv_offset, size_t *qkv_bytes) {
  Fp16State *f = h->f16;
  const mrf_config &c = h->cfg;
  const int nb = c.num_bands, D = c.dim, H = c.heads, A = attn_out_width(c), FF = c.ff_mult * D, MH = c.mask_hidden;
  const long long MBT = (long long)c.max_batch * c.max_frames, NT = MBT * nb;
  size_t off = 0;
  auto take = [&](size_t n) {
    const size_t o = off;
    off += (n + 255) & ~size_t(255);
    return o;
  };
  const size_t parts = (size_t)std::max(f->parts_res, f->parts_bs);
  const size_t oA = take((size_t)nb * MBT * f->k_bs * 2), oXh = take(NT * D * 2),
               oss = take(NT * 4 * parts), ossx = take(NT * 4 * parts), ossg = take(NT * 4 * parts);
  const size_t oQ = take(NT * f->ldq * 2);
  const size_t oO = take(NT * A * 2), oHh = take(NT * FF * 2), oH1 = take((size_t)nb * MBT * MH * 2),
               oH2 = take((size_t)nb * MBT * MH * 2);
  (void)H;
  if (qkv_offset) *qkv_offset = oQ;
  if (qkv_bytes) *qkv_bytes = oO - oQ;
  if (apply && f) {
    if (saved) *saved = {f->ss, f->Xh, f->QKV, f->O, f->Hh, f->H1, f->H2, f->A_bs, f->ssx, f->ssg};
    uint8_t *b = static_cast<uint8_t *>(base);
    f->A_bs = reinterpret_cast<__half *>(b + oA);
    f->Xh = reinterpret_cast<__half *>(b + oXh);
    f->ss = reinterpret_cast<float *>(b + oss);
    f->ssx = reinterpret_cast<float *>(b + ossx);
    f->ssg = reinterpret_cast<float *>(b + ossg);
    f->QKV = reinterpret_cast<__half *>(b + oQ);
    f->O = reinterpret_cast<__half *>(b + oO);
    f->Hh = reinterpret_cast<__half *>(b + oHh);
    f->H1 = reinterpret_cast<__half *>(b + oH1);
    f->H2 = reinterpret_cast<__half *>(b + oH2);
  }
  return off;
}

void fp16_restore_workspace(mrf_handle *h, const Fp16Workspace &s) {
  Fp16State *f = h->f16;
  f->ss = s.ss; f->Xh = s.Xh; f->QKV = s.QKV;
  f->O = s.O; f->Hh = s.Hh; f->H1 = s.H1; f->H2 = s.H2; f->A_bs = s.A_bs; f->ssx = s.ssx; f->ssg = s.ssg;
}

}  // namespace mrf
