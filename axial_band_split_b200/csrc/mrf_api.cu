// C ABI of the library (include/mrf.h): configuration and weight-table validation, weight
// repacking, workspace, the forward schedules, CUDA-graph replay and kernel timing.
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <algorithm>
#include <map>
#include <string>
#include <vector>

#include "mrf_handle.h"

using namespace mrf;

namespace {

thread_local std::string g_create_error;

mrf_status fail(mrf_handle *h, mrf_status s, const std::string &msg) {
  if (h) h->err = msg;
  else g_create_error = msg;
  return s;
}

bool cuda_ok(mrf_handle *h, cudaError_t e, const char *what, mrf_status *st) {
  if (e == cudaSuccess) return true;
  *st = fail(h, e == cudaErrorMemoryAllocation ? MRF_ENOMEM : MRF_ECUDA,
             std::string(what) + ": " + cudaGetErrorString(e));
  cudaGetLastError();
  return false;
}

std::string validate_config(const mrf_config &c) {
  if (c.sample_rate < 8000 || c.sample_rate > 384000) return "sample_rate out of range";
  if (c.n_fft < 16 || c.n_fft > 16384 || (c.n_fft & (c.n_fft - 1))) return "n_fft must be a power of two in [16, 16384]";
  if (c.audio_channels < 1 || c.audio_channels > 2) return "audio_channels must be 1 or 2";
  if (c.num_bands < 1 || c.num_bands > 128) return "num_bands out of range";
  if (c.dim < 16 || c.dim > 1024 || c.dim % 16) return "dim must be a multiple of 16 in [16, 1024]";
  if (c.depth < 0 || c.depth > 64) return "depth out of range";
  if (c.heads < 1 || c.heads > 32) return "heads out of range";
  if (c.dim_head < 2 || c.dim_head > 128 || (c.dim_head & 1)) return "dim_head must be even and <= 128";
  if (c.dim_head_v < 0 || c.dim_head_v > c.dim_head || (c.dim_head_v & 1) || head_v(c) > 64)
    return "dim_head_v must be 0 or even, at most dim_head and at most 64";
  if (c.ff_mult < 1 || c.ff_mult > 8) return "ff_mult out of range";
  if (c.mask_hidden < 16 || c.mask_hidden > 8192) return "mask_hidden out of range";
  if (c.mask_depth < 1 || c.mask_depth > 4) return "mask_depth out of range";
  if (c.ff_act != 0 && c.ff_act != 1) return "ff_act must be 0 (GELU) or 1 (GEGLU)";
  if (c.num_stems < 1 || c.num_stems > 4) return "num_stems must be in [1, 4]";
  if (c.max_batch < 1 || c.max_frames < 1) return "max_batch and max_frames must be >= 1";
  if ((long long)c.max_batch * c.max_frames > (1LL << 22)) return "max_batch * max_frames too large";
  if (!(c.rope_theta > 1.f)) return "rope_theta must be > 1";
  if (c.compute != MRF_FP16 && c.compute != MRF_BF16 && c.compute != MRF_FP32_DEBUG) return "compute mode not implemented";
  return "";
}

// Expected weight names and shapes from the configuration and the band tables.
std::map<std::string, std::vector<int64_t>> expected_weights(const mrf_config &c, const BandTables &t) {
  std::map<std::string, std::vector<int64_t>> e;
  const int64_t D = c.dim, A = attn_out_width(c), QKV = qkv_width(c), H = c.heads, FF = (int64_t)c.ff_mult * c.dim,
                MH = c.mask_hidden;
  for (int k = 0; k < c.num_bands; ++k) {
    const std::string p = "band_split.to_features." + std::to_string(k) + ".";
    e[p + "0.gamma"] = {t.width[k]};
    e[p + "1.weight"] = {D, t.width[k]};
    e[p + "1.bias"] = {D};
  }
  for (int l = 0; l < c.depth; ++l)
    for (int a = 0; a < 2; ++a) {
      const std::string p = "layers." + std::to_string(l) + "." + std::to_string(a) + ".";
      e[p + "layers.0.0.norm.gamma"] = {D};
      e[p + "layers.0.0.to_qkv.weight"] = {QKV, D};
      e[p + "layers.0.0.to_gates.weight"] = {H, D};
      e[p + "layers.0.0.to_gates.bias"] = {H};
      e[p + "layers.0.0.to_out.0.weight"] = {D, A};
      e[p + "layers.0.1.net.0.gamma"] = {D};
      const int64_t F1 = c.ff_act == 1 ? 2 * FF : FF;  // GEGLU: value and gate halves
      e[p + "layers.0.1.net.1.weight"] = {F1, D};
      e[p + "layers.0.1.net.1.bias"] = {F1};
      e[p + "layers.0.1.net.4.weight"] = {D, FF};
      e[p + "layers.0.1.net.4.bias"] = {D};
      e[p + "norm.gamma"] = {D};
    }
  for (int s = 0; s < c.num_stems; ++s)
  for (int k = 0; k < c.num_bands; ++k) {
    const std::string p = "mask_estimators." + std::to_string(s) + ".to_freqs." + std::to_string(k) + ".0.";
    std::vector<int64_t> dims = {D};
    for (int i = 0; i < c.mask_depth; ++i) dims.push_back(MH);
    dims.push_back(2 * (int64_t)t.width[k]);
    for (int i = 0; i + 1 < (int)dims.size(); ++i) {
      e[p + std::to_string(2 * i) + ".weight"] = {dims[i + 1], dims[i]};
      e[p + std::to_string(2 * i) + ".bias"] = {dims[i + 1]};
    }
  }
  return e;
}

mrf_status read_weights(const mrf_config &c, const BandTables &t, const mrf_tensor *w, int n,
                        std::map<std::string, HostW> *out) {
  auto exp = expected_weights(c, t);
  for (int i = 0; i < n; ++i) {
    const mrf_tensor &x = w[i];
    if (!x.name) return fail(nullptr, MRF_EWEIGHTS, "weight " + std::to_string(i) + " has no name");
    const std::string name(x.name);
    auto it = exp.find(name);
    if (it == exp.end()) return fail(nullptr, MRF_EWEIGHTS, "unexpected weight " + name);
    if (out->count(name)) return fail(nullptr, MRF_EWEIGHTS, "duplicate weight " + name);
    if (x.dtype != MRF_DTYPE_F32 && x.dtype != MRF_DTYPE_F16)
      return fail(nullptr, MRF_EWEIGHTS, "weight " + name + ": dtype must be f32 or f16");
    if (!x.host_data) return fail(nullptr, MRF_EINVAL, "weight " + name + ": null data");
    const auto &sh = it->second;
    if (x.ndim != (int)sh.size()) return fail(nullptr, MRF_ESHAPE, "weight " + name + ": wrong rank");
    size_t cnt = 1;
    for (int d = 0; d < x.ndim; ++d) {
      if (x.shape[d] != sh[d]) {
        char buf[160];
        snprintf(buf, sizeof buf, "weight %s: dim %d is %lld, expected %lld", name.c_str(), d,
                 (long long)x.shape[d], (long long)sh[d]);
        return fail(nullptr, MRF_ESHAPE, buf);
      }
      cnt *= (size_t)sh[d];
    }
    HostW hw;
    hw.shape = sh;
    hw.v.resize(cnt);
    if (x.dtype == MRF_DTYPE_F32) {
      memcpy(hw.v.data(), x.host_data, cnt * sizeof(float));
    } else {
      const __half *src = static_cast<const __half *>(x.host_data);
      for (size_t j = 0; j < cnt; ++j) hw.v[j] = __half2float(src[j]);
    }
    (*out)[name] = std::move(hw);
  }
  for (auto &kv : exp)
    if (!out->count(kv.first)) return fail(nullptr, MRF_EWEIGHTS, "missing weight " + kv.first);
  return MRF_OK;
}

}  // namespace

void *mrf_handle::alloc_bytes(size_t bytes) {
  if (fail_alloc_after >= 0 && n_allocs >= fail_alloc_after) return nullptr;
  void *p = nullptr;
  if (cudaMalloc(&p, bytes ? bytes : 16) != cudaSuccess) {
    cudaGetLastError();
    return nullptr;
  }
  ++n_allocs;
  allocs.push_back(p);
  return p;
}

bool mrf_handle::upload(void *dst, const void *src, size_t bytes) {
  return cudaMemcpy(dst, src, bytes, cudaMemcpyHostToDevice) == cudaSuccess;
}

void mrf_handle::begin(const char *name) {
  ++launch_counter;
  if (!timing) return;
  cudaEvent_t a, b;
  cudaEventCreate(&a);
  cudaEventCreate(&b);
  cudaEventRecord(a, cur_stream);
  pending.push_back({name, a, b});
}

void mrf_handle::end() {
  if (!timing || pending.empty()) return;
  cudaEventRecord(pending.back().e1, cur_stream);
}

// ------------------------------------------------------------------ packing (fp32 path)
namespace {

mrf_status pack_common(mrf_handle *h, std::map<std::string, HostW> &W) {
  const mrf_config &c = h->cfg;
  const BandTables &t = h->tab;
  const int nb = c.num_bands, D = c.dim;
  mrf_status st = MRF_OK;
  // tables
  h->d_feat_row = h->alloc<int32_t>(t.feat_row.size());
  h->d_feat_c = h->alloc<int32_t>(t.feat_c.size());
  h->d_src0 = h->alloc<int32_t>(t.src0.size());
  h->d_src1 = h->alloc<int32_t>(t.src1.size());
  h->d_row_weight = h->alloc<float>(t.row_weight.size());
  h->d_bands = h->alloc<BandDesc>(nb);
  if (!h->d_feat_row || !h->d_feat_c || !h->d_src0 || !h->d_src1 || !h->d_row_weight || !h->d_bands)
    return fail(h, MRF_ENOMEM, "device allocation failed (tables)");
  std::vector<BandDesc> bd(nb);
  long long woff = 0, w3off = 0;
  h->max_width = 0;
  for (int k = 0; k < nb; ++k) {
    bd[k] = {t.width[k], t.feat_off[k], (int)woff, (int)w3off};
    woff += (long long)t.width[k] * D;
    w3off += 2LL * t.width[k] * c.mask_hidden;
    h->max_width = std::max(h->max_width, t.width[k]);
  }
  h->bands = bd;
  // rope table: positions 0 .. max(max_frames, nb) - 1
  const int npos = std::max(c.max_frames, nb), half = c.dim_head / 2;
  std::vector<float2> rope((size_t)npos * half);
  for (int p = 0; p < npos; ++p)
    for (int i = 0; i < half; ++i) {
      const double ang = p * std::pow((double)c.rope_theta, -2.0 * i / c.dim_head);
      rope[(size_t)p * half + i] = make_float2((float)std::cos(ang), (float)std::sin(ang));
    }
  h->d_rope = h->alloc<float2>(rope.size());
  if (!h->d_rope) return fail(h, MRF_ENOMEM, "device allocation failed (rope)");
  // band split: gamma*sqrt(d_in) folded, transposed to [width][D] per band
  std::vector<float> bs((size_t)woff), bsb((size_t)nb * D);
  for (int k = 0; k < nb; ++k) {
    const std::string p = "band_split.to_features." + std::to_string(k) + ".";
    const auto &g = W[p + "0.gamma"].v;
    const auto &w = W[p + "1.weight"].v;
    const auto &b = W[p + "1.bias"].v;
    const int wd = t.width[k];
    const double s = std::sqrt((double)wd);
    for (int d = 0; d < D; ++d)
      for (int e = 0; e < wd; ++e)
        bs[bd[k].w_off + (size_t)e * D + d] = (float)((double)w[(size_t)d * wd + e] * g[e] * s);
    for (int d = 0; d < D; ++d) bsb[(size_t)k * D + d] = b[d];
  }
  h->w_bs = h->alloc<float>(bs.size());
  h->b_bs = h->alloc<float>(bsb.size());
  h->status = h->alloc<unsigned>(4);
  if (!h->w_bs || !h->b_bs || !h->status) return fail(h, MRF_ENOMEM, "device allocation failed (band split)");
  bool ok = h->upload(h->d_feat_row, t.feat_row.data(), t.feat_row.size() * 4) &&
            h->upload(h->d_feat_c, t.feat_c.data(), t.feat_c.size() * 4) &&
            h->upload(h->d_src0, t.src0.data(), t.src0.size() * 4) &&
            h->upload(h->d_src1, t.src1.data(), t.src1.size() * 4) &&
            h->upload(h->d_row_weight, t.row_weight.data(), t.row_weight.size() * 4) &&
            h->upload(h->d_bands, bd.data(), bd.size() * sizeof(BandDesc)) &&
            h->upload(h->d_rope, rope.data(), rope.size() * sizeof(float2)) &&
            h->upload(h->w_bs, bs.data(), bs.size() * 4) &&
            h->upload(h->b_bs, bsb.data(), bsb.size() * 4);
  if (!ok || cudaMemset(h->status, 0, 16) != cudaSuccess)
    return fail(h, MRF_ECUDA, "upload of tables failed");
  return st;
}

float *upload_f32(mrf_handle *h, const std::vector<float> &v) {
  float *p = h->alloc<float>(v.size());
  if (p && !h->upload(p, v.data(), v.size() * 4)) return nullptr;
  return p;
}

std::vector<float> scaled_gain(const std::vector<float> &g) {
  std::vector<float> o(g.size());
  const double s = std::sqrt((double)g.size());
  for (size_t i = 0; i < g.size(); ++i) o[i] = (float)(g[i] * s);
  return o;
}

// Mask-head last layer with its rows interleaved (value e, gate e) so that a GLU pair is
// two adjacent output columns.
void interleave_glu(const std::vector<float> &w, const std::vector<float> &b, int width, int hidden,
                    std::vector<float> *wo, std::vector<float> *bo) {
  for (int e = 0; e < width; ++e) {
    wo->insert(wo->end(), w.begin() + (size_t)e * hidden, w.begin() + (size_t)(e + 1) * hidden);
    wo->insert(wo->end(), w.begin() + (size_t)(width + e) * hidden,
               w.begin() + (size_t)(width + e + 1) * hidden);
    bo->push_back(b[e]);
    bo->push_back(b[width + e]);
  }
}

mrf_status pack_f32(mrf_handle *h, std::map<std::string, HostW> &W) {
  const mrf_config &c = h->cfg;
  const BandTables &t = h->tab;
  const int nb = c.num_bands, MH = c.mask_hidden;
  const long long MBT = (long long)c.max_batch * c.max_frames;
  h->trf.resize(2 * c.depth);
  for (int l = 0; l < c.depth; ++l)
    for (int a = 0; a < 2; ++a) {
      const std::string p = "layers." + std::to_string(l) + "." + std::to_string(a) + ".";
      TrF32 &x = h->trf[2 * l + a];
      x.g_attn = upload_f32(h, scaled_gain(W[p + "layers.0.0.norm.gamma"].v));
      x.wqkv = upload_f32(h, W[p + "layers.0.0.to_qkv.weight"].v);
      x.wg = upload_f32(h, W[p + "layers.0.0.to_gates.weight"].v);
      x.bg = upload_f32(h, W[p + "layers.0.0.to_gates.bias"].v);
      x.wo = upload_f32(h, W[p + "layers.0.0.to_out.0.weight"].v);
      x.g_ff = upload_f32(h, scaled_gain(W[p + "layers.0.1.net.0.gamma"].v));
      if (c.ff_act == 1) {  // GEGLU: (value, gate) rows paired for the epilogue
        const int FFh = c.ff_mult * c.dim;
        x.w1 = upload_f32(h, interleave_halves(W[p + "layers.0.1.net.1.weight"].v, FFh, c.dim));
        x.b1 = upload_f32(h, interleave_halves(W[p + "layers.0.1.net.1.bias"].v, FFh, 1));
      } else {
        x.w1 = upload_f32(h, W[p + "layers.0.1.net.1.weight"].v);
        x.b1 = upload_f32(h, W[p + "layers.0.1.net.1.bias"].v);
      }
      x.w2 = upload_f32(h, W[p + "layers.0.1.net.4.weight"].v);
      x.b2 = upload_f32(h, W[p + "layers.0.1.net.4.bias"].v);
      x.g_out = upload_f32(h, scaled_gain(W[p + "norm.gamma"].v));
      if (!x.g_attn || !x.wqkv || !x.wg || !x.bg || !x.wo || !x.g_ff || !x.w1 || !x.b1 || !x.w2 ||
          !x.b2 || !x.g_out)
        return fail(h, MRF_ENOMEM, "device allocation failed (transformer weights)");
    }
  // mask heads (one per stem): layers 0 .. mask_depth-1 stacked per band, last layer interleaved
  h->mf.w.resize(c.num_stems);
  h->mf.b.resize(c.num_stems);
  h->mf.w_last.resize(c.num_stems);
  h->mf.b_last.resize(c.num_stems);
  for (int s = 0; s < c.num_stems; ++s) {
    std::vector<std::vector<float>> mw(c.mask_depth), mb(c.mask_depth);
    std::vector<float> w_last, b_last;
    for (int k = 0; k < nb; ++k) {
      const std::string p = "mask_estimators." + std::to_string(s) + ".to_freqs." + std::to_string(k) + ".0.";
      for (int i = 0; i < c.mask_depth; ++i) {
        const auto &w = W[p + std::to_string(2 * i) + ".weight"].v;
        const auto &b = W[p + std::to_string(2 * i) + ".bias"].v;
        mw[i].insert(mw[i].end(), w.begin(), w.end());
        mb[i].insert(mb[i].end(), b.begin(), b.end());
      }
      const std::string q = p + std::to_string(2 * c.mask_depth);
      interleave_glu(W[q + ".weight"].v, W[q + ".bias"].v, t.width[k], MH, &w_last, &b_last);
    }
    h->mf.w[s].resize(c.mask_depth);
    h->mf.b[s].resize(c.mask_depth);
    for (int i = 0; i < c.mask_depth; ++i) {
      h->mf.w[s][i] = upload_f32(h, mw[i]);
      h->mf.b[s][i] = upload_f32(h, mb[i]);
      if (!h->mf.w[s][i] || !h->mf.b[s][i]) return fail(h, MRF_ENOMEM, "device allocation failed (mask head)");
    }
    h->mf.w_last[s] = upload_f32(h, w_last);
    h->mf.b_last[s] = upload_f32(h, b_last);
    if (!h->mf.w_last[s] || !h->mf.b_last[s]) return fail(h, MRF_ENOMEM, "device allocation failed (mask head)");
  }
  // groups of the mask-head GEMMs
  const int D = c.dim;
  std::vector<SimtGroup> g0(nb), g1(nb), g2(nb);
  for (int k = 0; k < nb; ++k) {
    g0[k] = {(long long)k * D, (long long)k * MH * D, (long long)k * MBT * MH, (long long)k * MH, nb * D, MH, MH, 0};
    g1[k] = {(long long)k * MBT * MH, (long long)k * MH * MH, (long long)k * MBT * MH, (long long)k * MH, MH, MH, MH, 0};
    g2[k] = {(long long)k * MBT * MH, (long long)h->bands[k].w3_off, (long long)t.feat_off[k],
             2LL * t.feat_off[k], MH, t.n_feat(), 2 * t.width[k], 0};
  }
  h->mf.g_first = h->alloc<SimtGroup>(nb);
  h->mf.g_mid = h->alloc<SimtGroup>(nb);
  h->mf.g_last = h->alloc<SimtGroup>(nb);
  if (!h->mf.g_first || !h->mf.g_mid || !h->mf.g_last) return fail(h, MRF_ENOMEM, "device allocation failed");
  if (!h->upload(h->mf.g_first, g0.data(), nb * sizeof(SimtGroup)) ||
      !h->upload(h->mf.g_mid, g1.data(), nb * sizeof(SimtGroup)) ||
      !h->upload(h->mf.g_last, g2.data(), nb * sizeof(SimtGroup)))
    return fail(h, MRF_ECUDA, "upload failed");
  // trunk groups (one group each)
  const int A = attn_out_width(c), QKVW = qkv_width(c), H = c.heads, FF = c.ff_mult * D;
  SimtGroup tg[5] = {
      {0, 0, 0, 0, D, QKVW, QKVW, 0},    // qkv
      {0, 0, 0, 0, D, H, H, 0},          // gates
      {0, 0, 0, 0, A, D, D, 0},          // out
      {0, 0, 0, 0, D, FF, c.ff_act == 1 ? 2 * FF : FF, 0},  // ff1 (GEGLU: 2 FF paired columns, FF outputs)
      {0, 0, 0, 0, FF, D, D, 0},         // ff2
  };
  h->d_tgroups = h->alloc<SimtGroup>(5);
  if (!h->d_tgroups || !h->upload(h->d_tgroups, tg, sizeof tg)) return fail(h, MRF_ENOMEM, "device allocation failed");
  // workspace
  const long long NT = MBT * nb;
  h->ws.X = h->alloc<float>(NT * D);
  h->ws.Xa = h->alloc<float>(NT * D);
  h->ws.QKV = h->alloc<float>(NT * QKVW);
  h->ws.G = h->alloc<float>(NT * H);
  h->ws.Q = h->alloc<float>(NT * H * c.dim_head);
  h->ws.K = h->alloc<float>(NT * H * c.dim_head);
  h->ws.V = h->alloc<float>(NT * A);
  h->ws.O = h->alloc<float>(NT * A);
  h->ws.Hf = h->alloc<float>(NT * FF);
  h->ws.H1 = h->alloc<float>((long long)nb * MBT * MH);
  h->ws.H2 = h->alloc<float>((long long)nb * MBT * MH);
  h->ws.Mg = h->alloc<float>(MBT * t.n_feat());
  if (!h->ws.X || !h->ws.Xa || !h->ws.QKV || !h->ws.G || !h->ws.Q || !h->ws.K || !h->ws.V ||
      !h->ws.O || !h->ws.Hf || !h->ws.H1 || !h->ws.H2 || !h->ws.Mg)
    return fail(h, MRF_ENOMEM, "device allocation failed (workspace)");
  return MRF_OK;
}

// ------------------------------------------------------------------ fp32 debug schedule
void schedule_f32(mrf_handle *h, const float *in, float *out, int B, int T) {
  const mrf_config &c = h->cfg;
  const int nb = c.num_bands, D = c.dim, H = c.heads, dh = c.dim_head, dv = head_v(c), A = attn_out_width(c),
            QKVW = qkv_width(c), FF = c.ff_mult * D;
  const long long NT = (long long)B * T * nb;
  const int R = h->tab.n_freqs * h->tab.channels;
  cudaStream_t st = h->cur_stream;
  Workspace &w = h->ws;
  SimtGroup *tg = h->d_tgroups;
  h->begin("band_split");
  launch_band_split(in, h->d_feat_row, h->d_feat_c, h->d_bands, nb, h->w_bs, h->b_bs, D, B, T, R,
                    w.X, nullptr, nullptr, st, h->max_width);
  h->end();
  for (int i = 0; i < 2 * c.depth; ++i) {
    const TrF32 &x = h->trf[i];
    const int axis = i & 1;
    h->begin("rownorm_f32"); launch_rownorm_f32(w.X, x.g_attn, w.Xa, NT, D, st); h->end();
    h->begin("gemm_f32"); launch_gemm_f32(w.Xa, x.wqkv, nullptr, w.QKV, tg + 0, 1, (int)NT, D, QKVW, kEpiStore, st); h->end();
    h->begin("gemm_f32"); launch_gemm_f32(w.Xa, x.wg, x.bg, w.G, tg + 1, 1, (int)NT, D, H, kEpiSigmoid, st); h->end();
    h->begin("rope_split_f32"); launch_rope_split_f32(w.QKV, h->d_rope, w.Q, w.K, w.V, B, T, nb, H, dh, dv, axis, st); h->end();
    h->begin("attention_f32"); launch_attention_f32(w.Q, w.K, w.V, w.G, w.O, B, T, nb, H, dh, dv, axis, st); h->end();
    h->begin("gemm_f32"); launch_gemm_f32(w.O, x.wo, nullptr, w.X, tg + 2, 1, (int)NT, A, D, kEpiResidual, st); h->end();
    h->begin("rownorm_f32"); launch_rownorm_f32(w.X, x.g_ff, w.Xa, NT, D, st); h->end();
    if (c.ff_act == 1) {
      h->begin("gemm_f32"); launch_gemm_f32(w.Xa, x.w1, x.b1, w.Hf, tg + 3, 1, (int)NT, D, 2 * FF, kEpiGeglu, st); h->end();
    } else {
      h->begin("gemm_f32"); launch_gemm_f32(w.Xa, x.w1, x.b1, w.Hf, tg + 3, 1, (int)NT, D, FF, kEpiGelu, st); h->end();
    }
    h->begin("gemm_f32"); launch_gemm_f32(w.Hf, x.w2, x.b2, w.X, tg + 4, 1, (int)NT, FF, D, kEpiResidual, st); h->end();
    h->begin("rownorm_f32"); launch_rownorm_f32(w.X, x.g_out, w.X, NT, D, st); h->end();
  }
  const int M = B * T, MH = c.mask_hidden;
  const long long per_stem = (long long)R * T * 2;  // one stem's masks of one window
  for (int s = 0; s < c.num_stems; ++s) {
    h->begin("gemm_f32");
    launch_gemm_f32(w.X, h->mf.w[s][0], h->mf.b[s][0], w.H1, h->mf.g_first, nb, M, D, MH, kEpiTanh, st);
    h->end();
    float *cur = w.H1, *nxt = w.H2;
    for (int i = 1; i < c.mask_depth; ++i) {
      h->begin("gemm_f32");
      launch_gemm_f32(cur, h->mf.w[s][i], h->mf.b[s][i], nxt, h->mf.g_mid, nb, M, MH, MH, kEpiTanh, st);
      h->end();
      std::swap(cur, nxt);
    }
    h->begin("gemm_f32");
    launch_gemm_f32(cur, h->mf.w_last[s], h->mf.b_last[s], w.Mg, h->mf.g_last, nb, M, MH, 2 * h->max_width,
                    kEpiGlu, st);
    h->end();
    h->begin("overlap_average");
    launch_overlap_average(w.Mg, h->tab.n_feat(), h->d_src0, h->d_src1, h->d_row_weight, out + s * per_stem,
                           c.num_stems * per_stem, h->apply_masks ? in : nullptr, B, T, R, st);
    h->end();
  }
}

void run_schedule(mrf_handle *h, const float *in, float *out, int B, int T) {
  h->launch_counter = 0;
  h->sched_error.clear();
  if (h->cfg.compute == MRF_FP32_DEBUG) schedule_f32(h, in, out, B, T);
  else schedule_fp16(h, in, out, B, T);
  h->last_launches = h->launch_counter;
  h->last_B = B;
  h->last_T = T;
  h->last_static = false;
}

}  // namespace

// ------------------------------------------------------------------ C ABI
extern "C" {

mrf_status mrf_band_tables(const mrf_config *cfg, int32_t *first_bin, int32_t *last_bin,
                           int32_t *width, int32_t *feat_row, float *row_weight, int32_t *n_feat) {
  if (!cfg) return fail(nullptr, MRF_EINVAL, "null config");
  BandTables t;
  const std::string e = build_band_tables(cfg->sample_rate, cfg->n_fft, cfg->num_bands,
                                          cfg->audio_channels, cfg->zero_dc != 0, &t);
  if (!e.empty()) return fail(nullptr, MRF_EINVAL, e);
  const int nb = cfg->num_bands;
  if (first_bin) memcpy(first_bin, t.first_bin.data(), nb * 4);
  if (last_bin) memcpy(last_bin, t.last_bin.data(), nb * 4);
  if (width) memcpy(width, t.width.data(), nb * 4);
  if (feat_row) memcpy(feat_row, t.feat_row.data(), t.feat_row.size() * 4);
  if (row_weight) memcpy(row_weight, t.row_weight.data(), t.row_weight.size() * 4);
  if (n_feat) *n_feat = t.n_feat();
  return MRF_OK;
}

mrf_status mrf_create(const mrf_config *cfg, const mrf_tensor *w, int n_w, mrf_handle **out) {
  g_create_error.clear();
  if (!out) return fail(nullptr, MRF_EINVAL, "null output handle pointer");
  *out = nullptr;
  if (!cfg) return fail(nullptr, MRF_EINVAL, "null config");
  if (!w || n_w <= 0) return fail(nullptr, MRF_EINVAL, "empty weight table");
  const std::string ce = validate_config(*cfg);
  if (!ce.empty()) return fail(nullptr, ce.find("implemented") != std::string::npos ? MRF_EUNSUPPORTED : MRF_EINVAL, ce);
  BandTables tab;
  const std::string te = build_band_tables(cfg->sample_rate, cfg->n_fft, cfg->num_bands,
                                           cfg->audio_channels, cfg->zero_dc != 0, &tab);
  if (!te.empty()) return fail(nullptr, MRF_EINVAL, te);
  if (cfg->compute != MRF_FP32_DEBUG) {
    const std::string fe = fp16_supported(*cfg, tab);
    if (!fe.empty()) return fail(nullptr, MRF_EUNSUPPORTED, fe);
  }
  std::map<std::string, HostW> W;
  mrf_status st = read_weights(*cfg, tab, w, n_w, &W);
  if (st != MRF_OK) return st;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return fail(nullptr, MRF_ECUDA, std::string("no CUDA device: ") + cudaGetErrorString(e));
  }
  mrf_handle *h = new (std::nothrow) mrf_handle();
  if (!h) return fail(nullptr, MRF_ENOMEM, "host allocation failed");
  h->cfg = *cfg;
  h->tab = std::move(tab);
  h->device = dev;
  if (const char *f = getenv("MRF_FAIL_ALLOC_AFTER")) h->fail_alloc_after = atoi(f);
  st = pack_common(h, W);
  if (st == MRF_OK) st = (cfg->compute == MRF_FP32_DEBUG) ? pack_f32(h, W) : pack_fp16(h, W);
  if (st == MRF_OK && cudaStreamCreateWithFlags(&h->cap_stream, cudaStreamNonBlocking) != cudaSuccess)
    st = fail(h, MRF_ECUDA, "stream creation failed");
  if (st == MRF_OK && cudaDeviceSynchronize() != cudaSuccess) st = fail(h, MRF_ECUDA, "device error during create");
  if (st != MRF_OK) {
    g_create_error = h->err;
    mrf_destroy(h);
    cudaGetLastError();
    return st;
  }
  *out = h;
  return MRF_OK;
}

}  // extern "C"

namespace {

// mrf_forward (apply = false: masks out) and mrf_forward_separate (apply = true: the masks
// multiplied into stft_repr).  The output holds B x num_stems x rows x T x 2 floats.
mrf_status forward_impl(mrf_handle *h, const float *in, float *out, int B, int T, void *stream, bool apply) {
  if (!h) return fail(nullptr, MRF_EINVAL, "null handle");
  if (!in || !out) return fail(h, MRF_EINVAL, "null stft_repr or output pointer");
  if (B < 1 || B > h->cfg.max_batch || T < 1 || T > h->cfg.max_frames)
    return fail(h, MRF_ESHAPE, "B or T outside [1, max_batch] x [1, max_frames]");
  if ((reinterpret_cast<uintptr_t>(in) | reinterpret_cast<uintptr_t>(out)) & 15)
    return fail(h, MRF_EINVAL, "stft_repr and the output must be 16-byte aligned");
  const size_t bytes = (size_t)B * h->tab.n_freqs * h->tab.channels * T * 2 * sizeof(float);
  const size_t out_bytes = bytes * h->cfg.num_stems;
  const char *a = reinterpret_cast<const char *>(in), *b = reinterpret_cast<const char *>(out);
  if (a < b + out_bytes && b < a + bytes) return fail(h, MRF_EINVAL, "stft_repr and the output overlap");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaGetLastError();
  mrf_status s = MRF_OK;
  h->apply_masks = apply;
  if (h->timing || !h->use_graph || h->stall_test) {  // a stalled forward is never recorded into a graph
    h->cur_stream = st;
    run_schedule(h, in, out, B, T);
    if (!h->sched_error.empty()) return fail(h, MRF_ECUDA, h->sched_error);
    if (!cuda_ok(h, cudaGetLastError(), "kernel launch", &s)) return s;
    return MRF_OK;
  }
  // CUDA graph per (B, T, in, out, apply): captured once on an internal stream, replayed on `st`
  GraphKey key{B, T, in, out, apply};
  cudaGraphExec_t exec = nullptr;
  for (auto &g : h->graphs)
    if (g.key == key) exec = g.exec;
  if (!exec) {
    h->cur_stream = h->cap_stream;
    if (!cuda_ok(h, cudaStreamBeginCapture(h->cap_stream, cudaStreamCaptureModeThreadLocal), "begin capture", &s)) return s;
    run_schedule(h, in, out, B, T);
    cudaGraph_t graph = nullptr;
    cudaError_t e = cudaStreamEndCapture(h->cap_stream, &graph);
    if (!h->sched_error.empty()) {
      if (graph) cudaGraphDestroy(graph);
      return fail(h, MRF_ECUDA, h->sched_error);
    }
    if (!cuda_ok(h, e, "end capture", &s)) return s;
    e = cudaGraphInstantiate(&exec, graph, 0);
    cudaGraphDestroy(graph);
    if (!cuda_ok(h, e, "graph instantiate", &s)) return s;
    if (h->graphs.size() >= 8) {
      cudaGraphExecDestroy(h->graphs.front().exec);
      h->graphs.erase(h->graphs.begin());
    }
    h->graphs.push_back({key, exec, h->last_launches});
  }
  for (auto &g : h->graphs)
    if (g.key == key) { h->last_launches = g.launches; h->last_B = B; h->last_T = T; h->last_static = false; }
  if (!cuda_ok(h, cudaGraphLaunch(exec, st), "graph launch", &s)) return s;
  return MRF_OK;
}

}  // namespace

extern "C" {

mrf_status mrf_forward(mrf_handle *h, const float *in, float *out, int B, int T, void *stream) {
  return forward_impl(h, in, out, B, T, stream, false);
}

mrf_status mrf_forward_separate(mrf_handle *h, const float *in, float *out, int B, int T, void *stream) {
  return forward_impl(h, in, out, B, T, stream, true);
}

}  // extern "C"

namespace {

// The host-buffer pipeline's one-time setup: two device slots of the largest input and output,
// the two copy streams and the ordering events, made on the current device at the first call.
mrf_status host_pipe_init(mrf_handle *h) {
  if (h->io_in[1]) return MRF_OK;
  const size_t maxb = (size_t)h->cfg.max_batch * h->tab.n_freqs * h->tab.channels * h->cfg.max_frames * 2 * sizeof(float);
  for (int s = 0; s < 2; ++s) {
    if (!h->io_in[s]) h->io_in[s] = static_cast<float *>(h->alloc_bytes(maxb));
    if (!h->io_out[s]) h->io_out[s] = static_cast<float *>(h->alloc_bytes(maxb * h->cfg.num_stems));
    if (!h->io_in[s] || !h->io_out[s]) return fail(h, MRF_ENOMEM, "device allocation failed (io buffers)");
  }
  mrf_status st = MRF_OK;
  if (!h->h2d_stream && !cuda_ok(h, cudaStreamCreateWithFlags(&h->h2d_stream, cudaStreamNonBlocking), "copy stream", &st)) return st;
  if (!h->d2h_stream && !cuda_ok(h, cudaStreamCreateWithFlags(&h->d2h_stream, cudaStreamNonBlocking), "copy stream", &st)) return st;
  cudaEvent_t *evs[8] = {&h->ev_in[0], &h->ev_in[1], &h->ev_fwd[0], &h->ev_fwd[1],
                         &h->ev_out[0], &h->ev_out[1], &h->ev_join, &h->ev_start};
  for (cudaEvent_t *e : evs)
    if (!*e && !cuda_ok(h, cudaEventCreateWithFlags(e, cudaEventDisableTiming), "event", &st)) return st;
  return MRF_OK;
}

// One call of the pipeline on slot io_next: H2D on h2d_stream after the forward that last read
// the slot's input (and, for the first call of a batch, after the work already on `stream`); the
// forward on `stream` after that copy and after the copy that last read the slot's output; D2H on
// d2h_stream after the forward.  (Waiting on an event that was never recorded returns at once,
// which covers a slot's first use.)
mrf_status host_pipe_call(mrf_handle *h, const float *in_host, float *out_host, int B, int T, void *stream) {
  if (!h) return fail(nullptr, MRF_EINVAL, "null handle");
  if (!in_host || !out_host) return fail(h, MRF_EINVAL, "null host buffer");
  if (B < 1 || B > h->cfg.max_batch || T < 1 || T > h->cfg.max_frames)
    return fail(h, MRF_ESHAPE, "B or T outside [1, max_batch] x [1, max_frames]");
  mrf_status s = host_pipe_init(h);
  if (s != MRF_OK) return s;
  const size_t bytes = (size_t)B * h->tab.n_freqs * h->tab.channels * T * 2 * sizeof(float);
  const size_t out_bytes = bytes * h->cfg.num_stems;
  const int k = h->io_next;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (!h->pipe_open) {  // a batch begins: its first copy follows what the caller enqueued before it
    if (!cuda_ok(h, cudaEventRecord(h->ev_start, st), "copy ordering", &s) ||
        !cuda_ok(h, cudaStreamWaitEvent(h->h2d_stream, h->ev_start, 0), "copy ordering", &s))
      return s;
    h->pipe_open = true;
  }
  if (!cuda_ok(h, cudaStreamWaitEvent(h->h2d_stream, h->ev_fwd[k], 0), "copy ordering", &s) ||
      !cuda_ok(h, cudaMemcpyAsync(h->io_in[k], in_host, bytes, cudaMemcpyHostToDevice, h->h2d_stream), "H2D copy", &s) ||
      !cuda_ok(h, cudaEventRecord(h->ev_in[k], h->h2d_stream), "copy ordering", &s) ||
      !cuda_ok(h, cudaStreamWaitEvent(st, h->ev_in[k], 0), "copy ordering", &s) ||
      !cuda_ok(h, cudaStreamWaitEvent(st, h->ev_out[k], 0), "copy ordering", &s))
    return s;
  s = mrf_forward(h, h->io_in[k], h->io_out[k], B, T, stream);
  if (s != MRF_OK) return s;
  if (!cuda_ok(h, cudaEventRecord(h->ev_fwd[k], st), "copy ordering", &s) ||
      !cuda_ok(h, cudaStreamWaitEvent(h->d2h_stream, h->ev_fwd[k], 0), "copy ordering", &s) ||
      !cuda_ok(h, cudaMemcpyAsync(out_host, h->io_out[k], out_bytes, cudaMemcpyDeviceToHost, h->d2h_stream), "D2H copy", &s) ||
      !cuda_ok(h, cudaEventRecord(h->ev_out[k], h->d2h_stream), "copy ordering", &s))
    return s;
  h->io_next = k ^ 1;
  return MRF_OK;
}

}  // namespace

extern "C" {

mrf_status mrf_forward_host_async(mrf_handle *h, const float *in_host, float *out_host, int B, int T, void *stream) {
  return host_pipe_call(h, in_host, out_host, B, T, stream);
}

mrf_status mrf_host_join(mrf_handle *h, void *stream) {
  if (!h) return fail(nullptr, MRF_EINVAL, "null handle");
  if (!h->d2h_stream) return MRF_OK;
  mrf_status s = MRF_OK;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (!cuda_ok(h, cudaEventRecord(h->ev_join, h->d2h_stream), "join", &s) ||
      !cuda_ok(h, cudaStreamWaitEvent(st, h->ev_join, 0), "join", &s))
    return s;
  h->pipe_open = false;
  return MRF_OK;
}

mrf_status mrf_forward_host(mrf_handle *h, const float *in_host, float *out_host, int B, int T,
                            void *stream) {
  mrf_status s = host_pipe_call(h, in_host, out_host, B, T, stream);
  if (s != MRF_OK) return s;
  s = mrf_host_join(h, stream);
  if (s != MRF_OK) return s;
  return mrf_sync_status(h, stream);
}

mrf_status mrf_sync_status(mrf_handle *h, void *stream) {
  if (!h) return fail(nullptr, MRF_EINVAL, "null handle");
  mrf_status s = MRF_OK;
  if (!cuda_ok(h, cudaStreamSynchronize(static_cast<cudaStream_t>(stream)), "stream sync", &s)) return s;
  unsigned word[4] = {0, 0, 0, 0};
  if (!cuda_ok(h, cudaMemcpy(word, h->status, sizeof word, cudaMemcpyDeviceToHost), "status read", &s)) return s;
  if (word[0] != kStatusOk) {
    cudaMemset(h->status, 0, sizeof word);
    char buf[128];
    snprintf(buf, sizeof buf, "a device-side bounded wait expired (code %u, site %u)", word[0], word[1]);
    return fail(h, MRF_ETIMEOUT, buf);
  }
  return MRF_OK;
}

void mrf_destroy(mrf_handle *h) {
  if (!h) return;
  for (auto &g : h->graphs) cudaGraphExecDestroy(g.exec);
  for (auto &p : h->pending) { cudaEventDestroy(p.e0); cudaEventDestroy(p.e1); }
  for (void *p : h->allocs) cudaFree(p);
  for (auto &p : h->sig_scratch) cudaFree(p.first);
  if (h->cap_stream) cudaStreamDestroy(h->cap_stream);
  for (cudaStream_t c : {h->h2d_stream, h->d2h_stream})
    if (c) { cudaStreamSynchronize(c); cudaStreamDestroy(c); }
  for (cudaEvent_t e : {h->ev_in[0], h->ev_in[1], h->ev_fwd[0], h->ev_fwd[1], h->ev_out[0], h->ev_out[1], h->ev_join,
                        h->ev_start})
    if (e) cudaEventDestroy(e);
  destroy_fp16(h);
  delete h;
}

const char *mrf_last_error(const mrf_handle *h) { return h ? h->err.c_str() : g_create_error.c_str(); }

mrf_status mrf_set_timing(mrf_handle *h, int enable) {
  if (!h) return fail(nullptr, MRF_EINVAL, "null handle");
  h->timing = enable != 0;
  return MRF_OK;
}

mrf_status mrf_set_graph(mrf_handle *h, int enable) {
  if (!h) return fail(nullptr, MRF_EINVAL, "null handle");
  h->use_graph = enable != 0;
  return MRF_OK;
}

mrf_status mrf_kernel_times(mrf_handle *h, mrf_kernel_time *out, int max_n, int *n_out) {
  if (!h || !n_out) return fail(h, MRF_EINVAL, "null argument");
  std::vector<mrf_kernel_time> acc;
  for (auto &p : h->pending) {
    if (cudaEventSynchronize(p.e1) != cudaSuccess) { cudaGetLastError(); return fail(h, MRF_ECUDA, "event wait failed"); }
    float ms = 0.f;
    cudaEventElapsedTime(&ms, p.e0, p.e1);
    cudaEventDestroy(p.e0);
    cudaEventDestroy(p.e1);
    mrf_kernel_time *slot = nullptr;
    for (auto &a : acc)
      if (!strncmp(a.name, p.name, sizeof a.name)) slot = &a;
    if (!slot) {
      acc.push_back({});
      slot = &acc.back();
      snprintf(slot->name, sizeof slot->name, "%s", p.name);
    }
    slot->launches++;
    slot->ms += ms;
  }
  h->pending.clear();
  *n_out = (int)acc.size();
  for (int i = 0; i < (int)acc.size() && i < max_n && out; ++i) out[i] = acc[i];
  return MRF_OK;
}

mrf_status mrf_debug_stall_next(mrf_handle *h) {
  if (!h) return fail(nullptr, MRF_EINVAL, "null handle");
  if (h->cfg.compute != MRF_FP16) return fail(h, MRF_EUNSUPPORTED, "the stall test runs the fp16 schedule");
  h->stall_test = true;  // consumed by the next forward, which runs eagerly
  return MRF_OK;
}

mrf_status mrf_debug_buffer(mrf_handle *h, const char *name, void *dst, size_t max_bytes, size_t *bytes_out) {
  if (!h || !name || !dst) return fail(h, MRF_EINVAL, "null argument");
  if (h->last_B < 1) return fail(h, MRF_EINVAL, "no forward has run");
  if (h->last_static)
    return fail(h, MRF_EINVAL, "the last forward ran in mrf_forward_static's shared scratch, which this hook does not read");
  const void *src = nullptr;
  size_t bytes = 0;
  const std::string n(name);
  const long long BT = (long long)h->last_B * h->last_T;
  if (h->cfg.compute == MRF_FP32_DEBUG) {
    if (n == "X") { src = h->ws.X; bytes = BT * h->cfg.num_bands * h->cfg.dim * sizeof(float); }
    else if (n == "M") { src = h->ws.Mg; bytes = BT * h->tab.n_feat() * sizeof(float); }
  } else if (!debug_buffer_fp16(h, n, &src, &bytes)) {
    src = nullptr;
  }
  if (!src) return fail(h, MRF_EINVAL, "unknown buffer " + n);
  bytes = std::min(bytes, max_bytes);
  mrf_status s = MRF_OK;
  if (!cuda_ok(h, cudaDeviceSynchronize(), "device sync", &s)) return s;
  cudaPointerAttributes attr{};
  const bool host_src = cudaPointerGetAttributes(&attr, src) == cudaSuccess && attr.type != cudaMemoryTypeDevice;
  cudaGetLastError();
  if (host_src) memcpy(dst, src, bytes);
  else if (!cuda_ok(h, cudaMemcpy(dst, src, bytes, cudaMemcpyDeviceToHost), "debug copy", &s)) return s;
  if (bytes_out) *bytes_out = bytes;
  return MRF_OK;
}

int mrf_launches_per_forward(const mrf_handle *h, int B, int T) {
  if (!h) return -1;
  return (h->last_B == B && h->last_T == T) ? h->last_launches : -1;
}

}  // extern "C"
