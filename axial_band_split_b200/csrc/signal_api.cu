// C ABI of the spectral front and back end and of the chunked separation loop (include/mrf.h:
// mrf_stft, mrf_istft, mrf_separate_audio).  Host orchestration only: every step runs in the
// kernels of k_signal.cu and in the model's forward.
#include <cmath>
#include <cstring>
#include <string>
#include <vector>

#include "../../include/mrf.h"
#include "mrf_handle.h"
#include "mrf_internal.h"

using namespace mrf;

namespace {

mrf_status sfail(mrf_handle *h, mrf_status s, const std::string &msg) {
  h->err = msg;
  return s;
}

bool sok(mrf_handle *h, cudaError_t e, const char *what, mrf_status *st) {
  if (e == cudaSuccess) return true;
  *st = sfail(h, e == cudaErrorMemoryAllocation ? MRF_ENOMEM : MRF_ECUDA, std::string(what) + ": " + cudaGetErrorString(e));
  cudaGetLastError();
  return false;
}

int log2_exact(int n) {
  int l = 0;
  while ((1 << l) < n) ++l;
  return (1 << l) == n ? l : -1;
}

// FFT twiddles exp(-2 pi i k / n), k < n/2, and the periodic Hann window of n, in double
// precision on the host, uploaded once.
mrf_status ensure_tables(mrf_handle *h) {
  if (h->d_tw) return MRF_OK;
  const int n = h->cfg.n_fft;
  if (log2_exact(n) < 0 || n > 4096) return sfail(h, MRF_EUNSUPPORTED, "n_fft must be a power of two <= 4096 for the STFT");
  std::vector<float2> tw(n / 2);
  std::vector<float> win(n);
  const double pi = 3.14159265358979323846;
  for (int k = 0; k < n / 2; ++k)
    tw[k] = make_float2((float)std::cos(2 * pi * k / n), (float)-std::sin(2 * pi * k / n));
  for (int i = 0; i < n; ++i) win[i] = (float)(0.5 - 0.5 * std::cos(2 * pi * i / n));
  float2 *dtw = h->alloc<float2>(n / 2);
  float *dwin = h->alloc<float>(n);
  if (!dtw || !dwin) return sfail(h, MRF_ENOMEM, "device allocation failed (FFT tables)");
  if (!h->upload(dtw, tw.data(), tw.size() * sizeof(float2)) || !h->upload(dwin, win.data(), win.size() * 4))
    return sfail(h, MRF_ECUDA, "upload failed (FFT tables)");
  if (!signal_kernels_init()) return sfail(h, MRF_ECUDA, "FFT kernels: shared-memory limit");
  h->d_tw = dtw;
  h->d_win = dwin;
  return MRF_OK;
}

// Grow-only scratch buffer `slot` of at least `bytes` (freed by mrf_destroy).
float *scratch(mrf_handle *h, size_t slot, size_t bytes) {
  if (h->sig_scratch.size() <= slot) h->sig_scratch.resize(slot + 1, {nullptr, 0});
  auto &e = h->sig_scratch[slot];
  if (e.second < bytes) {
    if (e.first) cudaFree(e.first);
    e = {nullptr, 0};
    void *p = nullptr;
    if (cudaMalloc(&p, bytes) != cudaSuccess) {
      cudaGetLastError();
      return nullptr;
    }
    e = {p, bytes};
  }
  return static_cast<float *>(e.first);
}

// The chunk loop's geometry for a mix of L samples ("Mel-Band RoFormer — ...", section
// "Verified inference hot path"): 8 s chunks (or chunk_samples), stride 0.9 chunk, fades of chunk / 10, the mix
// reflect-padded by the border chunk - stride when longer than two borders, a short last chunk
// padded by reflection when more than half a chunk remains (mode 1), by zeros otherwise (2).
struct ChunkGeometry {
  int chunk, stride, fade, border, Lp;
  bool padded;
  std::vector<int> off, n, mode;
};

ChunkGeometry chunk_geometry(int sample_rate, int chunk_samples, int L) {
  ChunkGeometry g;
  g.chunk = chunk_samples > 0 ? chunk_samples : sample_rate * 8;
  g.stride = (int)(g.chunk * 0.9);
  g.fade = g.chunk / 10;
  g.border = g.chunk - g.stride;
  g.padded = L > 2 * g.border;
  g.Lp = g.padded ? L + 2 * g.border : L;
  for (int o = 0; o < g.Lp; o += g.stride) {
    const int nk = std::min(g.chunk, g.Lp - o);
    g.off.push_back(o);
    g.n.push_back(nk);
    g.mode.push_back(nk == g.chunk ? 0 : (nk > g.chunk / 2 ? 1 : 2));
  }
  return g;
}

}  // namespace

extern "C" {

mrf_status mrf_stft(mrf_handle *h, const float *audio, float *stft_repr, int B, int L, int hop, void *stream) {
  if (!h) return MRF_EINVAL;
  if (!audio || !stft_repr) return sfail(h, MRF_EINVAL, "null audio or stft_repr pointer");
  const int n = h->cfg.n_fft;
  if (B < 1 || hop < 1 || L <= n / 2) return sfail(h, MRF_ESHAPE, "B >= 1, hop >= 1 and L > n_fft / 2 required");
  mrf_status s = ensure_tables(h);
  if (s != MRF_OK) return s;
  const int T = 1 + L / hop;
  cudaGetLastError();
  launch_stft(audio, stft_repr, h->d_tw, h->d_win, B, h->cfg.audio_channels, L, T, log2_exact(n), hop,
              static_cast<cudaStream_t>(stream));
  sok(h, cudaGetLastError(), "STFT launch", &s);
  return s;
}

mrf_status mrf_istft(mrf_handle *h, const float *spec, float *audio, int S, int T, int hop, int length,
                     void *stream) {
  if (!h) return MRF_EINVAL;
  if (!spec || !audio) return sfail(h, MRF_EINVAL, "null spec or audio pointer");
  if (S < 1 || T < 1 || hop < 1 || length < 1) return sfail(h, MRF_ESHAPE, "S, T, hop and length must be >= 1");
  mrf_status s = ensure_tables(h);
  if (s != MRF_OK) return s;
  const int n = h->cfg.n_fft, C = h->cfg.audio_channels;
  float *frames = scratch(h, 0, (size_t)S * C * T * n * sizeof(float));
  if (!frames) return sfail(h, MRF_ENOMEM, "device allocation failed (iSTFT frames)");
  cudaGetLastError();
  launch_istft(spec, frames, audio, h->d_tw, h->d_win, S, C, T, log2_exact(n), hop, length,
               static_cast<cudaStream_t>(stream));
  sok(h, cudaGetLastError(), "iSTFT launch", &s);
  return s;
}

mrf_status mrf_separate_audio(mrf_handle *h, const float *mix, float *stems, int L, int hop, void *stream) {
  return mrf_separate_audio_chunked(h, mix, stems, L, hop, 0, stream);
}

mrf_status mrf_separate_audio_chunked(mrf_handle *h, const float *mix, float *stems, int L, int hop,
                                      int chunk_samples, void *stream) {
  if (!h) return MRF_EINVAL;
  if (!mix || !stems) return sfail(h, MRF_EINVAL, "null mix or stems pointer");
  const mrf_config &c = h->cfg;
  const int C = c.audio_channels, S = c.num_stems, n = c.n_fft;
  if (hop < 1 || L < 2) return sfail(h, MRF_ESHAPE, "hop >= 1 and L >= 2 required");
  if (chunk_samples != 0 && (chunk_samples < 10 || chunk_samples <= n / 2))
    return sfail(h, MRF_EINVAL, "chunk_samples must be 0 (8 s) or at least 10 and above n_fft / 2");
  const ChunkGeometry g = chunk_geometry(c.sample_rate, chunk_samples, L);
  const int chunk = g.chunk, stride = g.stride, fade = g.fade, border = g.border;
  const int T = 1 + chunk / hop;
  if (T > c.max_frames) return sfail(h, MRF_ESHAPE, "max_frames is below the frames of one chunk");
  mrf_status s = ensure_tables(h);
  if (s != MRF_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const bool padded = g.padded;
  const int Lp = g.Lp;
  const int nb_max = std::min(std::min(c.max_batch, 16), (Lp + stride - 1) / stride);
  const size_t F = (size_t)n / 2 + 1;
  float *xp = scratch(h, 1, (size_t)C * Lp * 4);
  float *chunks = scratch(h, 2, (size_t)nb_max * C * chunk * 4);
  float *spec_in = scratch(h, 3, (size_t)nb_max * F * C * T * 2 * 4);
  float *spec_out = scratch(h, 4, (size_t)nb_max * S * F * C * T * 2 * 4);
  float *frames = scratch(h, 0, (size_t)nb_max * S * C * T * n * 4);
  float *est = scratch(h, 5, (size_t)nb_max * S * C * chunk * 4);
  float *acc = scratch(h, 6, (size_t)S * C * Lp * 4);
  float *counter = scratch(h, 7, (size_t)Lp * 4);
  if (!xp || !chunks || !spec_in || !spec_out || !frames || !est || !acc || !counter)
    return sfail(h, MRF_ENOMEM, "device allocation failed (separation buffers)");
  cudaGetLastError();
  if (!sok(h, cudaMemsetAsync(acc, 0, (size_t)S * C * Lp * 4, st), "memset", &s) ||
      !sok(h, cudaMemsetAsync(counter, 0, (size_t)Lp * 4, st), "memset", &s))
    return s;
  const float *src = mix;
  if (padded) {
    launch_pad_reflect(mix, xp, C, L, border, st);
    src = xp;
  }
  const std::vector<int> &offs = g.off;
  for (size_t k0 = 0; k0 < offs.size(); k0 += nb_max) {
    ChunkBatch cb{};
    cb.count = (int)std::min<size_t>(nb_max, offs.size() - k0);
    for (int k = 0; k < cb.count; ++k) {
      cb.off[k] = offs[k0 + k];
      cb.n[k] = g.n[k0 + k];
      cb.reflect[k] = g.mode[k0 + k] == 1;
    }
    launch_gather_chunks(src, chunks, cb, C, Lp, chunk, st);
    launch_stft(chunks, spec_in, h->d_tw, h->d_win, cb.count, C, chunk, T, log2_exact(n), hop, st);
    s = mrf_forward_separate(h, spec_in, spec_out, cb.count, T, stream);
    if (s != MRF_OK) return s;
    launch_istft(spec_out, frames, est, h->d_tw, h->d_win, cb.count * S, C, T, log2_exact(n), hop, chunk, st);
    for (int k = 0; k < cb.count; ++k)
      launch_accumulate_chunk(est + (size_t)k * S * C * chunk, acc, counter, S, C, Lp, chunk, fade, cb.off[k],
                              cb.n[k], cb.off[k] == 0, cb.off[k] + chunk >= Lp, st);
  }
  launch_finalize(acc, counter, stems, S, C, Lp, L, padded ? border : 0, st);
  sok(h, cudaGetLastError(), "separation launches", &s);
  return s;
}

mrf_status mrf_chunk_plan(int sample_rate, int chunk_samples, int L, int *chunk, int *border, int *padded_length,
                          int *n_chunks, int32_t *off, int32_t *valid, int32_t *mode, int max_chunks) {
  if (sample_rate < 1 || L < 2 || chunk_samples < 0 || (chunk_samples > 0 && chunk_samples < 10) || !chunk ||
      !border || !padded_length || !n_chunks)
    return MRF_EINVAL;
  const ChunkGeometry g = chunk_geometry(sample_rate, chunk_samples, L);
  *chunk = g.chunk;
  *border = g.padded ? g.border : 0;
  *padded_length = g.Lp;
  *n_chunks = (int)g.off.size();
  for (int i = 0; i < (int)g.off.size() && i < max_chunks; ++i) {
    if (off) off[i] = g.off[i];
    if (valid) valid[i] = g.n[i];
    if (mode) mode[i] = g.mode[i];
  }
  return MRF_OK;
}

}  // extern "C"
