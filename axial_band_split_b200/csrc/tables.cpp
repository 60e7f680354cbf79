// Band tables: Slaney mel bank -> binary incidence -> gather/average tables.
// See tables.h for the passage it follows.  The Slaney mel scale (Auditory Toolbox):
// 200/3 Hz per mel below 1 kHz, log steps of ln(6.4)/27 per mel above.
#include "tables.h"

#include <cmath>
#include <cstdio>

namespace mrf {
namespace {

constexpr double kHzPerMel = 200.0 / 3.0;
constexpr double kKneeHz = 1000.0;

double log_step() { return std::log(6.4) / 27.0; }

double to_mel(double hz) {
  if (hz < kKneeHz) return hz / kHzPerMel;
  return kKneeHz / kHzPerMel + std::log(hz / kKneeHz) / log_step();
}

double to_hz(double mel) {
  const double knee_mel = kKneeHz / kHzPerMel;
  if (mel < knee_mel) return mel * kHzPerMel;
  return kKneeHz * std::exp(log_step() * (mel - knee_mel));
}

}  // namespace

std::string build_band_tables(int sr, int n_fft, int nb, int C, bool zero_dc, BandTables *t) {
  if (sr <= 0 || n_fft < 4 || (n_fft & 1) || nb < 1 || C < 1) return "bad mel parameters";
  const int F = n_fft / 2 + 1;
  // centre frequencies of nb + 2 points equally spaced on the mel scale, 0 .. sr/2
  std::vector<double> pts(nb + 2);
  const double top = to_mel(sr / 2.0);
  for (int i = 0; i < nb + 2; ++i) pts[i] = to_hz(top * i / (nb + 1));
  // bin frequencies: linspace(0, sr/2, F)
  std::vector<double> ff(F);
  for (int f = 0; f < F; ++f) ff[f] = (sr / 2.0) * f / (F - 1);
  std::vector<uint8_t> inc(static_cast<size_t>(nb) * F, 0);
  for (int k = 0; k < nb; ++k) {
    const double lo = pts[k], mid = pts[k + 1], hi = pts[k + 2];
    for (int f = 0; f < F; ++f) {
      const double up = (ff[f] - lo) / (mid - lo);
      const double down = (hi - ff[f]) / (hi - mid);
      const double w = std::fmin(up, down);
      inc[static_cast<size_t>(k) * F + f] = w > 0.0;
    }
  }
  inc[0] = 1;                                          // DC -> band 0
  inc[static_cast<size_t>(nb - 1) * F + (F - 1)] = 1;  // Nyquist -> last band

  t->n_bands = nb; t->n_freqs = F; t->channels = C;
  t->first_bin.assign(nb, -1); t->last_bin.assign(nb, -1); t->n_bins.assign(nb, 0);
  t->width.assign(nb, 0); t->feat_off.assign(nb + 1, 0);
  t->feat_row.clear(); t->feat_c.clear();
  t->bands_per_bin.assign(F, 0);
  for (int k = 0; k < nb; ++k) {
    for (int f = 0; f < F; ++f) {
      if (!inc[static_cast<size_t>(k) * F + f]) continue;
      if (t->first_bin[k] < 0) t->first_bin[k] = f;
      else if (f != t->last_bin[k] + 1) return "band " + std::to_string(k) + " is not contiguous";
      t->last_bin[k] = f;
      t->n_bins[k]++;
      t->bands_per_bin[f]++;
    }
    if (t->n_bins[k] == 0) return "band " + std::to_string(k) + " is empty";
    t->width[k] = 2 * t->n_bins[k] * C;
    t->feat_off[k + 1] = t->feat_off[k] + t->width[k];
    for (int f = t->first_bin[k]; f <= t->last_bin[k]; ++f)
      for (int s = 0; s < C; ++s)
        for (int c = 0; c < 2; ++c) {
          t->feat_row.push_back(f * C + s);
          t->feat_c.push_back(c);
        }
  }
  for (int f = 0; f < F; ++f) {
    if (t->bands_per_bin[f] == 0) return "bin " + std::to_string(f) + " is in no band";
    if (t->bands_per_bin[f] > 2) return "bin " + std::to_string(f) + " is in more than two bands";
  }
  t->row_weight.assign(static_cast<size_t>(F) * C, 0.f);
  for (int f = 0; f < F; ++f)
    for (int s = 0; s < C; ++s)
      t->row_weight[f * C + s] = (zero_dc && f == 0) ? 0.f : 1.0f / t->bands_per_bin[f];
  t->src0.assign(static_cast<size_t>(F) * C * 2, -1);
  t->src1.assign(static_cast<size_t>(F) * C * 2, -1);
  for (int e = 0; e < t->n_feat(); ++e) {
    const int o = t->feat_row[e] * 2 + t->feat_c[e];
    if (t->src0[o] < 0) t->src0[o] = e;
    else t->src1[o] = e;
  }
  return "";
}

std::vector<float> interleave_halves(const std::vector<float> &w, int half_rows, int cols) {
  std::vector<float> out(w.size());
  for (int r = 0; r < half_rows; ++r)
    for (int h = 0; h < 2; ++h)
      for (int c = 0; c < cols; ++c)
        out[((size_t)2 * r + h) * cols + c] = w[((size_t)h * half_rows + r) * cols + c];
  return out;
}

}  // namespace mrf
