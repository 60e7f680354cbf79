// Band tables of the mel-band split, built on the host at create time.
//
// "Mel-Band RoFormer — architecture, inference hot path & RTX 3050 feasibility", section
// "The mel-band split, exactly": a Slaney mel filter bank of num_bands triangles over the
// n_fft/2+1 bins, binarised at weight > 0, DC forced into band 0 and Nyquist into the last
// band; freq_indices list each band's bins ascending with the channels interleaved
// (row f*C + s); num_bands_per_freq divides the overlap sum.
#pragma once
#include <cstdint>
#include <string>
#include <vector>

namespace mrf {

struct BandTables {
  int n_bands = 0, n_freqs = 0, channels = 0;
  std::vector<int32_t> first_bin, last_bin, n_bins, width;  // per band; width = 2 * n_bins * C
  std::vector<int32_t> feat_off;    // [n_bands + 1] prefix sums of width
  std::vector<int32_t> feat_row;    // [sum width] stft_repr row of each band feature
  std::vector<int32_t> feat_c;      // [sum width] complex part (0 re, 1 im)
  std::vector<int32_t> bands_per_bin;  // [n_freqs]
  std::vector<float> row_weight;    // [n_freqs * C]
  // Per output element (row, c): up to two source features (-1 when absent).
  std::vector<int32_t> src0, src1;  // [n_freqs * C * 2]
  int n_feat() const { return feat_off.empty() ? 0 : feat_off.back(); }
};

// Returns an empty string on success, else the reason the tables are invalid.
std::string build_band_tables(int sample_rate, int n_fft, int n_bands, int channels, bool zero_dc,
                              BandTables *out);

// Rows [v_0 .. v_{n-1}, g_0 .. g_{n-1}] (each `cols` wide) reordered as v_0, g_0, v_1, g_1, ...:
// the GEGLU projection's value and gate halves paired for an epilogue that reads neighbours.
std::vector<float> interleave_halves(const std::vector<float> &w, int half_rows, int cols);

}  // namespace mrf
