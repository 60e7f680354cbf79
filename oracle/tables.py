"""Band tables of the mel-band split (oracle; test infrastructure only).

Follows "Mel-Band RoFormer — architecture, inference hot path & RTX 3050 feasibility",
section "The mel-band split, exactly": a Slaney mel filter bank of n_bands triangles over
the n_fft/2+1 FFT bins, binarised (weight > 0), with DC forced into the first band and
Nyquist into the last; each band's bins in ascending order, stereo interleaved as rows
f*2 + s; the per-bin band count divides the overlap sum.  The gather/average layout
follows ``Core`` in package/scripts/export-roformer.py of "@audio/neural-separate 0.4.0 →
0.5.0" (each band's input columns, at most two sources per output column).

The Slaney mel scale is the Auditory Toolbox definition: linear at 200/3 Hz per mel
below 1 kHz, logarithmic above with a step of ln(6.4)/27 per mel.
"""
from __future__ import annotations

import math

import numpy as np

F_SP = 200.0 / 3.0
MIN_LOG_HZ = 1000.0
MIN_LOG_MEL = MIN_LOG_HZ / F_SP
LOGSTEP = math.log(6.4) / 27.0


def hz_to_mel(f):
    f = np.asarray(f, dtype=np.float64)
    lin = f / F_SP
    log = MIN_LOG_MEL + np.log(np.maximum(f, MIN_LOG_HZ) / MIN_LOG_HZ) / LOGSTEP
    return np.where(f >= MIN_LOG_HZ, log, lin)


def mel_to_hz(m):
    m = np.asarray(m, dtype=np.float64)
    lin = F_SP * m
    log = MIN_LOG_HZ * np.exp(LOGSTEP * (np.maximum(m, MIN_LOG_MEL) - MIN_LOG_MEL))
    return np.where(m >= MIN_LOG_MEL, log, lin)


def mel_filterbank(sr: int, n_fft: int, n_mels: int):
    """Triangular filters (n_mels, n_fft//2+1): n_mels+2 points equally spaced in mel
    from 0 to sr/2; filter i rises from point i to i+1 and falls to i+2."""
    fft_f = np.linspace(0.0, sr / 2.0, n_fft // 2 + 1)
    pts = mel_to_hz(np.linspace(hz_to_mel(0.0), hz_to_mel(sr / 2.0), n_mels + 2))
    w = np.zeros((n_mels, fft_f.size))
    for i in range(n_mels):
        rise = (fft_f - pts[i]) / (pts[i + 1] - pts[i])
        fall = (pts[i + 2] - fft_f) / (pts[i + 2] - pts[i + 1])
        w[i] = np.maximum(0.0, np.minimum(rise, fall))
    return w


def band_incidence(sr: int, n_fft: int, n_bands: int):
    """Binarised bank (n_bands, F) bool, DC forced into band 0 and Nyquist into the last."""
    inc = mel_filterbank(sr, n_fft, n_bands) > 0
    inc[0, 0] = True
    inc[-1, -1] = True
    return inc


def band_tables(sr: int, n_fft: int, n_bands: int, channels: int = 2, zero_dc: bool = False):
    """All integer tables of the split and the average.

    Returns a dict:
      first_bin, last_bin, n_bins : (n_bands,) int   each band's contiguous bin range
      widths      : (n_bands,) int     d_in = 2 (re, im) * n_bins * channels
      freq_rows   : (sum n_bins*channels,) int  gathered rows f*channels + s, band order
      feat_row    : (sum widths,) int  stft_repr row of each band feature, band order
      feat_c      : (sum widths,) int  complex part (0 re, 1 im) of each feature
      bands_per_bin : (F,) int         number of bands covering each bin
      row_weight  : (F*channels,) float  1 / bands_per_bin of the row's bin (0 at DC with zero_dc)
    Feature e of band k is (j*channels + s)*2 + c for the j-th bin of the band.
    """
    inc = band_incidence(sr, n_fft, n_bands)
    F = inc.shape[1]
    assert inc.any(axis=0).all(), "a bin belongs to no band"
    counts = inc.sum(axis=0)
    first, last, nb = [], [], []
    rows, feat_row, feat_c = [], [], []
    for k in range(n_bands):
        bins = np.nonzero(inc[k])[0]
        assert bins.size > 0 and np.all(np.diff(bins) == 1), "band not contiguous"
        first.append(int(bins[0]))
        last.append(int(bins[-1]))
        nb.append(int(bins.size))
        for f in bins:
            for s in range(channels):
                r = int(f) * channels + s
                rows.append(r)
                for c in range(2):
                    feat_row.append(r)
                    feat_c.append(c)
    w = 1.0 / np.repeat(counts, channels).astype(np.float64)
    if zero_dc:
        w[:channels] = 0.0
    nb = np.array(nb)
    return {
        "first_bin": np.array(first), "last_bin": np.array(last), "n_bins": nb,
        "widths": 2 * nb * channels, "freq_rows": np.array(rows),
        "feat_row": np.array(feat_row), "feat_c": np.array(feat_c),
        "bands_per_bin": counts.astype(np.int64), "row_weight": w,
    }
