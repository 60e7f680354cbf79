"""Pins of the oracle's band tables against what the pages print and the mel scale fixes."""
import numpy as np
import pytest

from conftest import read_golden
from oracle import tables


def golden_bins():
    return [int(v) for line in read_golden("mel60_band_bins.txt") for v in line.split()]


def test_slaney_mel_closed_forms():
    # linear part: 200/3 Hz per mel, so 1 kHz is mel 15; log part: 6.4x per 27 mels
    assert tables.hz_to_mel(1000.0) == pytest.approx(15.0, abs=1e-12)
    assert tables.hz_to_mel(6400.0) == pytest.approx(42.0, abs=1e-12)
    assert tables.hz_to_mel(500.0) == pytest.approx(7.5, abs=1e-12)
    assert tables.mel_to_hz(42.0) == pytest.approx(6400.0, rel=1e-13)
    f = np.array([0.0, 10.0, 999.0, 1000.0, 1001.0, 4321.0, 22050.0])
    assert np.allclose(tables.mel_to_hz(tables.hz_to_mel(f)), f, rtol=1e-13, atol=1e-10)
    # continuous at the 1 kHz knee
    assert tables.hz_to_mel(1000.0 - 1e-9) == pytest.approx(tables.hz_to_mel(1000.0), abs=1e-9)


def test_triangles_partition_of_unity():
    # between the second and the second-to-last mel point the falling edge of one
    # triangle and the rising edge of the next sum to one at every FFT bin
    sr, n_fft, nm = 44100, 2048, 60
    w = tables.mel_filterbank(sr, n_fft, nm)
    fft_f = np.linspace(0, sr / 2, n_fft // 2 + 1)
    pts = tables.mel_to_hz(np.linspace(0, tables.hz_to_mel(sr / 2), nm + 2))
    inside = (fft_f >= pts[1]) & (fft_f <= pts[nm])
    assert np.allclose(w[:, inside].sum(0), 1.0, atol=1e-12)
    # each triangle peaks at 1 exactly at its centre frequency
    assert np.all(w.max(1) <= 1.0 + 1e-12)


def test_vocals_band_counts_match_pages():
    t = tables.band_tables(44100, 2048, 60)
    assert list(t["n_bins"]) == golden_bins()
    assert int((t["bands_per_bin"] == 1).sum()) == 71
    assert int((t["bands_per_bin"] == 2).sum()) == 954
    assert int(t["n_bins"].sum()) == 1979
    assert int(t["widths"].sum()) == 7916
    assert t["widths"][0] == 2 * 7 * 2 and t["widths"][-1] == 2 * 130 * 2


@pytest.mark.parametrize("sr,n_fft,nb", [(44100, 2048, 60), (44100, 256, 8)])
def test_band_invariants(sr, n_fft, nb):
    t = tables.band_tables(sr, n_fft, nb)
    F = n_fft // 2 + 1
    inc = tables.band_incidence(sr, n_fft, nb)
    assert inc.shape == (nb, F)
    assert inc.any(0).all()                      # every bin covered
    assert inc.sum(0).max() <= 2                 # no bin in three bands
    assert inc[0, 0] and inc[-1, -1]             # DC in band 0, Nyquist in the last
    for k in range(nb):                          # contiguous, ascending, overlapping neighbours
        bins = np.nonzero(inc[k])[0]
        assert t["first_bin"][k] == bins[0] and t["last_bin"][k] == bins[-1]
        if k:
            assert t["first_bin"][k] >= t["first_bin"][k - 1]
    # gather rows: per band, bins ascending, stereo interleaved f*2+s
    off = 0
    for k in range(nb):
        rows = t["freq_rows"][off: off + 2 * t["n_bins"][k]]
        exp = [f * 2 + s for f in range(t["first_bin"][k], t["last_bin"][k] + 1) for s in (0, 1)]
        assert list(rows) == exp
        off += 2 * t["n_bins"][k]
    # feature e = (j*2+s)*2+c: row and complex part
    assert np.array_equal(t["feat_row"], np.repeat(t["freq_rows"], 2))
    assert np.array_equal(t["feat_c"], np.tile([0, 1], len(t["freq_rows"])))
    # average weights are 1/count, and weighting the count back gives one everywhere
    cnt = np.bincount(t["freq_rows"], minlength=2 * F)
    assert np.allclose(t["row_weight"] * cnt, 1.0)


def test_tiny_tables():
    t = tables.band_tables(44100, 256, 8)
    # no printed values for this size: the invariants above pin it; record the derived table
    assert list(t["n_bins"]) == [6, 6, 7, 12, 20, 31, 48, 77]
    assert int(t["widths"].sum()) == 828
    assert int((t["bands_per_bin"] == 1).sum()) == 51 and int((t["bands_per_bin"] == 2).sum()) == 78


def test_zero_dc_weight():
    t = tables.band_tables(44100, 2048, 60, zero_dc=True)
    assert t["row_weight"][0] == 0 and t["row_weight"][1] == 0
    assert t["row_weight"][2] > 0
