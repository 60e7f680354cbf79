"""Pins of oracle/signal.py (STFT, iSTFT, chunk loop) against the pages and closed forms."""
import math

import numpy as np

from oracle import signal


def test_frame_count_of_an_8s_chunk():
    # "Mel-Band RoFormer — architecture, ...", section "The two transformers are not the same
    # shape": center=True gives 1 + 352800/441
    # = 801 frames for an 8 s chunk
    x = np.zeros((1, 2, 352800))
    assert signal.stft(x).shape == (1, 2050, 801, 2)


def test_integer_bin_cosine_has_three_bins():
    # a periodic Hann window turns a cosine at bin k (amplitude A) into exactly three nonzero
    # bins in frames away from the edges: |X[k]| = A n / 4, |X[k +- 1]| = A n / 8
    n, hop, k, A = 256, 64, 17, 0.75
    L = 40 * hop
    t = np.arange(L)
    x = A * np.cos(2 * math.pi * k * t / n + 0.3)
    s = signal.stft(x[None, None], n_fft=n, hop=hop)          # (1, F, T, 2), one channel
    mag = np.hypot(s[0, :, :, 0], s[0, :, :, 1])               # (F, T)
    mid = mag[:, 5:-5]
    assert np.allclose(mid[k], A * n / 4, rtol=1e-12)
    assert np.allclose(mid[k - 1], A * n / 8, rtol=1e-12) and np.allclose(mid[k + 1], A * n / 8, rtol=1e-12)
    others = np.delete(mid, [k - 1, k, k + 1], axis=0)
    assert others.max() < 1e-9 * A * n


def test_stereo_rows_interleave_channels():
    # row f * 2 + s: the right channel alone only fills odd rows
    rng = np.random.Generator(np.random.PCG64(3))
    x = np.zeros((1, 2, 4000))
    x[0, 1] = rng.standard_normal(4000)
    s = signal.stft(x)
    assert np.abs(s[0, 0::2]).max() == 0 and np.abs(s[0, 1::2]).max() > 0


def test_istft_inverts_stft():
    rng = np.random.Generator(np.random.PCG64(4))
    x = rng.standard_normal((2, 2, 20000))
    y = signal.istft(signal.stft(x), channels=2, length=20000)
    assert np.abs(y - x).max() < 1e-10


def test_chunk_counts_follow_the_pages_formula():
    # "Mel-Band RoFormer — ...", section "The chunking arithmetic": n_chunks(d) = len(range(0, L,
    # 317520)), L = 44100 d
    # plus 2 * 35280 of reflect padding when 44100 d > 70560
    for d in (1.0, 1.7, 5.0, 8.0, 16.0, 60.0, 120.0):
        L = int(44100 * d)
        Lp = L + 2 * 35280 if L > 70560 else L
        _, border, lp, chunks, _ = signal.chunk_plan(L)
        assert lp == Lp and border == (35280 if L > 70560 else 0)
        assert len(chunks) == len(range(0, Lp, 317520))


def test_identity_estimate_returns_the_mix():
    # the fades are complementary across the stride and the counter normalises: an estimator
    # that returns its input gives back the mix, for padded and unpadded mixes and for both
    # tail paddings (reflect past half a chunk, zeros below)
    rng = np.random.Generator(np.random.PCG64(5))
    for L in (44100, 44100 * 3, 352800 + 20000, 352800 * 2 + 317520 // 3):
        mix = rng.standard_normal((2, L))
        out = signal.separate(mix, lambda part: part[None])
        assert out.shape == (1, 2, L)
        assert np.abs(out - mix).max() < 1e-12
