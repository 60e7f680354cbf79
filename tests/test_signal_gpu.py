"""STFT, iSTFT and the chunked separation loop through the C ABI (GPU) against oracle/signal.py.

"Mel-Band RoFormer — architecture, inference hot path & RTX 3050 feasibility", sections "The
forward chain" (torch.stft / istft with n_fft 2048, hop 441, Hann, center=True) and "Verified
inference hot path" (the chunk loop).  The transforms run in fp32: bar 1e-5 of the reference's
largest magnitude.  The separation with random weights carries the fp16 model's error: the
masks' bar (2e-2, 40 dB SNR) on the stems, relative to the mix's largest sample."""
import dataclasses

import numpy as np
import pytest

import synth
from oracle import model as oracle_model
from oracle import signal
from parity import snr_db

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")

HOP = 441


def make_model(cfg, W, max_batch=2, max_frames=801):
    from axial_band_split_b200 import mrf
    return mrf.Model(cfg, W, max_batch=max_batch, max_frames=max_frames, compute=mrf.MRF_FP16)


def weights(cfg):
    from axial_band_split_b200 import mrf
    return synth.make_weights(cfg, mrf.band_tables(cfg)["width"], fp16=True)


def rel(a, b):
    return float(np.abs(a - b).max() / np.abs(b).max())


def test_stft_and_istft_match_the_oracle():
    cfg = dataclasses.replace(synth.VOCALS, depth=0)
    m = make_model(cfg, weights(cfg))
    audio = np.stack([synth.synth_audio(44100, seed=s) for s in (1, 2)])          # (2, 2, L)
    got = m.stft(torch.from_numpy(audio.astype(np.float32)).cuda(), HOP).cpu().numpy()
    ref = signal.stft(audio.astype(np.float32))
    assert got.shape == ref.shape == (2, 2050, 101, 2)
    assert rel(got, ref) <= 1e-5, rel(got, ref)
    rng = np.random.Generator(np.random.PCG64(11))
    spec = rng.standard_normal((3, 2050, 40, 2)).astype(np.float32)             # not an STFT of anything
    length = 39 * HOP + 100
    got = m.istft(torch.from_numpy(spec).cuda(), HOP, length).cpu().numpy()
    ref = signal.istft(spec, channels=2, length=length)
    assert got.shape == ref.shape == (3, 2, length)
    assert rel(got, ref) <= 1e-5, rel(got, ref)
    m.close()


def identity_weights(cfg):
    # the last mask layer outputs value 1 (real parts), 0 (imaginary parts) and gate 30, so
    # every mask is 1 + 0i after the GLU (sigmoid(30) rounds to 1) and the overlap average
    W = weights(cfg)
    from axial_band_split_b200 import mrf
    widths = mrf.band_tables(cfg)["width"]
    last = 2 * cfg.mask_depth
    for k, d in enumerate(widths):
        p = f"mask_estimators.0.to_freqs.{k}.0.{last}."
        W[p + "weight"] = np.zeros_like(W[p + "weight"])
        b = np.zeros(2 * d, dtype=W[p + "bias"].dtype)
        b[0:d:2] = 1.0                                                          # value, real parts
        b[d:] = 30.0                                                            # gate
        W[p + "bias"] = b
    return W


@pytest.mark.parametrize("seconds", [1.0, 9.0, 20.0])
def test_separation_with_unit_masks_returns_the_mix(seconds):
    # 1 s: unpadded, one zero-padded chunk; 9 s: padded, last chunk zero-padded; 20 s: three
    # chunks, last one padded by reflection
    cfg = dataclasses.replace(synth.VOCALS, depth=1)
    m = make_model(cfg, identity_weights(cfg), max_batch=2)
    L = int(44100 * seconds)
    mix = synth.synth_audio(L, seed=3).astype(np.float32)
    out = m.separate_audio(torch.from_numpy(mix).cuda(), HOP).cpu().numpy()
    m.close()
    assert out.shape == (1, 2, L)
    err = float(np.abs(out[0] - mix).max()) / float(np.abs(mix).max())
    print(f"{seconds} s: max|stem - mix| / max|mix| = {err:.2e}")
    assert err <= 1e-5


def test_separation_matches_the_oracle():
    cfg = dataclasses.replace(synth.VOCALS, depth=1)
    W = weights(cfg)
    L = 88200                                                                   # 2 s: one chunk
    mix = synth.synth_audio(L, seed=4).astype(np.float32)
    m = make_model(cfg, W)
    got = m.separate_audio(torch.from_numpy(mix).cuda(), HOP).cpu().numpy()
    m.close()

    def estimate(part):
        x = signal.stft(part[None])
        spec = oracle_model.apply_masks(x, oracle_model.forward(x, cfg, W))
        return signal.istft(spec[0][None], channels=2, length=part.shape[-1])

    ref = signal.separate(mix.astype(np.float64), estimate)
    err = float(np.abs(got - ref).max()) / float(np.abs(mix).max())
    snr = snr_db(got, ref)
    print(f"separated audio: max|diff|/max|mix| = {err:.2e}, snr = {snr:.1f} dB")
    assert err <= 2e-2 and snr >= 40.0


def test_separation_with_short_chunks_matches_the_oracle():
    # chunks of 2 s instead of 8 s on a 5 s mix (padded, three chunks): the chunk-length
    # parameter of the separation loop against the oracle's loop with the same chunk
    cfg = dataclasses.replace(synth.VOCALS, depth=1)
    W = weights(cfg)
    L, chunk = 5 * 44100, 2 * 44100
    mix = synth.synth_audio(L, seed=5).astype(np.float32)
    m = make_model(cfg, W, max_batch=4)
    got = m.separate_audio(torch.from_numpy(mix).cuda(), HOP, chunk_samples=chunk).cpu().numpy()
    m.close()

    def estimate(part):
        x = signal.stft(part[None])
        spec = oracle_model.apply_masks(x, oracle_model.forward(x, cfg, W))
        return signal.istft(spec[0][None], channels=2, length=part.shape[-1])

    ref = signal.separate(mix.astype(np.float64), estimate, chunk=chunk)
    err = float(np.abs(got - ref).max()) / float(np.abs(mix).max())
    snr = snr_db(got, ref)
    print(f"2 s chunks: max|diff|/max|mix| = {err:.2e}, snr = {snr:.1f} dB")
    assert err <= 2e-2 and snr >= 40.0
