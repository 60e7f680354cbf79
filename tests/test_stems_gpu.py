"""More than one stem, and the separated spectra, through the C ABI (GPU) against the oracle.

One mask estimator per stem runs over the shared trunk ("Mel-Band RoFormer — architecture,
inference hot path & RTX 3050 feasibility", section "The forward chain": MaskEstimator per
stem; melband_deux and melband_karaoke are the pages' two-stem models), and
mrf_forward_separate multiplies each stem's complex mask into the mixture's STFT (same
section: multiply the original complex STFT).  Bars as in the other parity tests: fp16
max |diff| <= 2e-2 and SNR >= 40 dB on masks (on spectra the masks' bound times max |stft|),
fp32 debug <= 1e-4 relative."""
import dataclasses

import numpy as np
import pytest

import synth
from parity import case, rel_err, snr_db
from oracle import model as oracle_model

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


def run(cfg, W, x, compute, separate=False, max_batch=None, max_frames=None):
    from axial_band_split_b200 import mrf
    B, R, T, _ = x.shape
    m = mrf.Model(cfg, W, max_batch=max_batch or B, max_frames=max_frames or T, compute=compute)
    xd = torch.from_numpy(x).cuda()
    out = m.separate(xd) if separate else m.forward(xd)
    m.sync_status()
    torch.cuda.synchronize()
    res = out.cpu().numpy()
    m.close()
    return res


def check16(got, ref, what):
    err = float(np.abs(got - ref).max())
    snr = snr_db(got, ref)
    print(f"{what}: max|diff|={err:.3e} snr={snr:.1f} dB max|ref|={float(np.abs(ref).max()):.3e}")
    assert err <= 2e-2 and snr >= 40.0, what


@pytest.mark.parametrize("B,T", [(1, 32), (2, 17)])
def test_tiny_two_stems_fp32_and_fp16(B, T):
    from axial_band_split_b200 import mrf
    cfg = dataclasses.replace(synth.TINY, num_stems=2)
    W32, x = case(cfg, B, T, False)
    ref32 = oracle_model.forward(x, cfg, W32)
    got32 = run(cfg, W32, x, mrf.MRF_FP32_DEBUG, max_batch=2, max_frames=40)
    assert got32.shape == (B, 2) + x.shape[1:]
    assert rel_err(got32, ref32) <= 1e-4
    W16, _ = case(cfg, B, T, True)
    got16 = run(cfg, W16, x, mrf.MRF_FP16, max_batch=2, max_frames=40)
    check16(got16, oracle_model.forward(x, cfg, W16), f"tiny 2 stems B={B} T={T}")


def test_deux_two_stems_fp16():
    # the pages' melband_deux shape: dim 256, depth 12, two stems
    from axial_band_split_b200 import mrf
    cfg = synth.DEUX
    B, T = 1, 64
    W, x = case(cfg, B, T, True)
    got = run(cfg, W, x, mrf.MRF_FP16)
    check16(got, oracle_model.forward(x, cfg, W), "deux T=64")


def test_separate_spectra_fp16_and_fp32():
    from axial_band_split_b200 import mrf
    cfg = dataclasses.replace(synth.VOCALS, depth=1, num_stems=2)
    B, T = 1, 150
    W, x = case(cfg, B, T, True)
    masks = oracle_model.forward(x, cfg, W)
    ref = oracle_model.apply_masks(x, masks)
    got = run(cfg, W, x, mrf.MRF_FP16, separate=True)
    assert got.shape == ref.shape == (B, 2) + x.shape[1:]
    # the masks' bound carried through the product: |d(m x)| = |dm| |x| <= 2e-2 max|x|
    err = float(np.abs(got - ref).max())
    snr = snr_db(got, ref)
    scale = float(np.abs(x).max())
    print(f"separated spectra: max|diff|={err:.3e} (bound {2e-2 * scale:.3e}) snr={snr:.1f} dB")
    assert err <= 2e-2 * scale and snr >= 40.0
    cfg1 = synth.TINY
    W1, x1 = case(cfg1, 1, 32, False)
    ref1 = oracle_model.apply_masks(x1, oracle_model.forward(x1, cfg1, W1))
    got1 = run(cfg1, W1, x1, mrf.MRF_FP32_DEBUG, separate=True)
    assert rel_err(got1, ref1) <= 1e-4


def test_zero_dc_masks():
    # zero_dc: the DC rows' mask weight is 0 (the overlap average's row weight), both schedules
    from axial_band_split_b200 import mrf
    cfg = dataclasses.replace(synth.TINY, zero_dc=True)
    W32, x = case(cfg, 1, 32, False)
    ref = oracle_model.forward(x, cfg, W32)
    assert np.abs(ref[:, : cfg.audio_channels]).max() == 0          # rows f = 0
    got32 = run(cfg, W32, x, mrf.MRF_FP32_DEBUG, max_frames=40)
    assert rel_err(got32, ref) <= 1e-4 and np.abs(got32[:, : cfg.audio_channels]).max() == 0
    W16, _ = case(cfg, 1, 32, True)
    got16 = run(cfg, W16, x, mrf.MRF_FP16, max_frames=40)
    check16(got16, oracle_model.forward(x, cfg, W16), "tiny zero_dc")
    assert np.abs(got16[:, : cfg.audio_channels]).max() == 0


@pytest.mark.parametrize("B,T", [(1, 32), (2, 17)])
def test_geglu_tiny_fp32_and_fp16(B, T):
    # ff_act 1: the first feed-forward projection is [2 ff, dim], hidden = value * gelu(gate)
    from axial_band_split_b200 import mrf
    cfg = dataclasses.replace(synth.TINY, ff_act=1)
    W32, x = case(cfg, B, T, False)
    got32 = run(cfg, W32, x, mrf.MRF_FP32_DEBUG, max_batch=2, max_frames=40)
    assert rel_err(got32, oracle_model.forward(x, cfg, W32)) <= 1e-4
    W16, _ = case(cfg, B, T, True)
    got16 = run(cfg, W16, x, mrf.MRF_FP16, max_batch=2, max_frames=40)
    check16(got16, oracle_model.forward(x, cfg, W16), f"tiny GEGLU B={B} T={T}")


def test_geglu_vocals_depth1_fp16():
    from axial_band_split_b200 import mrf
    cfg = dataclasses.replace(synth.VOCALS, depth=1, ff_act=1)
    B, T = 1, 150
    W, x = case(cfg, B, T, True)
    got = run(cfg, W, x, mrf.MRF_FP16)
    check16(got, oracle_model.forward(x, cfg, W), "vocals depth 1 GEGLU")
