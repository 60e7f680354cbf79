"""The bf16 compute mode (MRF_BF16) against the float64 oracle, through the C ABI (GPU).

Same schedule and kernels as MRF_FP16 with bf16 operands and activations (tcgen05 kind::f16 with
both operands bf16, fp32 accumulation) and an fp32 master copy of the residual stream.  Weights
are rounded to bf16 once and the oracle uses the rounded values.  Bar (all mask elements): max
|diff| <= 2e-2 and SNR >= 40 dB."""
import dataclasses

import numpy as np
import pytest

import synth
from oracle import model as oracle_model
from parity import snr_db, widths

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


def run_bf16(cfg, B, T, seed=1):
    from axial_band_split_b200 import mrf
    W = synth.make_weights(cfg, widths(cfg), seed=0, bf16=True)
    x = synth.make_stft_repr(cfg, B, T, seed=seed)
    m = mrf.Model(cfg, W, max_batch=B, max_frames=T, compute=mrf.MRF_BF16)
    out = m.forward(torch.from_numpy(x).cuda())
    m.sync_status()
    got = out.cpu().numpy()
    m.close()
    return got, oracle_model.forward(x, cfg, W)


def check(got, ref, what):
    assert np.isfinite(got).all()
    err = float(np.abs(got - ref).max())
    snr = snr_db(got, ref)
    print(f"bf16 {what}: max|diff|={err:.3e} snr={snr:.1f} dB max|ref|={float(np.abs(ref).max()):.3e}")
    assert err <= 2e-2 and snr >= 40.0, f"{what}: max|diff|={err:.3e} snr={snr:.1f} dB"


@pytest.mark.parametrize("B,T", [(1, 32), (2, 17)])
def test_tiny_bf16(B, T):
    check(*run_bf16(synth.TINY, B, T), f"tiny B={B} T={T}")


def test_vocals_depth1_bf16():
    check(*run_bf16(dataclasses.replace(synth.VOCALS, depth=1), 1, 150), "vocals depth 1 T=150")


def test_vocals_full_depth_bf16():
    check(*run_bf16(synth.VOCALS, 1, 300), "vocals T=300")
