"""The fused feed-forward kernel (MRF_FF_FUSED=1: FF1, GELU and FF2 with the residual in one
launch on CTA pairs) against the float64 oracle and against the two-GEMM path (GPU).

Bar: max|diff| <= 2e-2 and SNR >= 40 dB against the oracle, as for every fp16 parity test.
Shapes: D = 384 (two FF2 pieces of 192 outputs) and D = 256 (one piece), a row count that is
not a multiple of the pair's 256-row tile, and more tiles than CTA pairs on the larger case."""
import dataclasses

import numpy as np
import pytest

import synth
from parity import case, snr_db
from oracle import model as oracle_model

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


def forward(cfg, B, T, W, x, fused, monkeypatch):
    from axial_band_split_b200 import mrf
    monkeypatch.setenv("MRF_FF_FUSED", "1" if fused else "0")
    m = mrf.Model(cfg, W, max_batch=B, max_frames=T, compute=mrf.MRF_FP16)
    m.set_graph(False)
    out = m.forward(torch.from_numpy(x).cuda())
    m.sync_status()
    res = out.cpu().numpy()
    m.close()
    return res


@pytest.mark.parametrize("name,B,T", [("vocals", 1, 150), ("vocals", 2, 37), ("deux", 1, 90)])
def test_fused_feed_forward(name, B, T, monkeypatch):
    base = synth.VOCALS if name == "vocals" else synth.DEUX
    cfg = dataclasses.replace(base, depth=1)
    W, x = case(cfg, B, T, True)
    got = forward(cfg, B, T, W, x, True, monkeypatch)
    two = forward(cfg, B, T, W, x, False, monkeypatch)
    ref = oracle_model.forward(x, cfg, W)
    assert np.isfinite(got).all()
    err, snr = float(np.abs(got - ref).max()), snr_db(got, ref)
    assert err <= 2e-2 and snr >= 40.0, f"fused: max|diff|={err:.3e} snr={snr:.1f} dB"
    # the same arithmetic up to fp32 summation order and one fewer fp16 rounding (the hidden
    # activations stay in fp16 either way)
    assert snr_db(got, two) >= 60.0
