"""CTA-pair GEMMs (cta_group::2, M = 256 tiles) against one CTA per M = 128 tile (GPU).

MRF_GEMM_PAIR, read when a model is created, selects which GEMMs pair: 0 none, 1 the trunk GEMMs
with K >= 1024 (FF2 of a D >= 256 model; the default), 2 every trunk GEMM and the mask MLP's tanh
layers (grouped by band).  A pair computes every
output element with the same K-ordered fp32 accumulation and the same epilogue arithmetic as a
single CTA, so the three modes give the same bits; each is also held to the fp16 parity bar
against the float64 oracle.  Shapes: a ragged row count (B T nb not a multiple of 256, so the
second CTA of the last pair reads past the end) and an odd batch of windows."""
import dataclasses

import numpy as np
import pytest

import synth
from parity import case, snr_db
from oracle import model as oracle_model

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


def forward(cfg, B, T, W, x, mode, monkeypatch):
    from axial_band_split_b200 import mrf
    monkeypatch.setenv("MRF_GEMM_PAIR", str(mode))
    m = mrf.Model(cfg, W, max_batch=B, max_frames=T, compute=mrf.MRF_FP16)
    m.set_graph(False)
    out = m.forward(torch.from_numpy(x).cuda())
    m.sync_status()
    res = out.cpu().numpy()
    m.close()
    return res


@pytest.mark.parametrize("name,B,T", [("vocals_d1", 1, 150), ("vocals_d1", 3, 37), ("tiny", 2, 17)])
def test_pair_modes_bit_identical(name, B, T, monkeypatch):
    cfg = dataclasses.replace(synth.VOCALS, depth=1) if name == "vocals_d1" else synth.TINY
    W, x = case(cfg, B, T, True)
    outs = [forward(cfg, B, T, W, x, mode, monkeypatch) for mode in (0, 1, 2)]
    ref = oracle_model.forward(x, cfg, W)
    for mode, got in zip((0, 1, 2), outs):
        assert np.isfinite(got).all()
        err, snr = float(np.abs(got - ref).max()), snr_db(got, ref)
        assert err <= 2e-2 and snr >= 40.0, f"pair mode {mode}: max|diff|={err:.3e} snr={snr:.1f} dB"
        assert np.array_equal(got, outs[0]), f"pair mode {mode} differs from one CTA per tile"
