"""fp32 debug schedule against the float64 oracle, through the C ABI (GPU).

Bar: max|diff| / max|ref| <= 1e-4 (fp32 accumulation throughout)."""
import dataclasses

import numpy as np
import pytest

import synth
from parity import case, oracle_masks, rel_err, snr_db

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


def run(cfg, B, T, W, x, compute, max_batch=None, max_frames=None, graph=True):
    from axial_band_split_b200 import mrf
    m = mrf.Model(cfg, W, max_batch=max_batch or B, max_frames=max_frames or T, compute=compute)
    m.set_graph(graph)
    xin = torch.from_numpy(x).cuda()
    out = m.forward(xin)
    m.sync_status()
    torch.cuda.synchronize()
    res = out.cpu().numpy()
    m.close()
    return res


@pytest.mark.parametrize("B,T", [(1, 32), (2, 17), (1, 1)])
def test_tiny_f32(B, T):
    from axial_band_split_b200 import mrf
    cfg = synth.TINY
    W, x = case(cfg, B, T, False)
    got = run(cfg, B, T, W, x, mrf.MRF_FP32_DEBUG, max_frames=40, max_batch=2)
    ref = oracle_masks(cfg, B, T, False)
    assert got.shape == ref.shape
    assert rel_err(got, ref) <= 1e-4, (rel_err(got, ref), snr_db(got, ref))


def test_vocals_f32_small_window():
    from axial_band_split_b200 import mrf
    cfg = dataclasses.replace(synth.VOCALS, depth=2)
    B, T = 1, 37
    W, x = case(cfg, B, T, False)
    got = run(cfg, B, T, W, x, mrf.MRF_FP32_DEBUG, graph=False)
    ref = oracle_masks(cfg, B, T, False)
    assert rel_err(got, ref) <= 1e-4, (rel_err(got, ref), snr_db(got, ref))


def test_graph_replay_matches_eager():
    from axial_band_split_b200 import mrf
    cfg = synth.TINY
    W, x = case(cfg, 1, 32, False)
    a = run(cfg, 1, 32, W, x, mrf.MRF_FP32_DEBUG, graph=True)
    b = run(cfg, 1, 32, W, x, mrf.MRF_FP32_DEBUG, graph=False)
    assert np.array_equal(a, b)
