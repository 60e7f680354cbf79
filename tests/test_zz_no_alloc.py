"""mrf_forward_static against mrf_forward (GPU).

mrf_forward_static serves callers that may not allocate device memory while they run the
model (a real-time audio callback, a host framework that owns all device allocations): it
runs the same fp16 forward with its workspace in a fixed array compiled into the library.
Two calls in a row must each match mrf_forward on the same handle and input within the
fp16 parity bar (max |diff| <= 2e-2, SNR >= 40 dB); a handle whose workspace does not fit
the array is refused with MRF_ESHAPE.  This file is collected last so a run that stops at
its first failure has run every other test before it."""
import numpy as np
import pytest

import synth
from parity import case, snr_db

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


def test_static_forward_matches_forward_twice():
    from axial_band_split_b200 import mrf
    cfg = synth.TINY
    B, T = 1, 32
    W, x = case(cfg, B, T, True)
    m = mrf.Model(cfg, W, max_batch=B, max_frames=T, compute=mrf.MRF_FP16)
    xin = torch.from_numpy(x).cuda()
    ref = m.forward(xin)
    m.sync_status()
    ref = ref.cpu().numpy()
    for _ in range(2):
        out = torch.full_like(xin, float("nan"))
        m.forward_static(xin, out)
        m.sync_status()
        got = out.cpu().numpy()
        err = float(np.abs(got - ref).max())
        assert err <= 2e-2 and snr_db(got, ref) >= 40.0, (err, snr_db(got, ref))
    m.close()


def test_static_forward_refuses_oversized_workspace():
    from axial_band_split_b200 import mrf
    cfg = synth.TINY
    W, x = case(cfg, 1, 32, True)
    m = mrf.Model(cfg, W, max_batch=8, max_frames=4096, compute=mrf.MRF_FP16)
    xin = torch.from_numpy(x).cuda()
    out = torch.empty_like(xin)
    with pytest.raises(mrf.MrfError) as e:
        m.forward_static(xin, out)
    assert e.value.status == -2 and "static scratch" in str(e.value)
    m.close()


def test_static_forward_after_separate_writes_masks():
    # a separate() call leaves the handle in its apply-masks state; the static entry point must
    # still write the masks, not the separated spectra
    from axial_band_split_b200 import mrf
    cfg = synth.TINY
    B, T = 1, 32
    W, x = case(cfg, B, T, True)
    m = mrf.Model(cfg, W, max_batch=B, max_frames=T, compute=mrf.MRF_FP16)
    xin = torch.from_numpy(x).cuda()
    ref = m.forward(xin).cpu().numpy()
    m.separate(xin)
    out = torch.full_like(xin, float("nan"))
    m.forward_static(xin, out)
    m.sync_status()
    got = out.cpu().numpy()
    assert np.abs(got - ref).max() <= 2e-2 and snr_db(got, ref) >= 40.0
    with pytest.raises(mrf.MrfError):          # the debug hook does not read the shared scratch
        m.debug_buffer("X", 16)
    m.close()


def test_static_forward_short_window_after_another_handle():
    # B*T below the handle's maximum, after a handle of another shape filled the shared scratch:
    # the rows past B*T hold that handle's bytes and must not reach the masks
    from axial_band_split_b200 import mrf
    import dataclasses
    other = dataclasses.replace(synth.TINY, dim=128, heads=2, dim_head=64)
    Wo, xo = case(other, 2, 40, True)
    mo = mrf.Model(other, Wo, max_batch=2, max_frames=40, compute=mrf.MRF_FP16)
    oo = torch.empty_like(torch.from_numpy(xo).cuda())
    mo.forward_static(torch.from_numpy(xo).cuda(), oo)
    mo.sync_status()
    mo.close()
    cfg = synth.TINY
    B, T = 1, 21
    W, x = case(cfg, B, T, True)
    m = mrf.Model(cfg, W, max_batch=2, max_frames=40, compute=mrf.MRF_FP16)
    xin = torch.from_numpy(x).cuda()
    ref = m.forward(xin).cpu().numpy()
    out = torch.full_like(xin, float("nan"))
    m.forward_static(xin, out)
    m.sync_status()
    got = out.cpu().numpy()
    assert np.isfinite(got).all()
    assert np.abs(got - ref).max() <= 2e-2 and snr_db(got, ref) >= 40.0
    m.close()
