"""The device failure path (GPU): a bounded wait that expires is reported, and the handle recovers.

mrf_debug_stall_next makes CTA 0 of the next forward's first tensor-core GEMM issue no loads (a
flag nothing sets).  Its MMA and epilogue waits expire after their ~2 s limit, record the site in
the device status word and return; no fault, trap or hang is involved.  mrf_sync_status reports
MRF_ETIMEOUT and clears the word; the next forward runs normally and matches the oracle."""
import time

import numpy as np
import pytest

import synth
from parity import case, oracle_masks, snr_db

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


def test_expired_wait_is_reported_and_the_handle_recovers():
    from axial_band_split_b200 import mrf
    cfg = synth.TINY
    W, x = case(cfg, 1, 32, True)
    m = mrf.Model(cfg, W, max_batch=1, max_frames=32, compute=mrf.MRF_FP16)
    xd = torch.from_numpy(x).cuda()
    m.forward(xd)
    m.sync_status()                                     # healthy to start with
    m.debug_stall_next()
    t0 = time.perf_counter()
    m.forward(xd)
    with pytest.raises(mrf.MrfError) as e:
        m.sync_status()
    waited = time.perf_counter() - t0
    assert e.value.status == -6 and "bounded wait expired" in str(e.value)
    assert 1.0 < waited < 30.0, waited
    out = m.forward(xd)                                  # the handle is usable again
    m.sync_status()
    got = out.cpu().numpy()
    m.close()
    ref = oracle_masks(cfg, 1, 32, True)
    assert float(np.abs(got - ref).max()) <= 2e-2 and snr_db(got, ref) >= 40.0
