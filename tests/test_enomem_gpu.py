"""Allocation failure at create (GPU): an injected device-allocation failure returns MRF_ENOMEM
and leaks nothing.

mrf_create allocates every device buffer through one allocator that fails once the handle has made
MRF_FAIL_ALLOC_AFTER allocations (a test hook read at create).  For failures injected at the first
allocation, in the middle of the weight upload and at the last workspace buffer, create must
return MRF_ENOMEM with a null handle, and the device's free memory must come back to what it was:
every buffer allocated before the failure is freed."""
import os

import pytest

import synth
from parity import case

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


def _allocations(mrf, cfg, W, compute):
    """How many device allocations a successful create makes (probed by failing late)."""
    lo, hi = 0, 100000
    while lo < hi:                      # smallest k whose injected failure lets create succeed
        mid = (lo + hi) // 2
        os.environ["MRF_FAIL_ALLOC_AFTER"] = str(mid)
        try:
            mrf.Model(cfg, W, max_batch=1, max_frames=32, compute=compute).close()
            hi = mid
        except mrf.MrfError:
            lo = mid + 1
        finally:
            del os.environ["MRF_FAIL_ALLOC_AFTER"]
    return lo


@pytest.mark.parametrize("compute", ["fp16", "fp32"])
def test_injected_allocation_failure_returns_enomem_and_leaks_nothing(compute):
    from axial_band_split_b200 import mrf
    cm = mrf.MRF_FP16 if compute == "fp16" else mrf.MRF_FP32_DEBUG
    cfg = synth.TINY
    W, _ = case(cfg, 1, 32, True)
    mrf.Model(cfg, W, max_batch=1, max_frames=32, compute=cm).close()   # warm: context, kernel attributes
    n = _allocations(mrf, cfg, W, cm)
    assert n > 10
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info()[0]
    for k in sorted({0, 1, n // 2, n - 1}):
        os.environ["MRF_FAIL_ALLOC_AFTER"] = str(k)
        try:
            with pytest.raises(mrf.MrfError) as e:
                mrf.Model(cfg, W, max_batch=1, max_frames=32, compute=cm)
            assert e.value.status == -3, (k, str(e.value))
        finally:
            del os.environ["MRF_FAIL_ALLOC_AFTER"]
        torch.cuda.synchronize()
        assert torch.cuda.mem_get_info()[0] == free0, f"device memory leaked after a failure at allocation {k}"
