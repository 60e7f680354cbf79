"""The host-buffer entry points (mrf_forward_host, and mrf_forward_host_async with mrf_host_join)
against the device-buffer forward and the float64 oracle (GPU).

The pipelined calls use two device slots in turn, copy on streams of their own and order copies
and forwards with events; every call's masks must equal, bit for bit, those of mrf_forward on
the same input copied by hand (the same kernels run on the same bytes), and one case is held to
the fp16 parity bar against the oracle.  Cases: more calls than slots with a different input
each (a slot overwritten before its predecessor's output was read would show up as another
call's masks), a pageable output buffer, a synchronous call between asynchronous ones, a join
with nothing pending, a smaller (B, T) after a larger one in the same slot, and a batch whose
input buffer is filled by work queued on its stream just before it."""
import numpy as np
import pytest

import synth
from parity import case, snr_db
from oracle import model as oracle_model

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


def model_for(cfg, W, B, T):
    from axial_band_split_b200 import mrf
    return mrf.Model(cfg, W, max_batch=B, max_frames=T, compute=mrf.MRF_FP16)


def device_masks(m, x):
    out = m.forward(torch.from_numpy(x).cuda())
    m.sync_status()
    return out.cpu().numpy()


@pytest.mark.parametrize("name,B,T", [("tiny", 2, 17), ("vocals_d1", 1, 150)])
def test_async_pipeline_matches_device_forward(name, B, T):
    import dataclasses
    cfg = dataclasses.replace(synth.VOCALS, depth=1) if name == "vocals_d1" else synth.TINY
    W, x0 = case(cfg, B, T, True)
    xs = [x0] + [synth.make_stft_repr(cfg, B, T, seed=10 + k) for k in range(4)]
    m = model_for(cfg, W, B, T)
    want = [device_masks(m, x) for x in xs]
    stream = torch.cuda.current_stream()
    m.host_join(stream)  # nothing pending yet
    ins = [torch.from_numpy(x).pin_memory() for x in xs]
    outs = [torch.full(w.shape, float("nan")).pin_memory() for w in want]
    outs[3] = torch.full(want[3].shape, float("nan"))  # pageable: its copy waits inside the call
    for k in range(len(xs)):
        m.forward_host_async(ins[k], outs[k], stream=stream)
    m.host_join(stream)
    m.sync_status(stream)
    for k in range(len(xs)):
        assert np.array_equal(outs[k].numpy(), want[k]), f"call {k} differs from the device forward"
    # a synchronous call between asynchronous ones
    o = torch.empty(want[0].shape).pin_memory()
    m.forward_host_async(ins[1], outs[1], stream=stream)
    m.forward_host(ins[0], o, stream=stream)
    assert np.array_equal(o.numpy(), want[0])
    assert np.array_equal(outs[1].numpy(), want[1])
    ref = oracle_model.forward(x0, cfg, W)
    got = outs[0].numpy()
    err, snr = float(np.abs(got - ref).max()), snr_db(got, ref)
    assert err <= 2e-2 and snr >= 40.0, f"max|diff|={err:.3e} snr={snr:.1f} dB"
    m.close()


def test_small_window_in_pipeline():
    """A window shorter than the one before it in the same slot: the masks of the short window
    must not depend on the longer window's bytes left in the slot."""
    cfg = synth.TINY
    B, T = 2, 17
    W, _ = case(cfg, B, T, True)
    m = model_for(cfg, W, B, T)
    xl = synth.make_stft_repr(cfg, B, T, seed=21)
    xsh = synth.make_stft_repr(cfg, 1, 5, seed=22)
    want = device_masks(m, xsh)
    stream = torch.cuda.current_stream()
    xl_t, xsh_t = torch.from_numpy(xl).pin_memory(), torch.from_numpy(xsh).pin_memory()
    ol, ol2, osh = m._out_like(xl_t, None), m._out_like(xl_t, None), m._out_like(xsh_t, None)
    m.forward_host_async(xl_t, ol, stream=stream)
    m.forward_host_async(xl_t, ol2, stream=stream)
    m.forward_host_async(xsh_t, osh, stream=stream)  # slot 0 again
    m.host_join(stream)
    m.sync_status(stream)
    assert np.array_equal(osh.numpy(), want)
    m.close()


@pytest.mark.parametrize("sync", [False, True])
def test_batch_copy_follows_stream_work(sync):
    """The first call of a batch copies its input only after the work already on its stream: the
    input buffer is filled by a device-to-host copy queued behind a ~25 ms sleep kernel, and the
    masks must be those of the new input, not of the zeros the buffer held before."""
    cfg = synth.TINY
    B, T = 2, 17
    W, _ = case(cfg, B, T, True)
    m = model_for(cfg, W, B, T)
    x1 = synth.make_stft_repr(cfg, B, T, seed=31)
    want = device_masks(m, x1)
    stream = torch.cuda.current_stream()
    xin = torch.zeros(x1.shape).pin_memory()
    out = m._out_like(xin, None)
    xd = torch.from_numpy(x1).cuda()
    torch.cuda.synchronize()
    torch.cuda._sleep(50_000_000)
    xin.copy_(xd, non_blocking=True)
    if sync:
        m.forward_host(xin, out, stream=stream)
    else:
        m.forward_host_async(xin, out, stream=stream)
        m.host_join(stream)
        m.sync_status(stream)
    assert np.array_equal(out.numpy(), want)
    m.close()
