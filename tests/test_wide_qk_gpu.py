"""Attention whose q and k are deeper than v, through the C ABI (GPU), against the oracle.

"evaluation.md", section "BS PolarFormer: the same quality for a quarter of the
arithmetic": that model's positional encoding doubles the depth of q and k (128) and leaves v at
64, and the fix it names is "a fused attention that tolerates v being narrower than q".  The
pages define neither PoPE nor that model's 62-band table, so the shape is built on this model's
60 mel bands with rotary positions on the 128-deep q and k (mrf_config.dim_head_v = 64): the
tensor-core kernel with two 64-wide q/k atoms per tile; a 32/16 head on the CUDA-core kernel;
and the fp32 debug schedule.  Bars as for the other configurations: fp16 max |diff| <= 2e-2 and
SNR >= 40 dB, fp32 debug <= 1e-4 relative."""
import dataclasses

import numpy as np
import pytest

import synth
from oracle import model as oracle_model
from parity import case, rel_err, snr_db

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


def run(cfg, B, T, compute, graph=True):
    from axial_band_split_b200 import mrf
    W, x = case(cfg, B, T, compute != mrf.MRF_FP32_DEBUG)
    m = mrf.Model(cfg, W, max_batch=B, max_frames=T, compute=compute)
    m.set_graph(graph)
    out = m.forward(torch.from_numpy(x).cuda())
    m.sync_status()
    got = out.cpu().numpy()
    m.close()
    return got, oracle_model.forward(x, cfg, W)


def check16(got, ref, what):
    assert np.isfinite(got).all()
    err, snr = float(np.abs(got - ref).max()), snr_db(got, ref)
    print(f"{what}: max|diff|={err:.3e} snr={snr:.1f} dB")
    assert err <= 2e-2 and snr >= 40.0, f"{what}: {err:.3e} {snr:.1f} dB"


@pytest.mark.parametrize("B,T", [(1, 150), (2, 260)])
def test_wide_qk_tensor_core_fp16(B, T):
    from axial_band_split_b200 import mrf
    check16(*run(synth.WIDE_QK, B, T, mrf.MRF_FP16), f"q,k 128 / v 64, B={B} T={T}")


def test_wide_qk_bf16():
    from axial_band_split_b200 import mrf
    cfg = synth.WIDE_QK
    W = synth.make_weights(cfg, oracle_model.band_tables(cfg.sample_rate, cfg.n_fft, cfg.num_bands)["widths"],
                           seed=0, bf16=True)
    x = synth.make_stft_repr(cfg, 1, 150, seed=1)
    m = mrf.Model(cfg, W, max_batch=1, max_frames=150, compute=mrf.MRF_BF16)
    got = m.forward(torch.from_numpy(x).cuda()).cpu().numpy()
    m.sync_status()
    m.close()
    check16(got, oracle_model.forward(x, cfg, W), "q,k 128 / v 64, bf16")


def test_wide_qk_fp32_debug():
    from axial_band_split_b200 import mrf
    got, ref = run(synth.WIDE_QK, 1, 64, mrf.MRF_FP32_DEBUG)
    print(f"fp32 debug: rel {rel_err(got, ref):.2e}")
    assert rel_err(got, ref) <= 1e-4


def test_narrow_v_cuda_core_kernel():
    # q, k 32 and v 16 per head: the CUDA-core attention of the tensor-core schedule, and the
    # fp32 debug schedule
    from axial_band_split_b200 import mrf
    cfg = dataclasses.replace(synth.TINY, dim_head=32, dim_head_v=16)
    got, ref = run(cfg, 2, 17, mrf.MRF_FP16)
    check16(got, ref, "tiny q,k 32 / v 16")
    got, ref = run(cfg, 2, 17, mrf.MRF_FP32_DEBUG)
    assert rel_err(got, ref) <= 1e-4
