"""Host-side checks of the C ABI: the library loads, exports every declared symbol,
builds the same band tables as the oracle bit for bit, and rejects bad arguments with
the documented status codes before touching a GPU."""
import ctypes
import dataclasses
import os
import re

import numpy as np
import pytest

import synth
from axial_band_split_b200 import mrf
from oracle import tables

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_symbols():
    src = open(os.path.join(ROOT, "include", "mrf.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(mrf_[a-z_]+)\s*\(", src)))


def test_exports_every_declared_symbol():
    L = mrf.lib()
    decl = declared_symbols()
    assert len(decl) >= 10
    for name in decl:
        assert hasattr(L, name), name
    assert sorted(mrf.EXPORTS) == decl


@pytest.mark.parametrize("cfg", [synth.VOCALS, synth.TINY,
                                 dataclasses.replace(synth.VOCALS, zero_dc=True)])
def test_band_tables_bit_exact_against_oracle(cfg):
    got = mrf.band_tables(cfg)
    ref = tables.band_tables(cfg.sample_rate, cfg.n_fft, cfg.num_bands, cfg.audio_channels, cfg.zero_dc)
    assert np.array_equal(got["first_bin"], ref["first_bin"])
    assert np.array_equal(got["last_bin"], ref["last_bin"])
    assert np.array_equal(got["width"], ref["widths"])
    assert np.array_equal(got["feat_row"], ref["feat_row"])
    # 1/1 and 1/2 are exact in float32; 0 at DC with zero_dc
    assert np.array_equal(got["row_weight"], ref["row_weight"].astype(np.float32))


def test_band_tables_rejects_bad_config():
    bad = dataclasses.replace(synth.VOCALS, num_bands=0)
    with pytest.raises(mrf.MrfError) as e:
        mrf.band_tables(bad)
    assert e.value.status == -1
    # far more bands than bins: some band is empty
    with pytest.raises(mrf.MrfError):
        mrf.band_tables(dataclasses.replace(synth.TINY, num_bands=120))


def tiny_weights(cfg=synth.TINY):
    widths = mrf.band_tables(cfg)["width"]
    return synth.make_weights(cfg, widths, fp16=False)


def test_create_validates_before_any_device_work():
    cfg = synth.TINY
    W = tiny_weights()
    with pytest.raises(mrf.MrfError) as e:                      # stems out of range
        mrf.Model(dataclasses.replace(cfg, num_stems=5), W)
    assert e.value.status == -1
    with pytest.raises(mrf.MrfError) as e:                      # a second stem without its weights
        mrf.Model(dataclasses.replace(cfg, num_stems=2), W)
    assert e.value.status == -7 and "mask_estimators.1." in str(e.value)
    with pytest.raises(mrf.MrfError) as e:                      # odd head width
        mrf.Model(dataclasses.replace(cfg, dim_head=15), W)
    assert e.value.status == -1
    W2 = dict(W)
    W2.pop("layers.0.1.norm.gamma")
    with pytest.raises(mrf.MrfError) as e:                      # missing weight
        mrf.Model(cfg, W2, max_frames=32, compute=mrf.MRF_FP32_DEBUG)
    assert e.value.status == -7 and "missing weight" in str(e.value)
    W3 = dict(W)
    W3["layers.0.0.layers.0.0.to_qkv.weight"] = W3["layers.0.0.layers.0.0.to_qkv.weight"][:-1]
    with pytest.raises(mrf.MrfError) as e:                      # wrong shape
        mrf.Model(cfg, W3, max_frames=32, compute=mrf.MRF_FP32_DEBUG)
    assert e.value.status == -2
    W4 = dict(W)
    W4["bogus.weight"] = np.zeros(3, np.float32)
    with pytest.raises(mrf.MrfError) as e:                      # unexpected name
        mrf.Model(cfg, W4, max_frames=32, compute=mrf.MRF_FP32_DEBUG)
    assert e.value.status == -7


def test_null_arguments():
    L = mrf.lib()
    h = ctypes.c_void_p()
    assert L.mrf_create(None, None, 0, ctypes.byref(h)) == -1
    assert L.mrf_forward(None, None, None, 1, 1, None) == -1
    assert L.mrf_sync_status(None, None) == -1
    L.mrf_destroy(None)
    assert L.mrf_launches_per_forward(None, 1, 1) == -1
    assert b"null" in L.mrf_last_error(None)


def test_accounting_matches_oracle_mac_count():
    # the bench's roofline numerators agree with the oracle's pinned MAC accounting
    from axial_band_split_b200 import accounting
    from oracle import model as om
    for cfg, B, T in [(synth.VOCALS, 1, 801), (synth.VOCALS, 1, 1100), (synth.TINY, 2, 32)]:
        widths = tables.band_tables(cfg.sample_rate, cfg.n_fft, cfg.num_bands)["widths"]
        m = om.mac_count(cfg, widths, B, T)
        assert accounting.total_flops(cfg, widths, B, T) == 2 * m["total"]
        assert accounting.attention_flops(cfg, widths, B, T) == 2 * (m["attn_time"] + m["attn_band"])
    assert accounting.audio_seconds(synth.VOCALS, 1, 1100) == pytest.approx(11.0)
