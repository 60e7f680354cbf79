"""Shared helpers of the GPU parity tests: seeded cases, the oracle run, error metrics."""
import functools

import numpy as np

import synth
from oracle import model as oracle_model
from oracle import tables as oracle_tables


def widths(cfg):
    return oracle_tables.band_tables(cfg.sample_rate, cfg.n_fft, cfg.num_bands, cfg.audio_channels)["widths"]


@functools.lru_cache(maxsize=8)
def case(cfg, B, T, fp16_weights, seed=1):
    """(weights, stft_repr) for a workload; weights rounded to fp16 when asked."""
    W = synth.make_weights(cfg, widths(cfg), seed=0, fp16=fp16_weights)
    x = synth.make_stft_repr(cfg, B, T, seed=seed)
    return W, x


@functools.lru_cache(maxsize=8)
def oracle_masks(cfg, B, T, fp16_weights, seed=1):
    W, x = case(cfg, B, T, fp16_weights, seed)
    return oracle_model.forward(x, cfg, W)


def rel_err(got, ref):
    return float(np.abs(got - ref).max() / max(np.abs(ref).max(), 1e-30))


def snr_db(got, ref):
    e = float(np.sum((got.astype(np.float64) - ref) ** 2))
    p = float(np.sum(ref.astype(np.float64) ** 2))
    return float("inf") if e == 0 else 10 * np.log10(p / e)
