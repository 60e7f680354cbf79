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


def _oracle_window(args):
    """Worker of oracle_windows: regenerate the seeded weights and inputs, run one window."""
    import os
    cfg, B, T, seed, b = args
    W, x = case(cfg, B, T, True, seed)
    return b, oracle_model.forward(x[b:b + 1], cfg, W)


def oracle_windows(cfg, B, T, seed=1, workers=4):
    """The oracle's masks for every window of a seeded B-window workload, windows in parallel
    processes (started with spawn, so a process that already holds a CUDA context is safe),
    each process with an equal share of the host's BLAS threads."""
    import concurrent.futures as cf
    import multiprocessing as mp
    import os
    workers = max(1, min(workers, B))
    threads = str(max(1, (os.cpu_count() or 1) // workers))
    env = {k: threads for k in ("OMP_NUM_THREADS", "OPENBLAS_NUM_THREADS", "MKL_NUM_THREADS")}
    old = {k: os.environ.get(k) for k in env}
    os.environ.update(env)
    try:
        with cf.ProcessPoolExecutor(workers, mp_context=mp.get_context("spawn")) as ex:
            res = dict(ex.map(_oracle_window, [(cfg, B, T, seed, b) for b in range(B)]))
    finally:
        for k, v in old.items():
            if v is None:
                os.environ.pop(k, None)
            else:
                os.environ[k] = v
    return np.concatenate([res[b] for b in range(B)])
