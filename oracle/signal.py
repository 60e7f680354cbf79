"""Spectral front and back end and the chunked separation loop, plain float64 NumPy (oracle;
test infrastructure only: only tests/, the smoke check and bench.py's CPU baseline use it).

Each function restates a step of "Mel-Band RoFormer — architecture, inference hot path & RTX
3050 feasibility":

* section "The forward chain": torch.stft with n_fft 2048, hop 441, a Hann window of 2048,
  center=True; the stereo channels merged into the frequency axis (row f * channels + s); the
  masks multiplied into the complex STFT; istft back to the waveform;
* section "Verified inference hot path", the chunk loop: 8 s chunks at a stride of 0.9 chunk,
  the mix reflect-padded by the border (chunk - stride) when it is longer than two borders, a
  short last chunk padded by reflection when more than half a chunk remains and by zeros
  otherwise, linear fades of chunk / 10 samples (fade-in forced to 1 on the first chunk,
  fade-out forced to 1 on the last), out += estimate * window and counter += window, then
  out / max(counter, 1e-8) and the border cropped.

Readings where the pages leave a detail open: the Hann window is periodic (torch.hann_window's
default); the STFT is unnormalised with reflect padding of n_fft / 2 on both sides ("musetric/
vocal-separation-roformer-onnx", section "Signature"); istft is torch.istft's definition: the
overlap-added windowed inverse real FFTs divided by the overlap-added squared window, the
first n_fft / 2 samples dropped, `length` samples kept; the fade-in and fade-out overrides are
independent conditions (a chunk that is both first and last gets neither fade); linspace(0, 1,
n) includes both ends.
"""
from __future__ import annotations

import math

import numpy as np


def hann(n: int) -> np.ndarray:
    """Periodic Hann window of length n: 0.5 - 0.5 cos(2 pi i / n)."""
    return 0.5 - 0.5 * np.cos(2.0 * math.pi * np.arange(n) / n)


def stft(audio, n_fft: int = 2048, hop: int = 441) -> np.ndarray:
    """audio (B, C, L) -> stft_repr (B, F*C, T, 2), F = n_fft/2 + 1, T = 1 + L // hop; row
    f * C + c, last axis (re, im)."""
    a = np.asarray(audio, dtype=np.float64)
    B, C, L = a.shape
    pad = n_fft // 2
    x = np.pad(a, ((0, 0), (0, 0), (pad, pad)), mode="reflect")
    T = 1 + (x.shape[-1] - n_fft) // hop
    w = hann(n_fft)
    frames = np.stack([x[..., t * hop: t * hop + n_fft] * w for t in range(T)], axis=2)  # (B, C, T, n)
    z = np.fft.rfft(frames, axis=-1)                                                    # (B, C, T, F)
    F = n_fft // 2 + 1
    out = np.empty((B, F, C, T, 2))
    out[..., 0] = np.transpose(z.real, (0, 3, 1, 2))
    out[..., 1] = np.transpose(z.imag, (0, 3, 1, 2))
    return out.reshape(B, F * C, T, 2)


def istft(spec, channels: int, length: int, n_fft: int = 2048, hop: int = 441) -> np.ndarray:
    """spec (..., F*C, T, 2) -> audio (..., C, length): per frame the inverse real FFT times
    the window, overlap-added at hop, divided by the overlap-added squared window, then the
    first n_fft/2 samples dropped and `length` kept (zeros past the signal's end)."""
    s = np.asarray(spec, dtype=np.float64)
    lead = s.shape[:-3]
    FC, T, _ = s.shape[-3:]
    F = FC // channels
    z = (s[..., 0] + 1j * s[..., 1]).reshape(lead + (F, channels, T))
    y = np.fft.irfft(np.moveaxis(z, -3, -1), n=n_fft, axis=-1)       # (..., C, T, n)
    w = hann(n_fft)
    total = n_fft + hop * (T - 1)
    sig = np.zeros(lead + (channels, total))
    env = np.zeros(total)
    for t in range(T):
        sig[..., t * hop: t * hop + n_fft] += y[..., t, :] * w
        env[t * hop: t * hop + n_fft] += w * w
    start = n_fft // 2
    keep = sig[..., start: start + length] / np.where(env[start: start + length] > 1e-11,
                                                       env[start: start + length], 1.0)
    if keep.shape[-1] < length:
        keep = np.concatenate([keep, np.zeros(lead + (channels, length - keep.shape[-1]))], axis=-1)
    return keep


def chunk_plan(length: int, sample_rate: int = 44100, chunk: int = 0):
    """The chunk loop's geometry for a mix of `length` samples: (chunk, border or 0 when the mix
    is not padded, padded length, [(offset, valid samples, tail padding mode or None)],
    fade window of the chunk).  `chunk` samples per chunk, 0 for the page's 8 s."""
    chunk = int(chunk) if chunk else int(sample_rate * 8)
    stride = int(chunk * 0.9)
    fade = chunk // 10
    border = chunk - stride
    padded = length > 2 * border
    Lp = length + 2 * border if padded else length
    chunks = []
    for off in range(0, Lp, stride):
        n = min(chunk, Lp - off)
        mode = None if n == chunk else ("reflect" if n > chunk // 2 else "zeros")
        chunks.append((off, n, mode))
    window = np.ones(chunk)
    window[:fade] = np.linspace(0.0, 1.0, fade)
    window[-fade:] = np.linspace(1.0, 0.0, fade)
    return chunk, (border if padded else 0), Lp, chunks, window


def separate(mix, estimate, sample_rate: int = 44100, chunk: int = 0):
    """The chunk loop: mix (C, L) -> stems (S, C, L), with estimate(chunk (C, chunk)) ->
    (S, C, chunk) the model run on one chunk; chunks of `chunk` samples (0: 8 s)."""
    mix = np.asarray(mix, dtype=np.float64)
    C, L = mix.shape
    chunk, border, Lp, chunks, window = chunk_plan(L, sample_rate, chunk)
    x = np.pad(mix, ((0, 0), (border, border)), mode="reflect") if border else mix
    out, counter = None, np.zeros(Lp)
    fade = chunk // 10
    for i, (off, n, mode) in enumerate(chunks):
        part = x[:, off: off + n]
        if mode == "reflect":
            part = np.pad(part, ((0, 0), (0, chunk - n)), mode="reflect")
        elif mode == "zeros":
            part = np.pad(part, ((0, 0), (0, chunk - n)))
        est = np.asarray(estimate(part), dtype=np.float64)
        if out is None:
            out = np.zeros((est.shape[0], C, Lp))
        w = window.copy()
        if off == 0:
            w[:fade] = 1.0
        if off + chunk >= Lp:
            w[-fade:] = 1.0
        out[..., off: off + n] += est[..., :n] * w[:n]
        counter[off: off + n] += w[:n]
    out = out / np.maximum(counter, 1e-8)
    return out[..., border: Lp - border] if border else out
