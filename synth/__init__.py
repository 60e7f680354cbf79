"""Seeded synthetic inputs shared by the CUDA path's tests/bench and by the oracle.

This module holds no arithmetic of the method itself (no band table, norm, attention,
mask head or overlap average). It produces:

* ``ModelConfig`` and the named workload presets (the model shapes of the Mel-Band
  RoFormer vocals checkpoint and a tiny correctness model);
* random-init weights for a given list of per-band input widths (the widths come from
  the caller, which derives them from its own band tables);
* synthetic stereo audio (harmonic tone stacks, pink noise, click transients) and its
  STFT in float64 (periodic Hann, centered, reflect padded, unnormalised), packed as
  ``stft_repr[B, F*2, T, 2]`` with row ``f*2 + s``.

Shapes and recipe follow "Mel-Band RoFormer — architecture, inference hot path & RTX 3050
feasibility" (section "The forward chain": n_fft 2048, hop 441, Hann, center, reflect;
stereo merged into the frequency axis) and the model card "musetric/vocal-separation-
roformer-onnx" (section "Signature": stft_repr float32 [1, 2050, T, 2]).  The tone stack
follows ``mixes()`` of package/scripts/export-roformer.py in "@audio/neural-separate 0.4.0
→ 0.5.0" (110..1760 Hz, amplitude 1/k, L/R scaled differently); the noise floor follows
``write()`` in package/scripts/reference.py on the same page (no band may be silent).
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np

__all__ = [
    "ModelConfig", "preset", "PRESETS", "weight_shapes", "make_weights", "round_bf16",
    "synth_audio", "stft_stereo", "make_stft_repr", "clip_chunks",
]


@dataclasses.dataclass(frozen=True)
class ModelConfig:
    """Hyper-parameters of one Mel-Band RoFormer core (the fields of its config.json)."""
    sample_rate: int = 44100
    n_fft: int = 2048
    hop: int = 441
    audio_channels: int = 2
    num_bands: int = 60
    dim: int = 384
    depth: int = 6
    heads: int = 8
    dim_head: int = 64
    dim_head_v: int = 0        # width of v per head; 0: dim_head (q, k and v equally wide)
    ff_mult: int = 4
    ff_act: int = 0            # feed-forward activation: 0 GELU (the pages), 1 GEGLU (variant)
    mask_hidden_mult: int = 4
    mask_depth: int = 2
    num_stems: int = 1
    zero_dc: bool = False
    rope_theta: float = 10000.0

    @property
    def n_freqs(self) -> int:
        return self.n_fft // 2 + 1

    @property
    def rows(self) -> int:
        return self.n_freqs * self.audio_channels

    @property
    def ff_inner(self) -> int:
        return self.dim * self.ff_mult

    @property
    def mask_hidden(self) -> int:
        return self.dim * self.mask_hidden_mult

    @property
    def head_v(self) -> int:
        return self.dim_head_v or self.dim_head

    @property
    def attn_inner(self) -> int:
        """Width of the attention output (heads x v width): the output projection's input."""
        return self.heads * self.head_v


# Workload presets: model, batch, frames.  "tiny" is the small correctness model;
# "vocals" is the dim-384 / depth-6 / 60-band vocals checkpoint shape.
TINY = ModelConfig(n_fft=256, num_bands=8, dim=64, depth=1, heads=4, dim_head=16)
# An attention whose q and k are twice as wide as v (the shape of the BS PolarFormer attention of
# "evaluation.md", section "BS PolarFormer: the same quality for a quarter of the
# arithmetic": 8 heads, q and k of 128 against v of 64), on the vocals band split, with rotary
# positions on q and k.
WIDE_QK = ModelConfig(dim=256, depth=1, heads=8, dim_head=128, dim_head_v=64)
VOCALS = ModelConfig()
DEUX = ModelConfig(dim=256, depth=12, num_stems=2)

PRESETS = {
    "tiny_T32": (TINY, 1, 32),
    "vocals_T801": (VOCALS, 1, 801),
    "vocals_T1100": (VOCALS, 1, 1100),
    "vocals_B8_T801": (VOCALS, 8, 801),
}


def preset(name: str):
    """(ModelConfig, B, T) of a named workload; ``vocals_T<n>`` gives any window length."""
    if name in PRESETS:
        return PRESETS[name]
    if name.startswith("vocals_T"):
        return VOCALS, 1, int(name[len("vocals_T"):])
    raise KeyError(name)


def weight_shapes(cfg: ModelConfig, widths):
    """Named parameter shapes in PyTorch [out, in] layout, in a fixed order.

    Names follow the checkpoint paths the pages print (band_split.to_features.*,
    layers.{l}.{0=time,1=band}.layers.0.{0=attn,1=ff}.*, mask_estimators.{s}.to_freqs.*).
    ``widths`` are the per-band input widths d_in = 2 * bins * channels.
    """
    D, A, H, FF, MH = cfg.dim, cfg.attn_inner, cfg.heads, cfg.ff_inner, cfg.mask_hidden
    QKV = H * (2 * cfg.dim_head + cfg.head_v)  # q and k of dim_head, v of head_v per head
    out = []
    for k, w in enumerate(widths):
        p = f"band_split.to_features.{k}."
        out += [(p + "0.gamma", (w,)), (p + "1.weight", (D, w)), (p + "1.bias", (D,))]
    for l in range(cfg.depth):
        for a in range(2):
            p = f"layers.{l}.{a}."
            q = p + "layers.0.0."
            out += [(q + "norm.gamma", (D,)), (q + "to_qkv.weight", (QKV, D)),
                    (q + "to_gates.weight", (H, D)), (q + "to_gates.bias", (H,)),
                    (q + "to_out.0.weight", (D, A))]
            f = p + "layers.0.1.net."
            F1 = 2 * FF if cfg.ff_act == 1 else FF  # GEGLU: value and gate halves
            out += [(f + "0.gamma", (D,)), (f + "1.weight", (F1, D)), (f + "1.bias", (F1,)),
                    (f + "4.weight", (D, FF)), (f + "4.bias", (D,))]
            out += [(p + "norm.gamma", (D,))]
    for s in range(cfg.num_stems):
        for k, w in enumerate(widths):
            p = f"mask_estimators.{s}.to_freqs.{k}.0."
            dims = [D] + [MH] * cfg.mask_depth + [2 * w]
            for i in range(len(dims) - 1):
                out += [(p + f"{2 * i}.weight", (dims[i + 1], dims[i])),
                        (p + f"{2 * i}.bias", (dims[i + 1],))]
    return out


def round_bf16(a):
    """float32 values rounded to bfloat16 (round to nearest, ties to even), returned as float32."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) & 0xFFFF0000
    return u.astype(np.uint32).view(np.float32)


def make_weights(cfg: ModelConfig, widths, seed: int = 0, fp16: bool = True, std: float = 0.02,
                 bf16: bool = False):
    """Random-init weights: every Linear weight and bias ~ N(0, std); every norm gamma
    1 + N(0, std).  With ``fp16`` (or ``bf16``) each tensor is rounded to float16 (bfloat16)
    once (round to nearest even) and returned as float32 holding exactly those values, so both
    sides of a comparison use the same rounded weights."""
    rng = np.random.Generator(np.random.PCG64(seed))
    out = {}
    for name, shape in weight_shapes(cfg, widths):
        a = rng.standard_normal(shape, dtype=np.float64) * std
        if name.endswith("gamma"):
            a = a + 1.0
        a = a.astype(np.float32)
        if bf16:
            a = round_bf16(a)
        elif fp16:
            a = a.astype(np.float16).astype(np.float32)
        out[name] = a
    return out


def _pink(rng, n):
    """Pink (1/f power) noise by shaping white noise's spectrum, unit RMS."""
    w = np.fft.rfft(rng.standard_normal(n))
    f = np.arange(w.size, dtype=np.float64)
    f[0] = 1.0
    x = np.fft.irfft(w / np.sqrt(f), n)
    return x / np.sqrt(np.mean(x * x))


def synth_audio(n_samples: int, seed: int = 1, sr: int = 44100, clicks: bool = False):
    """Stereo float64 audio (2, n): gliding harmonic tone stacks, different per channel,
    plus pink noise at -20 dBFS RMS, plus optional unit clicks every ~0.5 s at -6 dBFS."""
    rng = np.random.Generator(np.random.PCG64(seed))
    t = np.arange(n_samples, dtype=np.float64) / sr
    out = np.zeros((2, n_samples))
    for s, (base, gain) in enumerate(((110.0, 0.2), (146.8, 0.16))):
        glide = 1.0 + 0.02 * np.sin(2 * math.pi * 0.1 * t + s)
        phase = 2 * math.pi * np.cumsum(base * glide) / sr
        tone = sum(np.sin(phase * (2 ** (k - 1))) / k for k in range(1, 6))
        out[s] = gain * tone
    noise_rms = 10 ** (-20 / 20)
    out += noise_rms * np.stack([_pink(rng, n_samples), _pink(rng, n_samples)])
    if clicks:
        step = sr // 2
        for i in range(step // 3, n_samples, step):
            out[:, i] += 10 ** (-6 / 20)
    return out


def stft_stereo(audio, n_fft: int = 2048, hop: int = 441):
    """Complex STFT (channels, n_fft//2+1, frames) in float64: periodic Hann of n_fft,
    centered with reflect padding of n_fft//2, unnormalised; frames = 1 + n // hop."""
    audio = np.asarray(audio, dtype=np.float64)
    pad = n_fft // 2
    x = np.pad(audio, ((0, 0), (pad, pad)), mode="reflect")
    frames = 1 + (x.shape[1] - n_fft) // hop
    win = 0.5 - 0.5 * np.cos(2 * math.pi * np.arange(n_fft) / n_fft)
    idx = np.arange(n_fft)[None, :] + hop * np.arange(frames)[:, None]
    seg = x[:, idx] * win                                  # (C, frames, n_fft)
    spec = np.fft.rfft(seg, axis=-1)                        # (C, frames, F)
    return np.transpose(spec, (0, 2, 1))


def pack_stft_repr(spec):
    """(C, F, T) complex -> float32 [F*C, T, 2], row f*C + s."""
    C, F, T = spec.shape
    z = np.stack([spec.real, spec.imag], -1)               # (C, F, T, 2)
    return np.ascontiguousarray(np.transpose(z, (1, 0, 2, 3)).reshape(F * C, T, 2)).astype(np.float32)


def clip_chunks(B: int, T: int, hop: int = 441, stride: int = 317520, seed: int = 1, sr: int = 44100):
    """B chunks of (T-1)*hop samples cut at ``stride`` from one clip with clicks."""
    n = (T - 1) * hop
    clip = synth_audio(stride * (B - 1) + n, seed=seed, sr=sr, clicks=True)
    return [clip[:, i * stride: i * stride + n] for i in range(B)]


def make_stft_repr(cfg: ModelConfig, B: int, T: int, seed: int = 1):
    """Input ``stft_repr`` float32 [B, F*2, T, 2] for a workload.

    The tiny model takes i.i.d. N(0, 1) values; the full-size model takes the STFT of
    synthetic audio of (T-1)*hop samples (one clip cut into chunks when B > 1)."""
    if cfg.n_fft <= 256:
        rng = np.random.Generator(np.random.PCG64(seed + 1))
        return rng.standard_normal((B, cfg.rows, T, 2)).astype(np.float32)
    n = (T - 1) * cfg.hop
    if B == 1:
        chunks = [synth_audio(n, seed=seed, sr=cfg.sample_rate)]
    else:
        chunks = clip_chunks(B, T, hop=cfg.hop, seed=seed, sr=cfg.sample_rate)
    out = np.stack([pack_stft_repr(stft_stereo(c, cfg.n_fft, cfg.hop)) for c in chunks])
    assert out.shape == (B, cfg.rows, T, 2), out.shape
    return out
