"""Mel-Band RoFormer core forward, plain float64 NumPy (oracle; test infrastructure only).

Each function restates one step as the pages describe it:

* "Mel-Band RoFormer — architecture, inference hot path & RTX 3050 feasibility"
  (page 1): section "The forward chain" (gather, BandSplit, depth x (time, band)
  transformer, mask estimator, scatter-add then divide by the band count), section "The
  mel-band split, exactly" (RMSNorm is F.normalize(x) * sqrt(dim) * gamma), section "The two
  transformers are not the same shape" (own rotary embedding per transformer; to_qkv and
  to_out without bias, to_gates with bias, per-head sigmoid gate), section "Parameter
  accounting" (mask MLP Linear-Tanh-Linear-Tanh-Linear-GLU), section "FLOP shares".
* "@audio/neural-separate 0.4.0 → 0.5.0" (page 5), package/scripts/export-roformer.py,
  classes ``Block``, ``Attn``, ``FF`` and ``Mod.forward``: feed-forward is
  norm -> Linear -> GELU -> Linear with biases; each transformer ends with its own norm;
  attention is softmax(q k^T * scale) v with q, k rotated; the norm clamps ||x|| at 1e-12.
* "musetric/vocal-separation-roformer-onnx" (page 3), section "Signature": stft_repr
  [B, F*2, T, 2] in, per-bin complex masks of the same shape out, already averaged; with
  more than one stem, one mask per stem over the shared trunk (page 1, "The forward chain":
  MaskEstimator per stem), and the separated spectra are mask times mixture (complex).

Readings where the pages leave a value open: RoPE theta 10000 on interleaved pairs
(2i, 2i+1), positions 0..n-1 along the attended axis (the band index on the band axis);
attention scale dim_head**-0.5; gates from the normed input; first GLU half is the value.

No blocking, fusion or reordering beyond these definitions, except that attention loops
over sequences one at a time to bound memory (sequences are independent).
"""
from __future__ import annotations

import math

import numpy as np
from scipy.special import erf

from .tables import band_tables

NORM_EPS = 1e-12


def rms_norm(x, gamma):
    """x / max(||x||_2, 1e-12) * sqrt(d) * gamma over the last axis (no mean, no bias)."""
    d = x.shape[-1]
    n = np.sqrt(np.sum(x * x, axis=-1, keepdims=True))
    return x / np.maximum(n, NORM_EPS) * math.sqrt(d) * gamma


def gelu(x):
    """GELU with the exact error function: x * (1 + erf(x / sqrt 2)) / 2."""
    return 0.5 * x * (1.0 + erf(x / math.sqrt(2.0)))


def sigmoid(x):
    return 1.0 / (1.0 + np.exp(-x))


def rope_angles(n: int, dim_head: int, theta: float):
    """phi[p, i] = p * theta^(-2i/dim_head), p = 0..n-1, i = 0..dim_head/2-1."""
    inv = theta ** (-np.arange(0, dim_head, 2, dtype=np.float64) / dim_head)
    return np.arange(n, dtype=np.float64)[:, None] * inv[None, :]


def rope(x, theta: float):
    """Rotate interleaved pairs of the last axis by the position (second-to-last axis):
    (x_2i, x_2i+1) -> (x_2i cos phi - x_2i+1 sin phi, x_2i+1 cos phi + x_2i sin phi)."""
    n, dh = x.shape[-2], x.shape[-1]
    phi = rope_angles(n, dh, theta)
    c, s = np.cos(phi), np.sin(phi)
    x0, x1 = x[..., 0::2], x[..., 1::2]
    out = np.empty_like(x)
    out[..., 0::2] = x0 * c - x1 * s
    out[..., 1::2] = x1 * c + x0 * s
    return out


def softmax(s, axis=-1):
    m = np.max(s, axis=axis, keepdims=True)
    e = np.exp(s - m)
    return e / np.sum(e, axis=axis, keepdims=True)


def attend(q, k, v):
    """softmax(q k^T / sqrt(dh)) v over the key axis; q, k, v (..., n, dh)."""
    dh = q.shape[-1]
    s = np.matmul(q, np.swapaxes(k, -1, -2)) * (dh ** -0.5)
    return np.matmul(softmax(s), v)


def attention(x, w, heads: int, dim_head: int, theta: float, dim_head_v: int = 0):
    """Pre-norm gated multi-head attention over x (S sequences, n, D) -> (S, n, D).

    a = norm(x); [q; k; v] = a W_qkv^T with features ordered (which, head, d); q, k
    rotated; o_h = attend(q_h, k_h, v_h) * sigmoid(a W_g^T + b_g)_h; out = concat_h o_h W_o^T.
    With dim_head_v (v narrower than q and k, as in the PolarFormer attention of
    "evaluation.md", section "BS PolarFormer: the same quality for a quarter of the arithmetic")
    the projection's features are q (heads x dim_head), k (heads x dim_head), v (heads x
    dim_head_v), each ordered (head, d); the softmax scale stays dim_head^-0.5 (the q.k width).
    """
    S, n, D = x.shape
    dv = dim_head_v or dim_head
    A = heads * dv
    Aqk = heads * dim_head
    out = np.empty_like(x)
    for i in range(S):
        a = rms_norm(x[i], w["norm.gamma"])                          # (n, D)
        qkv = a @ w["to_qkv.weight"].T                                # (n, 2 Aqk + A)
        q = rope(np.transpose(qkv[:, :Aqk].reshape(n, heads, dim_head), (1, 0, 2)), theta)   # (h, n, dh)
        k = rope(np.transpose(qkv[:, Aqk:2 * Aqk].reshape(n, heads, dim_head), (1, 0, 2)), theta)
        v = np.transpose(qkv[:, 2 * Aqk:].reshape(n, heads, dv), (1, 0, 2))
        o = attend(q, k, v)                                          # (h, n, dh)
        g = sigmoid(a @ w["to_gates.weight"].T + w["to_gates.bias"])  # (n, h)
        o = o * np.transpose(g)[:, :, None]
        o = np.transpose(o, (1, 0, 2)).reshape(n, A)
        out[i] = o @ w["to_out.0.weight"].T
    return out


def feed_forward(x, w, ff_act: int = 0):
    """norm -> Linear(D, FF) + b -> GELU -> Linear(FF, D) + b.  ff_act 1 (the GEGLU variant):
    the first projection is Linear(D, 2 FF) and its halves combine as value * GELU(gate), the
    first half the value (Shazeer, "GLU Variants Improve Transformer", 2020)."""
    a = rms_norm(x, w["net.0.gamma"])
    y = a @ w["net.1.weight"].T + w["net.1.bias"]
    if ff_act == 1:
        value, gate = np.split(y, 2, axis=-1)
        h = value * gelu(gate)
    else:
        h = gelu(y)
    return h @ w["net.4.weight"].T + w["net.4.bias"]


def transformer(x, w, heads, dim_head, theta, ff_act: int = 0, dim_head_v: int = 0):
    """x += attn(x); x += ff(x); return norm_out(x).  x (S, n, D)."""
    aw = {k[len("layers.0.0."):]: v for k, v in w.items() if k.startswith("layers.0.0.")}
    fw = {k[len("layers.0.1."):]: v for k, v in w.items() if k.startswith("layers.0.1.")}
    x = attention(x, aw, heads, dim_head, theta, dim_head_v) + x
    x = feed_forward(x, fw, ff_act) + x
    return rms_norm(x, w["norm.gamma"])


def _sub(weights, prefix):
    return {k[len(prefix):]: v for k, v in weights.items() if k.startswith(prefix)}


def band_split(spec, tab, weights):
    """spec (rows, T, 2) -> X (T, n_bands, D): per band gather its features
    (j*2 + s)*2 + c, RMSNorm(d_in), Linear(d_in, D) with bias."""
    feats = spec[tab["feat_row"], :, tab["feat_c"]].T                # (T, sum d_in)
    nb = len(tab["widths"])
    off = np.concatenate([[0], np.cumsum(tab["widths"])])
    D = weights["band_split.to_features.0.1.bias"].shape[0]
    X = np.empty((spec.shape[1], nb, D), dtype=spec.dtype)
    for k in range(nb):
        p = f"band_split.to_features.{k}."
        xk = rms_norm(feats[:, off[k]:off[k + 1]], weights[p + "0.gamma"])
        X[:, k] = xk @ weights[p + "1.weight"].T + weights[p + "1.bias"]
    return X


def mask_estimator(X, tab, weights, stem: int = 0, mask_depth: int = 2):
    """Per band: Linear-Tanh x mask_depth, Linear(hidden, 2 d_in), GLU -> (T, sum d_in)."""
    nb = len(tab["widths"])
    out = []
    for k in range(nb):
        p = f"mask_estimators.{stem}.to_freqs.{k}.0."
        h = X[:, k]
        for i in range(mask_depth):
            h = np.tanh(h @ weights[p + f"{2 * i}.weight"].T + weights[p + f"{2 * i}.bias"])
        i = mask_depth
        y = h @ weights[p + f"{2 * i}.weight"].T + weights[p + f"{2 * i}.bias"]
        d = tab["widths"][k]
        out.append(y[:, :d] * sigmoid(y[:, d:]))
    return np.concatenate(out, axis=1)


def overlap_average(m, tab, n_rows: int):
    """Scatter-add band features back to rows, then weight each row by 1 / (bands over
    its bin) (0 at DC with zero_dc).  m (T, sum d_in) -> masks (rows, T, 2)."""
    T = m.shape[0]
    acc = np.zeros((n_rows, T, 2), dtype=m.dtype)
    np.add.at(acc, (tab["feat_row"], slice(None), tab["feat_c"]), m.T)
    return acc * tab["row_weight"][:, None, None]


def apply_masks(stft_repr, masks):
    """The separated spectra: each stem's complex mask times the mixture's complex STFT
    (page 1, section "The forward chain": multiply the original complex STFT).  stft_repr
    (B, R, T, 2) and masks (B, R, T, 2) or (B, stems, R, T, 2), the last axis (re, im)."""
    x = np.asarray(stft_repr, dtype=np.float64)
    m = np.asarray(masks, dtype=np.float64)
    xc = x[..., 0] + 1j * x[..., 1]
    mc = m[..., 0] + 1j * m[..., 1]
    if mc.ndim == xc.ndim + 1:  # one mixture under every stem's mask
        xc = xc[:, None]
    y = mc * xc
    return np.stack([y.real, y.imag], axis=-1)


def forward(stft_repr, cfg, weights, dtype=np.float64, return_stages: bool = False):
    """masks = core(stft_repr); stft_repr (B, F*C, T, 2) -> masks (B, F*C, T, 2)
    (or (B, stems, F*C, T, 2) for more than one stem).  ``cfg`` is any object with the
    model fields (sample_rate, n_fft, num_bands, audio_channels, dim, depth, heads,
    dim_head, mask_depth, num_stems, zero_dc, rope_theta)."""
    tab = band_tables(cfg.sample_rate, cfg.n_fft, cfg.num_bands, cfg.audio_channels, cfg.zero_dc)
    W = {k: np.asarray(v, dtype=dtype) for k, v in weights.items()}
    x_in = np.asarray(stft_repr, dtype=dtype)
    B, R, T, _ = x_in.shape
    outs, stages = [], []
    for b in range(B):
        st = {}
        X = band_split(x_in[b], tab, W)                               # (T, nb, D)
        st["band_split"] = X.copy()
        for l in range(cfg.depth):
            tw = _sub(W, f"layers.{l}.0.")
            bw = _sub(W, f"layers.{l}.1.")
            ff_act = getattr(cfg, "ff_act", 0)
            dv = getattr(cfg, "dim_head_v", 0)
            X = np.transpose(transformer(np.transpose(X, (1, 0, 2)), tw, cfg.heads,
                                         cfg.dim_head, cfg.rope_theta, ff_act, dv), (1, 0, 2))
            st[f"layer{l}.time"] = X.copy()
            X = transformer(X, bw, cfg.heads, cfg.dim_head, cfg.rope_theta, ff_act, dv)
            st[f"layer{l}.band"] = X.copy()
        per_stem = []
        for s in range(cfg.num_stems):
            m = mask_estimator(X, tab, W, s, cfg.mask_depth)
            st[f"mask{s}"] = m.copy()
            per_stem.append(overlap_average(m, tab, R))
        outs.append(per_stem[0] if cfg.num_stems == 1 else np.stack(per_stem))
        stages.append(st)
    out = np.stack(outs)
    return (out, stages) if return_stages else out


def param_count(cfg, widths):
    """Number of parameters of the core (weights, biases, norm gammas; the rotary
    embedding's fixed frequencies are not parameters)."""
    D, H, dh = cfg.dim, cfg.heads, cfg.dim_head
    dv = getattr(cfg, "dim_head_v", 0) or dh
    A = H * dv                      # attention output width (v)
    QKV = H * (2 * dh + dv)
    FF = D * cfg.ff_mult
    MH = D * cfg.mask_hidden_mult
    n = sum(w + D * w + D for w in widths)
    F1 = 2 * FF if getattr(cfg, "ff_act", 0) == 1 else FF   # GEGLU: value and gate halves
    per_tr = (D + QKV * D + H * D + H + D * A) + (D + F1 * D + F1 + D * FF + D) + D
    n += 2 * cfg.depth * per_tr
    for _ in range(cfg.num_stems):
        for w in widths:
            dims = [D] + [MH] * cfg.mask_depth + [2 * w]
            n += sum(dims[i] * dims[i + 1] + dims[i + 1] for i in range(len(dims) - 1))
    return n


def mac_count(cfg, widths, B: int, T: int):
    """Multiply-accumulates of one forward, by term (the FLOP accounting of the pages'
    section "FLOP shares"; FLOPs = 2 * MACs)."""
    D, H, dh = cfg.dim, cfg.heads, cfg.dim_head
    dv = getattr(cfg, "dim_head_v", 0) or dh
    A = H * dv                      # attention output width (v)
    FF = D * cfg.ff_mult
    MH = D * cfg.mask_hidden_mult
    nb = len(widths)
    tok = B * T * nb
    L = cfg.depth
    per_axis = {
        "qkv": L * tok * D * H * (2 * dh + dv),
        "gates": L * tok * D * H,
        "out": L * tok * A * D,
        "ff1": L * tok * D * FF * (2 if getattr(cfg, "ff_act", 0) == 1 else 1),
        "ff2": L * tok * FF * D,
    }
    attn_time = L * (B * nb * H) * T * T * (dh + dv)   # q k^T over dh, p v over dv
    attn_band = L * (B * T * H) * nb * nb * (dh + dv)
    band_split_m = B * T * D * sum(widths)
    mask = cfg.num_stems * B * T * sum(D * MH + (cfg.mask_depth - 1) * MH * MH + MH * 2 * w
                                       for w in widths)
    linear = 2 * sum(per_axis.values())
    return {
        "per_axis": per_axis, "linear_trunk": linear, "attn_time": attn_time,
        "attn_band": attn_band, "trunk": linear + attn_time + attn_band,
        "band_split": band_split_m, "mask": mask,
        "total": linear + attn_time + attn_band + band_split_m + mask,
    }
