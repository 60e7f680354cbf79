"""Algorithmic work of one core forward, per kernel kind (roofline numerators).

FLOPs count 2 per multiply-accumulate of the method's dense contractions, nothing padded
or skipped: the linear layers of "Mel-Band RoFormer — architecture, inference hot path &
RTX 3050 feasibility", section "FLOP shares" (to_qkv, to_gates, to_out, two feed-forward
projections per transformer; attention 2*n^2*dh MACs per head for q k^T and again for
p v), plus the band split and the mask MLP of section "Parameter accounting".  Bytes are
the minimum DRAM traffic of the memory-bound kernels (each input read once, each output
written once).
"""
from __future__ import annotations


def kernel_work(cfg, widths, B: int, T: int):
    """{kernel name: (kind, total per forward, launches per forward)}; kind is "flop" or "byte"."""
    D, H, dh = cfg.dim, cfg.heads, cfg.dim_head
    dv = getattr(cfg, "dim_head_v", 0) or dh   # v per head (q and k are dh deep)
    A = H * dv                                  # attention output width
    QKV = H * (2 * dh + dv)
    FF = D * cfg.ff_mult
    F1 = FF * (2 if getattr(cfg, "ff_act", 0) == 1 else 1)  # GEGLU: value and gate halves
    MH = D * cfg.mask_hidden_mult
    nb = cfg.num_bands
    L2 = 2 * cfg.depth
    BT = B * T
    NT = BT * nb
    n_feat = int(sum(widths))
    rows = (cfg.n_fft // 2 + 1) * cfg.audio_channels
    S = cfg.num_stems  # one mask estimator (and overlap average) per stem
    w = {
        "gemm_qkv": ("flop", L2 * 2 * NT * D * (QKV + H), L2),
        "attn_time_tc": ("flop", cfg.depth * 2 * (B * nb * H) * T * T * (dh + dv), cfg.depth),
        "attn_band_tc": ("flop", cfg.depth * 2 * (BT * H) * nb * nb * (dh + dv), cfg.depth),
        "gemm_out_resid": ("flop", L2 * 2 * NT * A * D, L2),
        "gemm_ff1_gelu": ("flop", L2 * 2 * NT * D * F1, L2),
        "gemm_ff1_geglu": ("flop", L2 * 2 * NT * D * F1, L2),   # the GEGLU variant's launch name
        "gemm_ff2_resid": ("flop", L2 * 2 * NT * FF * D, L2),
        # the fused feed-forward (both projections in one launch per transformer)
        "gemm_ff_fused": ("flop", L2 * 2 * NT * D * F1 + L2 * 2 * NT * FF * D, L2),
        "gemm_mask_tanh": ("flop", S * 2 * BT * nb * (D * MH + (cfg.mask_depth - 1) * MH * MH), S * cfg.mask_depth),
        "gemm_mask_glu": ("flop", S * 2 * BT * MH * 2 * n_feat, S),
        "band_split": ("flop", 2 * BT * D * n_feat, 1),
        "gemm_band_split": ("flop", 2 * BT * D * n_feat, 1),
        # stft_repr read once, normalised fp16 band features written once
        "band_gather": ("byte", B * rows * T * 2 * 4 + BT * n_feat * 2, 1),
        # fp32 debug schedule, per stem: mask features fp32 read once, masks fp32 written once (the
        # fp16 schedule averages inside the GLU GEMM's epilogue)
        "overlap_average": ("byte", S * (BT * n_feat * 4 + B * rows * T * 2 * 4), S),
    }
    return w


# entries that restate others' work (the SIMT band split; FF1 under its GEGLU launch name; FF1 and
# FF2 together in the fused feed-forward launch)
_ALIASES = ("band_split", "gemm_ff1_geglu", "gemm_ff_fused")


def total_flops(cfg, widths, B: int, T: int) -> int:
    """FLOPs of one forward: every contraction of the method."""
    return sum(v for name, (k, v, _) in kernel_work(cfg, widths, B, T).items()
               if k == "flop" and name not in _ALIASES)


def attention_flops(cfg, widths, B, T):
    w = kernel_work(cfg, widths, B, T)
    return w["attn_time_tc"][1] + w["attn_band_tc"][1]


def audio_seconds(cfg, B: int, T: int) -> float:
    """Seconds of audio in B windows of T frames: B * T * hop / sample_rate."""
    return B * T * cfg.hop / cfg.sample_rate
