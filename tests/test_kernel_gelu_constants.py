"""The FF1 epilogue's GELU constants, checked on the CPU.

The kernel (axial_band_split_b200/csrc/tc_math.cuh, gelu2) evaluates
GELU(y) = max(y, 0) - |y| erfc(|y| / sqrt 2) / 2 with erfc from Abramowitz & Stegun 7.1.28,
erfc(z) = (1 + a1 z + ... + a6 z^6)^-16, the polynomial taken in w = -|y| with 1/sqrt 2, the
sign of w^k and a factor 2^(1/16) folded into its coefficients.  The GPU parity tests bound the
whole forward at fp16 tolerance, which a slightly wrong coefficient could pass; this test
recomputes the folded coefficients from the published a_k, and emulates the kernel's float32
evaluation order against math.erf.  The GELU of the pages is the exact (erf) one: "Mel-Band
RoFormer — architecture, inference hot path & RTX 3050 feasibility", section "The two
transformers are not the same shape"."""
import math
import os
import re

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
# Abramowitz & Stegun 7.1.28
AS_7_1_28 = [1.0, 0.0705230784, 0.0422820123, 0.0092705272, 0.0001520143, 0.0002765672, 0.0000430638]


def kernel_coefficients():
    src = open(os.path.join(ROOT, "axial_band_split_b200", "csrc", "tc_math.cuh")).read()
    body = src[src.index("float2 gelu2("):]
    body = body[:body.index("\n}\n")]
    pairs = re.findall(r"make_float2\(([-+0-9.e]+)f, ([-+0-9.e]+)f\)", body)
    vals = [float(a) for a, b in pairs if a == b]
    # Horner order in the source: the degree-6 and degree-5 coefficients first, then 4 .. 0
    return vals[:7]


def test_folded_coefficients_match_the_published_ones():
    got = kernel_coefficients()
    assert len(got) == 7
    want = [2.0 ** (1 / 16) * AS_7_1_28[k] * 2.0 ** (-k / 2) * (-1) ** k for k in range(7)]
    horner = [want[6], want[5], want[4], want[3], want[2], want[1], want[0]]
    for g, w in zip(got, horner):
        assert np.float32(g) == np.float32(w), (g, w)


def test_kernel_evaluation_order_is_within_the_bound():
    c = [np.float32(v) for v in kernel_coefficients()]
    f32 = np.float32
    y = np.concatenate([np.linspace(-12, 12, 240001), [0.0, -0.0, 1e-30, -1e-30, 40.0, -40.0]]).astype(f32)
    w = (-np.abs(y)).astype(f32)
    q = (w * c[0] + c[1]).astype(f32)
    for k in range(2, 7):
        q = (w * q + c[k]).astype(f32)
    with np.errstate(over="ignore"):
        for _ in range(4):
            q = (q * q).astype(f32)
        e = (f32(1) / q).astype(f32)
    got = (w * e + np.maximum(y, f32(0))).astype(np.float64)
    ref = np.array([0.5 * float(v) * (1.0 + math.erf(float(v) / math.sqrt(2.0))) for v in y])
    # 7.1.28's |erfc error| <= 3e-7 times |y| / 2, plus float32 rounding of the terms
    assert np.abs(got - ref).max() < 1e-6
    assert got[np.argmin(np.abs(y - 40.0))] == 40.0 and got[np.argmin(np.abs(y + 40.0))] == 0.0
