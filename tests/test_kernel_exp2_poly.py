"""The attention softmax's polynomial exponential (axial_band_split_b200/csrc/k_attn_tc.cu,
exp2_poly2), checked on the CPU.

Part of the softmax's exponentials run on the FMA pipe instead of the MUFU: 2^x = 2^n * 2^f with
n = rint(x) (adding and subtracting 1.5 * 2^23 in float32), f = x - n in [-1/2, 1/2], 2^f by a
degree-3 polynomial fitted here (minimax of the relative error, Remez exchange), and n added to
the float's exponent field.  This test refits the polynomial, checks that the kernel's constants
are that fit, and emulates the kernel's float32 evaluation against exp2 over the range the
softmax uses (s - m in [-125, 8]; lower arguments are clamped to -125)."""
import os
import re

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def kernel_coefficients():
    src = open(os.path.join(ROOT, "axial_band_split_b200", "csrc", "k_attn_tc.cu")).read()
    body = src[src.index("float2 exp2_poly2("):]
    body = body[:body.index("\n}\n")]
    pairs = re.findall(r"f2_pack\(([-+0-9.e]+)f, ([-+0-9.e]+)f\)", body)
    vals = [float(a) for a, b in pairs if a == b and float(a) != 12582912.0]
    return vals  # Horner order: c3, c2, c1, c0


def remez_exp2(deg=3, a=-0.5, b=0.5, iters=40):
    """Minimax polynomial of 2^f on [a, b] in relative error (coefficients c0..c_deg)."""
    n = deg + 2
    x = 0.5 * (a + b) + 0.5 * (b - a) * np.cos(np.pi * np.arange(n)[::-1] / (n - 1))
    grid = np.linspace(a, b, 20001)
    for _ in range(iters):
        A = np.stack([x ** i for i in range(deg + 1)] + [((-1.0) ** np.arange(n)) * 2.0 ** x], axis=1)
        c = np.linalg.solve(A, 2.0 ** x)[:-1]
        err = np.polyval(c[::-1], grid) / 2.0 ** grid - 1.0
        ext = np.where(np.sign(np.diff(err)[1:]) != np.sign(np.diff(err)[:-1]))[0] + 1
        pts = [0] + list(ext) + [len(grid) - 1]
        sel = [pts[0]]
        for p in pts[1:]:
            if np.sign(err[p]) == np.sign(err[sel[-1]]):
                if abs(err[p]) > abs(err[sel[-1]]):
                    sel[-1] = p
            else:
                sel.append(p)
        while len(sel) > n:
            sel.pop(0 if abs(err[sel[0]]) < abs(err[sel[-1]]) else -1)
        if len(sel) == n:
            x = grid[sel]
    return c, float(np.abs(err).max())


def test_constants_are_the_minimax_fit():
    got = kernel_coefficients()
    assert len(got) == 4
    c, e = remez_exp2()
    assert e < 8e-5
    for g, w in zip(got, [c[3], c[2], c[1], c[0]]):
        assert abs(g - w) < 1e-6 * max(1.0, abs(w)), (g, w)


def test_kernel_evaluation_is_within_the_bound():
    c3, c2, c1, c0 = [np.float32(v) for v in kernel_coefficients()]
    f32 = np.float32
    x = np.concatenate([np.linspace(-125, 8, 1330001), [0.0, -0.5, 0.5, -124.99, 7.9999]]).astype(f32)
    xc = np.maximum(x, f32(-125))
    t = (xc + f32(12582912.0)).astype(f32)
    n = (t - f32(12582912.0)).astype(f32)
    fr = (xc - n).astype(f32)
    p = (fr * c3 + c2).astype(f32)
    p = (fr * p + c1).astype(f32)
    p = (fr * p + c0).astype(f32)
    bits = (p.view(np.uint32).astype(np.uint64) + (t.view(np.uint32).astype(np.uint64) << 23)) & 0xFFFFFFFF
    got = bits.astype(np.uint32).view(np.float32).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(got - ref) / ref
    assert rel.max() < 1e-4, rel.max()
    # far below the clamp the result is 2^-125 at most: zero once rounded to fp16
    assert got[0] <= 2.0 ** -124
