"""The epilogues' tanh and sigmoid (axial_band_split_b200/csrc/tc_math.cuh, tanh_mufu and
sigmoid_mufu), checked on the CPU.

The kernels evaluate tanh y = 1 - 2 / (1 + e^(2y)) and sigmoid x = 1 / (1 + e^-x), with
e^u = 2^(u log2 e) on the MUFU (ex2.approx, relative error about 2^-22) and rcp.approx
(about 2^-23).  This test reads the two constants from the source, checks them against
2 log2(e) and -log2(e), and emulates the float32 evaluation order with each approximate step
perturbed by its worst relative error in both directions: the absolute error must stay below
2e-6 everywhere, including the saturated limits.  The mask MLP's tanh and the gates' and GLU's
sigmoid are those of "Mel-Band RoFormer — architecture, inference hot path & RTX 3050
feasibility", section "Parameter accounting" (Linear-Tanh mask MLP, GLU) and section "The two
transformers are not the same shape" (sigmoid gates)."""
import math
import os
import re

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = open(os.path.join(ROOT, "axial_band_split_b200", "csrc", "tc_math.cuh")).read()
f32 = np.float32


def const(name):
    return float(re.search(rf"constexpr float {name} = ([-+0-9.e]+)f;", SRC).group(1))


def test_constants():
    assert f32(const("kTwoLog2e")) == f32(2.0 / math.log(2.0))
    assert f32(const("kNegLog2e")) == f32(-1.0 / math.log(2.0))


def emulate(x, scale, form, de, dr):
    u = (x * f32(scale)).astype(f32)
    with np.errstate(over="ignore"):
        e = (np.exp2(u.astype(np.float64)) * (1 + de)).astype(f32)
    d = (f32(1) + e).astype(f32)
    with np.errstate(divide="ignore"):
        r = ((1.0 / d.astype(np.float64)) * (1 + dr)).astype(f32)
    if form == "tanh":
        return (f32(-2) * r + f32(1)).astype(np.float64)
    return r.astype(np.float64)


def test_tanh_and_sigmoid_error_bound():
    x = np.concatenate([np.linspace(-60, 60, 600001), [0.0, -0.0, 1e-30, -1e-30, 88.0, -88.0, 1e4, -1e4]]).astype(f32)
    xd = x.astype(np.float64)
    want_t = np.tanh(xd)
    want_s = 1.0 / (1.0 + np.exp(-np.clip(xd, -700, 700)))
    for de in (-2.0 ** -22, 0.0, 2.0 ** -22):
        for dr in (-2.0 ** -23, 0.0, 2.0 ** -23):
            t = emulate(x, const("kTwoLog2e"), "tanh", de, dr)
            s = emulate(x, const("kNegLog2e"), "sigmoid", de, dr)
            assert np.abs(t - want_t).max() < 2e-6
            assert np.abs(s - want_s).max() < 2e-6
    t = emulate(x, const("kTwoLog2e"), "tanh", 0.0, 0.0)
    s = emulate(x, const("kNegLog2e"), "sigmoid", 0.0, 0.0)
    assert t[x == 1e4][0] == 1.0 and t[x == -1e4][0] == -1.0
    assert s[x == 1e4][0] == 1.0 and s[x == -1e4][0] == 0.0
    assert np.all(np.diff(t[:600001]) >= 0)  # monotone on the grid
