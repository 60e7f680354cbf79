"""Pins of the oracle's forward pass against what the pages and the mathematics fix."""
import cmath
import dataclasses
import math

import numpy as np
import pytest

import synth
from conftest import read_golden
from oracle import model, tables


def golden(name):
    d = dict(l.split() for l in read_golden("published_counts.txt"))
    return float(d[name])


def widths60():
    return tables.band_tables(44100, 2048, 60)["widths"]


# ---------------------------------------------------------------- module wiring
def test_param_counts_match_pages():
    w = widths60()
    assert model.param_count(synth.VOCALS, w) == golden("params_vocals")
    assert model.param_count(synth.DEUX, w) == golden("params_deux")
    # the deux mask head alone
    no_head = model.param_count(dataclasses.replace(synth.DEUX, num_stems=0), w)
    assert model.param_count(synth.DEUX, w) - no_head == golden("params_deux_mask_head")
    # the vocals trunk (both axes, all blocks): 23.7 M
    base = dataclasses.replace(synth.VOCALS, depth=0)
    trunk = model.param_count(synth.VOCALS, w) - model.param_count(base, w)
    assert round(trunk / 1e6, 1) == golden("trunk_params_vocals_millions")


def test_weight_table_matches_param_count():
    # the generator's named shapes add up to the same count (shapes of [1536,384],
    # [1536,1536], [56,1536], [1040,1536] as the pages print)
    w = widths60()
    shapes = dict(synth.weight_shapes(synth.VOCALS, w))
    assert sum(int(np.prod(s)) for s in shapes.values()) == golden("params_vocals")
    p = "mask_estimators.0.to_freqs."
    assert shapes[p + "0.0.0.weight"] == (1536, 384)
    assert shapes[p + "0.0.2.weight"] == (1536, 1536)
    assert shapes[p + "0.0.4.weight"] == (56, 1536)
    assert shapes[p + "59.0.4.weight"] == (1040, 1536)


def test_mac_accounting_matches_pages():
    m = model.mac_count(synth.VOCALS, widths60(), 1, 801)
    for term in ("qkv", "ff1", "ff2"):
        assert round(m["per_axis"][term] / 1e9, 2) == golden("macs_per_term_G")
    assert round(m["trunk"] / 1e9, 1) == golden("macs_trunk_G")
    assert round(m["attn_time"] / 1e9, 2) == golden("macs_attn_time_G")
    assert round(m["attn_band"] / 1e9, 2) == golden("macs_attn_band_G")
    D, A = 384, 512
    assert 2 * 60 * A == golden("macs_band_attn_per_token")
    assert D * 4 * D == golden("macs_ffn_projection_per_token")
    # 3.102 TFLOP per chunk: the page's total stands within 0.5 % of the term sum
    assert 2 * m["total"] / 1e12 == pytest.approx(golden("tflop_per_chunk"), rel=5e-3)


def test_frames_of_8s_chunk():
    spec = synth.stft_stereo(np.zeros((2, 352800)), 2048, 441)
    assert spec.shape == (2, 1025, int(golden("frames_8s")))


# ---------------------------------------------------------------- RMSNorm
def test_rmsnorm_properties():
    rng = np.random.default_rng(0)
    x = rng.standard_normal((5, 37))
    g = np.ones(37)
    y = model.rms_norm(x, g)
    assert np.allclose(np.linalg.norm(y, axis=1), math.sqrt(37))      # ||N(x)|| = sqrt(d)
    assert np.allclose(model.rms_norm(3.7 * x, g), y)                   # scale invariant
    assert not np.allclose(model.rms_norm(x + 1.0, g), y)               # not mean invariant
    z = model.rms_norm(np.zeros((2, 8)), np.ones(8))
    assert np.all(z == 0)                                               # zero row -> 0
    gam = rng.standard_normal(37)
    assert np.allclose(model.rms_norm(x, gam), y * gam)


def test_gelu_erf_values():
    # GELU(x) = x * Phi(x); Phi(1) = 0.841344746068542948..., Phi(2) = 0.977249868051820...
    assert model.gelu(np.array(1.0)) == pytest.approx(0.8413447460685429, abs=1e-15)
    assert model.gelu(np.array(-1.0)) == pytest.approx(-0.15865525393145707, abs=1e-15)
    assert model.gelu(np.array(2.0)) == pytest.approx(2 * 0.9772498680518208, abs=1e-14)
    assert model.gelu(np.array(0.0)) == 0.0


# ---------------------------------------------------------------- rotary embedding
def test_rope_equals_complex_rotation():
    # pair (x_2i, x_2i+1) as the complex number x_2i + i x_2i+1, multiplied by e^{i p theta^(-2i/d)}
    rng = np.random.default_rng(1)
    n, dh, theta = 7, 8, 10000.0
    x = rng.standard_normal((n, dh))
    y = model.rope(x, theta)
    for p in range(n):
        for i in range(dh // 2):
            z = complex(x[p, 2 * i], x[p, 2 * i + 1]) * cmath.exp(1j * p * theta ** (-2 * i / dh))
            assert y[p, 2 * i] == pytest.approx(z.real, abs=1e-12)
            assert y[p, 2 * i + 1] == pytest.approx(z.imag, abs=1e-12)


def test_rope_norm_and_relative_position():
    rng = np.random.default_rng(2)
    n, dh = 12, 16
    q = rng.standard_normal((n, dh))
    k = rng.standard_normal((n, dh))
    rq = model.rope(q, 10000.0)
    assert np.allclose(np.linalg.norm(rq.reshape(n, -1, 2), axis=-1),
                       np.linalg.norm(q.reshape(n, -1, 2), axis=-1))      # per pair norm kept
    assert np.allclose(rq[0], q[0])                                       # position 0 is identity
    # <R_m q, R_n k> depends on m - n only: same vectors placed at (m, n) and (m+s, n+s)
    qv, kv = q[0], k[0]
    def at(vec, p):
        tmp = np.zeros((p + 1, dh)); tmp[p] = vec
        return model.rope(tmp, 10000.0)[p]
    a = at(qv, 3) @ at(kv, 1)
    b = at(qv, 9) @ at(kv, 7)
    assert a == pytest.approx(b, abs=1e-12)
    # interleaved pairs to halves is one permutation of q's and k's features: q.k unchanged
    perm = np.concatenate([np.arange(0, dh, 2), np.arange(1, dh, 2)])
    rk = model.rope(k, 10000.0)
    assert np.allclose(rq[:, perm] @ rk[:, perm].T, rq @ rk.T)


# ---------------------------------------------------------------- attention
def brute_attend(q, k, v):
    n, dh = len(q), len(q[0])
    out = []
    for i in range(n):
        s = [sum(q[i][d] * k[j][d] for d in range(dh)) / math.sqrt(dh) for j in range(n)]
        m = max(s)
        e = [math.exp(x - m) for x in s]
        z = sum(e)
        out.append([sum(e[j] / z * v[j][d] for j in range(n)) for d in range(len(v[0]))])
    return np.array(out)


def test_attend_brute_force_and_properties():
    rng = np.random.default_rng(3)
    q, k, v = (rng.standard_normal((6, 4)) for _ in range(3))
    assert np.allclose(model.attend(q, k, v), brute_attend(q.tolist(), k.tolist(), v.tolist()), atol=1e-13)
    s = model.softmax(rng.standard_normal((5, 9)) * 30)
    assert np.allclose(s.sum(-1), 1.0)
    # n = 1: output is v
    assert np.allclose(model.attend(q[:1], k[:1], v[:1]), v[:1])
    # splitting the queries is exact
    full = model.attend(q, k, v)
    assert np.allclose(np.concatenate([model.attend(q[:2], k, v), model.attend(q[2:], k, v)]), full)


def brute_attention_layer(x, w, h, dh, theta):
    """Scalar loops over the definition: pre-norm, qkv features (which, head, d), RoPE on
    q and k, softmax attention per head, sigmoid gate per head from the normed input,
    heads concatenated head-major, output projection."""
    n, D = x.shape
    g = w["norm.gamma"]
    a = []
    for t in range(n):
        nrm = math.sqrt(sum(x[t, j] ** 2 for j in range(D)))
        a.append([x[t, j] / max(nrm, 1e-12) * math.sqrt(D) * g[j] for j in range(D)])
    Wq = w["to_qkv.weight"]
    def proj(which, head, t):
        return [sum(Wq[(which * h + head) * dh + d, j] * a[t][j] for j in range(D)) for d in range(dh)]
    def rot(vec, p):
        out = list(vec)
        for i in range(dh // 2):
            z = complex(vec[2 * i], vec[2 * i + 1]) * cmath.exp(1j * p * theta ** (-2 * i / dh))
            out[2 * i], out[2 * i + 1] = z.real, z.imag
        return out
    cat = [[0.0] * (h * dh) for _ in range(n)]
    for head in range(h):
        q = [rot(proj(0, head, t), t) for t in range(n)]
        k = [rot(proj(1, head, t), t) for t in range(n)]
        v = [proj(2, head, t) for t in range(n)]
        o = brute_attend(q, k, v)
        for t in range(n):
            gate = sum(w["to_gates.weight"][head, j] * a[t][j] for j in range(D)) + w["to_gates.bias"][head]
            sg = 1 / (1 + math.exp(-gate))
            for d in range(dh):
                cat[t][head * dh + d] = o[t][d] * sg
    Wo = w["to_out.0.weight"]
    return np.array([[sum(Wo[i, j] * cat[t][j] for j in range(h * dh)) for i in range(D)] for t in range(n)])


def test_attention_layer_brute_force():
    rng = np.random.default_rng(4)
    n, D, h, dh = 5, 6, 2, 4
    w = {"norm.gamma": 1 + 0.1 * rng.standard_normal(D),
         "to_qkv.weight": rng.standard_normal((3 * h * dh, D)),
         "to_gates.weight": rng.standard_normal((h, D)), "to_gates.bias": rng.standard_normal(h),
         "to_out.0.weight": rng.standard_normal((D, h * dh))}
    x = rng.standard_normal((1, n, D))
    got = model.attention(x, w, h, dh, 10000.0)[0]
    assert np.allclose(got, brute_attention_layer(x[0], w, h, dh, 10000.0), atol=1e-11)


def test_transformer_output_norm():
    rng = np.random.default_rng(5)
    cfg = synth.TINY
    widths = tables.band_tables(44100, 256, 8)["widths"]
    W = synth.make_weights(cfg, widths, seed=0, fp16=False)
    tw = {k[len("layers.0.0."):]: v.astype(np.float64) for k, v in W.items() if k.startswith("layers.0.0.")}
    tw["norm.gamma"] = np.ones(cfg.dim)
    y = model.transformer(rng.standard_normal((3, 5, cfg.dim)), tw, cfg.heads, cfg.dim_head, 10000.0)
    assert np.allclose(np.linalg.norm(y, axis=-1), math.sqrt(cfg.dim))


# ---------------------------------------------------------------- mask head and average
def test_glu_zero_gate_is_half_value():
    cfg = synth.TINY
    tab = tables.band_tables(44100, 256, 8)
    W = {k: v.astype(np.float64) for k, v in synth.make_weights(cfg, tab["widths"], fp16=False).items()}
    for k, d in enumerate(tab["widths"]):
        p = f"mask_estimators.0.to_freqs.{k}.0.4."
        W[p + "weight"][d:] = 0
        W[p + "bias"][d:] = 0
    X = np.random.default_rng(6).standard_normal((4, 8, cfg.dim))
    m = model.mask_estimator(X, tab, W)
    # reference value half: y = W4 tanh(W2 tanh(W0 x + b0) + b2) + b4 with the first d rows
    off = 0
    for k, d in enumerate(tab["widths"]):
        p = f"mask_estimators.0.to_freqs.{k}.0."
        h1 = np.tanh(X[:, k] @ W[p + "0.weight"].T + W[p + "0.bias"])
        assert np.all(np.abs(h1) < 1)
        h2 = np.tanh(h1 @ W[p + "2.weight"].T + W[p + "2.bias"])
        val = h2 @ W[p + "4.weight"][:d].T + W[p + "4.bias"][:d]
        assert np.allclose(m[:, off:off + d], 0.5 * val)
        off += d


def test_overlap_average_partition_of_unity_and_one_hot():
    tab = tables.band_tables(44100, 2048, 60)
    T, R = 3, 2050
    m = np.full((T, int(tab["widths"].sum())), 0.37)
    assert np.allclose(model.overlap_average(m, tab, R), 0.37)
    # one band's features at 1, all else 0: its rows get 1 / (bands over the bin)
    k = 20
    off = np.concatenate([[0], np.cumsum(tab["widths"])])
    m = np.zeros_like(m)
    m[:, off[k]:off[k + 1]] = 1.0
    out = model.overlap_average(m, tab, R)
    for f in range(tab["first_bin"][k], tab["last_bin"][k] + 1):
        assert np.allclose(out[2 * f: 2 * f + 2], 1.0 / tab["bands_per_bin"][f])
    assert out[: 2 * tab["first_bin"][k]].sum() == 0
    assert out[2 * tab["last_bin"][k] + 2:].sum() == 0


# ---------------------------------------------------------------- whole forward
def tiny_case(B=1, T=32, seed=2):
    cfg = synth.TINY
    widths = tables.band_tables(44100, 256, 8)["widths"]
    W = synth.make_weights(cfg, widths, seed=0, fp16=False)
    x = synth.make_stft_repr(cfg, B, T, seed=seed)
    return cfg, W, x


def test_forward_shapes_and_batching():
    cfg, W, x = tiny_case(B=2, T=9)
    out, st = model.forward(x, cfg, W, return_stages=True)
    assert out.shape == (2, 258, 9, 2)
    assert st[0]["band_split"].shape == (9, 8, 64)
    assert st[0]["mask0"].shape == (9, 828)
    for b in range(2):
        assert np.allclose(model.forward(x[b:b + 1], cfg, W)[0], out[b])


def test_time_transformer_keeps_bands_independent():
    # before the band transformer, band k's sequence depends on band k's input only
    cfg, W, x = tiny_case(T=6)
    _, st = model.forward(x, cfg, W, return_stages=True)
    tab = tables.band_tables(44100, 256, 8)
    x2 = x.copy()
    x2[0, : 2 * tab["first_bin"][1]] *= -1.3        # bins below band 1 belong to band 0 only
    _, st2 = model.forward(x2, cfg, W, return_stages=True)
    a, b = st[0]["layer0.time"], st2[0]["layer0.time"]
    assert not np.allclose(a[:, 0], b[:, 0])
    assert np.allclose(a[:, 1:], b[:, 1:])


def test_forward_fp32_close_to_fp64():
    cfg, W, x = tiny_case()
    a = model.forward(x, cfg, W, dtype=np.float64)
    b = model.forward(x, cfg, W, dtype=np.float32)
    assert np.abs(a - b).max() / np.abs(a).max() < 1e-4


def test_apply_masks_unit_and_imaginary_unit():
    # mask 1 passes the mixture through; mask i turns (re, im) into (-im, re)
    rng = np.random.Generator(np.random.PCG64(7))
    x = rng.standard_normal((2, 6, 5, 2))
    one = np.zeros_like(x)
    one[..., 0] = 1.0
    assert np.array_equal(model.apply_masks(x, one), x)
    i = np.zeros_like(x)
    i[..., 1] = 1.0
    y = model.apply_masks(x, i)
    assert np.array_equal(y[..., 0], -x[..., 1]) and np.array_equal(y[..., 1], x[..., 0])


def test_apply_masks_modulus_and_stems_summing_to_one():
    # |m x| = |m| |x| element by element; stems whose masks sum to 1 give back the mixture
    rng = np.random.Generator(np.random.PCG64(8))
    x = rng.standard_normal((1, 4, 3, 2))
    m = rng.standard_normal((1, 2, 4, 3, 2))
    y = model.apply_masks(x, m)
    mod = lambda a: np.hypot(a[..., 0], a[..., 1])
    assert np.allclose(mod(y), mod(m) * mod(x)[:, None], rtol=1e-12, atol=0)
    m[:, 1] = -m[:, 0]
    m[:, 1, ..., 0] += 1.0                                    # m1 = 1 - m0
    y = model.apply_masks(x, m)
    assert np.allclose(y.sum(axis=1), x, rtol=0, atol=1e-12)


def test_stems_share_the_trunk():
    # two stems: the same trunk output under two mask heads; stem 0 equals the one-stem model
    # built from stem 0's weights
    import dataclasses
    cfg, W, x = tiny_case()
    cfg2 = dataclasses.replace(cfg, num_stems=2)
    W2 = synth.make_weights(cfg2, tables.band_tables(44100, 256, 8)["widths"], fp16=False)
    two = model.forward(x, cfg2, W2)
    one = model.forward(x, cfg, {k: v for k, v in W2.items() if not k.startswith("mask_estimators.1.")})
    assert two.shape == (1, 2) + x.shape[1:]
    assert np.array_equal(two[:, 0], one)
    assert not np.allclose(two[:, 1], one)


def test_geglu_with_unit_value_half_is_the_gelu_block():
    # GEGLU(y) = value * GELU(gate): with the value half's weights 0 and biases 1 the block is
    # the GELU block whose first projection is the gate half (a swapped or missing half fails)
    import dataclasses
    cfg, W, x = tiny_case(T=5)
    g = dataclasses.replace(cfg, ff_act=1)
    widths = tables.band_tables(44100, 256, 8)["widths"]
    Wg = synth.make_weights(g, widths, seed=0, fp16=False)
    Wp = dict(Wg)
    FF = cfg.dim * cfg.ff_mult
    for l in range(cfg.depth):
        for a in range(2):
            p = f"layers.{l}.{a}.layers.0.1.net.1."
            w, b = Wg[p + "weight"].copy(), Wg[p + "bias"].copy()
            w[:FF] = 0.0
            b[:FF] = 1.0
            Wg[p + "weight"], Wg[p + "bias"] = w, b
            Wp[p + "weight"], Wp[p + "bias"] = w[FF:], b[FF:]
    assert np.allclose(model.forward(x, g, Wg), model.forward(x, cfg, Wp), rtol=0, atol=1e-12)


def test_geglu_parameter_count():
    # the first projection doubles: 2 * (D * FF + FF) more per transformer
    import dataclasses
    widths = tables.band_tables(44100, 2048, 60)["widths"]
    base = model.param_count(synth.VOCALS, widths)
    g = model.param_count(dataclasses.replace(synth.VOCALS, ff_act=1), widths)
    D, FF = 384, 1536
    assert g - base == 2 * 6 * (D * FF + FF) and g == 235_299_108


# ---------------------------------------------------------------- feed-forward and band split, by scalar loops
def brute_feed_forward(x, w, ff_act=0):
    """Scalar loops over the definition of the feed-forward block ("@audio/neural-separate
    0.4.0 → 0.5.0", package/scripts/export-roformer.py, class FF: norm, Linear with bias, GELU,
    Linear with bias): a = x / max(|x|, 1e-12) * sqrt(D) * gamma; h_i = gelu(W1[i] . a + b1[i])
    with gelu(y) = y (1 + erf(y / sqrt 2)) / 2 (math.erf); out_j = W2[j] . h + b2[j].  The GEGLU
    variant pairs h_i = (W1[i] . a + b1[i]) * gelu(W1[F + i] . a + b1[F + i])."""
    n, D = x.shape
    g, W1, b1, W2, b2 = w["net.0.gamma"], w["net.1.weight"], w["net.1.bias"], w["net.4.weight"], w["net.4.bias"]
    F = W2.shape[1]
    gelu = lambda y: 0.5 * y * (1.0 + math.erf(y / math.sqrt(2.0)))
    out = np.zeros((n, D))
    for t in range(n):
        nrm = math.sqrt(sum(x[t, j] ** 2 for j in range(D)))
        a = [x[t, j] / max(nrm, 1e-12) * math.sqrt(D) * g[j] for j in range(D)]
        y = [sum(W1[i, j] * a[j] for j in range(D)) + b1[i] for i in range(W1.shape[0])]
        h = [y[i] * gelu(y[F + i]) for i in range(F)] if ff_act == 1 else [gelu(y[i]) for i in range(F)]
        for o in range(D):
            out[t, o] = sum(W2[o, i] * h[i] for i in range(F)) + b2[o]
    return out


def _ff_weights(rng, D, F, ff_act=0):
    F1 = 2 * F if ff_act == 1 else F
    return {"net.0.gamma": 1 + 0.2 * rng.standard_normal(D), "net.1.weight": rng.standard_normal((F1, D)) / 2,
            "net.1.bias": rng.standard_normal(F1), "net.4.weight": rng.standard_normal((D, F)) / 3,
            "net.4.bias": rng.standard_normal(D)}


@pytest.mark.parametrize("ff_act", [0, 1])
def test_feed_forward_brute_force(ff_act):
    rng = np.random.default_rng(11 + ff_act)
    D, F = 6, 10
    w = _ff_weights(rng, D, F, ff_act)
    x = rng.standard_normal((5, D)) * 3
    assert np.allclose(model.feed_forward(x, w, ff_act), brute_feed_forward(x, w, ff_act), rtol=0, atol=1e-11)


def test_feed_forward_brute_force_catches_slips():
    # each plausible slip changes the result by far more than the 1e-11 of the test above
    rng = np.random.default_rng(13)
    D, F = 6, 10
    w = _ff_weights(rng, D, F)
    x = rng.standard_normal((5, D)) * 3
    ref = brute_feed_forward(x, w)
    for key in ("net.1.bias", "net.4.bias"):          # a dropped bias
        w2 = dict(w)
        w2[key] = np.zeros_like(w[key])
        assert np.abs(model.feed_forward(x, w2) - ref).max() > 1e-3
    w2 = dict(w)
    w2["net.0.gamma"] = w["net.0.gamma"] / math.sqrt(D)    # the norm's sqrt(D) left out
    assert np.abs(model.feed_forward(x, w2) - ref).max() > 1e-3
    # GELU after the second projection instead of the first, and no pre-norm at all
    a = model.rms_norm(x, w["net.0.gamma"])
    late = model.gelu((a @ w["net.1.weight"].T + w["net.1.bias"]) @ w["net.4.weight"].T + w["net.4.bias"])
    assert np.abs(late - ref).max() > 1e-3
    raw = model.gelu(x @ w["net.1.weight"].T + w["net.1.bias"]) @ w["net.4.weight"].T + w["net.4.bias"]
    assert np.abs(raw - ref).max() > 1e-3


def brute_transformer(x, w, h, dh, theta):
    """One transformer by scalar loops: x += attention(x); x += ff(x); x = norm_out(x)."""
    aw = {k[len("layers.0.0."):]: v for k, v in w.items() if k.startswith("layers.0.0.")}
    fw = {k[len("layers.0.1."):]: v for k, v in w.items() if k.startswith("layers.0.1.")}
    x = x + brute_attention_layer(x, aw, h, dh, theta)
    x = x + brute_feed_forward(x, fw)
    n, D = x.shape
    out = np.zeros_like(x)
    for t in range(n):
        nrm = math.sqrt(sum(x[t, j] ** 2 for j in range(D)))
        for j in range(D):
            out[t, j] = x[t, j] / max(nrm, 1e-12) * math.sqrt(D) * w["norm.gamma"][j]
    return out


def test_transformer_brute_force():
    rng = np.random.default_rng(14)
    n, D, h, dh, F = 4, 6, 2, 4, 8
    w = {"layers.0.0.norm.gamma": 1 + 0.1 * rng.standard_normal(D),
         "layers.0.0.to_qkv.weight": rng.standard_normal((3 * h * dh, D)) / 2,
         "layers.0.0.to_gates.weight": rng.standard_normal((h, D)),
         "layers.0.0.to_gates.bias": rng.standard_normal(h),
         "layers.0.0.to_out.0.weight": rng.standard_normal((D, h * dh)) / 2,
         "norm.gamma": 1 + 0.1 * rng.standard_normal(D)}
    w.update({"layers.0.1." + k: v for k, v in _ff_weights(rng, D, F).items()})
    x = rng.standard_normal((2, n, D))
    got = model.transformer(x, w, h, dh, 10000.0)
    for s in range(2):
        assert np.allclose(got[s], brute_transformer(x[s], w, h, dh, 10000.0), rtol=0, atol=1e-10)


def brute_band_split(spec, first_bin, last_bin, channels, weights):
    """BandSplit by scalar loops ("Mel-Band RoFormer — architecture, inference hot path & RTX 3050
    feasibility", section "The mel-band split, exactly"): band k's features at frame t are, for
    each bin f = first..last of the band in ascending order, each channel s and each complex part
    c, spec[f * C + s, t, c] (feature (j * C + s) * 2 + c for the j-th bin); then
    x / max(|x|, 1e-12) * sqrt(d_in) * gamma and Linear(d_in, D) with bias."""
    R, T, _ = spec.shape
    nb = len(first_bin)
    D = weights["band_split.to_features.0.1.bias"].shape[0]
    out = np.zeros((T, nb, D))
    for k in range(nb):
        p = f"band_split.to_features.{k}."
        g, W, b = weights[p + "0.gamma"], weights[p + "1.weight"], weights[p + "1.bias"]
        for t in range(T):
            feats = []
            for f in range(first_bin[k], last_bin[k] + 1):
                for s in range(channels):
                    for c in range(2):
                        feats.append(spec[f * channels + s, t, c])
            d = len(feats)
            nrm = math.sqrt(sum(v * v for v in feats))
            a = [feats[e] / max(nrm, 1e-12) * math.sqrt(d) * g[e] for e in range(d)]
            for o in range(D):
                out[t, k, o] = sum(W[o, e] * a[e] for e in range(d)) + b[o]
    return out


def test_band_split_brute_force():
    rng = np.random.default_rng(15)
    tab = tables.band_tables(44100, 256, 8)
    D = 5
    widths = tab["widths"]
    W = {}
    for k, d in enumerate(widths):
        p = f"band_split.to_features.{k}."
        W[p + "0.gamma"] = 1 + 0.2 * rng.standard_normal(d)
        W[p + "1.weight"] = rng.standard_normal((D, d))
        W[p + "1.bias"] = rng.standard_normal(D)
    spec = rng.standard_normal((258, 3, 2))
    spec[:, 2] = 0.0                                       # a silent frame: every band's norm clamps
    ref = brute_band_split(spec, tab["first_bin"], tab["last_bin"], 2, W)
    got = model.band_split(spec, tab, W)
    assert np.allclose(got, ref, rtol=0, atol=1e-11)
    # the silent frame gives exactly the biases (x / max(0, eps) = 0)
    for k in range(8):
        assert np.array_equal(got[2, k], W[f"band_split.to_features.{k}.1.bias"])


# ---------------------------------------------------------------- v narrower than q and k
def brute_attention_layer_wide_qk(x, w, h, dh, dv, theta):
    """Scalar loops for the attention whose q and k (dh per head) are wider than v (dv per head)
    ("evaluation.md", section "BS PolarFormer: the same quality for a quarter of the
    arithmetic"): projection features q (head, d < dh), then k (head, d < dh), then v (head, d <
    dv); softmax scale dh^-1/2; heads concatenated head-major (h * dv wide)."""
    n, D = x.shape
    g = w["norm.gamma"]
    a = []
    for t in range(n):
        nrm = math.sqrt(sum(x[t, j] ** 2 for j in range(D)))
        a.append([x[t, j] / max(nrm, 1e-12) * math.sqrt(D) * g[j] for j in range(D)])
    Wq = w["to_qkv.weight"]
    def feat(row, t):
        return sum(Wq[row, j] * a[t][j] for j in range(D))
    def rot(vec, p):
        out = list(vec)
        for i in range(len(vec) // 2):
            z = complex(vec[2 * i], vec[2 * i + 1]) * cmath.exp(1j * p * theta ** (-2 * i / len(vec)))
            out[2 * i], out[2 * i + 1] = z.real, z.imag
        return out
    cat = [[0.0] * (h * dv) for _ in range(n)]
    for head in range(h):
        q = [rot([feat(head * dh + d, t) for d in range(dh)], t) for t in range(n)]
        k = [rot([feat(h * dh + head * dh + d, t) for d in range(dh)], t) for t in range(n)]
        v = [[feat(2 * h * dh + head * dv + d, t) for d in range(dv)] for t in range(n)]
        o = brute_attend(q, k, v)
        for t in range(n):
            gate = sum(w["to_gates.weight"][head, j] * a[t][j] for j in range(D)) + w["to_gates.bias"][head]
            sg = 1 / (1 + math.exp(-gate))
            for d in range(dv):
                cat[t][head * dv + d] = o[t][d] * sg
    Wo = w["to_out.0.weight"]
    return np.array([[sum(Wo[i, j] * cat[t][j] for j in range(h * dv)) for i in range(D)] for t in range(n)])


def test_attention_layer_wide_qk_brute_force():
    rng = np.random.default_rng(16)
    n, D, h, dh, dv = 5, 6, 2, 8, 4
    w = {"norm.gamma": 1 + 0.1 * rng.standard_normal(D),
         "to_qkv.weight": rng.standard_normal((h * (2 * dh + dv), D)) / 2,
         "to_gates.weight": rng.standard_normal((h, D)), "to_gates.bias": rng.standard_normal(h),
         "to_out.0.weight": rng.standard_normal((D, h * dv))}
    x = rng.standard_normal((1, n, D))
    got = model.attention(x, w, h, dh, 10000.0, dim_head_v=dv)[0]
    assert np.allclose(got, brute_attention_layer_wide_qk(x[0], w, h, dh, dv, 10000.0), rtol=0, atol=1e-11)
    # with dv = dh the general layout is the (which, head, d) layout of the equal-width layer
    w2 = dict(w, **{"to_qkv.weight": rng.standard_normal((3 * h * dh, D)) / 2,
                    "to_out.0.weight": rng.standard_normal((D, h * dh))})
    assert np.allclose(model.attention(x, w2, h, dh, 10000.0, dim_head_v=dh),
                       model.attention(x, w2, h, dh, 10000.0), rtol=0, atol=0)


def test_wide_qk_parameter_and_mac_counts():
    # to_qkv is h (2 dh + dv) x D and to_out D x h dv; attention MACs per score are dh + dv
    import dataclasses
    w = widths60()
    base = dataclasses.replace(synth.WIDE_QK, dim_head_v=0, dim_head=64)
    D, H = 256, 8
    extra_qkv = H * (2 * 128 + 64) * D - 3 * H * 64 * D
    assert model.param_count(synth.WIDE_QK, w) - model.param_count(base, w) == 2 * (extra_qkv)
    m = model.mac_count(synth.WIDE_QK, w, 1, 100)
    assert m["attn_time"] == 1 * (60 * H) * 100 * 100 * (128 + 64)
    assert m["per_axis"]["qkv"] == 1 * 100 * 60 * D * H * (2 * 128 + 64)
