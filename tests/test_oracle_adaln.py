"""Pins for AdaLN modulation and the gated residual fused with it."""
from decimal import Decimal, getcontext
from fractions import Fraction

import numpy as np
import pytest
import torch

from conftest import closed_form, load_golden


def _bf16(orc, a):
    return orc.f64_to_bf16(np.asarray(a, dtype=np.float64))


def test_golden_d4(orc):
    g = load_golden("adaln_d4.json")
    x = _bf16(orc, [g["x"]]).reshape(1, 1, 4)
    y = orc.adaln_modulate(x, np.array([g["shift"]]), np.array([g["scale"]]), g["eps"])
    want = np.array([closed_form(e) for e in g["y"]])
    assert np.allclose(y.reshape(4), want, rtol=0, atol=1e-15)
    x2 = _bf16(orc, [g["x2"]]).reshape(1, 1, 4)
    y2 = orc.adaln_modulate(x2, np.zeros((1, 4)), np.zeros((1, 4)), g["eps2"])
    want2 = np.array([closed_form(e) for e in g["y2"]])
    assert np.allclose(y2.reshape(4), want2, rtol=0, atol=1e-14)


def _rand_bits(orc, shape, seed, scale=1.0, loc=0.0):
    rng = np.random.default_rng(seed)
    return _bf16(orc, rng.standard_normal(shape) * scale + loc)


def test_zero_modulation_is_library_layer_norm(orc):
    B, N, D, eps = 2, 7, 96, 1e-6
    x = _rand_bits(orc, (B, N, D), 3, scale=2.0, loc=0.5)
    y = orc.adaln_modulate(x, np.zeros((B, D)), np.zeros((B, D)), eps)
    ref = torch.nn.functional.layer_norm(torch.from_numpy(orc.bf16_to_f64(x)), (D,), eps=eps)
    assert np.allclose(y, ref.numpy(), rtol=0, atol=1e-13)


def test_normalised_row_moments(orc):
    """Before modulation: mean 0 and variance var/(var+eps) per row."""
    N, D, eps = 16, 256, 0.3
    x = _rand_bits(orc, (1, N, D), 4, scale=0.7, loc=-1.0)
    y = orc.adaln_modulate(x, np.zeros((1, D)), np.zeros((1, D)), eps)[0]
    xf = orc.bf16_to_f64(x)[0]
    var = xf.var(axis=1)
    assert np.allclose(y.mean(axis=1), 0.0, atol=1e-14)
    assert np.allclose(y.var(axis=1), var / (var + eps), rtol=1e-12, atol=0)


def test_scale_minus_one_gives_shift(orc):
    B, N, D = 2, 5, 40
    x = _rand_bits(orc, (B, N, D), 5)
    rng = np.random.default_rng(6)
    shift = rng.standard_normal((B, D))
    y = orc.adaln_modulate(x, shift, -np.ones((B, D)), 1e-6)
    assert np.array_equal(y, np.broadcast_to(shift[:, None, :], y.shape))


def test_shift_and_positive_scale_invariance(orc):
    """LN(a*x + b) == LN(x) for a > 0 when eps = 0 (integer rows stay exact)."""
    rng = np.random.default_rng(7)
    xi = rng.integers(-20, 20, (1, 6, 32)).astype(np.float64)
    xi[..., 0] = 25.0  # no constant rows
    a = _bf16(orc, xi)
    b = _bf16(orc, 4.0 * xi + 64.0)
    z = np.zeros((1, 32))
    ya = orc.adaln_modulate(a, z, z, 0.0)
    yb = orc.adaln_modulate(b, z, z, 0.0)
    assert np.allclose(ya, yb, rtol=0, atol=1e-14)


def test_batch_uses_its_own_modulation(orc):
    B, N, D = 3, 4, 24
    x = _rand_bits(orc, (B, N, D), 8)
    rng = np.random.default_rng(9)
    sh, sc = rng.standard_normal((B, D)), rng.standard_normal((B, D))
    y = orc.adaln_modulate(x, sh, sc, 1e-6)
    for b in range(B):
        yb = orc.adaln_modulate(x[b:b + 1], sh[b:b + 1], sc[b:b + 1], 1e-6)
        assert np.array_equal(y[b:b + 1], yb)


def _exact_adaln(xrow, shift, scale, eps):
    getcontext().prec = 60
    xs = [Fraction(v) for v in xrow]
    D = len(xs)
    mu = sum(xs) / D
    var = sum((v - mu) ** 2 for v in xs) / D
    den = (Decimal(var.numerator) / Decimal(var.denominator) + Decimal(Fraction(eps).numerator)
           / Decimal(Fraction(eps).denominator)).sqrt()
    out = []
    for v, s, c in zip(xs, shift, scale):
        d = v - mu
        n = (Decimal(d.numerator) / Decimal(d.denominator)) / den
        out.append(float(n * (1 + Decimal(c)) + Decimal(s)))
    return out


def test_exact_arithmetic_brute_force(orc):
    """Tiny rows against exact rationals with a 60-digit square root."""
    rng = np.random.default_rng(10)
    for D in (2, 3, 5, 8, 13):
        x = _rand_bits(orc, (1, 1, D), 100 + D, scale=3.0, loc=1000.0)
        sh = rng.standard_normal((1, D))
        sc = rng.standard_normal((1, D))
        y = orc.adaln_modulate(x, sh, sc, 1e-3)[0, 0]
        want = _exact_adaln(orc.bf16_to_f64(x)[0, 0], sh[0], sc[0], 1e-3)
        assert np.allclose(y, want, rtol=1e-12, atol=1e-12)


# ------------------------------------------------------- gated residual


def test_gated_golden(orc):
    g = load_golden("gated_residual_d4.json")
    x = _bf16(orc, g["x"]).reshape(2, 1, 4)
    r = _bf16(orc, g["r"]).reshape(2, 1, 4)
    gate = np.array([g["gate_row1"], g["gate_row2"]])
    z = np.zeros((2, 4))
    x_out, y = orc.gated_residual_adaln(x, r, gate, z, z, g["eps"])
    xo = orc.bf16_to_f64(x_out)
    assert np.array_equal(xo[0, 0], [closed_form(e) for e in g["x_out_row1"]])
    assert np.array_equal(xo[1, 0], [closed_form(e) for e in g["x_out_row2"]])
    assert np.allclose(y[0, 0], [closed_form(e) for e in g["y_row1"]], rtol=0, atol=1e-14)


def test_gated_zero_gate_or_zero_branch_is_adaln(orc):
    B, N, D, eps = 2, 6, 64, 1e-6
    x = _rand_bits(orc, (B, N, D), 11)
    r = _rand_bits(orc, (B, N, D), 12)
    rng = np.random.default_rng(13)
    sh, sc, gt = (rng.standard_normal((B, D)) * 0.1 for _ in range(3))
    ref = orc.adaln_modulate(x, sh, sc, eps)
    x0, y0 = orc.gated_residual_adaln(x, r, np.zeros((B, D)), sh, sc, eps)
    assert np.array_equal(x0, x) and np.array_equal(y0, ref)
    x1, y1 = orc.gated_residual_adaln(x, np.zeros_like(r), gt, sh, sc, eps)
    assert np.array_equal(x1, x) and np.array_equal(y1, ref)


def test_gated_residual_is_nearest_bf16_of_exact_sum(orc):
    B, N, D = 1, 8, 48
    x = _rand_bits(orc, (B, N, D), 14)
    r = _rand_bits(orc, (B, N, D), 15)
    gate = np.random.default_rng(16).standard_normal((B, D)).astype(np.float32).astype(np.float64)
    z = np.zeros((B, D))
    x_out, _ = orc.gated_residual_adaln(x, r, gate, z, z, 1e-6)
    xf, rf = orc.bf16_to_f64(x), orc.bf16_to_f64(r)
    got = orc.bf16_to_f64(x_out)
    up = orc.bf16_to_f64((x_out.astype(np.int64) + 1).astype(np.uint16))
    dn = orc.bf16_to_f64((x_out.astype(np.int64) - 1).astype(np.uint16))
    for idx in np.ndindex(x.shape):
        exact = Fraction(xf[idx]) + Fraction(gate[0, idx[2]]) * Fraction(rf[idx])
        e = abs(Fraction(got[idx]) - exact)
        assert e <= abs(Fraction(up[idx]) - exact) and e <= abs(Fraction(dn[idx]) - exact)


def test_gated_y_is_adaln_of_rounded_residual(orc):
    """The fused op equals the unfused chain: store x' in bf16, then AdaLN."""
    B, N, D, eps = 2, 5, 80, 1e-6
    x = _rand_bits(orc, (B, N, D), 17)
    r = _rand_bits(orc, (B, N, D), 18)
    rng = np.random.default_rng(19)
    sh, sc, gt = (rng.standard_normal((B, D)) * 0.3 for _ in range(3))
    x_out, y = orc.gated_residual_adaln(x, r, gt, sh, sc, eps)
    assert np.array_equal(y, orc.adaln_modulate(x_out, sh, sc, eps))


# ------------------------------------------- per-token modulation sets


def _token_case(orc, seed, B=2, N=5, D=16, S=3):
    rng = np.random.default_rng(seed)
    x = _bf16(orc, rng.standard_normal((B, N, D)))
    r = _bf16(orc, rng.standard_normal((B, N, D)))
    mods = [rng.standard_normal((B, S, D)) * 0.3 for _ in range(3)]
    idx = rng.integers(0, S, (B, N)).astype(np.uint8)
    return x, r, mods, idx


def test_token_sets_all_zero_are_per_sample(orc):
    """Every token on set 0 is the per-sample operator with set 0's vectors."""
    x, r, (g, sh, sc), idx = _token_case(orc, 1)
    idx[:] = 0
    y = orc.adaln_modulate_tok(x, sh, sc, idx, 1e-6)
    assert np.array_equal(y, orc.adaln_modulate(x, sh[:, 0], sc[:, 0], 1e-6))
    xo, y = orc.gated_residual_adaln_tok(x, r, g, sh, sc, idx, 1e-6)
    xo0, y0 = orc.gated_residual_adaln(x, r, g[:, 0], sh[:, 0], sc[:, 0], 1e-6)
    assert np.array_equal(xo, xo0) and np.array_equal(y, y0)


def test_token_sets_each_token_uses_its_own_set(orc):
    """Token (b, n) equals the per-sample operator run on that token alone
    with the vectors of set idx[b, n] of sample b."""
    x, r, (g, sh, sc), idx = _token_case(orc, 2)
    B, N, D = x.shape
    y = orc.adaln_modulate_tok(x, sh, sc, idx, 1e-6)
    xo, yg = orc.gated_residual_adaln_tok(x, r, g, sh, sc, idx, 1e-6)
    for b in range(B):
        for n in range(N):
            s = idx[b, n]
            one = orc.adaln_modulate(x[b:b + 1, n:n + 1], sh[b, s], sc[b, s], 1e-6)
            assert np.array_equal(y[b, n], one[0, 0])
            xo1, y1 = orc.gated_residual_adaln(x[b:b + 1, n:n + 1], r[b:b + 1, n:n + 1], g[b, s],
                                               sh[b, s], sc[b, s], 1e-6)
            assert np.array_equal(xo[b, n], xo1[0, 0]) and np.array_equal(yg[b, n], y1[0, 0])


def test_token_sets_closed_forms(orc):
    """Set 0 has zero modulation (a plain LayerNorm: row [1, 2, 3, 4] gives
    (x - 2.5) / sqrt(1.25 + eps)); set 1 has scale = -1 (y is its shift) and
    gate 0 (the residual passes unchanged)."""
    eps = 1e-6
    x = _bf16(orc, [[[1, 2, 3, 4], [1, 2, 3, 4], [-8, 0.5, 3, 7]]])
    r = _bf16(orc, np.full((1, 3, 4), 0.75))
    sh = np.array([[[0, 0, 0, 0], [0.5, -1.5, 2.0, 3.25]]])
    sc = np.array([[[0, 0, 0, 0], [-1, -1, -1, -1]]])
    g = np.array([[[1, 1, 1, 1], [0, 0, 0, 0]]])
    idx = np.array([[0, 1, 1]], np.uint8)
    y = orc.adaln_modulate_tok(x, sh, sc, idx, eps)
    ln = (np.array([1, 2, 3, 4]) - 2.5) / np.sqrt(1.25 + eps)
    assert np.allclose(y[0, 0], ln, rtol=1e-15, atol=1e-15)
    assert np.array_equal(y[0, 1], sh[0, 1]) and np.array_equal(y[0, 2], sh[0, 1])
    xo, yg = orc.gated_residual_adaln_tok(x, r, g, sh, sc, idx, eps)
    assert np.array_equal(xo[0, 1:], x[0, 1:])                       # gate 0
    assert np.array_equal(orc.bf16_to_f64(xo[0, 0]), [1.75, 2.75, 3.75, 4.75])
    assert np.allclose(yg[0, 0], ln, rtol=1e-15, atol=1e-15)        # LN is shift-invariant
    assert np.array_equal(yg[0, 2], sh[0, 1])


def test_token_set_out_of_range_is_an_error(orc):
    x, r, (g, sh, sc), idx = _token_case(orc, 3, S=2)
    idx[0, 0] = 2
    with pytest.raises(ValueError):
        orc.adaln_modulate_tok(x, sh, sc, idx, 1e-6)
    with pytest.raises(ValueError):
        orc.gated_residual_adaln_tok(x, r, g, sh, sc, idx, 1e-6)
