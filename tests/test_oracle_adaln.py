"""Pins for AdaLN modulation and the gated residual fused with it."""
from decimal import Decimal, getcontext
from fractions import Fraction

import numpy as np
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
