"""Pins for SwiGLU fused into the up-projection GEMM: out = silu(x Wg^T) * (x Wu^T)."""
import numpy as np
import torch

import oracle  # noqa: F401  (the oracle fixture comes from conftest)


def _bf(orc, a):
    return orc.f64_to_bf16(np.asarray(a, dtype=np.float64))


def _case(orc, seed, M=6, K=40, F=5, wscale=None):
    rng = np.random.default_rng(seed)
    x = _bf(orc, rng.standard_normal((M, K)))
    w = _bf(orc, rng.standard_normal((2 * F, K)) * (wscale or 1.0 / np.sqrt(K)))
    return x, w


def test_one_hot_weights_reduce_to_swiglu(orc):
    """With one-hot weight rows the products pick columns of x, and the fused
    operator is the pinned SwiGLU of those columns."""
    rng = np.random.default_rng(1)
    M, K, F = 7, 24, 6
    x = _bf(orc, rng.standard_normal((M, K)) * 2)
    a = rng.integers(0, K, F)
    b = rng.integers(0, K, F)
    wf = np.zeros((2 * F, K))
    wf[np.arange(F), a] = 1.0
    wf[F + np.arange(F), b] = 1.0
    out, _, _ = orc.swiglu_gemm(x, _bf(orc, wf))
    pair = np.concatenate([x[:, a], x[:, b]], axis=1)
    assert np.array_equal(out, orc.swiglu(pair))


def test_matches_float64_library_matmul(orc):
    x, w = _case(orc, 2, M=9, K=64, F=11)
    out, ga, ua = orc.swiglu_gemm(x, w)
    X = torch.from_numpy(orc.bf16_to_f64(x))
    W = torch.from_numpy(orc.bf16_to_f64(w))
    g = X @ W[:11].T
    u = X @ W[11:].T
    ref = torch.nn.functional.silu(g) * u
    assert np.allclose(out, ref.numpy(), rtol=1e-12, atol=1e-14)
    assert np.allclose(ga, (X.abs() @ W[:11].abs().T).numpy(), rtol=1e-12)
    assert np.allclose(ua, (X.abs() @ W[11:].abs().T).numpy(), rtol=1e-12)


def test_sign_symmetry_closed_form(orc):
    """silu(-g) = silu(g) - g, so out(x) + out(-x) = g * u."""
    x, w = _case(orc, 3, M=5, K=32, F=7)
    out_p, _, _ = orc.swiglu_gemm(x, w)
    out_n, _, _ = orc.swiglu_gemm(x ^ np.uint16(0x8000), w)
    X = orc.bf16_to_f64(x)
    Wf = orc.bf16_to_f64(w)
    gu = (X @ Wf[:7].T) * (X @ Wf[7:].T)
    assert np.allclose(out_p + out_n, gu, rtol=1e-11, atol=1e-13)


def test_linear_half_scales_exactly(orc):
    """Doubling the linear half's weights (exact in bf16) doubles the output
    exactly; zero input gives zero."""
    x, w = _case(orc, 4, M=4, K=48, F=6)
    w2 = w.copy()
    w2[6:] = _bf(orc, orc.bf16_to_f64(w[6:]) * 2)
    a, _, _ = orc.swiglu_gemm(x, w)
    b, _, _ = orc.swiglu_gemm(x, w2)
    assert np.array_equal(b, 2 * a)
    z, _, _ = orc.swiglu_gemm(np.zeros_like(x), w)
    assert not z.any()


def test_row_selection(orc):
    x, w = _case(orc, 5, M=10, K=16, F=3)
    full, fg, fu = orc.swiglu_gemm(x, w)
    rows = np.array([9, 0, 4])
    part, pg, pu = orc.swiglu_gemm(x, w, rows)
    assert np.array_equal(part, full[rows]) and np.array_equal(pg, fg[rows])
    assert np.array_equal(pu, fu[rows])


def test_hand_worked(orc):
    """K = 2, x = [1, 2].  Gate row [0.5, 0.25] gives g = 1 and linear row
    [2, -1] gives u = 0, so the output is 0; a zero gate row gives g = 0 and
    silu 0.  With linear row [3, 0] (u = 3) the output is 3 / (1 + e^-1)."""
    x = _bf(orc, [[1.0, 2.0]])
    w = _bf(orc, [[0.5, 0.25], [0.0, 0.0], [2.0, -1.0], [1.0, 1.0]])
    out, ga, ua = orc.swiglu_gemm(x, w)
    assert out[0, 0] == 0.0
    assert out[0, 1] == 0.0
    assert ga[0, 0] == 1.0 and ua[0, 0] == 4.0
    w2 = _bf(orc, [[0.5, 0.25], [3.0, 0.0]])
    out2, _, _ = orc.swiglu_gemm(x, w2)
    assert abs(out2[0, 0] - 3.0 / (1.0 + np.exp(-1.0))) < 1e-15
