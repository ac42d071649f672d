"""Pins for the gated residual fused into the down-projection GEMM:
x' = bf16(x + gate_b * (h w^T))."""
from fractions import Fraction

import numpy as np
import torch


def _bf(orc, a):
    return orc.f64_to_bf16(np.asarray(a, dtype=np.float64))


def _case(orc, seed, B=2, N=3, K=48, D=10):
    rng = np.random.default_rng(seed)
    h = _bf(orc, rng.standard_normal((B * N, K)))
    w = _bf(orc, rng.standard_normal((D, K)) / np.sqrt(K))
    x = _bf(orc, rng.standard_normal((B * N, D)))
    gate = rng.standard_normal((B, D)).astype(np.float32).astype(np.float64)
    return h, w, x, gate


def test_zero_gate_leaves_the_residual(orc):
    h, w, x, gate = _case(orc, 1)
    out, _, _ = orc.gemm_gated_residual(h, w, x, np.zeros_like(gate), 3)
    assert np.array_equal(out, x)


def test_one_hot_weights_reduce_to_the_gated_residual(orc):
    """One-hot weight rows make the product a column selection r = h[:, a];
    x' is then the pinned a2 residual update with that branch."""
    rng = np.random.default_rng(2)
    B, N, K, D = 2, 4, 16, 8
    h = _bf(orc, rng.standard_normal((B * N, K)))
    x = _bf(orc, rng.standard_normal((B * N, D)))
    gate = rng.standard_normal((B, D)).astype(np.float32).astype(np.float64)
    a = rng.integers(0, K, D)
    wf = np.zeros((D, K))
    wf[np.arange(D), a] = 1.0
    out, _, _ = orc.gemm_gated_residual(h, _bf(orc, wf), x, gate, N)
    r = h[:, a]
    z = np.zeros((B, D))
    x_ref, _ = orc.gated_residual_adaln(x.reshape(B, N, D), r.reshape(B, N, D), gate, z, z, 1e-6)
    assert np.array_equal(out, x_ref.reshape(B * N, D))


def test_nearest_bf16_and_library_matmul(orc):
    """dot equals float64 torch matmul; x' is a nearest bf16 of x + g dot."""
    h, w, x, gate = _case(orc, 3, B=2, N=4, K=64, D=12)
    out, dot, ad = orc.gemm_gated_residual(h, w, x, gate, 4)
    H = torch.from_numpy(orc.bf16_to_f64(h))
    Wf = torch.from_numpy(orc.bf16_to_f64(w))
    assert np.allclose(dot, (H @ Wf.T).numpy(), rtol=1e-12, atol=1e-14)
    assert np.allclose(ad, (H.abs() @ Wf.abs().T).numpy(), rtol=1e-12)
    xv = orc.bf16_to_f64(x)
    got = orc.bf16_to_f64(out)
    up = orc.bf16_to_f64((out.astype(np.int64) + 1).astype(np.uint16))
    dn = orc.bf16_to_f64((out.astype(np.int64) - 1).astype(np.uint16))
    for m in range(8):
        for n in range(12):
            exact = Fraction(xv[m, n]) + Fraction(gate[m // 4, n]) * Fraction(dot[m, n])
            e = abs(Fraction(got[m, n]) - exact)
            assert e <= abs(Fraction(up[m, n]) - exact) and e <= abs(Fraction(dn[m, n]) - exact)


def test_each_sample_uses_its_gate(orc):
    """Rows of sample b use gate row b: swapping the gate rows swaps the
    samples' results when the samples' inputs are swapped too."""
    h, w, x, gate = _case(orc, 4, B=2, N=3)
    out, _, _ = orc.gemm_gated_residual(h, w, x, gate, 3)
    perm = np.r_[3:6, 0:3]
    out2, _, _ = orc.gemm_gated_residual(h[perm], w, x[perm], gate[::-1].copy(), 3)
    assert np.array_equal(out2, out[perm])


def test_row_selection(orc):
    h, w, x, gate = _case(orc, 5, B=3, N=2)
    full, fd, _ = orc.gemm_gated_residual(h, w, x, gate, 2)
    rows = np.array([5, 0, 3])
    part, pd, _ = orc.gemm_gated_residual(h, w, x, gate, 2, rows)
    assert np.array_equal(part, full[rows]) and np.array_equal(pd, fd[rows])
