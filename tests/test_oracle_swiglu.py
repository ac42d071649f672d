"""Pins for SwiGLU: hand-worked closed forms, the library SiLU, limits."""
import numpy as np
import torch

from conftest import closed_form, load_golden


def test_golden(orc):
    g = load_golden("swiglu.json")
    inp = orc.f64_to_bf16(np.array(g["in"]))
    out = orc.swiglu(inp)
    want = np.array([[closed_form(e) for e in row] for row in g["out"]])
    assert np.allclose(out, want, rtol=1e-15, atol=0)


def test_matches_library_silu(orc):
    rng = np.random.default_rng(0)
    M, F = 33, 40
    inp = orc.f64_to_bf16(rng.standard_normal((M, 2 * F)) * 4)
    v = torch.from_numpy(orc.bf16_to_f64(inp))
    ref = torch.nn.functional.silu(v[:, :F]) * v[:, F:]
    assert np.allclose(orc.swiglu(inp), ref.numpy(), rtol=1e-14, atol=1e-300)


def test_limits(orc):
    F = 6
    a = np.array([0.0, 100.0, -100.0, 30.0, 1.0, -1.0])
    b = np.array([5.0, 1.0, 1.0, -2.0, 0.0, 1.0])
    out = orc.swiglu(orc.f64_to_bf16(np.concatenate([a, b])[None, :]))[0]
    assert out[0] == 0.0                       # silu(0) = 0
    assert out[1] == 100.0                     # silu(a) -> a for large a
    assert abs(out[2]) < 1e-40                 # silu(a) -> 0 for very negative a
    assert np.isclose(out[3], -60.0, rtol=1e-12)
    assert out[4] == 0.0                       # b = 0
    assert np.isclose(out[5], -1.0 / (1.0 + np.e), rtol=1e-15)
    zero = orc.swiglu(np.zeros((3, 2 * F), dtype=np.uint16))
    assert np.all(zero == 0.0)                 # SwiGLU(0) = 0


def test_rows_are_independent(orc):
    rng = np.random.default_rng(1)
    inp = orc.f64_to_bf16(rng.standard_normal((5, 16)))
    full = orc.swiglu(inp)
    for m in range(5):
        assert np.array_equal(full[m], orc.swiglu(inp[m:m + 1])[0])
