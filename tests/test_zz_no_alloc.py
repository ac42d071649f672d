"""The Cache-DiT check for callers that cannot allocate device memory.

Some callers cannot call cudaMalloc or pass this library a workspace: a
plugin inside a serving engine that owns all device memory through its own
pool, or a caller on a latency-critical path that cannot take the device-wide
synchronisation a fresh allocation can cause.  cachedit_residual_diff_noalloc
serves them from a fixed array inside the library.  Its results must match
the workspace entry point's, call after call, although every call reuses the
same array and finds the previous call's partial sums in it.

This file sorts last so that a run which stops at the first failure has
already run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

import dit_block_pass_b200 as dbp
from dit_block_pass_b200 import workloads as W
from parity import bits

A = 0x10000  # a 16-byte aligned fake address, never dereferenced by the host checks


def _lib():
    from dit_block_pass_b200 import build
    build.build()
    return dbp.library()


def test_noalloc_rejects_bad_arguments_on_the_host():
    """Checks that return before any CUDA call: too many samples, NULLs."""
    L = _lib()
    f = L.cachedit_residual_diff_noalloc
    assert f(A, A, 65, 4, 64, 0.04, A, A, None) == -2          # more than 64 samples
    assert f(A, A, 0, 4, 64, 0.04, A, A, None) == -2
    assert f(None, A, 1, 4, 64, 0.04, A, A, None) == -1
    assert f(A, A, 1, 4, 64, 0.04, None, A, None) == -1
    assert f(A, A, 1, 4, 60, 0.04, A, A, None) == -3
    assert f(A, A, 1, 4, 64, float("nan"), A, A, None) == -8


@pytest.mark.gpu
def test_noalloc_matches_the_workspace_entry_point_on_consecutive_calls(orc):
    _lib()
    dev = "cuda:0"
    cases = [
        W.Workload("a", B=3, T=1, Hg=1, Wg=301, D=512, H=4, hd=128, F=8, pairs=(22, 21, 21),
                   sigma_cache=(0.03, 0.05, 0.1)),
        W.Workload("b", B=2, T=2, Hg=24, Wg=42, D=3072, H=24, hd=128, F=8, pairs=(22, 21, 21),
                   sigma_cache=(0.1, 0.03), seed=7),
    ]
    inputs = []
    for wl in cases:
        prev, cur = W.cache_pair(wl, device=dev)
        inputs.append((prev.view(wl.B, wl.N, wl.D), cur.view(wl.B, wl.N, wl.D)))
    # two calls in a row, on different inputs, through the C ABI
    got = [dbp.cachedit_residual_diff_noalloc(p, c, 0.04) for p, c in inputs]
    got = [(r.cpu().numpy(), u.cpu().numpy()) for r, u in got]
    for (p, c), (rel, reuse) in zip(inputs, got):
        ref_rel, ref_reuse = dbp.cachedit_residual_diff(p, c, 0.04)
        ref_rel, ref_reuse = ref_rel.cpu().numpy(), ref_reuse.cpu().numpy()
        assert np.allclose(rel, ref_rel, rtol=1e-7, atol=0), (rel, ref_rel)
        assert np.array_equal(reuse, ref_reuse)
        # and against the fp64 oracle on the same bf16 inputs
        o_rel, o_reuse = orc.cachedit_residual_diff(bits(p), bits(c), 0.04)
        assert np.allclose(rel, o_rel, rtol=1e-7, atol=0), (rel, o_rel)
        assert np.all(np.abs(o_rel - 0.04) > 1e-6), "decision margin too small to be meaningful"
        assert np.array_equal(reuse, o_reuse)
    # and the first input again, after the array holds the second call's sums
    rel, reuse = dbp.cachedit_residual_diff_noalloc(*inputs[0], 0.04)
    assert np.allclose(rel.cpu().numpy(), got[0][0], rtol=1e-7, atol=0)
    assert np.array_equal(reuse.cpu().numpy(), got[0][1])


def _exact_pair(B, N, D, seed):
    """prev with values (+-1 or +-1.5) * 2^j and cur = (1 + c_b) * prev with
    c_b in {+-2^-4, +-2^-5, +-2^-6}: every product is a bf16 value (at most 8
    significant bits), so rel_b is |c_b| exactly, in any summation order that
    treats the two sums alike (scaling by a power of two commutes with
    rounding)."""
    rng = np.random.default_rng(seed)
    mant = rng.choice([1.0, 1.5], size=(B, N, D))
    sign = rng.choice([-1.0, 1.0], size=(B, N, D))
    expo = rng.integers(-3, 4, size=(B, N, D)).astype(np.float64)
    prev = sign * mant * np.exp2(expo)
    c = np.array([2.0 ** -4, -2.0 ** -4, 2.0 ** -5, -2.0 ** -5, 2.0 ** -6, -2.0 ** -6])[
        np.arange(B) % 6]
    cur = (1.0 + c[:, None, None]) * prev
    to = lambda a: torch.from_numpy(a).to(torch.bfloat16)
    tp, tc = to(prev), to(cur)
    assert np.array_equal(tp.double().numpy(), prev) and np.array_equal(tc.double().numpy(), cur)
    return tp, tc, np.abs(c)


@pytest.mark.gpu
@pytest.mark.parametrize("B,N,D", [(64, 300, 512), (6, 37, 72)])
def test_noalloc_matches_the_oracle_at_exact_thresholds(orc, B, N, D):
    """Against the fp64 oracle, not only the workspace entry point: rel is
    known exactly, and thresholds on and beside it check the strict < of the
    decision (B = 64 is the largest batch the fixed array takes)."""
    _lib()
    tp, tc, c = _exact_pair(B, N, D, seed=B)
    prev, cur = tp.to("cuda:0"), tc.to("cuda:0")
    pb = tp.contiguous().view(torch.int16).numpy().view(np.uint16)
    cb = tc.contiguous().view(torch.int16).numpy().view(np.uint16)
    rel_buf = torch.empty(B, dtype=torch.float64, device="cuda:0")
    reuse_buf = torch.empty(B, dtype=torch.uint8, device="cuda:0")
    for thr in (2.0 ** -5, np.nextafter(2.0 ** -5, 1.0), np.nextafter(2.0 ** -6, 0.0), 0.04):
        rel, reuse = dbp.cachedit_residual_diff_noalloc(prev, cur, float(thr), rel=rel_buf,
                                                        reuse=reuse_buf)
        assert rel is rel_buf and reuse is reuse_buf
        ref_rel, ref_reuse = orc.cachedit_residual_diff(pb, cb, float(thr))
        got_rel, got_reuse = rel.cpu().numpy(), reuse.cpu().numpy()
        assert np.array_equal(ref_rel, c), "the oracle must find rel = |c| exactly"
        assert np.array_equal(got_rel, ref_rel), (got_rel, ref_rel)
        assert np.array_equal(got_reuse, ref_reuse), (thr, got_reuse, ref_reuse)
        assert np.array_equal(got_reuse, (c < thr).astype(np.uint8))


@pytest.mark.gpu
def test_noalloc_checks_its_result_buffers():
    _lib()
    x = torch.zeros(4, 2, 64, dtype=torch.bfloat16, device="cuda:0")
    with pytest.raises(ValueError):
        dbp.cachedit_residual_diff_noalloc(x, x, 0.04,
                                           rel=torch.empty(3, dtype=torch.float64, device="cuda:0"))
    with pytest.raises(ValueError):
        dbp.cachedit_residual_diff_noalloc(x, x, 0.04,
                                           reuse=torch.empty(4, dtype=torch.float32, device="cuda:0"))


@pytest.mark.gpu
def test_noalloc_too_many_samples_is_a_clear_error():
    _lib()
    x = torch.zeros(65, 2, 64, dtype=torch.bfloat16, device="cuda:0")
    with pytest.raises(dbp.DitError) as e:
        dbp.cachedit_residual_diff_noalloc(x, x, 0.04)
    assert e.value.status == -2
