"""Tolerance rule for comparing CUDA bf16 outputs with the fp64 oracle.

The oracle's fp64 result is rounded once to bf16 (the reference value).  A
CUDA output passes when

    |gpu - ref| <= 2 * ulp_bf16(max(|ref|, 2^-12))          (every element)
    mean(|gpu - ref| / |ref|) <= 1e-3   over elements with |ref| >= 2^-12

ulp_bf16(m) = 2^(floor(log2 m) - 7) (8 significant bits).  The 2^-12 floor
keeps the rule meaningful where an output cancels to almost zero (for
example n*(1+scale) + shift ~ 0): there the fp32 arithmetic of the kernel
carries an absolute error near 1e-7 while a strict 2-ulp rule would demand
less than 1e-9.  Elements that pass without the floor are counted too.
NaN must match NaN and infinities must match exactly.
"""
from __future__ import annotations

import numpy as np

import oracle

FLOOR = 2.0 ** -12
MAX_ULPS = 2.0
MEAN_REL = 1e-3


def _ulp(mag: np.ndarray) -> np.ndarray:
    return np.exp2(np.floor(np.log2(mag)) - 7)


def compare_bf16(gpu_bits: np.ndarray, ref64: np.ndarray, what: str = "",
                 max_ulps: float = MAX_ULPS, mean_rel: float = MEAN_REL, floor: float = FLOOR):
    orc = oracle.default()
    gpu_bits = np.ascontiguousarray(gpu_bits, dtype=np.uint16).reshape(-1)
    ref64 = np.ascontiguousarray(ref64, dtype=np.float64).reshape(-1)
    assert gpu_bits.size == ref64.size, f"{what}: size mismatch"
    r = orc.bf16_to_f64(orc.f64_to_bf16(ref64))
    g = orc.bf16_to_f64(gpu_bits)
    nan = np.isnan(r)
    assert np.array_equal(np.isnan(g), nan), f"{what}: NaN positions differ"
    inf = np.isinf(r)
    assert np.array_equal(g[inf], r[inf]), f"{what}: infinities differ"
    keep = ~(nan | inf)
    r, g = r[keep], g[keep]
    err = np.abs(g - r)
    tol = max_ulps * _ulp(np.maximum(np.abs(r), floor))
    bad = np.nonzero(err > tol)[0]
    if bad.size:
        i = bad[:8]
        raise AssertionError(
            f"{what}: {bad.size} of {r.size} elements beyond {max_ulps} ulp; "
            f"first: ref={r[i].tolist()} gpu={g[i].tolist()}")
    big = np.abs(r) >= floor
    mre = float((err[big] / np.abs(r[big])).mean()) if big.any() else 0.0
    assert mre <= mean_rel, f"{what}: mean relative error {mre:.3g} > {mean_rel}"
    strict_tol = max_ulps * _ulp(np.maximum(np.abs(r), np.finfo(np.float64).tiny))
    nz = r != 0
    return {
        "n": int(r.size),
        "exact_frac": float((err == 0).mean()) if r.size else 1.0,
        "max_ulps": float((err / _ulp(np.maximum(np.abs(r), floor))).max()) if r.size else 0.0,
        "mean_rel": mre,
        "strict_fail": int((err[nz] > strict_tol[nz]).sum()),
    }


def bits(t) -> np.ndarray:
    """bf16 torch tensor -> host uint16 bit patterns."""
    import torch
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)
