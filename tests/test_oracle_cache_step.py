"""Pins for the Cache-DiT step cache: the cached residual of the skipped
blocks (store and reuse) and the reuse rule over a denoising run."""
import math
from fractions import Fraction

import numpy as np

import oracle
from conftest import load_golden


def _bits(orc, v):
    return orc.f64_to_bf16(np.asarray(v, dtype=np.float64))


def _val(orc, b):
    return orc.bf16_to_f64(np.asarray(b, dtype=np.uint16))


def test_residual_golden(orc):
    g = load_golden("residual_cache.json")
    for c in g["store"]:
        r = orc.residual_store(_bits(orc, [c["before"]]), _bits(orc, [c["after"]]))
        assert _val(orc, r)[0] == c["R"], c
    for c in g["apply"]:
        o = orc.residual_apply(_bits(orc, [c["h"]]), _bits(orc, [c["R"]]))
        assert _val(orc, o)[0] == c["out"], c


def _nearest_even(orc, got_bits, exact):
    """got is a nearest bf16 to the exact rational, and on a tie the one with
    the even significand."""
    got = Fraction(float(_val(orc, [got_bits])[0]))
    up = Fraction(float(_val(orc, [(int(got_bits) + 1) & 0xFFFF])[0]))
    dn = Fraction(float(_val(orc, [(int(got_bits) - 1) & 0xFFFF])[0]))
    e = abs(got - exact)
    assert e <= abs(up - exact) and e <= abs(dn - exact)
    if e == abs(up - exact) or e == abs(dn - exact):
        if e != 0:
            assert int(got_bits) % 2 == 0


def test_residual_is_nearest_even_of_exact_value(orc):
    """Brute force against exact rational arithmetic, over operands spread
    across 40 binades so that many differences are inexact in bf16."""
    rng = np.random.default_rng(5)
    a = _bits(orc, rng.standard_normal(600) * np.exp2(rng.integers(-20, 20, 600)))
    b = _bits(orc, rng.standard_normal(600) * np.exp2(rng.integers(-20, 20, 600)))
    r = orc.residual_store(a, b)
    o = orc.residual_apply(a, b)
    av, bv = _val(orc, a), _val(orc, b)
    for i in range(a.size):
        _nearest_even(orc, r[i], Fraction(float(bv[i])) - Fraction(float(av[i])))
        _nearest_even(orc, o[i], Fraction(float(av[i])) + Fraction(float(bv[i])))


def test_residual_round_trip_and_identities(orc):
    """store(x, x) = 0; apply(h, 0) = h; when after - before is a bf16 value
    (same binade, few bits), apply(before, store(before, after)) = after."""
    rng = np.random.default_rng(6)
    x = _bits(orc, rng.standard_normal(500))
    assert not _val(orc, orc.residual_store(x, x)).any()
    assert np.array_equal(orc.residual_apply(x, np.zeros_like(x)), x)
    before = _bits(orc, 1.0 + rng.integers(0, 128, 500) / 128.0)     # [1, 2), exact
    after = _bits(orc, 1.0 + rng.integers(0, 128, 500) / 128.0)
    r = orc.residual_store(before, after)
    assert np.array_equal(orc.residual_apply(before, r), after)


def test_residual_overflow_and_nan(orc):
    big = _bits(orc, [3.0e38, -3.0e38, float("nan")])
    r = orc.residual_store(_bits(orc, [-3.0e38, 3.0e38, 1.0]), big)
    v = _val(orc, r)
    assert v[0] == math.inf and v[1] == -math.inf and math.isnan(v[2])


def test_policy_golden():
    g = load_golden("cache_policy.json")
    for c in g["cases"]:
        rels = [float(x) for x in c["rels"]]
        got = oracle.cache_policy(rels, c["threshold"], c["warmup"], c["max_cached"])
        assert "".join("R" if d else "C" for d in got) == c["expect"], c


def test_policy_invariants():
    """A higher threshold never reuses less; the first step always computes;
    with a cap m, no m+1 reuses in a row; no reuse above the threshold."""
    rng = np.random.default_rng(7)
    for _ in range(200):
        rels = list(rng.exponential(0.05, 50))
        lo = oracle.cache_policy(rels, 0.04)
        hi = oracle.cache_policy(rels, 0.08)
        assert all(h or not l for l, h in zip(lo, hi))
        assert not lo[0] and not hi[0]
        assert all(not d or r < 0.04 for d, r in zip(lo[1:], rels[1:]))
        capped = oracle.cache_policy(rels, 0.08, max_cached_steps=3)
        runs = "".join("R" if d else "C" for d in capped).split("C")
        assert max(len(x) for x in runs) <= 3
