"""Pins for the Cache-DiT relative-L1 residual check."""
import numpy as np

from conftest import closed_form, load_golden


def test_golden(orc):
    for case in load_golden("cachedit.json")["cases"]:
        prev = orc.f64_to_bf16(np.array(case["prev"])).reshape(1, 1, -1)
        cur = orc.f64_to_bf16(np.array(case["cur"])).reshape(1, 1, -1)
        rel, reuse = orc.cachedit_residual_diff(prev, cur, case["threshold"])
        want = closed_form(case["rel"])
        assert rel[0] == want or np.isclose(rel[0], want, rtol=1e-15), case
        assert reuse[0] == case["reuse"], case


def _bits(orc, a):
    return orc.f64_to_bf16(np.asarray(a, dtype=np.float64))


def test_identical_inputs_reuse(orc):
    rng = np.random.default_rng(0)
    prev = _bits(orc, rng.standard_normal((2, 50, 24)))
    rel, reuse = orc.cachedit_residual_diff(prev, prev.copy(), 0.04)
    assert np.all(rel == 0.0) and np.all(reuse == 1)


def test_uniform_relative_change_is_exact(orc):
    """cur = (1 + c) * prev with bf16-exact products gives rel = |c| exactly."""
    rng = np.random.default_rng(1)
    vals = np.array([1.0, -1.0, 1.5, -1.5, 0.75, 2.0, -3.0, 0.375])
    prev_f = rng.choice(vals, (1, 64, 16))
    for c in (2.0 ** -5, -(2.0 ** -5), 2.0 ** -3):
        prev = _bits(orc, prev_f)
        cur = _bits(orc, prev_f * (1.0 + c))
        assert np.array_equal(orc.bf16_to_f64(cur), prev_f * (1.0 + c))
        rel, _ = orc.cachedit_residual_diff(prev, cur, 0.04)
        assert rel[0] == abs(c)


def test_sign_flip_gives_two(orc):
    rng = np.random.default_rng(2)
    prev_f = rng.standard_normal((1, 30, 8))
    prev = _bits(orc, prev_f)
    cur = _bits(orc, -orc.bf16_to_f64(prev))
    rel, reuse = orc.cachedit_residual_diff(prev, cur, 0.04)
    assert rel[0] == 2.0 and reuse[0] == 0


def test_per_sample_independence(orc):
    rng = np.random.default_rng(3)
    prev = _bits(orc, rng.standard_normal((2, 40, 32)))
    cur = prev.copy()
    cur[1] = _bits(orc, orc.bf16_to_f64(prev[1]) * 1.5)
    rel, reuse = orc.cachedit_residual_diff(prev, cur, 0.04)
    assert rel[0] == 0.0 and reuse[0] == 1
    assert np.isclose(rel[1], 0.5, rtol=1e-2) and reuse[1] == 0
    r1, _ = orc.cachedit_residual_diff(prev[1:], cur[1:], 0.04)
    assert r1[0] == rel[1]


def test_sums_split_additively(orc):
    """The sums over a sample equal the sums of its row shards (the basis of
    the sharded check)."""
    rng = np.random.default_rng(4)
    prev = _bits(orc, rng.standard_normal((1, 100, 64)))
    cur = _bits(orc, orc.bf16_to_f64(prev) + 0.05 * rng.standard_normal(prev.shape))
    num, den = orc.cachedit_sums(prev, cur)
    parts = [orc.cachedit_sums(prev[:, a:b], cur[:, a:b]) for a, b in ((0, 37), (37, 100))]
    assert np.isclose(num, sum(p[0] for p in parts), rtol=1e-14)
    assert np.isclose(den, sum(p[1] for p in parts), rtol=1e-14)


def test_noise_level_is_recovered(orc):
    """cur = prev + N(0, s^2) noise gives rel close to s * E|z| / E|prev| = s
    for N(0,1) prev (bf16 rounding of cur adds a little)."""
    rng = np.random.default_rng(5)
    pf = rng.standard_normal((1, 400, 256))
    prev = _bits(orc, pf)
    for s in (0.03, 0.1):
        cur = _bits(orc, orc.bf16_to_f64(prev) + s * rng.standard_normal(pf.shape))
        rel, _ = orc.cachedit_residual_diff(prev, cur, 0.04)
        assert s * 0.95 < rel[0] < s * 1.25
