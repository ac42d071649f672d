"""Pins for the SubBlock router: block means, summary dot products, top
n_keep key blocks per query block (ties to the lower index), kept indices in
increasing order."""
import math

import numpy as np
import pytest

from conftest import load_golden


def _bf(orc, a):
    return orc.f64_to_bf16(np.asarray(a, dtype=np.float64))


def test_keep_count(orc):
    assert orc.subblock_keep_count(977, 0.75) == 245          # ceil(244.25)
    assert orc.subblock_keep_count(977, 0.80) == 196          # ceil(195.4)
    assert orc.subblock_keep_count(8, 0.75) == 2
    assert orc.subblock_keep_count(3, 0.9) == 1               # at least one
    assert orc.subblock_keep_count(5, 0.0) == 5
    with pytest.raises(ValueError):
        orc.subblock_keep_count(5, 1.0)


def test_golden(orc):
    """Hand-worked: constant rows per block make every summary known."""
    g = load_golden("subblock_router.json")
    for c in g["cases"]:
        q = _bf(orc, c["q"])
        k = _bf(orc, c["k"])
        kept, scores = orc.subblock_router(q, k, 1, c["H"], c["hd"], c["block"], c["sparsity"])
        assert kept[0].tolist() == c["kept"], c["name"]
        if "scores" in c:
            assert np.allclose(scores[0], c["scores"], rtol=0, atol=1e-12), c["name"]


def _rand(orc, seed, B=2, N=45, H=3, hd=8):
    rng = np.random.default_rng(seed)
    q = _bf(orc, rng.standard_normal((B * N, H * hd)))
    k = _bf(orc, rng.standard_normal((B * N, H * hd)))
    return q, k


def test_selection_is_the_top_of_the_scores(orc):
    """Every kept block scores at least as high as every dropped one, the
    kept list is strictly increasing, and equal scores keep the lower index."""
    q, k = _rand(orc, 1)
    kept, sc = orc.subblock_router(q, k, 2, 3, 8, 4, 0.7)
    nb = sc.shape[-1]
    for b in range(2):
        for h in range(3):
            for i in range(nb):
                row = kept[b, h, i]
                assert np.all(np.diff(row) > 0)
                drop = np.setdiff1d(np.arange(nb), row)
                assert sc[b, h, i, row].min() >= sc[b, h, i, drop].max()


def test_means_and_scores_match_numpy(orc):
    """Scores equal the dot products of numpy block means (ragged last block
    averaged over its own length)."""
    B, N, H, hd, blk = 1, 45, 2, 8, 4
    q, k = _rand(orc, 2, B, N, H, hd)
    _, sc = orc.subblock_router(q, k, B, H, hd, blk, 0.5)
    Q = orc.bf16_to_f64(q).reshape(N, H, hd)
    K = orc.bf16_to_f64(k).reshape(N, H, hd)
    nb = math.ceil(N / blk)
    qm = np.stack([Q[j * blk:(j + 1) * blk].mean(0) for j in range(nb)])   # [nb, H, hd]
    km = np.stack([K[j * blk:(j + 1) * blk].mean(0) for j in range(nb)])
    ref = np.einsum("ihd,jhd->hij", qm, km)
    assert np.allclose(sc[0], ref, rtol=1e-12, atol=1e-14)


def test_invariances(orc):
    """Permuting tokens inside a block, and scaling k by 2 (exact), change
    nothing; sparsity 0 keeps every block."""
    B, N, H, hd, blk = 1, 32, 2, 8, 8
    q, k = _rand(orc, 3, B, N, H, hd)
    kept, _ = orc.subblock_router(q, k, B, H, hd, blk, 0.6)
    perm = np.concatenate([np.random.default_rng(4).permutation(blk) + j * blk
                           for j in range(N // blk)])
    kept_p, _ = orc.subblock_router(q[perm], k[perm], B, H, hd, blk, 0.6)
    assert np.array_equal(kept, kept_p)
    k2 = _bf(orc, orc.bf16_to_f64(k) * 2)
    kept_s, _ = orc.subblock_router(q, k2, B, H, hd, blk, 0.6)
    assert np.array_equal(kept, kept_s)
    all_, _ = orc.subblock_router(q, k, B, H, hd, blk, 0.0)
    assert np.array_equal(all_, np.broadcast_to(np.arange(N // blk), all_.shape))


def test_heads_and_samples_are_independent(orc):
    """Swapping two heads' columns swaps their selections; each sample is
    routed on its own tokens."""
    B, N, H, hd, blk = 2, 24, 2, 8, 4
    q, k = _rand(orc, 5, B, N, H, hd)
    kept, _ = orc.subblock_router(q, k, B, H, hd, blk, 0.5)
    sw = np.r_[hd:2 * hd, 0:hd]
    kept_sw, _ = orc.subblock_router(q[:, sw], k[:, sw], B, H, hd, blk, 0.5)
    assert np.array_equal(kept_sw, kept[:, ::-1])
    one, _ = orc.subblock_router(q[N:], k[N:], 1, H, hd, blk, 0.5)
    assert np.array_equal(one[0], kept[1])
