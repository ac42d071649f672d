"""Pins for block-sparse attention over the router's kept key blocks."""
import numpy as np
import torch


def _bf(orc, a):
    return orc.f64_to_bf16(np.asarray(a, dtype=np.float64))


def _qkv(orc, seed, B, N, H, hd):
    rng = np.random.default_rng(seed)
    return tuple(_bf(orc, rng.standard_normal((B * N, H * hd))) for _ in range(3))


def _all_blocks(B, H, nb):
    return np.broadcast_to(np.arange(nb, dtype=np.int32), (B, H, nb, nb)).copy()


def test_all_blocks_is_dense_attention(orc):
    """Keeping every block is plain attention: torch's float64
    scaled_dot_product_attention."""
    B, N, H, hd, blk = 2, 20, 2, 8, 4
    q, k, v = _qkv(orc, 1, B, N, H, hd)
    out = orc.block_sparse_attention(q, k, v, B, H, hd, blk, _all_blocks(B, H, 5))
    f = lambda a: torch.from_numpy(orc.bf16_to_f64(a)).view(B, N, H, hd).transpose(1, 2)
    ref = torch.nn.functional.scaled_dot_product_attention(f(q), f(k), f(v))
    assert np.allclose(out, ref.transpose(1, 2).reshape(B * N, H * hd).numpy(), rtol=1e-12,
                       atol=1e-13)


def test_single_block_and_ragged_tail(orc):
    """One kept block: attention restricted to its tokens (the ragged last
    block has 2 of 4); torch's attention on those keys only."""
    B, N, H, hd, blk = 1, 14, 1, 8, 4
    q, k, v = _qkv(orc, 2, B, N, H, hd)
    nb = 4
    for j in range(nb):
        kept = np.full((B, H, nb, 1), j, dtype=np.int32)
        out = orc.block_sparse_attention(q, k, v, B, H, hd, blk, kept)
        sl = slice(j * blk, min(N, (j + 1) * blk))
        f = lambda a: torch.from_numpy(orc.bf16_to_f64(a))[None, None]
        ref = torch.nn.functional.scaled_dot_product_attention(f(q), f(k[sl]), f(v[sl]))
        assert np.allclose(out, ref[0, 0].numpy(), rtol=1e-12, atol=1e-13), j


def test_zero_query_averages_the_kept_values(orc):
    """q = 0 gives equal weights: the mean of v over the kept tokens."""
    B, N, H, hd, blk = 1, 12, 1, 8, 4
    _, k, v = _qkv(orc, 3, B, N, H, hd)
    q = np.zeros_like(k)
    kept = np.array([[[[0, 2]], [[1, 2]], [[0, 1]]]], dtype=np.int32).reshape(1, 1, 3, 2)
    out = orc.block_sparse_attention(q, k, v, B, H, hd, blk, kept)
    V = orc.bf16_to_f64(v)
    for t in range(N):
        i = t // blk
        toks = np.concatenate([np.arange(j * blk, (j + 1) * blk) for j in kept[0, 0, i]])
        assert np.allclose(out[t], V[toks].mean(0), rtol=1e-13, atol=1e-14)


def test_invariances(orc):
    """The order of the kept list and of the tokens inside a kept block does
    not matter; doubling v (exact in bf16) doubles the output."""
    B, N, H, hd, blk = 1, 16, 1, 8, 4
    q, k, v = _qkv(orc, 4, B, N, H, hd)
    kept = np.array([[0, 3], [1, 2], [0, 2], [1, 3]], dtype=np.int32).reshape(1, 1, 4, 2)
    base = orc.block_sparse_attention(q, k, v, B, H, hd, blk, kept)
    rev = orc.block_sparse_attention(q, k, v, B, H, hd, blk, kept[..., ::-1].copy())
    assert np.allclose(rev, base, rtol=1e-13, atol=1e-14)
    perm = np.concatenate([np.random.default_rng(5).permutation(blk) + j * blk
                           for j in range(4)])
    out_p = orc.block_sparse_attention(q, k[perm], v[perm], B, H, hd, blk, kept)
    assert np.allclose(out_p, base, rtol=1e-12, atol=1e-13)
    v2 = _bf(orc, orc.bf16_to_f64(v) * 2)
    assert np.allclose(orc.block_sparse_attention(q, k, v2, B, H, hd, blk, kept), 2 * base,
                       rtol=1e-13, atol=1e-14)


def test_samples_and_heads_are_independent(orc):
    B, N, H, hd, blk = 2, 8, 2, 8, 4
    q, k, v = _qkv(orc, 6, B, N, H, hd)
    kept = np.array([0, 1, 1, 0, 1, 1, 0, 0], dtype=np.int32).reshape(B, H, 2, 1)
    out = orc.block_sparse_attention(q, k, v, B, H, hd, blk, kept)
    one = orc.block_sparse_attention(q[N:], k[N:], v[N:], 1, H, hd, blk, kept[1:])
    assert np.allclose(out[N:], one, rtol=0, atol=0)


def test_row_selection(orc):
    B, N, H, hd, blk = 2, 12, 2, 8, 4
    q, k, v = _qkv(orc, 7, B, N, H, hd)
    kept = np.array([[[[0], [2], [1]], [[1], [1], [0]]], [[[2], [0], [1]], [[0], [1], [2]]]],
                    dtype=np.int32)
    full = orc.block_sparse_attention(q, k, v, B, H, hd, blk, kept)
    rows = np.array([23, 0, 13, 5])
    part = orc.block_sparse_attention(q, k, v, B, H, hd, blk, kept, rows=rows)
    assert np.array_equal(part, full[rows])
