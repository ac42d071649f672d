"""The seeded input generators: exact integer hashing, subset consistency,
distributions, shapes of the H3-shaped workloads."""
import numpy as np
import torch

from dit_block_pass_b200 import workloads as W


def test_mul32_and_fmix32_are_exact():
    rng = np.random.default_rng(0)
    x = rng.integers(0, 2**32, 5000, dtype=np.int64)
    for c in (0x85EBCA6B, 0xC2B2AE35, 0x9E3779B1, 1, 0xFFFFFFFF):
        got = W._mul32(torch.from_numpy(x), c).numpy()
        want = np.array([(int(v) * c) & 0xFFFFFFFF for v in x], dtype=np.int64)
        assert np.array_equal(got, want)
    got = W._fmix32(torch.from_numpy(x)).numpy()
    want = np.array([W._fmix32_int(int(v)) for v in x], dtype=np.int64)
    assert np.array_equal(got, want)


def test_deterministic_and_row_subsets_agree():
    a = W.normal(0, 5, 300, 70)
    b = W.normal(0, 5, 300, 70)
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))
    rows = torch.tensor([0, 7, 150, 299])
    sub = W.normal(0, 5, 300, 70, row_ids=rows)
    assert torch.equal(sub.view(torch.int16), a[rows].view(torch.int16))
    # small chunks give the same values
    c = W.normal(0, 5, 300, 70, chunk=1000)
    assert torch.equal(c.view(torch.int16), a.view(torch.int16))
    # a different stream or seed differs
    assert not torch.equal(W.normal(0, 6, 300, 70), a)
    assert not torch.equal(W.normal(1, 5, 300, 70), a)


def test_large_indices_use_the_high_word():
    idx = torch.tensor([5, 5 + (1 << 32)], dtype=torch.int64)
    h = W.hash_bits(0, 1, idx)
    assert h[0] != h[1]


def test_distributions():
    v = W.normal(0, 1, 2000, 500, dtype=torch.float32)
    assert abs(v.mean().item()) < 0.01 and abs(v.std().item() - 1.0) < 0.01
    m = W.normal(0, 2, 1000, 100, sigma=0.1, dtype=torch.float32)
    assert abs(m.std().item() - 0.1) < 0.002
    w = W.normal(0, 3, 1000, 100, sigma=0.02, mean=1.0, dtype=torch.float32)
    assert abs(w.mean().item() - 1.0) < 0.001 and abs(w.std().item() - 0.02) < 0.001
    assert v.abs().max().item() < 4.5


def test_workload_shapes():
    c = W.CONFIGS
    assert c["tiny"].N == 48 and c["small"].N == 8064
    assert c["h3_5s"].N == 124992 and c["h3_10s"].N == 245952
    assert c["cfg_av"].N == 124992 + 1200 and c["cfg_av"].B == 2
    for wl in c.values():
        assert sum(wl.pairs) == wl.hd // 2 and wl.H * wl.hd == wl.D


def test_explicit_positions_for_audio(orc):
    wl = W.Workload("t", B=2, T=2, Hg=3, Wg=4, D=64, H=1, hd=64, F=64, pairs=(12, 10, 10),
                    n_audio=5)
    pos = W.positions(wl).numpy()
    assert pos.shape == (2 * wl.N, 3)
    video = orc.grid_positions(2, 3, 4, 0, 24)
    for b in range(2):
        blk = pos[b * wl.N:(b + 1) * wl.N]
        assert np.array_equal(blk[:24], video)
        assert np.array_equal(blk[24:, 0], np.arange(5)) and np.all(blk[24:, 1:] == 0)
    assert W.positions(W.CONFIGS["tiny"]) is None


def test_cache_pair_noise_per_sample():
    wl = W.Workload("t", B=2, T=4, Hg=8, Wg=8, D=256, H=2, hd=128, F=64, pairs=(22, 21, 21),
                    sigma_cache=(0.03, 0.1))
    prev, cur = W.cache_pair(wl)
    d = (cur.float() - prev.float()).reshape(2, -1)
    s = d.std(dim=1)
    assert 0.025 < s[0] < 0.04 and 0.09 < s[1] < 0.11
    rows = torch.tensor([3, 256 + 7])
    p2, c2 = W.cache_pair(wl, row_ids=rows)
    assert torch.equal(p2.view(torch.int16), prev[rows].view(torch.int16))
    assert torch.equal(c2.view(torch.int16), cur[rows].view(torch.int16))


def test_sample_rows_cover_boundaries():
    wl = W.CONFIGS["cfg_av"]
    rows = W.sample_rows(wl, 40).tolist()
    for b in range(wl.B):
        assert b * wl.N in rows and b * wl.N + wl.N - 1 in rows
    assert rows == sorted(set(rows))
