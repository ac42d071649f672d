"""The SubBlock router on the GPU against the oracle.  Scores are fp32 sums
on the GPU (three tf32 products of split means on the tensor cores for hd a
multiple of 32, fp32 FMAs otherwise) and fp64 in the oracle, so where two key
blocks' scores lie within the fp32 error of the selection threshold either may
be kept: the test checks that the kept list is valid (n_keep distinct
increasing indices) and agrees with the oracle's everywhere else.  The bound:
the block means sum at most `block` bf16 values in fp32, and a score carries
at most about (3 hd / 8) 2^-23 + 3 2^-20 of sum|q_d k_d| (the split-tf32 bound
checked score by score in test_gpu_qk_pool.py); tau = 2^-14 max_j |score_ij|
covers both with a wide margin."""
import numpy as np
import pytest
import torch

import dit_block_pass_b200 as dbp
from dit_block_pass_b200 import workloads as W
from parity import bits

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


@pytest.fixture(scope="module", autouse=True)
def _built():
    from dit_block_pass_b200 import build
    build.build()


def _check_rows(got, ref, S, n_keep, what):
    """got, ref: [..., n_keep] kept lists; S: [..., n_blocks] fp64 scores."""
    nb = S.shape[-1]
    got = got.reshape(-1, n_keep)
    ref = ref.reshape(-1, n_keep)
    S = S.reshape(-1, nb)
    differ = 0
    for r in range(got.shape[0]):
        g = got[r]
        assert np.all(np.diff(g) > 0) and g[0] >= 0 and g[-1] < nb, (what, r, g)
        tau = 2.0 ** -14 * np.abs(S[r]).max()
        thr = np.sort(S[r])[::-1][n_keep - 1]
        drop = np.setdiff1d(np.arange(nb), g)
        assert S[r, g].min() >= thr - tau, (what, r)
        if drop.size:
            assert S[r, drop].max() <= thr + tau, (what, r)
        sym = np.setxor1d(g, ref[r])
        assert np.all(np.abs(S[r, sym] - thr) <= tau), (what, r, sym)
        differ += sym.size > 0
    return differ


def _qkv(B, N, H, hd, seed):
    g = torch.Generator().manual_seed(seed)
    D = H * hd
    return torch.randn(B, N, 3 * D, generator=g).to(torch.bfloat16)


@pytest.mark.parametrize("B,N,H,hd,block,sp", [(2, 1000, 3, 64, 128, 0.75), (1, 8192, 4, 128, 128, 0.8),
                                               (2, 77, 2, 32, 16, 0.5), (1, 3000, 2, 128, 64, 0.0),
                                               (1, 4096 * 3 + 5, 2, 64, 8, 0.75),
                                               (1, 8 * 2100, 1, 32, 8, 0.75),
                                               (2, 1000, 3, 40, 16, 0.75),    # fp32 FMA scores
                                               (1, 1500, 2, 256, 8, 0.8)])    # 8 tf32 chunks
def test_router_matches_oracle(orc, B, N, H, hd, block, sp):
    qkv = _qkv(B, N, H, hd, N + H)
    D = H * hd
    g = qkv.to(DEV)
    kept = dbp.subblock_router(g[:, :, :D], g[:, :, D:2 * D], H, block, sp)
    torch.cuda.synchronize()
    flat = bits(qkv.view(B * N, 3 * D))
    ref, S = orc.subblock_router(flat[:, :D], flat[:, D:2 * D], B, H, hd, block, sp)
    n_keep = ref.shape[-1]
    assert kept.shape == ref.shape
    differ = _check_rows(kept.cpu().numpy(), ref, S, n_keep, f"{B}x{N}x{H}x{hd}/{block}")
    assert differ <= max(1, ref.size // n_keep // 100)       # near-ties are rare


def test_router_full_size_sampled_heads(orc):
    """h3_5s: 124,992 tokens, 40 heads x 128, blocks of 128 (977 blocks),
    sparsity 0.75 and 0.8; the oracle on two heads."""
    wl = W.CONFIGS["h3_5s"]
    N, H, hd, D = wl.N, wl.H, wl.hd, wl.D
    qkv = W.token_rows(wl, W.S_QKV, 3 * D, device=DEV).view(1, N, 3 * D)
    for sp in (0.75, 0.8):
        kept = dbp.subblock_router(qkv[:, :, :D], qkv[:, :, D:2 * D], H, 128, sp).cpu().numpy()
        for h in (0, 37):
            q = bits(qkv[0, :, h * hd:(h + 1) * hd])
            k = bits(qkv[0, :, D + h * hd:D + (h + 1) * hd])
            ref, S = orc.subblock_router(q, k, 1, 1, hd, 128, sp)
            n_keep = ref.shape[-1]
            assert n_keep == (245 if sp == 0.75 else 196)
            _check_rows(kept[0, h], ref[0, 0], S[0, 0], n_keep, f"h3 head {h} s={sp}")


def test_router_empty_and_errors():
    q = torch.zeros(1, 0, 128, dtype=torch.bfloat16, device=DEV)
    assert dbp.subblock_router(q, q, 2, 128, 0.75).shape == (1, 2, 0, 0)
    q = torch.zeros(1, 256, 128, dtype=torch.bfloat16, device=DEV)
    with pytest.raises(ValueError):
        dbp.subblock_router(q, q, 2, 128, 1.0)
    with pytest.raises(dbp.DitError):                       # hd = 12: not a multiple of 8
        dbp.subblock_router(q[:, :, :120], q[:, :, :120], 10, 128, 0.5)
