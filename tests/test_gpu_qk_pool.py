"""QK RMSNorm + 3D RoPE with the SubBlock block means fused in, then the
router from those means, on the GPU against the oracle.

Three checks per case:
  * q and k are the QK operator's results (the oracle, the parity rule);
  * each block mean is the mean of the kernel's own bf16 results within the
    bound of an fp32 sum: |err| <= (n-1) 2^-24 sum|x| / n + 2^-24 |mean|
    (recursive summation of n terms, one correctly rounded divide);
  * the kept lists from the means equal the oracle router's on the kernel's
    q and k except where two scores lie within the fp32 tie band of the
    threshold (as the router test), and agree with the oracle's QK followed
    by the oracle's router within that band widened by the largest score
    difference the two QK results cause.
"""
import numpy as np
import pytest
import torch

import dit_block_pass_b200 as dbp
from dit_block_pass_b200 import workloads as W
from parity import bits, compare_bf16
from test_gpu_subblock import _check_rows

pytestmark = pytest.mark.gpu
DEV = "cuda:0"
U = 2.0 ** -24


@pytest.fixture(scope="module", autouse=True)
def _built():
    from dit_block_pass_b200 import build
    build.build()


def _means64(x_bits, orc, B, N, block):
    """Exact block means (fp64) and sums of |x| of bf16 rows [B*N, D]."""
    x = orc.bf16_to_f64(x_bits).reshape(B, N, -1)
    nb = (N + block - 1) // block
    m = np.empty((B, nb, x.shape[-1]))
    a = np.empty_like(m)
    cnt = np.empty(nb)
    for j in range(nb):
        seg = x[:, j * block:(j + 1) * block]
        cnt[j] = seg.shape[1]
        m[:, j] = seg.sum(axis=1) / cnt[j]
        a[:, j] = np.abs(seg).sum(axis=1)
    return m, a, cnt


CASES = [
    # name, B, T, Hg, Wg, H, hd, block, layout, sparsity, audio tokens
    ("tiny-grid", 1, 2, 4, 6, 4, 64, 16, 0, 0.75, 0),
    ("ragged", 2, 3, 5, 7, 3, 128, 32, 0, 0.5, 0),       # 105 tokens: last block of 9
    ("rotate-half", 1, 4, 8, 10, 5, 128, 64, 1, 0.8, 0),
    ("hd32", 1, 2, 6, 9, 6, 32, 8, 0, 0.75, 0),
    ("audio", 2, 2, 4, 6, 2, 128, 16, 0, 0.75, 10),      # explicit positions
    ("h3-shape", 1, 2, 24, 42, 40, 128, 128, 0, 0.75, 0),  # 2,016 tokens, 16 blocks
]


@pytest.mark.parametrize("name,B,T,Hg,Wg,H,hd,block,layout,sp,audio", CASES)
def test_qk_pooled_then_router(orc, name, B, T, Hg, Wg, H, hd, block, layout, sp, audio):
    pairs = {32: (6, 5, 5), 64: (12, 10, 10), 128: (22, 21, 21)}[hd]
    wl = W.Workload(name, B=B, T=T, Hg=Hg, Wg=Wg, D=H * hd, H=H, hd=hd, F=8, pairs=pairs,
                    n_audio=audio, seed=11)
    N, D = wl.N, wl.D
    qkv_h = W.token_rows(wl, W.S_QKV, 3 * D)
    wq, wk = W.norm_weights(wl)
    pos = W.positions(wl)
    qkv = qkv_h.to(DEV).view(B, N, 3 * D)
    nb = (N + block - 1) // block
    means = torch.full((B, 2, nb, D), float("nan"), dtype=torch.float32, device=DEV)
    grid = None if pos is not None else (T, Hg, Wg)
    dbp.qk_rmsnorm_rope3d(qkv[:, :, :D], qkv[:, :, D:2 * D], wq.to(DEV), wk.to(DEV), H, pairs,
                          grid=grid, pos=None if pos is None else pos.to(DEV),
                          theta=wl.theta, eps=wl.eps, rope_layout=layout,
                          block_means=means, block=block)
    kept = dbp.subblock_router_means(means, N, H, block, sp)
    torch.cuda.synchronize()
    got = bits(qkv.view(B * N, 3 * D))
    hb = bits(qkv_h)
    p = pos.numpy() if pos is not None else orc.grid_positions(T, Hg, Wg, 0, N)
    p = np.ascontiguousarray(np.tile(p.reshape(-1, 3), (B if pos is None else 1, 1)))
    # 1. q and k: the QK operator
    ref = {}
    for t, w in ((0, wq), (1, wk)):
        ref[t] = orc.qk_rmsnorm_rope3d_ex(hb[:, t * D:(t + 1) * D], w.double().numpy(), H, hd, p,
                                          pairs, wl.theta, wl.eps, layout=layout)
        compare_bf16(got[:, t * D:(t + 1) * D], ref[t], f"{name} {'qk'[t]}")
    assert np.array_equal(got[:, 2 * D:], hb[:, 2 * D:]), "v changed"
    # 2. the means of the kernel's own results
    gm = means.cpu().numpy()
    for t in (0, 1):
        m, a, cnt = _means64(got[:, t * D:(t + 1) * D], orc, B, N, block)
        tol = 1.01 * ((cnt[None, :, None] - 1) * U * a / cnt[None, :, None] + U * np.abs(m)) + 1e-30
        err = np.abs(gm[:, t].astype(np.float64) - m)
        assert np.all(err <= tol), (name, t, float((err / tol).max()))
    # 3. the kept lists
    kept = kept.cpu().numpy()
    own, S_own = orc.subblock_router(got[:, :D], got[:, D:2 * D], B, H, hd, block, sp)
    n_keep = own.shape[-1]
    assert kept.shape == own.shape
    _check_rows(kept, own, S_own, n_keep, f"{name} vs router on the kernel's q, k")
    r_bits = {t: orc.f64_to_bf16(ref[t]).reshape(B * N, D) for t in (0, 1)}
    chain, S_chain = orc.subblock_router(r_bits[0], r_bits[1], B, H, hd, block, sp)
    delta = np.abs(S_own - S_chain).max(axis=-1, keepdims=True)
    _check_rows_band(kept, chain, S_chain, n_keep, delta, f"{name} vs oracle QK + router")


def _check_rows_band(got, ref, S, n_keep, delta, what):
    """As _check_rows, with the tie band widened per row by delta (the
    largest score difference between the two QK results)."""
    nb = S.shape[-1]
    got = got.reshape(-1, n_keep)
    ref = ref.reshape(-1, n_keep)
    S = S.reshape(-1, nb)
    delta = delta.reshape(-1)
    for r in range(got.shape[0]):
        g = got[r]
        assert np.all(np.diff(g) > 0) and g[0] >= 0 and g[-1] < nb, (what, r, g)
        tau = 2.0 ** -14 * np.abs(S[r]).max() + 2.0 * delta[r]
        thr = np.sort(S[r])[::-1][n_keep - 1]
        sym = np.setxor1d(g, ref[r])
        assert np.all(np.abs(S[r, sym] - thr) <= tau), (what, r, sym)


def test_pooled_means_repeat_bit_for_bit():
    """Fixed summation order: the same inputs give the same means."""
    wl = W.Workload("rep", B=1, T=3, Hg=24, Wg=42, D=5120, H=40, hd=128, F=8,
                    pairs=(22, 21, 21))
    N, D = wl.N, wl.D
    base = W.token_rows(wl, W.S_QKV, 2 * D, device=DEV).view(1, N, 2 * D)
    wq, wk = W.norm_weights(wl, device=DEV)
    outs = []
    for _ in range(2):
        x = base.clone()
        m = torch.empty(1, 2, (N + 127) // 128, D, dtype=torch.float32, device=DEV)
        dbp.qk_rmsnorm_rope3d(x[:, :, :D], x[:, :, D:], wq, wk, wl.H, wl.pairs,
                              grid=(wl.T, wl.Hg, wl.Wg), block_means=m)
        outs.append((x, m))
    assert torch.equal(outs[0][0], outs[1][0])
    assert torch.equal(outs[0][1].view(torch.int32), outs[1][1].view(torch.int32))


def test_pooled_argument_errors():
    x = torch.zeros(1, 64, 256, dtype=torch.bfloat16, device=DEV)
    w = torch.ones(64, dtype=torch.float32, device=DEV)
    m = torch.empty(1, 2, 4, 128, dtype=torch.float32, device=DEV)
    with pytest.raises(ValueError):            # wrong means shape
        dbp.qk_rmsnorm_rope3d(x[:, :, :128], x[:, :, 128:], w, w, 2, (12, 10, 10),
                              grid=(1, 8, 8), block_means=m[:, :, :3], block=16)
    with pytest.raises(ValueError):            # whole-row norm is not offered with means
        dbp.qk_rmsnorm_rope3d(x[:, :, :128], x[:, :, 128:], w, w, 2, (12, 10, 10),
                              grid=(1, 8, 8), block_means=m, block=16,
                              norm_width=dbp.NORM_ROW)
    L = dbp.library()
    A = x.data_ptr()
    f = L.dit_qk_rmsnorm_rope3d_pooled
    # block 0, k NULL, means overlapping q
    assert f(A, A + 256, 256, w.data_ptr(), w.data_ptr(), 0, 1, 64, 2, 64, 1, 8, 8, None, 0, 12,
             10, 10, 1e4, 1e-6, 0, 0, m.data_ptr(), None, None) == -2
    assert f(A, None, 256, w.data_ptr(), w.data_ptr(), 0, 1, 64, 2, 64, 1, 8, 8, None, 0, 12,
             10, 10, 1e4, 1e-6, 0, 16, m.data_ptr(), None, None) == -1
    assert f(A, A + 256, 256, w.data_ptr(), w.data_ptr(), 0, 1, 64, 2, 64, 1, 8, 8, None, 0, 12,
             10, 10, 1e4, 1e-6, 0, 16, A, None, None) == -7
