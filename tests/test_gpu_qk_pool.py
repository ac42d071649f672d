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


ROUTER_MEANS = [
    # B, N, H, hd, block, sparsity: several 128 x 256 score tiles with ragged
    # edges (tensor-core scores for hd a multiple of 32: 1 to 8 chunks
    # through the two-slot ring), and hd that takes the fp32 FMA scores (48)
    (2, 4800, 2, 128, 8, 0.75),      # 600 blocks: 5 x 3 tiles, last 88 x 88
    (1, 2016, 3, 96, 8, 0.8),        # 3 chunks of 32
    (1, 8 * 2100, 1, 32, 8, 0.75),   # 2,100 blocks: 17 x 9 tiles (selection past 2,048)
    (2, 1000, 2, 64, 16, 0.5),       # 63 blocks: one ragged tile
    (1, 3000, 2, 48, 16, 0.75),
    (1, 1500, 1, 160, 8, 0.75),      # 5 chunks
    (1, 700, 2, 256, 8, 0.75),       # 8 chunks
]


@pytest.mark.parametrize("B,N,H,hd,block,sp", ROUTER_MEANS)
def test_router_from_given_means(orc, B, N, H, hd, block, sp):
    """The router from means given directly: fp32 means of random bf16 q and
    k (exact means rounded once to fp32).  The scores the call leaves at the
    front of its workspace are checked one by one against the oracle's
    (fp64 means, fp64 sums) within the bound of the arithmetic used:
      fp32 FMA sums:      hd 2^-24 sum|q_d k_d|
      tf32 split (3 products of a high part with 10 stored bits and the
      remainder truncated to tf32): 3 2^-20 per product, plus 3 hd / 8
      tensor-core accumulations of at most 2^-23 each,
    both plus 2 2^-24 for the rounding of the means to fp32; and the kept
    lists as the router test."""
    D = H * hd
    g = torch.Generator().manual_seed(N + hd)
    x = torch.randn(B * N, 2 * D, generator=g).to(torch.bfloat16)
    xb = bits(x)
    nb = (N + block - 1) // block
    m, _, _ = _means64(xb, orc, B, N, block)                       # [B, nb, 2D]
    means = np.stack([m[:, :, :D], m[:, :, D:]], axis=1)           # [B, 2, nb, D]
    L = dbp.library()
    need = int(L.dit_subblock_means_workspace_bytes(B, N, H, hd, block))
    assert need >= B * H * nb * nb * 4
    ws = torch.full((need,), 0xFF, dtype=torch.uint8, device=DEV)
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    gm = torch.from_numpy(means.astype(np.float32)).to(DEV)
    kept = dbp.subblock_router_means(gm, N, H, block, sp, workspace=ws, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    ref, S = orc.subblock_router(xb[:, :D], xb[:, D:], B, H, hd, block, sp)
    got_s = ws[:B * H * nb * nb * 4].view(torch.float32).cpu().numpy().reshape(B, H, nb, nb)
    mq = means[:, 0].reshape(B, nb, H, hd).transpose(0, 2, 1, 3)    # [B, H, nb, hd]
    mk = means[:, 1].reshape(B, nb, H, hd).transpose(0, 2, 1, 3)
    absdot = np.einsum("bhid,bhjd->bhij", np.abs(mq), np.abs(mk))
    tc = hd % 32 == 0
    rel = (3 * 2.0 ** -20 + 3 * hd / 8 * 2.0 ** -23) if tc else hd * 2.0 ** -24
    tol = (rel + 2 * 2.0 ** -24) * absdot + 1e-30
    err = np.abs(got_s - S)
    assert np.all(err <= tol), (float((err / tol).max()), np.unravel_index(np.argmax(err / tol), err.shape))
    n_keep = ref.shape[-1]
    _check_rows(kept.cpu().numpy(), ref, S, n_keep, f"means {B}x{N}x{H}x{hd}/{block}")


def test_router_means_workspace_sizes():
    L = dbp.library()
    nb = (1000 + 15) // 16
    scores = 2 * 3 * nb * nb * 4
    assert L.dit_subblock_means_workspace_bytes(2, 1000, 3, 48, 16) == scores
    big = L.dit_subblock_means_workspace_bytes(2, 1000, 3, 64, 16)
    assert big >= scores + 2 * (2 * 2 * nb * 3 * 64 * 4)
    assert L.dit_subblock_means_workspace_bytes(2, 1000, 3, 64, 0) == 0


def test_router_scores_expired_wait_is_reported_and_the_context_survives(orc):
    """Failure path of the tensor-core score kernel: with its copy thread
    issuing nothing (test hook) every wait runs out after its 2 s bound; the
    kernel reports through the status word, frees its tensor memory and
    returns, and the router works in the same context afterwards."""
    B, N, H, hd, block = 1, 1024, 2, 64, 64
    D = H * hd
    g = torch.Generator().manual_seed(5)
    x = torch.randn(B * N, 2 * D, generator=g).to(torch.bfloat16)
    xb = bits(x)
    m, _, _ = _means64(xb, orc, B, N, block)
    gm = torch.from_numpy(np.stack([m[:, :, :D], m[:, :, D:]], axis=1).astype(np.float32)).to(DEV)
    L = dbp.library()
    need = int(L.dit_subblock_means_workspace_bytes(B, N, H, hd, block))
    ws = torch.empty(need, dtype=torch.uint8, device=DEV)
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    rc = L.dit_subblock_scores_stall_test(gm.data_ptr(), B, N, H, hd, block, ws.data_ptr(), need,
                                          st.data_ptr(), torch.cuda.current_stream().cuda_stream)
    assert rc == 0
    torch.cuda.synchronize()
    assert int(st.item()) == 1
    st.zero_()
    kept = dbp.subblock_router_means(gm, N, H, block, 0.75, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    ref, S = orc.subblock_router(xb[:, :D], xb[:, D:], B, H, hd, block, 0.75)
    _check_rows(kept.cpu().numpy(), ref, S, ref.shape[-1], "after the stall")


def test_pooled_expired_wait_is_reported_and_the_context_survives(orc):
    """Failure path of the QK operator with block means: with no copy issued
    (test hook) every wait of the copy ring runs out after its 2 s bound; the
    kernel reports through the status word and returns without touching q, k
    or the means, and the next launch in the same context is correct."""
    wl = W.Workload("stall", B=1, T=2, Hg=4, Wg=6, D=4 * 64, H=4, hd=64, F=8, pairs=(12, 10, 10))
    N, D = wl.N, wl.D
    qkv_h = W.token_rows(wl, W.S_QKV, 3 * D)
    wq, wk = W.norm_weights(wl)
    x = qkv_h.to(DEV).view(1, N, 3 * D)
    before = x.clone()
    means = torch.full((1, 2, (N + 15) // 16, D), 7.0, dtype=torch.float32, device=DEV)
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    L = dbp.library()
    wqg, wkg = wq.to(DEV), wk.to(DEV)
    rc = L.dit_qk_rmsnorm_rope3d_pooled_stall_test(
        x.data_ptr(), x.data_ptr() + 2 * D, 3 * D, wqg.data_ptr(), wkg.data_ptr(), 0, 1, N,
        wl.H, wl.hd, wl.T, wl.Hg, wl.Wg, None, 0, *wl.pairs, wl.theta, wl.eps, 0, 16,
        means.data_ptr(), st.data_ptr(), torch.cuda.current_stream().cuda_stream)
    assert rc == 0
    torch.cuda.synchronize()
    assert int(st.item()) == 1
    assert torch.equal(x.view(torch.int16), before.view(torch.int16))
    assert bool((means == 7.0).all())
    st.zero_()
    dbp.qk_rmsnorm_rope3d(x[:, :, :D], x[:, :, D:2 * D], wqg, wkg, wl.H, wl.pairs,
                          grid=(wl.T, wl.Hg, wl.Wg), theta=wl.theta, eps=wl.eps,
                          block_means=means, block=16, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    hb = bits(qkv_h)
    p = np.ascontiguousarray(orc.grid_positions(wl.T, wl.Hg, wl.Wg, 0, N).reshape(-1, 3))
    ref = orc.qk_rmsnorm_rope3d_ex(hb[:, :D], wq.double().numpy(), wl.H, wl.hd, p, wl.pairs,
                                   wl.theta, wl.eps, layout=0)
    compare_bf16(bits(x.view(N, 3 * D))[:, :D], ref, "q after the stall")
