"""Full-size parity at the H3-shaped workloads (5 s clip, 10 s clip, CFG pair
with joint audio), in the launch configuration the benchmark times.

Inputs are generated on the device by the seeded generator; a sample of rows
(always including every sample's first and last token) is regenerated on the
host and must match bit for bit, and the oracle runs on those host rows.  The
Cache-DiT check is compared on the whole tensors: its sums cover every
element.
"""
import numpy as np
import pytest
import torch

import dit_block_pass_b200 as dbp
from dit_block_pass_b200 import workloads as W
from parity import bits, compare_bf16

pytestmark = pytest.mark.gpu

DEV = "cuda:0"
SAMPLE = 96


@pytest.fixture(scope="module", autouse=True)
def _built():
    from dit_block_pass_b200 import build
    build.build()


def _free():
    torch.cuda.synchronize()
    torch.cuda.empty_cache()


def _same_rows(dev_rows: torch.Tensor, host_rows: torch.Tensor):
    assert np.array_equal(bits(dev_rows), bits(host_rows)), "device generator != host generator"


@pytest.mark.parametrize("name", ["h3_5s", "cfg_av", "h3_10s"])
def test_fullsize_adaln_and_gated(orc, name):
    wl = W.CONFIGS[name]
    B, N, D, M = wl.B, wl.N, wl.D, wl.M
    rows = W.sample_rows(wl, SAMPLE)
    mod = W.modulation(wl, device=DEV)
    modh = mod.cpu().double().numpy()
    x = W.token_rows(wl, W.S_X, D, device=DEV)
    xh = W.token_rows(wl, W.S_X, D, row_ids=rows)
    _same_rows(x[rows.to(DEV)], xh)
    y = dbp.adaln_modulate(x.view(B, N, D), mod[:, 0], mod[:, 1], wl.eps)
    ysel = bits(y.view(M, D)[rows.to(DEV)])
    del y
    r = W.token_rows(wl, W.S_R, D, device=DEV)
    rh = W.token_rows(wl, W.S_R, D, row_ids=rows)
    xo, y2 = dbp.gated_residual_adaln(x.view(B, N, D), r.view(B, N, D), mod[:, 2], mod[:, 3],
                                      mod[:, 4], wl.eps)
    xosel = bits(xo.view(M, D)[rows.to(DEV)])
    y2sel = bits(y2.view(M, D)[rows.to(DEV)])
    del x, r, xo, y2
    _free()
    samp = (rows // N).numpy()
    for b in range(B):
        sel = samp == b
        if not sel.any():
            continue
        xb = bits(xh[torch.from_numpy(sel)]).reshape(1, -1, D)
        rb = bits(rh[torch.from_numpy(sel)]).reshape(1, -1, D)
        ref = orc.adaln_modulate(xb, modh[b:b + 1, 0], modh[b:b + 1, 1], wl.eps)
        compare_bf16(ysel[sel], ref, f"{name} adaln sample {b}")
        rx, ry = orc.gated_residual_adaln(xb, rb, modh[b:b + 1, 2], modh[b:b + 1, 3],
                                          modh[b:b + 1, 4], wl.eps)
        assert np.array_equal(xosel[sel].reshape(-1), rx.reshape(-1))
        compare_bf16(y2sel[sel], ry, f"{name} gated sample {b}")


@pytest.mark.parametrize("name", ["h3_5s", "cfg_av", "h3_10s"])
def test_fullsize_swiglu(orc, name):
    wl = W.CONFIGS[name]
    rows = W.sample_rows(wl, SAMPLE)
    inp = W.token_rows(wl, W.S_SWIGLU, 2 * wl.F, device=DEV)
    out = dbp.swiglu(inp)
    inh = W.token_rows(wl, W.S_SWIGLU, 2 * wl.F, row_ids=rows)
    _same_rows(inp[rows.to(DEV)], inh)
    sel = bits(out[rows.to(DEV)])
    del inp, out
    _free()
    compare_bf16(sel, orc.swiglu(bits(inh)), f"{name} swiglu")


@pytest.mark.parametrize("name", ["h3_5s", "cfg_av", "h3_10s"])
def test_fullsize_qk_rope(orc, name):
    wl = W.CONFIGS[name]
    B, N, D, M = wl.B, wl.N, wl.D, wl.M
    rows = W.sample_rows(wl, SAMPLE)
    qkv = W.token_rows(wl, W.S_QKV, 3 * D, device=DEV)
    qh = W.token_rows(wl, W.S_QKV, 3 * D, row_ids=rows)
    _same_rows(qkv[rows.to(DEV)], qh)
    wq, wk = W.norm_weights(wl, device=DEV)
    v3 = qkv.view(B, N, 3 * D)
    pos = W.positions(wl, device=DEV)
    dbp.qk_rmsnorm_rope3d(v3[:, :, :D], v3[:, :, D:2 * D], wq, wk, wl.H, wl.pairs,
                          grid=None if pos is not None else (wl.T, wl.Hg, wl.Wg), pos=pos,
                          theta=wl.theta, eps=wl.eps)
    sel = bits(qkv[rows.to(DEV)])
    del qkv, v3
    _free()
    if pos is not None:
        p = pos.cpu().numpy()[rows.numpy()]
    else:
        p = orc.grid_positions(wl.T, wl.Hg, wl.Wg, 0, N)[(rows % N).numpy()]
    hb = bits(qh)
    rq = orc.qk_rmsnorm_rope3d(hb[:, :D], wq.cpu().double().numpy(), wl.H, wl.hd, p, wl.pairs,
                               wl.theta, wl.eps)
    rk = orc.qk_rmsnorm_rope3d(hb[:, D:2 * D], wk.cpu().double().numpy(), wl.H, wl.hd, p,
                               wl.pairs, wl.theta, wl.eps)
    compare_bf16(sel[:, :D], rq, f"{name} q")
    compare_bf16(sel[:, D:2 * D], rk, f"{name} k")
    assert np.array_equal(sel[:, 2 * D:], hb[:, 2 * D:]), "v changed"


@pytest.mark.parametrize("layout", [dbp.ROPE_INTERLEAVED, dbp.ROPE_HALF])
@pytest.mark.parametrize("name", ["h3_5s", "cfg_av"])
def test_fullsize_qk_whole_row_norm(orc, name, layout):
    """The whole-row norm options at full size (the persistent row kernel,
    as the benchmark times it), sampled rows against the oracle."""
    wl = W.CONFIGS[name]
    B, N, D, M = wl.B, wl.N, wl.D, wl.M
    rows = W.sample_rows(wl, SAMPLE)
    qkv = W.token_rows(wl, W.S_QKV, 3 * D, device=DEV)
    qh = W.token_rows(wl, W.S_QKV, 3 * D, row_ids=rows)
    _same_rows(qkv[rows.to(DEV)], qh)
    wq, wk = W.row_norm_weights(wl, device=DEV)
    v3 = qkv.view(B, N, 3 * D)
    pos = W.positions(wl, device=DEV)
    dbp.qk_rmsnorm_rope3d(v3[:, :, :D], v3[:, :, D:2 * D], wq, wk, wl.H, wl.pairs,
                          grid=None if pos is not None else (wl.T, wl.Hg, wl.Wg), pos=pos,
                          theta=wl.theta, eps=wl.eps, rope_layout=layout,
                          norm_width=dbp.NORM_ROW)
    sel = bits(qkv[rows.to(DEV)])
    del qkv, v3
    _free()
    if pos is not None:
        p = pos.cpu().numpy()[rows.numpy()]
    else:
        p = orc.grid_positions(wl.T, wl.Hg, wl.Wg, 0, N)[(rows % N).numpy()]
    hb = bits(qh)
    for t, w in ((0, wq), (1, wk)):
        ref = orc.qk_rmsnorm_rope3d_ex(hb[:, t * D:(t + 1) * D], w.cpu().double().numpy(), wl.H,
                                       wl.hd, np.ascontiguousarray(p), wl.pairs, wl.theta, wl.eps,
                                       layout=layout, norm=dbp.NORM_ROW)
        compare_bf16(sel[:, t * D:(t + 1) * D], ref, f"{name} {'qk'[t]} layout {layout}")
    assert np.array_equal(sel[:, 2 * D:], hb[:, 2 * D:]), "v changed"


def test_fullsize_qk_means_then_router(orc):
    """h3_5s: the QK operator with block means, then the router from those
    means (tensor-core scores, 977 blocks), against the oracle router on the
    kernel's own q and k for two heads (within the fp32 tie band)."""
    from test_gpu_subblock import _check_rows
    wl = W.CONFIGS["h3_5s"]
    N, D, H, hd = wl.N, wl.D, wl.H, wl.hd
    qkv = W.token_rows(wl, W.S_QKV, 3 * D, device=DEV).view(1, N, 3 * D)
    wq, wk = W.norm_weights(wl, device=DEV)
    nb = (N + 127) // 128
    means = torch.empty(1, 2, nb, D, dtype=torch.float32, device=DEV)
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    dbp.qk_rmsnorm_rope3d(qkv[:, :, :D], qkv[:, :, D:2 * D], wq, wk, H, wl.pairs,
                          grid=(wl.T, wl.Hg, wl.Wg), theta=wl.theta, eps=wl.eps,
                          block_means=means, block=128, status=st)
    kept = dbp.subblock_router_means(means, N, H, 128, 0.75, status=st).cpu().numpy()
    assert int(st.item()) == 0
    for h in (0, 29):
        q = bits(qkv[0, :, h * hd:(h + 1) * hd])
        k = bits(qkv[0, :, D + h * hd:D + (h + 1) * hd])
        ref, S = orc.subblock_router(q, k, 1, 1, hd, 128, 0.75)
        assert ref.shape[-1] == 245
        _check_rows(kept[0, h], ref[0, 0], S[0, 0], 245, f"h3 means head {h}")
    del qkv, means
    _free()


@pytest.mark.parametrize("name", ["h3_5s", "h3_10s", "cfg_av"])
def test_fullsize_cachedit(orc, name):
    wl = W.CONFIGS[name]
    B, N, D = wl.B, wl.N, wl.D
    rows = W.sample_rows(wl, SAMPLE)
    prev, cur = W.cache_pair(wl, device=DEV)
    ph, chh = W.cache_pair(wl, row_ids=rows)
    _same_rows(prev[rows.to(DEV)], ph)
    _same_rows(cur[rows.to(DEV)], chh)
    pb, cb = bits(prev).reshape(B, N, D), bits(cur).reshape(B, N, D)
    for thr in wl.thresholds:
        rel, reuse = dbp.cachedit_residual_diff(prev.view(B, N, D), cur.view(B, N, D), thr)
        ref_rel, ref_reuse = orc.cachedit_residual_diff(pb, cb, thr)
        rel, reuse = rel.cpu().numpy(), reuse.cpu().numpy()
        assert np.allclose(rel, ref_rel, rtol=1e-7, atol=0), (rel, ref_rel)
        assert np.all(np.abs(ref_rel - thr) > 1e-4), "decision margin too small to be meaningful"
        assert np.array_equal(reuse, ref_reuse), (rel, ref_rel, thr)
    del prev, cur
    _free()
