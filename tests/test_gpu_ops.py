"""CUDA path vs the fp64 oracle, element by element, through the C ABI.

Sizes: the tiny and small H3-shaped workloads (all elements), ragged shapes
(rows that are not a multiple of the warp width, odd token counts, several
samples), the largest supported widths and head sizes, and the degenerate
cases (empty inputs, constant rows, zero gates, identical residuals).
Every output buffer is guarded by canary padding on both sides.
"""
import numpy as np
import pytest
import torch

import dit_block_pass_b200 as dbp
from dit_block_pass_b200 import workloads as W
from parity import bits, compare_bf16

pytestmark = pytest.mark.gpu

DEV = "cuda:0"
CANARY = -12345.0


@pytest.fixture(scope="module", autouse=True)
def _built():
    from dit_block_pass_b200 import build
    build.build()
    assert torch.cuda.is_available()


def guarded(shape, dtype=torch.bfloat16, pad=64):
    n = int(np.prod(shape))
    buf = torch.full((pad + n + pad,), CANARY, dtype=dtype, device=DEV)
    view = buf[pad:pad + n].view(*shape)

    def check():
        head, tail = buf[:pad], buf[pad + n:]
        assert torch.all(head == CANARY) and torch.all(tail == CANARY), "write outside the output"
    return view, check


def rows(wl, stream, width):
    return W.token_rows(wl, stream, width)


def ragged(B=3, N=37, D=264, H=3, hd=64, pairs=(12, 10, 10)):
    return W.Workload("ragged", B=B, T=1, Hg=1, Wg=N, D=D, H=H, hd=hd, F=D, pairs=pairs,
                      sigma_cache=(0.03, 0.05, 0.1))


# ------------------------------------------------------------------ AdaLN

ADALN_CASES = ["tiny", "small", "ragged", "wide8192", "narrow8", "twosamples"]


def _adaln_wl(name):
    if name in W.CONFIGS:
        return W.CONFIGS[name]
    return {"ragged": ragged(), "wide8192": ragged(B=1, N=9, D=8192),
            "narrow8": ragged(B=2, N=5, D=8), "twosamples": ragged(B=2, N=300, D=5120)}[name]


@pytest.mark.parametrize("name", ADALN_CASES)
@pytest.mark.parametrize("mod_dtype", [torch.float32, torch.bfloat16])
def test_adaln_modulate(orc, name, mod_dtype):
    wl = _adaln_wl(name)
    B, N, D = wl.B, wl.N, wl.D
    x = rows(wl, W.S_X, D).view(B, N, D)
    mod = W.modulation(wl).to(mod_dtype)
    ref = orc.adaln_modulate(bits(x), mod[:, 0].double().numpy(), mod[:, 1].double().numpy(),
                             wl.eps)
    modg = mod.to(DEV)
    y, check = guarded((B, N, D))
    dbp.adaln_modulate(x.to(DEV), modg[:, 0], modg[:, 1], wl.eps, out=y)
    torch.cuda.synchronize()
    check()
    compare_bf16(bits(y), ref, f"adaln {name}")


def test_adaln_in_place_and_broadcast_modulation(orc):
    wl = ragged(B=2, N=50, D=1024)
    x = rows(wl, W.S_X, wl.D).view(2, 50, 1024)
    shift = W.normal(0, 77, 1, 1024, sigma=0.1, dtype=torch.float32)
    scale = W.normal(0, 78, 1, 1024, sigma=0.1, dtype=torch.float32)
    ref = orc.adaln_modulate(bits(x), np.repeat(shift.double().numpy(), 2, 0),
                             np.repeat(scale.double().numpy(), 2, 0), 1e-6)
    xg = x.to(DEV)
    dbp.adaln_modulate(xg, shift[0].to(DEV), scale[0].to(DEV), 1e-6, out=xg)  # [D] broadcast
    compare_bf16(bits(xg), ref, "adaln in place")


def test_adaln_degenerate_rows(orc):
    """Constant rows: with eps > 0 the output is the shift; with eps = 0 it
    is 0/0 = NaN on both sides.  scale = -1 gives the shift exactly."""
    D = 256
    x = torch.ones(1, 3, D, dtype=torch.bfloat16) * 1.5
    shift = W.normal(0, 5, 1, D, sigma=0.1, dtype=torch.float32)
    scale = W.normal(0, 6, 1, D, sigma=0.1, dtype=torch.float32)
    for eps in (1e-6, 0.0):
        ref = orc.adaln_modulate(bits(x), shift.double().numpy(), scale.double().numpy(), eps)
        y = dbp.adaln_modulate(x.to(DEV), shift.to(DEV), scale.to(DEV), eps)
        compare_bf16(bits(y), ref, f"constant rows eps={eps}")
    xr = W.normal(0, 7, 4, D).view(1, 4, D)
    y = dbp.adaln_modulate(xr.to(DEV), shift.to(DEV), -torch.ones(1, D, device=DEV), 1e-6)
    assert torch.equal(y.float().cpu(), shift.to(torch.bfloat16).float().expand(1, 4, D))


def test_adaln_empty():
    x = torch.empty(1, 0, 256, dtype=torch.bfloat16, device=DEV)
    y = dbp.adaln_modulate(x, torch.zeros(1, 256, device=DEV), torch.zeros(1, 256, device=DEV))
    assert y.shape == (1, 0, 256)


# --------------------------------------------------------- gated residual


@pytest.mark.parametrize("name", ADALN_CASES)
def test_gated_residual_adaln(orc, name):
    wl = _adaln_wl(name)
    B, N, D = wl.B, wl.N, wl.D
    x = rows(wl, W.S_X, D).view(B, N, D)
    r = rows(wl, W.S_R, D).view(B, N, D)
    mod = W.modulation(wl)
    g, sh, sc = (mod[:, i].double().numpy() for i in (2, 3, 4))
    ref_x, ref_y = orc.gated_residual_adaln(bits(x), bits(r), g, sh, sc, wl.eps)
    modg = mod.to(DEV)
    xo, c1 = guarded((B, N, D))
    y, c2 = guarded((B, N, D))
    dbp.gated_residual_adaln(x.to(DEV), r.to(DEV), modg[:, 2], modg[:, 3], modg[:, 4], wl.eps,
                             x_out=xo, y=y)
    torch.cuda.synchronize()
    c1()
    c2()
    # the new residual is bit-exact: one rounding of the exact x + gate*r
    assert np.array_equal(bits(xo).reshape(-1), ref_x.reshape(-1)), "x' not bit-exact"
    compare_bf16(bits(y), ref_y, f"gated y {name}")


def test_gated_residual_ties_and_in_place(orc):
    """Inputs built so that many x + g*r land exactly on bf16 rounding ties
    (and just beside them): the residual must still round once, to even."""
    D, N = 512, 40
    gen = torch.Generator().manual_seed(3)
    xf = torch.randint(-64, 64, (1, N, D), generator=gen).float() / 8.0 + 1.0
    rf = torch.ones(1, N, D)
    gate = (torch.randint(-8, 8, (1, D), generator=gen).float() * 2.0 ** -9)
    gate[0, ::3] += 2.0 ** -30   # just off the tie
    x, r = xf.to(torch.bfloat16), rf.to(torch.bfloat16)
    z = torch.zeros(1, D)
    ref_x, ref_y = orc.gated_residual_adaln(bits(x), bits(r), gate.double().numpy(),
                                            z.double().numpy(), z.double().numpy(), 1e-6)
    xg = x.to(DEV)
    _, y = dbp.gated_residual_adaln(xg, r.to(DEV), gate.to(DEV), z.to(DEV), z.to(DEV), 1e-6,
                                    x_out=xg)
    assert np.array_equal(bits(xg).reshape(-1), ref_x.reshape(-1))
    compare_bf16(bits(y), ref_y, "gated ties")


def test_gated_zero_gate_equals_adaln(orc):
    """gate = 0: the residual passes through bit for bit, and y is the AdaLN
    of x (both kernels within the tolerance of the oracle, and within one
    bf16 ulp of each other: they sum the row statistics in different
    orders)."""
    wl = ragged(B=2, N=30, D=640)
    x = rows(wl, W.S_X, wl.D).view(2, 30, 640)
    r = rows(wl, W.S_R, wl.D).view(2, 30, 640)
    mod = W.modulation(wl)
    mod[:, 2] = 0.0
    ref = orc.adaln_modulate(bits(x), mod[:, 3].double().numpy(), mod[:, 4].double().numpy(),
                             wl.eps)
    xg, modg = x.to(DEV), mod.to(DEV)
    xo, y = dbp.gated_residual_adaln(xg, r.to(DEV), modg[:, 2], modg[:, 3], modg[:, 4])
    y1 = dbp.adaln_modulate(xg, modg[:, 3], modg[:, 4])
    assert torch.equal(xo.view(torch.int16), xg.view(torch.int16))
    compare_bf16(bits(y), ref, "gated with zero gate")
    compare_bf16(bits(y1), ref, "adaln")
    assert compare_bf16(bits(y), orc.bf16_to_f64(bits(y1)), "gated vs adaln", max_ulps=1.0)


# ------------------------------------------- per-token modulation sets


def _fl2va_index(wl, S, seed=0):
    """Tokens of the first and last latent frames on set 1, a few random
    tokens on the other sets, the rest on set 0."""
    B, N = wl.B, wl.N
    idx = np.zeros((B, N), np.uint8)
    frame = wl.Hg * wl.Wg
    idx[:, :frame] = 1 % S
    idx[:, max(0, N - frame):] = 1 % S
    rng = np.random.default_rng(seed)
    pick = rng.random((B, N)) < 0.05
    idx[pick] = rng.integers(0, S, pick.sum())
    return idx


def _set_views(base, D, pad):
    """[B, S, D] views of the six DiT modulation vectors in a
    [B, S, 6, D + pad] buffer (pad > 0 breaks every set's 16-byte alignment)."""
    B, S = base.shape[:2]
    flat = base.reshape(B, S, 6 * (D + pad))
    return [flat[:, :, k * (D + pad):k * (D + pad) + D] for k in range(6)]


def _set_mods(wl, S, dtype, pad=0):
    B, D = wl.B, wl.D
    base = W.normal(wl.seed, 90, B * S * 6, D + pad, sigma=0.1, dtype=torch.float32)
    return base.view(B, S, 6, D + pad).to(dtype)


TOKEN_SET_CASES = [("ragged", 3, 0), ("twosamples", 3, 0), ("wide8192", 2, 0),
                   ("small", 4, 0), ("ragged", 3, 1)]


@pytest.mark.parametrize("name,S,pad", TOKEN_SET_CASES)
@pytest.mark.parametrize("mod_dtype", [torch.float32, torch.bfloat16])
def test_token_sets(orc, name, S, pad, mod_dtype):
    """AdaLN and the gated residual with a modulation set per token: first
    and last frames on their own set, scattered tokens on others."""
    wl = _adaln_wl(name)
    B, N, D = wl.B, wl.N, wl.D
    x = rows(wl, W.S_X, D).view(B, N, D)
    r = rows(wl, W.S_R, D).view(B, N, D)
    idx = _fl2va_index(wl, S)
    base = _set_mods(wl, S, mod_dtype, pad)
    m = [t.contiguous().double().numpy() for t in _set_views(base, D, pad)]
    ref_y = orc.adaln_modulate_tok(bits(x), m[0], m[1], idx, wl.eps)
    ref_xo, ref_y2 = orc.gated_residual_adaln_tok(bits(x), bits(r), m[2], m[3], m[4], idx, wl.eps)
    vg = _set_views(base.to(DEV), D, pad)
    idg = torch.from_numpy(idx).to(DEV)
    xg, rg = x.to(DEV), r.to(DEV)
    y = dbp.adaln_modulate(xg, vg[0], vg[1], wl.eps, set_index=idg)
    xo, y2 = dbp.gated_residual_adaln(xg, rg, vg[2], vg[3], vg[4], wl.eps, set_index=idg)
    torch.cuda.synchronize()
    compare_bf16(bits(y), ref_y, f"adaln sets {name}")
    assert np.array_equal(bits(xo), ref_xo), "gated x' differs"
    compare_bf16(bits(y2), ref_y2, f"gated sets {name}")
    # set 0 everywhere is the per-sample operator, bit for bit
    zero = torch.zeros_like(idg)
    y0 = dbp.adaln_modulate(xg, vg[0], vg[1], wl.eps, set_index=zero)
    y0s = dbp.adaln_modulate(xg, vg[0][:, 0], vg[1][:, 0], wl.eps)
    assert torch.equal(y0.view(torch.int16), y0s.view(torch.int16))


def test_token_set_out_of_range_gives_nan(orc):
    wl = ragged(B=2, N=40, D=512)
    B, N, D = wl.B, wl.N, wl.D
    x = rows(wl, W.S_X, D).view(B, N, D)
    r = rows(wl, W.S_R, D).view(B, N, D)
    bad = _fl2va_index(wl, 2)
    bad[1, 7] = 2
    bad[0, 0] = 255
    base = _set_mods(wl, 2, torch.float32)
    vg = _set_views(base.to(DEV), D, 0)
    badg = torch.from_numpy(bad).to(DEV)
    y = dbp.adaln_modulate(x.to(DEV), vg[0], vg[1], wl.eps, set_index=badg)
    xo, y2 = dbp.gated_residual_adaln(x.to(DEV), r.to(DEV), vg[2], vg[3], vg[4], wl.eps,
                                      set_index=badg)
    ok = torch.ones(B, N, dtype=torch.bool)
    ok[1, 7] = ok[0, 0] = False
    for t in (y, xo, y2):
        t = t.float().cpu()
        assert torch.isnan(t[~ok]).all() and not torch.isnan(t[ok]).any()
    m = [t.contiguous().double().numpy() for t in _set_views(base, D, 0)]
    ref = orc.adaln_modulate_tok(bits(x), m[0], m[1], np.where(bad < 2, bad, 0).astype(np.uint8),
                                 wl.eps)
    compare_bf16(bits(y.cpu()[ok]), ref[ok.numpy()], "valid rows")


def test_token_set_argument_errors():
    x = torch.zeros(1, 4, 64, dtype=torch.bfloat16, device=DEV)
    m = torch.zeros(1, 2, 64, device=DEV)
    with pytest.raises(ValueError):
        dbp.adaln_modulate(x, m, m, set_index=torch.zeros(1, 4, dtype=torch.int32, device=DEV))
    L = dbp.library()
    idx = torch.zeros(4, dtype=torch.uint8, device=DEV)
    y = torch.empty_like(x)
    for n_sets in (0, 256):
        assert L.dit_adaln_modulate_tok(x.data_ptr(), y.data_ptr(), m.data_ptr(), m.data_ptr(),
                                        0, 128, 64, idx.data_ptr(), n_sets, 1, 4, 64, 1e-6,
                                        None) == -2


# ------------------------------------------------------------------ SwiGLU


@pytest.mark.parametrize("name", ["tiny", "small", "ragged", "onevector", "manyrows"])
def test_swiglu(orc, name):
    if name in W.CONFIGS:
        wl = W.CONFIGS[name]
        M, F = wl.M, wl.F
        inp = rows(wl, W.S_SWIGLU, 2 * F)
    else:
        M, F = {"ragged": (37, 264), "onevector": (5, 8), "manyrows": (4099, 40)}[name]
        inp = W.normal(0, W.S_SWIGLU, M, 2 * F, sigma=3.0)
    ref = orc.swiglu(bits(inp))
    out, check = guarded((M, F))
    dbp.swiglu(inp.to(DEV), out=out)
    torch.cuda.synchronize()
    check()
    compare_bf16(bits(out), ref, f"swiglu {name}")


def test_swiglu_narrow_vectors_when_not_32_byte_aligned(orc):
    """F divisible by 16 but pointers only 16-byte aligned: the 16-byte path."""
    M, F = 333, 512
    inp = W.normal(0, 41, M, 2 * F, sigma=2.0)
    ref = orc.swiglu(bits(inp))
    ibuf = torch.zeros(M * 2 * F + 8, dtype=torch.bfloat16, device=DEV)
    ig = ibuf[8:].view(M, 2 * F)            # 16 bytes past a 256-byte boundary
    ig.copy_(inp.to(DEV))
    out, check = guarded((M, F), pad=72)    # 144-byte pad: 16 past a 32-byte boundary
    dbp.swiglu(ig, out=out)
    torch.cuda.synchronize()
    check()
    compare_bf16(bits(out), ref, "swiglu 16-byte path")


def test_swiglu_extremes(orc):
    a = torch.tensor([0.0, 1.0, -1.0, 20.0, -20.0, 80.0, -80.0, -100.0, 3e38, -3e38,
                      1e-30, -1e-30, 0.5, -0.5, 88.0, -88.0])
    b = torch.tensor([1.0, -2.0, 3.0, 0.5, 0.5, 1.0, 1.0, 1.0, 0.0, 0.0,
                      1.0, 1.0, 1e30, 1e30, 1.0, 1.0])
    inp = torch.cat([a, b]).to(torch.bfloat16).view(1, 32)
    ref = orc.swiglu(bits(inp))
    out = dbp.swiglu(inp.to(DEV))
    compare_bf16(bits(out), ref, "swiglu extremes")


def test_swiglu_empty():
    out = dbp.swiglu(torch.empty(0, 16, dtype=torch.bfloat16, device=DEV))
    assert out.shape == (0, 8)


# ----------------------------------------------------- QK RMSNorm + RoPE


def _qk_case(orc, wl, fused, which="qk", pos_mode="grid", w_dtype=torch.float32, offset=0,
             layout=dbp.ROPE_INTERLEAVED, norm=dbp.NORM_HEAD):
    B, N, H, hd = wl.B, wl.N, wl.H, wl.hd
    D = H * hd
    qkv = rows(wl, W.S_QKV, 3 * D)
    if not fused:
        q = qkv[:, :D].contiguous()
        k = qkv[:, D:2 * D].contiguous()
    wq, wk = W.norm_weights(wl) if norm == dbp.NORM_HEAD else W.row_norm_weights(wl)
    wq, wk = wq.to(w_dtype), wk.to(w_dtype)
    if pos_mode == "grid":
        pos = np.tile(orc.grid_positions(wl.T, wl.Hg, wl.Wg, offset, N), (B, 1))
    else:
        pos = W.positions(wl).numpy() if wl.explicit_positions else np.tile(
            orc.grid_positions(wl.T, wl.Hg, wl.Wg, 0, N), (B, 1))
    if layout == dbp.ROPE_INTERLEAVED and norm == dbp.NORM_HEAD:
        ref_q = orc.qk_rmsnorm_rope3d(bits(qkv[:, :D]), wq.double().numpy(), H, hd, pos,
                                      wl.pairs, wl.theta, wl.eps)
        ref_k = orc.qk_rmsnorm_rope3d(bits(qkv[:, D:2 * D]), wk.double().numpy(), H, hd, pos,
                                      wl.pairs, wl.theta, wl.eps)
    else:
        ref_q = orc.qk_rmsnorm_rope3d_ex(bits(qkv[:, :D]), wq.double().numpy(), H, hd, pos,
                                         wl.pairs, wl.theta, wl.eps, layout=layout, norm=norm)
        ref_k = orc.qk_rmsnorm_rope3d_ex(bits(qkv[:, D:2 * D]), wk.double().numpy(), H, hd, pos,
                                         wl.pairs, wl.theta, wl.eps, layout=layout, norm=norm)
    if fused:
        buf, check = guarded((B * N, 3 * D))
        buf.copy_(qkv.to(DEV))
        qg = buf.view(B, N, 3 * D)[:, :, :D]
        kg = buf.view(B, N, 3 * D)[:, :, D:2 * D]
    else:
        qg, c1 = guarded((B, N, D))
        kg, c2 = guarded((B, N, D))
        qg.copy_(q.view(B, N, D).to(DEV))
        kg.copy_(k.view(B, N, D).to(DEV))
        check = lambda: (c1(), c2())
    posg = torch.from_numpy(pos).to(DEV) if pos_mode == "explicit" else None
    dbp.qk_rmsnorm_rope3d(qg if "q" in which else None, kg if "k" in which else None,
                          wq.to(DEV), wk.to(DEV), H, wl.pairs,
                          grid=(wl.T, wl.Hg, wl.Wg) if posg is None else None, pos=posg,
                          pos_offset=offset, theta=wl.theta, eps=wl.eps, rope_layout=layout,
                          norm_width=norm)
    torch.cuda.synchronize()
    check()
    q_in = bits(qkv[:, :D])
    k_in = bits(qkv[:, D:2 * D])
    qo = bits(qg.reshape(B * N, D))
    ko = bits(kg.reshape(B * N, D))
    if "q" in which:
        compare_bf16(qo, ref_q, f"q {wl.name}")
    else:
        assert np.array_equal(qo, q_in), "q touched"
    if "k" in which:
        compare_bf16(ko, ref_k, f"k {wl.name}")
    else:
        assert np.array_equal(ko, k_in), "k touched"
    if fused:
        v_in = bits(qkv[:, 2 * D:])
        assert np.array_equal(bits(buf[:, 2 * D:]), v_in), "v touched"


@pytest.mark.parametrize("name", ["tiny", "small"])
@pytest.mark.parametrize("fused", [False, True])
def test_qk_rope(orc, name, fused):
    _qk_case(orc, W.CONFIGS[name], fused)


@pytest.mark.parametrize("hd,pairs,H", [(32, (6, 5, 5), 5), (64, (12, 10, 10), 3),
                                        (128, (22, 21, 21), 3), (256, (44, 42, 42), 2)])
def test_qk_head_dims_ragged(orc, hd, pairs, H):
    wl = W.Workload("ragged", B=2, T=3, Hg=5, Wg=7, D=H * hd, H=H, hd=hd, F=8, pairs=pairs)
    _qk_case(orc, wl, fused=True)


def test_qk_single_tensor_and_bf16_weights(orc):
    wl = W.CONFIGS["tiny"]
    _qk_case(orc, wl, fused=True, which="q", w_dtype=torch.bfloat16)
    _qk_case(orc, wl, fused=False, which="k")


def test_qk_explicit_positions_with_audio(orc):
    wl = W.Workload("av", B=2, T=3, Hg=4, Wg=5, D=256, H=2, hd=128, F=8, pairs=(22, 21, 21),
                    n_audio=23)
    _qk_case(orc, wl, fused=True, pos_mode="explicit")


def test_qk_shard_offset_matches_full(orc):
    """A sequence shard with pos_offset equals the same rows of the full run."""
    wl = W.Workload("g", B=1, T=4, Hg=6, Wg=10, D=256, H=2, hd=128, F=8, pairs=(22, 21, 21))
    N, D = wl.N, wl.D
    qkv = rows(wl, W.S_QKV, 3 * D).to(DEV)
    wq, wk = (w.to(DEV) for w in W.norm_weights(wl))
    full = qkv.clone().view(1, N, 3 * D)
    dbp.qk_rmsnorm_rope3d(full[:, :, :D], full[:, :, D:2 * D], wq, wk, 2, wl.pairs,
                          grid=(4, 6, 10))
    for a, b in ((0, 97), (97, 200), (200, 240)):
        part = qkv[a:b].clone().view(1, b - a, 3 * D)
        dbp.qk_rmsnorm_rope3d(part[:, :, :D], part[:, :, D:2 * D], wq, wk, 2, wl.pairs,
                              grid=(4, 6, 10), pos_offset=a)
        assert torch.equal(part.view(torch.int16), full[:, a:b].view(torch.int16))
    # and the shard against the oracle
    _qk_case(orc, wl, fused=True, offset=0)


OPTIONS = [(dbp.ROPE_HALF, dbp.NORM_HEAD), (dbp.ROPE_INTERLEAVED, dbp.NORM_ROW),
           (dbp.ROPE_HALF, dbp.NORM_ROW)]


@pytest.mark.parametrize("layout,norm", OPTIONS)
@pytest.mark.parametrize("name", ["tiny", "small"])
def test_qk_options(orc, name, layout, norm):
    """Rotate-half pairs and the whole-row norm against the oracle, fused qkv."""
    _qk_case(orc, W.CONFIGS[name], fused=True, layout=layout, norm=norm)


@pytest.mark.parametrize("layout,norm", OPTIONS)
@pytest.mark.parametrize("hd,pairs,H", [(32, (6, 5, 5), 5), (64, (12, 10, 10), 3),
                                        (128, (22, 21, 21), 3), (256, (44, 42, 42), 2),
                                        (128, (22, 21, 21), 40)])
def test_qk_options_head_dims_ragged(orc, hd, pairs, H, layout, norm):
    """Every head size; widths that leave a ragged last lane-vector pass,
    up to 5120 (H=40), where the row kernel holds 20 vectors a lane."""
    wl = W.Workload("ragged", B=2, T=3, Hg=5, Wg=7, D=H * hd, H=H, hd=hd, F=8, pairs=pairs)
    _qk_case(orc, wl, fused=True, layout=layout, norm=norm)


@pytest.mark.parametrize("layout,norm", OPTIONS)
def test_qk_options_single_tensor_separate_buffers_bf16_weights(orc, layout, norm):
    wl = W.CONFIGS["tiny"]
    _qk_case(orc, wl, fused=False, which="k", w_dtype=torch.bfloat16, layout=layout, norm=norm)
    _qk_case(orc, wl, fused=False, which="q", layout=layout, norm=norm, pos_mode="explicit")


@pytest.mark.parametrize("layout,norm", [(dbp.ROPE_INTERLEAVED, dbp.NORM_HEAD)] + OPTIONS)
@pytest.mark.parametrize("order", ["head_major", "token_major"])
def test_qk_separate_outputs(orc, layout, norm, order):
    """Results written to separate q/k buffers ([B, H, N, hd] for attention,
    or [B, N, H, hd]) equal the oracle; the fused qkv input stays as it was."""
    wl = W.Workload("o", B=2, T=3, Hg=5, Wg=7, D=3 * 128, H=3, hd=128, F=8, pairs=(22, 21, 21))
    B, N, H, hd, D = wl.B, wl.N, wl.H, wl.hd, wl.D
    qkv = rows(wl, W.S_QKV, 3 * D)
    wq, wk = W.norm_weights(wl) if norm == dbp.NORM_HEAD else W.row_norm_weights(wl)
    pos = np.tile(orc.grid_positions(wl.T, wl.Hg, wl.Wg, 0, N), (B, 1))
    refs = [orc.qk_rmsnorm_rope3d_ex(bits(qkv[:, a * D:(a + 1) * D]), w.double().numpy(), H, hd,
                                     pos, wl.pairs, wl.theta, wl.eps, layout=layout, norm=norm)
            for a, w in ((0, wq), (1, wk))]
    buf = qkv.to(DEV).view(B, N, 3 * D)
    before = buf.clone()
    if order == "head_major":
        q_out = torch.full((B, H, N, hd), 7.0, dtype=torch.bfloat16, device=DEV).transpose(1, 2)
        k_out = torch.full((B, H, N, hd), 7.0, dtype=torch.bfloat16, device=DEV).transpose(1, 2)
    else:
        q_out = torch.full((B, N, H, hd), 7.0, dtype=torch.bfloat16, device=DEV)
        k_out = torch.full((B, N, H, hd), 7.0, dtype=torch.bfloat16, device=DEV)
    dbp.qk_rmsnorm_rope3d(buf[:, :, :D], buf[:, :, D:2 * D], wq.to(DEV), wk.to(DEV), H, wl.pairs,
                          grid=(wl.T, wl.Hg, wl.Wg), theta=wl.theta, eps=wl.eps,
                          rope_layout=layout, norm_width=norm, q_out=q_out, k_out=k_out)
    torch.cuda.synchronize()
    assert torch.equal(buf.view(torch.int16), before.view(torch.int16)), "input changed"
    for o, ref, nm in ((q_out, refs[0], "q"), (k_out, refs[1], "k")):
        compare_bf16(bits(o.reshape(B * N, D)), ref, f"{nm} {order}")


def test_qk_option_errors():
    wl = W.CONFIGS["tiny"]
    D = wl.H * wl.hd
    x = torch.zeros(1, 4, 3 * D, dtype=torch.bfloat16, device=DEV)
    wq, wk = (w.to(DEV) for w in W.norm_weights(wl))
    rq, rk = (w.to(DEV) for w in W.row_norm_weights(wl))
    grid = (1, 1, 4)
    with pytest.raises(dbp.DitError) as e:
        dbp.qk_rmsnorm_rope3d(x[:, :, :D], x[:, :, D:2 * D], wq, wk, wl.H, wl.pairs, grid=grid,
                              rope_layout=2)
    assert e.value.status == -8
    with pytest.raises(ValueError):      # a head-sized weight for the whole-row norm
        dbp.qk_rmsnorm_rope3d(x[:, :, :D], None, wq, None, wl.H, wl.pairs, grid=grid,
                              norm_width=dbp.NORM_ROW)
    dbp.qk_rmsnorm_rope3d(x[:, :, :D], x[:, :, D:2 * D], rq, rk, wl.H, wl.pairs, grid=grid,
                          norm_width=dbp.NORM_ROW)
    torch.cuda.synchronize()
    assert torch.count_nonzero(x) == 0   # a zero row stays zero under either norm


def test_qk_zero_position_is_plain_rms_norm(orc):
    wl = W.Workload("z", B=1, T=1, Hg=1, Wg=1, D=512, H=4, hd=128, F=8, pairs=(22, 21, 21))
    x = W.normal(0, 9, 1, 512).view(1, 1, 512)
    wq, _ = W.norm_weights(wl)
    ref = orc.qk_rmsnorm_rope3d(bits(x.view(1, 512)), wq.double().numpy(), 4, 128,
                                np.zeros((1, 3), np.int32), wl.pairs, 1e4, 1e-6)
    xg = x.to(DEV)
    dbp.qk_rmsnorm_rope3d(xg, None, wq.to(DEV), None, 4, wl.pairs, grid=(1, 1, 1))
    compare_bf16(bits(xg), ref, "rms at position 0")


# -------------------------------------------------------------- Cache-DiT


def _cache_case(orc, wl, thresholds):
    B, N, D = wl.B, wl.N, wl.D
    prev, cur = W.cache_pair(wl)
    prev, cur = prev.view(B, N, D), cur.view(B, N, D)
    pg, cg = prev.to(DEV), cur.to(DEV)
    for thr in thresholds:
        ref_rel, ref_reuse = orc.cachedit_residual_diff(bits(prev), bits(cur), thr)
        rel, reuse = dbp.cachedit_residual_diff(pg, cg, thr)
        rel, reuse = rel.cpu().numpy(), reuse.cpu().numpy()
        assert np.allclose(rel, ref_rel, rtol=1e-7, atol=0), (rel, ref_rel)
        assert np.all(np.abs(ref_rel - thr) > 1e-6 * thr), "case too close to the threshold"
        assert np.array_equal(reuse, ref_reuse), (rel, ref_rel, thr)
    return pg, cg


@pytest.mark.parametrize("name", ["tiny", "small", "ragged"])
def test_cachedit(orc, name):
    wl = W.CONFIGS.get(name) or ragged()
    _cache_case(orc, wl, (0.04, 0.08, 0.2))


def test_cachedit_identical_and_sign_flip():
    x = W.normal(0, 1, 1000, 512).view(2, 500, 512).to(DEV)
    rel, reuse = dbp.cachedit_residual_diff(x, x.clone(), 0.04)
    assert rel.cpu().tolist() == [0.0, 0.0] and reuse.cpu().tolist() == [1, 1]
    rel, reuse = dbp.cachedit_residual_diff(x, -x, 0.04)
    assert rel.cpu().tolist() == [2.0, 2.0] and reuse.cpu().tolist() == [0, 0]
    z = torch.zeros(1, 10, 64, dtype=torch.bfloat16, device=DEV)
    rel, reuse = dbp.cachedit_residual_diff(z, z.clone(), 0.04)
    assert rel.item() == 0.0 and reuse.item() == 1
    one = z.clone()
    one[0, 3, 5] = 1.0
    rel, reuse = dbp.cachedit_residual_diff(z, one, 0.04)
    assert rel.item() == float("inf") and reuse.item() == 0


def test_cachedit_exact_relative_change():
    vals = torch.tensor([1.0, -1.0, 1.5, -1.5, 0.75, 2.0, -3.0, 0.375])
    idx = torch.randint(0, 8, (3, 200, 256), generator=torch.Generator().manual_seed(0))
    prev = vals[idx]
    cur = prev * (1 + 2.0 ** -5)
    rel, reuse = dbp.cachedit_residual_diff(prev.to(torch.bfloat16).to(DEV),
                                            cur.to(torch.bfloat16).to(DEV), 2.0 ** -5)
    assert rel.cpu().tolist() == [2.0 ** -5] * 3
    assert reuse.cpu().tolist() == [0, 0, 0]        # strict <


def test_cachedit_sums_and_decide_over_shards(orc):
    """Shard sums + decide over the gathered [R, B, 2] equal one full call."""
    wl = ragged(B=2, N=301, D=512)
    pg, cg = _cache_case(orc, wl, (0.04,))
    rel_full, reuse_full = dbp.cachedit_residual_diff(pg, cg, 0.04)
    parts = [dbp.cachedit_residual_sums(pg[:, a:b].contiguous(), cg[:, a:b].contiguous())
             for a, b in ((0, 100), (100, 250), (250, 301))]
    rel, reuse = dbp.cachedit_decide(torch.stack(parts), 0.04)
    assert torch.allclose(rel, rel_full, rtol=1e-12, atol=0)
    assert torch.equal(reuse, reuse_full)
    num, den = orc.cachedit_sums(bits(pg[1]), bits(cg[1]))
    s = dbp.cachedit_residual_sums(pg, cg).cpu().numpy()
    assert np.isclose(s[1, 0], num, rtol=1e-7) and np.isclose(s[1, 1], den, rtol=1e-7)


def test_cachedit_deterministic_and_empty():
    wl = ragged(B=1, N=2000, D=1024)
    prev, cur = (t.view(1, 2000, 1024).to(DEV) for t in W.cache_pair(wl))
    r1, _ = dbp.cachedit_residual_diff(prev, cur, 0.04)
    r2, _ = dbp.cachedit_residual_diff(prev, cur, 0.04)
    assert r1.item() == r2.item()
    e = torch.empty(2, 0, 64, dtype=torch.bfloat16, device=DEV)
    rel, reuse = dbp.cachedit_residual_diff(e, e, 0.04)
    assert rel.cpu().tolist() == [0.0, 0.0] and reuse.cpu().tolist() == [1, 1]


def test_launch_error_reports_status():
    """A bad argument raises DitError with the status and launches nothing."""
    x = torch.zeros(1, 4, 60, dtype=torch.bfloat16, device=DEV)
    with pytest.raises(dbp.DitError) as e:
        dbp.adaln_modulate(x, torch.zeros(1, 60, device=DEV), torch.zeros(1, 60, device=DEV))
    assert e.value.status == -3
