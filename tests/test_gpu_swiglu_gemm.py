"""SwiGLU fused into the up-projection GEMM and the gated residual fused
into the down-projection GEMM (tcgen05) against the fp64 oracle.  Tolerance, derived from the arithmetic: the tensor cores sum K
exact bf16 products in fp32, so |g_gpu - g| <= 2 K 2^-24 sum_k |x w| for any
summation order (the factor 2 is margin for the unit's internal order);
that error passes through silu(g) * u with |silu'| <= 1.1, and the result is
rounded once to bf16 (at most one bf16 ulp of slack, plus a few fp32 ulp for
the fast exp and divide)."""
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


def _ulp_bf16(a):
    a = np.maximum(np.abs(a), 2.0 ** -126)
    return np.exp2(np.floor(np.log2(a)) - 7)


def _gu(x_rows, w):
    """g and u in float64 (for the error bound only), F in chunks."""
    X = x_rows.double()
    F = w.shape[0] // 2
    g = torch.empty(X.shape[0], F, dtype=torch.float64)
    u = torch.empty_like(g)
    for a in range(0, F, 2048):
        b = min(F, a + 2048)
        g[:, a:b] = X @ w[a:b].double().T
        u[:, a:b] = X @ w[F + a:F + b].double().T
    return g.numpy(), u.numpy()


def _check(orc, x_rows, w, got, what=""):
    """Compare GPU rows (outputs of the rows x_rows) with the oracle under
    the derived bound."""
    ref, ga, ua = orc.swiglu_gemm(bits(x_rows), bits(w))
    K = x_rows.shape[1]
    g, u = _gu(x_rows, w)
    eg = 2.0 * K * 2.0 ** -24 * ga
    eu = 2.0 * K * 2.0 ** -24 * ua
    sg = g / (1.0 + np.exp(-g))
    bound = 1.1 * eg * np.abs(u) + np.abs(sg) * eu + eg * eu + _ulp_bf16(ref) + 1e-6 * np.abs(ref)
    out = orc.bf16_to_f64(bits(got))
    err = np.abs(out - ref)
    bad = err > bound
    assert not bad.any(), (what, int(bad.sum()), float((err / bound).max()))
    # and typically far inside it: nearly every output is within one bf16 ulp
    frac_close = float(np.mean(err <= _ulp_bf16(ref)))
    assert frac_close > 0.99, (what, frac_close)


def _inputs(M, K, F, seed, int_valued=False):
    g = torch.Generator().manual_seed(seed)
    if int_valued:
        x = torch.randint(-3, 4, (M, K), generator=g).to(torch.bfloat16)
        w = torch.randint(-2, 3, (2 * F, K), generator=g).to(torch.bfloat16) / 8
    else:
        x = torch.randn(M, K, generator=g).to(torch.bfloat16)
        w = (torch.randn(2 * F, K, generator=g) / K ** 0.5).to(torch.bfloat16)
    return x, w


@pytest.mark.parametrize("M,K,F", [(128, 64, 128), (256, 512, 256), (200, 136, 136),
                                   (1000, 1024, 384), (77, 5120, 72)])
def test_fused_gemm_matches_oracle(orc, M, K, F):
    x, w = _inputs(M, K, F, M + K + F)
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    out = dbp.swiglu_gemm(x.to(DEV), w.to(DEV), status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    _check(orc, x, w, out.cpu(), what=f"{M}x{K}x{F}")


def test_exact_products_locate_every_element(orc):
    """Small integer inputs make every dot product exact in fp32, so any
    misplaced tile, swizzle or K step shows as a large error."""
    M, K, F = 384, 320, 256
    x, w = _inputs(M, K, F, 5, int_valued=True)
    out = dbp.swiglu_gemm(x.to(DEV), w.to(DEV)).cpu()
    ref, _, _ = orc.swiglu_gemm(bits(x), bits(w))
    got = orc.bf16_to_f64(bits(out))
    assert np.all(np.abs(got - ref) <= _ulp_bf16(ref) + 1e-6 * np.abs(ref))


def test_against_the_unfused_chain():
    """The fused op against cuBLAS's bf16 GEMM followed by the one-pass SwiGLU:
    they differ only by the unfused chain's rounding of g and u to bf16."""
    M, K, F = 512, 1024, 512
    x, w = _inputs(M, K, F, 9)
    xg, wg = x.to(DEV), w.to(DEV)
    fused = dbp.swiglu_gemm(xg, wg).float()
    unfused = dbp.swiglu(xg @ wg.T).float()
    rel = ((fused - unfused).abs() / unfused.abs().clamp_min(1e-2)).max().item()
    assert rel < 0.05, rel


def test_full_size_sampled_rows(orc):
    """The h3_5s up-projection: x [124992, 5120], w [27648, 5120]; rows
    sampled across every row tile (first, last, ragged tail)."""
    wl = W.CONFIGS["h3_5s"]
    M, K, F = wl.M, wl.D, wl.F
    g = torch.Generator(device=DEV).manual_seed(1)
    xg = torch.randn(M, K, generator=g, device=DEV).to(torch.bfloat16)
    wg = (torch.randn(2 * F, K, generator=g, device=DEV) / K ** 0.5).to(torch.bfloat16)
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    out = dbp.swiglu_gemm(xg, wg, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    rows = np.array([0, 1, 127, 128, 5000, 65537, M - 129, M - 1])
    x_rows = xg[torch.from_numpy(rows).to(DEV)].cpu()
    got = out[torch.from_numpy(rows).to(DEV)].cpu()
    w_host = wg.cpu()
    _check(orc, x_rows, w_host, got, what="h3_5s rows")
    del xg, wg, out
    torch.cuda.empty_cache()


def test_empty_and_errors():
    x = torch.empty(0, 64, dtype=torch.bfloat16, device=DEV)
    w = torch.zeros(16, 64, dtype=torch.bfloat16, device=DEV)
    assert dbp.swiglu_gemm(x, w).shape == (0, 8)
    with pytest.raises(ValueError):
        dbp.swiglu_gemm(torch.zeros(4, 64, dtype=torch.bfloat16, device=DEV), w[:, :32].contiguous())


# ------------------------------------------ gated residual, down-projection


def _check_resid(orc, h_rows, w, x_rows, gate, N, got, rows_global, what=""):
    """x' within the derived bound: |g| * 2 K 2^-24 sum|h w| for the
    accumulation, plus one bf16 ulp for the final rounding."""
    B = gate.shape[0]
    # the oracle on the selected rows: pass them as their own samples
    ref, dot, ad = orc.gemm_gated_residual(bits(h_rows), bits(w), bits(x_rows),
                                           gate.double().numpy()[rows_global // N], 1)
    K = h_rows.shape[1]
    gv = np.abs(gate.double().numpy()[rows_global // N])
    bound = gv * 2.0 * K * 2.0 ** -24 * ad + _ulp_bf16(orc.bf16_to_f64(ref))
    out = orc.bf16_to_f64(bits(got))
    err = np.abs(out - orc.bf16_to_f64(ref))
    assert not (err > bound).any(), (what, int((err > bound).sum()))
    assert float(np.mean(err == 0)) > 0.95, (what, float(np.mean(err == 0)))
    del B


@pytest.mark.parametrize("B,N,K,D", [(1, 128, 64, 256), (2, 100, 512, 384), (3, 77, 136, 264),
                                     (1, 1000, 2048, 1024)])
@pytest.mark.parametrize("gate_dtype", [torch.float32, torch.bfloat16])
def test_down_projection_gated_residual(orc, B, N, K, D, gate_dtype):
    g = torch.Generator().manual_seed(B * 1000 + N + K + D)
    h = torch.randn(B, N, K, generator=g).to(torch.bfloat16)
    w = (torch.randn(D, K, generator=g) / K ** 0.5).to(torch.bfloat16)
    x = torch.randn(B, N, D, generator=g).to(torch.bfloat16)
    gate = (0.3 * torch.randn(B, D, generator=g)).to(gate_dtype)
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    out = dbp.gemm_gated_residual(h.to(DEV), w.to(DEV), x.to(DEV), gate.to(DEV), status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    M = B * N
    rows = np.arange(M)
    _check_resid(orc, h.view(M, K), w, x.view(M, D), gate.float(), N, out.view(M, D).cpu(), rows,
                 what=f"{B}x{N}x{K}x{D}")


def test_down_projection_in_place_and_zero_gate(orc):
    """In place on x; a zero gate leaves x bit for bit."""
    B, N, K, D = 2, 200, 256, 512
    g = torch.Generator().manual_seed(3)
    h = torch.randn(B, N, K, generator=g).to(torch.bfloat16).to(DEV)
    w = (torch.randn(D, K, generator=g) / K ** 0.5).to(torch.bfloat16).to(DEV)
    x = torch.randn(B, N, D, generator=g).to(torch.bfloat16).to(DEV)
    x0 = x.clone()
    dbp.gemm_gated_residual(h, w, x, torch.zeros(B, D, device=DEV), x_out=x)
    torch.cuda.synchronize()
    assert torch.equal(x.view(torch.int16), x0.view(torch.int16))
    gate = 0.5 * torch.ones(D, device=DEV)                  # one gate for every sample
    ref = dbp.gemm_gated_residual(h, w, x0, gate)
    dbp.gemm_gated_residual(h, w, x, gate, x_out=x)
    torch.cuda.synchronize()
    assert torch.equal(x.view(torch.int16), ref.view(torch.int16))


def test_down_projection_full_size_sampled_rows(orc):
    """The h3_5s down-projection: h [124992, 13824], w [5120, 13824]."""
    wl = W.CONFIGS["h3_5s"]
    M, K, D = wl.M, wl.F, wl.D
    gen = torch.Generator(device=DEV).manual_seed(2)
    h = torch.randn(1, M, K, generator=gen, device=DEV).to(torch.bfloat16)
    w = (torch.randn(D, K, generator=gen, device=DEV) / K ** 0.5).to(torch.bfloat16)
    x = torch.randn(1, M, D, generator=gen, device=DEV).to(torch.bfloat16)
    gate = 0.3 * torch.randn(1, D, generator=gen, device=DEV)
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    out = dbp.gemm_gated_residual(h, w, x, gate, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    rows = np.array([0, 255, 256, 70001, M - 257, M - 1])
    idx = torch.from_numpy(rows).to(DEV)
    _check_resid(orc, h[0, idx].cpu(), w.cpu(), x[0, idx].cpu(), gate.cpu(), M,
                 out[0, idx].cpu(), rows, what="h3_5s rows")
    del h, w, x, out
    torch.cuda.empty_cache()


def test_an_expired_wait_is_reported_and_the_context_survives(orc):
    """Failure path: with the copy warp disabled (test hook) every pipeline
    wait runs out after its 2 s bound; the kernel reports through the status
    word, frees its tensor memory and returns, and the next launch works."""
    M, K, F = 128, 64, 128
    x, w = _inputs(M, K, F, 11)
    xg, wg = x.to(DEV), w.to(DEV)
    out = torch.zeros(M, F, dtype=torch.bfloat16, device=DEV)
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    L = dbp.library()
    rc = L.dit_swiglu_gemm_stall_test(xg.data_ptr(), wg.data_ptr(), out.data_ptr(), M, K, F,
                                      st.data_ptr(), torch.cuda.current_stream().cuda_stream)
    assert rc == 0
    torch.cuda.synchronize()
    assert int(st.item()) == 1
    st.zero_()
    good = dbp.swiglu_gemm(xg, wg, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    _check(orc, x, w, good.cpu(), what="after the stall")
