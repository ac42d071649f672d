"""Block-sparse attention (tcgen05) against the fp64 oracle.  Tolerance,
derived from the arithmetic: the softmax weights enter P V as bf16 (relative
rounding at most 2^-9 each) and everything else is fp32, so an output
differs from the exact one by at most about 2^-8 * sum_u p_u |v_u| (p the
exact weights) plus one bf16 ulp of the output; a zero query makes every
weight exactly 1 and the output the mean of the kept values, which leaves
only fp32 summation and the final rounding."""
import numpy as np
import pytest
import torch

import dit_block_pass_b200 as dbp
from dit_block_pass_b200 import workloads as W
from parity import bits

pytestmark = pytest.mark.gpu
DEV = "cuda:0"
HD = 128


@pytest.fixture(scope="module", autouse=True)
def _built():
    from dit_block_pass_b200 import build
    build.build()


def _ulp_bf16(a):
    a = np.maximum(np.abs(a), 2.0 ** -126)
    return np.exp2(np.floor(np.log2(a)) - 7)


def _weights_abs_v(orc, q, k, v, kept, B, N, H, rows):
    """sum_u p_u |v_u| per (sampled row, head, d), fp64 (for the bound)."""
    Q = orc.bf16_to_f64(q)
    K = orc.bf16_to_f64(k)
    V = orc.bf16_to_f64(v)
    out = np.zeros((len(rows), H * HD))
    for n, t in enumerate(rows):
        b, tt = divmod(int(t), N)
        for h in range(H):
            blocks = kept[b, h, tt // 128]
            toks = np.concatenate([np.arange(j * 128, min(N, (j + 1) * 128)) for j in blocks])
            s = K[b * N + toks, h * HD:(h + 1) * HD] @ Q[t, h * HD:(h + 1) * HD] / np.sqrt(HD)
            p = np.exp(s - s.max())
            p /= p.sum()
            out[n, h * HD:(h + 1) * HD] = p @ np.abs(V[b * N + toks, h * HD:(h + 1) * HD])
    return out


def _case(orc, B, N, H, sparsity, seed, zero_q=False):
    g = torch.Generator().manual_seed(seed)
    D = H * HD
    qkv = torch.randn(B, N, 3 * D, generator=g).to(torch.bfloat16)
    if zero_q:
        qkv[:, :, :D] = 0
    x = qkv.to(DEV)
    q, k, v = x[:, :, :D], x[:, :, D:2 * D], x[:, :, 2 * D:]
    kept = dbp.subblock_router(k, k, H, 128, sparsity)     # any valid kept lists will do
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    out = dbp.block_sparse_attention(q, k, v, H, kept, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    flat = bits(qkv.view(B * N, 3 * D))
    qb, kb, vb = flat[:, :D], flat[:, D:2 * D], flat[:, 2 * D:]
    keptn = kept.cpu().numpy()
    got = orc.bf16_to_f64(bits(out.view(B * N, D)))
    ref = orc.block_sparse_attention(qb, kb, vb, B, H, HD, 128, keptn)
    return qb, kb, vb, keptn, got, ref, np.arange(B * N)


@pytest.mark.parametrize("B,N,H,sparsity", [(1, 512, 2, 0.5), (2, 1000, 2, 0.75),
                                            (1, 128, 1, 0.0), (3, 300, 1, 0.4),
                                            (1, 4096, 2, 0.8)])
def test_attention_matches_oracle(orc, B, N, H, sparsity):
    qb, kb, vb, kept, got, ref, rows = _case(orc, B, N, H, sparsity, B * N + H)
    bound = 2.0 ** -8 * _weights_abs_v(orc, qb, kb, vb, kept, B, N, H, rows) + \
        2 * _ulp_bf16(ref) + 1e-6
    err = np.abs(got - ref)
    assert not (err > bound).any(), (int((err > bound).sum()), float((err / bound).max()))
    # on average well inside it: bf16 output rounding alone averages about
    # 2^-10 of the output, and P's rounding adds a similar amount
    assert err.mean() < 2.0 ** -8 * np.abs(ref).mean()


def test_zero_query_is_the_mean_of_the_kept_values(orc):
    """q = 0: every kept key has weight exactly 1 before normalising, so the
    output is the mean of the kept values up to fp32 summation."""
    B, N, H = 2, 700, 2
    _, _, _, _, got, ref, _ = _case(orc, B, N, H, 0.6, 5, zero_q=True)
    assert np.all(np.abs(got - ref) <= _ulp_bf16(ref) + 1e-6)


def test_attention_full_size_sampled_tokens(orc):
    """The h3_5s clip: 124,992 tokens, 40 heads x 128, sparsity 0.75 (245 of
    977 key blocks per query block); the oracle on sampled tokens of two
    heads' query blocks."""
    wl = W.CONFIGS["h3_5s"]
    N, H, D = wl.N, wl.H, wl.D
    qkv = W.token_rows(wl, W.S_QKV, 3 * D, device=DEV).view(1, N, 3 * D)
    q, k, v = qkv[:, :, :D], qkv[:, :, D:2 * D], qkv[:, :, 2 * D:]
    kept = dbp.subblock_router(q, k, H, 128, 0.75)
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    out = dbp.block_sparse_attention(q, k, v, H, kept, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    keptn = kept.cpu().numpy()
    rows = np.array([0, 127, 64000, N - 1])
    # the oracle on the sampled query rows, over the whole clip's keys
    flat = qkv.view(N, 3 * D)
    qb = bits(flat[:, :D])
    kb = bits(flat[:, D:2 * D])
    vb = bits(flat[:, 2 * D:])
    ref = orc.block_sparse_attention(qb, kb, vb, 1, H, HD, 128, keptn, rows=rows)
    got = orc.bf16_to_f64(bits(out[0, torch.from_numpy(rows).to(DEV)]))
    bound = 2.0 ** -8 * np.abs(orc.bf16_to_f64(vb)).max(0) + 2 * _ulp_bf16(ref) + 1e-6
    assert np.all(np.abs(got - ref) <= bound)
    del qkv, out
    torch.cuda.empty_cache()


def test_attention_errors():
    x = torch.zeros(1, 256, 3 * 256, dtype=torch.bfloat16, device=DEV)
    q, k, v = x[:, :, :256], x[:, :, 256:512], x[:, :, 512:]
    kept = torch.zeros(1, 2, 2, 1, dtype=torch.int32, device=DEV)
    with pytest.raises(ValueError):
        dbp.block_sparse_attention(q, k, v, 2, kept[:, :1].contiguous())
    L = dbp.library()
    assert L.dit_block_sparse_attention(q.data_ptr(), k.data_ptr(), v.data_ptr(), 768,
                                        x.data_ptr(), 768, 1, 256, 4, 64, 128, kept.data_ptr(),
                                        1, 0.1, None, None) == -2          # hd 64
    assert L.dit_block_sparse_attention(q.data_ptr(), k.data_ptr(), v.data_ptr(), 768,
                                        x.data_ptr(), 768, 1, 256, 2, 128, 128, kept.data_ptr(),
                                        1, 0.1, None, None) == -7          # out over the inputs


def test_an_expired_wait_is_reported_and_the_context_survives(orc):
    """Failure path: with the copy warps issuing nothing (test hook) every
    wait of the pipeline runs out after its 2 s bound; the kernel reports
    through the status word, frees its tensor memory and returns, and the
    next launch in the same context is correct."""
    B, N, H = 1, 256, 1
    D = H * HD
    g = torch.Generator().manual_seed(3)
    qkv = torch.randn(B, N, 3 * D, generator=g).to(torch.bfloat16)
    x = qkv.to(DEV)
    q, k, v = x[:, :, :D], x[:, :, D:2 * D], x[:, :, 2 * D:]
    kept = dbp.subblock_router(k, k, H, 128, 0.5)
    out = torch.zeros(B, N, D, dtype=torch.bfloat16, device=DEV)
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    L = dbp.library()
    rc = L.dit_block_sparse_attention_stall_test(
        q.data_ptr(), k.data_ptr(), v.data_ptr(), 3 * D, out.data_ptr(), D, B, N, H, HD, 128,
        kept.data_ptr(), kept.shape[-1], HD ** -0.5, st.data_ptr(),
        torch.cuda.current_stream().cuda_stream)
    assert rc == 0
    torch.cuda.synchronize()
    assert int(st.item()) == 1
    assert L.dit_block_sparse_attention_stall_test(
        q.data_ptr(), k.data_ptr(), v.data_ptr(), 3 * D, out.data_ptr(), D, B, N, H, HD, 128,
        kept.data_ptr(), kept.shape[-1], HD ** -0.5, None, None) == -1     # status required
    st.zero_()
    good = dbp.block_sparse_attention(q, k, v, H, kept, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    flat = bits(qkv.view(B * N, 3 * D))
    ref = orc.block_sparse_attention(flat[:, :D], flat[:, D:2 * D], flat[:, 2 * D:], B, H, HD,
                                     128, kept.cpu().numpy())
    got = orc.bf16_to_f64(bits(good.view(B * N, D)))
    assert np.abs(got - ref).max() < 0.02
