"""The Cache-DiT step cache on the GPU against the oracle: the cached
residual store and reuse (bit for bit: both sides round the exact value
once), and whole denoising runs in which the reuse rule picks steps."""
import numpy as np
import pytest
import torch

import dit_block_pass_b200 as dbp
import oracle
from dit_block_pass_b200 import workloads as W
from parity import bits

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


@pytest.fixture(scope="module", autouse=True)
def _built():
    from dit_block_pass_b200 import build
    build.build()


def _pair(n, seed, spread=20):
    rng = np.random.default_rng(seed)
    a = torch.from_numpy(rng.standard_normal(n) * np.exp2(rng.integers(-spread, spread, n)))
    b = torch.from_numpy(rng.standard_normal(n) * np.exp2(rng.integers(-spread, spread, n)))
    return a.to(torch.bfloat16), b.to(torch.bfloat16)


@pytest.mark.parametrize("n", [8, 24, 4096 + 8, 3 * 2 ** 20 + 16, 5120 * 301])
def test_store_and_apply_bit_exact(orc, n):
    a, b = _pair(n, n)
    ag, bg = a.to(DEV), b.to(DEV)
    r = dbp.cachedit_residual_store(ag, bg)
    o = dbp.cachedit_residual_apply(ag, bg)
    torch.cuda.synchronize()
    assert np.array_equal(bits(r), orc.residual_store(bits(a), bits(b)))
    assert np.array_equal(bits(o), orc.residual_apply(bits(a), bits(b)))


def test_in_place_and_unaligned_wide_path(orc):
    """In place (out is an input) and 16-byte vectors (a 32-byte misaligned
    view), against the oracle."""
    a, b = _pair(8 * 1000 + 8, 3)
    buf = torch.empty(a.numel() + 8, dtype=torch.bfloat16, device=DEV)
    av = buf[8:]                                   # 16-byte aligned, not 32
    av.copy_(a.to(DEV))
    bg = b.to(DEV)
    dbp.cachedit_residual_apply(av, bg, out=av)
    torch.cuda.synchronize()
    assert np.array_equal(bits(av), orc.residual_apply(bits(a), bits(b)))
    ag = a.to(DEV)
    dbp.cachedit_residual_store(ag, bg, out=bg)      # residual written over `after`
    torch.cuda.synchronize()
    assert np.array_equal(bits(bg), orc.residual_store(bits(a), bits(b)))


def test_specials(orc):
    v = torch.tensor([3.0e38, -3.0e38, float("inf"), float("nan"), 0.0, -0.0, 1e-40, -1e-40],
                     dtype=torch.bfloat16)
    w = torch.tensor([3.0e38, 3.0e38, float("-inf"), 1.0, -0.0, -0.0, 1e-40, 1e-40],
                     dtype=torch.bfloat16)
    r = dbp.cachedit_residual_store(v.to(DEV), w.to(DEV)).cpu()
    o = dbp.cachedit_residual_apply(v.to(DEV), w.to(DEV)).cpu()
    for got, ref in ((r, orc.residual_store(bits(v), bits(w))),
                     (o, orc.residual_apply(bits(v), bits(w)))):
        g = bits(got)
        nan = np.isnan(orc.bf16_to_f64(ref))
        assert np.array_equal(np.isnan(orc.bf16_to_f64(g)), nan)
        assert np.array_equal(g[~nan], ref[~nan])


# ------------------------------------------------------------ denoising runs


def _run(wl, steps, sigmas, policy_args, side, orc=None):
    """A toy denoising run.  Step t: the first blocks add f_t (a base
    residual plus sigma_t noise), the remaining blocks add g_t; the cache
    reuses the stored residual of the remaining blocks when the rule allows.
    side = "gpu" (library) or "oracle".  Returns (decisions, rels, final h)."""
    B, N, D = wl.B, wl.N, wl.D
    M = B * N
    base = W.normal(wl.seed, 101, M, D)
    h = W.normal(wl.seed, 100, M, D)
    fs, gs = [], []
    for t in range(steps):
        z = W.normal(wl.seed, 200 + t, M, D, sigma=sigmas[t])
        fs.append((base.float() + z.float()).to(torch.bfloat16))
        gs.append(W.normal(wl.seed, 300 + t, M, D, sigma=0.5))
    decisions, rels = [], []
    prev_r1 = R = None
    if side == "gpu":
        pol = dbp.CachePolicy(*policy_args)
        h = h.to(DEV)
        fs = [f.to(DEV) for f in fs]
        gs = [g.to(DEV) for g in gs]
        ws = None
        for t in range(steps):
            h1 = (h.float() + fs[t].float()).to(torch.bfloat16)          # the first blocks
            r1 = dbp.cachedit_residual_store(h, h1)
            rel = None
            if prev_r1 is not None:
                rv, _ = dbp.cachedit_residual_diff(prev_r1.view(B, N, D), r1.view(B, N, D),
                                                   policy_args[0], workspace=ws)
                rel = float(rv.max().item())
            reuse = pol.decide(rel)
            if reuse:
                out = dbp.cachedit_residual_apply(h1, R)
            else:
                out = (h1.float() + gs[t].float()).to(torch.bfloat16)   # the remaining blocks
                R = dbp.cachedit_residual_store(h1, out)
            decisions.append(reuse)
            rels.append(rel)
            prev_r1, h = r1, out
        return decisions, rels, bits(h)
    hb = bits(h)
    fb = [bits(f) for f in fs]
    gb = [bits(g) for g in gs]
    for t in range(steps):
        h1 = orc.residual_apply(hb, fb[t])
        r1 = orc.residual_store(hb, h1)
        rel = None
        if prev_r1 is not None:
            rv, _ = orc.cachedit_residual_diff(prev_r1.reshape(B, N, D), r1.reshape(B, N, D),
                                               policy_args[0])
            rel = float(rv.max())
        rels.append(rel)
        reuse = oracle.cache_policy([np.nan if r is None else r for r in rels], *policy_args)[-1]
        if reuse:
            out = orc.residual_apply(h1, R)
        else:
            out = orc.residual_apply(h1, gb[t])
            R = orc.residual_store(h1, out)
        decisions.append(reuse)
        prev_r1, hb = r1, out
    return decisions, rels, hb


@pytest.mark.parametrize("policy_args", [(0.04, 0, 0), (0.08, 0, 0), (0.04, 2, 0), (0.08, 0, 2)])
def test_denoising_run_matches_the_oracle(orc, policy_args):
    wl = W.Workload("run", B=2, T=2, Hg=6, Wg=10, D=256, H=2, hd=128, F=8, pairs=(22, 21, 21))
    # first-block residual noise per step: quiet steps reuse, loud ones compute
    sigmas = [0.02, 0.02, 0.15, 0.02, 0.02, 0.02, 0.05, 0.02, 0.02, 0.3]
    dg, rg, hg = _run(wl, len(sigmas), sigmas, policy_args, "gpu")
    do, ro, ho = _run(wl, len(sigmas), sigmas, policy_args, "oracle", orc)
    assert dg == do
    for a, b in zip(rg[1:], ro[1:]):
        assert abs(a - b) <= 1e-6 * b
        assert abs(b - policy_args[0]) > 1e-3        # decisions far from the threshold
    assert np.array_equal(hg, ho)
    assert any(dg) and not all(dg[1:])               # the run mixes both kinds of step
