"""The C ABI without a GPU: the library loads, exports every function the
header declares, and rejects bad arguments on the host before touching CUDA
(only checks that return before any CUDA call are exercised here)."""
import ctypes
import os
import re

import pytest

from conftest import ROOT

HEADER = os.path.join(ROOT, "include", "dit_block.h")
E = {"NULL": -1, "SHAPE": -2, "ALIGN": -3, "DTYPE": -4, "WORKSPACE": -6, "OVERLAP": -7,
     "VALUE": -8}
A = 0x10000  # a 16-byte aligned fake address: never dereferenced by these calls


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    src = re.sub(r"//[^\n]*", "", src)
    names = re.findall(r"^[A-Za-z_][\w\s\*]*?\b([A-Za-z_]\w*)\s*\([^;{]*\)\s*;", src, flags=re.M)
    return sorted(set(names))


@pytest.fixture(scope="module")
def lib():
    from dit_block_pass_b200 import build
    import dit_block_pass_b200 as dbp
    build.build()
    return dbp.library()


def test_header_declares_the_hot_path():
    names = declared_functions()
    for n in ("dit_adaln_modulate", "dit_gated_residual_adaln", "dit_swiglu",
              "dit_qk_rmsnorm_rope3d", "dit_qk_rmsnorm_rope3d_ex", "cachedit_residual_diff",
              "cachedit_workspace_bytes",
              "cachedit_residual_sums", "cachedit_decide", "dit_status_string",
              "dit_abi_version"):
        assert n in names


def test_every_declared_symbol_is_exported(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name


def test_header_is_plain_c():
    """The header compiles as C99 with no CUDA include path."""
    import subprocess
    import tempfile
    with tempfile.TemporaryDirectory() as d:
        c = os.path.join(d, "t.c")
        open(c, "w").write('#include "dit_block.h"\nint main(void){return dit_abi_version();}\n')
        subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-fsyntax-only",
                        "-I", os.path.dirname(HEADER), c], check=True)


def test_status_strings_and_version(lib):
    assert lib.dit_abi_version() == 1
    assert lib.dit_status_string(0) == b"ok"
    for code in E.values():
        assert lib.dit_status_string(code) not in (b"ok", b"unknown status")


def test_workspace_size_is_host_only(lib):
    assert lib.cachedit_workspace_bytes(1, 124992, 5120) > 0
    assert lib.cachedit_workspace_bytes(2, 0, 8) == 2 * lib.cachedit_workspace_bytes(1, 0, 8)
    assert lib.cachedit_workspace_bytes(0, 10, 8) == 0


def test_swiglu_argument_errors(lib):
    f = lib.dit_swiglu
    assert f(None, A, 4, 8, None) == E["NULL"]
    assert f(A, A + 0x1000, -1, 8, None) == E["SHAPE"]
    assert f(A, A + 0x1000, 4, 0, None) == E["SHAPE"]
    assert f(A, A + 0x1000, 4, 12, None) == E["ALIGN"]         # F % 8
    assert f(A + 2, A + 0x1000, 4, 8, None) == E["ALIGN"]      # misaligned in
    assert f(A, A + 16, 4, 8, None) == E["OVERLAP"]            # out inside in
    assert f(A, A + 0x1000, 0, 8, None) == 0                   # empty: no launch


def test_adaln_argument_errors(lib):
    f = lib.dit_adaln_modulate
    ok = (A, A + 0x100000, A + 0x200000, A + 0x300000, 0, 0, 1, 4, 64, 1e-6, None)

    def call(**kw):
        names = ["x", "y", "shift", "scale", "dt", "ms", "B", "N", "D", "eps", "s"]
        a = dict(zip(names, ok))
        a.update(kw)
        return f(*[a[n] for n in names])

    assert call(x=None) == E["NULL"]
    assert call(shift=None) == E["NULL"]
    assert call(D=60) == E["ALIGN"]
    assert call(D=8200) == E["SHAPE"]
    assert call(B=-1) == E["SHAPE"]
    assert call(dt=7) == E["DTYPE"]
    assert call(eps=-1.0) == E["VALUE"]
    assert call(eps=float("nan")) == E["VALUE"]
    assert call(x=A + 8) == E["ALIGN"]
    assert call(scale=A + 0x300002) == E["ALIGN"]              # fp32 scale not 4-aligned
    assert call(y=A + 64) == E["OVERLAP"]                      # partial overlap
    assert call(N=0) == 0
    g = lib.dit_gated_residual_adaln
    base = [A, A + 0x100000, A + 0x200000, A + 0x300000, A + 0x400000, A + 0x500000,
            A + 0x600000, 0, 0, 1, 4, 64, 1e-6, None]
    bad = list(base)
    bad[1] = A  # r == x
    assert g(*bad) == E["OVERLAP"]
    bad = list(base)
    bad[2] = A  # x_out == x is allowed (in place): empty N makes it a no-op
    bad[10] = 0
    assert g(*bad) == 0
    bad = list(base)
    bad[4] = None
    assert g(*bad) == E["NULL"]


def test_qk_argument_errors(lib):
    f = lib.dit_qk_rmsnorm_rope3d
    names = ["q", "k", "rs", "wq", "wk", "wdt", "B", "N", "H", "hd", "T", "Hg", "Wg", "pos",
             "off", "pt", "ph", "pw", "theta", "eps", "s"]
    ok = dict(zip(names, [A, A + 2 * 256, 768, A + 0x900000, A + 0x900100, 0, 1, 48, 4, 64, 2, 4,
                          6, None, 0, 12, 10, 10, 1e4, 1e-6, None]))

    def call(**kw):
        a = dict(ok)
        a.update(kw)
        return f(*[a[n] for n in names])

    assert call(q=None, k=None) == E["NULL"]
    assert call(wq=None) == E["NULL"]
    assert call(hd=48, H=4) == E["SHAPE"]                       # unsupported head dim
    assert call(pt=11) == E["SHAPE"]                            # pairs do not sum to hd/2
    assert call(rs=200) == E["SHAPE"]                           # stride < H*hd
    assert call(rs=772) == E["ALIGN"]
    assert call(N=49) == E["SHAPE"]                             # beyond the grid
    assert call(off=1) == E["SHAPE"]
    assert call(k=A + 2 * 128) == E["OVERLAP"]                  # k inside q's row
    assert call(theta=0.0) == E["VALUE"]
    assert call(wdt=3) == E["DTYPE"]
    assert call(q=A + 4) == E["ALIGN"]
    assert call(N=0) == 0


def test_qk_option_argument_errors(lib):
    f = lib.dit_qk_rmsnorm_rope3d_ex
    names = ["q", "k", "rs", "wq", "wk", "wdt", "B", "N", "H", "hd", "T", "Hg", "Wg", "pos",
             "off", "pt", "ph", "pw", "theta", "eps", "layout", "norm", "out", "s"]
    ok = dict(zip(names, [A, A + 2 * 256, 768, A + 0x900000, A + 0x900100, 0, 1, 48, 4, 64, 2, 4,
                          6, None, 0, 12, 10, 10, 1e4, 1e-6, 0, 0, None, None]))

    def call(**kw):
        a = dict(ok)
        a.update(kw)
        return f(*[a[n] for n in names])

    assert call(layout=2) == E["VALUE"]
    assert call(layout=-1) == E["VALUE"]
    assert call(norm=2) == E["VALUE"]
    assert call(norm=1, wq=A + 0x900004) == E["ALIGN"]     # row weights are read 16 B at a time
    assert call(norm=1, wq=None) == E["NULL"]
    assert call(hd=48, H=4, layout=1) == E["SHAPE"]
    assert call(N=0, layout=1, norm=1) == 0

    # separate outputs: [B, N, H, hd] = [1, 48, 4, 64] with element strides
    import ctypes
    from dit_block_pass_b200 import QKOut
    O = A + 0x1000000                                   # well clear of the inputs
    head_major = (4 * 48 * 64, 64, 48 * 64)
    assert call(out=ctypes.byref(QKOut(O, O + 0x100000, *head_major)), N=0) == 0
    assert call(out=ctypes.byref(QKOut(O, None, *head_major))) == E["NULL"]
    assert call(out=ctypes.byref(QKOut(O + 4, O + 0x100000, *head_major))) == E["ALIGN"]
    assert call(out=ctypes.byref(QKOut(O, O + 0x100000, 4 * 48 * 64, 64, 44 * 64))) == E["SHAPE"]
    assert call(out=ctypes.byref(QKOut(O, O + 0x100000, 4 * 48 * 64, 60, 48 * 64))) == E["ALIGN"]
    assert call(out=ctypes.byref(QKOut(O, O + 0x100, *head_major))) == E["OVERLAP"]
    assert call(out=ctypes.byref(QKOut(A + 0x40, O, *head_major))) == E["OVERLAP"]  # on q


def test_cachedit_argument_errors(lib):
    f = lib.cachedit_residual_diff
    ws = lib.cachedit_workspace_bytes(1, 4, 64)
    assert f(None, A, 1, 4, 64, 0.04, A, A, A, ws, None) == E["NULL"]
    assert f(A, A, 0, 4, 64, 0.04, A, A, A, ws, None) == E["SHAPE"]
    assert f(A, A, 1, 4, 60, 0.04, A, A, A, ws, None) == E["ALIGN"]
    assert f(A, A, 1, 4, 64, 0.04, None, A, A, ws, None) == E["NULL"]
    assert f(A, A, 1, 4, 64, float("nan"), A, A, A, ws, None) == E["VALUE"]
    assert f(A, A, 1, 4, 64, 0.04, A, A, None, ws, None) == E["WORKSPACE"]
    assert f(A, A, 1, 4, 64, 0.04, A, A, A, ws - 1, None) == E["WORKSPACE"]
    assert lib.cachedit_decide(None, 1, 1, 0.04, A, A, None) == E["NULL"]
    assert lib.cachedit_decide(A, 0, 1, 0.04, A, A, None) == E["SHAPE"]
    assert lib.cachedit_decide(A + 4, 1, 1, 0.04, A, A, None) == E["ALIGN"]


def test_binding_refuses_cpu_tensors():
    import torch
    import dit_block_pass_b200 as dbp
    x = torch.zeros(1, 4, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        dbp.adaln_modulate(x, torch.zeros(1, 64), torch.zeros(1, 64))
    with pytest.raises(ValueError):
        dbp.swiglu(torch.zeros(4, 16, dtype=torch.bfloat16))


def test_cache_policy_matches_the_rule(lib):
    """The library's reuse rule against the oracle's, on golden and random
    runs (host code: no GPU)."""
    import numpy as np
    import oracle
    from conftest import load_golden
    from dit_block_pass_b200 import CachePolicy
    cases = [([float(x) for x in c["rels"]], c["threshold"], c["warmup"], c["max_cached"])
             for c in load_golden("cache_policy.json")["cases"]]
    rng = np.random.default_rng(11)
    for _ in range(300):
        cases.append((list(rng.exponential(0.05, 40)), float(rng.choice([0.04, 0.08])),
                      int(rng.integers(0, 5)), int(rng.integers(0, 4))))
    for rels, thr, warm, cap in cases:
        p = CachePolicy(thr, warm, cap)
        got = [p.decide(r) for r in rels]
        assert got == oracle.cache_policy(rels, thr, warm, cap)
        assert p.step == len(rels) and p.reused == sum(got) and p.computed == len(rels) - sum(got)


def test_cache_policy_and_step_cache_errors(lib):
    import ctypes
    from dit_block_pass_b200 import CachePolicyStruct
    s = CachePolicyStruct()
    assert lib.dit_cache_policy_init(None, 0.04, 0, 0) == E["NULL"]
    assert lib.dit_cache_policy_init(ctypes.byref(s), float("nan"), 0, 0) == E["VALUE"]
    assert lib.dit_cache_policy_init(ctypes.byref(s), 0.04, -1, 0) == E["VALUE"]
    assert lib.dit_cache_policy_decide(None, 0.0) == E["NULL"]
    for f in (lib.cachedit_residual_store, lib.cachedit_residual_apply):
        assert f(A, A + 0x10000, A + 0x20000, 0, None) == 0            # empty: no launch
        assert f(A, A + 0x10000, A + 0x20000, -8, None) == E["SHAPE"]
        assert f(None, A + 0x10000, A + 0x20000, 8, None) == E["NULL"]
        assert f(A, A + 0x10000, A + 0x20000, 12, None) == E["ALIGN"]
        assert f(A + 2, A + 0x10000, A + 0x20000, 8, None) == E["ALIGN"]
        assert f(A, A + 0x10000, A + 16, 64, None) == E["OVERLAP"]    # partly over an input


def test_swiglu_gemm_argument_errors(lib):
    f = lib.dit_swiglu_gemm
    assert f(A, A + 0x100000, A + 0x200000, 0, 64, 64, None, None) == 0      # empty M
    assert f(A, A + 0x100000, A + 0x200000, -1, 64, 64, None, None) == E["SHAPE"]
    assert f(A, A + 0x100000, A + 0x200000, 4, 0, 64, None, None) == E["SHAPE"]
    assert f(A, A + 0x100000, A + 0x200000, 4, 60, 64, None, None) == E["ALIGN"]
    assert f(A, A + 0x100000, A + 0x200000, 4, 64, 12, None, None) == E["ALIGN"]
    assert f(None, A + 0x100000, A + 0x200000, 4, 64, 64, None, None) == E["NULL"]
    assert f(A + 8, A + 0x100000, A + 0x200000, 4, 64, 64, None, None) == E["ALIGN"]
    assert f(A, A + 0x100000, A + 0x200000, 4, 64, 64, A + 2, None) == E["ALIGN"]
    assert f(A, A + 0x100000, A + 0x100, 4, 64, 64, None, None) == E["OVERLAP"]   # over x


def test_gemm_gated_residual_argument_errors(lib):
    f = lib.dit_gemm_gated_residual
    H, W_, X, O, G = A, A + 0x100000, A + 0x200000, A + 0x300000, A + 0x400000
    assert f(H, W_, X, O, G, 0, 64, 0, 4, 64, 64, None, None) == 0          # empty
    assert f(H, W_, X, O, G, 0, 64, 1, 4, 60, 64, None, None) == E["ALIGN"]
    assert f(H, W_, X, O, G, 2, 64, 1, 4, 64, 64, None, None) == E["DTYPE"]
    assert f(H, W_, X, O, None, 0, 64, 1, 4, 64, 64, None, None) == E["NULL"]
    assert f(H, W_, X, O, G + 2, 0, 64, 1, 4, 64, 64, None, None) == E["ALIGN"]
    assert f(H, W_, X, X + 16, G, 0, 64, 1, 4, 64, 64, None, None) == E["OVERLAP"]
    assert f(H, W_, X, H, G, 0, 64, 1, 4, 64, 64, None, None) == E["OVERLAP"]
    assert f(H, W_, X, O, G, 0, -1, 1, 4, 64, 64, None, None) == E["SHAPE"]


def test_subblock_router_host(lib):
    """The keep count equals the oracle's; argument errors launch nothing."""
    import oracle
    orc = oracle.default()
    for nb in (1, 3, 8, 100, 977, 1922, 8192):
        for sp in (0.0, 0.5, 0.75, 0.8, 0.99):
            assert lib.dit_subblock_keep_count(nb, sp) == orc.subblock_keep_count(nb, sp)
    assert lib.dit_subblock_keep_count(10, 1.0) == E["VALUE"]
    f = lib.dit_subblock_router
    ws = lib.dit_subblock_workspace_bytes(1, 256, 2, 64, 128)
    # block means (256-byte rounded), then the scores and the split means
    assert ws == 2048 + lib.dit_subblock_means_workspace_bytes(1, 256, 2, 64, 128)
    assert lib.dit_subblock_means_workspace_bytes(1, 256, 2, 64, 128) == 256 + 2 * 2048
    assert lib.dit_subblock_workspace_bytes(1, 256, 2, 48, 128) == 1536 + 32  # fp32 scores only
    assert f(A, A + 0x1000, 128, 1, 0, 2, 64, 128, 0.75, A + 0x2000, A + 0x3000, ws, None, None) == 0
    assert f(A, A + 0x1000, 128, 1, 256, 2, 60, 128, 0.75, A + 0x2000, A + 0x3000, ws, None, None) == E["SHAPE"]
    assert f(A, A + 0x1000, 128, 1, 256, 2, 64, 128, 1.0, A + 0x2000, A + 0x3000, ws, None, None) == E["VALUE"]
    assert f(A, A + 0x1000, 128, 1, 256, 2, 64, 128, 0.75, A + 0x2000, A + 0x3000, ws - 4, None, None) == E["WORKSPACE"]
    assert f(A, None, 128, 1, 256, 2, 64, 128, 0.75, A + 0x2000, A + 0x3000, ws, None, None) == E["NULL"]
    assert f(A, A + 0x1000, 120, 1, 256, 2, 64, 128, 0.75, A + 0x2000, A + 0x3000, ws, None, None) == E["SHAPE"]
    assert f(A, A + 0x1000, 128, 1, 128 * 8193, 2, 64, 128, 0.75, A + 0x2000, A + 0x3000, ws, None, None) == E["SHAPE"]
    # the score kernel's stall hook refuses what it does not test, before any launch
    g = lib.dit_subblock_scores_stall_test
    mws = lib.dit_subblock_means_workspace_bytes(1, 256, 2, 64, 128)
    assert g(A, 1, 256, 2, 64, 128, A + 0x2000, mws, None, None) == E["NULL"]           # status
    assert g(A, 1, 256, 2, 48, 128, A + 0x2000, mws, A + 0x100, None) == E["SHAPE"]      # FMA path
    assert g(A, 1, 256 * 1024, 2, 64, 8, A + 0x2000, mws, A + 0x100, None) == E["SHAPE"]  # too big
    assert g(A, 1, 256, 2, 64, 128, A + 0x2000, mws - 16, A + 0x100, None) == E["WORKSPACE"]


def test_cachedit_result_buffers_are_checked_before_the_call():
    """rel [B] float64 and reuse [B] uint8 reach the kernel as raw pointers,
    so the binding rejects a wrong dtype, a short or strided tensor, or one on
    another device before any call (checked here on CPU tensors)."""
    import torch
    import dit_block_pass_b200 as dbp
    prev = torch.zeros(3, 4, 8, dtype=torch.bfloat16)
    rel, reuse = dbp._result_buffers(prev, 3, None, None)
    assert rel.dtype == torch.float64 and reuse.dtype == torch.uint8 and rel.numel() == 3
    ok_rel, ok_reuse = torch.zeros(3, dtype=torch.float64), torch.zeros(3, dtype=torch.uint8)
    assert dbp._result_buffers(prev, 3, ok_rel, ok_reuse)[0] is ok_rel
    bad = [
        (torch.zeros(3, dtype=torch.float32), ok_reuse),           # rel float32
        (torch.zeros(2, dtype=torch.float64), ok_reuse),           # rel too short
        (torch.zeros(6, dtype=torch.float64)[::2], ok_reuse),      # rel strided
        (ok_rel, torch.zeros(3, dtype=torch.int32)),               # reuse int32
        (ok_rel, torch.zeros(2, dtype=torch.uint8)),               # reuse too short
        (ok_rel, torch.zeros(3, dtype=torch.uint8, device="meta")),  # another device
    ]
    for r, u in bad:
        with pytest.raises(ValueError):
            dbp._result_buffers(prev, 3, r, u)
