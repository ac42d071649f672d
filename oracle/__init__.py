"""fp64 CPU oracle for the DiT block memory-bound operators.

TEST INFRASTRUCTURE ONLY.  Only the test-suite, ``__graft_entry__.smoke()``
and the CPU-baseline leg of ``bench.py`` may import this package.  The CUDA
library never loads it and shares no code with it; a product call that reached
this module would be a CPU fallback, which the library does not have.

This module is argument marshalling around ``dit_oracle.c`` (numpy arrays in,
numpy arrays out).  bf16 tensors travel as ``uint16`` bit patterns; modulation
vectors and norm weights as ``float64`` (a float32 value widens exactly).
Outputs come back unrounded in fp64; ``f64_to_bf16`` rounds them once.
"""
from __future__ import annotations

import ctypes
import threading

import numpy as np

from . import build as _build

_u16p = ctypes.POINTER(ctypes.c_uint16)
_u8p = ctypes.POINTER(ctypes.c_uint8)
_i32p = ctypes.POINTER(ctypes.c_int32)
_f64p = ctypes.POINTER(ctypes.c_double)
_i64 = ctypes.c_int64
_int = ctypes.c_int
_dbl = ctypes.c_double


def _c(a: np.ndarray, dtype) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=dtype)


def _p(a: np.ndarray, ptype):
    return a.ctypes.data_as(ptype)


def _check(rc: int, what: str) -> None:
    if rc != 0:
        raise ValueError(f"oracle {what}: bad arguments (code {rc})")


class Oracle:
    """The oracle library at ``path`` (the built dit_oracle.c by default)."""

    def __init__(self, path: str | None = None):
        L = ctypes.CDLL(path or _build.build())
        L.dito_bf16_to_f64.argtypes = [ctypes.c_uint16]
        L.dito_bf16_to_f64.restype = _dbl
        L.dito_f64_to_bf16.argtypes = [_dbl]
        L.dito_f64_to_bf16.restype = ctypes.c_uint16
        L.dito_round_bf16.argtypes = [_f64p, _u16p, _i64]
        L.dito_widen_bf16.argtypes = [_u16p, _f64p, _i64]
        L.dito_adaln_modulate.argtypes = [_u16p, _f64p, _f64p, _i64, _int, _i64, _int,
                                          _dbl, _f64p, _f64p]
        L.dito_gated_residual_adaln.argtypes = [_u16p, _u16p, _f64p, _f64p, _f64p, _i64,
                                                _int, _i64, _int, _dbl, _u16p, _f64p, _f64p]
        L.dito_swiglu.argtypes = [_u16p, _i64, _int, _f64p]
        L.dito_grid_positions.argtypes = [_int, _int, _int, _i64, _i64, _i32p]
        L.dito_qk_rmsnorm_rope3d.argtypes = [_u16p, _i64, _f64p, _int, _i64, _int, _int,
                                             _i32p, _int, _int, _int, _dbl, _dbl, _f64p, _f64p]
        L.dito_qk_rmsnorm_rope3d_ex.argtypes = [_u16p, _i64, _f64p, _int, _i64, _int, _int,
                                                _i32p, _int, _int, _int, _dbl, _dbl, _int, _int,
                                                _f64p, _f64p]
        L.dito_cachedit_sums.argtypes = [_u16p, _u16p, _i64, _f64p, _f64p]
        L.dito_cachedit_decide.argtypes = [_dbl, _dbl, _dbl, _f64p]
        L.dito_cachedit_decide.restype = _int
        L.dito_cachedit_residual_diff.argtypes = [_u16p, _u16p, _int, _i64, _int, _dbl,
                                                  _f64p, _u8p]
        L.dito_adaln_modulate_tok.argtypes = [_u16p, _f64p, _f64p, _i64, _i64, _u8p, _int, _int,
                                              _i64, _int, _dbl, _f64p, _f64p]
        L.dito_gated_residual_adaln_tok.argtypes = [_u16p, _u16p, _f64p, _f64p, _f64p, _i64,
                                                    _i64, _u8p, _int, _int, _i64, _int, _dbl,
                                                    _u16p, _f64p, _f64p]
        L.dito_adaln_modulate_tok.restype = _int
        L.dito_gated_residual_adaln_tok.restype = _int
        _i64p = ctypes.POINTER(ctypes.c_int64)
        L.dito_swiglu_gemm.argtypes = [_u16p, _u16p, _i64, _int, _int, _i64p, _i64, _f64p,
                                       _f64p, _f64p]
        L.dito_swiglu_gemm.restype = _int
        L.dito_gemm_gated_residual.argtypes = [_u16p, _u16p, _u16p, _f64p, _i64, _i64, _i64,
                                               _int, _int, _i64p, _i64, _u16p, _f64p, _f64p]
        L.dito_gemm_gated_residual.restype = _int
        L.dito_subblock_keep_count.argtypes = [_i64, _dbl]
        L.dito_subblock_keep_count.restype = _int
        L.dito_subblock_router.argtypes = [_u16p, _u16p, _i64, _int, _i64, _int, _int, _int, _dbl,
                                           ctypes.POINTER(ctypes.c_int32), _f64p, _f64p]
        L.dito_subblock_router.restype = _int
        L.dito_block_sparse_attention.argtypes = [_u16p, _u16p, _u16p, _i64, _int, _i64, _int,
                                                  _int, _int, ctypes.POINTER(ctypes.c_int32),
                                                  _int, _dbl, ctypes.POINTER(ctypes.c_int64),
                                                  _i64, _f64p, _f64p]
        L.dito_block_sparse_attention.restype = _int
        L.dito_residual_store.argtypes = [_u16p, _u16p, _i64, _u16p]
        L.dito_residual_apply.argtypes = [_u16p, _u16p, _i64, _u16p]
        for name in ("dito_adaln_modulate", "dito_gated_residual_adaln", "dito_swiglu",
                     "dito_grid_positions", "dito_qk_rmsnorm_rope3d",
                     "dito_qk_rmsnorm_rope3d_ex", "dito_cachedit_residual_diff"):
            getattr(L, name).restype = _int
        self.lib = L

    # ------------------------------------------------------------- bf16

    def bf16_to_f64(self, h: np.ndarray) -> np.ndarray:
        h = _c(h, np.uint16)
        out = np.empty(h.shape, dtype=np.float64)
        self.lib.dito_widen_bf16(_p(h, _u16p), _p(out, _f64p), h.size)
        return out

    def f64_to_bf16(self, v: np.ndarray) -> np.ndarray:
        v = _c(v, np.float64)
        out = np.empty(v.shape, dtype=np.uint16)
        self.lib.dito_round_bf16(_p(v, _f64p), _p(out, _u16p), v.size)
        return out

    def f64_to_bf16_scalar(self, v: float) -> int:
        return int(self.lib.dito_f64_to_bf16(float(v)))

    # -------------------------------------------------------- operators

    def adaln_modulate(self, x, shift, scale, eps):
        """x: [B,N,D] bf16 bits; shift, scale: [B,D]. Returns y [B,N,D] fp64."""
        x = _c(x, np.uint16)
        B, N, D = x.shape
        shift = _c(shift, np.float64).reshape(B, D)
        scale = _c(scale, np.float64).reshape(B, D)
        y = np.empty((B, N, D), dtype=np.float64)
        work = np.empty(D, dtype=np.float64)
        _check(self.lib.dito_adaln_modulate(_p(x, _u16p), _p(shift, _f64p), _p(scale, _f64p), D,
                                            B, N, D, eps, _p(y, _f64p), _p(work, _f64p)),
               "adaln_modulate")
        return y

    def adaln_modulate_tok(self, x, shift, scale, set_index, eps):
        """x: [B,N,D] bf16 bits; shift, scale: [B,S,D] (S modulation sets);
        set_index: [B,N] uint8. Token (b, n) uses set set_index[b, n].
        Returns y [B,N,D] fp64."""
        x = _c(x, np.uint16)
        B, N, D = x.shape
        shift = _c(shift, np.float64).reshape(B, -1, D)
        S = shift.shape[1]
        scale = _c(scale, np.float64).reshape(B, S, D)
        idx = _c(set_index, np.uint8).reshape(B, N)
        y = np.empty((B, N, D), dtype=np.float64)
        work = np.empty(D, dtype=np.float64)
        _check(self.lib.dito_adaln_modulate_tok(
            _p(x, _u16p), _p(shift, _f64p), _p(scale, _f64p), S * D, D,
            _p(idx, _u8p), S, B, N, D, eps, _p(y, _f64p),
            _p(work, _f64p)), "adaln_modulate_tok")
        return y

    def gated_residual_adaln_tok(self, x, r, gate, shift, scale, set_index, eps):
        """As gated_residual_adaln with [B,S,D] modulation sets chosen per
        token by set_index [B,N] uint8. Returns (x_out bits, y fp64)."""
        x = _c(x, np.uint16)
        r = _c(r, np.uint16)
        B, N, D = x.shape
        gate = _c(gate, np.float64).reshape(B, -1, D)
        S = gate.shape[1]
        shift = _c(shift, np.float64).reshape(B, S, D)
        scale = _c(scale, np.float64).reshape(B, S, D)
        idx = _c(set_index, np.uint8).reshape(B, N)
        x_out = np.empty((B, N, D), dtype=np.uint16)
        y = np.empty((B, N, D), dtype=np.float64)
        work = np.empty(D, dtype=np.float64)
        _check(self.lib.dito_gated_residual_adaln_tok(
            _p(x, _u16p), _p(r, _u16p), _p(gate, _f64p), _p(shift, _f64p), _p(scale, _f64p),
            S * D, D, _p(idx, _u8p), S, B, N, D, eps,
            _p(x_out, _u16p), _p(y, _f64p), _p(work, _f64p)), "gated_residual_adaln_tok")
        return x_out, y

    def gated_residual_adaln(self, x, r, gate, shift, scale, eps):
        """x, r: [B,N,D] bf16 bits; gate/shift/scale [B,D].
        Returns (x_out [B,N,D] bf16 bits, y [B,N,D] fp64)."""
        x = _c(x, np.uint16)
        r = _c(r, np.uint16)
        B, N, D = x.shape
        gate = _c(gate, np.float64).reshape(B, D)
        shift = _c(shift, np.float64).reshape(B, D)
        scale = _c(scale, np.float64).reshape(B, D)
        x_out = np.empty((B, N, D), dtype=np.uint16)
        y = np.empty((B, N, D), dtype=np.float64)
        work = np.empty(D, dtype=np.float64)
        _check(self.lib.dito_gated_residual_adaln(_p(x, _u16p), _p(r, _u16p), _p(gate, _f64p),
                                                  _p(shift, _f64p), _p(scale, _f64p), D, B, N, D,
                                                  eps, _p(x_out, _u16p), _p(y, _f64p),
                                                  _p(work, _f64p)),
               "gated_residual_adaln")
        return x_out, y

    def swiglu(self, inp):
        """inp: [M, 2F] bf16 bits. Returns [M, F] fp64."""
        inp = _c(inp, np.uint16)
        M, F2 = inp.shape
        if F2 % 2:
            raise ValueError("swiglu input width must be even")
        F = F2 // 2
        out = np.empty((M, F), dtype=np.float64)
        _check(self.lib.dito_swiglu(_p(inp, _u16p), M, F, _p(out, _f64p)), "swiglu")
        return out

    def grid_positions(self, T, Hg, Wg, offset, N):
        """[N, 3] int32 (t, h, w) of global tokens offset .. offset+N-1."""
        pos = np.empty((N, 3), dtype=np.int32)
        _check(self.lib.dito_grid_positions(T, Hg, Wg, offset, N, _p(pos, _i32p)),
               "grid_positions")
        return pos

    def qk_rmsnorm_rope3d(self, x, w, H, hd, pos, pairs, theta, eps, row_stride=None):
        """x: token rows of bf16 bits ([R, row_stride] or [..., H*hd]); w: [hd];
        pos: [R, 3] int32. Returns [R, H*hd] fp64."""
        x = _c(x, np.uint16)
        if row_stride is None:
            row_stride = x.shape[-1]
        R = x.size // row_stride
        w = _c(w, np.float64).reshape(hd)
        pos = _c(pos, np.int32).reshape(R, 3)
        out = np.empty((R, H * hd), dtype=np.float64)
        work = np.empty(hd, dtype=np.float64)
        pt, ph, pw = pairs
        _check(self.lib.dito_qk_rmsnorm_rope3d(_p(x, _u16p), row_stride, _p(w, _f64p), 1, R, H,
                                               hd, _p(pos, _i32p), pt, ph, pw, theta, eps,
                                               _p(out, _f64p), _p(work, _f64p)),
               "qk_rmsnorm_rope3d")
        return out

    def qk_rmsnorm_rope3d_ex(self, x, w, H, hd, pos, pairs, theta, eps, layout=0, norm=0,
                             row_stride=None):
        """As qk_rmsnorm_rope3d with the two options: layout 0 interleaved pairs,
        1 rotate-half pairs; norm 0 per-head RMS with w [hd], 1 whole-row RMS with
        w [H*hd]. Returns [R, H*hd] fp64."""
        x = _c(x, np.uint16)
        if row_stride is None:
            row_stride = x.shape[-1]
        R = x.size // row_stride
        w = _c(w, np.float64).reshape(-1)
        if w.size != (hd if norm == 0 else H * hd):
            raise ValueError("weight size does not match the norm option")
        pos = _c(pos, np.int32).reshape(R, 3)
        out = np.empty((R, H * hd), dtype=np.float64)
        work = np.empty(H * hd, dtype=np.float64)
        pt, ph, pw = pairs
        _check(self.lib.dito_qk_rmsnorm_rope3d_ex(_p(x, _u16p), row_stride, _p(w, _f64p), 1, R, H,
                                                  hd, _p(pos, _i32p), pt, ph, pw, theta, eps,
                                                  layout, norm, _p(out, _f64p), _p(work, _f64p)),
               "qk_rmsnorm_rope3d_ex")
        return out

    def swiglu_gemm(self, x, w, rows=None):
        """x: [M, K] bf16 bits, w: [2F, K] bf16 bits (gate rows, then linear
        rows). Returns (out [R, F] fp64, g_abs, u_abs) for the rows `rows`
        of x (all when None); g_abs / u_abs are the sums of |x w| per output."""
        x = _c(x, np.uint16)
        w = _c(w, np.uint16)
        M, K = x.shape
        F = w.shape[0] // 2
        if w.shape != (2 * F, K):
            raise ValueError("w must be [2F, K]")
        r = None if rows is None else _c(rows, np.int64)
        R = M if r is None else r.size
        out = np.empty((R, F), dtype=np.float64)
        ga = np.empty((R, F), dtype=np.float64)
        ua = np.empty((R, F), dtype=np.float64)
        _check(self.lib.dito_swiglu_gemm(
            _p(x, _u16p), _p(w, _u16p), M, K, F,
            None if r is None else r.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)), R,
            _p(out, _f64p), _p(ga, _f64p), _p(ua, _f64p)), "swiglu_gemm")
        return out, ga, ua

    def gemm_gated_residual(self, h, w, x, gate, N, rows=None):
        """h: [M, K] bf16 bits, w: [D, K] bf16 bits, x: [M, D] bf16 bits,
        gate: [B, D] (B = M / N samples of N token rows).  Returns
        (x_out [R, D] bf16 bits, dot [R, D] fp64, abs_dot [R, D] fp64) for the
        rows `rows` (all when None)."""
        h = _c(h, np.uint16)
        w = _c(w, np.uint16)
        x = _c(x, np.uint16)
        M, K = h.shape
        D = w.shape[0]
        if w.shape != (D, K) or x.shape != (M, D):
            raise ValueError("shapes do not match")
        gate = _c(gate, np.float64).reshape(-1, D)
        r = None if rows is None else _c(rows, np.int64)
        R = M if r is None else r.size
        out = np.empty((R, D), dtype=np.uint16)
        dot = np.empty((R, D), dtype=np.float64)
        ad = np.empty((R, D), dtype=np.float64)
        _check(self.lib.dito_gemm_gated_residual(
            _p(h, _u16p), _p(w, _u16p), _p(x, _u16p), _p(gate, _f64p), D, M, N, K, D,
            None if r is None else r.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)), R,
            _p(out, _u16p), _p(dot, _f64p), _p(ad, _f64p)), "gemm_gated_residual")
        return out, dot, ad

    def subblock_keep_count(self, n_blocks, sparsity):
        n = self.lib.dito_subblock_keep_count(int(n_blocks), float(sparsity))
        _check(0 if n > 0 else n, "subblock_keep_count")
        return n

    def subblock_router(self, q, k, B, H, hd, block, sparsity, row_stride=None):
        """q, k: [B*N, >= H*hd] bf16 bits (rows `row_stride` apart).  Returns
        (kept [B, H, n_blocks, n_keep] int32, scores [B, H, n_blocks, n_blocks]
        fp64)."""
        q = _c(q, np.uint16)
        k = _c(k, np.uint16)
        if row_stride is None:
            row_stride = q.shape[-1]
        N = q.size // row_stride // B
        nb = (N + block - 1) // block
        n_keep = self.subblock_keep_count(nb, sparsity)
        kept = np.empty((B, H, nb, n_keep), dtype=np.int32)
        scores = np.empty((B, H, nb, nb), dtype=np.float64)
        work = np.empty(2 * nb * hd + 2 * nb, dtype=np.float64)
        rc = self.lib.dito_subblock_router(_p(q, _u16p), _p(k, _u16p), row_stride, B, N, H, hd,
                                           block, sparsity,
                                           kept.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)),
                                           _p(scores, _f64p), _p(work, _f64p))
        _check(0 if rc > 0 else rc, "subblock_router")
        return kept, scores

    def block_sparse_attention(self, q, k, v, B, H, hd, block, kept, scale=None,
                               row_stride=None, rows=None):
        """q, k, v: [B*N, >= H*hd] bf16 bits; kept: [B, H, n_blocks, n_keep]
        int32.  Returns out [R, H*hd] fp64 for the query rows `rows` (b*N + t;
        all B*N when None)."""
        q = _c(q, np.uint16)
        k = _c(k, np.uint16)
        v = _c(v, np.uint16)
        if row_stride is None:
            row_stride = q.shape[-1]
        N = q.size // row_stride // B
        kept = _c(kept, np.int32)
        n_keep = kept.shape[-1]
        if scale is None:
            scale = 1.0 / np.sqrt(hd)
        r = None if rows is None else _c(rows, np.int64)
        R = B * N if r is None else r.size
        out = np.empty((R, H * hd), dtype=np.float64)
        work = np.empty(n_keep * block, dtype=np.float64)
        _check(self.lib.dito_block_sparse_attention(
            _p(q, _u16p), _p(k, _u16p), _p(v, _u16p), row_stride, B, N, H, hd, block,
            kept.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)), n_keep, float(scale),
            None if r is None else r.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)), R,
            _p(out, _f64p), _p(work, _f64p)), "block_sparse_attention")
        return out

    def residual_store(self, before, after):
        """R = bf16(after - before), elementwise on bf16 bits."""
        before = _c(before, np.uint16)
        after = _c(after, np.uint16)
        if before.shape != after.shape:
            raise ValueError("shapes differ")
        out = np.empty(before.shape, dtype=np.uint16)
        self.lib.dito_residual_store(_p(before, _u16p), _p(after, _u16p), before.size,
                                     _p(out, _u16p))
        return out

    def residual_apply(self, h, residual):
        """out = bf16(h + R), elementwise on bf16 bits."""
        h = _c(h, np.uint16)
        residual = _c(residual, np.uint16)
        if h.shape != residual.shape:
            raise ValueError("shapes differ")
        out = np.empty(h.shape, dtype=np.uint16)
        self.lib.dito_residual_apply(_p(h, _u16p), _p(residual, _u16p), h.size, _p(out, _u16p))
        return out

    def cachedit_sums(self, prev, cur):
        """(sum |cur - prev|, sum |prev|) over all elements, fp64."""
        prev = _c(prev, np.uint16)
        cur = _c(cur, np.uint16)
        if prev.size != cur.size:
            raise ValueError("size mismatch")
        num = ctypes.c_double()
        den = ctypes.c_double()
        self.lib.dito_cachedit_sums(_p(prev, _u16p), _p(cur, _u16p), prev.size,
                                    ctypes.byref(num), ctypes.byref(den))
        return num.value, den.value

    def cachedit_decide(self, num, den, threshold):
        """(rel, reuse) from the two sums."""
        rel = ctypes.c_double()
        reuse = self.lib.dito_cachedit_decide(num, den, threshold, ctypes.byref(rel))
        return rel.value, int(reuse)

    def cachedit_residual_diff(self, prev, cur, threshold):
        """prev, cur: [B,N,D] bf16 bits. Returns (rel [B] fp64, reuse [B] uint8)."""
        prev = _c(prev, np.uint16)
        cur = _c(cur, np.uint16)
        B, N, D = prev.shape
        rel = np.empty(B, dtype=np.float64)
        reuse = np.empty(B, dtype=np.uint8)
        _check(self.lib.dito_cachedit_residual_diff(_p(prev, _u16p), _p(cur, _u16p), B, N, D,
                                                    threshold, _p(rel, _f64p), _p(reuse, _u8p)),
               "cachedit_residual_diff")
        return rel, reuse


_default = None
_lock = threading.Lock()


def default() -> Oracle:
    global _default
    with _lock:
        if _default is None:
            _default = Oracle()
    return _default


def __getattr__(name):
    # module-level access to the default oracle's methods: oracle.swiglu(...)
    if name.startswith("_"):
        raise AttributeError(name)
    return getattr(default(), name)


def cache_policy(rels, threshold, warmup_steps=0, max_cached_steps=0):
    """The Cache-DiT reuse rule over a denoising run, one decision per step.

    [REPORT], section "Só com três camadas de aceleração somadas chega-se a 6
    vezes": a residual-difference threshold decides whether a step reuses
    the results cached between neighbouring steps (0.04 conservative, 0.08 in
    the more aggressive stride mode).  rels[t] is the relative L1 difference
    of step t's first-block residual against step t-1's (rels[0] is ignored:
    the first step has nothing to compare with).  Step t reuses iff
        t >= 1 and t >= warmup_steps and rels[t] < threshold
        and (max_cached_steps == 0 or fewer than max_cached_steps steps in a
             row before t reused).
    Readings: the comparison is always with the previous step (neighbouring
    steps); warm-up and the cap on consecutive reuses are optional guards
    (0 = off) that the pages do not mention.  Returns a list of bools.
    """
    out = []
    run = 0
    for t, rel in enumerate(rels):
        reuse = (t >= 1 and t >= warmup_steps and rel < threshold
                 and (max_cached_steps == 0 or run < max_cached_steps))
        run = run + 1 if reuse else 0
        out.append(reuse)
    return out
