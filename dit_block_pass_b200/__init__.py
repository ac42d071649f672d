"""dit_block_pass_b200: B200-native (sm_100a) memory-bound operators of one
block of a dense single-stream video+audio diffusion transformer
(MiniMax-H3 shaped).

The compute lives in ``libdit_block.so`` (hand-written CUDA, C ABI declared in
``include/dit_block.h``).  This module only marshals torch tensors into that
ABI: it checks devices, dtypes and strides, passes raw pointers and the
current CUDA stream, and turns a negative status into an exception.  There
is no CPU fallback: without the built library every call raises.

Operators (see the header for the definitions):
  adaln_modulate, gated_residual_adaln, swiglu, qk_rmsnorm_rope3d,
  cachedit_residual_diff, cachedit_residual_sums, cachedit_decide.
"""
from __future__ import annotations

import ctypes
import os
import threading
from typing import Optional, Sequence

import torch

__all__ = [
    "DitError", "library", "library_path", "adaln_modulate", "gated_residual_adaln", "swiglu",
    "qk_rmsnorm_rope3d", "cachedit_workspace_bytes", "cachedit_residual_diff",
    "cachedit_residual_sums", "cachedit_decide", "cachedit_residual_diff_noalloc",
    "launch_counts", "QKOut", "CachePolicy", "swiglu_gemm", "gemm_gated_residual",
    "subblock_keep_count", "subblock_router", "subblock_router_means", "block_sparse_attention",
    "cachedit_residual_store",
    "cachedit_residual_apply", "F32", "BF16", "ROPE_INTERLEAVED", "ROPE_HALF", "NORM_HEAD", "NORM_ROW",
]

F32, BF16 = 0, 1
# options of qk_rmsnorm_rope3d
ROPE_INTERLEAVED, ROPE_HALF = 0, 1     # rotation pairs (2p, 2p+1) or (p, p + hd/2)
NORM_HEAD, NORM_ROW = 0, 1             # RMS over each head or over the whole H*hd row
_PKG = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_PKG, "libdit_block.so")
_lib = None
_lock = threading.Lock()

# kernels launched per call of each entry point (for launch accounting)
launch_counts = {
    "adaln_modulate": 1, "gated_residual_adaln": 1, "swiglu": 1, "qk_rmsnorm_rope3d": 1,
    "qk_rmsnorm_rope3d_ex": 1, "adaln_modulate_tok": 1, "gated_residual_adaln_tok": 1,
    "cachedit_residual_diff": 2, "cachedit_residual_sums": 2, "cachedit_decide": 1,
    "cachedit_residual_diff_noalloc": 2, "cachedit_residual_store": 1,
    "cachedit_residual_apply": 1, "swiglu_gemm": 1, "gemm_gated_residual": 1,
    "subblock_router": 4, "block_sparse_attention": 1, "qk_rmsnorm_rope3d_pooled": 1,
    "subblock_router_means": 3,        # 2 when hd is not a multiple of 32
}


class QKOut(ctypes.Structure):
    """dit_qk_out: output buffers and [B, N, H, hd] element strides."""
    _fields_ = [("q", ctypes.c_void_p), ("k", ctypes.c_void_p), ("stride_b", ctypes.c_int64),
                ("stride_n", ctypes.c_int64), ("stride_h", ctypes.c_int64)]


class CachePolicyStruct(ctypes.Structure):
    """dit_cache_policy."""
    _fields_ = [("threshold", ctypes.c_double), ("warmup_steps", ctypes.c_int),
                ("max_cached_steps", ctypes.c_int), ("step", ctypes.c_int), ("run", ctypes.c_int),
                ("computed", ctypes.c_int), ("reused", ctypes.c_int)]


class DitError(RuntimeError):
    def __init__(self, fn: str, status: int, msg: str):
        super().__init__(f"{fn} failed with status {status}: {msg}")
        self.status = status


def library_path() -> str:
    return _LIB_PATH


def library() -> ctypes.CDLL:
    """The loaded C library; raises if it has not been built."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(_LIB_PATH):
                raise RuntimeError(
                    f"{_LIB_PATH} is missing: build it with "
                    "`python -m dit_block_pass_b200.build` (nvcc, sm_100a). "
                    "There is no CPU fallback.")
            L = ctypes.CDLL(_LIB_PATH)
            vp, i64, i32, dbl, sz = (ctypes.c_void_p, ctypes.c_int64, ctypes.c_int,
                                     ctypes.c_double, ctypes.c_size_t)
            L.dit_abi_version.restype = i32
            L.dit_status_string.restype = ctypes.c_char_p
            L.dit_status_string.argtypes = [i32]
            L.dit_adaln_modulate.argtypes = [vp, vp, vp, vp, i32, i64, i32, i64, i32, dbl, vp]
            L.dit_gated_residual_adaln.argtypes = [vp, vp, vp, vp, vp, vp, vp, i32, i64, i32,
                                                   i64, i32, dbl, vp]
            L.dit_swiglu.argtypes = [vp, vp, i64, i32, vp]
            L.dit_adaln_modulate_tok.argtypes = [vp, vp, vp, vp, i32, i64, i64, vp, i32, i32,
                                                 i64, i32, dbl, vp]
            L.dit_gated_residual_adaln_tok.argtypes = [vp, vp, vp, vp, vp, vp, vp, i32, i64,
                                                       i64, vp, i32, i32, i64, i32, dbl, vp]
            L.dit_qk_rmsnorm_rope3d.argtypes = [vp, vp, i64, vp, vp, i32, i32, i64, i32, i32,
                                                i32, i32, i32, vp, i64, i32, i32, i32, dbl, dbl,
                                                vp]
            L.dit_qk_rmsnorm_rope3d_ex.argtypes = [vp, vp, i64, vp, vp, i32, i32, i64, i32,
                                                   i32, i32, i32, i32, vp, i64, i32, i32, i32,
                                                   dbl, dbl, i32, i32,
                                                   ctypes.POINTER(QKOut), vp]
            L.dit_qk_rmsnorm_rope3d_pooled.argtypes = [vp, vp, i64, vp, vp, i32, i32, i64, i32,
                                                       i32, i32, i32, i32, vp, i64, i32, i32,
                                                       i32, dbl, dbl, i32, i32, vp, vp, vp]
            L.dit_qk_rmsnorm_rope3d_pooled_stall_test.argtypes = [
                vp, vp, i64, vp, vp, i32, i32, i64, i32, i32, i32, i32, i32, vp, i64, i32, i32,
                i32, dbl, dbl, i32, i32, vp, vp, vp]
            L.dit_subblock_means_workspace_bytes.argtypes = [i32, i64, i32, i32, i32]
            L.dit_subblock_means_workspace_bytes.restype = sz
            L.dit_subblock_router_means.argtypes = [vp, i32, i64, i32, i32, i32, dbl, vp, vp, sz,
                                                    vp, vp]
            L.dit_swiglu_gemm.argtypes = [vp, vp, vp, i64, i32, i32, vp, vp]
            L.dit_block_sparse_attention.argtypes = [vp, vp, vp, i64, vp, i64, i32, i64, i32,
                                                     i32, i32, vp, i32, dbl, vp, vp]
            L.dit_block_sparse_attention_stall_test.argtypes = [vp, vp, vp, i64, vp, i64, i32,
                                                                i64, i32, i32, i32, vp, i32,
                                                                dbl, vp, vp]
            L.dit_subblock_keep_count.argtypes = [i64, dbl]
            L.dit_subblock_workspace_bytes.argtypes = [i32, i64, i32, i32, i32]
            L.dit_subblock_workspace_bytes.restype = sz
            L.dit_subblock_router.argtypes = [vp, vp, i64, i32, i64, i32, i32, i32, dbl, vp, vp,
                                              sz, vp, vp]
            L.dit_swiglu_gemm_stall_test.argtypes = [vp, vp, vp, i64, i32, i32, vp, vp]
            L.dit_subblock_scores_stall_test.argtypes = [vp, i32, i64, i32, i32, i32, vp, sz, vp,
                                                         vp]
            L.dit_gemm_gated_residual.argtypes = [vp, vp, vp, vp, vp, i32, i64, i32, i64, i32,
                                                  i32, vp, vp]
            L.cachedit_residual_store.argtypes = [vp, vp, vp, i64, vp]
            L.cachedit_residual_apply.argtypes = [vp, vp, vp, i64, vp]
            L.dit_cache_policy_init.argtypes = [ctypes.POINTER(CachePolicyStruct), dbl, i32, i32]
            L.dit_cache_policy_decide.argtypes = [ctypes.POINTER(CachePolicyStruct), dbl]
            L.cachedit_workspace_bytes.restype = sz
            L.cachedit_workspace_bytes.argtypes = [i32, i64, i32]
            L.cachedit_residual_diff.argtypes = [vp, vp, i32, i64, i32, dbl, vp, vp, vp, sz, vp]
            L.cachedit_residual_sums.argtypes = [vp, vp, i32, i64, i32, vp, vp, sz, vp]
            L.cachedit_decide.argtypes = [vp, i32, i32, dbl, vp, vp, vp]
            L.cachedit_residual_diff_noalloc.argtypes = [vp, vp, i32, i64, i32, dbl, vp, vp, vp]
            L.cachedit_residual_diff_noalloc.restype = i32
            for name in ("dit_adaln_modulate", "dit_gated_residual_adaln", "dit_swiglu",
                         "dit_adaln_modulate_tok", "dit_gated_residual_adaln_tok",
                         "cachedit_residual_store", "cachedit_residual_apply", "dit_swiglu_gemm",
                         "dit_gemm_gated_residual", "dit_subblock_keep_count",
                         "dit_swiglu_gemm_stall_test", "dit_subblock_scores_stall_test",
                         "dit_block_sparse_attention_stall_test",
                         "dit_qk_rmsnorm_rope3d_pooled_stall_test",
                         "dit_subblock_router", "dit_block_sparse_attention",
                         "dit_cache_policy_init", "dit_cache_policy_decide",
                         "dit_qk_rmsnorm_rope3d", "dit_qk_rmsnorm_rope3d_ex",
                         "dit_qk_rmsnorm_rope3d_pooled", "dit_subblock_router_means",
                         "cachedit_residual_diff",
                         "cachedit_residual_sums", "cachedit_decide"):
                getattr(L, name).restype = i32
            _lib = L
    return _lib


def _call(name: str, *args) -> None:
    L = library()
    st = getattr(L, name)(*args)
    if st != 0:
        raise DitError(name, st, L.dit_status_string(st).decode())


def _stream(t: torch.Tensor) -> int:
    return torch.cuda.current_stream(t.device).cuda_stream


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _need_cuda_bf16(name: str, t: torch.Tensor) -> None:
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor (there is no CPU path)")
    if t.dtype != torch.bfloat16:
        raise ValueError(f"{name} must be bfloat16, got {t.dtype}")


def _mod_dtype(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return F32
    if t.dtype == torch.bfloat16:
        return BF16
    raise ValueError(f"modulation/weight dtype must be float32 or bfloat16, got {t.dtype}")


def _mod_views(B: int, D: int, *mods: torch.Tensor):
    """Modulation vectors as [B, D] views (any batch stride, unit inner
    stride); returns (dtype code, batch stride in elements)."""
    dt = _mod_dtype(mods[0])
    stride = None
    for m in mods:
        if m.dtype != mods[0].dtype or not m.is_cuda or m.device != mods[0].device:
            raise ValueError("modulation vectors must share dtype and device")
        if m.dim() == 1:
            m = m.reshape(1, -1)
        if m.shape[-1] != D or m.stride(-1) != 1 or m.shape[0] not in (1, B):
            raise ValueError(f"modulation must be [B, D] (or [D]) with unit inner stride, got "
                             f"{tuple(m.shape)}")
        s = 0 if m.shape[0] == 1 else m.stride(0)
        if stride is None:
            stride = s
        elif s != stride:
            raise ValueError("modulation vectors must share one batch stride")
    return dt, stride


def _set_views(B: int, N: int, D: int, set_index: torch.Tensor, *mods: torch.Tensor):
    """Per-token modulation: vectors as [B, S, D] views (unit inner stride,
    shared strides; a sample stride of 0 broadcasts) and set_index [B, N]
    uint8.  Returns (dtype code, sample stride, set stride, S)."""
    dt = _mod_dtype(mods[0])
    if set_index.dtype != torch.uint8 or not set_index.is_cuda or \
            set_index.numel() != B * N or not set_index.is_contiguous():
        raise ValueError("set_index must be a contiguous CUDA uint8 [B, N] tensor")
    strides = None
    S = None
    for m in mods:
        if m.dtype != mods[0].dtype or not m.is_cuda or m.device != set_index.device:
            raise ValueError("modulation vectors must share dtype and device")
        if m.dim() != 3 or m.shape[0] not in (1, B) or m.shape[2] != D or m.stride(2) != 1:
            raise ValueError(f"modulation must be [B, S, D] with unit inner stride, got "
                             f"{tuple(m.shape)}")
        st = (0 if m.shape[0] == 1 else m.stride(0), m.stride(1))
        if strides is not None and (st != strides or m.shape[1] != S):
            raise ValueError("modulation vectors must share shape and strides")
        strides, S = st, m.shape[1]
    if not 1 <= S <= 255:
        raise ValueError("between 1 and 255 modulation sets")
    return dt, strides[0], strides[1], S


def _result_buffers(prev: torch.Tensor, B: int, rel: Optional[torch.Tensor],
                    reuse: Optional[torch.Tensor]):
    """The Cache-DiT outputs: caller tensors are checked before the kernel
    writes B float64 and B uint8 values through their pointers (contiguous,
    on prev's device, at least B elements); None allocates them."""
    rel = torch.empty(B, dtype=torch.float64, device=prev.device) if rel is None else rel
    reuse = torch.empty(B, dtype=torch.uint8, device=prev.device) if reuse is None else reuse
    for nm, t, dt in (("rel", rel, torch.float64), ("reuse", reuse, torch.uint8)):
        if not isinstance(t, torch.Tensor) or t.dtype != dt or t.device != prev.device or \
                not t.is_contiguous() or t.numel() < B:
            raise ValueError(f"{nm} must be a contiguous {dt} tensor of at least {B} elements "
                             f"on {prev.device}")
    return rel, reuse


def _rows3(name: str, t: torch.Tensor):
    if t.dim() != 3 or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous [B, N, D] tensor")
    return t.shape


# ---------------------------------------------------------------- operators


def adaln_modulate(x: torch.Tensor, shift: torch.Tensor, scale: torch.Tensor, eps: float = 1e-6,
                   out: Optional[torch.Tensor] = None,
                   set_index: Optional[torch.Tensor] = None) -> torch.Tensor:
    """y = LN(x) * (1 + scale) + shift per sample; x [B, N, D] bf16.  With
    ``set_index`` ([B, N] uint8) shift and scale are [B, S, D] modulation sets
    and token (b, n) uses set set_index[b, n] (an index >= S gives NaN)."""
    _need_cuda_bf16("x", x)
    B, N, D = _rows3("x", x)
    y = torch.empty_like(x) if out is None else out
    _need_cuda_bf16("out", y)
    if y.shape != x.shape or not y.is_contiguous():
        raise ValueError("out must match x")
    if set_index is None:
        dt, ms = _mod_views(B, D, shift, scale)
        _call("dit_adaln_modulate", x.data_ptr(), y.data_ptr(), shift.data_ptr(),
              scale.data_ptr(), dt, ms, B, N, D, float(eps), _stream(x))
        return y
    dt, ms, ss, S = _set_views(B, N, D, set_index, shift, scale)
    _call("dit_adaln_modulate_tok", x.data_ptr(), y.data_ptr(), shift.data_ptr(),
          scale.data_ptr(), dt, ms, ss, set_index.data_ptr(), S, B, N, D, float(eps), _stream(x))
    return y


def gated_residual_adaln(x: torch.Tensor, r: torch.Tensor, gate: torch.Tensor,
                         shift: torch.Tensor, scale: torch.Tensor, eps: float = 1e-6,
                         x_out: Optional[torch.Tensor] = None, y: Optional[torch.Tensor] = None,
                         set_index: Optional[torch.Tensor] = None):
    """x' = bf16(x + gate * r); y = AdaLN(x'). Returns (x', y).  With
    ``set_index`` ([B, N] uint8) gate, shift and scale are [B, S, D]
    modulation sets chosen per token (an index >= S gives NaN)."""
    _need_cuda_bf16("x", x)
    _need_cuda_bf16("r", r)
    B, N, D = _rows3("x", x)
    if r.shape != x.shape or not r.is_contiguous():
        raise ValueError("r must match x")
    if set_index is None:
        dt, ms = _mod_views(B, D, gate, shift, scale)
    else:
        dt, ms, ss, S = _set_views(B, N, D, set_index, gate, shift, scale)
    x_out = torch.empty_like(x) if x_out is None else x_out
    y = torch.empty_like(x) if y is None else y
    for nm, t in (("x_out", x_out), ("y", y)):
        _need_cuda_bf16(nm, t)
        if t.shape != x.shape or not t.is_contiguous():
            raise ValueError(f"{nm} must match x")
    if set_index is None:
        _call("dit_gated_residual_adaln", x.data_ptr(), r.data_ptr(), x_out.data_ptr(),
              y.data_ptr(), gate.data_ptr(), shift.data_ptr(), scale.data_ptr(), dt, ms, B, N, D,
              float(eps), _stream(x))
    else:
        _call("dit_gated_residual_adaln_tok", x.data_ptr(), r.data_ptr(), x_out.data_ptr(),
              y.data_ptr(), gate.data_ptr(), shift.data_ptr(), scale.data_ptr(), dt, ms, ss,
              set_index.data_ptr(), S, B, N, D, float(eps), _stream(x))
    return x_out, y


def swiglu(inp: torch.Tensor, out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """out = silu(inp[..., :F]) * inp[..., F:]; inp [..., 2F] bf16 contiguous."""
    _need_cuda_bf16("inp", inp)
    if not inp.is_contiguous() or inp.shape[-1] % 2:
        raise ValueError("inp must be contiguous with an even last dimension")
    F = inp.shape[-1] // 2
    M = inp.numel() // max(1, inp.shape[-1])
    if out is None:
        out = torch.empty(*inp.shape[:-1], F, dtype=inp.dtype, device=inp.device)
    _need_cuda_bf16("out", out)
    if out.numel() != M * F or not out.is_contiguous():
        raise ValueError("out must be contiguous [..., F]")
    _call("dit_swiglu", inp.data_ptr(), out.data_ptr(), M, F, _stream(inp))
    return out


def _token_rows(name: str, t: torch.Tensor, B: int, N: int, width: int) -> int:
    """Row stride (elements) of a [B, N, width] view with unit inner stride and
    uniformly strided token rows."""
    _need_cuda_bf16(name, t)
    if t.dim() != 3 or tuple(t.shape) != (B, N, width) or t.stride(2) != 1:
        raise ValueError(f"{name} must be a [B, N, H*hd] view with unit inner stride")
    rs = t.stride(1)
    if B > 1 and t.stride(0) != N * rs:
        raise ValueError(f"{name}: samples must be uniformly strided token rows")
    return rs


def qk_rmsnorm_rope3d(q: Optional[torch.Tensor], k: Optional[torch.Tensor],
                      w_q: Optional[torch.Tensor], w_k: Optional[torch.Tensor], heads: int,
                      pairs: Sequence[int], grid: Optional[Sequence[int]] = None,
                      pos: Optional[torch.Tensor] = None, pos_offset: int = 0,
                      theta: float = 10000.0, eps: float = 1e-6,
                      rope_layout: int = ROPE_INTERLEAVED, norm_width: int = NORM_HEAD,
                      q_out: Optional[torch.Tensor] = None,
                      k_out: Optional[torch.Tensor] = None,
                      block_means: Optional[torch.Tensor] = None, block: int = 128,
                      status: Optional[torch.Tensor] = None) -> None:
    """In place on q and k ([B, N, H*hd] views, e.g. slices of a fused qkv
    buffer): RMSNorm with weight w, then 3D RoPE with pair split
    ``pairs`` = (t, h, w).  Positions come from ``grid`` = (T, Hg, Wg) (token
    n at global index pos_offset + n) or from ``pos`` [B*N, 3] int32.
    ``norm_width`` NORM_HEAD normalises each head (w: [hd]), NORM_ROW the
    token's whole row (w: [H*hd]); ``rope_layout`` ROPE_INTERLEAVED rotates
    pairs (2p, 2p+1), ROPE_HALF pairs (p, p + hd/2).  With ``q_out``/``k_out``
    ([B, N, H, hd] views with any strides and a contiguous last dimension,
    e.g. ``torch.empty(B, H, N, hd).transpose(1, 2)`` for the head-major
    layout attention reads) q and k are only read and the results go there.
    With ``block_means`` (fp32 [B, 2, ceil(N/block), H*hd], contiguous) the
    call is in place with the per-head norm and also writes the mean of each
    block of ``block`` tokens of the rotated q ([:, 0]) and k ([:, 1]), the
    input of ``subblock_router_means``; ``status`` (int32 CUDA scalar) is set to
    1 if a wait of that path's copy pipeline expired."""
    ref = q if q is not None else k
    if ref is None:
        raise ValueError("q and k cannot both be None")
    B, N, width = ref.shape
    if width % heads:
        raise ValueError("last dimension must be heads * head_dim")
    hd = width // heads
    rs = None
    for nm, t in (("q", q), ("k", k)):
        if t is not None:
            s = _token_rows(nm, t, B, N, width)
            if rs is not None and s != rs:
                raise ValueError("q and k must share the row stride")
            rs = s
    w_dt = None
    for nm, t, w in (("w_q", q, w_q), ("w_k", k, w_k)):
        if t is not None:
            wn = hd if norm_width == NORM_HEAD else width
            if w is None or w.numel() != wn or not w.is_contiguous() or not w.is_cuda:
                raise ValueError(f"{nm} must be a contiguous CUDA [{wn}] tensor")
            d = _mod_dtype(w)
            if w_dt is not None and d != w_dt:
                raise ValueError("w_q and w_k must share a dtype")
            w_dt = d
    if pos is not None:
        if pos.dtype != torch.int32 or not pos.is_contiguous() or pos.numel() != B * N * 3 \
                or not pos.is_cuda:
            raise ValueError("pos must be a contiguous CUDA int32 [B*N, 3] tensor")
        T = Hg = Wg = 0
    else:
        if grid is None:
            raise ValueError("give grid=(T, Hg, Wg) or pos")
        T, Hg, Wg = grid
    pt, ph, pw = pairs
    if block_means is not None:
        nb = (N + block - 1) // block
        if q is None or k is None or q_out is not None or k_out is not None or \
                norm_width != NORM_HEAD:
            raise ValueError("block_means needs q and k, in place, with the per-head norm")
        if status is not None and (status.dtype != torch.int32 or not status.is_cuda):
            raise ValueError("status must be a CUDA int32 tensor")
        if block_means.dtype != torch.float32 or not block_means.is_contiguous() or \
                block_means.device != ref.device or \
                tuple(block_means.shape) != (B, 2, nb, width):
            raise ValueError(f"block_means must be a contiguous float32 [{B}, 2, {nb}, {width}] "
                             f"tensor on {ref.device}")
        _call("dit_qk_rmsnorm_rope3d_pooled", _ptr(q), _ptr(k), rs, _ptr(w_q), _ptr(w_k), w_dt,
              B, N, heads, hd, T, Hg, Wg, _ptr(pos), int(pos_offset), pt, ph, pw, float(theta),
              float(eps), int(rope_layout), int(block), block_means.data_ptr(), _ptr(status),
              _stream(ref))
        return
    out = None
    if q_out is not None or k_out is not None:
        strides = None
        for nm, t, o in (("q_out", q, q_out), ("k_out", k, k_out)):
            if t is None:
                continue
            if o is None:
                raise ValueError(f"{nm} is needed when the outputs are not in place")
            if o.shape != (B, N, heads, hd) or o.stride(-1) != 1 or o.dtype != torch.bfloat16 \
                    or o.device != ref.device:
                raise ValueError(f"{nm} must be a bfloat16 [B, N, H, hd] view with unit inner "
                                 f"stride on {ref.device}")
            s = tuple(o.stride()[:3])
            if strides is not None and s != strides:
                raise ValueError("q_out and k_out must share their strides")
            strides = s
        out = QKOut(_ptr(q_out) if q is not None else None,
                    _ptr(k_out) if k is not None else None, *strides)
    _call("dit_qk_rmsnorm_rope3d_ex", _ptr(q), _ptr(k), rs, _ptr(w_q), _ptr(w_k), w_dt, B, N,
          heads, hd, T, Hg, Wg, _ptr(pos), int(pos_offset), pt, ph, pw, float(theta), float(eps),
          int(rope_layout), int(norm_width), None if out is None else ctypes.byref(out),
          _stream(ref))


def cachedit_workspace_bytes(B: int, N: int, D: int) -> int:
    return int(library().cachedit_workspace_bytes(B, N, D))


def _workspace(prev: torch.Tensor, workspace: Optional[torch.Tensor]) -> torch.Tensor:
    B, N, D = prev.shape
    need = cachedit_workspace_bytes(B, N, D)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=prev.device)
    if workspace.numel() * workspace.element_size() < need or not workspace.is_contiguous() \
            or workspace.device != prev.device:
        raise ValueError(f"workspace needs {need} contiguous bytes on {prev.device}")
    return workspace


def cachedit_residual_diff(prev: torch.Tensor, cur: torch.Tensor, threshold: float,
                           workspace: Optional[torch.Tensor] = None, rel: Optional[torch.Tensor] = None,
                           reuse: Optional[torch.Tensor] = None):
    """Per sample rel = sum|cur-prev| / sum|prev| and reuse = rel < threshold.
    Returns device tensors (rel [B] float64, reuse [B] uint8)."""
    _need_cuda_bf16("prev", prev)
    _need_cuda_bf16("cur", cur)
    B, N, D = _rows3("prev", prev)
    if cur.shape != prev.shape or not cur.is_contiguous():
        raise ValueError("cur must match prev")
    ws = _workspace(prev, workspace)
    rel, reuse = _result_buffers(prev, B, rel, reuse)
    _call("cachedit_residual_diff", prev.data_ptr(), cur.data_ptr(), B, N, D, float(threshold),
          rel.data_ptr(), reuse.data_ptr(), ws.data_ptr(), ws.numel() * ws.element_size(),
          _stream(prev))
    return rel, reuse


def cachedit_residual_sums(prev: torch.Tensor, cur: torch.Tensor,
                           workspace: Optional[torch.Tensor] = None,
                           sums: Optional[torch.Tensor] = None) -> torch.Tensor:
    """[B, 2] float64 device tensor: (sum|cur-prev|, sum|prev|) per sample."""
    _need_cuda_bf16("prev", prev)
    _need_cuda_bf16("cur", cur)
    B, N, D = _rows3("prev", prev)
    if cur.shape != prev.shape or not cur.is_contiguous():
        raise ValueError("cur must match prev")
    ws = _workspace(prev, workspace)
    sums = torch.empty(B, 2, dtype=torch.float64, device=prev.device) if sums is None else sums
    if sums.dtype != torch.float64 or sums.device != prev.device or not sums.is_contiguous() \
            or sums.numel() < 2 * B:
        raise ValueError(f"sums must be a contiguous float64 tensor of at least {2 * B} "
                         f"elements on {prev.device}")
    _call("cachedit_residual_sums", prev.data_ptr(), cur.data_ptr(), B, N, D, sums.data_ptr(),
          ws.data_ptr(), ws.numel() * ws.element_size(), _stream(prev))
    return sums


def cachedit_decide(sums: torch.Tensor, threshold: float):
    """sums: [R, B, 2] float64 device tensor of partial sums (R shards).
    Returns (rel [B] float64, reuse [B] uint8) device tensors."""
    if sums.dtype != torch.float64 or not sums.is_cuda or not sums.is_contiguous():
        raise ValueError("sums must be a contiguous CUDA float64 tensor")
    if sums.dim() == 2:
        sums = sums.unsqueeze(0)
    R, B, two = sums.shape
    if two != 2:
        raise ValueError("sums must be [R, B, 2]")
    rel = torch.empty(B, dtype=torch.float64, device=sums.device)
    reuse = torch.empty(B, dtype=torch.uint8, device=sums.device)
    _call("cachedit_decide", sums.data_ptr(), R, B, float(threshold), rel.data_ptr(),
          reuse.data_ptr(), _stream(sums))
    return rel, reuse


def cachedit_residual_diff_noalloc(prev: torch.Tensor, cur: torch.Tensor, threshold: float,
                                   rel: Optional[torch.Tensor] = None,
                                   reuse: Optional[torch.Tensor] = None):
    """The Cache-DiT check for callers that cannot allocate device memory: the
    library keeps the partial sums in its own fixed 64 KB device array
    instead of a workspace (at most 64 samples).  Pass preallocated ``rel``
    [B] float64 and ``reuse`` [B] uint8 to allocate nothing at all.  Calls
    on one device share that array: order them (one stream, or synchronise)."""
    _need_cuda_bf16("prev", prev)
    _need_cuda_bf16("cur", cur)
    B, N, D = _rows3("prev", prev)
    if cur.shape != prev.shape or not cur.is_contiguous():
        raise ValueError("cur must match prev")
    rel, reuse = _result_buffers(prev, B, rel, reuse)
    _call("cachedit_residual_diff_noalloc", prev.data_ptr(), cur.data_ptr(), B, N, D,
          float(threshold), rel.data_ptr(), reuse.data_ptr(), _stream(prev))
    return rel, reuse


# ------------------------------------------------------ Cache-DiT step cache


def _elementwise(name: str, a: torch.Tensor, b: torch.Tensor, out: Optional[torch.Tensor]):
    for nm, t in (("a", a), ("b", b)):
        _need_cuda_bf16(nm, t)
        if not t.is_contiguous():
            raise ValueError(f"{name}: inputs must be contiguous")
    if a.shape != b.shape:
        raise ValueError(f"{name}: shapes differ")
    out = torch.empty_like(a) if out is None else out
    _need_cuda_bf16("out", out)
    if out.shape != a.shape or not out.is_contiguous():
        raise ValueError(f"{name}: out must match the inputs")
    return out


def cachedit_residual_store(before: torch.Tensor, after: torch.Tensor,
                            out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """The residual blocks added: bf16(after - before), elementwise."""
    out = _elementwise("cachedit_residual_store", before, after, out)
    _call("cachedit_residual_store", before.data_ptr(), after.data_ptr(), out.data_ptr(),
          before.numel(), _stream(before))
    return out


def cachedit_residual_apply(h: torch.Tensor, residual: torch.Tensor,
                            out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """A reusing step: bf16(h + residual), elementwise (out may be h)."""
    out = _elementwise("cachedit_residual_apply", h, residual, out)
    _call("cachedit_residual_apply", h.data_ptr(), residual.data_ptr(), out.data_ptr(),
          h.numel(), _stream(h))
    return out


class CachePolicy:
    """The Cache-DiT reuse rule (dit_cache_policy in the library): call
    decide(rel) once per denoising step; True = reuse the cached residual."""

    def __init__(self, threshold: float = 0.04, warmup_steps: int = 0,
                 max_cached_steps: int = 0):
        self._s = CachePolicyStruct()
        _call("dit_cache_policy_init", ctypes.byref(self._s), float(threshold),
              int(warmup_steps), int(max_cached_steps))

    def decide(self, rel: Optional[float]) -> bool:
        r = library().dit_cache_policy_decide(ctypes.byref(self._s),
                                             float("nan") if rel is None else float(rel))
        if r < 0:
            raise DitError("dit_cache_policy_decide", r, library().dit_status_string(r).decode())
        return bool(r)

    @property
    def step(self) -> int:
        return self._s.step

    @property
    def computed(self) -> int:
        return self._s.computed

    @property
    def reused(self) -> int:
        return self._s.reused


# ------------------------------------------- SwiGLU fused into the up-projection


def swiglu_gemm(x: torch.Tensor, w: torch.Tensor, out: Optional[torch.Tensor] = None,
                status: Optional[torch.Tensor] = None) -> torch.Tensor:
    """out = silu(x @ w[:F].T) * (x @ w[F:].T) on the tensor cores, the
    [M, 2F] product never written.  x [..., K] bf16, w [2F, K] bf16 (gate
    rows, then linear rows); returns [..., F].  ``status`` (int32 CUDA
    scalar) is set to 1 if a wait inside the kernel expired."""
    _need_cuda_bf16("x", x)
    _need_cuda_bf16("w", w)
    if not x.is_contiguous() or not w.is_contiguous() or w.dim() != 2 or w.shape[0] % 2:
        raise ValueError("x must be contiguous [..., K] and w contiguous [2F, K]")
    K = x.shape[-1]
    F = w.shape[0] // 2
    if w.shape[1] != K:
        raise ValueError("w must be [2F, K] with the K of x")
    M = x.numel() // max(1, K)
    if out is None:
        out = torch.empty(*x.shape[:-1], F, dtype=x.dtype, device=x.device)
    _need_cuda_bf16("out", out)
    if out.numel() != M * F or not out.is_contiguous():
        raise ValueError("out must be contiguous [..., F]")
    if status is not None and (status.dtype != torch.int32 or not status.is_cuda):
        raise ValueError("status must be a CUDA int32 tensor")
    _call("dit_swiglu_gemm", x.data_ptr(), w.data_ptr(), out.data_ptr(), M, K, F,
          _ptr(status), _stream(x))
    return out


def gemm_gated_residual(h: torch.Tensor, w: torch.Tensor, x: torch.Tensor, gate: torch.Tensor,
                        x_out: Optional[torch.Tensor] = None,
                        status: Optional[torch.Tensor] = None) -> torch.Tensor:
    """x' = bf16(x + gate_b * (h @ w.T)) on the tensor cores.  h [B, N, K],
    w [D, K], x [B, N, D] bf16; gate [B, D] or [D] (fp32 or bf16, unit inner
    stride).  x_out may be x.  Returns x'."""
    for nm, t in (("h", h), ("w", w), ("x", x)):
        _need_cuda_bf16(nm, t)
        if not t.is_contiguous():
            raise ValueError(f"{nm} must be contiguous")
    if h.dim() != 3 or x.dim() != 3 or w.dim() != 2:
        raise ValueError("h and x must be [B, N, .], w [D, K]")
    B, N, K = h.shape
    D = w.shape[0]
    if w.shape[1] != K or x.shape != (B, N, D):
        raise ValueError("shapes do not match: h [B, N, K], w [D, K], x [B, N, D]")
    dt, gs = _mod_views(B, D, gate)
    x_out = torch.empty_like(x) if x_out is None else x_out
    _need_cuda_bf16("x_out", x_out)
    if x_out.shape != x.shape or not x_out.is_contiguous():
        raise ValueError("x_out must match x")
    if status is not None and (status.dtype != torch.int32 or not status.is_cuda):
        raise ValueError("status must be a CUDA int32 tensor")
    _call("dit_gemm_gated_residual", h.data_ptr(), w.data_ptr(), x.data_ptr(), x_out.data_ptr(),
          gate.data_ptr(), dt, gs, B, N, K, D, _ptr(status), _stream(x))
    return x_out


# ------------------------------------------------------------ SubBlock router


def subblock_keep_count(n_blocks: int, sparsity: float) -> int:
    n = library().dit_subblock_keep_count(int(n_blocks), float(sparsity))
    if n < 0:
        raise DitError("dit_subblock_keep_count", n, library().dit_status_string(n).decode())
    return n


def subblock_router(q: torch.Tensor, k: torch.Tensor, heads: int, block: int = 128,
                    sparsity: float = 0.75, workspace: Optional[torch.Tensor] = None,
                    kept: Optional[torch.Tensor] = None,
                    status: Optional[torch.Tensor] = None) -> torch.Tensor:
    """The kept key blocks of every query block: int32 [B, H, n_blocks,
    n_keep], increasing.  q and k are [B, N, H*hd] views (e.g. slices of a
    fused qkv buffer) sharing one row stride.  ``status`` (int32 CUDA
    scalar) is set to 1 if a wait of the tensor-core score kernel expired."""
    _need_cuda_bf16("q", q)
    _need_cuda_bf16("k", k)
    B, N, width = q.shape
    if k.shape != q.shape or width % heads:
        raise ValueError("q and k must be [B, N, H*hd] of the same shape")
    hd = width // heads
    rs = _token_rows("q", q, B, N, width)
    if _token_rows("k", k, B, N, width) != rs:
        raise ValueError("q and k must share the row stride")
    nb = (N + block - 1) // block
    if not 0.0 <= sparsity < 1.0:
        raise ValueError("sparsity must be in [0, 1)")
    if nb == 0 or B == 0:
        return torch.empty(B, heads, nb, 0, dtype=torch.int32, device=q.device)
    n_keep = subblock_keep_count(nb, sparsity)
    need = int(library().dit_subblock_workspace_bytes(B, N, heads, hd, block))
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    if workspace.numel() * workspace.element_size() < need:
        raise ValueError(f"workspace needs {need} bytes")
    if kept is None:
        kept = torch.empty(B, heads, nb, n_keep, dtype=torch.int32, device=q.device)
    if kept.dtype != torch.int32 or kept.numel() != B * heads * nb * n_keep or \
            not kept.is_contiguous():
        raise ValueError(f"kept must be a contiguous int32 [B, H, {nb}, {n_keep}] tensor")
    if status is not None and (status.dtype != torch.int32 or not status.is_cuda):
        raise ValueError("status must be a CUDA int32 tensor")
    _call("dit_subblock_router", q.data_ptr(), k.data_ptr(), rs, B, N, heads, hd, block,
          float(sparsity), kept.data_ptr(), workspace.data_ptr(),
          workspace.numel() * workspace.element_size(), _ptr(status), _stream(q))
    return kept


def subblock_router_means(block_means: torch.Tensor, N: int, heads: int, block: int = 128,
                          sparsity: float = 0.75, workspace: Optional[torch.Tensor] = None,
                          kept: Optional[torch.Tensor] = None,
                          status: Optional[torch.Tensor] = None) -> torch.Tensor:
    """The router from block means (``qk_rmsnorm_rope3d(..., block_means=)``):
    fp32 [B, 2, n_blocks, H*hd] -> kept int32 [B, H, n_blocks, n_keep].
    ``status`` (int32 CUDA scalar) is set to 1 if a wait of the tensor-core
    score kernel expired."""
    if block_means.dtype != torch.float32 or not block_means.is_cuda or \
            not block_means.is_contiguous() or block_means.dim() != 4 or \
            block_means.shape[1] != 2:
        raise ValueError("block_means must be a contiguous CUDA float32 [B, 2, n_blocks, H*hd]")
    B, _, nb, width = block_means.shape
    if nb != (N + block - 1) // block or width % heads:
        raise ValueError("block_means does not match N, block and heads")
    hd = width // heads
    if not 0.0 <= sparsity < 1.0:
        raise ValueError("sparsity must be in [0, 1)")
    if nb == 0 or B == 0:
        return torch.empty(B, heads, nb, 0, dtype=torch.int32, device=block_means.device)
    n_keep = subblock_keep_count(nb, sparsity)
    need = int(library().dit_subblock_means_workspace_bytes(B, N, heads, hd, block))
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=block_means.device)
    if workspace.numel() * workspace.element_size() < need or \
            workspace.device != block_means.device or not workspace.is_contiguous():
        raise ValueError(f"workspace needs {need} contiguous bytes")
    if kept is None:
        kept = torch.empty(B, heads, nb, n_keep, dtype=torch.int32, device=block_means.device)
    if kept.dtype != torch.int32 or kept.numel() != B * heads * nb * n_keep or \
            not kept.is_contiguous() or kept.device != block_means.device:
        raise ValueError(f"kept must be a contiguous int32 [B, H, {nb}, {n_keep}] tensor")
    if status is not None and (status.dtype != torch.int32 or not status.is_cuda):
        raise ValueError("status must be a CUDA int32 tensor")
    _call("dit_subblock_router_means", block_means.data_ptr(), B, N, heads, hd, block,
          float(sparsity), kept.data_ptr(), workspace.data_ptr(),
          workspace.numel() * workspace.element_size(), _ptr(status), _stream(block_means))
    return kept


def block_sparse_attention(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, heads: int,
                           kept: torch.Tensor, scale: Optional[float] = None,
                           out: Optional[torch.Tensor] = None,
                           status: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Attention of every query block over its kept key blocks (blocks of
    128 tokens, head size 128).  q, k, v: [B, N, H*128] views sharing one row
    stride (e.g. slices of a fused qkv buffer); kept: int32 [B, H, n_blocks,
    n_keep] from subblock_router.  Returns [B, N, H*128] bf16."""
    for nm, t in (("q", q), ("k", k), ("v", v)):
        _need_cuda_bf16(nm, t)
    B, N, width = q.shape
    if k.shape != q.shape or v.shape != q.shape or width % heads:
        raise ValueError("q, k and v must be [B, N, H*hd] of the same shape")
    hd = width // heads
    rs = _token_rows("q", q, B, N, width)
    if _token_rows("k", k, B, N, width) != rs or _token_rows("v", v, B, N, width) != rs:
        raise ValueError("q, k and v must share the row stride")
    if kept.dtype != torch.int32 or kept.dim() != 4 or not kept.is_contiguous() or \
            kept.shape[:3] != (B, heads, (N + 127) // 128):
        raise ValueError("kept must be a contiguous int32 [B, H, n_blocks, n_keep] tensor")
    if out is None:
        out = torch.empty(B, N, width, dtype=torch.bfloat16, device=q.device)
    _need_cuda_bf16("out", out)
    os_ = _token_rows("out", out, B, N, width)
    if scale is None:
        scale = hd ** -0.5
    if status is not None and (status.dtype != torch.int32 or not status.is_cuda):
        raise ValueError("status must be a CUDA int32 tensor")
    if B * N == 0:
        return out
    _call("dit_block_sparse_attention", q.data_ptr(), k.data_ptr(), v.data_ptr(), rs,
          out.data_ptr(), os_, B, N, heads, hd, 128, kept.data_ptr(), kept.shape[3],
          float(scale), _ptr(status), _stream(q))
    return out
