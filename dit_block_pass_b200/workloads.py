"""Synthetic H3-shaped workloads and their seeded input generators.

This module builds INPUTS only: shapes, value distributions and the seeded
counter-based generator that fills them.  It holds none of the operators'
arithmetic, and both the CUDA path and the fp64 oracle draw their inputs from
it.

Generator.  Element ``i`` of tensor ``s`` (row-major index, int64) under seed
``seed`` is a pure function of ``(seed, s, i)``:

    key  = fmix32((seed * 0x9E3779B1 + s) mod 2^32)
    bits = fmix32(fmix32((i mod 2^32) xor key) xor (i >> 32))
    z    = Q[bits >> 16]              Q[j] = Phi^-1((j + 0.5) / 65536), float32
    v    = bf16(float32(z * sigma) + mean)     (or float32 for fp32 tensors)

``fmix32`` is the 32-bit finaliser of MurmurHash3 (Appleby).  Every step is
integer arithmetic, an exact table gather, one correctly rounded float32
multiply and add, and one round-to-nearest-even conversion, so the same
element comes out bit-identical on the CPU and on the GPU, and any subset of
rows can be generated on its own (the full-size parity tests check sampled
rows without generating the whole tensor on the host).  The quantile table
bounds |z| by about 4.3.

The workloads follow the H3-Base shapes: 1344x768 video at 24 fps through a
16x spatial / 4x temporal VAE gives a 31x48x84 latent grid for 5 s (124,992
tokens) and 61x48x84 for 10 s; model width 5120 in 40 heads of 128; SwiGLU
width 13,824.  ("MiniMax H3 mở trọng số: H3-Base có gì và còn thiếu gì?",
section "Kiến trúc: tạo hình và tiếng trong cùng một luồng"; "MiniMax-H3 no
SGLang em H200", test setup paragraph.)
"""
from __future__ import annotations

import dataclasses
from typing import Optional, Sequence

import torch

_M32 = 0xFFFFFFFF

# tensor stream ids
S_X, S_R, S_MOD, S_QKV, S_WQ, S_WK, S_SWIGLU, S_PREV, S_NOISE = range(1, 10)


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    T: int
    Hg: int
    Wg: int
    D: int
    H: int
    hd: int
    F: int
    pairs: tuple
    n_audio: int = 0
    theta: float = 10000.0
    eps: float = 1e-6
    thresholds: tuple = (0.04,)
    sigma_cache: tuple = (0.03,)     # per-sample noise of cur vs prev (cycled over B)
    seed: int = 0

    @property
    def n_video(self) -> int:
        return self.T * self.Hg * self.Wg

    @property
    def N(self) -> int:
        return self.n_video + self.n_audio

    @property
    def M(self) -> int:
        return self.B * self.N

    @property
    def explicit_positions(self) -> bool:
        return self.n_audio > 0

    def describe(self) -> str:
        s = (f"{self.name}: B={self.B}, grid T={self.T},H={self.Hg},W={self.Wg} "
             f"({self.n_video:,} video tokens")
        if self.n_audio:
            s += f" + {self.n_audio:,} audio tokens"
        s += (f"), D={self.D}, {self.H} heads x {self.hd}, SwiGLU [M,{2 * self.F}]->[M,{self.F}], "
              f"RoPE pairs t/h/w {'/'.join(map(str, self.pairs))}, bf16")
        return s


CONFIGS = {
    "tiny": Workload("tiny", B=1, T=2, Hg=4, Wg=6, D=256, H=4, hd=64, F=1024,
                     pairs=(12, 10, 10)),
    "small": Workload("small", B=1, T=8, Hg=24, Wg=42, D=3072, H=24, hd=128, F=8192,
                      pairs=(22, 21, 21)),
    "h3_5s": Workload("h3_5s", B=1, T=31, Hg=48, Wg=84, D=5120, H=40, hd=128, F=13824,
                      pairs=(22, 21, 21), thresholds=(0.04, 0.08)),
    "h3_10s": Workload("h3_10s", B=1, T=61, Hg=48, Wg=84, D=5120, H=40, hd=128, F=13824,
                       pairs=(22, 21, 21), thresholds=(0.04, 0.08)),
    "cfg_av": Workload("cfg_av", B=2, T=31, Hg=48, Wg=84, D=5120, H=40, hd=128, F=13824,
                       pairs=(22, 21, 21), n_audio=1200, thresholds=(0.04, 0.08),
                       sigma_cache=(0.03, 0.1)),
    # an 8-frame slice of the 5 s clip (32,256 tokens): same widths, so the
    # same kernels and launch shapes, at a size a profiler capture can hold;
    # every tensor is still larger than L2
    "h3_slice": Workload("h3_slice", B=1, T=8, Hg=48, Wg=84, D=5120, H=40, hd=128, F=13824,
                         pairs=(22, 21, 21), thresholds=(0.04, 0.08)),
}


# ------------------------------------------------------------ generator


def _mul32(x: torch.Tensor, c: int) -> torch.Tensor:
    """(x * c) mod 2^32 for int64 x in [0, 2^32), without int64 overflow."""
    lo, hi = c & 0xFFFF, c >> 16
    return (x * lo + (((x * hi) & 0xFFFF) << 16)) & _M32


def _fmix32(x: torch.Tensor) -> torch.Tensor:
    x = x ^ (x >> 16)
    x = _mul32(x, 0x85EBCA6B)
    x = x ^ (x >> 13)
    x = _mul32(x, 0xC2B2AE35)
    return x ^ (x >> 16)


def _fmix32_int(x: int) -> int:
    x &= _M32
    x ^= x >> 16
    x = (x * 0x85EBCA6B) & _M32
    x ^= x >> 13
    x = (x * 0xC2B2AE35) & _M32
    return x ^ (x >> 16)


def stream_key(seed: int, stream: int) -> int:
    return _fmix32_int(seed * 0x9E3779B1 + stream)


_QTABLE = {}


def _quantile_table(device) -> torch.Tensor:
    dev = torch.device(device)
    key = str(dev)
    if key not in _QTABLE:
        if "cpu" not in _QTABLE:
            p = (torch.arange(65536, dtype=torch.float64) + 0.5) / 65536.0
            _QTABLE["cpu"] = torch.special.ndtri(p).to(torch.float32)
        _QTABLE[key] = _QTABLE["cpu"].to(dev)
    return _QTABLE[key]


def hash_bits(seed: int, stream: int, idx: torch.Tensor) -> torch.Tensor:
    """32-bit hash of int64 element indices (values in [0, 2^32))."""
    key = stream_key(seed, stream)
    h = _fmix32((idx & _M32) ^ key)
    return _fmix32(h ^ (idx >> 32))


def _normal_f32(seed: int, stream: int, idx: torch.Tensor, sigma: float, mean: float) -> torch.Tensor:
    z = _quantile_table(idx.device)[hash_bits(seed, stream, idx) >> 16]
    v = z * torch.tensor(sigma, dtype=torch.float32, device=idx.device)
    if mean != 0.0:
        v = v + torch.tensor(mean, dtype=torch.float32, device=idx.device)
    return v


def normal(seed: int, stream: int, rows: int, cols: int, sigma: float = 1.0, mean: float = 0.0,
           dtype=torch.bfloat16, device="cpu", row_ids: Optional[torch.Tensor] = None,
           chunk: Optional[int] = None) -> torch.Tensor:
    """A [rows, cols] tensor (or [len(row_ids), cols] with row_ids) of
    ~N(mean, sigma^2) values of the given dtype; element (r, c) has index
    r*cols + c in the stream.  `chunk` elements are hashed at a time (only
    speed and memory depend on it)."""
    device = torch.device(device)
    if chunk is None:
        chunk = (1 << 24) if device.type == "cuda" else (1 << 20)
    if row_ids is not None:
        row_ids = row_ids.to(device=device, dtype=torch.int64)
        out_rows = row_ids.numel()
    else:
        out_rows = rows
    out = torch.empty(out_rows, cols, dtype=dtype, device=device)
    if out_rows == 0 or cols == 0:
        return out
    rows_per_chunk = max(1, chunk // cols)
    col = torch.arange(cols, dtype=torch.int64, device=device)
    for r0 in range(0, out_rows, rows_per_chunk):
        r1 = min(out_rows, r0 + rows_per_chunk)
        if row_ids is None:
            rr = torch.arange(r0, r1, dtype=torch.int64, device=device)
        else:
            rr = row_ids[r0:r1]
        idx = rr[:, None] * cols + col[None, :]
        out[r0:r1] = _normal_f32(seed, stream, idx, sigma, mean).to(dtype)
    return out


# ------------------------------------------------------------- inputs


def positions(wl: Workload, device="cpu") -> Optional[torch.Tensor]:
    """[B*N, 3] int32 (t, h, w) for workloads with appended audio tokens: the
    video tokens take their latent-grid coordinates (row-major), audio token j
    takes (j, 0, 0) (one temporal axis).  None when positions follow the grid."""
    if not wl.explicit_positions:
        return None
    t, h, w = torch.meshgrid(torch.arange(wl.T), torch.arange(wl.Hg), torch.arange(wl.Wg),
                             indexing="ij")
    video = torch.stack([t.reshape(-1), h.reshape(-1), w.reshape(-1)], dim=1)
    audio = torch.zeros(wl.n_audio, 3, dtype=torch.int64)
    audio[:, 0] = torch.arange(wl.n_audio)
    one = torch.cat([video, audio], dim=0).to(torch.int32)
    return one.repeat(wl.B, 1).to(device)


def modulation(wl: Workload, device="cpu", dtype=torch.float32) -> torch.Tensor:
    """[B, 6, D]: shift1, scale1, gate1, shift2, scale2, gate2 ~ N(0, 0.1)."""
    m = normal(wl.seed, S_MOD, wl.B * 6, wl.D, sigma=0.1, dtype=torch.float32, device=device)
    return m.reshape(wl.B, 6, wl.D).to(dtype)


def norm_weights(wl: Workload, device="cpu"):
    """RMSNorm weights w_q, w_k: [hd] fp32 ~ 1 + N(0, 0.02)."""
    wq = normal(wl.seed, S_WQ, 1, wl.hd, sigma=0.02, mean=1.0, dtype=torch.float32, device=device)
    wk = normal(wl.seed, S_WK, 1, wl.hd, sigma=0.02, mean=1.0, dtype=torch.float32, device=device)
    return wq.reshape(wl.hd), wk.reshape(wl.hd)


def row_norm_weights(wl: Workload, device="cpu"):
    """Whole-row RMSNorm weights w_q, w_k: [H*hd] fp32 ~ 1 + N(0, 0.02)."""
    D = wl.H * wl.hd
    wq = normal(wl.seed, S_WQ, 1, D, sigma=0.02, mean=1.0, dtype=torch.float32, device=device)
    wk = normal(wl.seed, S_WK, 1, D, sigma=0.02, mean=1.0, dtype=torch.float32, device=device)
    return wq.reshape(D), wk.reshape(D)


def token_rows(wl: Workload, stream: int, width: int, device="cpu", row_ids=None) -> torch.Tensor:
    """[B*N, width] bf16 ~N(0,1) token-major rows (all rows, or row_ids)."""
    return normal(wl.seed, stream, wl.M, width, device=device, row_ids=row_ids)


def cache_pair(wl: Workload, device="cpu", row_ids=None):
    """prev ~N(0,1) and cur = bf16(prev + N(0, sigma_b)) per sample, [rows, D]."""
    prev = token_rows(wl, S_PREV, wl.D, device=device, row_ids=row_ids)
    rows = (torch.arange(wl.M, device=device) if row_ids is None
            else row_ids.to(device=device, dtype=torch.int64))
    sig = torch.tensor([wl.sigma_cache[b % len(wl.sigma_cache)] for b in range(wl.B)],
                       dtype=torch.float32, device=device)
    noise = normal(wl.seed, S_NOISE, wl.M, wl.D, sigma=1.0, dtype=torch.float32, device=device,
                   row_ids=row_ids)
    noise = noise * sig[rows // wl.N][:, None]
    cur = (prev.to(torch.float32) + noise).to(torch.bfloat16)
    return prev, cur


def sample_rows(wl: Workload, count: int, seed: int = 1) -> torch.Tensor:
    """A sorted sample of token rows that always includes the first and last
    token of every sample (boundaries and the ragged tail)."""
    g = torch.Generator().manual_seed(seed)
    picks = set()
    for b in range(wl.B):
        picks.update({b * wl.N, b * wl.N + wl.N - 1})
    extra = torch.randint(0, wl.M, (max(0, count - len(picks)),), generator=g).tolist()
    picks.update(extra)
    return torch.tensor(sorted(picks), dtype=torch.int64)


def bits_u16(t: torch.Tensor):
    """bf16 tensor -> numpy uint16 bit patterns (host copy)."""
    import numpy as np
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def config_names() -> Sequence[str]:
    return list(CONFIGS)
