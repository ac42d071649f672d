"""Sequence sharding of the block op chain across ranks (one process per GPU).

Every operator of the chain is token-local except the Cache-DiT check, so a
clip's N tokens split into contiguous shards, one per rank, and each rank
runs the same kernels on its shard with no exchange:

  * AdaLN, gated residual + AdaLN and SwiGLU: nothing changes.
  * QK RMSNorm + 3D RoPE: the shard passes its first token's global index as
    ``pos_offset`` so every token keeps its place on the (T, H, W) grid (or
    the rank passes its slice of an explicit position table).
  * Cache-DiT: the relative L1 difference needs sums over the whole clip.
    Each rank computes its shard's (sum |cur - prev|, sum |prev|) per sample
    (2*B doubles), the ranks all-gather them, and every rank adds the
    gathered [R, B, 2] array in the same fixed order, so all ranks reach
    bit-identical rel values and the same reuse decision.  This is the only
    collective, 16*B bytes per rank, and it is latency bound.

The compute steps are injectable (``sums_fn``, ``decide_fn``) so that the
exchange logic can be exercised on CPU ranks with the gloo backend; by
default they are the CUDA library's entry points.
"""
from __future__ import annotations

from typing import Callable, Optional, Sequence, Tuple

import torch


def shard_range(n: int, rank: int, world: int) -> Tuple[int, int]:
    """Contiguous, balanced [start, stop) of n tokens for `rank` of `world`
    (the first n % world ranks take one extra token)."""
    if world < 1 or not 0 <= rank < world or n < 0:
        raise ValueError("bad shard arguments")
    base, extra = divmod(n, world)
    start = rank * base + min(rank, extra)
    return start, start + base + (1 if rank < extra else 0)


def qk_rmsnorm_rope3d_shard(q, k, w_q, w_k, heads: int, pairs: Sequence[int],
                            grid: Sequence[int], token_start: int, theta: float = 10000.0,
                            eps: float = 1e-6, op: Optional[Callable] = None) -> None:
    """QK RMSNorm + 3D RoPE on a shard whose first token is global token
    `token_start` of the (T, Hg, Wg) grid."""
    if op is None:
        from . import qk_rmsnorm_rope3d as op
    op(q, k, w_q, w_k, heads, pairs, grid=grid, pos_offset=token_start, theta=theta, eps=eps)


def cachedit_residual_diff_sharded(prev: torch.Tensor, cur: torch.Tensor, threshold: float,
                                   group=None, sums_fn: Optional[Callable] = None,
                                   decide_fn: Optional[Callable] = None):
    """Cache-DiT decision over a clip whose tokens are sharded across the
    ranks of `group`.  prev/cur are this rank's [B, N_shard, D] shards.
    Returns (rel [B], reuse [B]) identical on every rank."""
    import torch.distributed as dist
    if sums_fn is None:
        from . import cachedit_residual_sums as sums_fn
    if decide_fn is None:
        from . import cachedit_decide as decide_fn
    sums = sums_fn(prev, cur)                                  # [B, 2] float64
    world = dist.get_world_size(group)
    gathered = [torch.empty_like(sums) for _ in range(world)]
    dist.all_gather(gathered, sums.contiguous(), group=group)
    return decide_fn(torch.stack(gathered).contiguous(), threshold)   # [R, B, 2], rank order
