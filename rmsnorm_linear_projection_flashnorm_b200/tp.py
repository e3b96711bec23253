"""Row-parallel (d-split) tensor parallelism for the fused norm + projection.

When the input width d is sharded across ranks (each rank holds its own
contiguous columns of x, as the output of a column-parallel layer leaves
them, and the matching rows of the folded weight), the deferred
normalisation (FlashNorm talk summary, Proposal 2) needs exactly one
exchange: each rank computes the unscaled products and the sums of squares
of its columns into one fp32 buffer (``fn_norm_proj_partial``), one
all-reduce sums the buffers, and every rank finishes with the post-scale
(``fn_post_scale``: 1/rms from the full width, SwiGLU, bf16).

Host-side plumbing only: the arithmetic runs in the library's kernels, the
exchange is one ``torch.distributed.all_reduce`` (NCCL on GPUs).
"""
from __future__ import annotations

from typing import List, Optional, Tuple

import torch
import torch.distributed as dist


def rowparallel_slices(d: int, world: int, align: int = 64) -> List[Tuple[int, int]]:
    """Contiguous [start, stop) column ranges of d for `world` ranks: every
    boundary a multiple of `align` (64 for bf16 weights, 128 for fp8, the
    kernels' k-block sizes), sizes as even as that allows.  Raises
    ValueError when some rank would get no columns."""
    if d <= 0 or world <= 0 or align <= 0 or d % align:
        raise ValueError(f"d={d} must be a positive multiple of align={align}")
    blocks = d // align
    if blocks < world:
        raise ValueError(f"d={d} has {blocks} blocks of {align}: fewer than {world} ranks")
    out = []
    for r in range(world):
        b0 = r * blocks // world
        b1 = (r + 1) * blocks // world
        out.append((b0 * align, b1 * align))
    return out


def row_parallel_norm_proj(x_local: torch.Tensor, Wp_local: torch.Tensor, N: int, eps: float, d_total: int,
                           swiglu: bool = False, scales: Optional[torch.Tensor] = None, group=None,
                           ws=None) -> torch.Tensor:
    """y [M, N] (bf16) of RMSNorm(x) @ W with d split across the ranks of
    `group`: this rank passes its columns x_local [M, d_local] and its rows of
    the folded weight (and of the fp8 block scales).  Every rank returns the
    full y."""
    from . import torch_api as T
    M = x_local.shape[0]
    ncols = 2 * N if swiglu else N
    part = T.norm_proj_partial(x_local, Wp_local, ncols, scales=scales, ws=ws)
    world = dist.get_world_size(group) if dist.is_available() and dist.is_initialized() else 1
    if world > 1:
        dist.all_reduce(part, op=dist.ReduceOp.SUM, group=group)
    return T.post_scale(part, M, N, d_total, eps, swiglu=swiglu)
