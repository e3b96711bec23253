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
exchange is one ``torch.distributed.all_reduce`` (NCCL on GPUs), or a
reduce-scatter by rows followed by an all-gather of the bf16 outputs, which
moves fewer bytes.
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
                           ws=None, exchange: str = "allreduce") -> torch.Tensor:
    """y [M, N] (bf16) of RMSNorm(x) @ W with d split across the ranks of
    `group`: this rank passes its columns x_local [M, d_local] and its rows of
    the folded weight (and of the block scales).  Every rank returns the full y.

    exchange="allreduce": one all-reduce of the fp32 buffer [M, ncols] + [M],
    then every rank post-scales all rows.
    exchange="reduce_scatter": the fp32 products and sums of squares are
    reduce-scattered by rows (rank r gets rows [r M/W, (r+1) M/W)), each rank
    post-scales its own rows, and the bf16 outputs [M/W, N] are all-gathered.
    The sums are the same fp32 sums, so the result agrees with the all-reduce
    path; a ring exchange moves (W-1)/W (4 M ncols + 2 M N) bytes per rank
    instead of 2 (W-1)/W 4 M ncols: 0.625x for SwiGLU (ncols = 2N), 0.75x for
    a plain projection.  Needs M divisible by the world size; otherwise the
    all-reduce path is taken."""
    from . import torch_api as T
    if exchange not in ("allreduce", "reduce_scatter"):
        raise ValueError(f"exchange must be 'allreduce' or 'reduce_scatter', not {exchange!r}")
    M = x_local.shape[0]
    ncols = 2 * N if swiglu else N
    part = T.norm_proj_partial(x_local, Wp_local, ncols, scales=scales, ws=ws)
    world = dist.get_world_size(group) if dist.is_available() and dist.is_initialized() else 1
    if world == 1:
        return T.post_scale(part, M, N, d_total, eps, swiglu=swiglu)
    if exchange == "allreduce" or M % world:
        dist.all_reduce(part, op=dist.ReduceOp.SUM, group=group)
        return T.post_scale(part, M, N, d_total, eps, swiglu=swiglu)
    rank = dist.get_rank(group)
    Ml = M // world
    # this rank's rows: products [Ml, ncols], then their sums of squares, in the
    # layout fn_post_scale reads
    local = torch.empty(Ml * ncols + Ml, dtype=part.dtype, device=part.device)
    dist.reduce_scatter_tensor(local[:Ml * ncols].view(Ml, ncols), part[:M * ncols].view(M, ncols),
                               op=dist.ReduceOp.SUM, group=group)
    dist.reduce_scatter_tensor(local[Ml * ncols:], part[M * ncols:], op=dist.ReduceOp.SUM, group=group)
    y_local = T.post_scale(local, Ml, N, d_total, eps, swiglu=swiglu)
    y = torch.empty((M, N), dtype=y_local.dtype, device=y_local.device)
    dist.all_gather_into_tensor(y, y_local.contiguous(), group=group)
    return y
