"""Fold-time model transforms around the fused norm + projection.

Double-norm removal (FlashNorm talk summary, Proposal 3 "이중 정규화 제거"):
where two RMSNorms follow each other, as in Gemma-4-style blocks, the second
one undoes any scalar factor the first leaves on its output, so

    RMSNorm(RMSNorm(x; c*1); g) = RMSNorm(x; sign(c) * g)     (exactly when eps = 0)

and the pair becomes one norm, which then folds into the projection that
follows (Proposal 1).  With eps > 0 the first norm's output has a mean square
of c^2 * ms / (ms + eps) rather than c^2, which moves the result by a relative
O(eps / ms + eps / c^2).  A first norm whose gain is not one scalar changes the
direction of x, and the pair cannot be merged.
"""
from __future__ import annotations

from typing import Optional, Tuple

import torch


def double_norm_gain(g_first: torch.Tensor, g_second: torch.Tensor) -> torch.Tensor:
    """The gain of the single norm that replaces RMSNorm(.; g_first) followed
    by RMSNorm(.; g_second): sign(c) * g_second when g_first is the constant c.
    Raises ValueError when g_first is not one non-zero scalar repeated."""
    gf = g_first.detach().reshape(-1).to(torch.float64).cpu()
    if gf.numel() != g_second.numel():
        raise ValueError("the two norms act on different widths")
    c = float(gf[0])
    if not bool(torch.all(gf == c)):
        raise ValueError("the first norm's gain is not a single scalar: the pair cannot be merged")
    if c == 0.0 or c != c:
        raise ValueError("the first norm's gain is zero or NaN")
    return g_second if c > 0 else -g_second


def fold_double_norm(W0: torch.Tensor, g_first: torch.Tensor, g_second: torch.Tensor,
                     W1: Optional[torch.Tensor] = None, wtype: int = 0,
                     stream=None) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """Fold the merged norm of a back-to-back pair into the projection (or the
    gate/up pair) that follows; the fused calls then take the raw input of the
    first norm."""
    from . import torch_api as T
    g = double_norm_gain(g_first, g_second)
    return T.fold(W0, g.to(device=W0.device, dtype=torch.float32).contiguous(), W1, wtype=wtype, stream=stream)
