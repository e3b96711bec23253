"""torch-facing conveniences over the C ABI: allocate outputs and workspaces
with torch (device memory is torch's job here) and call the library.  No
arithmetic of the method happens in Python."""
from __future__ import annotations

from typing import Optional, Tuple

import torch

from . import (FN_W_BF16, FN_W_FP8_E4M3_B128, FN_W_MXFP8_E4M3, check, fn_adaln_shift_bias, fn_norm_proj_adaln,
               fn_norm_proj_swiglu_nvfp4_swizzled, fn_workspace_size_adaln, fn_fold_weights, fn_norm_proj, fn_norm_proj_swiglu,
               fn_norm_proj_partial, fn_norm_proj_swiglu_nvfp4, fn_post_scale, fn_query_device_status,
               fn_workspace_size)


def weight_type(Wp: torch.Tensor, scales: Optional[torch.Tensor]) -> int:
    """The fn_wtype of a folded weight: bf16, e4m3 with fp32 block scales, or
    MXFP8 (e4m3 with ue8m0 scale bytes)."""
    if Wp.dtype == torch.bfloat16:
        return FN_W_BF16
    return FN_W_MXFP8_E4M3 if scales is not None and scales.dtype == torch.uint8 else FN_W_FP8_E4M3_B128


def fold(W0: torch.Tensor, g: torch.Tensor, W1: Optional[torch.Tensor] = None, wtype: int = FN_W_BF16,
         stream=None) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """Fold g into W0 (and W1 for SwiGLU); returns (W', scales or None)."""
    d, N = W0.shape
    ncols = 2 * N if W1 is not None else N
    dev = W0.device
    if wtype == FN_W_BF16:
        Wp = torch.empty((d, ncols), dtype=torch.bfloat16, device=dev)
        scales = None
    elif wtype == FN_W_MXFP8_E4M3:
        Wp = torch.empty((d, ncols), dtype=torch.uint8, device=dev)
        scales = torch.empty(d * ncols // 32, dtype=torch.uint8, device=dev)   # chunked ue8m0 bytes
    else:
        Wp = torch.empty((d, ncols), dtype=torch.uint8, device=dev)
        scales = torch.empty((d // 128, ncols // 128), dtype=torch.float32, device=dev)
    check(fn_fold_weights(W0, W1, g, d, N, wtype, Wp, scales, stream), "fn_fold_weights")
    return Wp, scales


class Workspace:
    """A zero-initialised device workspace that grows on demand."""

    def __init__(self, device="cuda"):
        self.device = device
        self.buf = torch.zeros(256, dtype=torch.uint8, device=device)

    def get(self, M: int, d: int, N: int, wt: int, swiglu: bool) -> torch.Tensor:
        need = fn_workspace_size(M, d, N, wt, int(swiglu))
        if self.buf.numel() < need:
            self.buf = torch.zeros(need, dtype=torch.uint8, device=self.device)
        return self.buf

    def status(self, stream=None):
        return fn_query_device_status(self.buf, stream)


def norm_proj(x: torch.Tensor, Wp: torch.Tensor, N: int, eps: float, swiglu: bool = False,
              scales: Optional[torch.Tensor] = None, ws: Optional[Workspace] = None,
              out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """y = RMSNorm(x) @ W through the fused kernels (W' already folded)."""
    M, d = x.shape
    wt = weight_type(Wp, scales)
    if ws is None:
        ws = Workspace(x.device)
    buf = ws.get(M, d, N, wt, swiglu)
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=x.device)
    fn = fn_norm_proj_swiglu if swiglu else fn_norm_proj
    check(fn(x, M, d, Wp, scales, wt, N, eps, out, buf, buf.numel(), stream), fn.__name__)
    return out


def norm_proj_swiglu_nvfp4(x: torch.Tensor, Wp: torch.Tensor, N: int, eps: float, global_scale: torch.Tensor,
                           scales: Optional[torch.Tensor] = None, ws: Optional[Workspace] = None,
                           out: Optional[Tuple[torch.Tensor, torch.Tensor]] = None,
                           stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """SwiGLU output in NVFP4: (codes uint8 [M, N/2], e4m3 scale bytes uint8
    [M, N/16]); global_scale is a one-element fp32 device tensor."""
    M, d = x.shape
    wt = weight_type(Wp, scales)
    if ws is None:
        ws = Workspace(x.device)
    buf = ws.get(M, d, N, wt, True)
    if out is None:
        out = (torch.empty((M, N // 2), dtype=torch.uint8, device=x.device),
               torch.empty((M, N // 16), dtype=torch.uint8, device=x.device))
    q, sf = out
    check(fn_norm_proj_swiglu_nvfp4(x, M, d, Wp, scales, wt, N, eps, global_scale, q, sf, buf, buf.numel(), stream),
          "fn_norm_proj_swiglu_nvfp4")
    return q, sf


def norm_proj_swiglu_nvfp4_swizzled(x: torch.Tensor, Wp: torch.Tensor, N: int, eps: float,
                                    global_scale: torch.Tensor, scales: Optional[torch.Tensor] = None,
                                    ws: Optional[Workspace] = None, stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """SwiGLU output in NVFP4 with the scale bytes in the chunked (swizzled)
    layout: (codes uint8 [M, N/2], scale bytes uint8 [ceil(M/128)*128 * N/16],
    zero-initialised so the padding rows read as 0)."""
    M, d = x.shape
    wt = weight_type(Wp, scales)
    if ws is None:
        ws = Workspace(x.device)
    buf = ws.get(M, d, N, wt, True)
    q = torch.empty((M, N // 2), dtype=torch.uint8, device=x.device)
    sf = torch.zeros(((M + 127) // 128) * 128 * (N // 16), dtype=torch.uint8, device=x.device)
    check(fn_norm_proj_swiglu_nvfp4_swizzled(x, M, d, Wp, scales, wt, N, eps, global_scale, q, sf, buf, buf.numel(),
                                             stream), "fn_norm_proj_swiglu_nvfp4_swizzled")
    return q, sf


def norm_proj_partial(x: torch.Tensor, Wp: torch.Tensor, ncols: int, scales: Optional[torch.Tensor] = None,
                      ws: Optional[Workspace] = None, out: Optional[torch.Tensor] = None,
                      stream=None) -> torch.Tensor:
    """One rank's share of a row-parallel projection: fp32 [M * ncols + M]
    (unscaled x @ Wp in stored column order, then the rows' sums of squares)."""
    M, d = x.shape
    wt = weight_type(Wp, scales)
    if ws is None:
        ws = Workspace(x.device)
    buf = ws.get(M, d, ncols, wt, False)
    if out is None:
        out = torch.empty(M * ncols + M, dtype=torch.float32, device=x.device)
    check(fn_norm_proj_partial(x, M, d, Wp, scales, wt, ncols, out, buf, buf.numel(), stream), "fn_norm_proj_partial")
    return out


def post_scale(partial: torch.Tensor, M: int, N: int, d_total: int, eps: float, swiglu: bool = False,
               out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """bf16 [M, N] from a summed partial buffer (see fn_post_scale)."""
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=partial.device)
    check(fn_post_scale(partial, M, N, int(swiglu), d_total, eps, out, stream), "fn_post_scale")
    return out


def adaln_shift_bias(shift: torch.Tensor, W0: torch.Tensor, W1: Optional[torch.Tensor] = None,
                     stream=None) -> torch.Tensor:
    """fp32 [n_cond, ncols]: the AdaLN shift rows through the unfolded weight."""
    n_cond, d = shift.shape
    N = W0.shape[1]
    ncols = 2 * N if W1 is not None else N
    B = torch.empty((n_cond, ncols), dtype=torch.float32, device=shift.device)
    check(fn_adaln_shift_bias(shift, n_cond, W0, W1, d, N, B, stream), "fn_adaln_shift_bias")
    return B


def norm_proj_adaln(x: torch.Tensor, Wp: torch.Tensor, N: int, eps: float, adaln_scale: torch.Tensor,
                    shift_bias: torch.Tensor, adaln_index: torch.Tensor, swiglu: bool = False,
                    scales: Optional[torch.Tensor] = None, ws: Optional[Workspace] = None,
                    out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """The AdaLN-modulated fused call (see fn_norm_proj_adaln)."""
    M, d = x.shape
    wt = weight_type(Wp, scales)
    if ws is None:
        ws = Workspace(x.device)
    need = fn_workspace_size_adaln(d, N, wt, int(swiglu))
    if ws.buf.numel() < need:
        ws.buf = torch.zeros(need, dtype=torch.uint8, device=ws.device)
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=x.device)
    check(fn_norm_proj_adaln(x, M, d, Wp, scales, wt, N, int(swiglu), eps, adaln_scale, shift_bias, adaln_index,
                             adaln_scale.shape[0], out, ws.buf, ws.buf.numel(), stream), "fn_norm_proj_adaln")
    return out
