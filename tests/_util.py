"""Shared helpers for the GPU tests: run the library through its C ABI on torch
device buffers, and build oracle references from the oracle's own fold (never
from anything the CUDA path produced)."""
from __future__ import annotations

import numpy as np
import torch

import oracle as O
import rmsnorm_linear_projection_flashnorm_b200 as fnb
from rmsnorm_linear_projection_flashnorm_b200 import torch_api as T

BF16_TOL = 1e-2   # max|y - y_ref| <= 1e-2 (1 + |y_ref|), bf16 weights
FP8_TOL = 6e-2    # ... <= 6e-2 (1 + |y_ref|), fp8 e4m3 block-scaled weights


def rel_err(y, ref) -> float:
    """max |y - ref| / (1 + |ref|) over positions where ref is finite; NaN
    positions must coincide."""
    y = O.to_f64(y)
    ref = np.asarray(ref, dtype=np.float64)
    nan_y, nan_r = np.isnan(y), np.isnan(ref)
    assert np.array_equal(nan_y, nan_r), "NaN positions differ"
    ok = ~nan_r
    if not ok.any():
        return 0.0
    return float(np.max(np.abs(y[ok] - ref[ok]) / (1.0 + np.abs(ref[ok]))))


def fold_ref_bf16(W, g, col_chunk: int = 4096) -> np.ndarray:
    """The oracle's bf16 fold as float64 values, computed in column chunks."""
    d, N = W.shape
    out = np.empty((d, N), dtype=np.float64)
    for c0 in range(0, N, col_chunk):
        c1 = min(N, c0 + col_chunk)
        out[:, c0:c1] = O.bf16_from_bits(O.fold_bf16(W[:, c0:c1], g))
    return out


def gpu(t):
    return t.cuda(non_blocking=False)


def run(x, Wp, N, eps, swiglu=False, scales=None, ws=None):
    y = T.norm_proj(x, Wp, N, eps, swiglu=swiglu, scales=scales, ws=ws)
    torch.cuda.synchronize()
    return y


def sample_cols(N: int, seed: int, per_tile: int = 8, tile: int = 128) -> np.ndarray:
    rng = np.random.default_rng(20_000 + seed)
    cols = []
    for t0 in range(0, N, tile):
        cols.extend(rng.choice(np.arange(t0, min(N, t0 + tile)), size=min(per_tile, tile), replace=False))
    return np.unique(np.asarray(cols, dtype=np.int64))


def fold_fp8_ref(W0, g, W1=None, col_chunk: int = 1024):
    """The oracle's fp8 fold (codes, fp32 block scales), computed in column
    chunks of whole 128-column blocks; with W1 the gate/up tiles are
    interleaved per 128 columns like the stored layout."""
    def one(W):
        d, N = W.shape
        q = np.empty((d, N), dtype=np.uint8)
        s = np.empty((d // 128, N // 128), dtype=np.float32)
        for c0 in range(0, N, col_chunk):
            c1 = min(N, c0 + col_chunk)
            q[:, c0:c1], s[:, c0 // 128:c1 // 128] = O.fold_fp8(W[:, c0:c1], g)
        return q, s
    if W1 is None:
        return one(W0)
    qg, sg = one(W0)
    qu, su = one(W1)
    s = np.empty((sg.shape[0], 2 * sg.shape[1]), dtype=np.float32)
    s[:, 0::2], s[:, 1::2] = sg, su
    return O.interleave128(qg, qu), s
