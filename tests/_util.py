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


def check_nvfp4(q_packed, sf, ref, gs: float, tol: float, min_exact: float = 0.97) -> float:
    """Check the kernel's NVFP4 output (codes [M, N/2] bytes, scale bytes
    [M, N/16]) against the oracle's fp64 SwiGLU values `ref` [M, N].

    The kernel's fp32 value v lies within t = tol * (1 + |ref|) of ref, and a
    quantised code is a decision on v, so the check accepts every code some v
    in that band could give:
      * the scale byte must lie between the oracle's scale codes for the
        smallest and largest block maximum the band allows;
      * given the kernel's scale, each element's e2m1 value must lie between
        the oracle's roundings of the band's two ends;
      * blocks where ref holds a non-finite value must carry the NaN scale
        code 0x7F and zero codes.
    Returns the fraction of codes (scale and element) equal to the oracle's
    own encoding of ref, which must be at least `min_exact`."""
    q = O.nvfp4_unpack(np.asarray(q_packed, dtype=np.uint8))
    sf = np.asarray(sf, dtype=np.uint8)
    ref = np.asarray(ref, dtype=np.float64)
    M, N = ref.shape
    assert q.shape == (M, N) and sf.shape == (M, N // 16)
    gs = float(np.float32(gs))
    blocks = ref.reshape(M, N // 16, 16)
    bad_blk = ~np.all(np.isfinite(blocks), axis=2)
    assert np.all(sf[bad_blk] == 0x7F), "non-finite blocks must carry the NaN scale"
    assert np.all(q.reshape(M, N // 16, 16)[bad_blk] == 0), "non-finite blocks must carry zero codes"
    fin = np.where(np.isfinite(blocks), blocks, 0.0)
    t = tol * (1.0 + np.abs(fin))
    amax_lo = np.max(np.maximum(np.abs(fin) - t, 0.0), axis=2)
    amax_hi = np.max(np.abs(fin) + t, axis=2)
    s_lo = O.e4m3_decode(O.e4m3_encode(gs * amax_lo / O.E2M1_MAX))
    s_hi = O.e4m3_decode(O.e4m3_encode(gs * amax_hi / O.E2M1_MAX))
    s_got = np.where(bad_blk, 0.0, O.e4m3_decode(np.where(bad_blk, 0, sf)))
    ok_s = bad_blk | ((s_got >= s_lo) & (s_got <= s_hi))
    assert ok_s.all(), f"{int((~ok_s).sum())} scale codes outside the band"
    enc = np.where(s_got > 0, gs / np.where(s_got > 0, s_got, 1.0), 0.0)[:, :, None]
    v_lo = O.e2m1_round((fin - t) * enc)
    v_hi = O.e2m1_round((fin + t) * enc)
    v_got = O.e2m1_decode(q).reshape(M, N // 16, 16)
    ok_v = bad_blk[:, :, None] | ((v_got >= v_lo) & (v_got <= v_hi))
    assert ok_v.all(), f"{int((~ok_v).sum())} element codes outside the band"
    q_ref, sf_ref = O.nvfp4_quantize(ref, gs)
    same = np.count_nonzero(sf == sf_ref) + np.count_nonzero(O.e2m1_decode(q) == O.e2m1_decode(q_ref))
    frac = same / (sf.size + q.size)
    assert frac >= min_exact, f"only {frac:.4f} of the codes equal the oracle's encoding"
    return frac
