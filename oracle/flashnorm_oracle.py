"""Plain fp64 NumPy statement of what the fused norm+projection computes.

TEST INFRASTRUCTURE ONLY (see the package docstring): never called by the
library, shares no code with the CUDA path.

Sources.  The method is described on the FlashNorm talk summary ("RMS norm는
연산량 1할인데 왜 33번 호출로 속도를 갉아먹나", news.juniverse.app): Proposal 1
("웨이트리스 정규화", weightless normalisation) folds the norm gain into the
following projection offline; Proposal 2 ("지연된 정규화", deferred
normalisation) postpones the per-row 1/rms scalar until after the matmul;
Proposal 3 ("이중 정규화 제거") removes a back-to-back norm by scale invariance.
The SwiGLU epilogue (silu(gate) * up) is the activation of the fused FC1 on the
FlashInfer PR #5521 analysis ("Segmented Chain" baseline and "Register-level
SwiGLU" design item).  The pages print no formula; the readings used here are:

    ms[m]  = (1/d) * sum_k x[m,k]^2              mean over the full row (divisor d)
    r[m]   = 1 / sqrt(ms[m] + eps)               eps inside the square root
    h[m,k] = x[m,k] * r[m] * g[k]                normalised row times the gain
    y      = h @ W                               no bias
    silu(z) = z / (1 + exp(-z))
    swiglu  = silu(h @ W_gate) * (h @ W_up)

The oracle computes these the *unfolded* way: normalise first, then multiply.
All stored low-precision inputs are taken exactly as float64.

The fold (Proposal 1) and the fp8 block quantisation are encodings, so the
oracle spells out their rounding steps from the formats' definitions:

    W'      = RN_bf16( fp32(g[k]) * fp32(W[k,n]) )        one fp32 product, one RN
    fp8:    P = fp32(g[k]) * fp32(W[k,n]);  per 128x128 block b:
            s_b = fp32( amax_b(|P|) / 448 )  (s_b = 1 when amax_b = 0)
            q   = RN_e4m3_satfinite( fp32(P / s_b) )
    SwiGLU storage: 128-column tiles of the gate and up halves alternate,
            W'_cat[:, 256j : 256j+128]       = W'_gate[:, 128j : 128j+128]
            W'_cat[:, 256j+128 : 256j+256]   = W'_up  [:, 128j : 128j+128]

The quantising SwiGLU epilogue writes its output in NVFP4 for the next
projection (FlashInfer PR #4040 analysis: silu_and_mul fused with the NVFP4
quantisation, a block of SF_VEC_SIZE = 16 elements per scale factor and a
caller-supplied global scale).  That page names the parts but prints no
formula; the reading used here, per row m and block b of 16 consecutive
output columns, with gs the fp32 global scale:

    amax_b = max |y[m, 16b : 16b+16]|
    sf_b   = RN_e4m3_satfinite( gs * amax_b / 6 )     6: the largest e2m1 value
    q      = RN_e2m1_satfinite( y * gs / sf_b )        q = 0 where sf_b = 0
    a block holding a non-finite value: sf_b = the e4m3 NaN code, q = 0
    dequantised: e2m1(q) * e4m3(sf_b) / gs
    storage: two codes per byte, the even column in the low nibble;
             scale codes row-major [M, N/16]
"""
from __future__ import annotations

import math
from typing import Optional, Tuple

import numpy as np

__all__ = [
    "BF16", "E4M3", "round_to_format", "bf16_round", "bf16_bits", "bf16_from_bits",
    "e4m3_round", "e4m3_encode", "e4m3_decode", "to_f64",
    "rms_inv", "rmsnorm", "norm_proj", "silu", "norm_proj_swiglu",
    "fold_bf16", "interleave128", "deinterleave128", "fold_fp8", "dequant_fp8", "dequant_fp8_bf16_bits",
    "FP8_BLOCK", "E4M3_MAX",
    "E2M1", "E2M1_MAX", "NVFP4_BLOCK", "e2m1_round", "e2m1_encode", "e2m1_decode",
    "nvfp4_quantize", "nvfp4_pack", "nvfp4_unpack", "nvfp4_dequantize",
    "rowparallel_partial", "rowparallel_finish",
    "MX_BLOCK", "fold_mxfp8", "dequant_mxfp8",
    "sf_chunk_layout", "sf_chunk_unlayout", "mx_scale_store", "fold_mxfp8_stored",
    "adaln_modulate", "norm_proj_adaln", "norm_proj_adaln_swiglu", "adaln_shift_bias", "adaln_scaled_operand",
]

FP8_BLOCK = 128
E4M3_MAX = 448.0


# ---------------------------------------------------------------------------
# Number formats, from their definitions
# ---------------------------------------------------------------------------
class _Format:
    """A binary floating-point format: stored mantissa bits, exponent bias,
    largest finite value and what happens above it ("inf" or "sat")."""

    def __init__(self, name, man_bits, exp_bits, bias, max_finite, overflow):
        self.name = name
        self.man_bits = man_bits
        self.exp_bits = exp_bits
        self.bias = bias
        self.emin = 1 - bias                   # exponent of the smallest normal
        self.max_finite = max_finite
        self.overflow = overflow


# bfloat16: 1 sign, 8 exponent (bias 127), 7 mantissa bits; IEEE-style inf.
BF16 = _Format("bf16", 7, 8, 127, (2.0 - 2.0 ** -7) * 2.0 ** 127, "inf")
# e4m3 ("fn" variant): 1 sign, 4 exponent (bias 7), 3 mantissa bits, no inf;
# S.1111.111 is NaN, so the largest finite value is 1.75 * 2^8 = 448.
# Conversions here saturate to +-448 (the "satfinite" rounding).
E4M3 = _Format("e4m3", 3, 4, 7, 448.0, "sat")
# e2m1: 1 sign, 2 exponent (bias 1), 1 mantissa bit; no inf and no NaN.  The
# exponent field 0 holds the subnormal 0.5; the largest value is 1.5 * 2^2 = 6.
E2M1 = _Format("e2m1", 1, 2, 1, 6.0, "sat")
E2M1_MAX = 6.0
NVFP4_BLOCK = 16


def round_to_format(v, fmt: _Format) -> np.ndarray:
    """Round values to the nearest member of `fmt`, ties to even.

    Works in float64, where every step below is exact: the quantum of the
    binade holding |v| is a power of two, so |v| / quantum is exact and
    np.rint rounds half to even.  Below the smallest normal the quantum is
    fixed (subnormals).  Returns float64 values of the format.
    """
    v = np.asarray(v, dtype=np.float64)
    a = np.abs(v)
    _, ex = np.frexp(np.where(a > 0, a, 1.0))    # a = m * 2^ex, m in [0.5, 1)
    e = np.maximum(ex.astype(np.int64) - 1, fmt.emin)   # floor(log2 a), clamped
    quantum = np.ldexp(1.0, e - fmt.man_bits)
    r = np.rint(a / quantum) * quantum
    if fmt.overflow == "inf":
        r = np.where(r > fmt.max_finite, np.inf, r)
    else:
        r = np.where(r > fmt.max_finite, fmt.max_finite, r)
    r = np.where(np.isinf(a), np.inf if fmt.overflow == "inf" else fmt.max_finite, r)
    out = np.copysign(r, v)
    return np.where(np.isnan(v), np.nan, out)


def bf16_round(v) -> np.ndarray:
    return round_to_format(v, BF16)


def bf16_bits(v) -> np.ndarray:
    """uint16 bit patterns of RN_bf16(v).  A bf16 value is an fp32 value whose
    low 16 bits are zero, so the pattern is the top half of its fp32 bits."""
    r = bf16_round(v).astype(np.float32)
    bits = (r.view(np.uint32) >> 16).astype(np.uint16)
    return np.where(np.isnan(r), np.uint16(0x7FC0), bits).astype(np.uint16)


def bf16_from_bits(bits) -> np.ndarray:
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return b.view(np.float32).astype(np.float64)


def e4m3_round(v) -> np.ndarray:
    return round_to_format(v, E4M3)


def e4m3_encode(v) -> np.ndarray:
    """uint8 codes of RN_e4m3_satfinite(v): sign | exponent field | mantissa."""
    r = e4m3_round(v)
    sign = (np.signbit(r)).astype(np.uint8) << 7
    a = np.abs(r)
    nan = np.isnan(a)
    a = np.where(nan, 0.0, a)
    min_normal = 2.0 ** E4M3.emin
    _, ex = np.frexp(np.where(a > 0, a, 1.0))
    e = ex.astype(np.int64) - 1
    normal = a >= min_normal
    exp_field = np.where(normal, e + E4M3.bias, 0)
    mant = np.where(normal,
                    np.ldexp(a, -e) - 1.0,                   # in [0, 1)
                    a / min_normal)                          # subnormal: 0.mmm
    mant_field = np.rint(mant * 8.0).astype(np.int64)
    code = (exp_field.astype(np.int64) << 3) | mant_field
    code = np.where(a == 0, 0, code).astype(np.uint8) | sign
    return np.where(nan, np.uint8(0x7F), code).astype(np.uint8)


def e4m3_decode(code) -> np.ndarray:
    """float64 value of each uint8 e4m3 code (S.1111.111 decodes to NaN)."""
    c = np.asarray(code, dtype=np.uint8).astype(np.int64)
    s = np.where(c & 0x80, -1.0, 1.0)
    ef = (c >> 3) & 0xF
    mf = c & 0x7
    val = np.where(ef == 0,
                   np.ldexp(mf / 8.0, E4M3.emin),
                   np.ldexp(1.0 + mf / 8.0, ef - E4M3.bias))
    val = np.where((ef == 0xF) & (mf == 0x7), np.nan, val)
    return s * val


def to_f64(a) -> np.ndarray:
    """Stored values (NumPy array or a CPU torch tensor of any float dtype) as
    float64, exactly."""
    if hasattr(a, "detach"):
        a = a.detach().cpu()
        if str(a.dtype) in ("torch.bfloat16", "torch.float16"):
            a = a.float()
        a = a.double().numpy()
    return np.asarray(a, dtype=np.float64)


# ---------------------------------------------------------------------------
# The operation (FlashNorm talk: RMSNorm feeding its projection; unfolded form)
# ---------------------------------------------------------------------------
def rms_inv(x, eps: float) -> np.ndarray:
    """r[m] = 1 / sqrt(mean_k x[m,k]^2 + eps); the per-row scalar that
    Proposal 2 (deferred normalisation) postpones to after the matmul."""
    x = to_f64(x)
    ms = np.mean(x * x, axis=1)
    with np.errstate(divide="ignore", invalid="ignore"):
        return 1.0 / np.sqrt(ms + eps)


def rmsnorm(x, g, eps: float) -> np.ndarray:
    """h = (x * r) * g, the normalised activation an unfused chain writes."""
    x = to_f64(x)
    g = to_f64(g)
    with np.errstate(invalid="ignore"):
        return (x * rms_inv(x, eps)[:, None]) * g[None, :]


def _matmul_chunked(h: np.ndarray, W, col_chunk: Optional[int]) -> np.ndarray:
    W_is_np = isinstance(W, np.ndarray)
    ncols = W.shape[1]
    if col_chunk is None or col_chunk >= ncols:
        return h @ to_f64(W)
    out = np.empty((h.shape[0], ncols), dtype=np.float64)
    for c0 in range(0, ncols, col_chunk):
        c1 = min(ncols, c0 + col_chunk)
        out[:, c0:c1] = h @ to_f64(W[:, c0:c1] if W_is_np else W[:, c0:c1])
    return out


def norm_proj(x, g, W, eps: float, col_chunk: Optional[int] = None) -> np.ndarray:
    """y = RMSNorm(x; g, eps) @ W in float64, normalising first (unfolded)."""
    h = rmsnorm(x, g, eps)
    with np.errstate(invalid="ignore"):
        return _matmul_chunked(h, W, col_chunk)


def silu(z) -> np.ndarray:
    """silu(z) = z / (1 + exp(-z)); exp overflow for z << 0 gives -0."""
    z = np.asarray(z, dtype=np.float64)
    with np.errstate(over="ignore"):
        return z / (1.0 + np.exp(-z))


def norm_proj_swiglu(x, g, W_gate, W_up, eps: float,
                     col_chunk: Optional[int] = None) -> np.ndarray:
    """silu(h @ W_gate) * (h @ W_up) with h = RMSNorm(x; g, eps)."""
    h = rmsnorm(x, g, eps)
    with np.errstate(invalid="ignore"):
        return silu(_matmul_chunked(h, W_gate, col_chunk)) * _matmul_chunked(h, W_up, col_chunk)


# ---------------------------------------------------------------------------
# The offline fold (Proposal 1) and the weight encodings
# ---------------------------------------------------------------------------
def _gain_product_f32(W, g) -> np.ndarray:
    """fp32(g[k]) * fp32(W[k,n]) as an fp32 array (IEEE round-to-nearest)."""
    Wf = to_f64(W).astype(np.float32)
    gf = to_f64(g).astype(np.float32)
    return gf[:, None] * Wf


def fold_bf16(W, g) -> np.ndarray:
    """bf16 bit patterns [d, N] of W' = RN_bf16(fp32(g) * fp32(W))."""
    return bf16_bits(_gain_product_f32(W, g).astype(np.float64))


def interleave128(A: np.ndarray, B: np.ndarray) -> np.ndarray:
    """[d, 2N] with 128-column tiles alternating A, B, A, B, ..."""
    d, N = A.shape
    assert B.shape == (d, N) and N % 128 == 0
    out = np.empty((d, 2 * N), dtype=A.dtype)
    for j in range(N // 128):
        out[:, 256 * j: 256 * j + 128] = A[:, 128 * j: 128 * j + 128]
        out[:, 256 * j + 128: 256 * j + 256] = B[:, 128 * j: 128 * j + 128]
    return out


def deinterleave128(C: np.ndarray) -> Tuple[np.ndarray, np.ndarray]:
    d, N2 = C.shape
    N = N2 // 2
    A = np.empty((d, N), dtype=C.dtype)
    B = np.empty((d, N), dtype=C.dtype)
    for j in range(N // 128):
        A[:, 128 * j: 128 * j + 128] = C[:, 256 * j: 256 * j + 128]
        B[:, 128 * j: 128 * j + 128] = C[:, 256 * j + 128: 256 * j + 256]
    return A, B


def fold_fp8(W, g) -> Tuple[np.ndarray, np.ndarray]:
    """e4m3 codes [d, N] and fp32 block scales [d/128, N/128] of the folded
    weight: s_b = fp32(amax_b / 448) (1 for an all-zero block) and
    q = RN_e4m3_satfinite(fp32(P / s_b)), P = fp32(g) * fp32(W)."""
    P = _gain_product_f32(W, g)
    d, N = P.shape
    assert d % FP8_BLOCK == 0 and N % FP8_BLOCK == 0
    bd, bn = d // FP8_BLOCK, N // FP8_BLOCK
    blocks = np.abs(P).reshape(bd, FP8_BLOCK, bn, FP8_BLOCK)
    amax = blocks.max(axis=(1, 3)).astype(np.float32)
    s = np.where(amax > 0, amax / np.float32(E4M3_MAX), np.float32(1.0)).astype(np.float32)
    s_full = np.repeat(np.repeat(s, FP8_BLOCK, axis=0), FP8_BLOCK, axis=1)
    quot = (P / s_full).astype(np.float32)          # fp32 IEEE division
    return e4m3_encode(quot.astype(np.float64)), s


def dequant_fp8(q: np.ndarray, s: np.ndarray) -> np.ndarray:
    """float64 W_deq[k,n] = e4m3(q[k,n]) * s[k/128, n/128] (exact in fp64)."""
    s_full = np.repeat(np.repeat(to_f64(s), FP8_BLOCK, axis=0), FP8_BLOCK, axis=1)
    return e4m3_decode(q) * s_full


def dequant_fp8_bf16_bits(q: np.ndarray, s: np.ndarray) -> np.ndarray:
    """bf16 bit patterns of the on-chip dequantisation step: the e4m3 value
    (exact in fp32) times the fp32 block scale, rounded to fp32, then rounded
    once more to bf16 (the bf16 operand the tensor cores multiply)."""
    s_full = np.repeat(np.repeat(np.asarray(s, dtype=np.float32), FP8_BLOCK, axis=0), FP8_BLOCK, axis=1)
    prod = e4m3_decode(q).astype(np.float32) * s_full        # fp32 IEEE product
    return bf16_bits(prod.astype(np.float64))


# ---------------------------------------------------------------------------
# NVFP4 output encoding (quantising SwiGLU epilogue)
# ---------------------------------------------------------------------------
def e2m1_round(v) -> np.ndarray:
    return round_to_format(v, E2M1)


def e2m1_encode(v) -> np.ndarray:
    """4-bit codes (uint8 0..15) of RN_e2m1_satfinite(v): sign | exponent
    field (2 bits) | mantissa bit.  NaN has no code here; callers keep it out."""
    r = e2m1_round(v)
    sign = np.signbit(r).astype(np.uint8) << 3
    a = np.abs(np.where(np.isnan(r), 0.0, r))
    _, ex = np.frexp(np.where(a > 0, a, 1.0))
    e = ex.astype(np.int64) - 1                     # floor(log2 a)
    normal = a >= 1.0                               # smallest normal: 2^(1 - bias)
    exp_field = np.where(normal, e + E2M1.bias, 0)
    # normal: a = (1 + m/2) * 2^e; subnormal (field 0): a = m * 0.5
    mant_field = np.where(normal, np.rint((np.ldexp(a, -e) - 1.0) * 2.0), np.rint(a * 2.0)).astype(np.int64)
    code = (exp_field << 1) | mant_field
    return (np.where(a == 0, 0, code).astype(np.uint8) | sign).astype(np.uint8)


def e2m1_decode(code) -> np.ndarray:
    """float64 value of each 4-bit e2m1 code."""
    c = np.asarray(code, dtype=np.uint8).astype(np.int64)
    s = np.where(c & 0x8, -1.0, 1.0)
    ef = (c >> 1) & 0x3
    mf = c & 0x1
    val = np.where(ef == 0, mf * 0.5, np.ldexp(1.0 + mf / 2.0, ef - E2M1.bias))
    return s * val


def nvfp4_quantize(y, global_scale: float) -> Tuple[np.ndarray, np.ndarray]:
    """NVFP4 encoding of y [M, N] (N a multiple of 16) with the fp32 global
    scale gs, following the reading in the module docstring.  Returns the
    4-bit codes [M, N] (one per uint8) and the e4m3 scale codes [M, N/16].
    The arithmetic is float64; gs is taken as its fp32 value."""
    y = np.asarray(y, dtype=np.float64)
    M, N = y.shape
    assert N % NVFP4_BLOCK == 0
    gs = float(np.float32(global_scale))
    blocks = y.reshape(M, N // NVFP4_BLOCK, NVFP4_BLOCK)
    finite = np.all(np.isfinite(blocks), axis=2)                     # [M, N/16]
    amax = np.max(np.abs(np.where(np.isfinite(blocks), blocks, 0.0)), axis=2)
    sf = e4m3_encode(gs * amax / E2M1_MAX)
    sf = np.where(finite, sf, np.uint8(0x7F)).astype(np.uint8)
    sf_val = np.where(finite, e4m3_decode(np.where(finite, sf, 0)), 0.0)
    enc = np.where(sf_val > 0, gs / np.where(sf_val > 0, sf_val, 1.0), 0.0)
    scaled = np.where(finite[:, :, None], np.where(np.isfinite(blocks), blocks, 0.0) * enc[:, :, None], 0.0)
    codes = e2m1_encode(scaled).reshape(M, N)
    return codes, sf


def nvfp4_pack(codes) -> np.ndarray:
    """[M, N] 4-bit codes -> [M, N/2] bytes, the even column in the low nibble."""
    c = np.asarray(codes, dtype=np.uint8)
    return (c[:, 0::2] & 0xF) | ((c[:, 1::2] & 0xF) << 4)


def nvfp4_unpack(packed) -> np.ndarray:
    """[M, N/2] bytes -> [M, N] 4-bit codes."""
    b = np.asarray(packed, dtype=np.uint8)
    out = np.empty((b.shape[0], b.shape[1] * 2), dtype=np.uint8)
    out[:, 0::2] = b & 0xF
    out[:, 1::2] = b >> 4
    return out


def nvfp4_dequantize(codes, sf, global_scale: float) -> np.ndarray:
    """float64 e2m1(q) * e4m3(sf) / gs for codes [M, N] and scale codes [M, N/16]."""
    gs = float(np.float32(global_scale))
    scale = np.repeat(e4m3_decode(sf), NVFP4_BLOCK, axis=1)
    return e2m1_decode(codes) * scale / gs


# ---------------------------------------------------------------------------
# Row-parallel (d-split) form of the deferred normalisation
# ---------------------------------------------------------------------------
def rowparallel_partial(x_local, W_local) -> Tuple[np.ndarray, np.ndarray]:
    """One rank's share when the input width d is split across ranks: the
    unscaled products over this rank's columns of x (rows of W) and the sums
    of squares of those columns.  Proposal 2 (deferred normalisation) applies
    1/rms after the matmul, and both quantities are sums over k, so the shares
    of all ranks add up to the single-device values."""
    x = to_f64(x_local)
    return x @ to_f64(W_local), np.sum(x * x, axis=1)


def rowparallel_finish(acc, ssq, d_total: int, eps: float, swiglu: bool = False) -> np.ndarray:
    """The post-scale after the shares were summed: r = 1/sqrt(ssq/d + eps)
    with d the full width, then r * acc, or silu(r * gate) * (r * up) with the
    gate and up columns in the interleaved stored order."""
    acc = np.asarray(acc, dtype=np.float64)
    r = 1.0 / np.sqrt(np.asarray(ssq, dtype=np.float64) / d_total + eps)
    if not swiglu:
        return acc * r[:, None]
    gate, up = deinterleave128(acc)
    return silu(gate * r[:, None]) * (up * r[:, None])


# ---------------------------------------------------------------------------
# MXFP8 weights: e4m3 codes with one power-of-two (ue8m0) scale per 32 k values
# ---------------------------------------------------------------------------
MX_BLOCK = 32


def fold_mxfp8(W, g) -> Tuple[np.ndarray, np.ndarray]:
    """Folded weight P = fp32(g[k]) * fp32(W[k,n]) in the block-scaled form the
    tensor cores' kind::mxf8f6f4 MMAs read: per column n and block b of 32
    consecutive k, a shared exponent E (stored as the ue8m0 byte E + 127) with
        E = ceil(log2(amax_b / 448))      the smallest power of two that keeps
                                          every |P| / 2^E <= 448 (no saturation)
        q = RN_e4m3(P / 2^E)              (exact division by a power of two)
    An all-zero block stores E = -127 (byte 0) and zero codes.  Reading: the
    OCP MX rule floor(log2 amax) - 8 lets a block maximum land in [448, 512)
    and clamps it; the round-up rule loses no accuracy against the 128x128
    fp32-scaled format (the format study in the tests), so it is used here.
    Returns codes [d, N] and scale bytes [d/32, N]."""
    P = _gain_product_f32(W, g).astype(np.float64)
    d, N = P.shape
    assert d % MX_BLOCK == 0
    Pb = P.reshape(d // MX_BLOCK, MX_BLOCK, N)
    amax = np.max(np.abs(Pb), axis=1)                                   # [d/32, N]
    _, ex = np.frexp(np.where(amax > 0, amax / E4M3_MAX, 1.0))          # amax/448 = m * 2^ex, m in [0.5, 1)
    m = np.ldexp(np.where(amax > 0, amax / E4M3_MAX, 1.0), -ex)
    E = np.where(m == 0.5, ex - 1, ex)                                  # ceil(log2(amax/448))
    E = np.where(amax > 0, np.clip(E, -127, 127), -127).astype(np.int64)
    q = e4m3_encode(Pb / np.ldexp(1.0, E)[:, None, :])
    return q.reshape(d, N), (E + 127).astype(np.uint8)


def dequant_mxfp8(q: np.ndarray, sbytes: np.ndarray) -> np.ndarray:
    """float64 e4m3(q[k,n]) * 2^(s[k/32, n] - 127) (exact in fp64)."""
    scale = np.ldexp(1.0, np.asarray(sbytes, dtype=np.int64) - 127)
    return e4m3_decode(q) * np.repeat(scale, MX_BLOCK, axis=0)


# ---------------------------------------------------------------------------
# Scale bytes in the chunked layout that block-scaled tensor-core MMAs read
# ---------------------------------------------------------------------------
def sf_chunk_layout(S) -> np.ndarray:
    """Scale bytes S [R, C] (R rows along the M or N side of a block-scaled
    MMA, C scale columns along its K side) in the chunked layout the tensor
    cores read: the matrix is cut into chunks of 128 rows x 4 scale columns
    (512 bytes each, rows padded to a multiple of 128 and columns to a
    multiple of 4 with zero bytes), chunk (rb, cg) stored at byte
    512 * (rb * ceil(C/4) + cg), and inside a chunk the byte of row r, column c
    sits at 16 * (r mod 32) + 4 * ((r mod 128) div 32) + (c mod 4): 32
    sixteen-byte lines, line i holding rows i, i+32, i+64, i+96 of the chunk.
    This is the layout the FlashInfer PR #4040 analysis calls swizzled scale
    factors (is_swizzled), which a block-scaled GEMM consumes directly.
    Returns a flat uint8 array."""
    S = np.asarray(S, dtype=np.uint8)
    R, C = S.shape
    Rp, Cp = -(-R // 128) * 128, -(-C // 4) * 4
    r, c = np.indices((R, C))
    dest = 512 * ((r // 128) * (Cp // 4) + c // 4) + 16 * (r % 32) + 4 * ((r % 128) // 32) + (c % 4)
    out = np.zeros(Rp * Cp, dtype=np.uint8)
    out[dest.ravel()] = S.ravel()
    return out


def sf_chunk_unlayout(flat, R: int, C: int) -> np.ndarray:
    """Inverse of sf_chunk_layout: the [R, C] scale bytes back from the flat
    chunked array."""
    flat = np.asarray(flat, dtype=np.uint8)
    Cp = -(-C // 4) * 4
    r, c = np.indices((R, C))
    src = 512 * ((r // 128) * (Cp // 4) + c // 4) + 16 * (r % 32) + 4 * ((r % 128) // 32) + (c % 4)
    return flat[src]


def mx_scale_store(sb) -> np.ndarray:
    """MXFP8 scale bytes [d/32, ncols] (32-deep k blocks x stored columns) in
    the order the library stores them: 128-deep k groups (4 blocks) one after
    another; each group's [ncols, 4] slab, in the weight's MMA orientation
    (rows = output columns), laid out by sf_chunk_layout (one 512-byte chunk
    per 128 columns).  A row slice of the weight on 128-row boundaries
    therefore owns one contiguous range of scale bytes."""
    sb = np.asarray(sb, dtype=np.uint8)
    assert sb.shape[0] % 4 == 0
    return np.concatenate([sf_chunk_layout(sb[4 * kg: 4 * kg + 4, :].T) for kg in range(sb.shape[0] // 4)])


def fold_mxfp8_stored(W, g) -> Tuple[np.ndarray, np.ndarray]:
    """The MXFP8 fold as the library stores it: the e4m3 codes [d, N] of
    fold_mxfp8 and its scale bytes in the order of mx_scale_store."""
    q, sb = fold_mxfp8(W, g)
    return q, mx_scale_store(sb)


# ---------------------------------------------------------------------------
# AdaLN modulation after the norm (FlashInfer PR #5521 analysis, fused API)
# ---------------------------------------------------------------------------
# The PR #5521 analysis fuses "RMSNorm + AdaLN" into its FC1 and passes the
# norm weight, an AdaLN scale, an AdaLN shift and an index for AdaLN; it
# prints no formula.  Reading used here (adaptive layer norm applied to the
# normalised row, one scale row and one shift row per condition, selected by
# each token's index):
#
#     h[m, k] = RMSNorm(x; g, eps)[m, k] * scale[c_m, k] + shift[c_m, k],
#     c_m = index[m],   y = h @ W   (SwiGLU: silu(h @ W_gate) * (h @ W_up))
#
# `scale` is the effective multiplier, as g is (a DiT-style 1 + scale is the
# caller's conversion).


def adaln_modulate(x, g, eps: float, scale, shift, index) -> np.ndarray:
    """h = RMSNorm(x; g, eps) * scale[index] + shift[index], row by row."""
    idx = np.asarray(index, dtype=np.int64)
    with np.errstate(invalid="ignore"):
        return rmsnorm(x, g, eps) * to_f64(scale)[idx] + to_f64(shift)[idx]


def norm_proj_adaln(x, g, W, eps: float, scale, shift, index) -> np.ndarray:
    """y = (RMSNorm(x; g, eps) * scale[index] + shift[index]) @ W, normalising
    and modulating first (unfolded)."""
    h = adaln_modulate(x, g, eps, scale, shift, index)
    with np.errstate(invalid="ignore"):
        return h @ to_f64(W)


def norm_proj_adaln_swiglu(x, g, W_gate, W_up, eps: float, scale, shift, index) -> np.ndarray:
    """silu(h @ W_gate) * (h @ W_up) with h the AdaLN-modulated norm."""
    h = adaln_modulate(x, g, eps, scale, shift, index)
    with np.errstate(invalid="ignore"):
        return silu(h @ to_f64(W_gate)) * (h @ to_f64(W_up))


def adaln_shift_bias(shift, W) -> np.ndarray:
    """The shift's contribution to the projection, one row per condition:
    B[c, n] = sum_k shift[c, k] W[k, n] with the unfolded weight (the shift is
    added after the gain, so the gain does not multiply it).  With it the
    modulated projection splits into the deferred form
        y[m, :] = r[m] * ((x[m, :] * scale[c_m, :]) @ W') + B[c_m, :],
    W' = diag(g) W, which the kernels compute (the scale multiplies the raw
    activations, the 1/rms scalar stays deferred, the shift becomes a bias)."""
    return to_f64(shift) @ to_f64(W)


def adaln_scaled_operand(x, scale, index) -> np.ndarray:
    """The scaled activations as the tensor cores receive them in the deferred
    form: the fp32 product fp32(x[m, k]) * fp32(scale[c_m, k]) (IEEE
    round-to-nearest), rounded once more to bf16 (the MMA's operand format).
    Returned as float64 values."""
    idx = np.asarray(index, dtype=np.int64)
    prod = to_f64(x).astype(np.float32) * to_f64(scale).astype(np.float32)[idx]
    return bf16_round(prod.astype(np.float64))
