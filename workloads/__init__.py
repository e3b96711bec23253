"""Seeded synthetic inputs for the norm+projection workloads.

This module only draws random numbers and stores them in the dtypes the
workloads name.  It holds none of the method's arithmetic (no norm, no fold,
no matmul), so both the fp64 oracle and the CUDA path may take their inputs
from here without sharing any computation.

Recipe (one seed per workload; NumPy PCG64; draws in fp64, stored as bf16):

* x[m, k]   = N(0, 1) * s_m,  s_m = exp(U[ln 0.1, ln 10])  (per-row scale)
* outliers  = floor(d / 100) fixed columns of x multiplied by 20 (large
  prefill workload only)
* g[k]      = bf16(1 + 0.1 * N(0, 1)), handed to the library as fp32 holding
  bf16-representable values (a checkpoint stores its norm gain in bf16)
* W[k, n]   = bf16(N(0, 1/d)); SwiGLU workloads draw W_gate then W_up
* eps       = 1e-6

Each quantity has its own child stream of the seed, and x and its row scales
are drawn row-major, so the first M rows of a workload are the same for every
M it lists.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, Optional, Sequence, Tuple

import numpy as np
import torch

EPS = 1e-6


@dataclasses.dataclass(frozen=True)
class Workload:
    """One synthetic workload: shapes, epilogue and weight storage."""

    name: str
    Ms: Tuple[int, ...]
    d: int
    N: int            # output columns (per half for SwiGLU)
    swiglu: bool
    wtype: str        # "bf16", "fp8_e4m3_b128" or "mxfp8_e4m3"
    outliers: bool
    seed: int

    @property
    def ncols(self) -> int:
        """Columns of the stored (folded) weight: N, or 2N for gate|up."""
        return 2 * self.N if self.swiglu else self.N


WORKLOADS: Dict[str, Workload] = {
    w.name: w
    for w in (
        Workload("tiny", (4,), 256, 512, False, "bf16", False, 0),
        Workload("decode_qkv", (1, 8, 32, 64), 4096, 6144, False, "bf16", False, 1),
        Workload("ffn_swiglu", (16, 4096), 4096, 14336, True, "bf16", False, 2),
        Workload("prefill_swiglu_large", (16384,), 8192, 28672, True, "bf16", True, 3),
        Workload("fp8_swiglu", (1, 64, 256, 8192), 5120, 13824, True, "fp8_e4m3_b128", False, 4),
        # the fp8 workload's shapes and inputs with the weight folded to the
        # block-scaled MXFP8 format instead of 128x128 fp32 block scales
        Workload("mxfp8_swiglu", (1, 64, 256, 8192), 5120, 13824, True, "mxfp8_e4m3", False, 4),
    )
}
WORKLOAD_ORDER = ("tiny", "decode_qkv", "ffn_swiglu", "prefill_swiglu_large", "fp8_swiglu", "mxfp8_swiglu")

_CHUNK = 1 << 22  # elements per draw, bounds host memory for the large weights


def _streams(seed: int):
    """Independent child generators: g, W, row scales, x, outlier columns."""
    children = np.random.SeedSequence(seed).spawn(5)
    return [np.random.Generator(np.random.PCG64(c)) for c in children]


def _to_bf16(a64: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a64, dtype=np.float32)).to(torch.bfloat16)


def _normal_bf16(rng: np.random.Generator, rows: int, cols: int, std: float) -> torch.Tensor:
    out = torch.empty((rows, cols), dtype=torch.bfloat16)
    step = max(1, _CHUNK // max(cols, 1))
    for r0 in range(0, rows, step):
        r1 = min(rows, r0 + step)
        out[r0:r1] = _to_bf16(rng.standard_normal((r1 - r0, cols)) * std)
    return out


def gain(d: int, seed: int) -> torch.Tensor:
    """g = bf16(1 + 0.1 N(0,1)) as fp32 [d]."""
    rng = _streams(seed)[0]
    return _to_bf16(1.0 + 0.1 * rng.standard_normal(d)).to(torch.float32)


def weights(d: int, N: int, seed: int, halves: int = 1):
    """W ~ bf16(N(0, 1/d)) [d, N]; with halves=2 returns (W_gate, W_up)."""
    rng = _streams(seed)[1]
    std = 1.0 / math.sqrt(d)
    ws = tuple(_normal_bf16(rng, d, N, std) for _ in range(halves))
    return ws[0] if halves == 1 else ws


def row_scales(M: int, seed: int) -> np.ndarray:
    """Per-row scale s_m = exp(U[ln 0.1, ln 10]) as fp64 [M]."""
    rng = _streams(seed)[2]
    return np.exp(rng.uniform(math.log(0.1), math.log(10.0), size=M))


def outlier_columns(d: int, seed: int) -> np.ndarray:
    """floor(d/100) distinct column indices, sorted."""
    rng = _streams(seed)[4]
    k = d // 100
    return np.sort(rng.choice(d, size=k, replace=False))


def activations(M: int, d: int, seed: int, outliers: bool = False,
                zero_rows: Sequence[int] = ()) -> torch.Tensor:
    """x [M, d] bf16: N(0,1) times the row scale (times 20 on outlier columns)."""
    scales = row_scales(M, seed)
    rng = _streams(seed)[3]
    cols = outlier_columns(d, seed) if outliers else None
    out = torch.empty((M, d), dtype=torch.bfloat16)
    step = max(1, _CHUNK // max(d, 1))
    for r0 in range(0, M, step):
        r1 = min(M, r0 + step)
        a = rng.standard_normal((r1 - r0, d)) * scales[r0:r1, None]
        if cols is not None:
            a[:, cols] *= 20.0
        out[r0:r1] = _to_bf16(a)
    for r in zero_rows:
        out[r] = 0
    return out


def case(M: int, d: int, N: int, swiglu: bool, seed: int, outliers: bool = False,
         zero_rows: Sequence[int] = ()) -> dict:
    """A full input set: x, g, W (or W_gate, W_up), eps."""
    inp = {
        "x": activations(M, d, seed, outliers, zero_rows),
        "g": gain(d, seed),
        "eps": EPS,
    }
    if swiglu:
        inp["W_gate"], inp["W_up"] = weights(d, N, seed, halves=2)
    else:
        inp["W"] = weights(d, N, seed)
    return inp


def workload_case(name: str, M: Optional[int] = None) -> dict:
    """Inputs of a named workload at one of its M (default: the largest)."""
    w = WORKLOADS[name]
    M = max(w.Ms) if M is None else M
    return case(M, w.d, w.N, w.swiglu, w.seed, w.outliers)


def sample_rows(M: int, seed: int, per_tile: int = 2, tile: int = 128) -> np.ndarray:
    """Deterministic row sample: `per_tile` rows in every `tile`-row block,
    always including the rows with the smallest and largest row scale."""
    rng = np.random.Generator(np.random.PCG64(10_000 + seed))
    rows = []
    for t0 in range(0, M, tile):
        t1 = min(M, t0 + tile)
        k = min(per_tile, t1 - t0)
        rows.extend(rng.choice(np.arange(t0, t1), size=k, replace=False).tolist())
    s = row_scales(M, seed)
    rows.extend([int(np.argmin(s)), int(np.argmax(s))])
    return np.unique(np.asarray(rows, dtype=np.int64))


def device_inputs(w: Workload, M: int, device, seed_offset: int = 0):
    """The same distributions as the host recipe above, drawn on the device with
    torch's generator (seeded), for benchmark workloads whose host generation
    would take longer than the measurement: returns x [M, d] bf16, g [d] fp32
    (bf16-representable), and W [d, N] bf16 (or the pair W_gate, W_up).  The
    values differ from the host recipe's; only shapes and distributions match."""
    gen = torch.Generator(device=device)
    gen.manual_seed(1_000_003 * (w.seed + 1) + seed_offset)
    d, N = w.d, w.N
    g = (1.0 + 0.1 * torch.randn(d, generator=gen, device=device)).to(torch.bfloat16).to(torch.float32)
    std = 1.0 / math.sqrt(d)
    Ws = tuple((torch.randn((d, N), generator=gen, device=device) * std).to(torch.bfloat16)
               for _ in range(2 if w.swiglu else 1))
    u = torch.rand((M, 1), generator=gen, device=device, dtype=torch.float64)
    scale = torch.exp(math.log(0.1) + u * (math.log(10.0) - math.log(0.1))).to(torch.float32)
    colmul = torch.ones((1, d), dtype=torch.float32, device=device)
    if w.outliers:
        colmul[0, torch.randperm(d, generator=gen, device=device)[: d // 100]] = 20.0
    x = torch.empty((M, d), dtype=torch.bfloat16, device=device)
    step = max(1, (1 << 26) // d)
    for r0 in range(0, M, step):
        r1 = min(M, r0 + step)
        x[r0:r1] = (torch.randn((r1 - r0, d), generator=gen, device=device) * scale[r0:r1] * colmul).to(torch.bfloat16)
    return x, g, (Ws[0] if len(Ws) == 1 else Ws)
