"""GPU parity of the row-parallel (d-split) path: fn_norm_proj_partial on
each rank's slice of the input width, the shares summed, fn_post_scale.

One GPU stands in for the ranks: each slice's share is computed by the
library in turn and the shares are added on the device (what the all-reduce
does), then post-scaled; the result is compared with the fp64 oracle of the
whole (unsliced) projection.  With one slice the partial + post-scale route
must give the fused call's bits wherever both reduce every sum the same way:
on the tile path (each row's sum of squares is reduced in k order for every
column tile) and on decode shapes whose stream-K split cuts every column
tile at the same k points.  One test runs the real exchange through
torch.distributed (NCCL, world size 1).
"""
import datetime
import socket

import numpy as np
import pytest
import torch

import oracle as O
import rmsnorm_linear_projection_flashnorm_b200 as fnb
import workloads as WL
from rmsnorm_linear_projection_flashnorm_b200 import torch_api as T
from rmsnorm_linear_projection_flashnorm_b200 import tp
from tests._util import BF16_TOL, FP8_TOL, fold_fp8_ref, fold_ref_bf16, gpu, rel_err

pytestmark = pytest.mark.gpu
FP8 = fnb.FN_W_FP8_E4M3_B128


@pytest.fixture(scope="module", autouse=True)
def _lib():
    fnb.build()
    fnb.lib()
    torch.cuda.init()
    yield


def _fold(inp, swiglu, wt):
    g = inp["g"]
    W1 = gpu(inp["W_up"]) if swiglu else None
    W0 = gpu(inp["W_gate"] if swiglu else inp["W"])
    return T.fold(W0, gpu(g), W1, wtype=wt)


def _ref(inp, swiglu, wt, d):
    g = inp["g"]
    if wt == FP8:
        if swiglu:
            q, s = fold_fp8_ref(inp["W_gate"], g, inp["W_up"])
            Wg, Wu = O.deinterleave128(O.dequant_fp8(q, s))
            return O.norm_proj_swiglu(inp["x"], np.ones(d), Wg, Wu, inp["eps"])
        q, s = fold_fp8_ref(inp["W"], g)
        return O.norm_proj(inp["x"], np.ones(d), O.dequant_fp8(q, s), inp["eps"])
    if swiglu:
        return O.norm_proj_swiglu(inp["x"], np.ones(d), fold_ref_bf16(inp["W_gate"], g),
                                  fold_ref_bf16(inp["W_up"], g), inp["eps"])
    return O.norm_proj(inp["x"], np.ones(d), fold_ref_bf16(inp["W"], g), inp["eps"])


def _split_run(x, Wp, scales, N, eps, swiglu, wt, ranks):
    """Shares of `ranks` slices of d, summed on the device, post-scaled."""
    M, d = x.shape
    ncols = 2 * N if swiglu else N
    align = 128 if wt == FP8 else 64
    total = torch.zeros(M * ncols + M, dtype=torch.float32, device="cuda")
    for k0, k1 in tp.rowparallel_slices(d, ranks, align):
        sc = scales[k0 // 128:k1 // 128].contiguous() if scales is not None else None
        part = T.norm_proj_partial(x[:, k0:k1].contiguous(), Wp[k0:k1].contiguous(), ncols, scales=sc)
        total += part
    y = T.post_scale(total, M, N, d, eps, swiglu=swiglu)
    torch.cuda.synchronize()
    return y


@pytest.mark.parametrize("M,d,N,swiglu,wt,ranks", [
    (1, 1024, 384, False, 0, 2),      # decode, split tiles finished by the fix-up kernel
    (40, 768, 512, False, 0, 3),
    (8, 512, 256, True, 0, 2),
    (64, 256, 19200, False, 0, 2),    # 150 tiles: whole tiles in the decode kernel
    (200, 512, 384, False, 0, 2),     # tile kernel, ragged M, a half-filled last 256-column tile
    (130, 1024, 384, True, 0, 4),
    (3, 512, 256, True, FP8, 2),      # fp8 decode, in-kernel activation split
    (48, 768, 384, False, FP8, 3),    # fp8 decode, activations split once per call
    (100, 512, 256, True, FP8, 2),    # fp8 tile kernel
    (1100, 256, 256, False, FP8, 2),  # fp8, weight dequantised once per call
])
def test_row_parallel_matches_oracle(M, d, N, swiglu, wt, ranks):
    inp = WL.case(M, d, N, swiglu, seed=501)
    Wp, scales = _fold(inp, swiglu, wt)
    y = _split_run(gpu(inp["x"]), Wp, scales, N, inp["eps"], swiglu, wt, ranks)
    assert rel_err(y.cpu(), _ref(inp, swiglu, wt, d)) <= (FP8_TOL if wt == FP8 else BF16_TOL)


@pytest.mark.parametrize("M,d,N,swiglu,wt", [
    (8, 1024, 512, False, 0),         # decode: 64 iterations on 64 CTAs, every tile cut the same way
    (300, 512, 384, False, 0),        # tile kernel
    (130, 512, 384, True, 0),         # tile kernel: SwiGLU tiles are the same 256 stored columns
    (1, 1024, 512, False, FP8),       # fp8 decode: 32 iterations on 32 CTAs
])
def test_one_slice_is_bit_identical_to_the_fused_call(M, d, N, swiglu, wt):
    inp = WL.case(M, d, N, swiglu, seed=502)
    Wp, scales = _fold(inp, swiglu, wt)
    x = gpu(inp["x"])
    fused = T.norm_proj(x, Wp, N, inp["eps"], swiglu=swiglu, scales=scales)
    y = _split_run(x, Wp, scales, N, inp["eps"], swiglu, wt, 1)
    assert torch.equal(y, fused)


@pytest.mark.parametrize("M", [6, 90])
def test_row_parallel_nan_rows(M):
    """A zero row with eps = 0 has no finite 1/rms: NaN, as in the fused call."""
    inp = WL.case(M, 512, 256, False, seed=503)
    inp["x"][2] = 0
    inp["eps"] = 0.0
    Wp, _ = _fold(inp, False, 0)
    y = _split_run(gpu(inp["x"]), Wp, None, 256, 0.0, False, 0, 2).cpu().float().numpy()
    assert np.all(np.isnan(y[2])) and np.all(np.isfinite(np.delete(y, 2, axis=0)))


def test_row_parallel_through_torch_distributed():
    """The exchange itself through torch.distributed: one NCCL rank, whose
    all-reduce leaves the buffer as it is; the result matches the oracle."""
    import torch.distributed as dist
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1,
                            timeout=datetime.timedelta(seconds=60))
    try:
        inp = WL.case(16, 1024, 512, True, seed=504)
        Wp, _ = _fold(inp, True, 0)
        x = gpu(inp["x"])
        y = tp.row_parallel_norm_proj(x, Wp, 512, inp["eps"], 1024, swiglu=True)
        torch.cuda.synchronize()
        assert rel_err(y.cpu(), _ref(inp, True, 0, 1024)) <= BF16_TOL
    finally:
        dist.destroy_process_group()
