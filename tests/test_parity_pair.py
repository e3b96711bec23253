"""GPU parity of the tile kernel on pairs of SMs (2-CTA clusters, 256 x 256 or
256 x 512 tiles, tcgen05.mma.cta_group::2), which the library runs for bf16
weights at M >= 512.

Against the fp64 oracle on the stored folded weight within 1e-2 (1 + |y_ref|),
against the single-SM tile kernel (FN_DEBUG_FORCE_PATH = 3) within the same
bound, bit-identical over repeated calls, and the bounded waits of both CTAs
of a pair: a withheld arrival times out in both and the next call is correct.
Shapes cover ragged rows (the second CTA of the last pair partly or wholly
past M), an odd number of 128-column blocks (the second CTA's weight half past
the last column), a long k range, and more tiles than pairs (a partial second
wave).
"""
import numpy as np
import pytest
import torch

import oracle as O
import rmsnorm_linear_projection_flashnorm_b200 as fnb
import workloads as WL
from rmsnorm_linear_projection_flashnorm_b200 import torch_api as T
from tests._util import BF16_TOL, fold_ref_bf16, gpu, rel_err, run

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    fnb.build()
    fnb.lib()
    yield
    fnb.fn_set_debug(fnb.FN_DEBUG_FORCE_PATH, 0)


@pytest.fixture(autouse=True, params=[1, 2], ids=["tile256x256", "tile256x512"])
def pair_tile(request):
    """Every test runs with both pair tiles: 256 x 256 (one pair MMA per K step,
    two accumulators) and 256 x 512 (two pair MMAs per K step into one
    512-column accumulator)."""
    assert fnb.fn_set_debug(fnb.FN_DEBUG_PAIR_TILE, request.param) == fnb.FN_OK
    yield request.param
    fnb.fn_set_debug(fnb.FN_DEBUG_PAIR_TILE, 0)


def _case(M, d, N, swiglu, seed):
    inp = WL.case(M, d, N, swiglu, seed=seed)
    g = inp["g"]
    if swiglu:
        Wp, _ = T.fold(gpu(inp["W_gate"]), gpu(g), gpu(inp["W_up"]))
        ref = O.norm_proj_swiglu(inp["x"], np.ones(d), fold_ref_bf16(inp["W_gate"], g),
                                 fold_ref_bf16(inp["W_up"], g), inp["eps"])
    else:
        Wp, _ = T.fold(gpu(inp["W"]), gpu(g))
        ref = O.norm_proj(inp["x"], np.ones(d), fold_ref_bf16(inp["W"], g), inp["eps"])
    return inp, Wp, ref


@pytest.mark.parametrize("M,d,N,swiglu", [
    (512, 256, 512, False),
    (600, 512, 384, False),    # ragged rows; 3 column blocks: the last tile's second half is past N
    (520, 640, 640, True),     # 5 output blocks of 128: the wide tile's last second MMA is past N
    (700, 384, 256, True),     # the last pair: CTA 0 partly, CTA 1 wholly past M
    (1024, 1024, 1280, True),
    (777, 4096, 256, False),   # long k range
    # 80 and 90 tiles of 256 x 512 on 74 pairs: a second, partial wave of
    # tiles (plain; SwiGLU with ragged rows)
    (512, 256, 20480, False),
    (600, 256, 7680, True),
])
def test_pair_kernel_against_oracle_and_single_sm(M, d, N, swiglu):
    inp, Wp, ref = _case(M, d, N, swiglu, seed=240 + M)
    x = gpu(inp["x"])
    y = run(x, Wp, N, inp["eps"], swiglu=swiglu)
    assert rel_err(y, ref) <= BF16_TOL
    assert fnb.fn_set_debug(fnb.FN_DEBUG_FORCE_PATH, 3) == fnb.FN_OK
    try:
        y1 = run(x, Wp, N, inp["eps"], swiglu=swiglu)
    finally:
        fnb.fn_set_debug(fnb.FN_DEBUG_FORCE_PATH, 0)
    assert rel_err(y1, ref) <= BF16_TOL
    assert rel_err(y, y1.cpu().double().numpy()) <= BF16_TOL


def test_pair_kernel_non_finite_and_zero_rows():
    M, d, N = 640, 256, 256
    x = WL.activations(M, d, 250).clone()
    x[3] = 0
    x[300, 5] = float("inf")
    x[513, 7] = float("nan")
    inp = WL.case(M, d, N, False, seed=250)
    Wp, _ = T.fold(gpu(inp["W"]), gpu(inp["g"]))
    y = run(gpu(x), Wp, N, inp["eps"])
    ref = O.norm_proj(x, np.ones(d), fold_ref_bf16(inp["W"], inp["g"]), inp["eps"])
    assert torch.all(y[3].float() == 0)
    assert torch.all(torch.isnan(y[300].float())) and torch.all(torch.isnan(y[513].float()))
    assert rel_err(y, ref) <= BF16_TOL


def test_pair_kernel_repeated_calls_bit_identical():
    M, d, N = 1024, 512, 512
    inp, Wp, _ = _case(M, d, N, True, seed=251)
    x = gpu(inp["x"])
    ws = T.Workspace()
    first = run(x, Wp, N, inp["eps"], swiglu=True, ws=ws).clone()
    for _ in range(100):
        assert torch.equal(run(x, Wp, N, inp["eps"], swiglu=True, ws=ws), first)
    assert ws.status()[0] == fnb.FN_OK


@pytest.mark.parametrize("swiglu", [False, True])
def test_pair_kernel_withheld_arrival_times_out_cleanly(swiglu):
    M, d, N = 600, 512, 512
    inp, Wp, ref = _case(M, d, N, swiglu, seed=252)
    x = gpu(inp["x"])
    ws = T.Workspace()
    assert fnb.fn_set_debug(fnb.FN_DEBUG_WAIT_BUDGET_NS, 20_000_000) == fnb.FN_OK
    assert fnb.fn_set_debug(fnb.FN_DEBUG_WITHHOLD_ARRIVE, 1) == fnb.FN_OK
    try:
        T.norm_proj(x, Wp, N, 1e-6, swiglu=swiglu, ws=ws)
        st, word = ws.status()
    finally:
        fnb.fn_set_debug(fnb.FN_DEBUG_WITHHOLD_ARRIVE, 0)
        fnb.fn_set_debug(fnb.FN_DEBUG_WAIT_BUDGET_NS, 2_000_000_000)
    assert st == fnb.FN_ERR_TIMEOUT and (word >> 8) != 0
    ws.buf.zero_()
    y = T.norm_proj(x, Wp, N, 1e-6, swiglu=swiglu, ws=ws)
    torch.cuda.synchronize()
    assert ws.status()[0] == fnb.FN_OK
    assert rel_err(y, ref) <= BF16_TOL
