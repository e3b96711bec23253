"""GPU parity with fp8 (e4m3, 128x128 block-scaled) folded weights.

The activations stay bf16; the kernels convert each staged e4m3 weight tile
to bf16 on chip (fp32 product with the block scale, one rounding) and run the
bf16 MMA.  Kernel parity is against the oracle evaluated on the stored,
dequantised weight W_deq = e4m3(q) * s (exact in fp64) with g = 1, within
6e-2 (1 + |y_ref|).  The oracle's own fold provides W_deq; the GPU folds the
same weights itself, and the fold's bit-exactness is a separate test.
"""
import numpy as np
import pytest
import torch

import oracle as O
import rmsnorm_linear_projection_flashnorm_b200 as fnb
import workloads as WL
from rmsnorm_linear_projection_flashnorm_b200 import torch_api as T
from tests._util import FP8_TOL, fold_fp8_ref, gpu, rel_err, run, sample_cols

pytestmark = pytest.mark.gpu
FP8 = fnb.FN_W_FP8_E4M3_B128


@pytest.fixture(scope="module", autouse=True)
def _lib():
    fnb.build()
    fnb.lib()
    yield
    fnb.fn_set_debug(fnb.FN_DEBUG_FORCE_PATH, 0)


def test_dequant_step_bit_exact():
    inp = WL.case(4, 256, 384, False, seed=130)
    q, s = fold_fp8_ref(inp["W"], inp["g"])
    qd, sd = gpu(torch.from_numpy(q)), gpu(torch.from_numpy(s))
    W = torch.empty((256, 384), dtype=torch.bfloat16, device="cuda")
    assert fnb.fn_dequant_fp8(qd, sd, 256, 384, W, None) == fnb.FN_OK
    torch.cuda.synchronize()
    got = W.cpu().view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(got, O.dequant_fp8_bf16_bits(q, s))


def _case(M, d, N, swiglu, seed):
    inp = WL.case(M, d, N, swiglu, seed=seed)
    x, g = inp["x"], inp["g"]
    if swiglu:
        Wq, s = T.fold(gpu(inp["W_gate"]), gpu(g), gpu(inp["W_up"]), wtype=FP8)
        q, sr = fold_fp8_ref(inp["W_gate"], g, inp["W_up"])
        Wg, Wu = O.deinterleave128(O.dequant_fp8(q, sr))
        ref = O.norm_proj_swiglu(x, np.ones(d), Wg, Wu, inp["eps"])
    else:
        Wq, s = T.fold(gpu(inp["W"]), gpu(g), wtype=FP8)
        q, sr = fold_fp8_ref(inp["W"], g)
        ref = O.norm_proj(x, np.ones(d), O.dequant_fp8(q, sr), inp["eps"])
    y = run(gpu(x), Wq, N, inp["eps"], swiglu=swiglu, scales=s)
    return y, ref


@pytest.mark.parametrize("M,d,N,swiglu", [
    (5, 256, 384, False),      # decode, odd number of 128-column blocks
    (200, 256, 384, False),    # tile path: the last 256-column tile is half past the weight
    (40, 384, 256, True),      # decode SwiGLU
    (300, 512, 384, True),     # tile SwiGLU, ragged M
    (64, 128, 128, False),     # single k block, single tile
    (129, 640, 640, True),
    (1100, 256, 256, True),    # M >= 1024: the weight is dequantised once into the workspace
    (1024, 384, 384, False),
])
def test_fp8_small(M, d, N, swiglu):
    y, ref = _case(M, d, N, swiglu, seed=131)
    assert rel_err(y, ref) <= FP8_TOL


@pytest.mark.parametrize("path", [1, 2])
def test_fp8_both_paths_at_small_m(path):
    fnb.fn_set_debug(fnb.FN_DEBUG_FORCE_PATH, path)
    try:
        for M, sw in ((3, False), (33, True)):
            y, ref = _case(M, 256, 256, sw, seed=132)
            assert rel_err(y, ref) <= FP8_TOL
    finally:
        fnb.fn_set_debug(fnb.FN_DEBUG_FORCE_PATH, 0)


@pytest.fixture(scope="module")
def fp8_workload():
    w = WL.WORKLOADS["fp8_swiglu"]
    inp = WL.workload_case("fp8_swiglu", max(w.Ms))
    g = inp["g"]
    Wq, s = T.fold(gpu(inp["W_gate"]), gpu(g), gpu(inp["W_up"]), wtype=FP8)
    q, sr = fold_fp8_ref(inp["W_gate"], g, inp["W_up"])
    Wg, Wu = O.deinterleave128(O.dequant_fp8(q, sr))
    torch.cuda.synchronize()
    return w, inp, Wq, s, Wg, Wu


@pytest.mark.parametrize("M", [1, 64, 256])
def test_fp8_workload(fp8_workload, M):
    w, inp, Wq, s, Wg, Wu = fp8_workload
    x = inp["x"][:M]
    y = run(gpu(x), Wq, w.N, inp["eps"], swiglu=True, scales=s)
    ref = O.norm_proj_swiglu(x, np.ones(w.d), Wg, Wu, inp["eps"])
    assert rel_err(y, ref) <= FP8_TOL


@pytest.mark.slow
def test_fp8_workload_prefill_sampled(fp8_workload):
    w, inp, Wq, s, Wg, Wu = fp8_workload
    M = max(w.Ms)
    y = run(gpu(inp["x"]), Wq, w.N, inp["eps"], swiglu=True, scales=s)
    rows = WL.sample_rows(M, w.seed)
    ref = O.norm_proj_swiglu(inp["x"][rows], np.ones(w.d), Wg, Wu, inp["eps"])
    assert rel_err(y.cpu()[rows], ref) <= FP8_TOL
