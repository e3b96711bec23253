"""GPU parity of the decode kernel that gives each thread-block cluster a group
of T adjacent 64-column boxes of W' and splits their k range across the
cluster's S CTAs (bf16 weights, plain projection, bf16 output, M <= 64).  The
partial sums are reduced through distributed shared memory in rank (= k)
order, so one kernel finishes the call: no fix-up kernel.

Checked against the fp64 oracle on the stored folded weight (bf16 W', g = 1)
at the bf16 bound 1e-2 (1 + |y_ref|): the decode QKV shape at every M of its
workload (where the automatic plan picks this kernel), every (T, S) plan
forced on a small shape with a ragged last group and an uneven k split, each
padded row count (16, 32, 64), non-finite and zero rows, bit-identical
repeats, and a withheld arrival that must time out cleanly.  That the call ran
this kernel is read from the library's launch counter: one launch per call,
where stream-K launches its kernel and the fix-up.
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

GROUPS_OFF = 1


def forced(t, s):
    return 2 | (t << 4) | (s << 8)


@pytest.fixture(scope="module", autouse=True)
def _lib():
    fnb.build()
    fnb.lib()
    torch.cuda.init()
    yield
    fnb.fn_set_debug(fnb.FN_DEBUG_DECODE_GROUPS, 0)


def _fold(inp):
    Wp, _ = T.fold(gpu(inp["W"]), gpu(inp["g"]))
    return Wp


def _counted(x, Wp, N, eps, ws=None):
    """One call; returns (y, kernels it launched)."""
    n0 = fnb.fn_kernel_launches()
    y = run(x, Wp, N, eps, ws=ws)
    return y, fnb.fn_kernel_launches() - n0


@pytest.mark.parametrize("M", [1, 8, 32, 64])
def test_decode_qkv_shape_one_kernel(M):
    """d = 4096, N = 6144: the automatic plan takes the cluster kernel (one
    launch); stream-K (forced) needs its fix-up kernel (two).  Both match the
    oracle."""
    w = WL.WORKLOADS["decode_qkv"]
    inp = WL.workload_case("decode_qkv", M)
    Wp = _fold(inp)
    x = gpu(inp["x"])
    ref = O.norm_proj(inp["x"], np.ones(w.d), fold_ref_bf16(inp["W"], inp["g"]), inp["eps"])
    y, n = _counted(x, Wp, w.N, inp["eps"])
    assert n == 1
    assert rel_err(y, ref) <= BF16_TOL
    assert rel_err(y, O.norm_proj(inp["x"], inp["g"], inp["W"], inp["eps"])) <= BF16_TOL   # end to end
    fnb.fn_set_debug(fnb.FN_DEBUG_DECODE_GROUPS, GROUPS_OFF)
    try:
        y_sk, n_sk = _counted(x, Wp, w.N, inp["eps"])
    finally:
        fnb.fn_set_debug(fnb.FN_DEBUG_DECODE_GROUPS, 0)
    assert n_sk == 2
    assert rel_err(y_sk, ref) <= BF16_TOL


PLANS = [(1, 2), (1, 8), (2, 2), (2, 4), (2, 8), (3, 2), (3, 3), (3, 4), (3, 6), (3, 8)]


@pytest.mark.parametrize("M", [1, 20, 64])
@pytest.mark.parametrize("t,s", PLANS)
def test_forced_plans(M, t, s):
    """N = 640 (10 boxes: with T = 3 the last group holds one box and two boxes
    of zero fill), d = 1216 (19 k blocks, split unevenly over S CTAs)."""
    d, N = 1216, 640
    inp = WL.case(M, d, N, False, seed=300 + 10 * t + s)
    Wp = _fold(inp)
    fnb.fn_set_debug(fnb.FN_DEBUG_DECODE_GROUPS, forced(t, s))
    try:
        y, n = _counted(gpu(inp["x"]), Wp, N, inp["eps"])
    finally:
        fnb.fn_set_debug(fnb.FN_DEBUG_DECODE_GROUPS, 0)
    assert n == 1
    ref = O.norm_proj(inp["x"], np.ones(d), fold_ref_bf16(inp["W"], inp["g"]), inp["eps"])
    assert rel_err(y, ref) <= BF16_TOL


@pytest.mark.parametrize("M", [3, 40])
def test_zero_and_non_finite_rows(M):
    """A zero row gives zeros; an inf or NaN makes its row NaN; other rows are
    unaffected (their partials and sums of squares travel separately)."""
    d, N = 512, 384
    x = WL.activations(M, d, 310).clone()
    x[0] = 0
    x[1, 7] = float("inf")
    x[2, 300] = float("nan")
    inp = WL.case(M, d, N, False, seed=310)
    Wp = _fold(inp)
    fnb.fn_set_debug(fnb.FN_DEBUG_DECODE_GROUPS, forced(3, 4))
    try:
        y, n = _counted(gpu(x), Wp, N, 1e-6)
    finally:
        fnb.fn_set_debug(fnb.FN_DEBUG_DECODE_GROUPS, 0)
    assert n == 1
    assert torch.all(y[0].float() == 0)
    assert torch.all(torch.isnan(y[1:3].float()))
    ref = O.norm_proj(x, np.ones(d), fold_ref_bf16(inp["W"], inp["g"]), 1e-6)
    assert rel_err(y, ref) <= BF16_TOL


@pytest.mark.parametrize("M", [8, 64])
def test_repeated_calls_bit_identical_and_timeout(M):
    """Repeats of the decode QKV shape give the same bits; a withheld reducer
    arrival makes the epilogue's bounded wait give up with FN_ERR_TIMEOUT, the
    cluster still meets at its barriers and exits, and the next call (zeroed
    workspace) is correct."""
    w = WL.WORKLOADS["decode_qkv"]
    inp = WL.workload_case("decode_qkv", M)
    Wp = _fold(inp)
    x = gpu(inp["x"])
    ws = T.Workspace()
    first, n = _counted(x, Wp, w.N, inp["eps"], ws=ws)
    first = first.clone()
    assert n == 1
    for _ in range(100):
        assert torch.equal(run(x, Wp, w.N, inp["eps"], ws=ws), first)
    assert ws.status()[0] == fnb.FN_OK
    assert fnb.fn_set_debug(fnb.FN_DEBUG_WAIT_BUDGET_NS, 20_000_000) == fnb.FN_OK
    assert fnb.fn_set_debug(fnb.FN_DEBUG_WITHHOLD_ARRIVE, 1) == fnb.FN_OK
    try:
        T.norm_proj(x, Wp, w.N, inp["eps"], ws=ws)
        st, word = ws.status()
    finally:
        fnb.fn_set_debug(fnb.FN_DEBUG_WITHHOLD_ARRIVE, 0)
        fnb.fn_set_debug(fnb.FN_DEBUG_WAIT_BUDGET_NS, 2_000_000_000)
    assert st == fnb.FN_ERR_TIMEOUT and (word >> 8) != 0
    ws.buf.zero_()
    assert torch.equal(run(x, Wp, w.N, inp["eps"], ws=ws), first)
    assert ws.status()[0] == fnb.FN_OK
