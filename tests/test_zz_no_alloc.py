"""fn_norm_proj_static: the entry point for callers that cannot allocate device
memory (stream capture, plug-ins whose host owns all allocations, loops that
must not synchronise through cudaMalloc).  Its scratch is a fixed array inside
the library; its results must match fn_norm_proj, which uses a caller-provided
workspace, and the fp64 oracle, on consecutive calls (the array keeps the
previous call's contents).

This file is collected last on purpose, so a run that stops at the first
failure has already run every other test."""
import numpy as np
import pytest
import torch

import oracle as O
import rmsnorm_linear_projection_flashnorm_b200 as fnb
import workloads as WL
from rmsnorm_linear_projection_flashnorm_b200 import torch_api as T
from tests._util import BF16_TOL, FP8_TOL, fold_fp8_ref, fold_ref_bf16, rel_err

pytestmark = pytest.mark.gpu
STATIC_BYTES = 8 << 20


@pytest.fixture(scope="module", autouse=True)
def _lib():
    fnb.build()
    fnb.lib()


def _nonblocking_stream():
    """A stream created with cudaStreamNonBlocking (no implicit ordering with
    the legacy default stream), wrapped for torch."""
    from cuda.bindings import runtime as rt
    err, s = rt.cudaStreamCreateWithFlags(rt.cudaStreamNonBlocking)
    assert err == rt.cudaError_t.cudaSuccess
    return torch.cuda.ExternalStream(int(s)), s


def _destroy(raw):
    from cuda.bindings import runtime as rt
    rt.cudaStreamDestroy(raw)


@pytest.mark.parametrize("M,d,N,fp8", [(8, 4096, 6144, False), (200, 1024, 1536, False), (32, 1024, 2048, True)])
def test_static_scratch_matches_workspace_entry_point(M, d, N, fp8):
    """Two calls in a row with different inputs on a non-blocking stream:
    the same bits as fn_norm_proj with its own workspace, and within the
    kernel tolerance of the oracle.  The shapes cover the bf16 decode path
    (split-K partials in the scratch), the tile path (status word only) and
    the fp8 decode path at 17..64 rows (activations split into the scratch)."""
    wt = fnb.FN_W_FP8_E4M3_B128 if fp8 else fnb.FN_W_BF16
    assert fnb.fn_workspace_size(M, d, N, wt, 0) <= STATIC_BYTES
    inp = WL.case(M, d, N, False, seed=120)
    Wp, s = T.fold(inp["W"].cuda(), inp["g"].cuda(), wtype=wt)
    if fp8:
        q, sr = fold_fp8_ref(inp["W"], inp["g"])
        Wref, tol = O.dequant_fp8(q, sr), FP8_TOL
    else:
        Wref, tol = fold_ref_bf16(inp["W"], inp["g"]), BF16_TOL
    xs_host = [inp["x"], WL.activations(M, d, seed=121)]
    stream, raw = _nonblocking_stream()
    try:
        with torch.cuda.stream(stream):
            xs = [x.cuda() for x in xs_host]
            outs = []
            for x in xs:                                  # two calls in a row, different inputs
                y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
                st = fnb.fn_norm_proj_static(x, M, d, Wp, s, wt, N, 1e-6, y, stream)
                assert st == fnb.FN_OK, fnb.status_string(st)
                ref = T.norm_proj(x, Wp, N, 1e-6, scales=s, stream=stream)   # the workspace entry point
                outs.append((y, ref))
            stream.synchronize()
        assert fnb.fn_query_static_status(stream)[0] == fnb.FN_OK
        for (y, ref), xh in zip(outs, xs_host):
            assert torch.equal(y, ref)                    # same kernels, same order: same bits
            assert rel_err(y.cpu(), O.norm_proj(xh, np.ones(d), Wref, 1e-6)) <= tol
    finally:
        _destroy(raw)


def test_static_scratch_rejects_sizes_beyond_its_maximum():
    # M = 64 on the decode QKV shape needs about 9.8 MB of split-K partials on
    # 148 SMs, more than the 8 MiB array; fp8 weights at 8192 rows need the
    # split activations (84 MB) and, for NVFP4 or partial outputs, a bf16 copy
    # of the weight.  Small real buffers stand in for the operands: the size
    # check rejects the call before anything is launched.
    d, N = 4096, 6144
    assert fnb.fn_workspace_size(64, d, N, fnb.FN_W_BF16, 0) > STATIC_BYTES
    assert fnb.fn_workspace_size(32, d, N, fnb.FN_W_BF16, 0) <= STATIC_BYTES
    x = torch.zeros(1024, dtype=torch.bfloat16, device="cuda")
    Wp = torch.zeros(1024, dtype=torch.bfloat16, device="cuda")
    y = torch.zeros(1024, dtype=torch.bfloat16, device="cuda")
    st = fnb.fn_norm_proj_static(x, 64, d, Wp, None, fnb.FN_W_BF16, N, 1e-6, y, None)
    assert st == fnb.FN_ERR_WORKSPACE
    d8, N8 = 5120, 13824
    assert fnb.fn_workspace_size(8192, d8, N8, fnb.FN_W_FP8_E4M3_B128, 0) > STATIC_BYTES
    sc = torch.ones(64, dtype=torch.float32, device="cuda")
    st = fnb.fn_norm_proj_static(x, 8192, d8, Wp, sc, fnb.FN_W_FP8_E4M3_B128, N8, 1e-6, y, None)
    assert st == fnb.FN_ERR_WORKSPACE
    torch.cuda.synchronize()


def test_static_timeout_is_reported_and_cleared():
    """A wait that cannot complete (the reducers withhold their first
    arrival, a flag that nothing sets) gives up after its budget and records
    FN_ERR_TIMEOUT in the static scratch; fn_query_static_status reports it
    once and clears it, and the next call is correct."""
    M, d, N = 8, 512, 512
    inp = WL.case(M, d, N, False, seed=122)
    Wp, _ = T.fold(inp["W"].cuda(), inp["g"].cuda())
    x = inp["x"].cuda()
    y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    assert fnb.fn_set_debug(fnb.FN_DEBUG_WAIT_BUDGET_NS, 20_000_000) == fnb.FN_OK   # 20 ms
    assert fnb.fn_set_debug(fnb.FN_DEBUG_WITHHOLD_ARRIVE, 1) == fnb.FN_OK
    try:
        st = fnb.fn_norm_proj_static(x, M, d, Wp, None, fnb.FN_W_BF16, N, 1e-6, y, None)
        assert st == fnb.FN_OK
        st, word = fnb.fn_query_static_status(None)
    finally:
        fnb.fn_set_debug(fnb.FN_DEBUG_WITHHOLD_ARRIVE, 0)
        fnb.fn_set_debug(fnb.FN_DEBUG_WAIT_BUDGET_NS, 2_000_000_000)
    assert st == fnb.FN_ERR_TIMEOUT and (word & 0xFF) == fnb.FN_ERR_TIMEOUT and (word >> 8) != 0
    assert fnb.fn_query_static_status(None) == (fnb.FN_OK, 0)
    assert fnb.fn_norm_proj_static(x, M, d, Wp, None, fnb.FN_W_BF16, N, 1e-6, y, None) == fnb.FN_OK
    assert fnb.fn_query_static_status(None)[0] == fnb.FN_OK
    ref = O.norm_proj(inp["x"], np.ones(d), fold_ref_bf16(inp["W"], inp["g"]), 1e-6)
    assert rel_err(y.cpu(), ref) <= BF16_TOL
