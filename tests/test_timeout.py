"""Bounded waits: a device-side wait that cannot complete gives up after its
time budget, records FN_ERR_TIMEOUT in the workspace status word and lets the
kernel tear down (drain its copies and MMAs, free TMEM) and exit.  The context
stays usable.

The failure is made by a test knob that makes the sum-of-squares reducers
withhold their first arrival, so the epilogue's wait on that barrier never
completes: a flag that nothing sets.  No fault, trap or endless loop is used.
"""
import numpy as np
import pytest
import torch

import rmsnorm_linear_projection_flashnorm_b200 as fnb
import workloads as WL
from rmsnorm_linear_projection_flashnorm_b200 import torch_api as T
from tests._util import BF16_TOL, fold_ref_bf16, gpu, rel_err
import oracle as O

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("M,swiglu", [(8, False), (40, True), (300, False), (200, True)])
def test_withheld_arrival_times_out_cleanly(M, swiglu):
    fnb.build()
    d, N = 512, 512
    inp = WL.case(M, d, N, swiglu, seed=110)
    if swiglu:
        Wp, _ = T.fold(gpu(inp["W_gate"]), gpu(inp["g"]), gpu(inp["W_up"]))
    else:
        Wp, _ = T.fold(gpu(inp["W"]), gpu(inp["g"]))
    x = gpu(inp["x"])
    ws = T.Workspace()
    assert fnb.fn_set_debug(fnb.FN_DEBUG_WAIT_BUDGET_NS, 20_000_000) == fnb.FN_OK   # 20 ms
    assert fnb.fn_set_debug(fnb.FN_DEBUG_WITHHOLD_ARRIVE, 1) == fnb.FN_OK
    try:
        T.norm_proj(x, Wp, N, 1e-6, swiglu=swiglu, ws=ws)
        st, word = ws.status()
    finally:
        fnb.fn_set_debug(fnb.FN_DEBUG_WITHHOLD_ARRIVE, 0)
        fnb.fn_set_debug(fnb.FN_DEBUG_WAIT_BUDGET_NS, 2_000_000_000)
    assert st == fnb.FN_ERR_TIMEOUT
    assert (word & 0xFF) == fnb.FN_ERR_TIMEOUT and (word >> 8) != 0
    # the context is still usable, and a zeroed workspace gives correct results
    ws.buf.zero_()
    y = T.norm_proj(x, Wp, N, 1e-6, swiglu=swiglu, ws=ws)
    torch.cuda.synchronize()
    assert ws.status()[0] == fnb.FN_OK
    if swiglu:
        ref = O.norm_proj_swiglu(inp["x"], np.ones(d), fold_ref_bf16(inp["W_gate"], inp["g"]),
                                 fold_ref_bf16(inp["W_up"], inp["g"]), 1e-6)
    else:
        ref = O.norm_proj(inp["x"], np.ones(d), fold_ref_bf16(inp["W"], inp["g"]), 1e-6)
    assert rel_err(y, ref) <= BF16_TOL
