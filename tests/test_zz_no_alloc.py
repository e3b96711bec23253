"""fn_norm_proj_static: the entry point for callers that cannot allocate device
memory (stream capture, plug-ins whose host owns all allocations, loops that
must not synchronise through cudaMalloc).  Its scratch is a fixed array inside
the library; its results must match fn_norm_proj, which uses a caller-provided
workspace, on consecutive calls (the array keeps the previous call's contents).

This file is collected last on purpose, so a run that stops at the first
failure has already run every other test."""
import numpy as np
import pytest
import torch

import rmsnorm_linear_projection_flashnorm_b200 as fnb
import workloads as WL
from rmsnorm_linear_projection_flashnorm_b200 import torch_api as T
from tests._util import BF16_TOL, rel_err

pytestmark = pytest.mark.gpu


def test_static_scratch_matches_workspace_entry_point():
    fnb.build()
    d, N = 4096, 6144
    inp = WL.case(8, d, N, False, seed=120)
    Wp, _ = T.fold(inp["W"].cuda(), inp["g"].cuda())
    xs = [inp["x"].cuda(), WL.activations(8, d, seed=121).cuda()]
    for x in xs:                                    # two calls in a row, different inputs
        ref = T.norm_proj(x, Wp, N, 1e-6)           # existing entry point, own workspace
        y = torch.empty_like(ref)
        st = fnb.fn_norm_proj_static(x, 8, d, Wp, None, fnb.FN_W_BF16, N, 1e-6, y, None)
        assert st == fnb.FN_OK, fnb.status_string(st)
        torch.cuda.synchronize()
        assert rel_err(y.cpu(), ref.cpu().double().numpy()) <= BF16_TOL
        assert torch.equal(y, ref)                  # same kernels, same order: same bits


def test_static_scratch_rejects_sizes_beyond_its_maximum():
    fnb.build()
    # M = 64 on the decode QKV shape needs about 9.8 MB of split-K partials on
    # 148 SMs, more than the 8 MiB array; the pointers are never touched
    d, N = 4096, 6144
    assert fnb.fn_workspace_size(64, d, N, fnb.FN_W_BF16, 0) > (8 << 20)
    st = fnb.fn_norm_proj_static(1 << 20, 64, d, 1 << 30, None, fnb.FN_W_BF16, N, 1e-6, 1 << 34, None)
    assert st == fnb.FN_ERR_WORKSPACE
    assert fnb.fn_workspace_size(32, d, N, fnb.FN_W_BF16, 0) <= (8 << 20)
