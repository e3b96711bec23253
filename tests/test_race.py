"""Synchronisation tests for the join the FlashNorm talk got wrong.

The talk ("실제 버그" / "원인" / "수정" bullets) describes a post-scale that read
an unfinished matmul's old buffer: unit tests and perplexity passed, and only
long generation showed one-step-delayed repetition.  So these tests launch
many calls back to back with inputs that change every call, and demand that
each output is bit-identical to the same call run alone.
"""
import numpy as np
import pytest
import torch

import oracle as O
import rmsnorm_linear_projection_flashnorm_b200 as fnb
import workloads as WL
from rmsnorm_linear_projection_flashnorm_b200 import torch_api as T
from tests._util import BF16_TOL, fold_ref_bf16, gpu, rel_err

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    fnb.build()
    fnb.lib()


def _setup(M, d, N, swiglu, seed):
    inp = WL.case(M, d, N, swiglu, seed=seed)
    if swiglu:
        Wp, _ = T.fold(gpu(inp["W_gate"]), gpu(inp["g"]), gpu(inp["W_up"]))
    else:
        Wp, _ = T.fold(gpu(inp["W"]), gpu(inp["g"]))
    return inp, Wp


@pytest.mark.parametrize("M,calls", [(8, 10_000), (256, 1_000)])
def test_repeated_launches_bit_identical(M, calls):
    """One stream, identical inputs, many launches: every output has the same bits."""
    d, N = 4096, 6144 if M <= 64 else 1024
    inp, Wp = _setup(M, d, N, False, seed=100)
    x = gpu(inp["x"])
    ws = T.Workspace()
    ref = T.norm_proj(x, Wp, N, 1e-6, ws=ws).clone()
    y = torch.empty_like(ref)
    bad = torch.zeros((), dtype=torch.int64, device="cuda")
    for _ in range(calls):
        T.norm_proj(x, Wp, N, 1e-6, ws=ws, out=y)
        bad += (y.view(torch.int16) != ref.view(torch.int16)).sum()
    torch.cuda.synchronize()
    assert int(bad) == 0
    assert ws.status()[0] == fnb.FN_OK


@pytest.mark.parametrize("M,swiglu", [(4, False), (48, True), (192, False), (130, True)])
def test_alternating_inputs(M, swiglu):
    """A, B, A, B, ... into the same output buffer: each equals its solo result."""
    d, N = 1024, 512
    inpA, Wp = _setup(M, d, N, swiglu, seed=101)
    xA = gpu(inpA["x"])
    xB = gpu(WL.activations(M, d, seed=102))
    ws = T.Workspace()
    yA = T.norm_proj(xA, Wp, N, 1e-6, swiglu=swiglu, ws=ws).clone()
    yB = T.norm_proj(xB, Wp, N, 1e-6, swiglu=swiglu, ws=ws).clone()
    assert not torch.equal(yA, yB)
    y = torch.empty_like(yA)
    bad = torch.zeros((), dtype=torch.int64, device="cuda")
    for i in range(400):
        want = yA if i % 2 == 0 else yB
        T.norm_proj(xA if i % 2 == 0 else xB, Wp, N, 1e-6, swiglu=swiglu, ws=ws, out=y)
        bad += (y.view(torch.int16) != want.view(torch.int16)).sum()
    torch.cuda.synchronize()
    assert int(bad) == 0


@pytest.mark.parametrize("M", [1, 16, 96])
def test_chained_generation(M):
    """x_{t+1} = first d columns of y_t, as in autoregressive generation.  The
    back-to-back chain must reproduce the step-by-step (synchronised) chain
    bit for bit, and stay within the oracle's bound."""
    d, N, steps = 512, 1024, 64
    inp, Wp = _setup(M, d, N, False, seed=103)
    ws = T.Workspace()
    # step-by-step reference, synchronising after every call
    x = gpu(inp["x"])
    solo = []
    for _ in range(steps):
        y = T.norm_proj(x, Wp, N, 1e-6, ws=ws)
        torch.cuda.synchronize()
        solo.append(y.clone())
        x = y[:, :d].contiguous()
    # the same chain with no host synchronisation between launches
    x = gpu(inp["x"])
    outs = [torch.empty((M, N), dtype=torch.bfloat16, device="cuda") for _ in range(steps)]
    for t in range(steps):
        T.norm_proj(x, Wp, N, 1e-6, ws=ws, out=outs[t])
        x = outs[t][:, :d].contiguous()
    torch.cuda.synchronize()
    for t in range(steps):
        assert torch.equal(outs[t], solo[t]), f"step {t} differs"
    # the last step against the oracle on its own (stored) input
    x_last = solo[-2][:, :d].cpu()
    ref = O.norm_proj(x_last, np.ones(d), fold_ref_bf16(inp["W"], inp["g"]), 1e-6)
    assert rel_err(solo[-1], ref) <= BF16_TOL


def test_two_streams_distinct_workspaces():
    d, N = 2048, 2048
    inp, Wp = _setup(32, d, N, False, seed=104)
    x1 = gpu(inp["x"])
    x2 = gpu(WL.activations(32, d, seed=105))
    ref1 = T.norm_proj(x1, Wp, N, 1e-6).clone()
    ref2 = T.norm_proj(x2, Wp, N, 1e-6).clone()
    s1, s2 = torch.cuda.Stream(), torch.cuda.Stream()
    w1, w2 = T.Workspace(), T.Workspace()
    y1 = torch.empty_like(ref1)
    y2 = torch.empty_like(ref2)
    torch.cuda.synchronize()
    for _ in range(100):
        with torch.cuda.stream(s1):
            T.norm_proj(x1, Wp, N, 1e-6, ws=w1, out=y1, stream=s1)
        with torch.cuda.stream(s2):
            T.norm_proj(x2, Wp, N, 1e-6, ws=w2, out=y2, stream=s2)
    torch.cuda.synchronize()
    assert torch.equal(y1, ref1) and torch.equal(y2, ref2)
