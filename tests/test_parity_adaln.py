"""GPU parity of the AdaLN-modulated fused call (the "RMSNorm + AdaLN" front
of the fused FC1 on the FlashInfer PR #5521 analysis): per-token index into
scale and shift rows applied after the norm.

The kernel computes r * ((x * scale[c]) @ W') + B[c] with W' the stored
folded weight and B = shift @ W the fp32 shift bias.  Kernel parity is
against the oracle on the stored operands (the deferred split, pinned on CPU
against the unfolded definition): the scaled activations as the MMA takes
them (one bf16 rounding of the fp32 product) through W', times the 1/rms of
the raw rows, plus the shift through the original W, within 1e-2 (1 + |y_ref|)
for bf16 weights and 6e-2 for e4m3 weights.  The plain projection is also compared end to end with the oracle's
unfolded definition (original W and g) under a looser sanity bound, since the
modulated activations take one more bf16 rounding than the plain path.
"""
import numpy as np
import pytest
import torch

import oracle as O
import rmsnorm_linear_projection_flashnorm_b200 as fnb
import workloads as WL
from rmsnorm_linear_projection_flashnorm_b200 import torch_api as T
from tests._util import BF16_TOL, FP8_TOL, fold_fp8_ref, fold_ref_bf16, gpu, rel_err

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    fnb.build()
    fnb.lib()


def _cond(n_cond, d, M, seed):
    rng = np.random.default_rng(seed)
    scale = (1.0 + 0.3 * rng.standard_normal((n_cond, d))).astype(np.float32)
    shift = (0.5 * rng.standard_normal((n_cond, d))).astype(np.float32)
    index = rng.integers(0, n_cond, M).astype(np.int32)
    return scale, shift, index


def _run(M, d, N, swiglu, n_cond, seed, wt=fnb.FN_W_BF16, index=None):
    inp = WL.case(M, d, N, swiglu, seed=seed)
    scale, shift, idx = _cond(n_cond, d, M, seed)
    if index is not None:
        idx = index
    g = inp["g"]
    W0 = inp["W_gate"] if swiglu else inp["W"]
    W1 = inp["W_up"] if swiglu else None
    Wp, s = T.fold(gpu(W0), gpu(g), gpu(W1) if swiglu else None, wtype=wt)
    B = T.adaln_shift_bias(gpu(torch.from_numpy(shift)), gpu(W0), gpu(W1) if swiglu else None)
    y = T.norm_proj_adaln(gpu(inp["x"]), Wp, N, inp["eps"], gpu(torch.from_numpy(scale)), B,
                          gpu(torch.from_numpy(idx)), swiglu=swiglu, scales=s)
    torch.cuda.synchronize()
    # oracle on the stored operands: the scaled activations as the MMA takes
    # them (bf16) through the stored W', the deferred 1/rms of the raw rows,
    # the shift through the original W
    safe = np.clip(idx, 0, n_cond - 1)
    xm = O.adaln_scaled_operand(inp["x"], scale, safe)
    r = O.rms_inv(inp["x"], inp["eps"])[:, None]
    if wt == fnb.FN_W_BF16:
        Ws = [fold_ref_bf16(W0, g)] + ([fold_ref_bf16(W1, g)] if swiglu else [])
    else:
        q, sr = fold_fp8_ref(W0, g, W1)
        deq = O.dequant_fp8(q, sr)
        Ws = list(O.deinterleave128(deq)) if swiglu else [deq]
    parts = [r * (xm @ Wsi) for Wsi in Ws]
    biases = [O.adaln_shift_bias(shift, O.to_f64(Wo))[safe] for Wo in ([W0, W1] if swiglu else [W0])]
    if swiglu:
        ref = O.silu(parts[0] + biases[0]) * (parts[1] + biases[1])
    else:
        ref = parts[0] + biases[0]
    return y, ref, inp, scale, shift, idx


@pytest.mark.parametrize("M,d,N,n_cond", [
    (1, 256, 384, 1),      # a decode-sized batch still runs on the tile kernel
    (8, 512, 256, 3),
    (100, 256, 640, 4),    # ragged row tile, odd number of 128-column blocks
    (300, 512, 384, 2),
    (64, 1024, 512, 5),
])
def test_adaln_plain(M, d, N, n_cond):
    y, ref, inp, scale, shift, idx = _run(M, d, N, False, n_cond, seed=200 + M)
    assert rel_err(y, ref) <= BF16_TOL
    # End to end against the unfolded definition (original W and g): besides
    # the stored bf16 W', the modulated activations x * scale are rounded to
    # bf16 for the MMA, one rounding more than the plain path, which moves
    # results by about 1e-2 (1 + |y|); the gate is the kernel parity above,
    # this bound only catches gross departures.
    e2e = O.norm_proj_adaln(inp["x"], inp["g"], inp["W"], inp["eps"], scale, shift, idx)
    assert rel_err(y, e2e) <= 2 * BF16_TOL


@pytest.mark.parametrize("M,d,N,n_cond", [(1, 256, 256, 2), (40, 512, 384, 3), (260, 384, 256, 4)])
def test_adaln_swiglu(M, d, N, n_cond):
    y, ref, *_ = _run(M, d, N, True, n_cond, seed=210 + M)
    assert rel_err(y, ref) <= BF16_TOL


@pytest.mark.parametrize("M,swiglu", [(16, False), (200, True)])
def test_adaln_fp8_weights(M, swiglu):
    """e4m3 weights with 128x128 scales go through the bf16 conversion first."""
    y, ref, *_ = _run(M, 512, 256, swiglu, 3, seed=220 + M, wt=fnb.FN_W_FP8_E4M3_B128)
    assert rel_err(y, ref) <= FP8_TOL


def test_adaln_invalid_index_gives_nan_rows():
    M, n_cond = 6, 3
    idx = np.array([0, 5, 1, -1, 2, 2], dtype=np.int32)
    y, ref, *_ = _run(M, 256, 256, False, n_cond, seed=230, index=idx)
    yf = y.float().cpu()
    assert torch.all(torch.isnan(yf[1])) and torch.all(torch.isnan(yf[3]))
    good = [0, 2, 4, 5]
    assert rel_err(y.cpu()[good], ref[good]) <= BF16_TOL


def test_adaln_shift_bias_matches_oracle():
    d, N, n_cond = 512, 384, 4
    inp = WL.case(1, d, N, True, seed=231)
    _, shift, _ = _cond(n_cond, d, 1, 231)
    B = T.adaln_shift_bias(gpu(torch.from_numpy(shift)), gpu(inp["W_gate"]), gpu(inp["W_up"]))
    torch.cuda.synchronize()
    want = O.interleave128(O.adaln_shift_bias(shift, O.to_f64(inp["W_gate"])),
                           O.adaln_shift_bias(shift, O.to_f64(inp["W_up"])))
    got = B.cpu().double().numpy()
    assert np.max(np.abs(got - want) / (1 + np.abs(want))) <= 1e-5


def test_adaln_repeated_calls_bit_identical():
    M, d, N = 200, 512, 512
    inp = WL.case(M, d, N, True, seed=232)
    scale, shift, idx = _cond(3, d, M, 232)
    Wp, _ = T.fold(gpu(inp["W_gate"]), gpu(inp["g"]), gpu(inp["W_up"]))
    B = T.adaln_shift_bias(gpu(torch.from_numpy(shift)), gpu(inp["W_gate"]), gpu(inp["W_up"]))
    args = (gpu(inp["x"]), Wp, N, inp["eps"], gpu(torch.from_numpy(scale)), B, gpu(torch.from_numpy(idx)))
    ws = T.Workspace()
    first = T.norm_proj_adaln(*args, swiglu=True, ws=ws).clone()
    for _ in range(100):
        assert torch.equal(T.norm_proj_adaln(*args, swiglu=True, ws=ws), first)
    assert ws.status()[0] == fnb.FN_OK
