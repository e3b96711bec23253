"""GPU parity with MXFP8 folded weights: e4m3 codes with one ue8m0 scale per
32 k values of each column, in the chunked layout block-scaled tensor-core
MMAs read.

The fold must be bit-identical to the oracle's (codes and scale bytes, plain
and gate/up interleaved).  At M <= 64 the codes and scales go to the
block-scaled MMAs as stored and the bf16 activations are split exactly into
two e4m3 parts sharing a power-of-two scale, so the products are those of the
stored weight; at M > 64 with bf16 output the promotion tile kernel does the
same with block-scaled MMAs over each tile's whole k range, and the other
tile-path forms (and FN_DEBUG_FORCE_PATH 4) convert the weight to bf16 once
per call (an exact conversion, checked bit for bit).  Kernel parity is
therefore against the oracle on the dequantised stored weight e4m3(q) * 2^E
(exact in fp64) with g = 1, and every case holds the bf16 bound
1e-2 (1 + |y_ref|), tighter than the 6e-2 bound stated for fp8 weights.
"""
import numpy as np
import pytest
import torch

import oracle as O
import rmsnorm_linear_projection_flashnorm_b200 as fnb
import workloads as WL
from rmsnorm_linear_projection_flashnorm_b200 import torch_api as T
from tests._util import BF16_TOL, check_nvfp4, gpu, rel_err, run

pytestmark = pytest.mark.gpu
MX = fnb.FN_W_MXFP8_E4M3


@pytest.fixture(scope="module", autouse=True)
def _lib():
    fnb.build()
    fnb.lib()
    yield
    fnb.fn_set_debug(fnb.FN_DEBUG_FORCE_PATH, 0)


def mx_ref(W0, g, W1=None):
    """The oracle's MXFP8 fold in the stored order: codes [d, ncols], scale
    bytes, and the dequantised stored weight (fp64, stored column order)."""
    if W1 is None:
        q, sb = O.fold_mxfp8(W0, g)
    else:
        qg, sg = O.fold_mxfp8(W0, g)
        qu, su = O.fold_mxfp8(W1, g)
        q, sb = O.interleave128(qg, qu), O.interleave128(sg, su)
    return q, O.mx_scale_store(sb), O.dequant_mxfp8(q, sb)


def _case(M, d, N, swiglu, seed, x=None):
    inp = WL.case(M, d, N, swiglu, seed=seed)
    if x is not None:
        inp["x"] = x
    x, g = inp["x"], inp["g"]
    if swiglu:
        Wq, s = T.fold(gpu(inp["W_gate"]), gpu(g), gpu(inp["W_up"]), wtype=MX)
        Wg, Wu = O.deinterleave128(mx_ref(inp["W_gate"], g, inp["W_up"])[2])
        ref = O.norm_proj_swiglu(x, np.ones(d), Wg, Wu, inp["eps"])
    else:
        Wq, s = T.fold(gpu(inp["W"]), gpu(g), wtype=MX)
        ref = O.norm_proj(x, np.ones(d), mx_ref(inp["W"], g)[2], inp["eps"])
    y = run(gpu(x), Wq, N, inp["eps"], swiglu=swiglu, scales=s)
    return y, ref


@pytest.mark.parametrize("d,N,swiglu", [(256, 384, False), (512, 256, True), (1024, 640, False)])
def test_mxfp8_fold_bit_exact(d, N, swiglu):
    inp = WL.case(2, d, N, swiglu, seed=160)
    g = inp["g"]
    if swiglu:
        Wq, s = T.fold(gpu(inp["W_gate"]), gpu(g), gpu(inp["W_up"]), wtype=MX)
        q, flat, _ = mx_ref(inp["W_gate"], g, inp["W_up"])
    else:
        W = inp["W"].clone()
        W[32:64, 5] = 0                                     # an all-zero block
        W[64:96, 7] = (W[64:96, 7].float() * 1e-30).to(torch.bfloat16)   # tiny values, subnormal codes
        Wq, s = T.fold(gpu(W), gpu(g), wtype=MX)
        q, flat, _ = mx_ref(W, g)
    torch.cuda.synchronize()
    assert np.array_equal(Wq.cpu().numpy(), q)
    assert np.array_equal(s.cpu().numpy(), flat)


def test_mxfp8_dequant_bit_exact():
    d, ncols = 256, 384
    inp = WL.case(2, d, ncols, False, seed=161)
    q, flat, deq = mx_ref(inp["W"], inp["g"])
    W = torch.empty((d, ncols), dtype=torch.bfloat16, device="cuda")
    assert fnb.fn_dequant_mxfp8(gpu(torch.from_numpy(q)), gpu(torch.from_numpy(flat)), d, ncols, W, None) == fnb.FN_OK
    torch.cuda.synchronize()
    got = W.cpu().view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(got, O.bf16_bits(deq))


@pytest.mark.parametrize("M", [1, 2, 15, 16, 17, 31, 32, 33, 63, 64])
@pytest.mark.parametrize("swiglu", [False, True])
def test_mxfp8_decode_m_ladder(M, swiglu):
    """Every padded row count of the block-scaled decode kernel (16, 32, 64)."""
    y, ref = _case(M, 512, 768 if not swiglu else 384, swiglu, seed=170 + M)
    assert rel_err(y, ref) <= BF16_TOL


@pytest.mark.parametrize("M,d,N,swiglu", [
    (5, 256, 384, False),      # odd number of 128-column blocks
    (40, 384, 256, True),
    (64, 128, 128, False),     # single k group, single tile
    (8, 2048, 1024, True),     # k split across CTAs: fix-up kernel
    (200, 256, 384, False),    # tile path: block-scaled promotion kernel
    (300, 512, 384, True),
])
def test_mxfp8_small(M, d, N, swiglu):
    y, ref = _case(M, d, N, swiglu, seed=171)
    assert rel_err(y, ref) <= BF16_TOL


@pytest.mark.parametrize("M,d,N,swiglu", [
    (65, 128, 128, False),     # one k group, one ragged row block
    (129, 1024, 640, False),   # odd number of 128-column blocks, ragged rows
    (250, 2048, 896, True),    # several k groups and tiles
    (700, 768, 2304, True),    # 6 x 9 tiles: a last partial wave split in k over CTA pairs
    (1030, 512, 1280, False),  # several row blocks, ragged
])
def test_mxfp8_promotion_kernel(M, d, N, swiglu):
    """MXFP8 at M > 64 with bf16 output: x split per 32-deep block into e4m3
    hi/lo planes with ue8m0 scales, block-scaled MMAs on the stored codes."""
    y, ref = _case(M, d, N, swiglu, seed=178 + M)
    assert rel_err(y, ref) <= BF16_TOL


@pytest.mark.parametrize("M,swiglu", [(200, False), (300, True)])
def test_mxfp8_dequant_once_route(M, swiglu):
    """The tile path's other route (the weight converted to bf16 once per call),
    which NVFP4, partial and AdaLN outputs take, forced for a bf16 output."""
    fnb.fn_set_debug(fnb.FN_DEBUG_FORCE_PATH, 4)
    try:
        y, ref = _case(M, 512, 384, swiglu, seed=179)
    finally:
        fnb.fn_set_debug(fnb.FN_DEBUG_FORCE_PATH, 0)
    assert rel_err(y, ref) <= BF16_TOL


def test_mxfp8_promotion_repeated_calls_and_timeout():
    """320 tiles on the SMs: whole waves, then a tail split in k over CTA pairs
    whose halves are added in a fixed order, so repeated calls give the same
    bits.  A withheld scaler arrival (each CTA has several tiles, so its MMA
    issuer waits for the accumulator) times out cleanly: the status word
    reports it and the next call is correct."""
    M, d, N = 2048, 256, 2560
    inp = WL.case(M, d, N, True, seed=180)
    Wq, s = T.fold(gpu(inp["W_gate"]), gpu(inp["g"]), gpu(inp["W_up"]), wtype=MX)
    x = gpu(inp["x"])
    ws = T.Workspace()
    first = run(x, Wq, N, 1e-6, swiglu=True, scales=s, ws=ws).clone()
    Wg, Wu = O.deinterleave128(mx_ref(inp["W_gate"], inp["g"], inp["W_up"])[2])
    ref = O.norm_proj_swiglu(inp["x"], np.ones(d), Wg, Wu, 1e-6)
    assert rel_err(first, ref) <= BF16_TOL
    for _ in range(50):
        assert torch.equal(run(x, Wq, N, 1e-6, swiglu=True, scales=s, ws=ws), first)
    assert ws.status()[0] == fnb.FN_OK
    assert fnb.fn_set_debug(fnb.FN_DEBUG_WAIT_BUDGET_NS, 20_000_000) == fnb.FN_OK
    assert fnb.fn_set_debug(fnb.FN_DEBUG_WITHHOLD_ARRIVE, 1) == fnb.FN_OK
    try:
        T.norm_proj(x, Wq, N, 1e-6, swiglu=True, scales=s, ws=ws)
        st, word = ws.status()
    finally:
        fnb.fn_set_debug(fnb.FN_DEBUG_WITHHOLD_ARRIVE, 0)
        fnb.fn_set_debug(fnb.FN_DEBUG_WAIT_BUDGET_NS, 2_000_000_000)
    assert st == fnb.FN_ERR_TIMEOUT and (word >> 8) != 0
    ws.buf.zero_()
    assert torch.equal(run(x, Wq, N, 1e-6, swiglu=True, scales=s, ws=ws), first)
    assert ws.status()[0] == fnb.FN_OK


@pytest.mark.parametrize("M", [8, 100])
def test_mxfp8_row_parallel_shares(M):
    """Two ranks' shares of a row-parallel split (rows [0, d/2) and [d/2, d)
    of the weight; each rank's scale bytes are one contiguous range), summed
    and post-scaled, against the oracle of the whole projection."""
    d, N = 512, 384
    inp = WL.case(M, d, N, False, seed=176)
    Wq, s = T.fold(gpu(inp["W"]), gpu(inp["g"]), wtype=MX)
    half_sf = s.numel() // 2
    x = gpu(inp["x"])
    tot = None
    for r in range(2):
        xs = x[:, r * d // 2:(r + 1) * d // 2].contiguous()
        Ws = Wq[r * d // 2:(r + 1) * d // 2].contiguous()
        ss = s[r * half_sf:(r + 1) * half_sf].contiguous()
        part = T.norm_proj_partial(xs, Ws, N, scales=ss)
        tot = part.clone() if tot is None else tot + part
    y = T.post_scale(tot, M, N, d, inp["eps"])
    torch.cuda.synchronize()
    ref = O.norm_proj(inp["x"], np.ones(d), mx_ref(inp["W"], inp["g"])[2], inp["eps"])
    assert rel_err(y, ref) <= BF16_TOL


def test_mxfp8_timeout_is_reported():
    """A withheld arrival (the sums-of-squares warp never signals its first
    segment) makes the epilogue's bounded wait give up with FN_ERR_TIMEOUT."""
    M, d, N = 8, 512, 512
    inp = WL.case(M, d, N, False, seed=177)
    Wq, s = T.fold(gpu(inp["W"]), gpu(inp["g"]), wtype=MX)
    x = gpu(inp["x"])
    ws = T.Workspace()
    assert fnb.fn_set_debug(fnb.FN_DEBUG_WAIT_BUDGET_NS, 20_000_000) == fnb.FN_OK
    assert fnb.fn_set_debug(fnb.FN_DEBUG_WITHHOLD_ARRIVE, 1) == fnb.FN_OK
    try:
        T.norm_proj(x, Wq, N, 1e-6, scales=s, ws=ws)
        st, word = ws.status()
    finally:
        fnb.fn_set_debug(fnb.FN_DEBUG_WITHHOLD_ARRIVE, 0)
        fnb.fn_set_debug(fnb.FN_DEBUG_WAIT_BUDGET_NS, 2_000_000_000)
    assert st == fnb.FN_ERR_TIMEOUT and (word >> 8) != 0
    ws.buf.zero_()
    y = T.norm_proj(x, Wq, N, 1e-6, scales=s, ws=ws)
    torch.cuda.synchronize()
    assert ws.status()[0] == fnb.FN_OK
    ref = O.norm_proj(inp["x"], np.ones(d), mx_ref(inp["W"], inp["g"])[2], 1e-6)
    assert rel_err(y, ref) <= BF16_TOL


@pytest.fixture(scope="module")
def mx_workload():
    w = WL.WORKLOADS["fp8_swiglu"]
    inp = WL.workload_case("fp8_swiglu", 256)
    g = inp["g"]
    Wq, s = T.fold(gpu(inp["W_gate"]), gpu(g), gpu(inp["W_up"]), wtype=MX)
    Wg, Wu = O.deinterleave128(mx_ref(inp["W_gate"], g, inp["W_up"])[2])
    torch.cuda.synchronize()
    return w, inp, Wq, s, Wg, Wu


@pytest.mark.parametrize("M", [1, 64, 256])
def test_mxfp8_fp8_workload(mx_workload, M):
    """The fp8 SwiGLU workload's shape (d = 5120, 2 x 13824 columns) with the
    weight folded to MXFP8 instead of 128x128 fp32 block scales."""
    w, inp, Wq, s, Wg, Wu = mx_workload
    x = inp["x"][:M]
    y = run(gpu(x), Wq, w.N, inp["eps"], swiglu=True, scales=s)
    ref = O.norm_proj_swiglu(x, np.ones(w.d), Wg, Wu, inp["eps"])
    assert rel_err(y, ref) <= BF16_TOL
