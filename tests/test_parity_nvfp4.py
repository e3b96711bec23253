"""GPU parity of the quantising SwiGLU epilogue (NVFP4 output) against the
fp64 oracle, through the C ABI.

The kernels encode their fp32 SwiGLU value; the oracle encodes its fp64
value.  A code is a decision taken on that value, so the check (see
tests/_util.check_nvfp4) accepts every code a value within the kernel
tolerance could give, requires nearly all codes to equal the oracle's own
encoding, and checks the non-finite blocks exactly.  Cases cover the decode
kernel (bf16 and fp8 weights, whole tiles and tiles finished by the fix-up
kernel), the tile kernel (bf16, fp8 converted per tile and fp8 dequantised
once), ragged M, several global scales (including saturation and subnormal
scales), NaN rows and repeated calls.
"""
import numpy as np
import pytest
import torch

import oracle as O
import rmsnorm_linear_projection_flashnorm_b200 as fnb
import workloads as WL
from rmsnorm_linear_projection_flashnorm_b200 import torch_api as T
from tests._util import BF16_TOL, FP8_TOL, check_nvfp4, fold_fp8_ref, fold_ref_bf16, gpu

pytestmark = pytest.mark.gpu
FP8 = fnb.FN_W_FP8_E4M3_B128


@pytest.fixture(scope="module", autouse=True)
def _lib():
    fnb.build()
    fnb.lib()
    torch.cuda.init()
    yield
    fnb.fn_set_debug(fnb.FN_DEBUG_FORCE_PATH, 0)


def _prepare(M, d, N, wt, seed, x=None, eps=None):
    inp = WL.case(M, d, N, True, seed=seed)
    if x is not None:
        inp["x"] = x
    if eps is not None:
        inp["eps"] = eps
    g = inp["g"]
    if wt == FP8:
        Wq, s = T.fold(gpu(inp["W_gate"]), gpu(g), gpu(inp["W_up"]), wtype=FP8)
        q, sr = fold_fp8_ref(inp["W_gate"], g, inp["W_up"])
        Wg, Wu = O.deinterleave128(O.dequant_fp8(q, sr))
    else:
        Wq, _ = T.fold(gpu(inp["W_gate"]), gpu(g), gpu(inp["W_up"]))
        s = None
        Wg, Wu = fold_ref_bf16(inp["W_gate"], g), fold_ref_bf16(inp["W_up"], g)
    ref = O.norm_proj_swiglu(inp["x"], np.ones(d), Wg, Wu, inp["eps"])
    return inp, Wq, s, ref


def _run_nvfp4(inp, Wq, s, N, gs, ws=None):
    gsd = torch.tensor([gs], dtype=torch.float32, device="cuda")
    q, sf = T.norm_proj_swiglu_nvfp4(gpu(inp["x"]), Wq, N, inp["eps"], gsd, scales=s, ws=ws)
    torch.cuda.synchronize()
    return q.cpu().numpy(), sf.cpu().numpy()


def _gs_for(ref):
    """The usual choice: the tensor maximum maps to the largest scale x value."""
    amax = np.max(np.abs(ref[np.isfinite(ref)]))
    return float(np.float32(448.0 * 6.0 / amax))


@pytest.mark.parametrize("M,d,N,wt", [
    (1, 512, 256, 0),        # decode: every tile split, finished by the fix-up kernel
    (5, 256, 19200, 0),      # decode: 150 tiles on 148 SMs, whole tiles in the decode kernel
    (33, 384, 640, 0),
    (64, 256, 19200, 0),
    (65, 256, 512, 0),       # tile kernel
    (200, 512, 384, 0),      # tile kernel, ragged M
    (3, 256, 19200, FP8),    # fp8 decode, whole tiles
    (40, 384, 256, FP8),     # fp8 decode with the activations split once per call, fix-up
    (64, 512, 640, FP8),
    (130, 256, 384, FP8),    # fp8 tile kernel (per-tile conversion)
    (1100, 256, 256, FP8),   # fp8, weight dequantised once into the workspace
])
def test_nvfp4_small(M, d, N, wt):
    inp, Wq, s, ref = _prepare(M, d, N, wt, seed=401)
    gs = _gs_for(ref)
    q, sf = _run_nvfp4(inp, Wq, s, N, gs)
    check_nvfp4(q, sf, ref, gs, FP8_TOL if wt == FP8 else BF16_TOL)


@pytest.mark.parametrize("gs", [1.0, 1e6, 1e-3])
@pytest.mark.parametrize("M", [4, 96])
def test_nvfp4_global_scales(M, gs):
    """gs = 1 gives scales near one, 1e6 saturates every scale at 448 and the
    large elements at +-6, 1e-3 puts the scales in e4m3's subnormal range
    (the smallest round to zero)."""
    inp, Wq, s, ref = _prepare(M, 256, 512, 0, seed=402)
    q, sf = _run_nvfp4(inp, Wq, s, 512, gs)
    check_nvfp4(q, sf, ref, gs, BF16_TOL)
    if gs == 1e6:
        assert np.all(sf == 0x7E)


@pytest.mark.parametrize("M,wt", [(6, 0), (70, 0), (6, FP8), (70, FP8)])
def test_nvfp4_nan_rows(M, wt):
    """A zero row with eps = 0 has no finite 1/rms: its blocks carry the NaN
    scale code and zero codes; the other rows are unaffected."""
    inp = WL.case(M, 256, 256, True, seed=403)
    x = inp["x"].clone()
    x[1] = 0
    x[M - 1] = 0
    inp, Wq, s, ref = _prepare(M, 256, 256, wt, seed=403, x=x, eps=0.0)
    assert np.all(np.isnan(ref[1])) and np.all(np.isfinite(ref[0]))
    gs = _gs_for(ref)
    q, sf = _run_nvfp4(inp, Wq, s, 256, gs)
    check_nvfp4(q, sf, ref, gs, FP8_TOL if wt == FP8 else BF16_TOL)
    assert np.all(sf[1] == 0x7F) and np.all(sf[0] != 0x7F)


def test_nvfp4_ffn_decode_workload():
    w = WL.WORKLOADS["ffn_swiglu"]
    inp, Wq, s, ref = _prepare(16, w.d, w.N, 0, seed=w.seed)
    gs = _gs_for(ref)
    q, sf = _run_nvfp4(inp, Wq, s, w.N, gs)
    frac = check_nvfp4(q, sf, ref, gs, BF16_TOL)
    assert frac > 0.99


@pytest.mark.parametrize("M,wt", [(16, 0), (300, 0), (48, FP8)])
def test_nvfp4_repeated_calls_bit_identical(M, wt):
    inp, Wq, s, ref = _prepare(M, 512, 1024, wt, seed=404)
    ws = T.Workspace()
    gs = _gs_for(ref)
    q0, sf0 = _run_nvfp4(inp, Wq, s, 1024, gs, ws=ws)
    for _ in range(20):
        q1, sf1 = _run_nvfp4(inp, Wq, s, 1024, gs, ws=ws)
        assert np.array_equal(q0, q1) and np.array_equal(sf0, sf1)
    assert ws.status()[0] == fnb.FN_OK


def _sample_blocks(N: int, seed: int) -> np.ndarray:
    """One whole 16-column block in every 128-column output tile."""
    rng = np.random.default_rng(30_000 + seed)
    return np.array([t * 8 + int(rng.integers(0, 8)) for t in range(N // 128)], dtype=np.int64)


def _check_sampled(q, sf, rows, blocks, ref, gs, tol):
    cols = (blocks[:, None] * 16 + np.arange(16)[None, :]).reshape(-1)
    codes = O.nvfp4_unpack(q[rows])[:, cols]
    return check_nvfp4(O.nvfp4_pack(codes), sf[rows][:, blocks], ref, gs, tol)


def test_nvfp4_ffn_prefill_workload_sampled():
    """FFN SwiGLU at M = 4096 (tile kernel) on the full workload, checked on
    the deterministic row sample and one whole scale block per output tile."""
    w = WL.WORKLOADS["ffn_swiglu"]
    M = 4096
    inp = WL.workload_case("ffn_swiglu", M)
    x, g, Wg, Wu = inp["x"], inp["g"], inp["W_gate"], inp["W_up"]
    Wp, _ = T.fold(gpu(Wg), gpu(g), gpu(Wu))
    rows = WL.sample_rows(M, w.seed)
    blocks = _sample_blocks(w.N, w.seed)
    cols = (blocks[:, None] * 16 + np.arange(16)[None, :]).reshape(-1)
    ref = O.norm_proj_swiglu(x[rows], np.ones(w.d), fold_ref_bf16(Wg[:, cols], g), fold_ref_bf16(Wu[:, cols], g),
                             inp["eps"])
    gs = _gs_for(ref)
    q, sf = _run_nvfp4(inp, Wp, None, w.N, gs)
    assert _check_sampled(q, sf, rows, blocks, ref, gs, BF16_TOL) > 0.99


@pytest.fixture(scope="module")
def fp8_workload():
    w = WL.WORKLOADS["fp8_swiglu"]
    inp = WL.workload_case("fp8_swiglu", 256)
    g = inp["g"]
    Wq, s = T.fold(gpu(inp["W_gate"]), gpu(g), gpu(inp["W_up"]), wtype=FP8)
    q, sr = fold_fp8_ref(inp["W_gate"], g, inp["W_up"])
    Wg, Wu = O.deinterleave128(O.dequant_fp8(q, sr))
    torch.cuda.synchronize()
    return w, inp, Wq, s, Wg, Wu


@pytest.mark.parametrize("M", [1, 64, 256])
def test_nvfp4_fp8_workload(fp8_workload, M):
    """The fp8 SwiGLU workload (d = 5120, N = 13824): decode kernel with the
    in-kernel and the once-per-call activation split, and the tile kernel."""
    w, inp, Wq, s, Wg, Wu = fp8_workload
    x = inp["x"][:M]
    ref = O.norm_proj_swiglu(x, np.ones(w.d), Wg, Wu, inp["eps"])
    gs = _gs_for(ref)
    q, sf = _run_nvfp4({"x": x, "eps": inp["eps"]}, Wq, s, w.N, gs)
    assert check_nvfp4(q, sf, ref, gs, FP8_TOL) > 0.99


@pytest.mark.parametrize("M,d,N,wt", [
    (1, 512, 256, 0),        # decode, fix-up kernel writes the scales
    (5, 256, 19200, 0),      # decode, whole tiles staged and stored by the decode kernel
    (200, 512, 384, 0),      # tile kernel, ragged M (padding rows of the last 128-row block)
    (40, 384, 256, FP8),     # fp8 decode
    (130, 256, 384, FP8),    # fp8 tile kernel
    (300, 256, 512, 2),      # MXFP8 weights (tile path after the exact bf16 conversion)
    (17, 256, 512, 2),       # MXFP8 decode
])
def test_nvfp4_swizzled_scales(M, d, N, wt):
    """The swizzled entry point writes the same codes as the row-major one and
    its scale bytes are exactly the row-major bytes in the oracle's chunked
    layout (sf_chunk_layout, pinned on CPU); the row-major result itself is
    checked against the oracle's encoding."""
    inp = WL.case(M, d, N, True, seed=190 + M)
    g = inp["g"]
    Wq, s = T.fold(gpu(inp["W_gate"]), gpu(g), gpu(inp["W_up"]), wtype=wt)
    gsd = torch.tensor([448.0 * 6.0 / 6.0], dtype=torch.float32, device="cuda")
    x = gpu(inp["x"])
    q0, sf0 = T.norm_proj_swiglu_nvfp4(x, Wq, N, inp["eps"], gsd, scales=s)
    q1, sf1 = T.norm_proj_swiglu_nvfp4_swizzled(x, Wq, N, inp["eps"], gsd, scales=s)
    torch.cuda.synchronize()
    assert torch.equal(q0, q1)
    sf_rm = sf0.cpu().numpy()
    assert np.array_equal(sf1.cpu().numpy(), O.sf_chunk_layout(sf_rm))
    assert np.array_equal(O.sf_chunk_unlayout(sf1.cpu().numpy(), M, N // 16), sf_rm)
    if wt == 0:
        Wg, Wu = fold_ref_bf16(inp["W_gate"], g), fold_ref_bf16(inp["W_up"], g)
        ref = O.norm_proj_swiglu(inp["x"], np.ones(d), Wg, Wu, inp["eps"])
        check_nvfp4(q0.cpu().numpy(), sf_rm, ref, float(gsd.item()), BF16_TOL)
