"""GPU parity with fp8 (e4m3, 128x128 block-scaled) folded weights.

The activations stay bf16.  At M > 64 the kernels convert each staged e4m3
weight tile to bf16 on chip (fp32 product with the block scale, one rounding)
and run the bf16 MMA (at M >= 1024 after one dequantisation into the
workspace); at M <= 64 the e4m3 codes go to the tensor cores as they are and
the activations are split exactly into two e4m3 parts per 128-deep k block.

Each path is held to the bf16-weight bound, 1e-2 (1 + |y_ref|), against the
oracle evaluated on the weight that path multiplies (g = 1): bf16(e4m3(q) * s)
for the tile paths, the exact e4m3(q) * s for the decode paths; after that
step both paths only accumulate in fp32 and round the output once.  Every
case is also held to the format's bound, 6e-2 (1 + |y_ref|), against the exact
dequantised weight.  The oracle's own fold and dequantisation give both
weights; the GPU folds the same weights itself, and the fold's and the
dequantisation step's bit-exactness are separate tests.
"""
import numpy as np
import pytest
import torch

import oracle as O
import rmsnorm_linear_projection_flashnorm_b200 as fnb
import workloads as WL
from rmsnorm_linear_projection_flashnorm_b200 import torch_api as T
from tests._util import BF16_TOL, FP8_TOL, fold_fp8_ref, gpu, rel_err, run, sample_cols

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


def _tile_path(M, force=0):
    """True where the e4m3 weight reaches the tensor cores as bf16(q * s): the
    tile kernel's converter warps and the dequantise-once route, which the
    library takes for fp8 weights only when forced (FN_DEBUG_FORCE_PATH = 4)
    or for NVFP4, partial and AdaLN outputs.  The decode kernels (M <= 64) and
    the block-scale promotion kernel (M > 64) multiply the e4m3 codes exactly
    and apply s to fp32 sums."""
    return force == 4


def _stored_weight(q, sr, tile):
    """The weight each path multiplies: the exact q * s for the decode and
    promotion kernels, its one bf16 rounding for the converting paths (the
    oracle's own rounding)."""
    if tile:
        return O.bf16_from_bits(O.dequant_fp8_bf16_bits(q, sr))
    return O.dequant_fp8(q, sr)


def _case(M, d, N, swiglu, seed, x=None, force=0):
    """Kernel output and two references: the oracle on the weight this path
    stores (the bf16-weight bound applies, since everything after that is fp32
    accumulation and one output rounding) and the oracle on the exact dequant
    q * s (the format's own bound)."""
    inp = WL.case(M, d, N, swiglu, seed=seed)
    if x is not None:
        inp["x"] = x
    x, g = inp["x"], inp["g"]
    tile = _tile_path(M, force)
    if swiglu:
        Wq, s = T.fold(gpu(inp["W_gate"]), gpu(g), gpu(inp["W_up"]), wtype=FP8)
        q, sr = fold_fp8_ref(inp["W_gate"], g, inp["W_up"])
        refs = []
        for w in (_stored_weight(q, sr, tile), O.dequant_fp8(q, sr)):
            Wg, Wu = O.deinterleave128(w)
            refs.append(O.norm_proj_swiglu(x, np.ones(d), Wg, Wu, inp["eps"]))
    else:
        Wq, s = T.fold(gpu(inp["W"]), gpu(g), wtype=FP8)
        q, sr = fold_fp8_ref(inp["W"], g)
        refs = [O.norm_proj(x, np.ones(d), w, inp["eps"])
                for w in (_stored_weight(q, sr, tile), O.dequant_fp8(q, sr))]
    y = run(gpu(x), Wq, N, inp["eps"], swiglu=swiglu, scales=s)
    return y, refs[0], refs[1]


def _check(y, ref_stored, ref_exact):
    assert rel_err(y, ref_stored) <= BF16_TOL
    assert rel_err(y, ref_exact) <= FP8_TOL


@pytest.mark.parametrize("M,d,N,swiglu", [
    (5, 256, 384, False),      # decode, odd number of 128-column blocks
    (200, 256, 384, False),    # tile path: the last 256-column tile is half past the weight
    (40, 384, 256, True),      # SwiGLU at 40 rows: the promotion kernel (33..64 rows)
    (300, 512, 384, True),     # tile SwiGLU, ragged M
    (64, 128, 128, False),     # single k block, single tile
    (129, 640, 640, True),
    (1100, 256, 256, True),    # M >= 1024: the weight is dequantised once into the workspace
    (1024, 384, 384, False),
])
def test_fp8_small(M, d, N, swiglu):
    _check(*_case(M, d, N, swiglu, seed=131))


@pytest.mark.parametrize("path", [1, 2])
def test_fp8_both_paths_at_small_m(path):
    fnb.fn_set_debug(fnb.FN_DEBUG_FORCE_PATH, path)
    try:
        for M, sw in ((3, False), (33, True)):
            _check(*_case(M, 256, 256, sw, seed=132, force=path))
    finally:
        fnb.fn_set_debug(fnb.FN_DEBUG_FORCE_PATH, 0)


@pytest.mark.parametrize("M,d,N,swiglu", [
    (65, 256, 384, False),     # smallest tile-path M; 3 column blocks: the last tile's second half is past N
    (200, 1024, 512, True),
    (333, 4096, 256, False),   # long k range, ragged rows
    (130, 512, 1280, True),
    (256, 256, 9472, True),    # 148 tiles: one whole wave, no split tail
    (128, 256, 12800, True),   # 100 tiles: a last wave too full to split in k
])
def test_fp8_promotion_kernel(M, d, N, swiglu):
    """The block-scale promotion kernel (x split once into exact e4m3 parts,
    each 128-deep k block's exact sums scaled and added in fp32) is held to the
    bf16-weight bound against the exact dequantised weight.  On 148 SMs the
    first four shapes end in a last wave of at most 74 tiles, which CTA pairs
    split in k and reduce over distributed shared memory; the last two do not."""
    y, ref, ref_exact = _case(M, d, N, swiglu, seed=160 + M)
    assert rel_err(y, ref_exact) <= BF16_TOL
    _check(y, ref, ref_exact)


@pytest.mark.parametrize("M,d,N,swiglu", [(200, 256, 384, False), (300, 512, 384, True), (1100, 256, 256, True)])
def test_fp8_converting_routes(M, d, N, swiglu):
    """The routes that convert the weight to bf16 (on chip per tile below 1024
    rows, once per call into the workspace from 1024), which NVFP4, partial and
    AdaLN outputs use, forced here for bf16 output."""
    fnb.fn_set_debug(fnb.FN_DEBUG_FORCE_PATH, 4)
    try:
        _check(*_case(M, d, N, swiglu, seed=170 + M, force=4))
    finally:
        fnb.fn_set_debug(fnb.FN_DEBUG_FORCE_PATH, 0)


def test_fp8_promotion_wide_dynamic_range_is_exact():
    """Activations spanning 2^-18 .. 2^10 inside one k block still meet the
    bf16-weight bound: the split of each (row, k block) is exact above 2^-9 of
    the block's largest magnitude."""
    M, d, N = 100, 512, 384
    x = WL.activations(M, d, 161).float()
    mult = torch.ones(d)
    mult[0::4] = 2.0 ** 10
    mult[1::8] = 2.0 ** -12
    mult[3::16] = 2.0 ** -18
    x = (x * mult).to(torch.bfloat16)
    for swiglu in (False, True):
        y, ref, _ = _case(M, d, N, swiglu, seed=161, x=x)
        assert rel_err(y, ref) <= BF16_TOL


def test_fp8_promotion_repeated_calls_and_timeout():
    """Bit-identical repeats, and a withheld scaler arrival times out cleanly:
    the status word reports it and the next call is correct."""
    M, d, N = 300, 1024, 512
    inp = WL.case(M, d, N, True, seed=162)
    Wq, s = T.fold(gpu(inp["W_gate"]), gpu(inp["g"]), gpu(inp["W_up"]), wtype=FP8)
    x = gpu(inp["x"])
    ws = T.Workspace()
    first = run(x, Wq, N, 1e-6, swiglu=True, scales=s, ws=ws).clone()
    for _ in range(100):
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


@pytest.mark.parametrize("M", [1, 2, 15, 16, 17, 31, 32, 33, 63, 64])
@pytest.mark.parametrize("swiglu", [False, True])
def test_fp8_decode_m_ladder(M, swiglu):
    """Every padded row count of the decode kernel (16, 32, 64 rows) and both
    scaler layouts (all rows per thread, or half of them)."""
    _check(*_case(M, 512, 768 if not swiglu else 384, swiglu, seed=140 + M))


def test_fp8_decode_wide_dynamic_range_is_exact():
    """Per row and 128-deep k block the decode kernel scales x by a power of
    two and splits it into two e4m3 parts whose sum is the bf16 value; the
    products with the e4m3 weight are then exact, so even activations that
    span 2^-20 .. 2^12 inside one k block meet the bf16-weight bound."""
    M, d, N = 6, 512, 384
    x = WL.activations(M, d, 150).float()
    mult = torch.ones(d)
    mult[0::4] = 2.0 ** 10
    mult[1::8] = 2.0 ** -12
    mult[3::16] = 2.0 ** -18
    x = (x * mult).to(torch.bfloat16)
    for swiglu in (False, True):
        y, ref, _ = _case(M, d, N, swiglu, seed=150, x=x)
        assert rel_err(y, ref) <= BF16_TOL


@pytest.mark.parametrize("M", [3, 200])
def test_fp8_non_finite_rows_give_nan_rows(M):
    """An inf or NaN in a row makes that row's outputs NaN (its sum of squares
    is not finite), as in the oracle; the other rows are unaffected."""
    d, N = 256, 256
    x = WL.activations(M, d, 151).clone()
    x[1, 7] = float("inf")
    x[2, 200] = float("nan")
    y, ref, ref_exact = _case(M, d, N, False, seed=151, x=x)
    assert torch.all(torch.isnan(y[1:3].float()))
    _check(y, ref, ref_exact)      # NaN positions coincide, the rest within bound


@pytest.mark.parametrize("M,swiglu", [(1, True), (40, False), (64, True)])
def test_fp8_decode_repeated_calls_bit_identical(M, swiglu):
    d, N = 1024, 1024
    inp = WL.case(M, d, N, swiglu, seed=152)
    if swiglu:
        Wq, s = T.fold(gpu(inp["W_gate"]), gpu(inp["g"]), gpu(inp["W_up"]), wtype=FP8)
    else:
        Wq, s = T.fold(gpu(inp["W"]), gpu(inp["g"]), wtype=FP8)
    x = gpu(inp["x"])
    ws = T.Workspace()
    first = run(x, Wq, N, 1e-6, swiglu=swiglu, scales=s, ws=ws).clone()
    for _ in range(200):
        assert torch.equal(run(x, Wq, N, 1e-6, swiglu=swiglu, scales=s, ws=ws), first)
    assert ws.status()[0] == fnb.FN_OK


@pytest.fixture(scope="module")
def fp8_workload():
    w = WL.WORKLOADS["fp8_swiglu"]
    inp = WL.workload_case("fp8_swiglu", max(w.Ms))
    g = inp["g"]
    Wq, s = T.fold(gpu(inp["W_gate"]), gpu(g), gpu(inp["W_up"]), wtype=FP8)
    q, sr = fold_fp8_ref(inp["W_gate"], g, inp["W_up"])
    exact = O.deinterleave128(O.dequant_fp8(q, sr))
    stored = O.deinterleave128(_stored_weight(q, sr, True))
    torch.cuda.synchronize()
    return w, inp, Wq, s, exact, stored


def _workload_refs(x, w, inp, exact, stored, M):
    """(reference on the weight this M's path multiplies, reference on q * s)."""
    mine = stored if _tile_path(M) else exact
    return tuple(O.norm_proj_swiglu(x, np.ones(w.d), Wg, Wu, inp["eps"]) for Wg, Wu in (mine, exact))


@pytest.mark.parametrize("M", [1, 64, 256])
def test_fp8_workload(fp8_workload, M):
    w, inp, Wq, s, exact, stored = fp8_workload
    x = inp["x"][:M]
    y = run(gpu(x), Wq, w.N, inp["eps"], swiglu=True, scales=s)
    _check(y, *_workload_refs(x, w, inp, exact, stored, M))


@pytest.mark.slow
def test_fp8_workload_prefill_sampled(fp8_workload):
    w, inp, Wq, s, exact, stored = fp8_workload
    M = max(w.Ms)
    y = run(gpu(inp["x"]), Wq, w.N, inp["eps"], swiglu=True, scales=s)
    rows = WL.sample_rows(M, w.seed)
    _check(y.cpu()[rows], *_workload_refs(inp["x"][rows], w, inp, exact, stored, M))
