"""GPU parity: the CUDA path against the fp64 oracle, through the C ABI.

Three levels, as the norm+projection's stored formats allow:
  fold parity   fn_fold_weights is bit-identical to the oracle's fold;
  kernel parity the fused kernels match the oracle evaluated on the stored
                folded weight (bf16 W', g = 1) within 1e-2 (1 + |y_ref|);
  end to end    plain projections also match the oracle with the original
                W and g (unfolded) within the same bound.
Large workloads are checked on a deterministic sample: two rows in every
128-row block plus the smallest- and largest-scale rows, against eight columns
in every 128-column output block, so every output tile is visited.
"""
import numpy as np
import pytest
import torch

import oracle as O
import rmsnorm_linear_projection_flashnorm_b200 as fnb
import workloads as WL
from rmsnorm_linear_projection_flashnorm_b200 import torch_api as T
from tests._util import BF16_TOL, fold_ref_bf16, gpu, rel_err, run, sample_cols

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    fnb.build()
    fnb.lib()
    torch.cuda.init()
    yield
    fnb.fn_set_debug(fnb.FN_DEBUG_FORCE_PATH, 0)


def _bits16(t):
    return t.detach().cpu().view(torch.int16).numpy().view(np.uint16)


# ---------------------------------------------------------------------------
# fold (Proposal 1), bit-exact
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("d,N,swiglu", [(256, 512, False), (512, 384, True), (4096, 6144, False)])
def test_fold_bf16_bit_exact(d, N, swiglu):
    inp = WL.case(4, d, N, swiglu, seed=31)
    g = inp["g"]
    if swiglu:
        Wg, Wu = inp["W_gate"], inp["W_up"]
        Wp, _ = T.fold(gpu(Wg), gpu(g), gpu(Wu))
        want = O.interleave128(O.fold_bf16(Wg, g), O.fold_bf16(Wu, g))
    else:
        Wp, _ = T.fold(gpu(inp["W"]), gpu(g))
        want = O.fold_bf16(inp["W"], g)
    torch.cuda.synchronize()
    assert np.array_equal(_bits16(Wp), want)


def test_fold_bf16_general_gain_rounds_once_per_step():
    """A gain that is not bf16-representable: fp32 product rounds, then bf16."""
    inp = WL.case(4, 256, 256, False, seed=32)
    g = torch.linspace(0.31, 1.73, 256, dtype=torch.float32)
    Wp, _ = T.fold(gpu(inp["W"]), gpu(g))
    torch.cuda.synchronize()
    assert np.array_equal(_bits16(Wp), O.fold_bf16(inp["W"], g))


@pytest.mark.parametrize("d,N,swiglu", [(256, 384, False), (384, 256, True)])
def test_fold_fp8_bit_exact(d, N, swiglu):
    inp = WL.case(4, d, N, swiglu, seed=33)
    g = inp["g"]
    if swiglu:
        Wg, Wu = inp["W_gate"], inp["W_up"]
        Wq, s = T.fold(gpu(Wg), gpu(g), gpu(Wu), wtype=fnb.FN_W_FP8_E4M3_B128)
        qg, sg = O.fold_fp8(Wg, g)
        qu, su = O.fold_fp8(Wu, g)
        want_q = O.interleave128(qg, qu)
        want_s = np.empty((d // 128, 2 * N // 128), dtype=np.float32)
        want_s[:, 0::2], want_s[:, 1::2] = sg, su
    else:
        Wq, s = T.fold(gpu(inp["W"]), gpu(g), wtype=fnb.FN_W_FP8_E4M3_B128)
        want_q, want_s = O.fold_fp8(inp["W"], g)
    torch.cuda.synchronize()
    assert np.array_equal(Wq.cpu().numpy(), want_q)
    assert np.array_equal(s.cpu().numpy().view(np.uint32), want_s.view(np.uint32))


# ---------------------------------------------------------------------------
# fused norm + projection
# ---------------------------------------------------------------------------
def _plain_case(M, d, N, seed, eps=1e-6, zero_rows=()):
    inp = WL.case(M, d, N, False, seed=seed, zero_rows=zero_rows)
    x, g, W = inp["x"], inp["g"], inp["W"]
    Wp, _ = T.fold(gpu(W), gpu(g))
    y = run(gpu(x), Wp, N, eps)
    ref_c2 = O.norm_proj(x, np.ones(d), fold_ref_bf16(W, g), eps)
    return y, ref_c2, inp


def _swiglu_case(M, d, N, seed, eps=1e-6):
    inp = WL.case(M, d, N, True, seed=seed)
    x, g, Wg, Wu = inp["x"], inp["g"], inp["W_gate"], inp["W_up"]
    Wp, _ = T.fold(gpu(Wg), gpu(g), gpu(Wu))
    y = run(gpu(x), Wp, N, eps, swiglu=True)
    ref = O.norm_proj_swiglu(x, np.ones(d), fold_ref_bf16(Wg, g), fold_ref_bf16(Wu, g), eps)
    return y, ref, inp


def test_tiny_workload():
    w = WL.WORKLOADS["tiny"]
    inp = WL.workload_case("tiny")
    x, g, W = inp["x"], inp["g"], inp["W"]
    Wp, _ = T.fold(gpu(W), gpu(g))
    y = run(gpu(x), Wp, w.N, inp["eps"])
    assert rel_err(y, O.norm_proj(x, np.ones(w.d), fold_ref_bf16(W, g), inp["eps"])) <= BF16_TOL
    assert rel_err(y, O.norm_proj(x, g, W, inp["eps"])) <= BF16_TOL     # end to end


@pytest.mark.parametrize("M", [1, 8, 32, 64])
def test_decode_qkv_workload(M):
    w = WL.WORKLOADS["decode_qkv"]
    inp = WL.workload_case("decode_qkv", M)
    x, g, W = inp["x"], inp["g"], inp["W"]
    Wp, _ = T.fold(gpu(W), gpu(g))
    y = run(gpu(x), Wp, w.N, inp["eps"])
    assert rel_err(y, O.norm_proj(x, np.ones(w.d), fold_ref_bf16(W, g), inp["eps"])) <= BF16_TOL
    assert rel_err(y, O.norm_proj(x, g, W, inp["eps"])) <= BF16_TOL     # end to end


@pytest.mark.parametrize("M", [1, 2, 7, 15, 16, 17, 31, 33, 48, 63, 64])
def test_decode_m_ladder(M):
    y, ref, _ = _plain_case(M, 512, 384, seed=40 + M)
    assert rel_err(y, ref) <= BF16_TOL


@pytest.mark.parametrize("M,d,N", [(65, 256, 256), (300, 512, 768), (128, 64, 128), (1000, 320, 640)])
def test_tile_path_plain_ragged(M, d, N):
    y, ref, _ = _plain_case(M, d, N, seed=50)
    assert rel_err(y, ref) <= BF16_TOL


@pytest.mark.parametrize("M,d,N", [(5, 384, 384), (16, 256, 128), (64, 640, 512), (200, 384, 384),
                                   (129, 256, 640)])
def test_swiglu_small(M, d, N):
    y, ref, _ = _swiglu_case(M, d, N, seed=60)
    assert rel_err(y, ref) <= BF16_TOL


@pytest.mark.parametrize("path", [1, 2])
def test_both_paths_agree_with_oracle_at_small_m(path):
    fnb.fn_set_debug(fnb.FN_DEBUG_FORCE_PATH, path)
    try:
        for M in (1, 9, 40):
            y, ref, _ = _plain_case(M, 512, 256, seed=70)
            assert rel_err(y, ref) <= BF16_TOL
            y, ref, _ = _swiglu_case(M, 256, 256, seed=71)
            assert rel_err(y, ref) <= BF16_TOL
    finally:
        fnb.fn_set_debug(fnb.FN_DEBUG_FORCE_PATH, 0)


def test_single_k_block_and_single_tile():
    y, ref, _ = _plain_case(3, 64, 128, seed=80)
    assert rel_err(y, ref) <= BF16_TOL
    y, ref, _ = _plain_case(130, 64, 128, seed=81)
    assert rel_err(y, ref) <= BF16_TOL


@pytest.mark.parametrize("M", [4, 200])
def test_zero_rows(M):
    zero = (0, M - 1)
    y, ref, _ = _plain_case(M, 256, 256, seed=90, eps=1e-6, zero_rows=zero)
    assert torch.all(y[list(zero)] == 0)
    assert rel_err(y, ref) <= BF16_TOL
    y, ref, _ = _plain_case(M, 256, 256, seed=90, eps=0.0, zero_rows=zero)
    assert torch.all(torch.isnan(y[list(zero)].float()))
    assert rel_err(y, ref) <= BF16_TOL        # NaN positions coincide, others within bound


def test_empty_batch_launches_nothing():
    ws = T.Workspace()
    st = fnb.fn_norm_proj(0, 0, 256, 0, None, fnb.FN_W_BF16, 256, 1e-6, 0, ws.buf, ws.buf.numel(), None)
    assert st == fnb.FN_OK


def test_ffn_swiglu_decode_workload():
    w = WL.WORKLOADS["ffn_swiglu"]
    y, ref, _ = _swiglu_case(16, w.d, w.N, seed=w.seed)
    assert rel_err(y, ref) <= BF16_TOL


def _sampled_swiglu_workload(name, M):
    w = WL.WORKLOADS[name]
    inp = WL.workload_case(name, M)
    x, g, Wg, Wu = inp["x"], inp["g"], inp["W_gate"], inp["W_up"]
    Wp, _ = T.fold(gpu(Wg), gpu(g), gpu(Wu))
    y = run(gpu(x), Wp, w.N, inp["eps"], swiglu=True)
    rows = WL.sample_rows(M, w.seed)
    cols = sample_cols(w.N, w.seed)
    ref = O.norm_proj_swiglu(x[rows], np.ones(w.d), fold_ref_bf16(Wg[:, cols], g),
                             fold_ref_bf16(Wu[:, cols], g), inp["eps"])
    got = y.cpu()[rows][:, cols]
    return got, ref


def test_ffn_swiglu_prefill_workload_sampled():
    got, ref = _sampled_swiglu_workload("ffn_swiglu", 4096)
    assert rel_err(got, ref) <= BF16_TOL


@pytest.mark.slow
def test_large_prefill_workload_sampled():
    got, ref = _sampled_swiglu_workload("prefill_swiglu_large", 16384)
    assert rel_err(got, ref) <= BF16_TOL


def test_repeated_calls_bit_identical():
    inp = WL.case(32, 1024, 768, False, seed=95)
    Wp, _ = T.fold(gpu(inp["W"]), gpu(inp["g"]))
    x = gpu(inp["x"])
    ws = T.Workspace()
    first = run(x, Wp, 768, 1e-6, ws=ws).clone()
    for _ in range(50):
        assert torch.equal(run(x, Wp, 768, 1e-6, ws=ws), first)
    assert ws.status()[0] == fnb.FN_OK


@pytest.mark.parametrize("cluster", [0, 1])
@pytest.mark.parametrize("M,d,N,swiglu", [(1, 4096, 6144, False), (40, 4096, 6144, False), (8, 1024, 1024, True),
                                          (64, 640, 1280, True), (17, 2048, 256, False)])
def test_decode_cluster_and_stream_k_agree_with_oracle(cluster, M, d, N, swiglu):
    """The decode path either splits K inside thread-block clusters (reduced over
    distributed shared memory) or uses stream-K with the fix-up kernel; both
    must match the oracle."""
    fnb.fn_set_debug(fnb.FN_DEBUG_CLUSTER, cluster)
    try:
        if swiglu:
            y, ref, _ = _swiglu_case(M, d, N, seed=97)
        else:
            y, ref, _ = _plain_case(M, d, N, seed=97)
        assert rel_err(y, ref) <= BF16_TOL
    finally:
        fnb.fn_set_debug(fnb.FN_DEBUG_CLUSTER, 1)


@pytest.mark.parametrize("M", [3, 200])
def test_non_finite_rows_give_nan_rows(M):
    """An inf or NaN in a row makes that row's outputs NaN (its sum of squares
    is not finite), as in the oracle; the other rows are unaffected."""
    d, N = 256, 256
    x = WL.activations(M, d, 96).clone()
    x[1, 7] = float("inf")
    x[2, 200] = float("nan")
    inp = WL.case(M, d, N, False, seed=96)
    Wp, _ = T.fold(gpu(inp["W"]), gpu(inp["g"]))
    y = run(gpu(x), Wp, N, 1e-6)
    ref = O.norm_proj(x, np.ones(d), fold_ref_bf16(inp["W"], inp["g"]), 1e-6)
    assert torch.all(torch.isnan(y[1:3].float()))
    assert rel_err(y, ref) <= BF16_TOL


@pytest.mark.parametrize("M,swiglu", [(1, False), (48, True), (130, False)])
def test_long_k(M, swiglu):
    """d = 16384: 256 k blocks per column tile, so stream-K ranges span many
    blocks and the tile kernel runs a long main loop."""
    d, N = 16384, 256
    if swiglu:
        y, ref, _ = _swiglu_case(M, d, N, seed=94)
    else:
        y, ref, _ = _plain_case(M, d, N, seed=94)
    assert rel_err(y, ref) <= BF16_TOL
