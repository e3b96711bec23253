"""Pins for the fp64 oracle, run on the CPU.

Each check ties the oracle to something other than itself: the number
formats' definitions (hand-derived golden points), torch's own casts and
norm routine, explicit-loop brute force with math.fsum, closed forms, and
the identities the FlashNorm talk relies on (Proposal 1: folding the gain is
exact in real arithmetic; Proposal 3: RMSNorm is scale invariant).  The
planted-mistake tests at the end show that the pins catch a dropped or
misplaced term, a wrong divisor, a transposed operand and a swapped half.
"""
import math
import os

import numpy as np
import pytest
import torch

import oracle as O
from tests._golden import read_golden
import workloads as WL


# ---------------------------------------------------------------------------
# number formats
# ---------------------------------------------------------------------------


def test_e4m3_golden_points(golden_dir):
    rows = read_golden(os.path.join(golden_dir, "e4m3_points.txt"))
    vals = np.array([v for v, _ in rows])
    want = np.array([c for _, c in rows], dtype=np.uint8)
    got = O.e4m3_encode(vals)
    assert np.array_equal(got, want), list(zip(vals, got, want))


def test_bf16_golden_points(golden_dir):
    rows = read_golden(os.path.join(golden_dir, "bf16_points.txt"))
    vals = np.array([v for v, _ in rows])
    want = np.array([c for _, c in rows], dtype=np.uint16)
    got = O.bf16_bits(vals)
    assert np.array_equal(got, want), [(v, hex(g), hex(w)) for v, g, w in zip(vals, got, want)]


def _random_f32(n, seed, lo=-45, hi=38):
    rng = np.random.default_rng(seed)
    mag = 10.0 ** rng.uniform(lo, hi, size=n)
    v = (mag * rng.choice([-1.0, 1.0], size=n)).astype(np.float32)
    # exact ties of the 16-bit cut: low half 0x8000 with both parities of bit 16
    bits = rng.integers(0, 2 ** 31, size=n // 4, dtype=np.uint64).astype(np.uint32)
    ties = ((bits & np.uint32(0xFFFF0000)) | np.uint32(0x8000)).view(np.float32)
    return np.concatenate([v, ties[np.isfinite(ties)]])


def test_bf16_round_matches_torch_cast():
    v = _random_f32(200_000, 1)
    want = torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = O.bf16_bits(v.astype(np.float64))
    assert np.array_equal(got, want)


def test_e4m3_round_matches_torch_cast_in_range():
    # torch's cast gives NaN above 464 instead of saturating, so compare below it
    rng = np.random.default_rng(2)
    v = (rng.uniform(-463.9, 463.9, size=100_000)).astype(np.float32)
    v2 = (10.0 ** rng.uniform(-5, 2.6, size=100_000) * rng.choice([-1, 1], size=100_000)).astype(np.float32)
    grid = O.e4m3_decode(np.arange(256, dtype=np.uint8))
    grid = grid[np.isfinite(grid) & (np.abs(grid) < 448)]
    mids = ((grid[:-1] + grid[1:]) / 2).astype(np.float32) if len(grid) > 1 else np.zeros(0, np.float32)
    allv = np.concatenate([v, v2, np.sort(grid).astype(np.float32), np.sort(mids)])
    allv = allv[np.abs(allv) < 464]
    want = torch.from_numpy(allv).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = O.e4m3_encode(allv.astype(np.float64))
    # torch keeps the sign of a zero result; so does the oracle
    assert np.array_equal(got, want)


def test_e4m3_decode_all_codes_match_torch():
    codes = np.arange(256, dtype=np.uint8)
    want = torch.from_numpy(codes).view(torch.float8_e4m3fn).float().numpy().astype(np.float64)
    got = O.e4m3_decode(codes)
    assert np.array_equal(np.isnan(got), np.isnan(want))
    ok = ~np.isnan(want)
    assert np.array_equal(got[ok], want[ok])


def test_e4m3_saturation_by_definition():
    v = np.array([448.0, 449.0, 500.0, 1e30, np.inf, -np.inf, -470.0])
    r = O.e4m3_round(v)
    assert np.array_equal(r, [448, 448, 448, 448, 448, -448, -448])
    assert np.isnan(O.e4m3_round(np.array([np.nan]))[0])


def test_e4m3_encode_decode_roundtrip():
    codes = np.arange(256, dtype=np.uint8)
    vals = O.e4m3_decode(codes)
    finite = np.isfinite(vals)
    back = O.e4m3_encode(vals[finite])
    assert np.array_equal(back, codes[finite])


# ---------------------------------------------------------------------------
# the operation: brute force, closed forms, identities
# ---------------------------------------------------------------------------
def _tiny(seed=0, M=4, d=8, N=8):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((M, d)) * np.exp(rng.uniform(np.log(0.1), np.log(10), size=(M, 1)))
    g = 1 + 0.1 * rng.standard_normal(d)
    W = rng.standard_normal((d, N)) / math.sqrt(d)
    W2 = rng.standard_normal((d, N)) / math.sqrt(d)
    return x, g, W, W2


def _brute_norm_proj(x, g, W, eps):
    M, d = x.shape
    N = W.shape[1]
    out = [[0.0] * N for _ in range(M)]
    for m in range(M):
        ms = math.fsum(x[m, k] * x[m, k] for k in range(d)) / d
        inv = 1.0 / math.sqrt(ms + eps)
        h = [x[m, k] * inv * g[k] for k in range(d)]
        for n in range(N):
            out[m][n] = math.fsum(h[k] * W[k, n] for k in range(d))
    return np.array(out)


def _brute_silu(z):
    return z / (1.0 + math.exp(-z)) if z > -700 else -0.0


def _rel(a, b):
    return float(np.max(np.abs(a - b) / (1.0 + np.abs(b))))


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_norm_proj_brute_force_4x8x8(seed):
    x, g, W, _ = _tiny(seed)
    for eps in (0.0, 1e-6, 0.5):
        assert _rel(O.norm_proj(x, g, W, eps), _brute_norm_proj(x, g, W, eps)) <= 1e-14


@pytest.mark.parametrize("seed", [0, 1])
def test_swiglu_brute_force(seed):
    x, g, Wg, Wu = _tiny(seed)
    eps = 1e-6
    G = _brute_norm_proj(x, g, Wg, eps)
    U = _brute_norm_proj(x, g, Wu, eps)
    want = np.array([[_brute_silu(G[m, n]) * U[m, n] for n in range(G.shape[1])] for m in range(G.shape[0])])
    assert _rel(O.norm_proj_swiglu(x, g, Wg, Wu, eps), want) <= 1e-14


def test_matches_torch_rms_norm_then_matmul():
    x, g, W, _ = _tiny(3, M=16, d=64, N=32)
    eps = 1e-6
    xt = torch.from_numpy(x)
    ref_g1 = (torch.nn.functional.rms_norm(xt, (x.shape[1],), eps=eps) @ torch.from_numpy(W)).numpy()
    assert _rel(O.norm_proj(x, np.ones(x.shape[1]), W, eps), ref_g1) <= 1e-13
    ref = (torch.nn.functional.rms_norm(xt, (x.shape[1],), weight=torch.from_numpy(g), eps=eps)
           @ torch.from_numpy(W)).numpy()
    assert _rel(O.norm_proj(x, g, W, eps), ref) <= 1e-13


def test_silu_closed_forms_and_torch():
    z = np.linspace(-50, 50, 2001)
    s = O.silu(z)
    assert O.silu(np.array([0.0]))[0] == 0.0
    # silu(z) - silu(-z) = z  (sigma(z) + sigma(-z) = 1)
    assert np.max(np.abs((s - O.silu(-z)) - z)) <= 1e-12
    assert abs(O.silu(np.array([40.0]))[0] - 40.0) <= 1e-12
    assert abs(O.silu(np.array([-800.0]))[0]) == 0.0
    ref = torch.nn.functional.silu(torch.from_numpy(z)).numpy()
    assert np.max(np.abs(s - ref)) <= 1e-14


def test_constant_row_closed_form():
    rng = np.random.default_rng(5)
    d, N = 32, 16
    g = 1 + 0.1 * rng.standard_normal(d)
    W = rng.standard_normal((d, N))
    for c in (3.5, -0.25):
        x = np.full((1, d), c)
        want = math.copysign(1.0, c) * (g[:, None] * W).sum(axis=0)
        assert _rel(O.norm_proj(x, g, W, 0.0)[0], want) <= 1e-14


def test_zero_row():
    rng = np.random.default_rng(6)
    W = rng.standard_normal((16, 8))
    g = np.ones(16)
    x = np.zeros((2, 16))
    assert np.all(O.norm_proj(x, g, W, 1e-6) == 0.0)
    assert np.all(np.isnan(O.norm_proj(x, g, W, 0.0)))


def test_fold_identity_real_arithmetic():
    """Proposal 1: x_hat @ (diag(g) W) equals (x_hat * g) @ W (fp64, no rounding)."""
    for name in ("tiny", "decode_qkv"):
        inp = WL.workload_case(name)
        x, g, W, eps = inp["x"], O.to_f64(inp["g"]), O.to_f64(inp["W"]), inp["eps"]
        folded = O.norm_proj(x, np.ones_like(g), g[:, None] * W, eps)
        unfolded = O.norm_proj(x, g, W, eps)
        assert _rel(folded, unfolded) <= 1e-12


@pytest.mark.parametrize("a", [1e-3, 0.5, 3.0, 1e3])
def test_scale_invariance(a):
    """Proposal 3: RMSNorm(a x) = RMSNorm(x) for a > 0, exactly when eps = 0."""
    x, g, W, _ = _tiny(7, M=8, d=64, N=16)
    assert _rel(O.rmsnorm(a * x, g, 0.0), O.rmsnorm(x, g, 0.0)) <= 1e-12
    # eps > 0: exact invariance is lost, by no more than the first-order bound
    eps = 1e-6
    h1 = O.rmsnorm(a * x, g, eps)
    h0 = O.rmsnorm(x, g, eps)
    ms = np.mean(x * x, axis=1)
    lo = ms + min(eps, eps / a ** 2)
    bound = np.abs(x * g) * 0.5 * lo[:, None] ** -1.5 * eps * abs(1 - 1 / a ** 2)
    assert np.all(np.abs(h1 - h0) <= bound * (1 + 1e-9) + 1e-15)


def test_back_to_back_norm_removal():
    """Proposal 3: a weightless RMSNorm followed by RMSNorm equals the second alone."""
    x, g, W, _ = _tiny(8, M=8, d=64, N=16)
    inner = O.rmsnorm(x, np.ones(x.shape[1]), 0.0)
    assert _rel(O.rmsnorm(inner, g, 0.0), O.rmsnorm(x, g, 0.0)) <= 1e-12
    assert _rel(O.norm_proj(inner, g, W, 0.0), O.norm_proj(x, g, W, 0.0)) <= 1e-12


# ---------------------------------------------------------------------------
# the fold and the weight encodings
# ---------------------------------------------------------------------------
def test_fold_bf16_matches_torch_route():
    inp = WL.case(4, 256, 512, False, seed=11)
    g, W = inp["g"], inp["W"]
    want = (g[:, None] * W.float()).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(O.fold_bf16(W, g), want)
    # a gain that is not bf16-representable: fp32 product rounds, then bf16 rounds
    g2 = torch.linspace(0.3, 1.7, 256, dtype=torch.float32)
    want2 = (g2[:, None] * W.float()).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(O.fold_bf16(W, g2), want2)


def test_interleave_layout_brute_force():
    d, N = 3, 384
    A = np.arange(d * N).reshape(d, N)
    B = -1 - np.arange(d * N).reshape(d, N)
    C = O.interleave128(A, B)
    for k in range(d):
        for n in range(N):
            j, c = divmod(n, 128)
            assert C[k, 256 * j + c] == A[k, n]
            assert C[k, 256 * j + 128 + c] == B[k, n]
    A2, B2 = O.deinterleave128(C)
    assert np.array_equal(A2, A) and np.array_equal(B2, B)


def test_fold_fp8_properties():
    inp = WL.case(4, 256, 384, False, seed=12)
    W, g = inp["W"], inp["g"]
    W = W.clone()
    W[128:256, 256:384] = 0           # one all-zero block
    q, s = O.fold_fp8(W, g)
    assert q.shape == (256, 384) and s.shape == (2, 3) and s.dtype == np.float32
    P = O.to_f64(g)[:, None] * O.to_f64(W)          # exact: bf16 * bf16 fits fp32
    vals = O.e4m3_decode(q)
    for bi in range(2):
        for bj in range(3):
            blk = vals[128 * bi:128 * bi + 128, 128 * bj:128 * bj + 128]
            pb = P[128 * bi:128 * bi + 128, 128 * bj:128 * bj + 128]
            if bi == 1 and bj == 2:
                assert s[bi, bj] == 1.0 and np.all(blk == 0)
                continue
            amax = np.max(np.abs(pb))
            assert abs(s[bi, bj] - amax / 448) <= 2 ** -24 * amax / 448
            assert np.max(np.abs(blk)) == 448.0        # the amax element lands on 448
            # dequantised error within half an e4m3 step (plus fp32 quotient rounding)
            deq = blk * float(s[bi, bj])
            step = np.where(np.abs(pb) / s[bi, bj] >= 2 ** -6,
                            2.0 ** (np.floor(np.log2(np.maximum(np.abs(pb) / s[bi, bj], 2 ** -6))) - 3),
                            2.0 ** -9) * s[bi, bj]
            assert np.all(np.abs(deq - pb) <= 0.5 * step * (1 + 1e-6) + 1e-30)
    # torch's own e4m3 cast of the same fp32 quotient gives the same codes
    s_full = np.repeat(np.repeat(s, 128, 0), 128, 1)
    quot = (P.astype(np.float32) / s_full).astype(np.float32)
    want = torch.from_numpy(quot).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(q, want)


def test_dequant_bf16_rounding_matches_torch_route():
    """bf16(fp32(e4m3(q)) * s): torch computes the same product and cast."""
    rng = np.random.default_rng(13)
    q = rng.integers(0, 256, size=(256, 384), dtype=np.uint8)
    q[(q & 0x7F) == 0x7F] = 0                                  # no NaN codes
    s = (10.0 ** rng.uniform(-4, 1, size=(2, 3))).astype(np.float32)
    got = O.dequant_fp8_bf16_bits(q, s)
    qt = torch.from_numpy(q).view(torch.float8_e4m3fn).float()
    st = torch.from_numpy(np.repeat(np.repeat(s, 128, 0), 128, 1))
    want = (qt * st).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(got, want)


def test_dequant_exact():
    q = np.array([[0x38, 0x7E], [0x01, 0xC0]], dtype=np.uint8)
    q = np.tile(q, (64, 64))
    s = np.array([[0.5]], dtype=np.float32)
    d = O.dequant_fp8(q, s)
    assert d[0, 0] == 0.5 and d[0, 1] == 224.0 and d[1, 0] == 2.0 ** -10 and d[1, 1] == -1.0


# ---------------------------------------------------------------------------
# planted mistakes: each must be caught by at least one pin above
# ---------------------------------------------------------------------------
def _pins_pass(norm_proj, norm_proj_swiglu, interleave):
    """Re-run the independent pins against a candidate implementation."""
    try:
        for seed in (0, 1):
            x, g, W, W2 = _tiny(seed)
            for eps in (0.0, 1e-6, 0.5):
                if _rel(norm_proj(x, g, W, eps), _brute_norm_proj(x, g, W, eps)) > 1e-14:
                    return False
            G = _brute_norm_proj(x, g, W, 1e-6)
            U = _brute_norm_proj(x, g, W2, 1e-6)
            want = np.array([[_brute_silu(G[m, n]) * U[m, n] for n in range(8)] for m in range(4)])
            if _rel(norm_proj_swiglu(x, g, W, W2, 1e-6), want) > 1e-14:
                return False
        A = np.arange(2 * 256).reshape(2, 256)
        C = interleave(A, -A - 1)
        if not (C[1, 256 + 5] == A[1, 128 + 5] and C[0, 128] == -A[0, 0] - 1):
            return False
        return True
    except Exception:
        return False


def _swiglu_from(np_fn):
    return lambda x, g, Wg, Wu, eps: O.silu(np_fn(x, g, Wg, eps)) * np_fn(x, g, Wu, eps)


def _mut_eps_outside(x, g, W, eps):
    ms = np.mean(x * x, axis=1)
    with np.errstate(divide="ignore"):
        return ((x * (1 / np.sqrt(ms) + eps)[:, None]) * g) @ W


def _mut_divisor(x, g, W, eps):
    ms = np.sum(x * x, axis=1) / (x.shape[1] - 1)
    return ((x / np.sqrt(ms + eps)[:, None]) * g) @ W


def _mut_gain_on_output(x, g, W, eps):
    return (O.rmsnorm(x, np.ones_like(g), eps) @ W) * g[None, :W.shape[1]]


def _mut_transposed(x, g, W, eps):
    return O.rmsnorm(x, g, eps) @ W.T


def _mut_no_norm(x, g, W, eps):
    return (x * g) @ W


def test_pins_accept_the_oracle():
    assert _pins_pass(O.norm_proj, O.norm_proj_swiglu, O.interleave128)


@pytest.mark.parametrize("mutant", [_mut_eps_outside, _mut_divisor, _mut_gain_on_output,
                                    _mut_transposed, _mut_no_norm])
def test_pins_catch_planted_norm_mistakes(mutant):
    assert not _pins_pass(mutant, _swiglu_from(mutant), O.interleave128)


def test_pins_catch_planted_swiglu_mistakes():
    up_gate_swapped = lambda x, g, Wg, Wu, eps: O.silu(O.norm_proj(x, g, Wu, eps)) * O.norm_proj(x, g, Wg, eps)
    silu_sign = lambda x, g, Wg, Wu, eps: (lambda z: z / (1 + np.exp(z)))(O.norm_proj(x, g, Wg, eps)) * O.norm_proj(x, g, Wu, eps)
    assert not _pins_pass(O.norm_proj, up_gate_swapped, O.interleave128)
    assert not _pins_pass(O.norm_proj, silu_sign, O.interleave128)
    swapped_interleave = lambda A, B: O.interleave128(B, A)
    assert not _pins_pass(O.norm_proj, O.norm_proj_swiglu, swapped_interleave)


# ---------------------------------------------------------------------------
# row-parallel (d-split) form: shares over any partition of d add up to the
# single-device result (the definition computed the unfolded way)
# ---------------------------------------------------------------------------
def _partition(d, parts, rng):
    cuts = np.sort(rng.choice(np.arange(1, d), size=parts - 1, replace=False)) if parts > 1 else np.array([], int)
    edges = np.concatenate([[0], cuts, [d]])
    return list(zip(edges[:-1], edges[1:]))


@pytest.mark.parametrize("parts", [1, 2, 3, 7])
@pytest.mark.parametrize("swiglu", [False, True])
def test_rowparallel_shares_add_up(parts, swiglu):
    rng = np.random.default_rng(parts * 10 + swiglu)
    M, d, N = 5, 48, 256
    x = rng.standard_normal((M, d)) * np.exp(rng.uniform(-2, 2, (M, 1)))
    Wg = rng.standard_normal((d, N)) / np.sqrt(d)
    Wu = rng.standard_normal((d, N)) / np.sqrt(d)
    W = O.interleave128(Wg, Wu) if swiglu else Wg
    acc = np.zeros((M, W.shape[1]))
    ssq = np.zeros(M)
    for k0, k1 in _partition(d, parts, rng):
        a, s = O.rowparallel_partial(x[:, k0:k1], W[k0:k1])
        acc += a
        ssq += s
    y = O.rowparallel_finish(acc, ssq, d, 1e-6, swiglu)
    want = (O.norm_proj_swiglu(x, np.ones(d), Wg, Wu, 1e-6) if swiglu else O.norm_proj(x, np.ones(d), Wg, 1e-6))
    assert np.max(np.abs(y - want) / (1 + np.abs(want))) < 1e-12


def test_rowparallel_finish_closed_form():
    """A constant row c with eps = 0: r = 1/|c|, so y = sign(c) * sum_k W[k]."""
    d, N = 16, 128
    W = np.random.default_rng(2).standard_normal((d, N))
    x = np.full((1, d), -3.0)
    acc, ssq = O.rowparallel_partial(x, W)
    y = O.rowparallel_finish(acc, ssq, d, 0.0)
    assert np.allclose(y[0], -W.sum(axis=0), rtol=1e-13, atol=1e-13)
