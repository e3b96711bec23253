"""Pins for the oracle's MXFP8 weight fold (e4m3 codes with one ue8m0 scale
per 32 k values per column), run on the CPU.

Checks against torch's own e4m3 cast, a brute-force search for the shared
exponent, the defining property of the round-up exponent rule, closed forms
and the format's rounding bound.  The kernel for this format is not built
yet; the oracle comes first.
"""
import numpy as np
import pytest
import torch

import oracle as O
import workloads as WL


def _product(W, g):
    return (np.asarray(g, dtype=np.float32)[:, None] * np.asarray(W, dtype=np.float32)).astype(np.float64)


@pytest.fixture(scope="module")
def folded():
    inp = WL.case(4, 256, 384, False, seed=21)
    W, g = O.to_f64(inp["W"]), O.to_f64(inp["g"])
    W[32:64, 5] = 0.0                                  # an all-zero block
    W[64:96, 7] *= 1e-30                               # a block of tiny values (subnormal e4m3 codes)
    q, s = O.fold_mxfp8(W, g)
    return W, g, q, s


def test_codes_match_torch_cast(folded):
    W, g, q, s = folded
    P = _product(W, g)
    scale = np.repeat(np.ldexp(1.0, s.astype(np.int64) - 127), 32, axis=0)
    want = torch.from_numpy(P / scale).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(q, want)


def test_shared_exponent_brute_force(folded):
    W, g, q, s = folded
    P = _product(W, g)
    d, N = P.shape
    for b in range(d // 32):
        for n in range(0, N, 7):
            amax = float(np.max(np.abs(P[32 * b:32 * b + 32, n])))
            if amax == 0.0:
                assert s[b, n] == 0
                continue
            E = -127
            while amax > 448.0 * 2.0 ** E:          # the smallest E with amax / 2^E <= 448
                E += 1
            assert s[b, n] == E + 127, (b, n, amax)


def test_block_maxima_fill_the_top_binade(folded):
    W, g, q, s = folded
    blocks = q.reshape(-1, 32, q.shape[1]).transpose(0, 2, 1)     # [d/32, N, 32]
    vals = np.abs(O.e4m3_decode(blocks)).max(axis=2)
    nz = s > 0
    assert np.all(vals[nz] >= 224.0) and np.all(vals <= 448.0)
    assert np.all(blocks[~nz] == 0) and (~nz).any()


def test_dequantised_error_bound(folded):
    W, g, q, s = folded
    P = _product(W, g)
    deq = O.dequant_mxfp8(q, s)
    step = np.repeat(np.ldexp(1.0, s.astype(np.int64) - 127), 32, axis=0)
    # e4m3: half an ulp is at most 2^-4 of the value for normals, 2^-10 of the scale below 2^-6
    assert np.all(np.abs(deq - P) <= np.maximum(np.abs(P) * 2.0 ** -4, step * 2.0 ** -10) * (1 + 1e-12))


@pytest.mark.parametrize("k", [-20, -3, 0, 5])
def test_exact_blocks_round_trip(k):
    """A block whose maximum is 448 * 2^k of e4m3 values times 2^k: E = k and
    the codes reproduce it exactly (g = 1)."""
    rng = np.random.default_rng(k + 40)
    codes = rng.integers(0, 0x7F, (64, 128)).astype(np.uint8)
    vals = O.e4m3_decode(codes)
    vals[0, :] = 448.0
    vals[32, :] = -448.0
    W = vals * 2.0 ** k
    q, s = O.fold_mxfp8(W, np.ones(64))
    assert np.all(s == k + 127)
    assert np.array_equal(O.dequant_mxfp8(q, s), W)
