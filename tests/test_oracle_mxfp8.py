"""Pins for the oracle's MXFP8 weight fold (e4m3 codes with one ue8m0 scale
per 32 k values per column), run on the CPU.

Checks against torch's own e4m3 cast, a brute-force search for the shared
exponent, the defining property of the round-up exponent rule, closed forms
and the format's rounding bound.  The kernel for this format is not built
yet; the oracle comes first.
"""
import os

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


# ---------------------------------------------------------------------------
# the chunked scale layout (block-scaled tensor-core MMAs; NVFP4 swizzled scales)
# ---------------------------------------------------------------------------
def _golden_positions(golden_dir):
    rows = []
    with open(os.path.join(golden_dir, "sf_chunk_points.txt")) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                r, c, off = line.split()[:3]
                rows.append((int(r), int(c), int(off)))
    return rows


def test_sf_chunk_golden_positions(golden_dir):
    S = np.zeros((256, 8), dtype=np.uint8)
    pts = _golden_positions(golden_dir)
    for i, (r, c, _) in enumerate(pts):
        S[r, c] = i + 1
    flat = O.sf_chunk_layout(S)
    assert flat.size == 256 * 8
    for i, (_, _, off) in enumerate(pts):
        assert flat[off] == i + 1, (pts[i], int(np.argmax(flat == i + 1)))


def test_sf_chunk_reshape_form():
    """The same layout written as a reshape and a transposition: rows split
    into (block, group of 32, lane), columns into (chunk, slot); the chunk
    is [lane][group][slot]."""
    rng = np.random.default_rng(3)
    R, C = 384, 12
    S = rng.integers(0, 256, (R, C)).astype(np.uint8)
    t = S.reshape(R // 128, 4, 32, C // 4, 4)             # [block][group][lane][chunk][slot]
    want = t.transpose(0, 3, 2, 1, 4).reshape(-1)         # [block][chunk][lane][group][slot]
    assert np.array_equal(O.sf_chunk_layout(S), want)


def test_sf_chunk_padding_and_inverse():
    rng = np.random.default_rng(4)
    R, C = 200, 6                                          # ragged: padded to 256 x 8
    S = rng.integers(1, 256, (R, C)).astype(np.uint8)
    flat = O.sf_chunk_layout(S)
    assert flat.size == 256 * 8
    assert np.count_nonzero(flat) == R * C                 # padding bytes are zero
    assert np.array_equal(O.sf_chunk_unlayout(flat, R, C), S)
    assert sorted(flat[flat > 0].tolist()) == sorted(S.ravel().tolist())


def test_sf_chunk_planted_mistake_is_caught(golden_dir, monkeypatch):
    """A layout with the lane and row-group roles swapped fails the golden positions."""
    def wrong(S):
        S = np.asarray(S, dtype=np.uint8)
        R, C = S.shape
        r, c = np.indices((R, C))
        dest = 512 * ((r // 128) * (C // 4) + c // 4) + 4 * (r % 32) + 128 * ((r % 128) // 32) + (c % 4)
        out = np.zeros(R * C, dtype=np.uint8)
        out[dest.ravel()] = S.ravel()
        return out
    monkeypatch.setattr(O, "sf_chunk_layout", wrong)
    with pytest.raises(AssertionError):
        test_sf_chunk_golden_positions(golden_dir)


def test_stored_mxfp8_fold_is_the_fold_in_chunks():
    inp = WL.case(4, 256, 384, False, seed=22)
    q, sb = O.fold_mxfp8(inp["W"], inp["g"])
    q2, flat = O.fold_mxfp8_stored(inp["W"], inp["g"])
    assert np.array_equal(q, q2) and flat.size == 256 * 384 // 32
    # column n, k block j: k group j div 4 (3 chunks of 128 columns each), chunk n div 128
    for n in (0, 31, 32, 127, 128, 300, 383):
        for j in (0, 3, 4, 7):
            off = 512 * ((j // 4) * 3 + n // 128) + 16 * (n % 32) + 4 * ((n % 128) // 32) + j % 4
            assert flat[off] == sb[j, n]
    # a 128-row slice of the weight owns a contiguous range of the scale bytes
    q3, flat3 = O.fold_mxfp8_stored(inp["W"][128:], inp["g"][128:])
    assert np.array_equal(flat3, flat[flat.size // 2:])
