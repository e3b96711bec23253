"""Pins for the oracle's NVFP4 output encoding (the quantising SwiGLU
epilogue), run on the CPU.

The encoding follows the FlashInfer PR #4040 analysis (SwiGLU fused with its
NVFP4 quantisation: e2m1 elements, one scale factor per 16 elements, a global
scale).  Each check ties the oracle to something other than itself: the e2m1
format's definition (hand-derived golden points and its eight magnitudes),
torch's own e4m3 cast, a brute-force nearest-value search, closed forms and
the rounding error bound of the format.  The planted-mistake tests show that
a wrong constant or a swapped nibble order fails them.
"""
import math
import os

import numpy as np
import pytest
import torch

import oracle as O
from tests._golden import read_golden
import oracle.flashnorm_oracle as OF

# The eight e2m1 magnitudes in code order (OCP Microscaling formats
# specification, FP4 E2M1): code i holds E2M1_VALUES[i], its mantissa bit is i & 1.
E2M1_VALUES = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]




def test_e2m1_golden_points(golden_dir):
    rows = read_golden(os.path.join(golden_dir, "e2m1_points.txt"))
    vals = np.array([v for v, _ in rows])
    want = np.array([c for _, c in rows], dtype=np.uint8)
    got = O.e2m1_encode(vals)
    assert np.array_equal(got, want), [(v, hex(g), hex(w)) for v, g, w in zip(vals, got, want)]


def test_e2m1_code_table():
    got = O.e2m1_decode(np.arange(16))
    assert list(got[:8]) == E2M1_VALUES
    assert list(-got[8:]) == E2M1_VALUES and all(np.signbit(got[8:]))
    assert np.array_equal(O.e2m1_encode(got), np.arange(16, dtype=np.uint8))


def _brute_e2m1(x):
    """Nearest of the eight magnitudes by search, ties to the even code,
    saturating at 6; the sign is carried over (so -0 keeps its sign)."""
    a = abs(x)
    best = None
    for i, v in enumerate(E2M1_VALUES):
        d = abs(a - v)
        if best is None or d < best[0] or (d == best[0] and i % 2 == 0):
            best = (d, i)
    code = best[1]
    if a > 6.0:
        code = 7
    return code | (8 if math.copysign(1.0, x) < 0 else 0)


def test_e2m1_rounding_brute_force():
    grid = np.arange(-8.0, 8.0 + 1e-9, 1.0 / 64)
    rng = np.random.default_rng(7)
    rnd = rng.uniform(-10, 10, 4000)
    tiny = rng.uniform(-0.3, 0.3, 500)
    vals = np.concatenate([grid, rnd, tiny])
    got = O.e2m1_encode(vals)
    want = np.array([_brute_e2m1(float(v)) for v in vals], dtype=np.uint8)
    bad = np.nonzero(got != want)[0]
    assert bad.size == 0, [(vals[i], got[i], want[i]) for i in bad[:10]]


def _torch_e4m3_code(t):
    return int(torch.tensor([t], dtype=torch.float64).to(torch.float8_e4m3fn).view(torch.uint8)[0])


def _brute_nvfp4(y, gs):
    """Pure-Python loops over rows and 16-element blocks; the scale rounding by
    torch's e4m3 cast, the element rounding by the nearest-value search."""
    M, N = len(y), len(y[0])
    codes = [[0] * N for _ in range(M)]
    sfs = [[0] * (N // 16) for _ in range(M)]
    for m in range(M):
        for b in range(N // 16):
            blk = y[m][16 * b:16 * b + 16]
            amax = max(abs(v) for v in blk)
            sf = _torch_e4m3_code(gs * amax / 6.0)
            sfs[m][b] = sf
            sf_val = float(torch.tensor([sf], dtype=torch.uint8).view(torch.float8_e4m3fn).to(torch.float64)[0])
            for j, v in enumerate(blk):
                codes[m][16 * b + j] = _brute_e2m1(v * gs / sf_val) if sf_val > 0 else _brute_e2m1(v * 0.0)
    return np.array(codes, dtype=np.uint8), np.array(sfs, dtype=np.uint8)


@pytest.mark.parametrize("gs", [1.0, 37.5, 1.0 / 3.0])
def test_nvfp4_brute_force_small(gs):
    rng = np.random.default_rng(11)
    y = rng.standard_normal((5, 48)) * np.exp(rng.uniform(-3, 3, (5, 1)))
    y[2, 16:32] = 0.0                       # an all-zero block
    y[3, :16] *= 1e-4                       # a block whose scale is subnormal
    gs = float(np.float32(gs))
    codes, sf = O.nvfp4_quantize(y, gs)
    bc, bs = _brute_nvfp4(y.tolist(), gs)
    assert np.array_equal(sf, bs)
    assert np.array_equal(codes, bc)


@pytest.mark.parametrize("k", [-9, -7, -6, -1, 0, 3, 8])
def test_nvfp4_exact_blocks(k):
    """A block of e2m1 values times 2^k whose maximum is 6 * 2^k has the scale
    2^k exactly (gs = 1) and round-trips exactly."""
    rng = np.random.default_rng(k + 20)
    vals = np.array(E2M1_VALUES)[rng.integers(0, 8, (3, 64))] * rng.choice([-1.0, 1.0], (3, 64))
    vals[:, ::16] = 6.0                      # every block holds the maximum
    y = vals * 2.0 ** k
    codes, sf = O.nvfp4_quantize(y, 1.0)
    assert np.all(O.e4m3_decode(sf) == 2.0 ** k)
    assert np.array_equal(O.nvfp4_dequantize(codes, sf, 1.0), y)


def test_nvfp4_error_bound():
    """Rounding error of each element, in units of the block's step: at most
    half the e2m1 spacing at its magnitude; the block maximum, scaled, stays
    within 6 * (1 + 2^-4) (the e4m3 scale's relative rounding)."""
    rng = np.random.default_rng(3)
    y = rng.standard_normal((64, 256)) * np.exp(rng.uniform(-4, 4, (64, 1)))
    gs = float(np.float32(448.0 * 6.0 / np.max(np.abs(y))))
    codes, sf = O.nvfp4_quantize(y, gs)
    sfv = np.repeat(O.e4m3_decode(sf), 16, axis=1)
    assert np.all(sfv >= 2.0 ** -6)          # normal scales in this range
    scaled = y * gs / sfv
    assert np.max(np.abs(scaled)) <= 6.0 * (1 + 2.0 ** -4)
    q = O.e2m1_decode(codes)
    half_step = np.where(np.abs(scaled) < 2, 0.25, np.where(np.abs(scaled) < 4, 0.5, 1.0))
    assert np.all(np.abs(q - scaled) <= half_step)
    # and the dequantised value agrees in real units
    deq = O.nvfp4_dequantize(codes, sf, gs)
    assert np.allclose(deq, q * sfv / gs, rtol=0, atol=0)


def test_nvfp4_special_blocks():
    y = np.ones((4, 32))
    y[0, :16] = 0.0
    y[1, 5] = np.nan
    y[2, 20] = -np.inf
    y[3, :16] = 1e-9                         # scale underflows to zero
    codes, sf = O.nvfp4_quantize(y, 1.0)
    assert sf[0, 0] == 0 and np.all(codes[0, :16] == 0)
    assert sf[1, 0] == 0x7F and np.all(codes[1, :16] == 0) and sf[1, 1] != 0x7F
    assert sf[2, 1] == 0x7F and np.all(codes[2, 16:] == 0) and sf[2, 0] != 0x7F
    assert sf[3, 0] == 0 and np.all(codes[3, :16] == 0)
    assert np.all(np.isnan(O.nvfp4_dequantize(codes, sf, 1.0)[1, :16]))
    # saturation: a huge global scale clamps the scale to 448 and the codes to +-6
    y2 = np.linspace(-1, 1, 32).reshape(1, 32)
    c2, s2 = O.nvfp4_quantize(y2, 1e6)
    assert np.all(s2 == 0x7E)
    assert np.all(O.e2m1_decode(c2)[0, [0, 31]] == [-6.0, 6.0])


def test_nvfp4_pack_layout():
    codes = np.array([[0x1, 0x2, 0xF, 0x0, 0x8, 0x7]], dtype=np.uint8)
    packed = O.nvfp4_pack(codes)
    assert packed.tolist() == [[0x21, 0x0F, 0x78]]
    assert np.array_equal(O.nvfp4_unpack(packed), codes)


def test_planted_wrong_constant_fails(monkeypatch):
    monkeypatch.setattr(OF, "E2M1_MAX", 4.0)
    with pytest.raises(AssertionError):
        test_nvfp4_exact_blocks(0)


def test_planted_swapped_nibbles_fail(monkeypatch):
    monkeypatch.setattr(OF, "nvfp4_pack", lambda c: (np.asarray(c)[:, 1::2] & 0xF) | ((np.asarray(c)[:, 0::2] & 0xF) << 4))
    monkeypatch.setattr(O, "nvfp4_pack", OF.nvfp4_pack)
    with pytest.raises(AssertionError):
        test_nvfp4_pack_layout()


# ---------------------------------------------------------------------------
# the GPU tests' band check, exercised on oracle encodings
# ---------------------------------------------------------------------------
def _band_case():
    rng = np.random.default_rng(5)
    ref = rng.standard_normal((8, 64)) * np.exp(rng.uniform(-2, 2, (8, 1)))
    ref[3, 5] = np.nan
    tol = 1e-2
    gs = float(np.float32(448.0 * 6.0 / np.nanmax(np.abs(ref))))
    # a stand-in for the kernel's value: anywhere inside the tolerance band
    v = ref + rng.uniform(-0.9, 0.9, ref.shape) * tol * (1.0 + np.abs(ref))
    q, sf = O.nvfp4_quantize(v, gs)
    return ref, tol, gs, q, sf


def test_band_check_accepts_values_inside_the_band():
    from tests._util import check_nvfp4
    ref, tol, gs, q, sf = _band_case()
    frac = check_nvfp4(O.nvfp4_pack(q), sf, ref, gs, tol, min_exact=0.8)
    assert 0.8 <= frac <= 1.0


@pytest.mark.parametrize("mistake", ["swap_nibbles", "scale_up", "wrong_gs", "nan_scale_lost", "code_flip"])
def test_band_check_rejects_planted_mistakes(mistake):
    from tests._util import check_nvfp4
    ref, tol, gs, q, sf = _band_case()
    q, sf = q.copy(), sf.copy()
    if mistake == "swap_nibbles":
        packed = O.nvfp4_pack(q)
        packed = ((packed & 0xF) << 4) | (packed >> 4)
    else:
        if mistake == "scale_up":
            sf[0, 0] += 2                   # two e4m3 steps above the band
        elif mistake == "wrong_gs":
            q, sf = O.nvfp4_quantize(ref, gs * 3.0)
        elif mistake == "nan_scale_lost":
            sf[3, 0] = 0x30
        elif mistake == "code_flip":
            i = int(np.argmax(np.abs(O.e2m1_decode(q[0]))))
            q[0, i] ^= 0x8                  # the sign of the largest element
        packed = O.nvfp4_pack(q)
    with pytest.raises(AssertionError):
        check_nvfp4(packed, sf, ref, gs, tol, min_exact=0.8)
