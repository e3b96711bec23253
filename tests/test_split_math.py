"""The arithmetic fact the fp8 decode kernel rests on, checked on the CPU.

With fp8 e4m3 weights and bf16 activations, the decode kernel feeds the e4m3
weight codes to an 8-bit tensor-core MMA and converts the activations
instead: per row and 128-deep k block it scales x by a power of two so that
the largest magnitude lies in [128, 256) and splits each scaled value a into
hi = e4m3(a) and lo = e4m3(a - hi).  The claim is that a == hi + lo exactly
for every |a| >= 1/4 (a bf16 value has 8 significant bits; hi keeps the top
4 and lo the rest), and that below 1/4 the error is at most 2^-10.  Checked
exhaustively over every bf16 value in the range, with the oracle's e4m3
rounding (written from the format definition) and, independently, with
torch's float8_e4m3fn cast.
"""
import numpy as np
import torch

import oracle as O


def _all_bf16(lo_exp: int, hi_exp: int) -> np.ndarray:
    """Every positive and negative finite bf16 value with lo_exp <= exponent < hi_exp."""
    bits = np.arange(0, 1 << 16, dtype=np.uint32)
    f32 = (bits << 16).view(np.float32)
    vals = f32[np.isfinite(f32) & (f32 != 0)].astype(np.float64)
    exp = np.floor(np.log2(np.abs(vals)))
    return vals[(exp >= lo_exp) & (exp < hi_exp)]


def _split(a: np.ndarray, rnd):
    hi = rnd(a)
    lo = rnd(a - hi)        # a - hi is exact in fp64 (and in the kernel's fp32 and f16 steps)
    return hi, lo


def _torch_e4m3(v: np.ndarray) -> np.ndarray:
    return torch.from_numpy(v.astype(np.float32)).to(torch.float8_e4m3fn).to(torch.float64).numpy()


def test_split_is_exact_from_a_quarter_to_256():
    a = _all_bf16(-2, 8)                      # 1/4 <= |a| < 256
    for rnd in (O.e4m3_round, _torch_e4m3):
        hi, lo = _split(a, rnd)
        assert np.array_equal(hi + lo, a)
        # both parts are e4m3 values in range (no saturation)
        assert np.all(np.abs(hi) <= 448) and np.all(np.abs(lo) <= 448)
        assert np.array_equal(rnd(hi), hi) and np.array_equal(rnd(lo), lo)


def test_split_error_below_a_quarter_is_bounded():
    a = _all_bf16(-40, -2)                    # 2^-40 <= |a| < 1/4
    hi, lo = _split(a, O.e4m3_round)
    assert np.max(np.abs(hi + lo - a)) <= 2.0 ** -10


def test_power_of_two_scaling_reaches_the_range():
    """The per-block exponent e = 134 - E(amax) (E the biased bf16 exponent of
    the block's largest magnitude) puts amax * 2^e in [128, 256), exactly."""
    for amax in _all_bf16(-100, 100)[::97]:
        amax = abs(amax)
        E = int(np.floor(np.log2(amax))) + 127
        e = 134 - E
        assert 128 <= amax * 2.0 ** e < 256
