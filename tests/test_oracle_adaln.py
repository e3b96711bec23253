"""Pins for the oracle's AdaLN-modulated norm + projection (the "RMSNorm +
AdaLN" front of the fused FC1 on the FlashInfer PR #5521 analysis: the norm
weight, an AdaLN scale, an AdaLN shift and a per-token index), run on the CPU.

Each check ties the oracle to something other than itself: explicit-loop
brute force with math.fsum on tiny inputs, closed forms (a zero row sees only
its shift; unit scale and zero shift give the plain norm), the deferred split
the kernels compute (scale on the raw activations, the 1/rms scalar after the
matmul, the shift as a bias through the unfolded weight) agreeing to 1e-12,
scale invariance at eps = 0, and row permutation.  The planted-mistake tests
show that a shift applied before the norm, a dropped scale, the gain
multiplying the shift, or a wrong index all fail them.
"""
import math

import numpy as np
import pytest

import oracle as O
import oracle.flashnorm_oracle as OF
import workloads as WL


def _case(M=4, d=8, N=8, n_cond=3, seed=0):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((M, d)) * rng.uniform(0.1, 10, (M, 1))
    g = 1.0 + 0.1 * rng.standard_normal(d)
    W = rng.standard_normal((d, N)) / math.sqrt(d)
    W2 = rng.standard_normal((d, N)) / math.sqrt(d)
    scale = 1.0 + 0.3 * rng.standard_normal((n_cond, d))
    shift = 0.5 * rng.standard_normal((n_cond, d))
    index = rng.integers(0, n_cond, M)
    return x, g, W, W2, scale, shift, index


def _brute(x, g, W, eps, scale, shift, index):
    M, d = x.shape
    N = W.shape[1]
    out = np.zeros((M, N))
    for m in range(M):
        ms = math.fsum(x[m, k] * x[m, k] for k in range(d)) / d
        r = 1.0 / math.sqrt(ms + eps)
        c = int(index[m])
        h = [x[m, k] * r * g[k] * scale[c, k] + shift[c, k] for k in range(d)]
        for n in range(N):
            out[m, n] = math.fsum(h[k] * W[k, n] for k in range(d))
    return out


@pytest.mark.parametrize("eps", [0.0, 1e-6, 0.5])
def test_adaln_brute_force(eps):
    x, g, W, W2, scale, shift, index = _case(seed=1)
    want = _brute(x, g, W, eps, scale, shift, index)
    got = O.norm_proj_adaln(x, g, W, eps, scale, shift, index)
    assert np.max(np.abs(got - want) / (1 + np.abs(want))) <= 1e-14


def test_adaln_swiglu_brute_force():
    x, g, W, W2, scale, shift, index = _case(seed=2)
    a = _brute(x, g, W, 1e-6, scale, shift, index)
    b = _brute(x, g, W2, 1e-6, scale, shift, index)
    want = np.array([[ai / (1 + math.exp(-ai)) * bi for ai, bi in zip(ra, rb)] for ra, rb in zip(a, b)])
    got = O.norm_proj_adaln_swiglu(x, g, W, W2, 1e-6, scale, shift, index)
    assert np.max(np.abs(got - want) / (1 + np.abs(want))) <= 1e-13


def test_adaln_zero_row_sees_only_its_shift():
    x, g, W, W2, scale, shift, index = _case(M=5, seed=3)
    x[2] = 0.0
    y = O.norm_proj_adaln(x, g, W, 1e-6, scale, shift, index)
    want = np.array([math.fsum(shift[index[2], k] * W[k, n] for k in range(W.shape[0])) for n in range(W.shape[1])])
    assert np.max(np.abs(y[2] - want)) <= 1e-14


def test_adaln_unit_scale_zero_shift_is_the_plain_norm():
    x, g, W, W2, scale, shift, index = _case(M=6, d=16, N=12, seed=4)
    y = O.norm_proj_adaln(x, g, W, 1e-6, np.ones_like(scale), np.zeros_like(shift), index)
    want = _brute(x, g, W, 1e-6, np.ones_like(scale), np.zeros_like(shift), index)
    assert np.max(np.abs(y - want) / (1 + np.abs(want))) <= 1e-14
    assert np.max(np.abs(y - O.norm_proj(x, g, W, 1e-6)) / (1 + np.abs(y))) <= 1e-14


@pytest.mark.parametrize("eps", [0.0, 1e-6])
def test_adaln_deferred_split(eps):
    """The form the kernels compute: the scale on the raw activations, the
    folded weight, 1/rms after the matmul, the shift as a per-condition bias
    through the unfolded weight."""
    inp = WL.case(16, 256, 128, False, seed=5)
    x, g, W = O.to_f64(inp["x"]), O.to_f64(inp["g"]), O.to_f64(inp["W"])
    rng = np.random.default_rng(5)
    scale = 1.0 + 0.3 * rng.standard_normal((4, 256))
    shift = 0.5 * rng.standard_normal((4, 256))
    index = rng.integers(0, 4, 16)
    y = O.norm_proj_adaln(x, g, W, eps, scale, shift, index)
    r = O.rms_inv(x, eps)
    B = O.adaln_shift_bias(shift, W)
    deferred = r[:, None] * ((x * scale[index]) @ (g[:, None] * W)) + B[index]
    assert np.max(np.abs(y - deferred) / (1 + np.abs(y))) <= 1e-12


def test_adaln_scale_invariance_at_eps_zero():
    """The modulation follows the norm, so scaling a row of x by a > 0 leaves
    its output unchanged (exactly at eps = 0)."""
    x, g, W, W2, scale, shift, index = _case(M=6, d=16, N=12, seed=6)
    y = O.norm_proj_adaln(x, g, W, 0.0, scale, shift, index)
    for a in (1e-3, 0.5, 3.0, 1e3):
        ya = O.norm_proj_adaln(a * x, g, W, 0.0, scale, shift, index)
        assert np.max(np.abs(ya - y) / (1 + np.abs(y))) <= 1e-12


def test_adaln_rows_permute_with_their_index():
    x, g, W, W2, scale, shift, index = _case(M=7, d=16, N=12, seed=7)
    perm = np.random.default_rng(7).permutation(7)
    y = O.norm_proj_adaln(x, g, W, 1e-6, scale, shift, index)
    yp = O.norm_proj_adaln(x[perm], g, W, 1e-6, scale, shift, index[perm])
    assert np.array_equal(yp, y[perm])


def test_adaln_scaled_operand_matches_torch_casts():
    """fp32 product then one round-to-nearest-even to bf16, checked against
    torch's own fp32 multiply and bf16 cast on the CPU."""
    import torch
    x = WL.activations(8, 256, 9)
    rng = np.random.default_rng(9)
    scale = (1.0 + 0.3 * rng.standard_normal((3, 256))).astype(np.float32)
    index = rng.integers(0, 3, 8)
    want = (x.float() * torch.from_numpy(scale)[torch.from_numpy(index)]).to(torch.bfloat16).double().numpy()
    assert np.array_equal(O.adaln_scaled_operand(x, scale, index), want)


@pytest.mark.parametrize("mistake", ["shift_before_norm", "scale_dropped", "gain_on_shift", "index_off_by_one"])
def test_adaln_planted_mistakes_are_caught(mistake, monkeypatch):
    def wrong(x, g, eps, scale, shift, index):
        idx = np.asarray(index, dtype=np.int64)
        sc, sh = O.to_f64(scale), O.to_f64(shift)
        if mistake == "shift_before_norm":
            return O.rmsnorm(O.to_f64(x) + sh[idx], g, eps) * sc[idx]
        if mistake == "scale_dropped":
            return O.rmsnorm(x, g, eps) + sh[idx]
        if mistake == "gain_on_shift":
            return (O.rmsnorm(x, np.ones(len(g)), eps) * sc[idx] + sh[idx]) * O.to_f64(g)
        return O.rmsnorm(x, g, eps) * sc[(idx + 1) % sc.shape[0]] + sh[(idx + 1) % sc.shape[0]]
    monkeypatch.setattr(OF, "adaln_modulate", wrong)
    with pytest.raises(AssertionError):
        test_adaln_brute_force(1e-6)
