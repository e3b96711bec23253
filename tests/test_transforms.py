"""Fold-time transforms on the CPU: double-norm removal (FlashNorm talk,
Proposal 3) against the oracle's two-norm chain."""
import numpy as np
import pytest
import torch

import oracle as O
from rmsnorm_linear_projection_flashnorm_b200 import transforms as TR


def _inputs(seed=3, M=6, d=64, N=32):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((M, d)) * np.exp(rng.uniform(np.log(0.1), np.log(10), (M, 1)))
    g = 1 + 0.1 * rng.standard_normal(d)
    W = rng.standard_normal((d, N)) / np.sqrt(d)
    return x, g, W


@pytest.mark.parametrize("c", [1.0, 0.25, 7.5, -2.0])
def test_merged_gain_reproduces_the_pair(c):
    x, g, W = _inputs()
    d = x.shape[1]
    merged = TR.double_norm_gain(torch.full((d,), c), torch.from_numpy(g)).numpy()
    # eps = 0: exact
    pair = O.norm_proj(O.rmsnorm(x, np.full(d, c), 0.0), g, W, 0.0)
    one = O.norm_proj(x, merged, W, 0.0)
    assert np.max(np.abs(pair - one) / (1 + np.abs(pair))) < 1e-12
    # eps > 0: within the first-order effect of eps on both norms
    eps = 1e-6
    pair = O.norm_proj(O.rmsnorm(x, np.full(d, c), eps), g, W, eps)
    one = O.norm_proj(x, merged, W, eps)
    ms = np.mean(x * x, axis=1, keepdims=True)
    assert np.all(np.abs(pair - one) <= (eps / ms + eps / c ** 2) * (np.abs(one) + 1e-12) * 2)


def test_non_scalar_first_gain_is_refused():
    x, g, W = _inputs()
    d = x.shape[1]
    with pytest.raises(ValueError):
        TR.double_norm_gain(torch.from_numpy(g), torch.from_numpy(g))
    with pytest.raises(ValueError):
        TR.double_norm_gain(torch.zeros(d), torch.from_numpy(g))
    with pytest.raises(ValueError):
        TR.double_norm_gain(torch.ones(d + 1), torch.from_numpy(g))
    # and the refusal is right: with a non-scalar first gain the pair differs from any single norm
    pair = O.norm_proj(O.rmsnorm(x, g, 0.0), g, W, 0.0)
    one = O.norm_proj(x, g, W, 0.0)
    assert np.max(np.abs(pair - one)) > 1e-3
