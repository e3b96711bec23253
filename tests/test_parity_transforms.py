"""GPU check of the double-norm removal transform (FlashNorm talk, Proposal 3):
the merged norm folded into W and run by the fused call on the raw input
matches the oracle's two-norm chain on the original (unfolded) weight."""
import numpy as np
import pytest
import torch

import oracle as O
import rmsnorm_linear_projection_flashnorm_b200 as fnb
import workloads as WL
from rmsnorm_linear_projection_flashnorm_b200 import torch_api as T
from rmsnorm_linear_projection_flashnorm_b200 import transforms as TR
from tests._util import BF16_TOL, gpu, rel_err

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    fnb.build()
    fnb.lib()
    torch.cuda.init()
    yield


@pytest.mark.parametrize("M,c", [(8, 0.5), (200, -3.0)])
def test_double_norm_removal(M, c):
    d, N = 512, 384
    inp = WL.case(M, d, N, False, seed=601)
    x, g, W, eps = inp["x"], inp["g"], inp["W"], inp["eps"]
    Wp, _ = TR.fold_double_norm(gpu(W), torch.full((d,), c), gpu(g))
    y = T.norm_proj(gpu(x), Wp, N, eps)
    torch.cuda.synchronize()
    ref = O.norm_proj(O.rmsnorm(x, np.full(d, c), eps), g, W, eps)
    assert rel_err(y.cpu(), ref) <= BF16_TOL
