"""The software exponential the kernels run on the FMA pipes, checked on the
device against an fp64 reference: its error must stay within the bound its
derivation (derive_exp2_poly.py, Remez exchange) states, plus fp32 rounding."""
import numpy as np
import pytest
import torch

from token_level_sparse_causal_b200 import build, hs2

pytestmark = pytest.mark.gpu


def test_fma_exp2_within_derived_bounds():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    build.build()
    dev = torch.device("cuda:0")
    xs = np.concatenate([np.linspace(-125.0, 10.0, 2_000_001), np.linspace(-1.0, 1.0, 200_001),
                         -np.random.default_rng(0).random(100_000) * 60.0]).astype(np.float32)
    x = torch.from_numpy(xs).to(dev)
    y0, y3, y4 = torch.empty_like(x), torch.empty_like(x), torch.empty_like(x)
    hs2.hs2_exp2_check(x, y0, y3, y4)
    hs2.hs2_sync()
    ref = np.exp2(xs.astype(np.float64))
    rel = lambda y: np.abs(y.cpu().numpy().astype(np.float64) / ref - 1.0)
    slack = 4 * 2.0 ** -24          # fp32 rounding of the reduction, Horner steps and result
    assert rel(y3).max() <= 7.48e-5 + slack
    assert rel(y4).max() <= 2.642e-6 + slack
    assert rel(y0).max() <= 2.0 ** -21   # the hardware approximation itself, for comparison
