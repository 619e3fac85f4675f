"""The experts' elementwise activations on the GPU against fp64 references.

GELU is the exact erf form (erf by Abramowitz & Stegun 7.1.26, absolute
error <= 1.5e-7 for the formula, rearranged as max(x, 0) - 0.5|x| P(t)
exp(-x^2/2) and evaluated on packed fp32x2 arithmetic, two values per
call: |GELU error| <= 4e-7 max(1, |x|)); SiLU is x / (1 + exp(-x)). The
inputs have odd and even lengths, so both halves of the packed pair and a
lone tail element are exercised.
"""

import numpy as np
import pytest
import torch
from scipy.special import expit, ndtr

pytestmark = pytest.mark.gpu


def _run(act, x64):
    from mixture_experts_layer_33_b200 import moe
    x = torch.tensor(x64, dtype=torch.float32, device="cuda")
    y = torch.empty_like(x)
    moe.activation(x, y, act)
    torch.cuda.synchronize()
    return x.double().cpu().numpy(), y.double().cpu().numpy()


def test_gelu_matches_exact_erf_form():
    from mixture_experts_layer_33_b200 import moe
    x64 = np.concatenate([np.linspace(-12, 12, 200001), [0.0, -0.0, 1e-30, -1e-30, 40.0, -40.0]])
    x, y = _run(moe.GELU_ERF, x64)
    ref = x * ndtr(x)
    # 0.5*|x| times the fp32-evaluated erf error (< 6e-7, with margin for the
    # hardware exponential), plus a few fp32 ulps of |y|.
    bound = 0.5 * np.abs(x) * 1e-6 + 4 * np.finfo(np.float32).eps * np.abs(ref) + 1e-30
    assert np.all(np.abs(y - ref) <= bound)
    assert y[-2] == 40.0 and y[-1] == 0.0
    # Odd length: the last element runs alone in its pair.
    x, y = _run(moe.GELU_ERF, x64[:-1])
    ref = x * ndtr(x)
    bound = 0.5 * np.abs(x) * 1e-6 + 4 * np.finfo(np.float32).eps * np.abs(ref) + 1e-30
    assert np.all(np.abs(y - ref) <= bound)
    assert y[-1] == 40.0


def test_gelu_in_place():
    from mixture_experts_layer_33_b200 import moe
    x64 = np.linspace(-6, 6, 1001)
    x = torch.tensor(x64, dtype=torch.float32, device="cuda")
    y = torch.empty_like(x)
    moe.activation(x, y, moe.GELU_ERF)
    moe.activation(x, x, moe.GELU_ERF)
    torch.cuda.synchronize()
    assert torch.equal(x, y)


def test_silu_matches_definition():
    from mixture_experts_layer_33_b200 import moe
    x64 = np.linspace(-80, 80, 160001)
    x, y = _run(moe.SWIGLU, x64)
    ref = x * expit(x)
    assert np.all(np.abs(y - ref) <= 8 * np.finfo(np.float32).eps * np.abs(ref) + 1e-37)
