"""CPU checks of the O comparison used by the GPU parity tests: the bf16
output's own rounding is allowed on top of the 1e-2 bound, and nothing more."""
import numpy as np
import torch

from parity_utils import TOL_BF16, o_error


def _bf16(x):
    return torch.tensor(x, dtype=torch.float64).to(torch.bfloat16).double().numpy()


def test_exactly_rounded_bf16_output_can_exceed_the_absolute_bound():
    # a value just below the midpoint of two bf16 neighbours near 4 (spacing 2^-5)
    x = np.array([4.0 + 0.5 * 2.0 ** -5 - 1e-6, -5.99])
    r = _bf16(x)
    assert np.abs(r - x).max() > TOL_BF16["o"]         # the literal bound fails...
    assert o_error(r, x) <= 0.0                        # ...on pure output rounding


def test_real_errors_are_not_hidden():
    x = np.array([0.5, -0.25, 3.0])
    bad = x + np.array([0.0, 2e-2, 0.0])
    assert o_error(bad, x) > TOL_BF16["o"]
    bad_large = x + np.array([0.0, 0.0, 2e-2 + 3.0 * 2.0 ** -8])
    assert o_error(bad_large, x) > TOL_BF16["o"] - 1e-12
    assert o_error(x, x, dtype="fp32") == 0.0
