"""CPU checks of the O comparison used by the GPU parity tests: the 16-bit
output's own rounding (half a unit in the last place of the value's binade)
is allowed on top of the 1e-2 bound, and nothing more."""
import numpy as np
import torch

from parity_utils import TOL_BF16, half_ulp, o_error


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
    # 3.0 lies in [2, 4): half a unit is 2^-7, half of the old |x| * 2^-8 allowance
    bad_large = x + np.array([0.0, 0.0, 1e-2 + 2.0 ** -7 + 1e-6])
    assert o_error(bad_large, x) > TOL_BF16["o"]
    assert o_error(x, x, dtype="fp32") == 0.0


def test_half_ulp_is_the_largest_rounding_error_of_each_binade():
    rng = np.random.default_rng(7)
    for dtype, tdt in (("bf16", torch.bfloat16), ("fp16", torch.float16)):
        x = np.concatenate([rng.uniform(-9, 9, 20000), rng.uniform(-1e-3, 1e-3, 2000),
                            2.0 ** np.arange(-6, 4)])
        # fp32 values, as the kernels round from fp32 (a float64 -> 16-bit
        # conversion may pass through fp32 and round twice)
        x = x.astype(np.float32).astype(np.float64)
        r = torch.tensor(x, dtype=torch.float64).to(tdt).double().numpy()
        err = np.abs(r - x)
        hu = half_ulp(x, dtype)
        assert (err <= hu + 1e-300).all()
        # and it is tight: some values in each sampled binade round by nearly that much
        big = np.abs(x) >= 1.0
        assert (err[big] / hu[big]).max() > 0.99
    # exact values of the bound
    assert half_ulp(np.array([1.0, 1.99, 4.0, 7.9]), "bf16").tolist() == [2.0 ** -8, 2.0 ** -8, 2.0 ** -6, 2.0 ** -6]
    assert half_ulp(np.array([1.0, 3.0]), "fp16").tolist() == [2.0 ** -11, 2.0 ** -10]
    assert half_ulp(np.array([2.0 ** -20]), "fp16")[0] == 2.0 ** -25
    assert half_ulp(np.array([0.0]))[0] == 0.0
