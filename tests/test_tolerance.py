"""CPU checks of the attention acceptance bound used by the GPU parity tests: the
half-ulp term is the actual bf16 rounding error, and the bound is the stated 2e-2 wherever
a bf16 output can meet it."""
import numpy as np
import torch

from helpers import ATOL, F16_BUDGET, attention_bound, half_ulp_bf16


def test_half_ulp_bounds_bf16_rounding_and_is_attained():
    rng = np.random.default_rng(3)
    x = (rng.standard_normal(200_000) * np.exp2(rng.integers(-10, 12, 200_000))).astype(np.float32)
    r = torch.from_numpy(x).to(torch.bfloat16).float().numpy().astype(np.float64)
    err = np.abs(r - x.astype(np.float64))
    h = half_ulp_bf16(x)
    assert (err <= h).all()
    # ties land exactly on the half ulp: 1 + 2^-8 rounds to 1 (even), error = 2^-8
    assert half_ulp_bf16(np.array([1.0 + 2.0 ** -8]))[0] == 2.0 ** -8
    assert np.isclose((err / h).max(), 1.0, rtol=1e-2)


def test_bound_is_the_stated_absolute_value_below_four():
    ref = np.linspace(-3.999, 3.999, 10_001)
    assert (attention_bound(ref) == ATOL).all()


def test_bound_above_four_is_output_rounding_plus_f16_budget():
    for v, expect in ((4.0, max(ATOL, 2.0 ** -6 + 4 * F16_BUDGET)),
                      (7.99, 2.0 ** -6 + 7.99 * F16_BUDGET),
                      (8.0, 2.0 ** -5 + 8 * F16_BUDGET),
                      (-20.0, 2.0 ** -4 + 20 * F16_BUDGET)):
        assert np.isclose(attention_bound(np.array([v]))[0], expect, rtol=0, atol=1e-15)
    # never looser than 5e-3 relative, the old rule's slope, anywhere from 4 up
    ref = np.exp2(np.linspace(2, 8, 5000))
    assert (attention_bound(ref) <= np.maximum(ATOL, 5e-3 * ref) + 1e-15).all()
