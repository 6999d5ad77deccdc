"""CPU checks of the comparison helpers the chained recurrent-core tests use:
the bf16 ulp against torch's own bf16 spacing, the chain allowance's
recursion, and the rounding-noise allowance's scale."""
import numpy as np
import torch

from parity import bf16_ulp, chain_allowance, rounding_noise_allowance


def test_bf16_ulp_is_the_spacing_of_bf16_values():
    rng = np.random.default_rng(0)
    v = np.concatenate([rng.standard_normal(2000) * 10.0 ** rng.integers(-6, 4, 2000),
                        [1.0, 2.0, 0.5, 3.999, -7.0, 2.0 ** -20]])
    t = torch.tensor(np.abs(v), dtype=torch.float32).to(torch.bfloat16)
    up = torch.nextafter(t, torch.full_like(t, float("inf")))
    spacing = (up.float() - t.float()).numpy().astype(np.float64)
    # the rounded value's binade (a value just below a power of two may round up into the next)
    assert np.array_equal(bf16_ulp(t.float().numpy()), spacing)


def test_chain_allowance_adds_one_ulp_per_rounding_twice():
    u = [np.full(3, 1.5), np.full(3, 1.5)]
    # A1 = ulp(1.5) = 2^-7; A2 = A1 + ulp(1.5 + 2 A1) = 2 * 2^-7; allowance 2 * A2
    assert np.allclose(chain_allowance(u), 4 * 2.0 ** -7)
    # an element that grows into the next binade takes that binade's ulp
    a = chain_allowance([np.array([1.99]), np.array([1.99])])
    assert a[0] == 2 * (2.0 ** -7 + 2.0 ** -6)


def test_rounding_noise_allowance_scales_with_the_noise():
    r = np.zeros((4, 4))
    e = np.full((4, 4), 1e-3)
    assert np.isclose(rounding_noise_allowance(r, e), 6 * np.sqrt(2) * 1e-3)
    assert rounding_noise_allowance(r, r) == 0.0
