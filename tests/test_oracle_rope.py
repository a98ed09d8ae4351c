"""Pins for the oracle's RoPE (rotate-half pairs (i, i+d/2), theta_i =
base^(-2i/d)).  Each test checks a fact that holds independently of how the
oracle computes the rotation: identity at position 0, norm preservation,
the relative-position property, a complex-number formulation written with
numpy, the inverse rotation, and the unit-circle special case."""
import numpy as np
import pytest

import oracle


def _complex_rope(x, pos, base):
    """(x_i + i x_{i+d/2}) * exp(i * pos * base^(-2i/d)), independent numpy form."""
    d = x.shape[-1]
    h = d // 2
    z = x[..., :h] + 1j * x[..., h:]
    freqs = np.power(float(base), -np.arange(0, d, 2, dtype=np.float64) / d)
    z = z * np.exp(1j * pos * freqs)
    return np.concatenate([z.real, z.imag], axis=-1)


@pytest.mark.parametrize("d,base", [(64, 1e4), (128, 5e5), (8, 10.0)])
def test_position_zero_is_identity_bit_exact(d, base):
    x = np.random.default_rng(0).standard_normal((5, d))
    assert np.array_equal(oracle.rope(x, 0, base), x)


@pytest.mark.parametrize("pos", [1, 17, 4096, 131072])
def test_pair_norms_preserved(pos):
    d = 128
    x = np.random.default_rng(pos).standard_normal((4, d))
    y = oracle.rope(x, pos, 5e5)
    h = d // 2
    n_in = x[:, :h] ** 2 + x[:, h:] ** 2
    n_out = y[:, :h] ** 2 + y[:, h:] ** 2
    assert np.allclose(n_out, n_in, rtol=1e-12, atol=0)


def test_relative_position_property():
    rng = np.random.default_rng(3)
    d, base = 128, 5e5
    q, k = rng.standard_normal(d), rng.standard_normal(d)
    m, n = 1000, 37
    ref = oracle.rope(q, m, base) @ oracle.rope(k, n, base)
    for shift in (1, 250, 9999):
        got = oracle.rope(q, m + shift, base) @ oracle.rope(k, n + shift, base)
        assert abs(got - ref) <= 1e-9 * max(1.0, abs(ref))


@pytest.mark.parametrize("d,base,pos", [(64, 1e4, 255), (128, 5e5, 100_000), (128, 5e5, 3)])
def test_matches_complex_formulation(d, base, pos):
    x = np.random.default_rng(d + pos).standard_normal((3, d))
    # the angle pos * theta_i carries ~pos * 2^-52 of rounding from theta_i
    # (library pow vs C pow may differ by an ulp), so the bound grows with pos
    assert np.allclose(oracle.rope(x, pos, base), _complex_rope(x, pos, base),
                       rtol=0, atol=1e-13 + 2e-15 * pos)


def test_inverse_rotation_recovers_input():
    x = np.random.default_rng(9).standard_normal((2, 128))
    y = oracle.rope(oracle.rope(x, 54321, 5e5), -54321, 5e5)
    assert np.allclose(y, x, rtol=0, atol=1e-12)


@pytest.mark.parametrize("pos", [1, 2, 7, 1000])
def test_unit_circle_first_pair(pos):
    # d = 2: one pair with theta_0 = base^0 = 1, so (1, 0) goes to (cos p, sin p)
    y = oracle.rope(np.array([1.0, 0.0]), pos, 1e4)
    assert np.allclose(y, [np.cos(pos), np.sin(pos)], rtol=0, atol=1e-15)


def test_frequency_schedule_per_pair():
    # only pair i nonzero: its rotation angle is pos * base^(-2i/d) (mod 2 pi)
    d, base, pos = 16, 100.0, 3
    for i in range(d // 2):
        x = np.zeros(d)
        x[i] = 1.0
        y = oracle.rope(x, pos, base)
        ang = np.arctan2(y[i + d // 2], y[i])
        want = np.angle(np.exp(1j * pos * base ** (-2.0 * i / d)))
        assert abs(ang - want) < 1e-13
        others = np.delete(y, [i, i + d // 2])
        assert not others.any()
