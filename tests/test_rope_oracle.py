"""Pins for the oracle's rotary position encoding (no GPU).

The rotation is checked against complex multiplication (a different route to
the same closed form), hand-evaluated angles at small d with a chosen base,
and the properties that define a rotary encoding: position 0 is the identity,
each pair keeps its length, rotations compose additively, and the product of a
rotated query and key depends only on the distance of their positions.  Four
plausible mistakes planted in copies of the rotation each fail a pin."""
import cmath
import math

import numpy as np
import pytest

import oracle


def pin_identity(rope):
    x = np.random.default_rng(0).standard_normal((3, 2, 16))
    np.testing.assert_array_equal(rope(x, [0, 0, 0]), x)


def pin_complex(rope):
    # d = 2: one pair (x0, x1) with theta_0 = base^0 = 1, so the rotation is
    # multiplication of x0 + i x1 by e^{i p}, whatever the base
    x0, x1 = 0.3, -1.7
    for p in (0, 1, 5, 1000, 131071):
        z = complex(x0, x1) * cmath.exp(1j * p)
        got = rope(np.array([[x0, x1]]), [p], base=12345.0)[0]
        assert got[0] == pytest.approx(z.real, abs=1e-12)
        assert got[1] == pytest.approx(z.imag, abs=1e-12)


def pin_d4_by_hand(rope):
    # d = 4, base 100: pairs (x0, x2) with theta 1 and (x1, x3) with theta 100^(-1/2) = 0.1
    x = np.array([[1.0, 2.0, 3.0, 4.0]])
    a0, a1 = 3.0, 0.3                                           # position 3
    want = [1 * math.cos(a0) - 3 * math.sin(a0), 2 * math.cos(a1) - 4 * math.sin(a1),
            1 * math.sin(a0) + 3 * math.cos(a0), 2 * math.sin(a1) + 4 * math.cos(a1)]
    np.testing.assert_allclose(rope(x, [3], base=100.0)[0], want, atol=1e-12)


def pin_pair_length(rope):
    rng = np.random.default_rng(1)
    x = rng.standard_normal((50, 4, 64))
    y = rope(x, rng.integers(0, 100000, 50))
    np.testing.assert_allclose(y[..., :32] ** 2 + y[..., 32:] ** 2, x[..., :32] ** 2 + x[..., 32:] ** 2,
                               rtol=1e-12)


def pin_compose(rope):
    rng = np.random.default_rng(2)
    x = rng.standard_normal((20, 128))
    a, b = rng.integers(0, 5000, 20), rng.integers(0, 5000, 20)
    np.testing.assert_allclose(rope(rope(x, a), b), rope(x, a + b), atol=1e-9)


def pin_relative(rope):
    rng = np.random.default_rng(3)
    q, k = rng.standard_normal((1, 128)), rng.standard_normal((1, 128))
    ref = (rope(q, [700]) * rope(k, [650])).sum()
    for shift in (1, 17, 4096, 100000):
        assert (rope(q, [700 + shift]) * rope(k, [650 + shift])).sum() == pytest.approx(ref, abs=1e-9)
    assert (rope(q, [701]) * rope(k, [650])).sum() != pytest.approx(ref, abs=1e-6)


PINS = [pin_identity, pin_complex, pin_d4_by_hand, pin_pair_length, pin_compose, pin_relative]


@pytest.mark.parametrize("pin", PINS, ids=lambda f: f.__name__)
def test_oracle_rope_meets_pin(pin):
    pin(oracle.rope)


def test_rejects_odd_d():
    with pytest.raises(ValueError):
        oracle.rope(np.zeros((1, 3)), [1])


# ----------------------------------------------------------------- planted mistakes
def _rot(x, ang, lo_idx, hi_idx, sign=1.0):
    x = np.asarray(x, dtype=np.float64)
    shape = (x.shape[0],) + (1,) * (x.ndim - 2) + (ang.shape[1],)
    c, s = np.cos(ang).reshape(shape), sign * np.sin(ang).reshape(shape)
    out = x.copy()
    lo, hi = x[..., lo_idx], x[..., hi_idx]
    out[..., lo_idx] = lo * c - hi * s
    out[..., hi_idx] = lo * s + hi * c
    return out


def mutant_interleaved(x, positions, base=10000.0):
    d = np.asarray(x).shape[-1]
    return _rot(x, oracle.rope_angles(positions, d, base), np.arange(0, d, 2), np.arange(1, d, 2))


def mutant_sign(x, positions, base=10000.0):
    d = np.asarray(x).shape[-1]
    return _rot(x, oracle.rope_angles(positions, d, base), np.arange(d // 2), np.arange(d // 2, d), -1.0)


def mutant_exponent(x, positions, base=10000.0):
    d = np.asarray(x).shape[-1]
    p = np.asarray(positions, dtype=np.float64).reshape(-1)
    ang = p[:, None] * np.power(base, -np.arange(d // 2) / d)[None, :]
    return _rot(x, ang, np.arange(d // 2), np.arange(d // 2, d))


def mutant_relative_position(x, positions, base=10000.0):
    # positions counted from the first one given (re-indexed) instead of absolute
    p = np.asarray(positions).reshape(-1)
    return oracle.rope(x, p - p.min(), base)


@pytest.mark.parametrize("mutant", [mutant_interleaved, mutant_sign, mutant_exponent,
                                    mutant_relative_position], ids=lambda f: f.__name__)
def test_planted_mistake_fails_a_pin(mutant):
    failed = []
    for pin in PINS:
        try:
            pin(mutant)
        except AssertionError:
            failed.append(pin.__name__)
    assert failed, f"{mutant.__name__} passed every pin"
