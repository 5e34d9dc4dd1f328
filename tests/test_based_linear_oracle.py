"""Pins for the oracle's Taylor linear attention (the Based linear branch; no GPU).

The kernel is checked through two routes (the closed form 1 + x + x^2/2 and the
dot product of the explicit features), the recurrent state form against the
parallel form at every position, and the properties of a normalised positive
kernel: weights non-negative and summing to one (a constant v comes back
unchanged), and the first position returning v_0.  Planted mistakes fail a pin."""
import math

import numpy as np
import pytest

import oracle


def rnd(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


def pin_feature_route(fwd_unused, feats, kern):
    q, k = rnd((7, 5), 1), rnd((9, 5), 2)
    for scale in (1.0, 0.3):
        np.testing.assert_allclose(feats(q, scale) @ feats(k, scale).T, kern(q, k, scale), rtol=1e-12, atol=1e-12)


def pin_closed_form_by_hand(fwd_unused, feats, kern):
    # d = 1: x = s q k; kappa = 1 + x + x^2/2
    got = kern(np.array([[2.0]]), np.array([[3.0]]), 0.5)[0, 0]
    assert got == pytest.approx(1 + 3.0 + 4.5)


def pin_recurrent_equals_parallel(fwd, feats, kern, state_fn=None, step_fn=None):
    B, L, H, d, dv, scale = 2, 23, 3, 4, 5, 0.5
    q, k, v = rnd((B, L, H, d), 3), rnd((B, L, H, d), 4), rnd((B, L, H, dv), 5)
    par = fwd(q, k, v, scale)
    F = 1 + d + d * d
    S, z = np.zeros((B, H, F, dv)), np.zeros((B, H, F))
    for t in range(L):
        out, S, z = oracle.based_linear_decode(q[:, t], k[:, t], v[:, t], S, z, scale)
        np.testing.assert_allclose(out, par[:, t], rtol=1e-10, atol=1e-10)
    S2, z2 = oracle.based_linear_state(k, v, scale)
    np.testing.assert_allclose(S, S2, rtol=1e-10, atol=1e-9)
    np.testing.assert_allclose(z, z2, rtol=1e-10, atol=1e-9)


def pin_convex_combination(fwd, feats, kern):
    q, k = rnd((1, 30, 2, 4), 6), rnd((1, 30, 2, 4), 7)
    v = np.full((1, 30, 2, 3), 0.75)
    np.testing.assert_allclose(fwd(q, k, v, 0.5), 0.75, rtol=1e-12)
    v = rnd((1, 30, 2, 3), 8)
    out = fwd(q, k, v, 0.5)
    np.testing.assert_allclose(out[:, 0], v[:, 0], rtol=1e-12)            # position 0 sees itself only
    lo, hi = np.minimum.accumulate(v, axis=1), np.maximum.accumulate(v, axis=1)
    assert (out >= lo - 1e-12).all() and (out <= hi + 1e-12).all()       # convex combination of the seen v


PINS = [pin_feature_route, pin_closed_form_by_hand, pin_recurrent_equals_parallel, pin_convex_combination]


@pytest.mark.parametrize("pin", PINS, ids=lambda f: f.__name__)
def test_oracle_meets_pin(pin):
    pin(oracle.based_linear_fwd, oracle.taylor_features, oracle.taylor_kernel)


def test_kernel_is_positive():
    x = np.linspace(-50, 50, 10001)
    assert (1 + x + x * x / 2 > 0).all()


# ----------------------------------------------------------------- planted mistakes
def feats_no_sqrt2(u, scale):
    f = oracle.taylor_features(u, scale)
    d = np.asarray(u).shape[-1]
    f[..., 1 + d:] *= math.sqrt(2.0)
    return f


def kern_no_constant(q, k, scale):
    return oracle.taylor_kernel(q, k, scale) - 1.0


def fwd_non_causal(q, k, v, scale):
    q, k, v = (np.asarray(t, dtype=np.float64) for t in (q, k, v))
    B, L, H, _ = q.shape
    out = np.zeros(v.shape)
    for b in range(B):
        for h in range(H):
            a = oracle.taylor_kernel(q[b, :, h], k[b, :, h], scale)
            out[b, :, h] = (a @ v[b, :, h]) / a.sum(axis=1, keepdims=True)
    return out


@pytest.mark.parametrize("mistake", ["no_sqrt2", "no_constant", "non_causal"])
def test_planted_mistake_fails_a_pin(mistake):
    fwd, feats, kern = oracle.based_linear_fwd, oracle.taylor_features, oracle.taylor_kernel
    if mistake == "no_sqrt2":
        feats = feats_no_sqrt2
    elif mistake == "no_constant":
        kern = kern_no_constant
    else:
        fwd = fwd_non_causal
    failed = []
    for pin in PINS:
        try:
            pin(fwd, feats, kern)
        except AssertionError:
            failed.append(pin.__name__)
    assert failed, mistake


def test_hand_worked_example():
    """tests/golden/hand_based_linear_d2.json: a two-token prefill and one decode step
    with dk = 2, dv = 1, worked by hand (the derivation is in the file)."""
    import json
    import os
    g = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "hand_based_linear_d2.json")))
    s = g["scale"]
    q = np.array(g["q"])[None, :, None, :]
    k = np.array(g["k"])[None, :, None, :]
    v = np.array(g["v"])[None, :, None, :]
    np.testing.assert_allclose(oracle.based_linear_fwd(q, k, v, s)[0, :, 0], g["out"], rtol=1e-14)
    S, z = oracle.based_linear_state(k, v, s)
    np.testing.assert_allclose(S[0, 0], g["S"], rtol=1e-14, atol=1e-14)
    np.testing.assert_allclose(z[0, 0], g["z"], rtol=1e-14, atol=1e-14)
    out, S2, z2 = oracle.based_linear_decode(np.array(g["q_next"])[None, None], np.array(g["k_next"])[None, None],
                                             np.array(g["v_next"])[None, None], S, z, s)
    np.testing.assert_allclose(out[0, 0], g["out_next"], rtol=1e-14)
    np.testing.assert_allclose(S2[0, 0], g["S_next"], rtol=1e-14, atol=1e-14)
    np.testing.assert_allclose(z2[0, 0], g["z_next"], rtol=1e-14, atol=1e-14)
