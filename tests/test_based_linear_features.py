"""The feature map the tensor-core prefill of the Based linear branch works in,
checked on the CPU against the oracle (no GPU, no CUDA code involved).

The kernel keeps each symmetric product once: features [sqrt(s) u (16), 1,
(s/sqrt(2)) u_a^2 and s u_a u_b for a < b (136, a-major)], 153 in all.  Its dot
products must equal the oracle's Taylor kernel 1 + x + x^2/2, and a state summed
in that basis must map back to the oracle's interface layout [1, linear, all 256
products] by copying the linear and constant rows and splitting each off-diagonal
row as row / sqrt(2) into (a, b) and (b, a)."""
import math

import numpy as np

import oracle

D = 16


def pairs():
    return [(a, b) for a in range(D) for b in range(a, D)]


def compact_features(u, s):
    u = np.asarray(u, np.float64)
    lin = math.sqrt(s) * u
    one = np.ones(u.shape[:-1] + (1,))
    prods = np.stack([(s / math.sqrt(2.0) if a == b else s) * u[..., a] * u[..., b] for a, b in pairs()], axis=-1)
    return np.concatenate([lin, one, prods], axis=-1)


def to_interface(Sc):
    """Compact state rows [..., 153, C] -> interface rows [..., 273, C]."""
    out = np.zeros(Sc.shape[:-2] + (1 + D + D * D, Sc.shape[-1]))
    out[..., 1:1 + D, :] = Sc[..., :D, :]
    out[..., 0, :] = Sc[..., D, :]
    for p, (a, b) in enumerate(pairs()):
        row = Sc[..., D + 1 + p, :]
        if a == b:
            out[..., 1 + D + D * a + a, :] = row
        else:
            out[..., 1 + D + D * a + b, :] = row / math.sqrt(2.0)
            out[..., 1 + D + D * b + a, :] = row / math.sqrt(2.0)
    return out


def test_feature_count():
    assert compact_features(np.zeros((1, D)), 0.25).shape[-1] == 153


def test_compact_features_reproduce_the_taylor_kernel():
    g = np.random.default_rng(4)
    q, k = g.standard_normal((9, D)), g.standard_normal((11, D))
    for s in (0.25, 0.1, 1.0):
        got = compact_features(q, s) @ compact_features(k, s).T
        np.testing.assert_allclose(got, oracle.taylor_kernel(q, k, s), rtol=1e-12, atol=1e-12)


def test_compact_state_maps_back_to_the_interface_layout():
    g = np.random.default_rng(5)
    B, L, H, dv, s = 2, 13, 3, 5, 0.25
    k, v = g.standard_normal((B, L, H, D)), g.standard_normal((B, L, H, dv))
    fk = compact_features(k, s)                                            # [B, L, H, 153]
    Sc = np.einsum("blhf,blhc->bhfc", fk, v)
    zc = fk.sum(axis=1)[..., None]
    S, z = oracle.based_linear_state(k, v, s)
    np.testing.assert_allclose(to_interface(Sc), S, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(to_interface(zc)[..., 0], z, rtol=1e-12, atol=1e-12)
