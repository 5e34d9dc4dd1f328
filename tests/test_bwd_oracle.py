"""Pins for the oracle's backward pass (no GPU).

The gradients are checked against torch autograd through the library's
scaled_dot_product_attention with the same boolean mask (float64), against
central finite differences of the oracle's own forward (C code, a different
implementation) on tiny inputs, and against identities: the value gradient
sums to the output gradient's column sums, and keys outside every row's
visible set get no gradient.  Planted mistakes each fail a pin."""
import math

import numpy as np
import pytest
import torch

import oracle


def rand(B, L, Hq, Hkv, d, seed):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(B, L, Hq, d, generator=g, dtype=torch.float64)
    k = torch.randn(B, L, Hkv, d, generator=g, dtype=torch.float64)
    v = torch.randn(B, L, Hkv, d, generator=g, dtype=torch.float64)
    do = torch.randn(B, L, Hq, d, generator=g, dtype=torch.float64)
    return q, k, v, do


def autograd_reference(q, k, v, do, window, n_sink, scale):
    q, k, v = (t.clone().requires_grad_(True) for t in (q, k, v))
    G = q.shape[2] // k.shape[2]
    mask = torch.from_numpy(oracle.visible_mask(q.shape[1], window, n_sink))
    kk = k.repeat_interleave(G, dim=2)
    vv = v.repeat_interleave(G, dim=2)
    out = torch.nn.functional.scaled_dot_product_attention(
        q.transpose(1, 2), kk.transpose(1, 2), vv.transpose(1, 2), attn_mask=mask, scale=scale)
    out.transpose(1, 2).backward(do)
    return q.grad.numpy(), k.grad.numpy(), v.grad.numpy()


def pin_autograd(bwd):
    for (B, L, Hq, Hkv, d, w, s) in [(2, 37, 4, 2, 8, 9, 3), (1, 50, 3, 1, 16, 50, 0), (1, 29, 2, 2, 4, 1, 5),
                                     (1, 64, 4, 4, 8, 16, 20)]:
        q, k, v, do = rand(B, L, Hq, Hkv, d, L + w)
        scale = 1 / math.sqrt(d)
        got = bwd(q, k, v, do, w, s, scale)
        want = autograd_reference(q, k, v, do, w, s, scale)
        for g_, w_, name in zip(got, want, ("dq", "dk", "dv")):
            np.testing.assert_allclose(g_, w_, atol=1e-10, err_msg=name)


def pin_finite_differences(bwd):
    # loss = sum(dO * out) through the C oracle's forward; central differences in each input
    B, L, Hq, Hkv, d, w, s = 1, 7, 2, 1, 3, 3, 2
    q, k, v, do = (t.numpy() for t in rand(B, L, Hq, Hkv, d, 5))
    scale = 0.7
    grads = bwd(q, k, v, do, w, s, scale)
    loss = lambda qq, kk, vv: float((oracle.swa_fwd(qq, kk, vv, w, s, scale)[0] * do).sum())
    eps = 1e-5
    for gi, arr in enumerate((q, k, v)):
        num = np.zeros_like(arr)
        for idx in np.ndindex(arr.shape):
            plus, minus = arr.copy(), arr.copy()
            plus[idx] += eps
            minus[idx] -= eps
            args_p = [q, k, v]
            args_m = [q, k, v]
            args_p[gi], args_m[gi] = plus, minus
            num[idx] = (loss(*args_p) - loss(*args_m)) / (2 * eps)
        np.testing.assert_allclose(grads[gi], num, atol=1e-7)


def pin_identities(bwd):
    q, k, v, do = rand(1, 40, 2, 2, 8, 7)
    dq, dk, dv = bwd(q, k, v, do, 6, 2, 0.5)
    # every row's weights sum to one, so the value gradient of a head sums to dO's column sums
    np.testing.assert_allclose(dv.sum(axis=1), do.numpy().sum(axis=1), atol=1e-10)
    # and each row's score gradient sums to zero, so dK summed over keys is scale * sum_t dS_t. q_t = 0
    assert np.abs(dk.sum(axis=1)).max() < 1e-10


PINS = [pin_autograd, pin_finite_differences, pin_identities]


@pytest.mark.parametrize("pin", PINS, ids=lambda f: f.__name__)
def test_oracle_bwd_meets_pin(pin):
    pin(oracle.swa_bwd)


def test_window_one_gradients():
    q, k, v, do = rand(1, 12, 2, 1, 4, 3)
    dq, dk, dv = oracle.swa_bwd(q, k, v, do, 1, 0, 0.3)
    # window 1: every row attends to itself with weight one, so out = v: dv = sum of dO over
    # the heads, and nothing depends on q or k
    np.testing.assert_allclose(dv[:, :, 0], do.numpy().sum(axis=2), atol=1e-12)
    assert np.abs(dq).max() < 1e-12 and np.abs(dk).max() < 1e-12


# ----------------------------------------------------------------- planted mistakes
def _variant(mistake):
    def bwd(q, k, v, dout, window, n_sink, scale):
        q, k, v, do = (oracle._f64(t) for t in (q, k, v, dout))
        B, L, Hq, d = q.shape
        Hkv = k.shape[2]
        G = Hq // Hkv
        M = oracle.visible_mask(L, window, n_sink)
        dq, dk, dv = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
        for b in range(B):
            for h in range(Hq):
                kh = (h % Hkv) if mistake == "gqa_interleaved" else h // G
                s = scale * (q[b, :, h] @ k[b, :, kh].T)
                s = np.where(M, s, -np.inf)
                p = np.exp(s - s.max(axis=1, keepdims=True))
                p /= p.sum(axis=1, keepdims=True)
                dp = do[b, :, h] @ v[b, :, kh].T
                corr = 0.0 if mistake == "no_row_term" else (p * dp).sum(axis=1, keepdims=True)
                ds = p * (dp - corr)
                sc = 1.0 if mistake == "no_scale" else scale
                dq[b, :, h] = sc * (ds @ k[b, :, kh])
                dk[b, :, kh] += sc * ((ds if mistake == "transposed" else ds.T) @ q[b, :, h])
                if mistake == "dv_overwrite":
                    dv[b, :, kh] = p.T @ do[b, :, h]
                else:
                    dv[b, :, kh] += p.T @ do[b, :, h]
        return dq, dk, dv
    return bwd


@pytest.mark.parametrize("mistake", ["gqa_interleaved", "no_row_term", "no_scale", "transposed", "dv_overwrite"])
def test_planted_mistake_fails_a_pin(mistake):
    bwd = _variant(mistake)
    failed = []
    for pin in PINS:
        try:
            pin(bwd)
        except AssertionError:
            failed.append(pin.__name__)
    assert failed, mistake
