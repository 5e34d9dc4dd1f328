"""Pins for the fp64 oracle: nothing here retypes the oracle's own code.

Each check ties the oracle to something outside it:
  * torch's scaled_dot_product_attention (a library routine) given a dense
    boolean mask enumerated from the set definition of the visible keys
    ("Sliding-window beats linear attention", sections 1 and 3);
  * the library's own causal mode when the window covers the sequence;
  * closed forms (window 1, constant keys, hand-derived golden files);
  * invariants (weights non-negative and summing to one, permutation of the
    visible keys, sinks inside the window counted once).
"""
import json
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
import workloads

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def visible_literal(t, j, w, s):
    """The set definition, literally: key j is visible from query t."""
    return j <= t and (j >= t - w + 1 or j < s)


def dense_mask(L, w, s):
    return torch.tensor([[visible_literal(t, j, w, s) for j in range(L)] for t in range(L)])


def sdpa_masked(q, k, v, w, s, scale):
    """Library attention with a literal mask. q [L,Hq,d], k/v [L,Hkv,d] float64 tensors."""
    L, Hq, d = q.shape
    G = Hq // k.shape[1]
    kk = k.repeat_interleave(G, dim=1)        # query head h reads KV head h // G
    vv = v.repeat_interleave(G, dim=1)
    m = dense_mask(L, w, s)
    o = F.scaled_dot_product_attention(q.transpose(0, 1), kk.transpose(0, 1), vv.transpose(0, 1),
                                       attn_mask=m, scale=scale)
    return o.transpose(0, 1)


def lse_masked(q, k, w, s, scale):
    """log-sum-exp over visible scores via torch.logsumexp. Returns [L, Hq]."""
    L, Hq, d = q.shape
    G = Hq // k.shape[1]
    kk = k.repeat_interleave(G, dim=1)
    sc = torch.einsum("thc,jhc->htj", q, kk) * scale
    sc = sc.masked_fill(~dense_mask(L, w, s), float("-inf"))
    return torch.logsumexp(sc, dim=-1).transpose(0, 1)


def rand(shape, seed):
    g = torch.Generator().manual_seed(seed)
    return torch.randn(shape, generator=g, dtype=torch.float64)


@pytest.mark.parametrize("L", [1, 2, 5, 9, 16])
def test_brute_force_all_windows_and_sinks(L):
    Hq, Hkv, d = 4, 2, 3
    q, k, v = rand((L, Hq, d), 1), rand((L, Hkv, d), 2), rand((L, Hkv, d), 3)
    scale = 0.7
    for w in range(1, L + 2):
        for s in range(0, L + 1):
            ref = sdpa_masked(q, k, v, w, s, scale).numpy()
            ref_lse = lse_masked(q, k, w, s, scale).numpy()
            out, lse = oracle.swa_rows(q, list(range(L)), k, v, w, s, scale)
            np.testing.assert_allclose(out, ref, rtol=0, atol=1e-12, err_msg=f"w={w} s={s}")
            np.testing.assert_allclose(lse, ref_lse, rtol=0, atol=1e-12, err_msg=f"w={w} s={s}")


def test_window_covering_sequence_is_full_causal_attention():
    L, Hq, Hkv, d = 40, 6, 2, 8
    q, k, v = rand((1, L, Hq, d), 4), rand((1, L, Hkv, d), 5), rand((1, L, Hkv, d), 6)
    scale = 1 / math.sqrt(d)
    G = Hq // Hkv
    ref = F.scaled_dot_product_attention(
        q[0].transpose(0, 1), k[0].repeat_interleave(G, 1).transpose(0, 1),
        v[0].repeat_interleave(G, 1).transpose(0, 1), is_causal=True, scale=scale).transpose(0, 1)
    for w in (L, L + 1, 10 * L):
        out, _ = oracle.swa_fwd(q, k, v, w, 0, scale)
        np.testing.assert_allclose(out[0], ref.numpy(), rtol=0, atol=1e-12)


def test_window_one_returns_own_value():
    L, Hq, Hkv, d = 33, 4, 4, 16
    q, k, v = rand((1, L, Hq, d), 7), rand((1, L, Hkv, d), 8), rand((1, L, Hkv, d), 9)
    scale = 0.25
    out, lse = oracle.swa_fwd(q, k, v, 1, 0, scale)
    np.testing.assert_allclose(out[0], v[0].numpy(), rtol=0, atol=1e-13)
    own = scale * (q[0] * k[0]).sum(-1)                                 # [L, H]
    np.testing.assert_allclose(lse[0].T, own.numpy(), rtol=0, atol=1e-13)


@pytest.mark.parametrize("w,s", [(64, 4), (5, 0), (5, 3), (3, 7), (1, 2), (300, 4)])
def test_constant_keys_give_mean_of_visible_values(w, s):
    L, Hq, Hkv, d = 256, 2, 2, 4
    q, v = rand((1, L, Hq, d), 10), rand((1, L, Hkv, d), 11)
    k = torch.zeros(1, L, Hkv, d, dtype=torch.float64)
    out, lse = oracle.swa_fwd(q, k, v, w, s, 0.3)
    for t in range(L):
        vis = [j for j in range(L) if visible_literal(t, j, w, s)]
        np.testing.assert_allclose(out[0, t], v[0, vis].mean(0).numpy(), rtol=0, atol=1e-12)
        np.testing.assert_allclose(lse[0, :, t], math.log(len(vis)), rtol=0, atol=1e-12)
        assert oracle.visible_count(t, w, s) == len(vis)


def test_tiny_visible_count_total():
    # 256 rows, window 64, 4 sinks: sum over t of min(t+1, 64) = 14368 plus
    # 6 + 189*4 = 762 sink keys left of the window -> 15130 visible pairs per head.
    w = workloads.WORKLOADS["tiny"]
    total = sum(oracle.visible_count(t, w.window, w.n_sink) for t in range(w.L))
    assert total == 15130


def test_weights_are_a_distribution_on_the_visible_set():
    L, Hq, Hkv, d = 50, 4, 2, 8
    q, k, v = rand((L, Hq, d), 12), rand((L, Hkv, d), 13), rand((L, Hkv, d), 14)
    w_, s_, scale = 7, 3, 0.4
    out, _ = oracle.swa_rows(q, list(range(L)), k, v, w_, s_, scale)
    for t in (0, 1, 2, 5, 6, 9, 10, 30, 49):
        for h in range(Hq):
            wt = oracle.swa_weights(q[t], t, k, h, w_, s_, scale)
            assert (wt >= 0).all()
            assert abs(wt.sum() - 1) < 1e-14
            for j in range(L):
                if not visible_literal(t, j, w_, s_):
                    assert wt[j] == 0.0
                else:
                    assert wt[j] > 0.0
            np.testing.assert_allclose(wt @ v[:, h // 2].numpy(), out[t, h], rtol=0, atol=1e-13)


def test_permuting_visible_keys_leaves_rows_unchanged():
    L, Hq, Hkv, d = 60, 2, 1, 5
    q, k, v = rand((L, Hq, d), 15), rand((L, Hkv, d), 16), rand((L, Hkv, d), 17)
    w_, s_ = 9, 4
    rng = np.random.default_rng(0)
    for t in (3, 20, 59):
        vis = np.array([j for j in range(L) if visible_literal(t, j, w_, s_)])
        perm = vis[rng.permutation(len(vis))]
        k2, v2 = k.clone(), v.clone()
        k2[vis], v2[vis] = k[perm], v[perm]
        o1, l1 = oracle.swa_rows(q[t:t + 1], [t], k, v, w_, s_, 0.5)
        o2, l2 = oracle.swa_rows(q[t:t + 1], [t], k2, v2, w_, s_, 0.5)
        np.testing.assert_allclose(o1, o2, rtol=0, atol=1e-13)
        np.testing.assert_allclose(l1, l2, rtol=0, atol=1e-13)
        # and the result really depends on which keys are visible
        k3 = k.clone()
        k3[vis[0]] += 1.0
        o3, _ = oracle.swa_rows(q[t:t + 1], [t], k3, v, w_, s_, 0.5)
        assert np.abs(o3 - o1).max() > 1e-6


def test_sinks_inside_the_window_are_counted_once():
    L, Hq, Hkv, d = 40, 2, 2, 4
    q, k, v = rand((L, Hq, d), 18), rand((L, Hkv, d), 19), rand((L, Hkv, d), 20)
    w_ = 16
    o0, l0 = oracle.swa_rows(q, list(range(L)), k, v, w_, 0, 0.5)
    for s_ in (1, 4, 16, 40):
        o1, l1 = oracle.swa_rows(q, list(range(L)), k, v, w_, s_, 0.5)
        np.testing.assert_allclose(o1[:w_], o0[:w_], rtol=0, atol=0)      # rows t <= w-1
        np.testing.assert_allclose(l1[:w_], l0[:w_], rtol=0, atol=0)
        assert np.abs(o1[w_:] - o0[w_:]).max() > 1e-6


@pytest.mark.parametrize("name", ["hand_sinks_d1.json", "hand_gqa_d2.json"])
def test_golden_hand_examples(name):
    g = json.load(open(os.path.join(GOLDEN, name)))
    L, Hq, Hkv, d = g["L"], g["Hq"], g["Hkv"], g["d"]
    q = np.array(g["q"], dtype=np.float64).reshape(1, L, Hq, d)
    k = np.array(g["k"], dtype=np.float64).reshape(1, L, Hkv, d)
    v = np.array(g["v"], dtype=np.float64).reshape(1, L, Hkv, d)
    out, lse = oracle.swa_fwd(q, k, v, g["window"], g["n_sink"], g["scale"])
    np.testing.assert_allclose(out.reshape(-1), np.array(g["out"]).reshape(-1), rtol=0, atol=1e-14)
    np.testing.assert_allclose(lse[0].T.reshape(-1), np.array(g["lse"]).reshape(-1), rtol=0,
                               atol=1e-14)


def test_varlen_equals_each_sequence_alone():
    lens = [5, 1, 17, 9]
    cu = workloads.cu_seqlens_of(lens)
    Hq, Hkv, d = 4, 2, 8
    T = cu[-1]
    q, k, v = rand((T, Hq, d), 21), rand((T, Hkv, d), 22), rand((T, Hkv, d), 23)
    out, lse = oracle.swa_fwd_varlen(q, k, v, cu, 4, 2, 0.35)
    for i, n in enumerate(lens):
        a = cu[i]
        o, l_ = oracle.swa_fwd(q[None, a:a + n], k[None, a:a + n], v[None, a:a + n], 4, 2, 0.35)
        np.testing.assert_array_equal(out[a:a + n], o[0])
        np.testing.assert_array_equal(lse[:, a:a + n], l_[0])


def test_batched_fwd_matches_rows_and_lse_layout():
    B, L, Hq, Hkv, d = 3, 21, 4, 1, 6
    q, k, v = rand((B, L, Hq, d), 24), rand((B, L, Hkv, d), 25), rand((B, L, Hkv, d), 26)
    out, lse = oracle.swa_fwd(q, k, v, 6, 2, 0.4)
    for b in range(B):
        ref = sdpa_masked(q[b], k[b], v[b], 6, 2, 0.4).numpy()
        np.testing.assert_allclose(out[b], ref, rtol=0, atol=1e-12)
        np.testing.assert_allclose(lse[b].T, lse_masked(q[b], k[b], 6, 2, 0.4).numpy(), rtol=0,
                                   atol=1e-12)


def test_decode_oracle_is_prefill_row():
    B, P, Hq, Hkv, d = 2, 30, 4, 2, 8
    q, k, v = rand((B, P, Hq, d), 27), rand((B, P, Hkv, d), 28), rand((B, P, Hkv, d), 29)
    out, lse = oracle.swa_fwd(q, k, v, 8, 3, 0.5)
    pos = [29, 11]
    o, l_ = oracle.swa_decode(torch.stack([q[0, 29], q[1, 11]]), k, v, pos, 8, 3, 0.5)
    np.testing.assert_array_equal(o[0], out[0, 29])
    np.testing.assert_array_equal(o[1], out[1, 11])
    np.testing.assert_array_equal(l_[0], lse[0, :, 29])


def test_ring_model_holds_exactly_the_visible_keys():
    """After writing positions 0..p, the ring slots plus the sink slots that lie
    left of the window hold exactly the keys of S(p) (as a multiset)."""
    B, Hkv, d, w_, s_ = 1, 1, 1, 5, 2
    P = 23
    k = np.arange(P, dtype=np.float64).reshape(1, P, 1, 1) + 100.0
    kc = np.zeros((B, Hkv, w_, d))
    vc = np.zeros_like(kc)
    sk = np.zeros((B, Hkv, s_, d))
    sv = np.zeros_like(sk)
    for p in range(P):
        oracle.ring_append(kc, vc, sk, sv, k[:, p], k[:, p], [p], w_, s_)
        ring = [kc[0, 0, i, 0] for i in range(min(p + 1, w_))]
        sinks = [sk[0, 0, j, 0] for j in range(s_) if j < p - w_ + 1]
        got = sorted(ring + sinks)
        want = sorted(100.0 + j for j in range(P) if visible_literal(p, j, w_, s_))
        assert got == want, p
    kc2, _, sk2, _ = oracle.ring_fill(k, k, w_, s_)
    np.testing.assert_array_equal(kc2, kc)
    np.testing.assert_array_equal(sk2, sk)
