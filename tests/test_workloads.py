"""Seeded input recipes: determinism, shapes and the sink-key bias."""
import math

import torch

import workloads
from workloads import WORKLOADS


def test_prefill_inputs_are_deterministic_and_rounded():
    w = WORKLOADS["gqa8b_prefill"]
    a = workloads.make_prefill(w, L=300)
    b = workloads.make_prefill(w, L=300)
    for x, y in zip(a, b):
        assert x.dtype == torch.bfloat16
        assert torch.equal(x, y)
    q, k, v = a
    assert q.shape == (1, 300, 32, 128) and k.shape == (1, 300, 8, 128) and v.shape == k.shape


def test_tiny_stays_fp32():
    q, k, v = workloads.make_prefill(WORKLOADS["tiny"])
    assert q.dtype == torch.float32 and q.shape == (1, 256, 2, 64)


def test_sink_bias_raises_sink_score_spread():
    """With the bias, scaled scores of the sink keys spread about sqrt(5) times
    wider than those of ordinary keys (variance 1 + 4 along the query mean)."""
    w = WORKLOADS["gqa8b_prefill"]
    q, k, _ = workloads.make_prefill(w, L=2048, dtype="f32")
    G = w.G
    s_sink, s_other = [], []
    for kvh in range(w.Hkv):
        qq = q[0, :, kvh * G:(kvh + 1) * G].reshape(-1, w.d)
        s_sink.append((qq @ k[0, :w.n_sink, kvh].T).flatten() * w.scale)
        s_other.append((qq @ k[0, 100:104, kvh].T).flatten() * w.scale)
    r = torch.cat(s_sink).std() / torch.cat(s_other).std()
    assert 1.8 < r < 2.7, r


def test_unbiased_workload_untouched():
    w = WORKLOADS["based_local"]
    q, k, v = workloads.make_prefill(w, B=1, L=64, dtype="f32")
    g = torch.Generator().manual_seed(0)
    q0 = torch.randn(1, 64, 16, 64, generator=g)
    k0 = torch.randn(1, 64, 16, 64, generator=g)
    assert torch.equal(q, q0) and torch.equal(k, k0)


def test_varlen_layout():
    w = WORKLOADS["packed_long"]
    q, k, v, cu = workloads.make_varlen(w, seqlens=(7, 130, 1), dtype="f32")
    assert cu == [0, 7, 137, 138]
    assert q.shape == (138, 32, 128) and k.shape == (138, 8, 128)


def test_decode_inputs():
    w = WORKLOADS["decode"]
    di = workloads.make_decode(w, B=2, prefix=40, steps=3, chunk=16)
    assert di.prefix_k.shape == (2, 40, 8, 128)
    assert di.q.shape == (3, 2, 32, 128) and di.k_new.shape == (3, 2, 8, 128)
    di2 = workloads.make_decode(w, B=2, prefix=40, steps=3, chunk=16)
    assert torch.equal(di.prefix_k, di2.prefix_k) and torch.equal(di.v_new, di2.v_new)
    # sink keys carry the bias: their norm is well above sqrt(d)
    n_sink = di.prefix_k[:, :4].float().norm(dim=-1).mean()
    n_rest = di.prefix_k[:, 4:].float().norm(dim=-1).mean()
    assert n_sink > 1.8 * n_rest


def test_sample_rows_cover_edges():
    rows = workloads.sample_rows(32768, 4096, 4)
    for t in (0, 1, 4095, 4096, 4099, 32767, 128, 127):
        assert t in rows
    assert len(rows) < 600
    assert math.isclose(len(set(rows)), len(rows))
