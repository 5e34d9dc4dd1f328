"""GPU parity of the backward pass (through the C ABI) against the oracle.

The forward runs on the GPU (its out and lse are part of the path under test);
the oracle computes the gradients from q, k, v and dout alone.

Tolerance: the pages state none for gradients.  A gradient element sums up to L
products whose factors P and dS are rounded to bf16 for the tensor cores, so the
forward's bounds (max 1e-2, mean 1e-3) are applied relative to the gradient's
own scale where that exceeds one: max|err| <= 1e-2 max(1, max|ref|) and
mean|err| <= 1e-3 max(1, mean|ref|)."""
import math

import numpy as np
import pytest
import torch

import oracle
import sink_aware_sliding_b200 as swa

pytestmark = pytest.mark.gpu


def assert_grad_close(got, want, what):
    g = got.detach().cpu().double().numpy()
    err = np.abs(g - want)
    mx_allow = 1e-2 * max(1.0, float(np.abs(want).max()))
    mn_allow = 1e-3 * max(1.0, float(np.abs(want).mean()))
    assert np.isfinite(g).all(), f"{what}: non-finite"
    assert err.max() <= mx_allow and err.mean() <= mn_allow, (
        f"{what}: max {err.max():.3e} (allowed {mx_allow:.3e}) mean {err.mean():.3e} (allowed {mn_allow:.3e})")


def run_bwd(B, L, Hq, Hkv, d, window, n_sink, seed):
    g = torch.Generator().manual_seed(seed)
    q, k, v, do = (torch.randn(*sh, generator=g).bfloat16() for sh in
                   ((B, L, Hq, d), (B, L, Hkv, d), (B, L, Hkv, d), (B, L, Hq, d)))
    qd, kd, vd, dod = (t.cuda() for t in (q, k, v, do))
    out = torch.empty_like(qd)
    lse = torch.empty(B, Hq, L, device="cuda")
    swa.swa_fwd(qd, kd, vd, out, lse, window, n_sink)
    dq = torch.full((B, L, Hq, d), float("nan"), device="cuda")
    dk = torch.full((B, L, Hkv, d), float("nan"), device="cuda")
    dv = torch.full_like(dk, float("nan"))
    swa.swa_bwd(qd, kd, vd, out, dod, lse, dq, dk, dv, window, n_sink)
    torch.cuda.synchronize()
    assert swa.swa_device_error() == 0
    return (q, k, v, do), (dq, dk, dv)


@pytest.mark.parametrize("B,L,Hq,Hkv,d,window,n_sink", [
    (1, 128, 2, 2, 64, 64, 0),         # one tile
    (2, 300, 4, 2, 64, 64, 4),         # GQA, ragged tail, sinks
    (1, 520, 2, 2, 128, 200, 0),       # window wider than a tile
    (1, 384, 4, 1, 128, 1000, 0),      # full causal, four query heads per KV head
    (1, 700, 2, 2, 64, 64, 200),       # sink prefix spanning two key tiles
    (2, 77, 2, 2, 128, 16, 4),         # a single partial tile per sequence
    (1, 1024, 4, 4, 64, 128, 0),       # Based-like window
    (1, 600, 2, 1, 64, 100, 130),      # sinks longer than the window
])
def test_bwd_matches_oracle(B, L, Hq, Hkv, d, window, n_sink):
    (q, k, v, do), (dq, dk, dv) = run_bwd(B, L, Hq, Hkv, d, window, n_sink, B * L + window + n_sink)
    rq, rk, rv = oracle.swa_bwd(q, k, v, do, window, n_sink, 1 / math.sqrt(d))
    assert_grad_close(dq, rq, "dq")
    assert_grad_close(dk, rk, "dk")
    assert_grad_close(dv, rv, "dv")


def test_bwd_window_one_is_exact():
    # out = v: dv = dout summed over the query heads of each KV head, dq = dk = 0
    (q, k, v, do), (dq, dk, dv) = run_bwd(1, 300, 4, 2, 128, 1, 0, 5)
    want = do.double().view(1, 300, 2, 2, 128).sum(dim=3).numpy()
    np.testing.assert_allclose(dv.cpu().double().numpy(), want, atol=1e-5)
    assert dq.abs().max().item() < 1e-5 and dk.abs().max().item() < 1e-5


def test_bwd_repeat_is_deterministic():
    _, (a1, b1, c1) = run_bwd(1, 400, 2, 2, 128, 100, 4, 9)
    _, (a2, b2, c2) = run_bwd(1, 400, 2, 2, 128, 100, 4, 9)
    assert torch.equal(a1, a2) and torch.equal(b1, b2) and torch.equal(c1, c2)


def test_bwd_gqa_sink_biased_long_sequence():
    """Near the benchmarked backward shape: four query heads per KV head, d = 128,
    sink keys biased toward the queries (the 8B-shaped workload's recipe), and a
    sequence of 32 query tiles, so the dK/dV tile that holds the sink prefix is seen
    by every later query tile of all four heads."""
    import workloads
    B, L, Hq, Hkv, d, window, n_sink = 1, 4096, 8, 2, 128, 1024, 4
    g = torch.Generator().manual_seed(41)
    q = torch.randn(B, L, Hq, d, generator=g)
    k = torch.randn(B, L, Hkv, d, generator=g)
    v = torch.randn(B, L, Hkv, d, generator=g)
    do = torch.randn(B, L, Hq, d, generator=g)
    workloads._bias_sinks_(k[0], q[0], n_sink, Hq // Hkv)
    q, k, v, do = (t.bfloat16() for t in (q, k, v, do))
    qd, kd, vd, dod = (t.cuda() for t in (q, k, v, do))
    out = torch.empty_like(qd)
    lse = torch.empty(B, Hq, L, device="cuda")
    swa.swa_fwd(qd, kd, vd, out, lse, window, n_sink)
    dq = torch.full((B, L, Hq, d), float("nan"), device="cuda")
    dk = torch.full((B, L, Hkv, d), float("nan"), device="cuda")
    dv = torch.full_like(dk, float("nan"))
    swa.swa_bwd(qd, kd, vd, out, dod, lse, dq, dk, dv, window, n_sink)
    torch.cuda.synchronize()
    assert swa.swa_device_error() == 0
    rq, rk, rv = oracle.swa_bwd(q, k, v, do, window, n_sink, 1 / math.sqrt(d))
    assert_grad_close(dq, rq, "dq")
    assert_grad_close(dk, rk, "dk")
    assert_grad_close(dv, rv, "dv")
    # the sink keys carry gradient from every query tile
    assert np.abs(rk[0, :n_sink]).max() > 0


def test_bwd_benchmark_shape_identities():
    """The benchmarked backward shape itself (B=1, Hq=32, Hkv=8, L=8192, d=128, window
    4096, 4 sink-biased keys) against two identities that hold at any size: every row
    of P sums to one, so the dV of a KV head summed over positions equals dout summed
    over positions and over its query heads; every row of dS sums to zero, so the dK
    of a KV head sums to zero over positions."""
    import workloads
    w = workloads.WORKLOADS["gqa8b_prefill"]
    q, k, v = workloads.make_prefill(w, device="cuda", L=8192)
    gen = torch.Generator(device="cuda").manual_seed(workloads.SEED + 1)
    do = torch.randn(q.shape, generator=gen, device="cuda").bfloat16()
    out = torch.empty_like(q)
    lse = torch.empty(1, w.Hq, 8192, device="cuda")
    swa.swa_fwd(q, k, v, out, lse, w.window, w.n_sink)
    dq = torch.empty(q.shape, device="cuda")
    dk = torch.empty(k.shape, device="cuda")
    dv = torch.empty_like(dk)
    swa.swa_bwd(q, k, v, out, do, lse, dq, dk, dv, w.window, w.n_sink)
    torch.cuda.synchronize()
    assert swa.swa_device_error() == 0
    assert torch.isfinite(dq).all() and torch.isfinite(dk).all() and torch.isfinite(dv).all()
    G = w.Hq // w.Hkv
    want_dv = do.double().sum(dim=1).view(1, w.Hkv, G, w.d).sum(dim=2)       # [1, Hkv, d]
    got_dv = dv.double().sum(dim=1)
    # P is rounded to bf16 (relative 2^-9 per weight) before P^T dout: the column sums
    # agree to that relative precision of the summed magnitudes
    scale_dv = do.double().abs().sum(dim=1).view(1, w.Hkv, G, w.d).sum(dim=2)
    assert ((got_dv - want_dv).abs() <= 4e-3 * scale_dv + 1e-3).all()
    got_dk = dk.double().sum(dim=1)
    scale_dk = dk.double().abs().sum(dim=1)
    assert ((got_dk.abs()) <= 1e-2 * scale_dk + 1e-3).all()
