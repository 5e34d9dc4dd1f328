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
