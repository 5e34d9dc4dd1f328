"""GPU parity of the Based linear branch (Taylor-kernel linear attention)
through the C ABI: the chunked prefill (outputs and final recurrent state) and
the recurrent decode step, against the oracle's fp64 definitions.

Outputs are normalised averages of the values, compared under the usual
max-abs 1e-2 / mean-abs 1e-3 bounds.  The state is a sum of n products
phi(k_s) v_s in which the prefill kernel rounds each feature to bf16 (relative
error <= 2^-9; the values are bf16 already) and accumulates in fp32 (the
summation bound gamma_n ~ n 2^-24).  Each entry is checked against
(2^-8 + 2 (n + 4) 2^-24) sum_s |phi(k_s)| |v_s|: twice the feature rounding,
twice the fp32 summation bound.  The CUDA-core form of the same chunked step,
fp32 throughout, must meet the fp32 part alone."""
import numpy as np
import pytest
import torch

import oracle
import sink_aware_sliding_b200 as swa
import workloads
from tests.helpers import assert_close

pytestmark = pytest.mark.gpu
W = workloads.LINEAR_WORKLOADS["based_linear"]
DEV = "cuda"


def run_fwd(q, k, v, out_dtype=torch.float32, with_state=True, simt=False):
    B, L, H, _ = q.shape
    out = torch.empty(B, L, H, W.dv, device=DEV, dtype=out_dtype)
    S = torch.full((B, H, W.F, W.dv), float("nan"), device=DEV) if with_state else None
    z = torch.full((B, H, W.F), float("nan"), device=DEV) if with_state else None
    prev = swa.swa_set_debug_flags(8) if simt else None
    try:
        swa.swa_based_linear_fwd(q.to(DEV), k.to(DEV), v.to(DEV), out, S, z, W.scale)
        torch.cuda.synchronize()
    finally:
        if simt:
            swa.swa_set_debug_flags(prev)
    assert swa.swa_device_error() == 0
    return out, S, z


def state_bound(k, v, n, bf16_features=True):
    fk = np.abs(oracle.taylor_features(k, W.scale))                    # [B, L, H, F]
    av = np.abs(v.double().numpy())
    sS = np.einsum("blhf,blhc->bhfc", fk, av)
    sz = fk.sum(axis=1)
    c = 2.0 * (n + 4) * 2.0 ** -24 + (2.0 ** -8 if bf16_features else 0.0)
    return c * sS + 1e-30, c * sz + 1e-30


def assert_state_close(S, z, k, v, what, bf16_features=True):
    wS, wz = oracle.based_linear_state(k, v, W.scale)
    bS, bz = state_bound(k, v, k.shape[1], bf16_features)
    for got, want, bound, name in ((S, wS, bS, "S"), (z, wz, bz, "z")):
        g = got.cpu().double().numpy()
        assert np.isfinite(g).all(), f"{what}: {name} not fully written"
        worst = float((np.abs(g - want) / bound).max())
        assert worst <= 1.0, f"{what}: {name} exceeds the fp32 summation bound by x{worst:.2f}"


@pytest.mark.parametrize("B,L,H", [(2, 200, 3), (1, 128, 2), (1, 129, 1), (1, 1, 2), (3, 127, 1), (1, 700, 2)])
def test_prefill_matches_oracle(B, L, H):
    w = workloads.LinearWorkload("t", B=B, L=L, H=H, dk=W.dk, dv=W.dv)
    q, k, v = workloads.make_based_linear(w, seed=11 + L)
    out, S, z = run_fwd(q, k, v)
    assert_close(out, oracle.based_linear_fwd(q, k, v, W.scale), f"based linear B={B} L={L} H={H}")
    assert_state_close(S, z, k, v, f"state B={B} L={L} H={H}")
    out16, _, _ = run_fwd(q, k, v, out_dtype=torch.bfloat16, with_state=False)
    assert_close(out16, oracle.based_linear_fwd(q, k, v, W.scale), f"bf16 out L={L}")


@pytest.mark.parametrize("L", [1, 64, 200])
def test_cuda_core_form_matches_oracle(L):
    """The fp32 CUDA-core form of the chunked step (a test hook selects it)."""
    w = workloads.LinearWorkload("t", B=2, L=L, H=2, dk=W.dk, dv=W.dv)
    q, k, v = workloads.make_based_linear(w, seed=3 + L)
    out, S, z = run_fwd(q, k, v, simt=True)
    assert_close(out, oracle.based_linear_fwd(q, k, v, W.scale), f"CUDA-core form L={L}")
    assert_state_close(S, z, k, v, f"CUDA-core state L={L}", bf16_features=False)


def test_expired_wait_reports_timeout_and_context_survives():
    w = workloads.LinearWorkload("t", B=2, L=300, H=2, dk=W.dk, dv=W.dv)
    q, k, v = workloads.make_based_linear(w, seed=21)
    out = torch.zeros(2, 300, 2, W.dv, device=DEV)
    S = torch.zeros(2, 2, W.F, W.dv, device=DEV)
    z = torch.zeros(2, 2, W.F, device=DEV)
    assert swa.swa_device_error() == 0
    prev_t = swa.swa_set_wait_timeout_ns(50_000_000)
    prev_f = swa.swa_set_debug_flags(1)                        # the MMA warp issues nothing
    try:
        swa.swa_based_linear_fwd(q.to(DEV), k.to(DEV), v.to(DEV), out, S, z, W.scale)
        assert swa.swa_device_error() == swa.SWA_ERR_DEVICE_TIMEOUT
    finally:
        swa.swa_set_debug_flags(prev_f)
        swa.swa_set_wait_timeout_ns(prev_t)
    out2, S2, z2 = run_fwd(q, k, v)
    assert_close(out2, oracle.based_linear_fwd(q, k, v, W.scale), "after timeout")


def test_prefill_other_scale():
    """scale = 0.1 instead of 1/sqrt(dk): sqrt(scale) is no longer a power of two,
    so the linear features carry their own bf16 rounding."""
    w = workloads.LinearWorkload("t", B=2, L=300, H=2, dk=W.dk, dv=W.dv)
    q, k, v = workloads.make_based_linear(w, seed=31)
    out = torch.empty(2, 300, 2, W.dv, device=DEV)
    S = torch.full((2, 2, W.F, W.dv), float("nan"), device=DEV)
    z = torch.full((2, 2, W.F), float("nan"), device=DEV)
    swa.swa_based_linear_fwd(q.to(DEV), k.to(DEV), v.to(DEV), out, S, z, 0.1)
    torch.cuda.synchronize()
    assert swa.swa_device_error() == 0
    assert_close(out, oracle.based_linear_fwd(q, k, v, 0.1), "scale 0.1")
    wS, wz = oracle.based_linear_state(k, v, 0.1)
    fk = np.abs(oracle.taylor_features(k, 0.1))
    c = 2.0 * (300 + 4) * 2.0 ** -24 + 2.0 ** -8
    bS = c * np.einsum("blhf,blhc->bhfc", fk, np.abs(v.double().numpy())) + 1e-30
    bz = c * fk.sum(axis=1) + 1e-30
    assert (np.abs(S.cpu().double().numpy() - wS) <= bS).all()
    assert (np.abs(z.cpu().double().numpy() - wz) <= bz).all()


def test_empty_sequence_writes_a_zero_state():
    q = torch.empty(2, 0, 2, W.dk, dtype=torch.bfloat16)
    v = torch.empty(2, 0, 2, W.dv, dtype=torch.bfloat16)
    out, S, z = run_fwd(q, q, v)
    assert out.numel() == 0
    assert (S == 0).all() and (z == 0).all()


def test_decode_continues_the_prefill_state():
    w = workloads.LinearWorkload("t", B=3, L=136, H=2, dk=W.dk, dv=W.dv)
    q, k, v = workloads.make_based_linear(w, seed=5)
    L0 = 130
    _, S, z = run_fwd(q[:, :L0].contiguous(), k[:, :L0].contiguous(), v[:, :L0].contiguous())
    rS, rz = oracle.based_linear_state(k[:, :L0], v[:, :L0], W.scale)
    full = oracle.based_linear_fwd(q, k, v, W.scale)
    for t in range(L0, w.L):
        out = torch.empty(w.B, w.H, W.dv, device=DEV, dtype=torch.float32)
        qt, kt, vt = (x[:, t].contiguous() for x in (q, k, v))
        swa.swa_based_linear_decode(qt.to(DEV), kt.to(DEV), vt.to(DEV), S, z, out, W.scale)
        torch.cuda.synchronize()
        ro, rS, rz = oracle.based_linear_decode(qt, kt, vt, rS, rz, W.scale)
        assert_close(out, ro, f"decode step {t}")
        # the recurrent step reproduces row t of the parallel form
        assert_close(out, full[:, t], f"decode step {t} vs prefill row")
    assert_state_close(S, z, k, v, "state after decode")


def test_decode_bf16_output_and_fresh_state():
    w = workloads.LinearWorkload("t", B=4, L=1, H=3, dk=W.dk, dv=W.dv)
    q, k, v = workloads.make_based_linear(w, seed=9)
    S = torch.zeros(w.B, w.H, W.F, W.dv, device=DEV)
    z = torch.zeros(w.B, w.H, W.F, device=DEV)
    out = torch.empty(w.B, w.H, W.dv, device=DEV, dtype=torch.bfloat16)
    qt, kt, vt = (x[:, 0].contiguous() for x in (q, k, v))
    swa.swa_based_linear_decode(qt.to(DEV), kt.to(DEV), vt.to(DEV), S, z, out, W.scale)
    torch.cuda.synchronize()
    ro, _, _ = oracle.based_linear_decode(qt, kt, vt, np.zeros((4, 3, W.F, W.dv)), np.zeros((4, 3, W.F)), W.scale)
    # a single visible token: the output is that token's value
    np.testing.assert_allclose(ro, vt.double().numpy(), atol=1e-12)
    assert_close(out, ro, "decode from an empty state")


def test_full_size_sampled_heads():
    """The benchmarked shape (B=8, L=2048, H=16): every row of four (sequence,
    head) pairs and their final state against the oracle run on those heads."""
    q, k, v = workloads.make_based_linear(W)
    out, S, z = run_fwd(q, k, v)
    for b, h in ((0, 0), (3, 7), (5, 15), (7, 9)):
        qs, ks, vs = (x[b:b + 1, :, h:h + 1] for x in (q, k, v))
        assert_close(out[b:b + 1, :, h:h + 1], oracle.based_linear_fwd(qs, ks, vs, W.scale), f"full size b={b} h={h}")
        assert_state_close(S[b:b + 1, h:h + 1], z[b:b + 1, h:h + 1], ks, vs, f"full-size state b={b} h={h}")
    assert torch.isfinite(out).all()
