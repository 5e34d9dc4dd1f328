"""GPU parity of the short-window stream kernel (d = 64, bf16 inputs, window up to
129 keys, no sink prefix), which swa_fwd / swa_fwd_varlen choose for those shapes.

Every case is checked against the oracle, and, where the pair kernel applies (an
even head count), against it on the same inputs (debug flag 4 turns the stream
kernel off).  The stream kernel works on 64-key sub-tiles and the pair kernel on
128-key tiles, so their running maxima and summation orders differ and the two
agree within the oracle bounds, not bit for bit.  The ranges of query tiles a CTA streams
cross heads and sequences, start in the middle of sequences and can be a single
tile; the cases below make all of that happen."""
import math

import numpy as np
import pytest
import torch

import oracle
import sink_aware_sliding_b200 as swa
import workloads
from tests.helpers import assert_close
from workloads import WORKLOADS

pytestmark = pytest.mark.gpu


class flags:
    def __init__(self, f):
        self.f = f

    def __enter__(self):
        self.prev = swa.swa_set_debug_flags(self.f)

    def __exit__(self, *exc):
        swa.swa_set_debug_flags(self.prev)


def rand_qkv(B, L, Hq, Hkv, d, seed):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(B, L, Hq, d, generator=g).bfloat16()
    k = torch.randn(B, L, Hkv, d, generator=g).bfloat16()
    v = torch.randn(B, L, Hkv, d, generator=g).bfloat16()
    return q, k, v


def run(q, k, v, window, out_dtype, flag=0):
    B, L, Hq, d = q.shape
    out = torch.empty(q.shape, device="cuda", dtype=out_dtype)
    lse = torch.empty(B, Hq, L, device="cuda", dtype=torch.float32)
    with flags(flag):
        swa.swa_fwd(q, k, v, out, lse, window, 0)
    torch.cuda.synchronize()
    assert swa.swa_device_error() == 0
    return out, lse


@pytest.mark.parametrize("B,L,Hq,Hkv,window", [
    (2, 520, 4, 4, 128),     # Based-like, ragged tail
    (1, 2048, 2, 2, 129),    # widest window the kernel takes
    (3, 300, 3, 1, 64),      # odd head count, GQA 3, window smaller than a tile
    (1, 1000, 4, 2, 2),      # window 2
    (2, 700, 2, 2, 1),       # window 1: one key tile per query tile
    (4, 128, 8, 8, 128),     # one tile per sequence: every range crosses sequences
    (1, 77, 1, 1, 100),      # a single partial tile
    (1, 5000, 1, 1, 127),    # one long stream per CTA range
])
def test_stream_matches_oracle_and_pair_kernel(B, L, Hq, Hkv, window):
    q, k, v = rand_qkv(B, L, Hq, Hkv, 64, B * L + window)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    ro, rl = oracle.swa_fwd(q, k, v, window, 0, 1 / 8)
    # P is rounded to bf16 for the PV product (relative error up to 2^-8 per
    # weight).  With only a few visible keys one weight carries most of a row's
    # mass, so a row can be off by up to 2^-8 of the largest |v|; with wider
    # windows these errors average out far below 1e-2.
    max_abs = 1e-2 if window > 8 else max(1e-2, 2.0 ** -8 * float(v.float().abs().max()) + 1e-3)
    for od in (torch.float32, torch.bfloat16):
        out, lse = run(qd, kd, vd, window, od)
        assert_close(out, ro, f"stream out[{od}]", max_abs=max_abs)
        assert_close(lse, rl, f"stream lse[{od}]")
        if Hq % 2 == 0:                     # the pair kernel applies (odd Hq: one-tile kernel)
            pout, plse = run(qd, kd, vd, window, od, flag=4)
            assert_close(out, pout.double().cpu(), f"stream vs pair out[{od}]", max_abs=max_abs)
            assert_close(lse, plse.double().cpu(), f"stream vs pair lse[{od}]")


def test_stream_varlen_matches_oracle():
    seqlens = [1, 130, 128, 0, 900, 255, 257, 3]
    cu = workloads.cu_seqlens_of(seqlens)
    T, Hq, Hkv, d, window = cu[-1], 4, 2, 64, 128
    g = torch.Generator().manual_seed(9)
    q = torch.randn(T, Hq, d, generator=g).bfloat16()
    k = torch.randn(T, Hkv, d, generator=g).bfloat16()
    v = torch.randn(T, Hkv, d, generator=g).bfloat16()
    ro, rl = oracle.swa_fwd_varlen(q, k, v, cu, window, 0, 1 / 8)
    cu_d = torch.tensor(cu, dtype=torch.int32, device="cuda")
    for od in (torch.float32, torch.bfloat16):
        for flag in (0, 4):
            out = torch.empty(T, Hq, d, device="cuda", dtype=od)
            lse = torch.empty(Hq, T, device="cuda", dtype=torch.float32)
            with flags(flag):
                swa.swa_fwd_varlen(q.cuda(), k.cuda(), v.cuda(), out, lse, cu_d, window, 0)
            torch.cuda.synchronize()
            assert swa.swa_device_error() == 0
            assert_close(out, ro, f"varlen out[{od}, flag {flag}]")
            assert_close(lse, rl, f"varlen lse[{od}, flag {flag}]")


def test_based_local_stream_against_pair_kernel():
    """The benchmark workload in its launch configuration: every element of the
    stream kernel's output against the pair kernel's (checked against the oracle at
    this size in the prefill tests), and sampled rows against the oracle."""
    w = WORKLOADS["based_local"]
    q, k, v = workloads.make_prefill(w, device="cuda")
    out, lse = run(q, k, v, w.window, torch.float32)
    pout, plse = run(q, k, v, w.window, torch.float32, flag=4)
    err = (out - pout).abs()
    assert err.max().item() <= 1e-2 and err.mean().item() <= 1e-3
    assert (lse - plse).abs().max().item() <= 1e-2
    rows = workloads.sample_rows(w.L, w.window, w.n_sink, n_random=64)
    for b in (0, w.B - 1):
        ro, rl = oracle.swa_rows(q[b, rows].cpu(), rows, k[b].cpu(), v[b].cpu(), w.window, 0, w.scale)
        assert_close(out[b, rows], ro, f"based b={b} sampled rows out")
        assert_close(lse[b][:, rows].transpose(0, 1), rl, f"based b={b} sampled rows lse")


def test_stream_wait_timeout_reports_and_recovers():
    q, k, v = (t.cuda() for t in rand_qkv(2, 1024, 4, 4, 64, 3))
    prev_t = swa.swa_set_wait_timeout_ns(50_000_000)
    try:
        with flags(1):
            out, lse = torch.empty_like(q), torch.empty(2, 4, 1024, device="cuda")
            swa.swa_fwd(q, k, v, out, lse, 128, 0)
            torch.cuda.synchronize()
        assert swa.swa_device_error() == swa.SWA_ERR_DEVICE_TIMEOUT
    finally:
        swa.swa_set_wait_timeout_ns(prev_t)
    out, lse = run(q, k, v, 128, torch.float32)
    ro, rl = oracle.swa_fwd(q.cpu(), k.cpu(), v.cpu(), 128, 0, 1 / 8)
    assert_close(out, ro, "after timeout out")
