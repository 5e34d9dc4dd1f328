"""GPU parity of the prefill kernel against the fp64 oracle (through the C ABI)."""
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


def gpu_fwd(q, k, v, window, n_sink, scale=None, out_dtype=None):
    q, k, v = (t.cuda().contiguous() for t in (q, k, v))
    B, L, Hq, d = q.shape
    out = torch.empty(q.shape, device="cuda", dtype=out_dtype or q.dtype)
    lse = torch.empty(B, Hq, L, device="cuda", dtype=torch.float32)
    swa.swa_fwd(q, k, v, out, lse, window, n_sink, scale)
    torch.cuda.synchronize()
    assert swa.swa_device_error() == 0
    return out, lse


def rand_qkv(B, L, Hq, Hkv, d, seed, dtype=torch.bfloat16):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(B, L, Hq, d, generator=g).to(dtype)
    k = torch.randn(B, L, Hkv, d, generator=g).to(dtype)
    v = torch.randn(B, L, Hkv, d, generator=g).to(dtype)
    return q, k, v


class one_tile_kernel:
    """Within the block, swa_fwd uses the one-query-tile kernel even where the
    two-tile kernel applies (test hook, debug flag bit 1)."""

    def __enter__(self):
        self.prev = swa.swa_set_debug_flags(2)

    def __exit__(self, *exc):
        swa.swa_set_debug_flags(self.prev)


def check_full(q, k, v, window, n_sink, what, both_kernels=True):
    """bf16 inputs are run twice: with fp32 output (the arithmetic, strict bound)
    and with bf16 output (the bound plus the output's own rounding); and, where
    the two-tile kernel applies, once more through the one-tile kernel."""
    scale = 1.0 / math.sqrt(q.shape[-1])
    ro, rl = oracle.swa_fwd(q, k, v, window, n_sink, scale)
    outs = [torch.float32] if q.dtype == torch.float32 else [torch.float32, torch.bfloat16]
    for od in outs:
        out, lse = gpu_fwd(q, k, v, window, n_sink, scale, out_dtype=od)
        assert_close(out, ro, f"{what} out[{od}]")
        assert_close(lse, rl, f"{what} lse[{od}]")
    if both_kernels:
        with one_tile_kernel():
            out, lse = gpu_fwd(q, k, v, window, n_sink, scale, out_dtype=outs[-1])
        assert_close(out, ro, f"{what} out[one-tile kernel]")
        assert_close(lse, rl, f"{what} lse[one-tile kernel]")


def test_tiny_workload_fp32():
    w = WORKLOADS["tiny"]
    q, k, v = workloads.make_prefill(w)
    assert q.dtype == torch.float32
    check_full(q, k, v, w.window, w.n_sink, "tiny")


@pytest.mark.parametrize("B,L,Hq,Hkv,d,window,n_sink", [
    (2, 1000, 8, 2, 128, 300, 4),      # GQA, ragged tail, sinks
    (2, 520, 4, 4, 64, 128, 0),        # Based-like local window, d = 64
    (1, 384, 4, 1, 128, 1000, 0),      # window covers the sequence: full causal
    (1, 300, 2, 2, 128, 1, 0),         # window 1
    (1, 700, 4, 2, 128, 64, 200),      # sink prefix wider than a key tile
    (1, 600, 2, 1, 64, 100, 130),      # sinks longer than the window
    (3, 77, 4, 2, 128, 16, 4),         # a single partial tile per sequence
    (2, 1, 4, 4, 128, 8, 4),           # one token
    (1, 2048, 8, 8, 64, 128, 4),       # several q tiles, d = 64 with sinks
    (2, 700, 3, 1, 128, 200, 4),       # odd head count (one-tile kernel only)
    (1, 900, 6, 2, 128, 256, 4),       # G = 3: head pairs straddle KV heads
    (1, 900, 6, 2, 64, 256, 4),        # same at d = 64 (two-tile kernel, separate K/V)
    (4, 1024, 16, 16, 64, 128, 0),     # many units per CTA, d = 64, G = 1
    (1, 4096, 32, 8, 128, 512, 4),     # many units per CTA, GQA
    (1, 500, 4, 2, 128, 40, 4),        # sink tile is the first band tile
    (1, 500, 4, 2, 64, 40, 70),        # sink prefix across the first band tile, d = 64
    (2, 640, 4, 2, 64, 200, 4),        # d = 64 GQA: TMA-store epilogue over several units
    (1, 900, 4, 2, 128, 256, 16),      # 16 sinks: the widest sink mini-tile
    (1, 900, 4, 2, 64, 256, 17),       # 17 sinks: a whole masked sink tile again
    (1, 700, 4, 4, 128, 200, 1),       # a single sink
    (1, 1200, 2, 1, 64, 300, 16),      # mini-tile at d = 64 with the TMA-store epilogue
])
def test_prefill_matches_oracle(B, L, Hq, Hkv, d, window, n_sink):
    q, k, v = rand_qkv(B, L, Hq, Hkv, d, seed=B * 1000 + L)
    check_full(q, k, v, window, n_sink, f"B{B} L{L} H{Hq}/{Hkv} d{d} w{window} s{n_sink}")


def test_window_one_returns_v():
    q, k, v = rand_qkv(1, 260, 2, 2, 128, seed=5)
    out, _ = gpu_fwd(q, k, v, 1, 0)
    assert torch.equal(out.cpu(), v)


def test_fp32_d64_edges():
    q, k, v = rand_qkv(2, 333, 4, 2, 64, seed=9, dtype=torch.float32)
    check_full(q, k, v, 50, 3, "fp32 GQA")


def test_sink_stress_mass_on_sinks():
    """Queries share a direction c and the sink keys point along c, so the sinks
    take most of the softmax mass; the kernel must still match."""
    B, L, H, d, w, s = 1, 1500, 2, 128, 256, 4
    g = torch.Generator().manual_seed(11)
    c = torch.randn(d, generator=g)
    c = c / c.norm()
    q = torch.randn(B, L, H, d, generator=g) + 3.0 * c
    k = torch.randn(B, L, H, d, generator=g)
    k[:, :s] += 3.0 * math.sqrt(d) * c
    v = torch.randn(B, L, H, d, generator=g)
    q, k, v = q.bfloat16(), k.bfloat16(), v.bfloat16()
    wts = oracle.swa_weights(q[0, L - 1], L - 1, k[0], 0, w, s, 1 / math.sqrt(d))
    assert wts[:s].sum() > 0.9
    check_full(q, k, v, w, s, "sink stress")


def test_varlen_matches_oracle():
    lens = [1, 127, 128, 129, 700, 3, 256]
    cu = workloads.cu_seqlens_of(lens)
    T, Hq, Hkv, d, w, s = cu[-1], 8, 2, 128, 64, 4
    g = torch.Generator().manual_seed(3)
    q = torch.randn(T, Hq, d, generator=g).bfloat16()
    k = torch.randn(T, Hkv, d, generator=g).bfloat16()
    v = torch.randn(T, Hkv, d, generator=g).bfloat16()
    out = torch.empty(T, Hq, d, device="cuda", dtype=torch.bfloat16)
    lse = torch.empty(Hq, T, device="cuda", dtype=torch.float32)
    cu_d = torch.tensor(cu, dtype=torch.int32, device="cuda")
    swa.swa_fwd_varlen(q.cuda(), k.cuda(), v.cuda(), out, lse, cu_d, w, s)
    torch.cuda.synchronize()
    ro, rl = oracle.swa_fwd_varlen(q, k, v, cu, w, s, 1 / math.sqrt(d))
    assert_close(out, ro, "varlen out")
    assert_close(lse, rl, "varlen lse")


def test_based_local_full_size():
    w = WORKLOADS["based_local"]
    q, k, v = workloads.make_prefill(w)
    check_full(q, k, v, w.window, w.n_sink, "based_local")


def _sampled_rows_check(q, k, v, out, lse, window, n_sink, rows, what):
    """q/k/v on the host [L, H, d] of one sequence; out [L, Hq, d], lse [Hq, L] from the GPU."""
    d = q.shape[-1]
    ro, rl = oracle.swa_rows(q[rows], rows, k, v, window, n_sink, 1 / math.sqrt(d))
    assert_close(out[rows], ro, what + " out")
    assert_close(lse[:, rows].T, rl, what + " lse")


def test_gqa8b_full_size_sampled_rows():
    w = WORKLOADS["gqa8b_prefill"]
    q, k, v = workloads.make_prefill(w, device="cuda")
    out = torch.empty_like(q)
    lse = torch.empty(1, w.Hq, w.L, device="cuda", dtype=torch.float32)
    swa.swa_fwd(q, k, v, out, lse, w.window, w.n_sink)
    torch.cuda.synchronize()
    assert swa.swa_device_error() == 0
    rows = workloads.sample_rows(w.L, w.window, w.n_sink)
    _sampled_rows_check(q[0].cpu(), k[0].cpu(), v[0].cpu(), out[0].cpu(), lse[0].cpu(), w.window,
                        w.n_sink, rows, "gqa8b")


def test_packed_long_sampled_rows():
    w = WORKLOADS["packed_long"]
    q, k, v, cu = workloads.make_varlen(w, device="cuda")
    T = cu[-1]
    out = torch.empty_like(q)
    lse = torch.empty(w.Hq, T, device="cuda", dtype=torch.float32)
    swa.swa_fwd_varlen(q, k, v, out, lse, torch.tensor(cu, dtype=torch.int32, device="cuda"),
                       w.window, w.n_sink)
    torch.cuda.synchronize()
    assert swa.swa_device_error() == 0
    qh, kh, vh, oh, lh = q.cpu(), k.cpu(), v.cpu(), out.cpu(), lse.cpu()
    for i, n in enumerate(w.seqlens):
        a = cu[i]
        rows = workloads.sample_rows(n, w.window, w.n_sink, n_random=64, seed=i)
        _sampled_rows_check(qh[a:a + n], kh[a:a + n], vh[a:a + n], oh[a:a + n], lh[:, a:a + n],
                            w.window, w.n_sink, rows, f"packed seq {i}")


def test_repeat_calls_are_deterministic():
    q, k, v = rand_qkv(1, 1024, 8, 2, 128, seed=21)
    o1, l1 = gpu_fwd(q, k, v, 200, 4)
    o2, l2 = gpu_fwd(q, k, v, 200, 4)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
