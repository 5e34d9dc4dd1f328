"""GPU parity of the ring-buffer cache kernels and the split-K decode (through the C ABI)."""
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


class Cache:
    def __init__(self, B, Hkv, d, window, n_sink):
        z = dict(device="cuda", dtype=torch.bfloat16)
        self.kc = torch.zeros(B, Hkv, window, d, **z)
        self.vc = torch.zeros(B, Hkv, window, d, **z)
        self.sk = torch.zeros(B, Hkv, max(n_sink, 1), d, **z)
        self.sv = torch.zeros(B, Hkv, max(n_sink, 1), d, **z)
        self.window, self.n_sink = window, n_sink

    def fill(self, k, v):
        swa.swa_cache_fill(k.cuda().contiguous(), v.cuda().contiguous(), self.kc, self.vc, self.sk,
                           self.sv, self.window, self.n_sink)

    def append(self, k_new, v_new, pos):
        swa.swa_cache_append(k_new.cuda().contiguous(), v_new.cuda().contiguous(), pos, self.kc,
                             self.vc, self.sk, self.sv, self.window, self.n_sink)


def rand(shape, seed):
    g = torch.Generator().manual_seed(seed)
    return torch.randn(*shape, generator=g).bfloat16()


def decode(cache, q, pos, Hkv):
    B, Hq, d = q.shape
    out = torch.empty(B, Hq, d, device="cuda", dtype=torch.bfloat16)
    lse = torch.empty(B, Hq, device="cuda", dtype=torch.float32)
    nbytes = swa.swa_decode_workspace_bytes(B, Hq, Hkv, d, cache.window, cache.n_sink)
    ws = torch.empty(nbytes // 4 + 64, device="cuda", dtype=torch.float32)
    swa.swa_decode(q.cuda().contiguous(), cache.kc, cache.vc, cache.sk, cache.sv, pos, out, lse,
                   cache.window, cache.n_sink, ws)
    torch.cuda.synchronize()
    return out, lse


@pytest.mark.parametrize("P", [1, 4, 63, 64, 68, 199])
def test_cache_fill_bit_exact(P):
    B, Hkv, d, W, S = 3, 2, 128, 64, 4
    k, v = rand((B, P, Hkv, d), P), rand((B, P, Hkv, d), P + 1)
    c = Cache(B, Hkv, d, W, S)
    c.fill(k, v)
    torch.cuda.synchronize()
    kc, vc, sk, sv = oracle.ring_fill(k.view(torch.int16).numpy(), v.view(torch.int16).numpy(), W, S)
    np.testing.assert_array_equal(c.kc.cpu().view(torch.int16).numpy(), kc)
    np.testing.assert_array_equal(c.vc.cpu().view(torch.int16).numpy(), vc)
    np.testing.assert_array_equal(c.sk.cpu().view(torch.int16).numpy(), sk)
    np.testing.assert_array_equal(c.sv.cpu().view(torch.int16).numpy(), sv)


def test_cache_append_bit_exact():
    B, Hkv, d, W, S = 4, 2, 64, 16, 3
    c = Cache(B, Hkv, d, W, S)
    kc = np.zeros((B, Hkv, W, d), np.int16)
    vc, sk, sv = np.zeros_like(kc), np.zeros((B, Hkv, S, d), np.int16), np.zeros((B, Hkv, S, d), np.int16)
    start = np.array([0, 2, 15, 40])
    for step in range(40):
        pos = start + step
        kn, vn = rand((B, Hkv, d), 100 + step), rand((B, Hkv, d), 200 + step)
        c.append(kn, vn, torch.tensor(pos, dtype=torch.int32, device="cuda"))
        oracle.ring_append(kc, vc, sk, sv, kn.view(torch.int16).numpy(), vn.view(torch.int16).numpy(),
                           pos, W, S)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(c.kc.cpu().view(torch.int16).numpy(), kc)
    np.testing.assert_array_equal(c.vc.cpu().view(torch.int16).numpy(), vc)
    np.testing.assert_array_equal(c.sk.cpu().view(torch.int16).numpy(), sk)
    np.testing.assert_array_equal(c.sv.cpu().view(torch.int16).numpy(), sv)


@pytest.mark.parametrize("Hq,Hkv,d", [(8, 2, 128), (4, 4, 64), (8, 1, 128), (6, 2, 64)])
def test_decode_matches_oracle_at_mixed_positions(Hq, Hkv, d):
    W, S = 64, 4
    pos = [0, 3, 62, 63, 64, 67, 68, 200, 1000]
    B, P = len(pos), max(pos) + 1
    k, v = rand((B, P, Hkv, d), 1), rand((B, P, Hkv, d), 2)
    q = rand((B, Hq, d), 3)
    c = Cache(B, Hkv, d, W, S)
    # each sequence b holds positions 0..pos[b]: fill with its first pos[b] tokens, then append pos[b]
    for b in range(B):
        cb = Cache(1, Hkv, d, W, S)
        if pos[b] > 0:
            cb.fill(k[b:b + 1, :pos[b]], v[b:b + 1, :pos[b]])
        for name in ("kc", "vc", "sk", "sv"):
            getattr(c, name)[b].copy_(getattr(cb, name)[0])
    pos_d = torch.tensor(pos, dtype=torch.int32, device="cuda")
    c.append(k[torch.arange(B), pos], v[torch.arange(B), pos], pos_d)
    out, lse = decode(c, q, pos_d, Hkv)
    ro, rl = oracle.swa_decode(q, k, v, pos, W, S, 1 / math.sqrt(d))
    assert_close(out, ro, "decode out")
    assert_close(lse, rl, "decode lse")


def test_decode_reproduces_last_prefill_row():
    B, Hq, Hkv, d, W, S = 2, 8, 2, 128, 96, 4
    for P in (1, S, W - 1, W, W + S, 3 * W + 7):
        g = torch.Generator().manual_seed(P)
        q = torch.randn(B, P, Hq, d, generator=g).bfloat16()
        k = torch.randn(B, P, Hkv, d, generator=g).bfloat16()
        v = torch.randn(B, P, Hkv, d, generator=g).bfloat16()
        out = torch.empty(B, P, Hq, d, device="cuda", dtype=torch.bfloat16)
        lse = torch.empty(B, Hq, P, device="cuda", dtype=torch.float32)
        swa.swa_fwd(q.cuda(), k.cuda(), v.cuda(), out, lse, W, S)
        c = Cache(B, Hkv, d, W, S)
        if P > 1:
            c.fill(k[:, :P - 1], v[:, :P - 1])
        pos = torch.full((B,), P - 1, dtype=torch.int32, device="cuda")
        c.append(k[:, P - 1], v[:, P - 1], pos)
        do, dl = decode(c, q[:, P - 1], pos, Hkv)
        assert_close(do, out[:, P - 1], f"P={P} decode vs prefill out")
        assert_close(dl, lse[:, :, P - 1], f"P={P} decode vs prefill lse")


def test_step_by_step_decode_wraps_around():
    B, Hq, Hkv, d, W, S = 2, 4, 1, 64, 32, 4
    n = 2 * W + S + 3
    k, v, q = rand((B, n, Hkv, d), 7), rand((B, n, Hkv, d), 8), rand((B, n, Hq, d), 9)
    c = Cache(B, Hkv, d, W, S)
    for p in range(n):
        pos = torch.full((B,), p, dtype=torch.int32, device="cuda")
        c.append(k[:, p], v[:, p], pos)
        out, lse = decode(c, q[:, p], pos, Hkv)
        ro, rl = oracle.swa_decode(q[:, p], k, v, [p] * B, W, S, 1 / math.sqrt(d))
        assert_close(out, ro, f"step {p} out")
        assert_close(lse, rl, f"step {p} lse")


def test_decode_workload_sampled():
    """The decode workload's shapes (B=64, Hq=32, Hkv=8, d=128, window 4096 + 4 sinks)
    after a 16384-token prefix, checked on a few steps and sequences."""
    w = WORKLOADS["decode"]
    di = workloads.make_decode(w, device="cuda", steps=3)
    c = Cache(w.B, w.Hkv, w.d, w.window, w.n_sink)
    c.fill(di.prefix_k, di.prefix_v)
    for i in range(3):
        p = w.prefix + i
        pos = torch.full((w.B,), p, dtype=torch.int32, device="cuda")
        c.append(di.k_new[i], di.v_new[i], pos)
        out, lse = decode(c, di.q[i], pos, w.Hkv)
        for b in (0, 37, 63):
            kh = torch.cat([di.prefix_k[b], di.k_new[:i + 1, b]], 0)[None].cpu()
            vh = torch.cat([di.prefix_v[b], di.v_new[:i + 1, b]], 0)[None].cpu()
            ro, rl = oracle.swa_decode(di.q[i, b:b + 1].cpu(), kh, vh, [p], w.window, w.n_sink,
                                       w.scale)
            assert_close(out[b:b + 1], ro, f"step {i} b {b} out")
            assert_close(lse[b:b + 1], rl, f"step {i} b {b} lse")


def _decode_workload_check(name, steps, rows, out_dtype):
    w = WORKLOADS[name]
    di = workloads.make_decode(w, device="cuda", steps=steps)
    c = Cache(w.B, w.Hkv, w.d, w.window, w.n_sink)
    c.fill(di.prefix_k, di.prefix_v)
    nbytes = swa.swa_decode_workspace_bytes(w.B, w.Hq, w.Hkv, w.d, w.window, w.n_sink)
    ws = torch.empty(nbytes, device="cuda", dtype=torch.uint8)
    for i in range(steps):
        p = w.prefix + i
        pos = torch.full((w.B,), p, dtype=torch.int32, device="cuda")
        c.append(di.k_new[i], di.v_new[i], pos)
        out = torch.empty(w.B, w.Hq, w.d, device="cuda", dtype=out_dtype)
        lse = torch.empty(w.B, w.Hq, device="cuda", dtype=torch.float32)
        swa.swa_decode(di.q[i], c.kc, c.vc, c.sk, c.sv, pos, out, lse, w.window, w.n_sink, ws)
        torch.cuda.synchronize()
        for b in rows:
            kh = torch.cat([di.prefix_k[b], di.k_new[:i + 1, b]], 0)[None].cpu()
            vh = torch.cat([di.prefix_v[b], di.v_new[:i + 1, b]], 0)[None].cpu()
            ro, rl = oracle.swa_decode(di.q[i, b:b + 1].cpu(), kh, vh, [p], w.window, w.n_sink, w.scale)
            assert_close(out[b:b + 1], ro, f"{name} step {i} b {b} out")
            assert_close(lse[b:b + 1], rl, f"{name} step {i} b {b} lse")


def test_decode_workload_sampled_f32_output_strict_bound():
    """The decode workload with a float32 output: the kernels' arithmetic is held to
    max-abs 1e-2 and mean-abs 1e-3 with no allowance for a final bf16 rounding."""
    _decode_workload_check("decode", 2, (0, 21, 63), torch.float32)


@pytest.mark.parametrize("out_dtype", [torch.bfloat16, torch.float32])
def test_decode_single_sequence_workload(out_dtype):
    """One sequence (B=1, Hq=32, Hkv=8, d=128, window 4096 + 4 sinks) after a 16384-token
    prefix: the split grid is sized by the visible keys, not the GPU."""
    _decode_workload_check("decode_b1", 3, (0,), out_dtype)


def test_decode_early_positions_few_keys():
    """Positions 0..5 of a single sequence: far fewer keys than warps in the grid, so
    most warps take no piece and every piece still holds a key."""
    B, Hq, Hkv, d, W, S = 1, 32, 8, 128, 4096, 4
    n = 6
    k, v, q = rand((B, n, Hkv, d), 17), rand((B, n, Hkv, d), 18), rand((B, n, Hq, d), 19)
    c = Cache(B, Hkv, d, W, S)
    for p in range(n):
        pos = torch.full((B,), p, dtype=torch.int32, device="cuda")
        c.append(k[:, p], v[:, p], pos)
        out, lse = decode(c, q[:, p], pos, Hkv)
        ro, rl = oracle.swa_decode(q[:, p], k, v, [p], W, S, 1 / math.sqrt(d))
        assert_close(out, ro, f"pos {p} out")
        assert_close(lse, rl, f"pos {p} lse")
