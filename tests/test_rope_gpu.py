"""GPU parity of the rotary position encoding: in-place q/k rotation, the fused
rotate-then-append of a decode step, and the decode kernel that rotates its
query itself (all through the C ABI), against the oracle's fp64 rotation.

Rotated values are stored in bf16, so an element may differ from the exact
rotation by half a bf16 ulp (correct rounding) plus the fp32 rotation error,
bounded here by 2e-6 of the pair's length.  Attention results built on rotated
inputs are compared with the oracle's attention over bf16-rounded rotations
(the kernels consume bf16 operands), under the usual bounds."""
import math

import numpy as np
import pytest
import torch

import oracle
import sink_aware_sliding_b200 as swa
from tests.helpers import assert_close, bf16_half_ulp

pytestmark = pytest.mark.gpu
BASE = 10000.0


def rand(shape, seed):
    g = torch.Generator().manual_seed(seed)
    return torch.randn(*shape, generator=g).bfloat16()


def bf16(x64: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(x64)).float().bfloat16()


def assert_rotation_close(got, want, what):
    g = got.detach().cpu().double().numpy()
    d = want.shape[-1]
    mag = np.sqrt(want[..., : d // 2] ** 2 + want[..., d // 2:] ** 2)
    mag = np.concatenate([mag, mag], axis=-1)
    err = np.abs(g - want)
    tol = bf16_half_ulp(want) + 2e-6 * mag + 1e-30
    worst = float((err - tol).max())
    assert worst <= 0, f"{what}: exceeds the rotation bound by {worst:.3e} (max err {err.max():.3e})"


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("kind", ["qk", "q_only", "k_only"])
def test_rope_qk_matches_oracle(d, kind):
    T, Hq, Hkv = 300, 8, 2
    q, k = rand((T, Hq, d), 1), rand((T, Hkv, d), 2)
    rng = np.random.default_rng(d)
    pos = np.concatenate([[0, 1, 2, 4095, 4096, 131071, 10 ** 9, 2 ** 31 - 1],
                          rng.integers(0, 300000, T - 8)]).astype(np.int32)
    pos_d = torch.from_numpy(pos).cuda()
    qd, kd = q.cuda(), k.cuda()
    if kind == "qk":
        swa.swa_rope_qk(qd, kd, pos_d, BASE)
    elif kind == "q_only":
        swa.swa_rope_qk(qd, None, pos_d, BASE)
    else:
        swa.swa_rope_qk(kd, None, pos_d, BASE)
    torch.cuda.synchronize()
    if kind in ("qk", "q_only"):
        assert_rotation_close(qd, oracle.rope(q, pos, BASE), "q")
    else:
        assert torch.equal(qd.cpu(), q)
    if kind in ("qk", "k_only"):
        assert_rotation_close(kd, oracle.rope(k, pos, BASE), "k")
    else:
        assert torch.equal(kd.cpu(), k)


def test_rope_qk_other_base_and_batch_layout():
    B, L, Hq, Hkv, d = 3, 70, 4, 4, 128
    q, k = rand((B, L, Hq, d), 3), rand((B, L, Hkv, d), 4)
    pos = np.tile(np.arange(L, dtype=np.int32), B)
    qd, kd = q.cuda(), k.cuda()
    swa.swa_rope_qk(qd, kd, torch.from_numpy(pos).cuda(), 500000.0)
    torch.cuda.synchronize()
    assert_rotation_close(qd, oracle.rope(q.reshape(B * L, Hq, d), pos, 500000.0).reshape(B, L, Hq, d), "q")
    assert_rotation_close(kd, oracle.rope(k.reshape(B * L, Hkv, d), pos, 500000.0).reshape(B, L, Hkv, d), "k")


def test_rope_cache_append_matches_oracle():
    B, Hkv, d, W, S = 4, 2, 128, 16, 3
    z = dict(device="cuda", dtype=torch.bfloat16)
    kc, vc = torch.zeros(B, Hkv, W, d, **z), torch.zeros(B, Hkv, W, d, **z)
    sk, sv = torch.zeros(B, Hkv, S, d, **z), torch.zeros(B, Hkv, S, d, **z)
    okc, ovc = np.zeros((B, Hkv, W, d)), np.zeros((B, Hkv, W, d))
    osk, osv = np.zeros((B, Hkv, S, d)), np.zeros((B, Hkv, S, d))
    start = np.array([0, 2, 15, 100000])
    for step in range(40):
        pos = start + step
        kn, vn = rand((B, Hkv, d), 100 + step), rand((B, Hkv, d), 200 + step)
        swa.swa_rope_cache_append(kn.cuda(), vn.cuda(), torch.tensor(pos, dtype=torch.int32, device="cuda"),
                                  kc, vc, sk, sv, W, S, BASE)
        oracle.ring_append(okc, ovc, osk, osv, oracle.rope(kn, pos, BASE), vn.double().numpy(), pos, W, S)
    torch.cuda.synchronize()
    assert_rotation_close(kc, okc, "ring keys")
    assert_rotation_close(sk, osk, "sink keys")
    np.testing.assert_array_equal(vc.cpu().double().numpy(), ovc)
    np.testing.assert_array_equal(sv.cpu().double().numpy(), osv)


def _rotated_history(k):
    """bf16(rope(k[b])) for every sequence b of k [B, P, Hkv, d], positions 0..P-1."""
    B, P = k.shape[:2]
    return torch.stack([bf16(oracle.rope(k[b], np.arange(P), BASE)) for b in range(B)])


@pytest.mark.parametrize("Hq,Hkv,d", [(8, 2, 128), (4, 4, 64), (6, 2, 64)])
def test_decode_rope_matches_oracle_at_mixed_positions(Hq, Hkv, d):
    W, S = 64, 4
    pos = [0, 3, 62, 63, 64, 67, 200, 1000]
    B, P = len(pos), max(pos) + 1
    k, v, q = rand((B, P, Hkv, d), 1), rand((B, P, Hkv, d), 2), rand((B, Hq, d), 3)
    z = dict(device="cuda", dtype=torch.bfloat16)
    kc, vc = torch.zeros(B, Hkv, W, d, **z), torch.zeros(B, Hkv, W, d, **z)
    sk, sv = torch.zeros(B, Hkv, S, d, **z), torch.zeros(B, Hkv, S, d, **z)
    for b in range(B):
        # positions 0 .. pos[b]-1 rotated on the device, then filled; pos[b] appended below
        if pos[b] > 0:
            kb = k[b:b + 1, :pos[b]].cuda().contiguous()
            swa.swa_rope_qk(kb, None, torch.arange(pos[b], dtype=torch.int32, device="cuda"), BASE)
            one = [t[b:b + 1] for t in (kc, vc, sk, sv)]
            tmp = [torch.zeros_like(t) for t in one]
            swa.swa_cache_fill(kb, v[b:b + 1, :pos[b]].cuda().contiguous(), *tmp, W, S)
            for dst, src in zip(one, tmp):
                dst.copy_(src)
    pos_d = torch.tensor(pos, dtype=torch.int32, device="cuda")
    idx = torch.arange(B)
    swa.swa_rope_cache_append(k[idx, pos].cuda().contiguous(), v[idx, pos].cuda().contiguous(), pos_d,
                              kc, vc, sk, sv, W, S, BASE)
    out = torch.empty(B, Hq, d, **z)
    lse = torch.empty(B, Hq, device="cuda", dtype=torch.float32)
    ws = torch.empty(swa.swa_decode_workspace_bytes(B, Hq, Hkv, d, W, S), device="cuda", dtype=torch.uint8)
    swa.swa_decode_rope(q.cuda(), kc, vc, sk, sv, pos_d, out, lse, W, S, ws, BASE)
    torch.cuda.synchronize()
    q_rot = bf16(oracle.rope(q, pos, BASE))
    ro, rl = oracle.swa_decode(q_rot, _rotated_history(k), v, pos, W, S, 1 / math.sqrt(d))
    assert_close(out, ro, "decode_rope out")
    assert_close(lse, rl, "decode_rope lse")


def test_prefill_then_decode_with_rope():
    """Prefill on rotated q/k, then decode steps that rotate on the device, against the
    oracle's prefill rows of the whole rotated sequence."""
    B, Hq, Hkv, d, W, S, P, n_dec = 2, 8, 2, 128, 96, 4, 300, 4
    n = P + n_dec
    q, k, v = rand((B, n, Hq, d), 11), rand((B, n, Hkv, d), 12), rand((B, n, Hkv, d), 13)
    pos_all = np.tile(np.arange(P, dtype=np.int32), B)
    qd, kd, vd = q[:, :P].cuda().contiguous(), k[:, :P].cuda().contiguous(), v[:, :P].cuda().contiguous()
    swa.swa_rope_qk(qd, kd, torch.from_numpy(pos_all).cuda(), BASE)
    out = torch.empty(B, P, Hq, d, device="cuda", dtype=torch.bfloat16)
    lse = torch.empty(B, Hq, P, device="cuda", dtype=torch.float32)
    swa.swa_fwd(qd, kd, vd, out, lse, W, S)
    z = dict(device="cuda", dtype=torch.bfloat16)
    kc, vc = torch.zeros(B, Hkv, W, d, **z), torch.zeros(B, Hkv, W, d, **z)
    sk, sv = torch.zeros(B, Hkv, S, d, **z), torch.zeros(B, Hkv, S, d, **z)
    swa.swa_cache_fill(kd, vd, kc, vc, sk, sv, W, S)
    ws = torch.empty(swa.swa_decode_workspace_bytes(B, Hq, Hkv, d, W, S), device="cuda", dtype=torch.uint8)
    dec_out, dec_lse = [], []
    for i in range(n_dec):
        p = P + i
        pos = torch.full((B,), p, dtype=torch.int32, device="cuda")
        swa.swa_rope_cache_append(k[:, p].cuda().contiguous(), v[:, p].cuda().contiguous(), pos,
                                  kc, vc, sk, sv, W, S, BASE)
        o = torch.empty(B, Hq, d, **z)
        l_ = torch.empty(B, Hq, device="cuda", dtype=torch.float32)
        swa.swa_decode_rope(q[:, p].cuda().contiguous(), kc, vc, sk, sv, pos, o, l_, W, S, ws, BASE)
        dec_out.append(o)
        dec_lse.append(l_)
    torch.cuda.synchronize()
    qr = torch.stack([bf16(oracle.rope(q[b], np.arange(n), BASE)) for b in range(B)])
    kr = torch.stack([bf16(oracle.rope(k[b], np.arange(n), BASE)) for b in range(B)])
    ro, rl = oracle.swa_fwd(qr, kr, v, W, S, 1 / math.sqrt(d))
    assert_close(out, ro[:, :P], "rope prefill out")
    assert_close(lse, rl[:, :, :P], "rope prefill lse")
    for i in range(n_dec):
        assert_close(dec_out[i], ro[:, P + i], f"rope decode step {i} out")
        assert_close(dec_lse[i], rl[:, :, P + i], f"rope decode step {i} lse")
