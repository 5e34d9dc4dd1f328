"""GPU parity of a hybrid decode step (the Based layer's two branches side by
side): the window branch appends to its ring cache and decodes over it (d = 64,
window 128, no sinks) and the linear branch takes its recurrent step on the state
its prefill left, each against the oracle, for a few generated tokens."""
import math

import numpy as np
import pytest
import torch

import oracle
import sink_aware_sliding_b200 as swa
import workloads
from tests.helpers import assert_close

pytestmark = pytest.mark.gpu


def test_hybrid_decode_steps():
    B, H, d, W, P, n = 2, 2, 64, 128, 200, 3
    g = torch.Generator().manual_seed(17)
    k = torch.randn(B, P + n, H, d, generator=g).bfloat16()
    v = torch.randn(B, P + n, H, d, generator=g).bfloat16()
    q = torch.randn(B, P + n, H, d, generator=g).bfloat16()
    lw = workloads.LinearWorkload("t", B=B, L=P + n, H=H, dk=16, dv=64)
    ql, kl, vl = workloads.make_based_linear(lw, seed=23)
    dev = "cuda"
    z16 = dict(device=dev, dtype=torch.bfloat16)
    kc, vc = torch.zeros(B, H, W, d, **z16), torch.zeros(B, H, W, d, **z16)
    sk = torch.zeros(B, H, 1, d, **z16)
    swa.swa_cache_fill(k[:, :P].contiguous().to(dev), v[:, :P].contiguous().to(dev), kc, vc, sk, sk, W, 0)
    S = torch.empty(B, H, lw.F, lw.dv, device=dev)
    zs = torch.empty(B, H, lw.F, device=dev)
    swa.swa_based_linear_fwd(ql[:, :P].contiguous().to(dev), kl[:, :P].contiguous().to(dev),
                             vl[:, :P].contiguous().to(dev), torch.empty(B, P, H, lw.dv, device=dev), S, zs,
                             lw.scale)
    ws = torch.empty(swa.swa_decode_workspace_bytes(B, H, H, d, W, 0), device=dev, dtype=torch.uint8)
    out_w = torch.empty(B, H, d, device=dev, dtype=torch.bfloat16)
    lse = torch.empty(B, H, device=dev)
    out_l = torch.empty(B, H, lw.dv, device=dev)
    full_l = oracle.based_linear_fwd(ql, kl, vl, lw.scale)
    for t in range(P, P + n):
        pos = torch.full((B,), t, dtype=torch.int32, device=dev)
        swa.swa_cache_append(k[:, t].contiguous().to(dev), v[:, t].contiguous().to(dev), pos, kc, vc, sk, sk, W, 0)
        swa.swa_decode(q[:, t].contiguous().to(dev), kc, vc, sk, sk, pos, out_w, lse, W, 0, ws)
        swa.swa_based_linear_decode(ql[:, t].contiguous().to(dev), kl[:, t].contiguous().to(dev),
                                    vl[:, t].contiguous().to(dev), S, zs, out_l, lw.scale)
        torch.cuda.synchronize()
        assert swa.swa_device_error() == 0
        ro, rl = oracle.swa_decode(q[:, t], k, v, [t] * B, W, 0, 1.0 / math.sqrt(d))
        assert_close(out_w, ro, f"window branch, position {t}")
        assert_close(lse, rl, f"window branch lse, position {t}")
        assert_close(out_l, full_l[:, t], f"linear branch, position {t}")


@pytest.mark.parametrize("Hq,Hkv,W,S,P", [(2, 2, 128, 0, 200), (4, 2, 64, 4, 70), (4, 1, 32, 3, 2)])
def test_fused_hybrid_decode_steps(Hq, Hkv, W, S, P):
    """swa_hybrid_decode (both branches in one launch) against the oracle for a few
    generated tokens, and its cache contents against swa_cache_append's, bit for bit.
    Covers grouped query heads (one block per query head reads the KV head another
    block appends to), sinks, the ring's wrap-around and a prefix shorter than the
    window."""
    B, d, n = 2, 64, 4
    g = torch.Generator().manual_seed(31 + Hq + W)
    k = torch.randn(B, P + n, Hkv, d, generator=g).bfloat16()
    v = torch.randn(B, P + n, Hkv, d, generator=g).bfloat16()
    q = torch.randn(B, P + n, Hq, d, generator=g).bfloat16()
    Hl = 3
    lw = workloads.LinearWorkload("t", B=B, L=P + n, H=Hl, dk=16, dv=64)
    ql, kl, vl = workloads.make_based_linear(lw, seed=29)
    dev = "cuda"
    z16 = dict(device=dev, dtype=torch.bfloat16)
    caches = []
    for _ in range(2):                     # fused, and the separate append as reference
        kc, vc = torch.zeros(B, Hkv, W, d, **z16), torch.zeros(B, Hkv, W, d, **z16)
        sk, sv = torch.zeros(B, Hkv, max(S, 1), d, **z16), torch.zeros(B, Hkv, max(S, 1), d, **z16)
        swa.swa_cache_fill(k[:, :P].contiguous().to(dev), v[:, :P].contiguous().to(dev), kc, vc, sk, sv, W, S)
        caches.append((kc, vc, sk, sv))
    S_l = torch.empty(B, Hl, lw.F, lw.dv, device=dev)
    z_l = torch.empty(B, Hl, lw.F, device=dev)
    swa.swa_based_linear_fwd(ql[:, :P].contiguous().to(dev), kl[:, :P].contiguous().to(dev),
                             vl[:, :P].contiguous().to(dev), torch.empty(B, P, Hl, lw.dv, device=dev), S_l, z_l,
                             lw.scale)
    out_w = torch.empty(B, Hq, d, **z16)
    lse = torch.empty(B, Hq, device=dev)
    out_l = torch.empty(B, Hl, lw.dv, **z16)
    full_l = oracle.based_linear_fwd(ql, kl, vl, lw.scale)
    kc, vc, sk, sv = caches[0]
    for t in range(P, P + n):
        pos = torch.full((B,), t, dtype=torch.int32, device=dev)
        kn, vn = k[:, t].contiguous().to(dev), v[:, t].contiguous().to(dev)
        swa.swa_hybrid_decode(q[:, t].contiguous().to(dev), kn, vn, pos, kc, vc, sk, sv, out_w, lse, W, S,
                              ql[:, t].contiguous().to(dev), kl[:, t].contiguous().to(dev),
                              vl[:, t].contiguous().to(dev), S_l, z_l, out_l, scale_l=lw.scale)
        rk, rv, rsk, rsv = caches[1]
        swa.swa_cache_append(kn, vn, pos, rk, rv, rsk, rsv, W, S)
        torch.cuda.synchronize()
        assert swa.swa_device_error() == 0
        ro, rl = oracle.swa_decode(q[:, t], k, v, [t] * B, W, S, 1.0 / math.sqrt(d))
        assert_close(out_w, ro, f"window branch, position {t}")
        assert_close(lse, rl, f"window branch lse, position {t}")
        assert_close(out_l, full_l[:, t], f"linear branch, position {t}")
        for a_, b_ in zip(caches[0], caches[1]):
            assert torch.equal(a_, b_), f"cache contents differ after position {t}"


def test_fused_hybrid_decode_rejects_unsupported():
    z = torch.zeros(1, 1, 128, device="cuda", dtype=torch.bfloat16)
    pos = torch.zeros(1, dtype=torch.int32, device="cuda")
    st = torch.zeros(1, 1, 273, 64, device="cuda")
    zs = torch.zeros(1, 1, 273, device="cuda")
    ql = torch.zeros(1, 1, 16, device="cuda", dtype=torch.bfloat16)
    vl = torch.zeros(1, 1, 64, device="cuda", dtype=torch.bfloat16)
    with pytest.raises(swa.SwaError) as e:          # d = 128: the fused window branch is d = 64 only
        swa.swa_hybrid_decode(z, z, z, pos, z, z, None, None, z, None, 4, 0, ql, ql, vl, st, zs, vl)
    assert e.value.status == swa.SWA_ERR_UNSUPPORTED
