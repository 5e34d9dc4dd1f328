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
