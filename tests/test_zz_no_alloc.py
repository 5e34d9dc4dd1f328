"""swa_decode_noalloc: the decode step for callers that cannot allocate device
memory (their host framework owns every allocation, or allocation is forbidden
after start-up).  It must give the same results as swa_decode, which takes its
scratch from the caller, on two calls in a row that share the library's fixed
scratch array.

The file name sorts last so that pytest collects it after every other test file:
a run that stops at the first failure has then run everything else first, and the
array is exercised after the other tests have used the library on the same
device.  Nothing here depends on what the other tests did: the cases also pass in
a fresh process."""
import ctypes
import math

import pytest
import torch

import oracle
import sink_aware_sliding_b200 as swa
from tests.helpers import assert_close

pytestmark = pytest.mark.gpu


def _setup(B, Hq, Hkv, d, W, S, pos, seed):
    g = torch.Generator().manual_seed(seed)
    P = max(pos) + 1
    k = torch.randn(B, P, Hkv, d, generator=g).bfloat16()
    v = torch.randn(B, P, Hkv, d, generator=g).bfloat16()
    z = dict(device="cuda", dtype=torch.bfloat16)
    kc, vc = torch.zeros(B, Hkv, W, d, **z), torch.zeros(B, Hkv, W, d, **z)
    sk, sv = torch.zeros(B, Hkv, S, d, **z), torch.zeros(B, Hkv, S, d, **z)
    for b in range(B):
        # cache of sequence b holds positions 0..pos[b]
        swa.swa_cache_fill(k[b:b + 1, :pos[b] + 1].cuda().contiguous(), v[b:b + 1, :pos[b] + 1].cuda().contiguous(),
                           kc[b:b + 1], vc[b:b + 1], sk[b:b + 1], sv[b:b + 1], W, S)
    return k, v, (kc, vc, sk, sv)


def test_noalloc_matches_decode_on_two_calls_in_a_row():
    B, Hq, Hkv, d, W, S = 6, 8, 2, 128, 64, 4
    pos = [0, 5, 63, 64, 70, 300]
    k, v, (kc, vc, sk, sv) = _setup(B, Hq, Hkv, d, W, S, pos, seed=1)
    pos_d = torch.tensor(pos, dtype=torch.int32, device="cuda")
    ws = torch.empty(swa.swa_decode_workspace_bytes(B, Hq, Hkv, d, W, S), dtype=torch.uint8, device="cuda")
    for call in range(2):
        q = torch.randn(B, Hq, d, generator=torch.Generator().manual_seed(10 + call)).bfloat16().cuda()
        ref_out = torch.empty(B, Hq, d, device="cuda", dtype=torch.bfloat16)
        ref_lse = torch.empty(B, Hq, device="cuda", dtype=torch.float32)
        swa.swa_decode(q, kc, vc, sk, sv, pos_d, ref_out, ref_lse, W, S, ws)
        out = torch.empty_like(ref_out)
        lse = torch.empty_like(ref_lse)
        swa.swa_decode_noalloc(q, kc, vc, sk, sv, pos_d, out, lse, W, S)
        torch.cuda.synchronize()
        assert_close(out, ref_out.double(), f"call {call} out vs swa_decode")
        assert_close(lse, ref_lse, f"call {call} lse vs swa_decode")
        # and both against the definition
        ro, rl = oracle.swa_decode(q, k, v, pos, W, S, 1 / math.sqrt(d))
        assert_close(out, ro, f"call {call} out vs oracle")
        assert_close(lse, rl, f"call {call} lse vs oracle")


def test_noalloc_larger_then_smaller_batch_d64_no_sinks_no_lse():
    """A call with more sequences leaves partial states in the shared array beyond
    what the next, smaller call writes; the smaller call (d = 64, no sinks, no lse)
    must not read them."""
    Hq, Hkv, d, W, S = 4, 2, 64, 48, 0
    for B, pos, seed in ((7, [0, 9, 47, 48, 60, 130, 200], 3), (2, [5, 100], 4)):
        k, v, (kc, vc, sk, sv) = _setup(B, Hq, Hkv, d, W, S, pos, seed=seed)
        pos_d = torch.tensor(pos, dtype=torch.int32, device="cuda")
        ws = torch.empty(swa.swa_decode_workspace_bytes(B, Hq, Hkv, d, W, S), dtype=torch.uint8, device="cuda")
        q = torch.randn(B, Hq, d, generator=torch.Generator().manual_seed(20 + B)).bfloat16().cuda()
        ref = torch.empty(B, Hq, d, device="cuda", dtype=torch.bfloat16)
        swa.swa_decode(q, kc, vc, sk, sv, pos_d, ref, None, W, S, ws)
        out = torch.empty_like(ref)
        swa.swa_decode_noalloc(q, kc, vc, sk, sv, pos_d, out, None, W, S)
        torch.cuda.synchronize()
        assert_close(out, ref.double(), f"B={B} out vs swa_decode")
        ro, _ = oracle.swa_decode(q, k, v, pos, W, S, 1 / math.sqrt(d))
        assert_close(out, ro, f"B={B} out vs oracle")


def test_noalloc_rejects_sizes_beyond_its_scratch():
    # 4096 sequences x 8 KV heads need far more than the fixed 8 MiB of scratch; the
    # arguments are otherwise valid, so the size is what is rejected.
    B, Hq, Hkv, d, W, S = 4096, 32, 8, 128, 4096, 4
    need = swa.swa_decode_workspace_bytes(B, Hq, Hkv, d, W, S)
    assert need > 8 << 20
    z = dict(device="cuda", dtype=torch.bfloat16)
    q = torch.zeros(B, Hq, d, **z)
    kc = torch.zeros(B, Hkv, 16, d, **z)          # only pointers are checked before the size
    sk = torch.zeros(B, Hkv, S, d, **z)
    pos = torch.zeros(B, dtype=torch.int32, device="cuda")
    out = torch.empty_like(q)
    with pytest.raises(swa.SwaError) as e:
        swa.swa_decode_noalloc(q, kc, kc, sk, sk, pos, out, None, W, S)
    assert e.value.status == swa.SWA_ERR_UNSUPPORTED
    # invalid arguments are reported as such whatever the size
    lib = swa.library()
    st = lib.swa_decode_noalloc(None, None, None, None, None, None, None, None, B, Hq, Hkv, d, W, S,
                                ctypes.c_float(0.1), None)
    assert st == swa.SWA_ERR_INVALID_ARG
