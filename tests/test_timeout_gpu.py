"""Failure detection without a GPU fault: every device-side barrier wait of the
prefill kernels has a time limit.  A test hook makes the load warp issue no
copies, so the waits run out; the kernel must report SWA_ERR_DEVICE_TIMEOUT,
free its tensor memory and return, and the context must stay usable."""
import math

import pytest
import torch

import oracle
import sink_aware_sliding_b200 as swa
from tests.helpers import assert_close

pytestmark = pytest.mark.gpu


def _inputs(Hq, Hkv, d=128, L=512):
    g = torch.Generator().manual_seed(5)
    q = torch.randn(1, L, Hq, d, generator=g).bfloat16()
    k = torch.randn(1, L, Hkv, d, generator=g).bfloat16()
    v = torch.randn(1, L, Hkv, d, generator=g).bfloat16()
    return q, k, v


@pytest.mark.parametrize("kernel_flags", [0, 2], ids=["two-tile", "one-tile"])
def test_expired_wait_reports_timeout_and_context_survives(kernel_flags):
    q, k, v = _inputs(8, 2)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    out = torch.zeros_like(qd)
    lse = torch.zeros(1, 8, 512, device="cuda")
    assert swa.swa_device_error() == 0
    prev_t = swa.swa_set_wait_timeout_ns(50_000_000)          # 50 ms
    prev_f = swa.swa_set_debug_flags(1 | kernel_flags)
    try:
        swa.swa_fwd(qd, kd, vd, out, lse, 128, 4)
        assert swa.swa_device_error() == swa.SWA_ERR_DEVICE_TIMEOUT
        assert swa.swa_device_error() == 0                     # reading clears it
    finally:
        swa.swa_set_debug_flags(prev_f)
        swa.swa_set_wait_timeout_ns(prev_t)
    # the same call now runs normally on the same context
    swa.swa_fwd(qd, kd, vd, out, lse, 128, 4)
    assert swa.swa_device_error() == 0
    ro, rl = oracle.swa_fwd(q, k, v, 128, 4, 1 / math.sqrt(128))
    assert_close(out, ro, "after timeout: out")
    assert_close(lse, rl, "after timeout: lse")

