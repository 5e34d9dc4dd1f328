"""GPU parity of the Hadamard output projection against the oracle (C ABI)."""
import numpy as np
import pytest
import torch

import oracle
import sink_aware_sliding_b200 as swa
from tests.helpers import assert_close

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("n,rows", [(32, 5), (64, 130), (128, 7), (256, 33), (512, 3), (1024, 300),
                                    (2048, 65), (4096, 77), (8192, 9)])
def test_hadamard_matches_oracle(n, rows):
    g = torch.Generator().manual_seed(n + rows)
    y = torch.randn(rows, n, generator=g).bfloat16()
    alpha = torch.randn(n, generator=g) * 0.5 + 1.0
    beta = torch.randn(n, generator=g) * 0.1
    want = oracle.hadamard_proj(y, alpha, beta)
    for dt in (torch.float32, torch.bfloat16):
        z = torch.empty(rows, n, device="cuda", dtype=dt)
        swa.swa_hadamard_proj(y.cuda(), alpha.cuda(), beta.cuda(), z)
        torch.cuda.synchronize()
        assert_close(z, want, f"n={n} rows={rows} out={dt}")


def test_hadamard_of_attention_output_layout():
    """The projection reads the prefill output [T, Hq, d] as rows of n = Hq * d."""
    T, Hq, d = 96, 32, 128
    g = torch.Generator().manual_seed(3)
    y = torch.randn(T, Hq, d, generator=g).bfloat16()
    alpha, beta = torch.ones(Hq * d), torch.zeros(Hq * d)
    z = torch.empty(T, Hq, d, device="cuda", dtype=torch.float32)
    swa.swa_hadamard_proj(y.cuda(), alpha.cuda(), beta.cuda(), z)
    torch.cuda.synchronize()
    want = oracle.hadamard_proj(y.reshape(T, -1), alpha, beta).reshape(T, Hq, d)
    assert_close(z, want, "attention layout")
    # orthonormal: the l2 norm of every row is kept
    np.testing.assert_allclose(z.cpu().double().reshape(T, -1).norm(dim=1).numpy(),
                               y.double().reshape(T, -1).norm(dim=1).numpy(), rtol=1e-5)


def test_hadamard_full_size_sampled_rows():
    """The benchmark's projection (32768 x 4096) in its launch configuration; rows sampled."""
    import workloads as wl
    w = wl.PROJ_WORKLOADS["hadamard_proj"]
    y, alpha, beta = wl.make_hadamard(w, device="cuda")
    z = torch.empty_like(y)
    swa.swa_hadamard_proj(y, alpha, beta, z)
    torch.cuda.synchronize()
    g = torch.Generator().manual_seed(11)
    rows = sorted(set([0, 1, w.T - 1] + torch.randint(0, w.T, (61,), generator=g).tolist()))
    idx = torch.tensor(rows)
    want = oracle.hadamard_proj(y.cpu()[idx], alpha.cpu(), beta.cpu())
    assert_close(z.cpu()[idx], want, "hadamard full size")
