"""Shared test helpers: tolerances and comparison against the oracle."""
import numpy as np
import torch

# Bounds for bf16 inputs with fp32 accumulation, as the method's acceptance
# criterion states: max-abs 1e-2 and mean-abs 1e-3 on outputs (and on LSE).
MAX_ABS = 1e-2
MEAN_ABS = 1e-3


def to64(t) -> np.ndarray:
    if isinstance(t, np.ndarray):
        return t.astype(np.float64)
    return t.detach().to("cpu", torch.float64).numpy()


def bf16_half_ulp(x: np.ndarray) -> np.ndarray:
    """Half the spacing of bf16 numbers at |x| (8 significant bits): the largest
    error of rounding x to bf16 with round-to-nearest-even."""
    ax = np.abs(x)
    e = np.floor(np.log2(np.where(ax > 0, ax, 1.0)))
    return np.where(ax > 0, 2.0 ** (e - 8), 2.0 ** -134)


def assert_close(got, want, what: str, max_abs: float = MAX_ABS, mean_abs: float = MEAN_ABS):
    """max|got - want| <= max_abs and mean|got - want| <= mean_abs.

    When ``got`` is a bf16 tensor, each element may in addition differ by the
    half-ulp of rounding the exact value to bf16: a bf16 output cannot hold the
    oracle's value more closely than that (half an ulp is 0.0156 at |x| in [4, 8),
    above the 1e-2 bound by itself).  The mean bound takes the mean of the same
    allowance: if the fp32 result g32 meets mean|g32 - want| <= mean_abs, then
    bf16(g32) meets mean|bf16(g32) - want| <= mean_abs + mean(half-ulp), and
    nothing tighter holds for O(1) outputs, whose rounding alone averages about
    a quarter ulp (0.002 at |x| near 1.5).  The strict bounds are checked on the
    fp32-output modes of the same kernels.
    """
    out_bf16 = hasattr(got, "dtype") and got.dtype == torch.bfloat16
    g, w = to64(got), to64(want)
    assert g.shape == w.shape, f"{what}: shape {g.shape} vs {w.shape}"
    assert np.isfinite(g).all(), f"{what}: non-finite values"
    err = np.abs(g - w)
    hu = bf16_half_ulp(w) if out_bf16 else np.zeros_like(w)
    allow = max_abs + hu
    excess = float((err - allow).max()) if err.size else -1.0
    mx, mn = float(err.max()) if err.size else 0.0, float(err.mean()) if err.size else 0.0
    mean_allow = mean_abs + (float(hu.mean()) if err.size else 0.0)
    assert excess <= 0 and mn <= mean_allow, (
        f"{what}: max_abs={mx:.3e} (allowance exceeded by {excess:.3e}) mean_abs={mn:.3e}")
    return mx, mn
