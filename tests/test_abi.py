"""The C-ABI library loads and exports what include/swa.h declares (no GPU needed)."""
import ctypes
import os
import re

import pytest

import sink_aware_sliding_b200 as swa
from sink_aware_sliding_b200 import build as swa_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "swa.h")


@pytest.fixture(scope="module")
def lib():
    swa_build.build()
    return swa.library()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(swa_[a-z_0-9]+)\s*\(", text)))


def test_header_declares_the_binding_exports():
    assert declared_functions() == sorted(swa.EXPORTS)


def test_every_declared_symbol_is_exported(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name
        ctypes.cast(getattr(lib, name), ctypes.c_void_p)


def test_status_strings(lib):
    assert swa.swa_status_string(0) == "ok"
    assert "invalid" in swa.swa_status_string(1)
    assert "timed out" in swa.swa_status_string(4)
    assert swa.swa_status_string(99) == "unknown status"
    assert swa.swa_version() == 0x000100


def _fwd(lib, **kw):
    args = dict(q=None, k=None, v=None, out=None, lse=None, B=1, Hq=4, Hkv=2, L=16, d=128,
                window=8, n_sink=4, scale=0.1, dtype=0, stream=None)
    args.update(kw)
    return lib.swa_fwd(args["q"], args["k"], args["v"], args["out"], args["lse"], args["B"],
                       args["Hq"], args["Hkv"], args["L"], args["d"], args["window"],
                       args["n_sink"], ctypes.c_float(args["scale"]), args["dtype"], args["stream"])


def test_argument_checks_happen_before_any_device_work(lib):
    # These all return from host-side validation without touching CUDA.
    assert _fwd(lib, Hq=3, Hkv=2) == swa.SWA_ERR_INVALID_ARG
    assert _fwd(lib, window=0) == swa.SWA_ERR_INVALID_ARG
    assert _fwd(lib, n_sink=-1) == swa.SWA_ERR_INVALID_ARG
    assert _fwd(lib, scale=0.0) == swa.SWA_ERR_INVALID_ARG
    assert _fwd(lib, scale=float("inf")) == swa.SWA_ERR_INVALID_ARG
    assert _fwd(lib, dtype=7) == swa.SWA_ERR_INVALID_ARG
    assert _fwd(lib, d=96) == swa.SWA_ERR_UNSUPPORTED
    assert _fwd(lib, d=128, dtype=1) == swa.SWA_ERR_UNSUPPORTED
    assert _fwd(lib, B=0) == swa.SWA_OK                     # empty: nothing to launch
    assert _fwd(lib, L=0) == swa.SWA_OK
    assert _fwd(lib) == swa.SWA_ERR_INVALID_ARG             # null pointers
    assert _fwd(lib, q=16, k=32, v=48, out=64 + 8) == swa.SWA_ERR_INVALID_ARG  # misaligned
    assert lib.swa_decode_workspace_bytes(1, 12, 1, 128, 64, 4) == 0    # G = 12 > 8
    assert lib.swa_decode_workspace_bytes(1, 4, 3, 128, 64, 4) == 0     # Hq % Hkv != 0
    assert lib.swa_decode_workspace_bytes(1, 4, 1, 80, 64, 4) == 0      # d = 80


def test_rope_and_hadamard_argument_checks(lib):
    D = ctypes.c_double
    # rotary encoding: the base and d are checked first, then empty work returns OK
    assert lib.swa_rope_qk(None, None, None, 10, 4, 2, 128, D(0.0), None) == swa.SWA_ERR_INVALID_ARG
    assert lib.swa_rope_qk(None, None, None, 10, 4, 2, 128, D(float("nan")), None) == swa.SWA_ERR_INVALID_ARG
    assert lib.swa_rope_qk(None, None, None, -1, 4, 2, 128, D(1e4), None) == swa.SWA_ERR_INVALID_ARG
    assert lib.swa_rope_qk(None, None, None, 10, 4, 2, 96, D(1e4), None) == swa.SWA_ERR_UNSUPPORTED
    assert lib.swa_rope_qk(None, None, None, 0, 4, 2, 128, D(1e4), None) == swa.SWA_OK
    assert lib.swa_rope_qk(None, None, None, 10, 4, 2, 128, D(1e4), None) == swa.SWA_ERR_INVALID_ARG
    assert lib.swa_rope_cache_append(None, None, None, None, None, None, None, 1, 2, 128, 64, 4,
                                     D(-1.0), None) == swa.SWA_ERR_INVALID_ARG
    assert lib.swa_decode_rope(None, None, None, None, None, None, None, None, 1, 4, 2, 128, 64, 4,
                               ctypes.c_float(0.1), D(float("inf")), None, 0, None) == swa.SWA_ERR_INVALID_ARG
    # Hadamard projection: n must be a power of two in [32, 8192]
    for n in (16, 48, 16384):
        assert lib.swa_hadamard_proj(None, None, None, None, 4, n, 0, None) == swa.SWA_ERR_UNSUPPORTED
    assert lib.swa_hadamard_proj(None, None, None, None, 4, 64, 2, None) == swa.SWA_ERR_INVALID_ARG
    assert lib.swa_hadamard_proj(None, None, None, None, 0, 64, 0, None) == swa.SWA_OK
    assert lib.swa_hadamard_proj(None, None, None, None, 4, 64, 0, None) == swa.SWA_ERR_INVALID_ARG


def test_based_linear_argument_checks(lib):
    F = ctypes.c_float
    fwd = lambda **kw: lib.swa_based_linear_fwd(None, None, None, None, kw.get("state"), kw.get("zsum"),
                                                kw.get("B", 1), kw.get("L", 8), kw.get("H", 2), kw.get("dk", 16),
                                                kw.get("dv", 64), F(kw.get("scale", 0.25)), kw.get("dtype", 0), None)
    assert lib.swa_based_linear_state_features(16) == 273
    assert fwd(dk=32) == swa.SWA_ERR_UNSUPPORTED
    assert fwd(dv=128) == swa.SWA_ERR_UNSUPPORTED
    assert fwd(scale=0.0) == swa.SWA_ERR_INVALID_ARG
    assert fwd(dtype=7) == swa.SWA_ERR_INVALID_ARG
    assert fwd(H=0) == swa.SWA_ERR_INVALID_ARG
    assert fwd() == swa.SWA_ERR_INVALID_ARG                       # null tensors
    buf = ctypes.create_string_buffer(64)
    assert fwd(state=ctypes.addressof(buf)) == swa.SWA_ERR_INVALID_ARG   # state without zsum
    assert fwd(B=0) == swa.SWA_OK
    assert fwd(L=0) == swa.SWA_OK                                 # nothing to write
    dec = lambda **kw: lib.swa_based_linear_decode(None, None, None, None, None, None, kw.get("B", 1), 2,
                                                   kw.get("dk", 16), 64, F(0.25), 0, None)
    assert dec(dk=8) == swa.SWA_ERR_UNSUPPORTED
    assert dec() == swa.SWA_ERR_INVALID_ARG
    assert dec(B=0) == swa.SWA_OK


def test_based_linear_binding_checks_shapes(lib):
    # shape and dtype checks happen in the binding before any device work (CPU tensors)
    import torch
    bf = dict(dtype=torch.bfloat16)
    q = torch.zeros(1, 8, 2, 16, **bf)
    v = torch.zeros(1, 8, 2, 64, **bf)
    out = torch.zeros(1, 8, 2, 64, **bf)
    with pytest.raises(ValueError):
        swa.swa_based_linear_fwd(q, torch.zeros(1, 8, 2, 8, **bf), v, out)          # k shape
    with pytest.raises(ValueError):
        swa.swa_based_linear_fwd(q, q, v, torch.zeros(1, 8, 2, 32, **bf))          # out shape
    with pytest.raises(ValueError):
        swa.swa_based_linear_fwd(q, q, v, out, torch.zeros(1, 2, 100, 64), torch.zeros(1, 2, 100))
    with pytest.raises(ValueError):
        swa.swa_based_linear_fwd(q, q, v, out, torch.zeros(1, 2, 273, 64), None)
    qd = torch.zeros(1, 2, 16, **bf)
    vd = torch.zeros(1, 2, 64, **bf)
    with pytest.raises(ValueError):
        swa.swa_based_linear_decode(qd, qd, vd, torch.zeros(1, 2, 273, 64, dtype=torch.float64),
                                    torch.zeros(1, 2, 273), torch.zeros(1, 2, 64))
    with pytest.raises(ValueError):
        swa.swa_based_linear_decode(qd, qd, vd, torch.zeros(1, 2, 273, 64), torch.zeros(1, 2, 272),
                                    torch.zeros(1, 2, 64))


def test_decode_ex_hybrid_and_backward_argument_checks(lib):
    F = ctypes.c_float
    Z = ctypes.c_size_t(0)

    def dex(B=1, Hq=4, Hkv=2, d=128, W=64, S=4, scale=0.1, out_dtype=2):
        return lib.swa_decode_ex(None, None, None, None, None, None, None, None, B, Hq, Hkv, d, W, S,
                                 F(scale), out_dtype, None, Z, None)
    assert dex(out_dtype=1) == swa.SWA_ERR_INVALID_ARG            # f32 inputs: no decode
    assert dex(out_dtype=7) == swa.SWA_ERR_INVALID_ARG
    assert dex(scale=0.0) == swa.SWA_ERR_INVALID_ARG
    assert dex(Hq=3) == swa.SWA_ERR_INVALID_ARG
    assert dex(B=0) == swa.SWA_OK
    assert dex() == swa.SWA_ERR_INVALID_ARG                       # null tensors

    def hyb(B=1, Hq=4, Hkv=2, d=64, W=128, S=0, scale=0.125, H_l=2, dk=16, dv=64, scale_l=0.25):
        return lib.swa_hybrid_decode(None, None, None, None, None, None, None, None, None, None,
                                     B, Hq, Hkv, d, W, S, F(scale), None, None, None, None, None, None,
                                     H_l, dk, dv, F(scale_l), None)
    assert hyb(d=128) == swa.SWA_ERR_UNSUPPORTED                  # the window branch is d = 64 only
    assert hyb(W=600) == swa.SWA_ERR_UNSUPPORTED                  # window + sinks above 512 keys
    assert hyb(dk=8) == swa.SWA_ERR_UNSUPPORTED
    assert hyb(scale_l=0.0) == swa.SWA_ERR_INVALID_ARG
    assert hyb(Hq=3) == swa.SWA_ERR_INVALID_ARG
    assert hyb(H_l=0) == swa.SWA_ERR_INVALID_ARG
    assert hyb(B=0) == swa.SWA_OK
    assert hyb() == swa.SWA_ERR_INVALID_ARG                       # null tensors

    def bwd(B=1, Hq=4, Hkv=2, L=16, d=128, W=8, S=4, scale=0.1):
        return lib.swa_bwd(None, None, None, None, None, None, None, None, None, B, Hq, Hkv, L, d, W, S,
                           F(scale), None)
    assert bwd(d=96) == swa.SWA_ERR_UNSUPPORTED
    assert bwd(Hq=3) == swa.SWA_ERR_INVALID_ARG
    assert bwd(W=0) == swa.SWA_ERR_INVALID_ARG
    assert bwd(L=0) == swa.SWA_OK
    assert bwd() == swa.SWA_ERR_INVALID_ARG                       # null tensors
