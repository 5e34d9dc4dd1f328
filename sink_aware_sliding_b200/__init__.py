"""Python binding of libswa (causal sliding-window attention with attention sinks, B200).

Argument marshalling only: every function passes raw device pointers, sizes
and the current CUDA stream to the C ABI declared in ``include/swa.h``; all of
the work runs in the library's sm_100a kernels.  There is no fallback: if
``libswa.so`` is missing or cannot be loaded, every call raises.

Tensors are PyTorch tensors on a CUDA device (PyTorch only supplies memory and
streams).  Layouts follow ``swa.h``:
    prefill      q [B, L, Hq, d], k/v [B, L, Hkv, d], out like q, lse [B, Hq, L]
    varlen       q [T, Hq, d], k/v [T, Hkv, d], cu_seqlens int32 [n+1], lse [Hq, T]
    ring cache   kcache/vcache [B, Hkv, window, d], sink_k/sink_v [B, Hkv, n_sink, d]
    decode       q [B, Hq, d], pos int32 [B], out [B, Hq, d], lse [B, Hq]
"""
from __future__ import annotations

import ctypes
import math
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libswa.so")

SWA_OK = 0
SWA_ERR_INVALID_ARG = 1
SWA_ERR_UNSUPPORTED = 2
SWA_ERR_CUDA = 3
SWA_ERR_DEVICE_TIMEOUT = 4
SWA_ERR_WORKSPACE = 5
SWA_DTYPE_BF16 = 0
SWA_DTYPE_F32 = 1
SWA_DTYPE_BF16_F32OUT = 2

# Every entry point of include/swa.h.
EXPORTS = (
    "swa_fwd", "swa_fwd_varlen", "swa_cache_fill", "swa_cache_append",
    "swa_decode_workspace_bytes", "swa_decode", "swa_status_string", "swa_device_error",
    "swa_set_wait_timeout_ns", "swa_set_debug_flags", "swa_version", "swa_decode_noalloc",
    "swa_hadamard_proj", "swa_rope_qk", "swa_rope_cache_append", "swa_decode_rope", "swa_bwd",
    "swa_based_linear_state_features", "swa_based_linear_fwd", "swa_based_linear_decode",
    "swa_decode_ex", "swa_debug_error_word", "swa_hybrid_decode",
)

_lib = None


class SwaError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {swa_status_string(status)} (status {status})")


def _load():
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing; build it with `python -m sink_aware_sliding_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    P, I, F, LL, SZ = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_longlong, ctypes.c_size_t
    lib.swa_fwd.argtypes = [P, P, P, P, P, I, I, I, I, I, I, I, F, I, P]
    lib.swa_fwd_varlen.argtypes = [P, P, P, P, P, P, I, LL, I, I, I, I, I, F, I, P]
    lib.swa_cache_fill.argtypes = [P, P, I, P, P, P, P, I, I, I, I, I, P]
    lib.swa_cache_append.argtypes = [P, P, P, P, P, P, P, I, I, I, I, I, P]
    lib.swa_decode_workspace_bytes.argtypes = [I, I, I, I, I, I]
    lib.swa_decode_workspace_bytes.restype = SZ
    lib.swa_decode.argtypes = [P, P, P, P, P, P, P, P, I, I, I, I, I, I, F, P, SZ, P]
    lib.swa_decode_ex.argtypes = [P, P, P, P, P, P, P, P, I, I, I, I, I, I, F, I, P, SZ, P]
    lib.swa_decode_noalloc.argtypes = [P, P, P, P, P, P, P, P, I, I, I, I, I, I, F, P]
    lib.swa_hadamard_proj.argtypes = [P, P, P, P, LL, I, I, P]
    lib.swa_hybrid_decode.argtypes = [P, P, P, P, P, P, P, P, P, P, I, I, I, I, I, I, F,
                                      P, P, P, P, P, P, I, I, I, F, P]
    D = ctypes.c_double
    lib.swa_rope_qk.argtypes = [P, P, P, LL, I, I, I, D, P]
    lib.swa_rope_cache_append.argtypes = [P, P, P, P, P, P, P, I, I, I, I, I, D, P]
    lib.swa_decode_rope.argtypes = [P, P, P, P, P, P, P, P, I, I, I, I, I, I, F, D, P, SZ, P]
    lib.swa_bwd.argtypes = [P, P, P, P, P, P, P, P, P, I, I, I, I, I, I, I, F, P]
    lib.swa_based_linear_state_features.argtypes = [I]
    lib.swa_based_linear_fwd.argtypes = [P, P, P, P, P, P, I, I, I, I, I, F, I, P]
    lib.swa_based_linear_decode.argtypes = [P, P, P, P, P, P, I, I, I, I, F, I, P]
    lib.swa_status_string.argtypes = [I]
    lib.swa_status_string.restype = ctypes.c_char_p
    lib.swa_device_error.argtypes = [P]
    lib.swa_debug_error_word.argtypes = [P]
    lib.swa_set_wait_timeout_ns.argtypes = [ctypes.c_ulonglong]
    lib.swa_set_wait_timeout_ns.restype = ctypes.c_ulonglong
    lib.swa_set_debug_flags.argtypes = [I]
    for name in ("swa_fwd", "swa_fwd_varlen", "swa_cache_fill", "swa_cache_append", "swa_decode",
                 "swa_decode_ex", "swa_debug_error_word", "swa_decode_noalloc", "swa_hybrid_decode", "swa_hadamard_proj", "swa_rope_qk", "swa_rope_cache_append",
                 "swa_decode_rope", "swa_bwd", "swa_based_linear_state_features", "swa_based_linear_fwd",
                 "swa_based_linear_decode",
                 "swa_device_error", "swa_set_debug_flags", "swa_version"):
        getattr(lib, name).restype = I
    _lib = lib
    return lib


def library():
    """The loaded ctypes library (raises if libswa.so is missing)."""
    return _load()


def _check(st: int, where: str) -> None:
    if st != SWA_OK:
        raise SwaError(st, where)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        import torch
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _dtype_code(t, out) -> int:
    import torch
    if t.dtype == torch.bfloat16 and out.dtype == torch.bfloat16:
        return SWA_DTYPE_BF16
    if t.dtype == torch.bfloat16 and out.dtype == torch.float32:
        return SWA_DTYPE_BF16_F32OUT
    if t.dtype == torch.float32 and out.dtype == torch.float32:
        return SWA_DTYPE_F32
    raise TypeError(f"unsupported dtypes {t.dtype} -> {out.dtype}")


def _scale(scale, d):
    return 1.0 / math.sqrt(d) if scale is None else float(scale)


def _need(cond: bool, msg: str):
    if not cond:
        raise ValueError(msg)


def swa_status_string(status: int) -> str:
    return _load().swa_status_string(int(status)).decode()


def swa_version() -> int:
    return _load().swa_version()


def swa_fwd(q, k, v, out, lse, window: int, n_sink: int, scale=None, stream=None) -> None:
    """Prefill; q [B, L, Hq, d], k/v [B, L, Hkv, d]; writes out (like q) and lse [B, Hq, L] (or None)."""
    _need(q.dim() == 4 and k.dim() == 4 and v.shape == k.shape and out.shape == q.shape, "shapes")
    _need(all(t.is_contiguous() for t in (q, k, v, out)), "tensors must be contiguous")
    _need(q.dtype == k.dtype == v.dtype, "q, k, v must share a dtype")
    B, L, Hq, d = q.shape
    _need(k.shape[0] == B and k.shape[1] == L and k.shape[3] == d, "k/v shape")
    if lse is not None:
        _need(lse.shape == (B, Hq, L) and lse.is_contiguous(), "lse shape")
    st = _load().swa_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, Hq, k.shape[2], L, d,
                         int(window), int(n_sink), _scale(scale, d), _dtype_code(q, out), _stream(stream))
    _check(st, "swa_fwd")


def swa_fwd_varlen(q, k, v, out, lse, cu_seqlens, window: int, n_sink: int, scale=None,
                   stream=None) -> None:
    """Packed prefill; q [T, Hq, d], k/v [T, Hkv, d], cu_seqlens int32 [n+1] on the device."""
    _need(q.dim() == 3 and k.dim() == 3 and v.shape == k.shape and out.shape == q.shape, "shapes")
    _need(all(t.is_contiguous() for t in (q, k, v, out, cu_seqlens)), "tensors must be contiguous")
    import torch
    _need(cu_seqlens.dtype == torch.int32 and cu_seqlens.dim() == 1, "cu_seqlens must be int32 [n+1]")
    T, Hq, d = q.shape
    if lse is not None:
        _need(lse.shape == (Hq, T) and lse.is_contiguous(), "lse shape")
    st = _load().swa_fwd_varlen(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), _ptr(cu_seqlens),
                                cu_seqlens.numel() - 1, T, Hq, k.shape[1], d, int(window),
                                int(n_sink), _scale(scale, d), _dtype_code(q, out), _stream(stream))
    _check(st, "swa_fwd_varlen")


def swa_cache_fill(k, v, kcache, vcache, sink_k, sink_v, window: int, n_sink: int,
                   stream=None) -> None:
    """Write prefix positions 0..P-1 of k/v [B, P, Hkv, d] into an empty ring cache."""
    B, P, Hkv, d = k.shape
    st = _load().swa_cache_fill(_ptr(k), _ptr(v), P, _ptr(kcache), _ptr(vcache), _ptr(sink_k),
                                _ptr(sink_v), B, Hkv, d, int(window), int(n_sink), _stream(stream))
    _check(st, "swa_cache_fill")


def swa_cache_append(k_new, v_new, pos, kcache, vcache, sink_k, sink_v, window: int, n_sink: int,
                     stream=None) -> None:
    """Write k_new/v_new [B, Hkv, d] at positions pos (int32 [B], device) into the ring cache."""
    B, Hkv, d = k_new.shape
    st = _load().swa_cache_append(_ptr(k_new), _ptr(v_new), _ptr(pos), _ptr(kcache), _ptr(vcache),
                                  _ptr(sink_k), _ptr(sink_v), B, Hkv, d, int(window), int(n_sink),
                                  _stream(stream))
    _check(st, "swa_cache_append")


def swa_rope_cache_append(k_new, v_new, pos, kcache, vcache, sink_k, sink_v, window: int, n_sink: int,
                          rope_base: float = 10000.0, stream=None) -> None:
    """swa_cache_append with k_new rotated at pos[b] (rotary encoding) before it is stored."""
    B, Hkv, d = k_new.shape
    st = _load().swa_rope_cache_append(_ptr(k_new), _ptr(v_new), _ptr(pos), _ptr(kcache), _ptr(vcache),
                                       _ptr(sink_k), _ptr(sink_v), B, Hkv, d, int(window), int(n_sink),
                                       float(rope_base), _stream(stream))
    _check(st, "swa_rope_cache_append")


def swa_rope_qk(q, k, positions, rope_base: float = 10000.0, stream=None) -> None:
    """Rotate q [..., Hq, d] and k [..., Hkv, d] (bf16, contiguous; k may be None) in place;
    the leading dimensions flatten to tokens, token t at positions[t] (int32, device)."""
    import torch
    _need(q.dtype == torch.bfloat16 and q.is_contiguous(), "q bf16 contiguous")
    Hq, d = q.shape[-2], q.shape[-1]
    T = q.numel() // (Hq * d)
    Hkv = 0
    if k is not None:
        _need(k.dtype == torch.bfloat16 and k.is_contiguous() and k.shape[-1] == d, "k bf16 contiguous")
        Hkv = k.shape[-2]
        _need(k.numel() == T * Hkv * d, "k tokens")
    _need(positions.dtype == torch.int32 and positions.numel() == T, "positions int32 [T]")
    st = _load().swa_rope_qk(_ptr(q), _ptr(k) if k is not None else None, _ptr(positions), T, Hq, Hkv, d,
                             float(rope_base), _stream(stream))
    _check(st, "swa_rope_qk")


def swa_decode_workspace_bytes(B: int, Hq: int, Hkv: int, d: int, window: int, n_sink: int) -> int:
    return int(_load().swa_decode_workspace_bytes(B, Hq, Hkv, d, window, n_sink))


def swa_decode(q, kcache, vcache, sink_k, sink_v, pos, out, lse, window: int, n_sink: int,
               workspace, scale=None, stream=None) -> None:
    """One decode step; q [B, Hq, d] bf16 at positions pos; writes out [B, Hq, d] and lse [B, Hq].
    out is bf16 (swa_decode) or float32 (swa_decode_ex with a float32 output)."""
    import torch
    B, Hq, d = q.shape
    Hkv = kcache.shape[1]
    _need(out.dtype in (torch.bfloat16, torch.float32), "out bf16 or float32")
    args = (_ptr(q), _ptr(kcache), _ptr(vcache), _ptr(sink_k), _ptr(sink_v), _ptr(pos), _ptr(out), _ptr(lse),
            B, Hq, Hkv, d, int(window), int(n_sink), _scale(scale, d))
    ws = (_ptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream))
    if out.dtype == torch.float32:
        _check(_load().swa_decode_ex(*args, SWA_DTYPE_BF16_F32OUT, *ws), "swa_decode_ex")
    else:
        _check(_load().swa_decode(*args, *ws), "swa_decode")


def swa_decode_rope(q, kcache, vcache, sink_k, sink_v, pos, out, lse, window: int, n_sink: int,
                    workspace, rope_base: float = 10000.0, scale=None, stream=None) -> None:
    """swa_decode with q rotated at pos[b] inside the kernel (the cache holds rotated keys)."""
    B, Hq, d = q.shape
    Hkv = kcache.shape[1]
    st = _load().swa_decode_rope(_ptr(q), _ptr(kcache), _ptr(vcache), _ptr(sink_k), _ptr(sink_v),
                                 _ptr(pos), _ptr(out), _ptr(lse), B, Hq, Hkv, d, int(window), int(n_sink),
                                 _scale(scale, d), float(rope_base), _ptr(workspace),
                                 workspace.numel() * workspace.element_size(), _stream(stream))
    _check(st, "swa_decode_rope")


def swa_decode_noalloc(q, kcache, vcache, sink_k, sink_v, pos, out, lse, window: int, n_sink: int,
                       scale=None, stream=None) -> None:
    """swa_decode for callers that cannot allocate device memory: the split-K
    scratch lives in a fixed 8 MiB array inside the library instead of a
    caller-provided workspace.  Calls that overlap on the GPU share that array
    and must not run concurrently; sizes needing more than 8 MiB raise."""
    B, Hq, d = q.shape
    Hkv = kcache.shape[1]
    st = _load().swa_decode_noalloc(_ptr(q), _ptr(kcache), _ptr(vcache), _ptr(sink_k), _ptr(sink_v),
                                    _ptr(pos), _ptr(out), _ptr(lse), B, Hq, Hkv, d, int(window),
                                    int(n_sink), _scale(scale, d), _stream(stream))
    _check(st, "swa_decode_noalloc")


def swa_bwd(q, k, v, out, dout, lse, dq, dk, dv, window: int, n_sink: int, scale=None, stream=None) -> None:
    """Gradients dq [B, L, Hq, d], dk, dv [B, L, Hkv, d] (float32) of the forward
    out = swa_fwd(q, k, v), given dout (bf16) and the forward's out (bf16) and lse."""
    import torch
    B, L, Hq, d = q.shape
    Hkv = k.shape[2]
    for t, name in ((q, "q"), (k, "k"), (v, "v"), (out, "out"), (dout, "dout")):
        _need(t.dtype == torch.bfloat16 and t.is_contiguous(), f"{name} bf16 contiguous")
    for t, name in ((dq, "dq"), (dk, "dk"), (dv, "dv"), (lse, "lse")):
        _need(t.dtype == torch.float32 and t.is_contiguous(), f"{name} float32 contiguous")
    st = _load().swa_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(dout), _ptr(lse), _ptr(dq), _ptr(dk),
                         _ptr(dv), B, Hq, Hkv, L, d, int(window), int(n_sink), _scale(scale, d), _stream(stream))
    _check(st, "swa_bwd")


def swa_based_linear_state_features(dk: int) -> int:
    return int(_load().swa_based_linear_state_features(int(dk)))


def swa_based_linear_fwd(q, k, v, out, state=None, zsum=None, scale=None, stream=None) -> None:
    """Causal Taylor linear attention: q, k [B, L, H, dk], v [B, L, H, dv] bf16 -> out (bf16 or
    float32); state [B, H, F, dv] / zsum [B, H, F] float32, if given, receive the final state."""
    import torch
    _need(q.dim() == 4, "q [B, L, H, dk]")
    B, L, H, dk = q.shape
    dv = v.shape[-1]
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _need(t.dtype == torch.bfloat16 and t.is_contiguous(), f"{n} bf16 contiguous")
    _need(k.shape == q.shape, "k shape == q shape")
    _need(v.dim() == 4 and v.shape[:3] == q.shape[:3], "v [B, L, H, dv]")
    _need(out.shape == v.shape and out.is_contiguous() and out.dtype in (torch.bfloat16, torch.float32),
          "out [B, L, H, dv] bf16 or float32, contiguous")
    _need((state is None) == (zsum is None), "state and zsum together")
    if state is not None:
        F = 1 + dk + dk * dk
        _need(state.shape == (B, H, F, dv) and state.dtype == torch.float32 and state.is_contiguous(),
              "state [B, H, F, dv] float32 contiguous")
        _need(zsum.shape == (B, H, F) and zsum.dtype == torch.float32 and zsum.is_contiguous(),
              "zsum [B, H, F] float32 contiguous")
    code = SWA_DTYPE_F32 if out.dtype == torch.float32 else SWA_DTYPE_BF16
    st = _load().swa_based_linear_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(state), _ptr(zsum), B, L, H, dk, dv,
                                      ctypes.c_float(scale if scale is not None else 1.0 / math.sqrt(dk)), code,
                                      _stream(stream))
    _check(st, "swa_based_linear_fwd")


def swa_based_linear_decode(q, k, v, state, zsum, out, scale=None, stream=None) -> None:
    """One token per sequence: q, k [B, H, dk], v [B, H, dv] bf16; state/zsum float32 updated
    in place; out [B, H, dv]."""
    import torch
    _need(q.dim() == 3, "q [B, H, dk]")
    B, H, dk = q.shape
    dv = v.shape[-1]
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _need(t.dtype == torch.bfloat16 and t.is_contiguous(), f"{n} bf16 contiguous")
    _need(k.shape == q.shape and v.dim() == 3 and v.shape[:2] == q.shape[:2], "k [B, H, dk], v [B, H, dv]")
    F = 1 + dk + dk * dk
    _need(state.shape == (B, H, F, dv) and state.dtype == torch.float32 and state.is_contiguous(),
          "state [B, H, F, dv] float32 contiguous")
    _need(zsum.shape == (B, H, F) and zsum.dtype == torch.float32 and zsum.is_contiguous(),
          "zsum [B, H, F] float32 contiguous")
    _need(out.shape == v.shape and out.is_contiguous() and out.dtype in (torch.bfloat16, torch.float32),
          "out [B, H, dv] bf16 or float32, contiguous")
    code = SWA_DTYPE_F32 if out.dtype == torch.float32 else SWA_DTYPE_BF16
    st = _load().swa_based_linear_decode(_ptr(q), _ptr(k), _ptr(v), _ptr(state), _ptr(zsum), _ptr(out), B, H, dk, dv,
                                         ctypes.c_float(scale if scale is not None else 1.0 / math.sqrt(dk)), code,
                                         _stream(stream))
    _check(st, "swa_based_linear_decode")


def swa_hybrid_decode(q, k_new, v_new, pos, kcache, vcache, sink_k, sink_v, out, lse, window: int, n_sink: int,
                      ql, kl, vl, state, zsum, out_l, scale=None, scale_l=None, stream=None) -> None:
    """One hybrid decode step in one launch: the window branch (append k_new/v_new
    [B, Hkv, d] at pos, decode q [B, Hq, d] into out, lse) and the linear branch
    (ql, kl [B, H_l, 16], vl [B, H_l, 64]; state/zsum updated; out_l [B, H_l, 64])."""
    import torch
    B, Hq, d = q.shape
    Hkv = kcache.shape[1]
    H_l, dk = ql.shape[1], ql.shape[2]
    dv = vl.shape[-1]
    for t, n in ((q, "q"), (k_new, "k_new"), (v_new, "v_new"), (out, "out"), (ql, "ql"), (kl, "kl"), (vl, "vl"),
                 (out_l, "out_l")):
        _need(t.dtype == torch.bfloat16 and t.is_contiguous(), f"{n} bf16 contiguous")
    _need(state.dtype == torch.float32 and zsum.dtype == torch.float32, "state, zsum float32")
    _need(pos.dtype == torch.int32 and pos.numel() == B, "pos int32 [B]")
    st = _load().swa_hybrid_decode(_ptr(q), _ptr(k_new), _ptr(v_new), _ptr(pos), _ptr(kcache), _ptr(vcache),
                                   _ptr(sink_k), _ptr(sink_v), _ptr(out), _ptr(lse), B, Hq, Hkv, d, int(window),
                                   int(n_sink), _scale(scale, d), _ptr(ql), _ptr(kl), _ptr(vl), _ptr(state),
                                   _ptr(zsum), _ptr(out_l), H_l, dk, dv,
                                   ctypes.c_float(scale_l if scale_l is not None else 1.0 / math.sqrt(dk)),
                                   _stream(stream))
    _check(st, "swa_hybrid_decode")


def swa_hadamard_proj(y, alpha, beta, z, stream=None) -> None:
    """z = alpha * (y H) + beta per row of n = alpha.numel() elements; y bf16 holding a
    whole number of rows in any contiguous shape (e.g. an attention output [T, Hq, d]
    with n = Hq * d), z of the same shape in bf16 or float32, alpha/beta [n] float32.
    H is the orthonormal Walsh-Hadamard matrix of size n."""
    import torch
    n = alpha.numel()
    _need(y.dtype == torch.bfloat16 and y.is_contiguous() and z.is_contiguous(), "y bf16 contiguous")
    _need(z.shape == y.shape, "z shape")
    _need(alpha.dtype == beta.dtype == torch.float32 and beta.numel() == n, "alpha/beta float32 [n]")
    _need(n > 0 and y.numel() % n == 0, "y holds a whole number of rows of n")
    code = SWA_DTYPE_F32 if z.dtype == torch.float32 else SWA_DTYPE_BF16
    st = _load().swa_hadamard_proj(_ptr(y), _ptr(alpha), _ptr(beta), _ptr(z), y.numel() // n, n, code,
                                   _stream(stream))
    _check(st, "swa_hadamard_proj")


def swa_device_error(stream=None) -> int:
    return _load().swa_device_error(_stream(stream))


def swa_debug_error_word(stream=None) -> int:
    return _load().swa_debug_error_word(_stream(stream))


def swa_set_wait_timeout_ns(ns: int) -> int:
    return int(_load().swa_set_wait_timeout_ns(int(ns)))


def swa_set_debug_flags(flags: int) -> int:
    return _load().swa_set_debug_flags(int(flags))
