"""fp64 CPU oracle for sink-aware sliding-window attention.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline and reference legs may import this package.  The CUDA
library never calls it, imports nothing from it and shares no code with it.

The arithmetic lives in ``swa_oracle.c`` (plain C, double precision, OpenMP
over query rows); this module only marshals numpy arrays through ctypes and
holds the plain model of the ring-buffer KV cache (slot bookkeeping, no
arithmetic on values), the Hadamard output projection and the rotary position
encoding, both in numpy float64.

Parity pins: every function here is checked by the ``-m "not gpu"`` tests
against closed forms, a library causal-attention routine, brute-force masks
built from the set definition, and hand-derived golden values.
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "swa_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None
_lib_path = _LIB

_dp = ctypes.POINTER(ctypes.c_double)
_i64p = ctypes.POINTER(ctypes.c_int64)


def build(force: bool = False) -> str:
    """Compile swa_oracle.c into liboracle.so (gcc, -O2, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def use_library(path: str) -> None:
    """Point the wrappers at another build of swa_oracle.c (the tests use this to
    show that a deliberately broken copy fails the pins)."""
    global _lib, _lib_path
    with _lock:
        _lib, _lib_path = None, path


def _load():
    global _lib
    with _lock:
        if _lib is None:
            if _lib_path == _LIB:
                build()
            lib = ctypes.CDLL(_lib_path)
            lib.oracle_swa_rows.argtypes = [_dp, _i64p, ctypes.c_int64, _dp, _dp, ctypes.c_int64,
                                            ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int64,
                                            ctypes.c_int64, ctypes.c_double, _dp, _dp, ctypes.c_int]
            lib.oracle_swa_weights.argtypes = [_dp, ctypes.c_int64, _dp, ctypes.c_int64, ctypes.c_int,
                                               ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int64,
                                               ctypes.c_int64, ctypes.c_double, _dp]
            lib.oracle_swa_fwd.argtypes = [_dp, _dp, _dp, _dp, _dp, ctypes.c_int, ctypes.c_int,
                                           ctypes.c_int, ctypes.c_int64, ctypes.c_int, ctypes.c_int64,
                                           ctypes.c_int64, ctypes.c_double, ctypes.c_int]
            lib.oracle_swa_fwd_varlen.argtypes = [_dp, _dp, _dp, _dp, _dp, _i64p, ctypes.c_int,
                                                  ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                                  ctypes.c_int64, ctypes.c_int64, ctypes.c_double,
                                                  ctypes.c_int]
            lib.oracle_visible_count.argtypes = [ctypes.c_int64, ctypes.c_int64, ctypes.c_int64]
            lib.oracle_visible_count.restype = ctypes.c_int64
            lib.oracle_num_threads.argtypes = [ctypes.c_int]
            for f in (lib.oracle_swa_rows, lib.oracle_swa_weights, lib.oracle_swa_fwd,
                      lib.oracle_swa_fwd_varlen, lib.oracle_num_threads):
                f.restype = ctypes.c_int
            _lib = lib
    return _lib


def _f64(x) -> np.ndarray:
    """Exact float64 copy of a numpy array or a (CPU or CUDA) torch tensor."""
    if hasattr(x, "detach"):
        x = x.detach().to("cpu")
        import torch
        x = x.to(torch.float64).numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _p(a: np.ndarray):
    return a.ctypes.data_as(_dp)


def num_threads(n: int = 0) -> int:
    """Threads the oracle's OpenMP loops use (n > 0 sets it)."""
    return _load().oracle_num_threads(int(n))


def visible_count(t: int, window: int, n_sink: int) -> int:
    return int(_load().oracle_visible_count(int(t), int(window), int(n_sink)))


def swa_rows(q_rows, t_rows, k, v, window: int, n_sink: int, scale: float, threads: int = 0):
    """Selected rows of one sequence.

    q_rows [n, Hq, d]; t_rows [n] positions; k, v [L, Hkv, d].
    Returns out [n, Hq, d] and lse [n, Hq] (float64).
    """
    q = _f64(q_rows)
    k = _f64(k)
    v = _f64(v)
    t = np.ascontiguousarray(np.asarray(t_rows, dtype=np.int64))
    n, Hq, d = q.shape
    L, Hkv, _ = k.shape
    out = np.zeros((n, Hq, d))
    lse = np.zeros((n, Hq))
    rc = _load().oracle_swa_rows(_p(q), t.ctypes.data_as(_i64p), n, _p(k), _p(v), L, Hq, Hkv, d,
                                 int(window), int(n_sink), float(scale), _p(out), _p(lse),
                                 int(threads))
    if rc != 0:
        raise ValueError("oracle_swa_rows rejected its arguments")
    return out, lse


def swa_weights(q_row, t: int, k, h: int, window: int, n_sink: int, scale: float):
    """Attention weights over keys 0..L-1 of query head h at row t; q_row [Hq, d], k [L, Hkv, d]."""
    q = _f64(q_row)
    k = _f64(k)
    Hq, d = q.shape
    L, Hkv, _ = k.shape
    w = np.zeros(L)
    rc = _load().oracle_swa_weights(_p(q), int(t), _p(k), L, Hq, Hkv, d, int(h), int(window),
                                    int(n_sink), float(scale), _p(w))
    if rc != 0:
        raise ValueError("oracle_swa_weights rejected its arguments")
    return w


def swa_fwd(q, k, v, window: int, n_sink: int, scale: float, threads: int = 0):
    """q [B, L, Hq, d], k/v [B, L, Hkv, d] -> out [B, L, Hq, d], lse [B, Hq, L] (float64)."""
    q = _f64(q)
    k = _f64(k)
    v = _f64(v)
    B, L, Hq, d = q.shape
    Hkv = k.shape[2]
    out = np.zeros_like(q)
    lse = np.zeros((B, Hq, L))
    rc = _load().oracle_swa_fwd(_p(q), _p(k), _p(v), _p(out), _p(lse), B, Hq, Hkv, L, d,
                                int(window), int(n_sink), float(scale), int(threads))
    if rc != 0:
        raise ValueError("oracle_swa_fwd rejected its arguments")
    return out, lse


def swa_fwd_varlen(q, k, v, cu_seqlens, window: int, n_sink: int, scale: float, threads: int = 0):
    """Packed q [T, Hq, d], k/v [T, Hkv, d], cu_seqlens [n+1] -> out [T, Hq, d], lse [Hq, T]."""
    q = _f64(q)
    k = _f64(k)
    v = _f64(v)
    cu = np.ascontiguousarray(np.asarray(cu_seqlens, dtype=np.int64))
    T, Hq, d = q.shape
    Hkv = k.shape[1]
    out = np.zeros_like(q)
    lse = np.zeros((Hq, T))
    rc = _load().oracle_swa_fwd_varlen(_p(q), _p(k), _p(v), _p(out), _p(lse),
                                       cu.ctypes.data_as(_i64p), len(cu) - 1, Hq, Hkv, d,
                                       int(window), int(n_sink), float(scale), int(threads))
    if rc != 0:
        raise ValueError("oracle_swa_fwd_varlen rejected its arguments")
    return out, lse


def swa_decode(q, k_hist, v_hist, pos, window: int, n_sink: int, scale: float, threads: int = 0):
    """Decode by definition: row t = pos[b] of sequence b, whose keys/values at
    positions 0..pos[b] are k_hist[b, :pos[b]+1] (k_hist/v_hist [B, P, Hkv, d]).

    q [B, Hq, d] -> out [B, Hq, d], lse [B, Hq].
    """
    q = _f64(q)
    B, Hq, d = q.shape
    out = np.zeros((B, Hq, d))
    lse = np.zeros((B, Hq))
    for b in range(B):
        p = int(pos[b])
        o, l_ = swa_rows(q[b:b + 1], [p], k_hist[b, :p + 1], v_hist[b, :p + 1], window, n_sink,
                         scale, threads)
        out[b], lse[b] = o[0], l_[0]
    return out, lse


# ---------------------------------------------------------------------------
# Ring-buffer KV cache model (slot bookkeeping only).
#
# "Sliding-window beats linear attention", section 1: sliding-window attention
# keeps a fixed-size memory at inference, and the first tokens (sinks) must
# stay.  Reading used throughout: position p lives in ring slot p mod w; the
# positions p < n_sink are also kept in pinned sink slot p and are never
# evicted.  Writing position p overwrites (evicts) position p - w.
# ---------------------------------------------------------------------------

def ring_fill(k, v, window: int, n_sink: int):
    """Cache contents after positions 0..P-1 of k/v [B, P, Hkv, d] were written.

    Returns kcache, vcache [B, Hkv, window, d] and sink_k, sink_v [B, Hkv, n_sink, d]
    (numpy, same dtype as the input; untouched slots are zero).
    """
    k = np.asarray(k)
    v = np.asarray(v)
    B, P, Hkv, d = k.shape
    kc = np.zeros((B, Hkv, window, d), dtype=k.dtype)
    vc = np.zeros_like(kc)
    sk = np.zeros((B, Hkv, n_sink, d), dtype=k.dtype)
    sv = np.zeros_like(sk)
    for p in range(P):
        ring_append(kc, vc, sk, sv, k[:, p], v[:, p], np.full(B, p), window, n_sink)
    return kc, vc, sk, sv


def ring_append(kc, vc, sk, sv, k_new, v_new, pos, window: int, n_sink: int) -> None:
    """In place: write position pos[b] (k_new/v_new [B, Hkv, d]) into the cache arrays."""
    for b in range(len(pos)):
        p = int(pos[b])
        kc[b, :, p % window] = k_new[b]
        vc[b, :, p % window] = v_new[b]
        if p < n_sink:
            sk[b, :, p] = k_new[b]
            sv[b, :, p] = v_new[b]


# ---------------------------------------------------------------------------
# Hadamard output projection ("Rethinking Attention Output Projection:
# Structured Hadamard Transforms for Efficient Transformers", section 2,
# Methodology): MHA_Had(X) = alpha * (Y H) + beta, with H the fixed Walsh-
# Hadamard matrix, which preserves the l2 norm (so it is orthonormal).
# Reading: H is the Sylvester-ordered matrix of size n = Hq * d (a power of two),
# H[i, j] = (-1)^popcount(i & j) / sqrt(n); Y is one token's attention output
# with the heads concatenated (head-major, h * d + c).
# ---------------------------------------------------------------------------

def hadamard_matrix(n: int) -> np.ndarray:
    """Sylvester Walsh-Hadamard matrix of size n, normalised to be orthonormal."""
    if n < 1 or n & (n - 1):
        raise ValueError("n must be a power of two")
    i = np.arange(n, dtype=np.int64)
    bits = np.bitwise_and(i[:, None], i[None, :])
    pop = np.zeros_like(bits)
    while bits.any():
        pop += bits & 1
        bits >>= 1
    return np.where(pop % 2 == 0, 1.0, -1.0) / np.sqrt(n)


def hadamard_proj(y, alpha, beta) -> np.ndarray:
    """alpha * (y @ H) + beta for rows y [N, n] (any float input), in float64."""
    y = _f64(y)
    n = y.shape[-1]
    H = hadamard_matrix(n)
    return _f64(alpha) * (y.reshape(-1, n) @ H).reshape(y.shape) + _f64(beta)


# ---------------------------------------------------------------------------
# Rotary position encoding on the sliding-window branch ("Simple linear
# attention language models balance the recall-throughput tradeoff", proposed
# method: the window attention uses rotary position encoding, the linear branch
# none).  The page gives no formula; reading used: the RoFormer rotation with
# the rotate-half pairing.  For i < d/2 the pair (x[i], x[i + d/2]) of a vector
# at absolute position p turns by the angle p * theta_i, theta_i =
# base^(-2i/d):
#     x'[i]       = x[i] cos(p theta_i) - x[i + d/2] sin(p theta_i)
#     x'[i + d/2] = x[i] sin(p theta_i) + x[i + d/2] cos(p theta_i)
# Positions are absolute token positions (a cached key keeps the rotation of
# its own position; nothing is re-indexed inside the window).
# ---------------------------------------------------------------------------

def rope_angles(positions, d: int, base: float) -> np.ndarray:
    """Angles p * base^(-2i/d), shape [len(positions), d/2], float64."""
    if d < 2 or d % 2:
        raise ValueError("d must be even")
    p = np.asarray(positions, dtype=np.float64).reshape(-1)
    theta = np.power(float(base), -2.0 * np.arange(d // 2, dtype=np.float64) / d)
    return p[:, None] * theta[None, :]


def rope(x, positions, base: float = 10000.0) -> np.ndarray:
    """Rotate x [N, ..., d] (any float input) at positions [N]; float64 result."""
    x = _f64(x)
    d = x.shape[-1]
    ang = rope_angles(positions, d, base)                     # [N, d/2]
    if ang.shape[0] != x.shape[0]:
        raise ValueError("one position per leading index")
    shape = (x.shape[0],) + (1,) * (x.ndim - 2) + (d // 2,)
    c, s = np.cos(ang).reshape(shape), np.sin(ang).reshape(shape)
    lo, hi = x[..., : d // 2], x[..., d // 2:]
    return np.concatenate([lo * c - hi * s, lo * s + hi * c], axis=-1)


# ---------------------------------------------------------------------------
# Backward pass of sink-aware sliding-window attention: gradients of the loss
# with respect to q, k and v given dO = dL/dout, for the visible set of
# "Sliding-window beats linear attention" (sections 1 and 3).  Written out from
# the definition P = softmax over the visible keys, out = P V:
#     dV = P^T dO,  dP = dO V^T,  dS = P * (dP - rowsum(P * dP)),
#     dQ = scale * dS K,  dK = scale * dS^T Q,
# the gradients of a KV head summed over the query heads that read it.
# Dense per (sequence, head) in float64; sizes up to a few thousand rows.
# ---------------------------------------------------------------------------

def visible_mask(L: int, window: int, n_sink: int) -> np.ndarray:
    """Boolean [L, L]: row t sees key j iff j <= t and (j >= t - window + 1 or j < n_sink)."""
    t = np.arange(L)[:, None]
    j = np.arange(L)[None, :]
    return (j <= t) & ((j >= t - window + 1) | (j < n_sink))


def swa_bwd(q, k, v, dout, window: int, n_sink: int, scale: float):
    """q, dout [B, L, Hq, d]; k, v [B, L, Hkv, d] -> dq, dk, dv (float64, same shapes)."""
    q, k, v, do = _f64(q), _f64(k), _f64(v), _f64(dout)
    B, L, Hq, d = q.shape
    Hkv = k.shape[2]
    G = Hq // Hkv
    M = visible_mask(L, window, n_sink)
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    for b in range(B):
        for h in range(Hq):
            kh = h // G
            s = scale * (q[b, :, h] @ k[b, :, kh].T)
            s = np.where(M, s, -np.inf)
            p = np.exp(s - s.max(axis=1, keepdims=True))
            p /= p.sum(axis=1, keepdims=True)
            dp = do[b, :, h] @ v[b, :, kh].T
            ds = p * (dp - (p * dp).sum(axis=1, keepdims=True))
            dq[b, :, h] = scale * (ds @ k[b, :, kh])
            dk[b, :, kh] += scale * (ds.T @ q[b, :, h])
            dv[b, :, kh] += p.T @ do[b, :, h]
    return dq, dk, dv


# ---------------------------------------------------------------------------
# The linear-attention branch of the Based hybrid ("Simple linear attention
# language models balance the recall-throughput tradeoff", proposed method: a
# linear attention whose feature dimension sets the recurrent state size, with no
# position encoding, next to the sliding window).  The sink page defines linear
# attention as a kernel approximation of softmax attention; neither page gives
# the feature map.  Reading used: the second-order Taylor approximation of exp,
#     kappa(q, k) = 1 + x + x^2 / 2,  x = scale * q.k   (> 0 for every x),
# with causal normalisation
#     out_t = sum_{s<=t} kappa(q_t, k_s) v_s / sum_{s<=t} kappa(q_t, k_s).
# Its explicit features, phi(u) = [1, sqrt(scale) u, scale (u outer u) / sqrt(2)]
# (F = 1 + d + d^2 entries, the outer product row-major), give kappa(q, k) =
# phi(q).phi(k), the recurrent state S_t = sum_{s<=t} phi(k_s) v_s^T [F, dv] and
# z_t = sum_{s<=t} phi(k_s) [F], and out_t = phi(q_t) S_t / phi(q_t).z_t.
# ---------------------------------------------------------------------------

def taylor_kernel(q, k, scale: float) -> np.ndarray:
    """kappa(q_i, k_j) = 1 + x + x^2/2 with x = scale q_i.k_j, for q [n, d], k [m, d]."""
    x = scale * (_f64(q) @ _f64(k).T)
    return 1.0 + x + 0.5 * x * x


def taylor_features(u, scale: float) -> np.ndarray:
    """phi(u) for rows u [..., d]: [1, sqrt(scale) u, scale vec(u u^T) / sqrt(2)], float64."""
    u = _f64(u)
    d = u.shape[-1]
    outer = (u[..., :, None] * u[..., None, :]).reshape(u.shape[:-1] + (d * d,))
    one = np.ones(u.shape[:-1] + (1,))
    return np.concatenate([one, math.sqrt(scale) * u, scale * outer / math.sqrt(2.0)], axis=-1)


def based_linear_fwd(q, k, v, scale: float) -> np.ndarray:
    """Causal Taylor linear attention: q, k [B, L, H, d], v [B, L, H, dv] -> out [B, L, H, dv]."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, L, H, _ = q.shape
    out = np.zeros(v.shape[:3] + (v.shape[3],))
    causal = np.tril(np.ones((L, L), dtype=bool))
    for b in range(B):
        for h in range(H):
            a = np.where(causal, taylor_kernel(q[b, :, h], k[b, :, h], scale), 0.0)
            out[b, :, h] = (a @ v[b, :, h]) / a.sum(axis=1, keepdims=True)
    return out


def based_linear_state(k, v, scale: float):
    """State after positions 0..L-1: S [B, H, F, dv] and z [B, H, F] (float64)."""
    fk = taylor_features(k, scale)                                  # [B, L, H, F]
    S = np.einsum("blhf,blhc->bhfc", fk, _f64(v))
    z = fk.sum(axis=1)
    return S, z


def based_linear_decode(q, k, v, S, z, scale: float):
    """One recurrent step for q, k [B, H, d], v [B, H, dv] and the state before it:
    returns out [B, H, dv] and the new state (the token attends to itself)."""
    fk, fq = taylor_features(k, scale), taylor_features(q, scale)   # [B, H, F]
    S = _f64(S) + fk[..., :, None] * _f64(v)[..., None, :]
    z = _f64(z) + fk
    out = np.einsum("bhf,bhfc->bhc", fq, S) / np.einsum("bhf,bhf->bh", fq, z)[..., None]
    return out, S, z
