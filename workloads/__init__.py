"""Seeded synthetic workloads for sink-aware sliding-window attention.

This module is shared by the tests, the benchmark and the oracle's callers.
It holds shapes and random-number recipes only: none of the attention
arithmetic lives here, so neither the CUDA path nor the oracle can lean on
it for a result.

Input recipe (applies to every workload):
  * fp32 draws from N(0, 1) with a ``torch.Generator`` seeded 0, drawn in the
    order q, k, v (decode: the prefix q, k, v, then per generated step q,
    k_new, v_new);
  * optional sink bias: for each (sequence, KV head) let q_bar be the fp32
    mean of q over all positions of the sequence and the G query heads of
    that KV head, u = q_bar / |q_bar|, and add 2 * sqrt(d) * u to the keys at
    positions 0 .. n_sink-1.  The bias is applied before rounding, so the
    sink keys draw scores with about sqrt(5) times the spread of the others;
  * rounding to bf16 with round-to-nearest-even (``Tensor.to``), except for
    the fp32 tiny case, which stays fp32.

q and k are taken as already position-rotated: the sliding-window branch of
the Based hybrid applies its rotary encoding before attention ("Simple linear
attention language models balance the recall-throughput tradeoff", proposed
method), so the attention kernel itself sees no positions.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional, Sequence

import torch

SEED = 0


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    kind: str                      # "prefill", "varlen" or "decode"
    Hq: int
    Hkv: int
    d: int
    window: int
    n_sink: int
    dtype: str                     # "bf16" or "f32"
    B: int = 1
    L: int = 0                     # prefill sequence length
    seqlens: tuple = ()            # varlen: lengths of the packed sequences
    sink_bias: bool = False
    prefix: int = 0                # decode: tokens already in context
    steps: int = 0                 # decode: generated tokens
    rope_base: float = 0.0         # > 0: rotary encoding applied on the device (decode steps)
    note: str = ""

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    def describe(self) -> dict:
        out = {"workload": self.name, "kind": self.kind, "Hq": self.Hq, "Hkv": self.Hkv,
               "d": self.d, "window": self.window, "n_sink": self.n_sink,
               "dtype": self.dtype, "sink_bias": self.sink_bias}
        if self.kind == "prefill":
            out.update(B=self.B, L=self.L)
        elif self.kind == "varlen":
            out.update(seqlens=list(self.seqlens))
        else:
            out.update(B=self.B, prefix=self.prefix, steps=self.steps)
        if self.rope_base > 0:
            out.update(rope_base=self.rope_base)
        return out


WORKLOADS = {
    "tiny": Workload(
        "tiny", "prefill", Hq=2, Hkv=2, d=64, window=64, n_sink=4, dtype="f32", B=1, L=256,
        note="small fp32 case the oracle finishes in seconds"),
    "based_local": Workload(
        "based_local", "prefill", Hq=16, Hkv=16, d=64, window=128, n_sink=0, dtype="bf16",
        B=8, L=2048, note="sliding-window branch of a Based-style hybrid layer"),
    "gqa8b_prefill": Workload(
        "gqa8b_prefill", "prefill", Hq=32, Hkv=8, d=128, window=4096, n_sink=4, dtype="bf16",
        B=1, L=32768, sink_bias=True, note="8B-shaped GQA prefill with biased sink keys"),
    "decode": Workload(
        "decode", "decode", Hq=32, Hkv=8, d=128, window=4096, n_sink=4, dtype="bf16",
        B=64, prefix=16384, steps=1024, sink_bias=True,
        note="ring-buffer decode after a 16384-token prefix"),
    "decode_rope": Workload(
        "decode_rope", "decode", Hq=32, Hkv=8, d=128, window=4096, n_sink=4, dtype="bf16",
        B=64, prefix=16384, steps=1024, sink_bias=True, rope_base=10000.0,
        note="the decode workload with the rotary encoding fused into append and decode"),
    "decode_b1": Workload(
        "decode_b1", "decode", Hq=32, Hkv=8, d=128, window=4096, n_sink=4, dtype="bf16",
        B=1, prefix=16384, steps=1024, sink_bias=True,
        note="the decode workload for a single sequence (latency-bound serving case)"),
    "packed_long": Workload(
        "packed_long", "varlen", Hq=32, Hkv=8, d=128, window=2048, n_sink=4, dtype="bf16",
        seqlens=(131072, 65536, 16384, 1000), note="four packed sequences"),
}


def _gen(device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(SEED)
    return g


def _normal(g: torch.Generator, shape, device) -> torch.Tensor:
    return torch.randn(tuple(shape), generator=g, device=device, dtype=torch.float32)


def _round(x: torch.Tensor, dtype: str) -> torch.Tensor:
    if dtype == "bf16":
        return x.to(torch.bfloat16)
    if dtype == "f32":
        return x.contiguous()
    raise ValueError(dtype)


def sink_direction(q_sum: torch.Tensor) -> torch.Tensor:
    """Unit vector along a summed query tensor [..., d] (any positive scale of the mean)."""
    n = q_sum.norm(dim=-1, keepdim=True).clamp_min(1e-30)
    return q_sum / n


def _bias_sinks_(k: torch.Tensor, q: torch.Tensor, n_sink: int, G: int) -> None:
    """In place: k [L, Hkv, d] of one sequence, q [L, Hq, d] of the same sequence."""
    L, Hkv, d = k.shape
    s = min(n_sink, L)
    if s == 0:
        return
    qs = q.double().sum(dim=0).view(Hkv, G, d).sum(dim=1)          # [Hkv, d]
    u = sink_direction(qs).float()
    k[:s] += (2.0 * math.sqrt(d)) * u.unsqueeze(0)


def make_prefill(w: Workload, device="cpu", B: Optional[int] = None, L: Optional[int] = None,
                 dtype: Optional[str] = None):
    """q [B, L, Hq, d], k/v [B, L, Hkv, d] as the workload describes.

    B, L and dtype may be overridden to make a smaller case of the same recipe.
    """
    B = w.B if B is None else B
    L = w.L if L is None else L
    dt = w.dtype if dtype is None else dtype
    g = _gen(device)
    q = _normal(g, (B, L, w.Hq, w.d), device)
    k = _normal(g, (B, L, w.Hkv, w.d), device)
    v = _normal(g, (B, L, w.Hkv, w.d), device)
    if w.sink_bias:
        for b in range(B):
            _bias_sinks_(k[b], q[b], w.n_sink, w.G)
    return _round(q, dt), _round(k, dt), _round(v, dt)


def cu_seqlens_of(seqlens: Sequence[int]) -> list:
    cu = [0]
    for n in seqlens:
        cu.append(cu[-1] + int(n))
    return cu


def make_varlen(w: Workload, device="cpu", seqlens: Optional[Sequence[int]] = None,
                dtype: Optional[str] = None):
    """Packed q [T, Hq, d], k/v [T, Hkv, d] and cu_seqlens (python list, length n+1)."""
    seqlens = tuple(w.seqlens if seqlens is None else seqlens)
    dt = w.dtype if dtype is None else dtype
    cu = cu_seqlens_of(seqlens)
    T = cu[-1]
    g = _gen(device)
    q = _normal(g, (T, w.Hq, w.d), device)
    k = _normal(g, (T, w.Hkv, w.d), device)
    v = _normal(g, (T, w.Hkv, w.d), device)
    if w.sink_bias:
        for i in range(len(seqlens)):
            a, b = cu[i], cu[i + 1]
            _bias_sinks_(k[a:b], q[a:b], w.n_sink, w.G)
    return _round(q, dt), _round(k, dt), _round(v, dt), cu


@dataclasses.dataclass
class DecodeInputs:
    prefix_k: torch.Tensor      # [B, P, Hkv, d]
    prefix_v: torch.Tensor      # [B, P, Hkv, d]
    q: torch.Tensor             # [S, B, Hq, d]   query of generated step i (position P + i)
    k_new: torch.Tensor         # [S, B, Hkv, d]
    v_new: torch.Tensor         # [S, B, Hkv, d]


def make_decode(w: Workload, device="cpu", B: Optional[int] = None, prefix: Optional[int] = None,
                steps: Optional[int] = None, dtype: Optional[str] = None,
                chunk: int = 1024) -> DecodeInputs:
    """Decode workload: a prefix (positions 0..P-1) then ``steps`` generated tokens.

    The prefix queries are drawn (in chunks of ``chunk`` positions) only to set
    the sink-bias direction; they are not kept.
    """
    B = w.B if B is None else B
    P = w.prefix if prefix is None else prefix
    S = w.steps if steps is None else steps
    dt = w.dtype if dtype is None else dtype
    g = _gen(device)
    qsum = torch.zeros(B, w.Hkv, w.d, dtype=torch.float64, device=device)
    for p0 in range(0, P, chunk):
        n = min(chunk, P - p0)
        qc = _normal(g, (B, n, w.Hq, w.d), device)
        qsum += qc.double().sum(dim=1).view(B, w.Hkv, w.G, w.d).sum(dim=2)
        del qc
    pk = _normal(g, (B, P, w.Hkv, w.d), device)
    pv = _normal(g, (B, P, w.Hkv, w.d), device)
    if w.sink_bias and P > 0:
        s = min(w.n_sink, P)
        u = sink_direction(qsum).float()                               # [B, Hkv, d]
        pk[:, :s] += (2.0 * math.sqrt(w.d)) * u.unsqueeze(1)
    qs = torch.empty(S, B, w.Hq, w.d, dtype=torch.float32, device=device)
    ks = torch.empty(S, B, w.Hkv, w.d, dtype=torch.float32, device=device)
    vs = torch.empty(S, B, w.Hkv, w.d, dtype=torch.float32, device=device)
    for i in range(S):
        qs[i] = _normal(g, (B, w.Hq, w.d), device)
        ks[i] = _normal(g, (B, w.Hkv, w.d), device)
        vs[i] = _normal(g, (B, w.Hkv, w.d), device)
    return DecodeInputs(_round(pk, dt), _round(pv, dt), _round(qs, dt), _round(ks, dt), _round(vs, dt))


def sample_rows(L: int, window: int, n_sink: int, block: int = 128, n_random: int = 256,
                seed: int = 1) -> list:
    """Query rows checked one by one at full size: the sink and window edges, a few
    q-block edges, the last 64 rows and ``n_random`` seeded random rows."""
    rows = set(range(min(L, n_sink + 2)))
    for t in range(window - 2, window + n_sink + 2):
        if 0 <= t < L:
            rows.add(t)
    for m0 in (0, block, L // 2 - (L // 2) % block, L - L % block if L % block else L - block):
        for t in (m0 - 1, m0, m0 + 1, m0 + block - 1):
            if 0 <= t < L:
                rows.add(t)
    rows.update(range(max(0, L - 64), L))
    g = torch.Generator().manual_seed(seed)
    if L > 0:
        rows.update(torch.randint(0, L, (n_random,), generator=g).tolist())
    return sorted(rows)


@dataclasses.dataclass(frozen=True)
class ProjWorkload:
    """Output projection after attention: T token rows of n = Hq * d features."""
    name: str
    T: int
    n: int
    out_dtype: str = "bf16"
    note: str = ""

    def describe(self) -> dict:
        return {"workload": self.name, "kind": "hadamard_proj", "T": self.T, "n": self.n,
                "in_dtype": "bf16", "out_dtype": self.out_dtype}


# backward passes: (forward workload, sequence length or None for the workload's own)
BWD_WORKLOADS = {
    "bwd_based_local": ("based_local", None),
    "bwd_gqa8b_L8192": ("gqa8b_prefill", 8192),
}

ROPE_WORKLOADS = {
    # rotary encoding of the 8B-shaped prefill's q and k before attention
    "rope_qk_gqa8b": dict(T=32768, Hq=32, Hkv=8, d=128, rope_base=10000.0),
}

PROJ_WORKLOADS = {
    "hadamard_proj": ProjWorkload(
        "hadamard_proj", T=32768, n=4096,
        note="Hadamard output projection of the 8B-shaped prefill's attention output (32 x 128)"),
}


def make_hadamard(w: ProjWorkload, device="cpu", T: Optional[int] = None):
    """y [T, n] bf16 from N(0, 1); alpha [n] = 1 + 0.5 N(0, 1); beta [n] = 0.1 N(0, 1) (fp32),
    drawn in that order from the seed-0 generator."""
    T = w.T if T is None else T
    g = _gen(device)
    y = _normal(g, (T, w.n), device).to(torch.bfloat16)
    alpha = 1.0 + 0.5 * _normal(g, (w.n,), device)
    beta = 0.1 * _normal(g, (w.n,), device)
    return y, alpha, beta


@dataclasses.dataclass(frozen=True)
class LinearWorkload:
    """The linear-attention branch of a Based-style hybrid layer: H heads with
    feature dimension dk (q, k) and value dimension dv, no position encoding."""
    name: str
    B: int
    L: int
    H: int
    dk: int
    dv: int
    note: str = ""

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.dk)

    @property
    def F(self) -> int:
        return 1 + self.dk + self.dk * self.dk

    def describe(self) -> dict:
        return {"workload": self.name, "kind": "based_linear", "B": self.B, "L": self.L, "H": self.H,
                "dk": self.dk, "dv": self.dv, "features": self.F, "dtype": "bf16"}


LINEAR_WORKLOADS = {
    # the linear branch next to the based_local sliding-window branch (same B, L, heads,
    # head dim 64): feature dimension 16 gives a recurrent state of (1 + 16 + 256) x 65
    # floats per head, about the size of the window-128 branch's 2 x 128 x 64 cache
    "based_linear": LinearWorkload("based_linear", B=8, L=2048, H=16, dk=16, dv=64,
                                   note="linear-attention branch of a Based-style hybrid layer"),
}


def make_based_linear(w: LinearWorkload, device="cpu", B: Optional[int] = None, L: Optional[int] = None,
                      seed: int = SEED):
    """q, k [B, L, H, dk] and v [B, L, H, dv] bf16, each N(0, 1), drawn in that order."""
    B = w.B if B is None else B
    L = w.L if L is None else L
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    q = _normal(g, (B, L, w.H, w.dk), device)
    k = _normal(g, (B, L, w.H, w.dk), device)
    v = _normal(g, (B, L, w.H, w.dv), device)
    return q.to(torch.bfloat16), k.to(torch.bfloat16), v.to(torch.bfloat16)
