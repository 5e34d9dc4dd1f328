#!/usr/bin/env python
"""Benchmark of sink-aware sliding-window attention on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl swa|reference]
                    [--workloads packed_long,gqa8b_prefill,based_local,decode,...]

Prints ONE JSON line on rank 0.  The headline (`value`) is the prefill
throughput in TFLOP/s of the long-context packed prefill (sequences of 131072,
65536, 16384 and 1000 tokens, Hq=32, Hkv=8, d=128, window 2048, 4 sinks), the
largest workload that fits one GPU, counting 4*d FLOPs per visible (query, key)
pair, against the bf16 tensor roofline.  The same line carries, under
"workloads", the other workloads measured the same way: the 8B-shaped GQA
prefill and the Based-style local-window prefill (TFLOP/s against the tensor or
the HBM roofline), the ring-buffer decode at B=64 and B=1 (HBM GB/s and
tokens/s), the same decode with the rotary encoding fused into append and
decode, the rotary encoding of the GQA prefill's q and k, the Hadamard output
projection of the GQA prefill's output (HBM GB/s), the backward pass of the
Based-shaped and (at L=8192) the 8B-shaped prefill, the Based hybrid's
linear-attention branch (prefill in TFLOP/s of the recurrent form's FLOPs, and
its recurrent decode step in HBM GB/s), and the hybrid layer's decode (window
branch and linear branch side by side, GB/s and tokens/s).

Timing: inputs are generated on the device and stay resident; W untimed
warm-up steps; K timed steps between a barrier plus device synchronisation on
both sides; each prefill step is timed with CUDA events on the launching
stream, with a 512 MiB buffer written between steps so L2 (126 MB) holds
nothing of the next step's inputs; the decode cache (1.07 GB) is larger than
L2 by itself.  Multi-GPU runs are replicas (weak scaling): every rank runs the
same workload on its own GPU, times are reduced with a max over ranks.

`e2e` is the same metric through the C ABI with the inputs in pinned host
memory: each step copies its inputs host->device, runs the kernel(s) and
copies the outputs back, all inside the timed region.

`cpu_baseline` is the fp64 oracle on the host cores: over the headline's
sampled query rows (the sink and window edges, query-block edges, the last 64
rows and 256 seeded random rows of every sequence, all heads), as a rate on
the sample's visible pairs with the whole workload's time extrapolated from it;
the Based-style prefill in full; the GQA prefill on sampled rows; the decode on
four full steps.  `--impl reference` times the same oracle on the headline's
sample (the reference arm); it runs on rank 0 only.
"""
from __future__ import annotations

import argparse
import hashlib
import re
import json
import math
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "sink-SWA prefill TFLOP/s (visible pairs) & decode HBM GB/s, % of B200 roofline"
HEADLINE = "packed_long"
L2_FLUSH_BYTES = 512 << 20
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# --------------------------------------------------------------------------- counting
def visible_pairs(L: int, w: int, s: int) -> int:
    """Sum over query rows t < L of the number of visible keys min(t+1, w) + clamp(t-w+1, 0, s)."""
    if L <= 0:
        return 0
    band = L * (L + 1) // 2 if L <= w else w * (w + 1) // 2 + (L - w) * w
    n = L - w                      # rows whose window starts past position 0
    if n <= 0:
        sinks = 0
    elif n <= s:
        sinks = n * (n + 1) // 2
    else:
        sinks = s * (s + 1) // 2 + (n - s) * s
    return band + sinks


def prefill_flops(w, seqlens) -> int:
    return 4 * w.d * w.Hq * sum(visible_pairs(n, w.window, w.n_sink) for n in seqlens)


def prefill_bytes(w, T: int, in_bytes: int = 2, out_bytes: int = 2) -> int:
    return T * (w.Hq + 2 * w.Hkv) * w.d * in_bytes + T * w.Hq * w.d * out_bytes + T * w.Hq * 4


def decode_step_bytes(w, pos: int) -> int:
    keys = min(pos + 1, w.window) + min(max(pos - w.window + 1, 0), w.n_sink)
    cache = w.B * w.Hkv * keys * w.d * 2 * 2
    qo = 2 * w.B * w.Hq * w.d * 2 + w.B * w.Hq * 4
    append = 2 * (2 * w.B * w.Hkv * w.d * 2)     # read k_new, v_new and write them
    return cache + qo + append


def decode_step_flops(w, pos: int) -> int:
    keys = min(pos + 1, w.window) + min(max(pos - w.window + 1, 0), w.n_sink)
    return 4 * w.d * w.B * w.Hq * keys


# --------------------------------------------------------------------------- distributed
def dist_env():
    return int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")), \
        int(os.environ.get("LOCAL_RANK", "0"))


def reduce_max(x: float, device=None) -> float:
    """Max of a float over all ranks (identity without a process group)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(device=None):
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        if device is not None and device.type == "cuda":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


# --------------------------------------------------------------------------- clocks
class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML while active (read only)."""

    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x2: "applications_clocks_setting", 0x1: "gpu_idle"}

    def __init__(self, torch_device):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self._stop = threading.Event()
        self._thread = None
        self._h = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            h = None
            try:
                import torch
                uuid = str(torch.cuda.get_device_properties(torch_device).uuid)
                h = pynvml.nvmlDeviceGetHandleByUUID(uuid if uuid.startswith("GPU-") else "GPU-" + uuid)
            except Exception:
                h = None
            if h is None:
                vis = os.environ.get("CUDA_VISIBLE_DEVICES", "")
                idx = int(vis.split(",")[torch_device.index]) if vis and vis.split(",")[0].isdigit() \
                    else torch_device.index
                h = pynvml.nvmlDeviceGetHandleByIndex(idx)
            self._h = h
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self._h = None

    def _reasons_now(self):
        nv = self._nv
        for fn in ("nvmlDeviceGetCurrentClocksEventReasons", "nvmlDeviceGetCurrentClocksThrottleReasons"):
            if hasattr(nv, fn):
                try:
                    return getattr(nv, fn)(self._h)
                except Exception:
                    pass
        return 0

    def _run(self):
        nv = self._nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
                bits = self._reasons_now()
                for b, name in self.REASONS.items():
                    if bits & b and name != "gpu_idle":
                        self.reasons.add(name)
            except Exception:
                pass
            self._stop.wait(0.02)

    def __enter__(self):
        if self._h is not None:
            self._stop.clear()
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()
        return self

    def __exit__(self, *exc):
        if self._thread is not None:
            self._stop.set()
            self._thread.join()
            self._thread = None

    def summary(self):
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                "samples": len(self.samples)}


# --------------------------------------------------------------------------- helpers
def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        d = json.load(open(p))
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "source": "measured"}
    except Exception:
        return dict(PEAKS_FALLBACK, source="fallback")


def _code_only(text: str) -> str:
    """C/C++ source without its comments and with runs of white space collapsed."""
    text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
    text = re.sub(r"//[^\n]*", " ", text)
    return " ".join(text.split())


def kernel_source_hash(files=None) -> str:
    """Hash of the kernel sources (all of them, or the named files of csrc/).  Comments
    and white space are left out, so editing a comment keeps a capture valid."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "sink_aware_sliding_b200", "csrc")
    names = sorted(files) if files else sorted(n for n in os.listdir(csrc) if n.endswith((".cu", ".cuh", ".h")))
    for name in names:
        h.update(_code_only(open(os.path.join(csrc, name), encoding="utf-8").read()).encode())
    return h.hexdigest()[:16]


def profiled_traffic(workload: str):
    """DRAM bytes per launch of the workload's dominant kernel from the committed ncu
    summary, or None if the kernels changed since it was taken."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        d = json.load(open(p))
    except Exception:
        return None
    e = d.get(workload)
    if not e or e.get("kernel_hash") != kernel_source_hash(e.get("sources")):
        return None
    return e.get("dram_bytes_per_launch")


class Timer:
    """CUDA events around single launches on the current stream."""

    def __init__(self, torch):
        self.torch = torch
        self.pairs = []

    def __call__(self, fn):
        t = self.torch
        e0, e1 = t.cuda.Event(enable_timing=True), t.cuda.Event(enable_timing=True)
        e0.record()
        fn()
        e1.record()
        self.pairs.append((e0, e1))

    def ms(self):
        self.torch.cuda.synchronize()
        return [a.elapsed_time(b) for a, b in self.pairs]


# --------------------------------------------------------------------------- workloads (GPU)
def bench_prefill(name, steps, warmup, dev, flush, peaks, sampler):
    import torch

    import sink_aware_sliding_b200 as swa
    import workloads as wl
    w = wl.WORKLOADS[name]
    varlen = w.kind == "varlen"
    if varlen:
        q, k, v, cu = wl.make_varlen(w, device=dev)
        seqlens, T = list(w.seqlens), cu[-1]
        cu_d = torch.tensor(cu, dtype=torch.int32, device=dev)
        lse = torch.empty(w.Hq, T, device=dev, dtype=torch.float32)
    else:
        q, k, v = wl.make_prefill(w, device=dev)
        seqlens, T = [w.L] * w.B, w.B * w.L
        lse = torch.empty(w.B, w.Hq, w.L, device=dev, dtype=torch.float32)
    out = torch.empty_like(q)

    def run(qq=q, kk=k, vv=v, oo=out, ll=lse):
        if varlen:
            swa.swa_fwd_varlen(qq, kk, vv, oo, ll, cu_d, w.window, w.n_sink)
        else:
            swa.swa_fwd(qq, kk, vv, oo, ll, w.window, w.n_sink)

    for _ in range(warmup):
        flush.fill_(1)
        run()
    torch.cuda.synchronize()
    if swa.swa_device_error() != 0:
        raise RuntimeError(f"{name}: device wait timed out")
    timer = Timer(torch)
    barrier(dev)
    torch.cuda.synchronize()
    with sampler:
        for _ in range(steps):
            flush.fill_(1)             # evict the previous step's data from L2 (untimed)
            timer(run)
        torch.cuda.synchronize()
    barrier(dev)
    per = timer.ms()
    ms = reduce_max(sum(per), dev) / steps
    flops = prefill_flops(w, seqlens)
    alg_bytes = prefill_bytes(w, T)
    tflops = flops / (ms * 1e-3) / 1e12
    gbs = alg_bytes / (ms * 1e-3) / 1e9
    hbm_bound = flops / alg_bytes < peaks["bf16_tflops"] * 1e12 / (peaks["hbm_gbs"] * 1e9)

    # end to end through the C ABI with pinned host buffers
    hq, hk, hv = (t.cpu().pin_memory() for t in (q, k, v))
    ho = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    hl = torch.empty(lse.shape, dtype=lse.dtype).pin_memory()
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)

    def e2e_step():
        dq.copy_(hq, non_blocking=True)
        dk.copy_(hk, non_blocking=True)
        dv.copy_(hv, non_blocking=True)
        run(dq, dk, dv, out, lse)
        ho.copy_(out, non_blocking=True)
        hl.copy_(lse, non_blocking=True)

    for _ in range(max(1, warmup // 2)):
        e2e_step()
    torch.cuda.synchronize()
    e2e_steps = max(3, steps // 2)
    barrier(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(e2e_steps):
        e2e_step()
    e1.record()
    torch.cuda.synchronize()
    barrier(dev)
    e2e_ms = reduce_max(e0.elapsed_time(e1), dev) / e2e_steps
    h2d = sum(t.numel() * t.element_size() for t in (q, k, v))
    d2h = out.numel() * out.element_size() + lse.numel() * lse.element_size()

    if hbm_bound:
        roof = {"bound": "hbm", "achieved": round(gbs, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": round(gbs / peaks["hbm_gbs"], 4), "peak_source": peaks["source"]}
    else:
        roof = {"bound": "tensor", "achieved": round(tflops, 1), "peak": peaks["bf16_tflops"],
                "unit": "TFLOP/s", "frac": round(tflops / peaks["bf16_tflops"], 4),
                "frac_of_sustained": round(tflops / peaks["bf16_tflops_sustained"], 4),
                "peak_source": peaks["source"]}
    roof["traffic"] = profiled_traffic(name)
    roof["algorithmic_bytes_per_launch"] = alg_bytes
    roof["flops_per_launch"] = flops
    return {
        "config": w.describe(), "value": round(tflops, 2), "unit": "TFLOP/s", "ms_per_step": round(ms, 5),
        "achieved_gbs": round(gbs, 1), "roofline": roof,
        "e2e": {"value": round(flops / (e2e_ms * 1e-3) / 1e12, 3), "unit": "TFLOP/s",
                "ms_per_step": round(e2e_ms, 4), "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": steps, "l2": "flushed between steps (512 MiB write)",
    }


def bench_hadamard(name, steps, warmup, dev, flush, peaks, sampler):
    """Hadamard output projection over T token rows: read y (bf16), write z (bf16)."""
    import torch

    import sink_aware_sliding_b200 as swa
    import workloads as wl
    w = wl.PROJ_WORKLOADS[name]
    y, alpha, beta = wl.make_hadamard(w, device=dev)
    z = torch.empty_like(y)

    def run(yy=y, zz=z):
        swa.swa_hadamard_proj(yy, alpha, beta, zz)

    for _ in range(warmup):
        flush.fill_(1)
        run()
    torch.cuda.synchronize()
    timer = Timer(torch)
    barrier(dev)
    torch.cuda.synchronize()
    with sampler:
        for _ in range(steps):
            flush.fill_(1)
            timer(run)
        torch.cuda.synchronize()
    barrier(dev)
    ms = reduce_max(sum(timer.ms()), dev) / steps
    alg_bytes = 2 * w.T * w.n * 2 + 2 * w.n * 4
    gbs = alg_bytes / (ms * 1e-3) / 1e9

    hy = y.cpu().pin_memory()
    hz = torch.empty(z.shape, dtype=z.dtype).pin_memory()
    dy = torch.empty_like(y)

    def e2e_step():
        dy.copy_(hy, non_blocking=True)
        run(dy, z)
        hz.copy_(z, non_blocking=True)

    for _ in range(3):
        e2e_step()
    torch.cuda.synchronize()
    barrier(dev)
    n_e2e = max(3, steps // 2)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(n_e2e):
        e2e_step()
    e1.record()
    torch.cuda.synchronize()
    barrier(dev)
    e2e_ms = reduce_max(e0.elapsed_time(e1), dev) / n_e2e
    roof = {"bound": "hbm", "achieved": round(gbs, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
            "frac": round(gbs / peaks["hbm_gbs"], 4), "peak_source": peaks["source"],
            "traffic": profiled_traffic(name), "algorithmic_bytes_per_launch": alg_bytes}
    return {
        "config": w.describe(), "value": round(gbs, 1), "unit": "GB/s", "ms_per_step": round(ms, 5),
        "tokens_per_s": round(w.T / (ms * 1e-3), 1), "roofline": roof,
        "e2e": {"value": round(alg_bytes / (e2e_ms * 1e-3) / 1e9, 1), "unit": "GB/s",
                "ms_per_step": round(e2e_ms, 4), "h2d_bytes_per_step": y.numel() * 2,
                "d2h_bytes_per_step": z.numel() * 2},
        "gpu_launches": steps, "l2": "flushed between steps (512 MiB write)",
    }


def bench_rope_qk(name, steps, warmup, dev, flush, peaks, sampler):
    """Rotary encoding of a prefill's q and k in place (HBM-bound: read and write both)."""
    import torch

    import sink_aware_sliding_b200 as swa
    import workloads as wl
    c = wl.ROPE_WORKLOADS[name]
    T, Hq, Hkv, d, base = c["T"], c["Hq"], c["Hkv"], c["d"], c["rope_base"]
    g = torch.Generator(device=dev)
    g.manual_seed(wl.SEED)
    q = torch.randn(T, Hq, d, generator=g, device=dev).bfloat16()
    k = torch.randn(T, Hkv, d, generator=g, device=dev).bfloat16()
    pos = torch.arange(T, dtype=torch.int32, device=dev)

    def run(qq=q, kk=k):
        swa.swa_rope_qk(qq, kk, pos, base)

    for _ in range(warmup):
        flush.fill_(1)
        run()
    torch.cuda.synchronize()
    timer = Timer(torch)
    barrier(dev)
    torch.cuda.synchronize()
    with sampler:
        for _ in range(steps):
            flush.fill_(1)
            timer(run)
        torch.cuda.synchronize()
    barrier(dev)
    ms = reduce_max(sum(timer.ms()), dev) / steps
    alg_bytes = 2 * T * (Hq + Hkv) * d * 2 + 4 * T
    gbs = alg_bytes / (ms * 1e-3) / 1e9

    hq, hk = q.cpu().pin_memory(), k.cpu().pin_memory()
    dq, dk = torch.empty_like(q), torch.empty_like(k)

    def e2e_step():
        dq.copy_(hq, non_blocking=True)
        dk.copy_(hk, non_blocking=True)
        run(dq, dk)
        hq.copy_(dq, non_blocking=True)
        hk.copy_(dk, non_blocking=True)

    for _ in range(3):
        e2e_step()
    torch.cuda.synchronize()
    barrier(dev)
    n_e2e = max(3, steps // 2)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(n_e2e):
        e2e_step()
    e1.record()
    torch.cuda.synchronize()
    barrier(dev)
    e2e_ms = reduce_max(e0.elapsed_time(e1), dev) / n_e2e
    nb = (q.numel() + k.numel()) * 2
    roof = {"bound": "hbm", "achieved": round(gbs, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
            "frac": round(gbs / peaks["hbm_gbs"], 4), "peak_source": peaks["source"],
            "traffic": profiled_traffic(name), "algorithmic_bytes_per_launch": alg_bytes}
    return {
        "config": {"workload": name, "kind": "rope_qk", "T": T, "Hq": Hq, "Hkv": Hkv, "d": d,
                   "rope_base": base, "dtype": "bf16"},
        "value": round(gbs, 1), "unit": "GB/s", "ms_per_step": round(ms, 5), "roofline": roof,
        "e2e": {"value": round(alg_bytes / (e2e_ms * 1e-3) / 1e9, 1), "unit": "GB/s",
                "ms_per_step": round(e2e_ms, 4), "h2d_bytes_per_step": nb, "d2h_bytes_per_step": nb},
        "gpu_launches": steps, "l2": "flushed between steps (512 MiB write)",
    }


def based_linear_flops(w, tokens: int) -> float:
    """Algorithmic FLOPs of the linear branch: the recurrent form's 4 F (dv + 1) per token and
    head (adding phi(k) [v; 1]^T to the state, reading phi(q) against it)."""
    return 4.0 * w.F * (w.dv + 1) * tokens * w.H


def based_linear_bytes(w, tokens: int) -> int:
    """HBM bytes of a linear-branch prefill: q, k, v read and the bf16 output written
    (2 (2 dk + dv) + 2 dv bytes per token and head) plus the fp32 final state and
    normaliser (F (dv + 1) floats per sequence and head)."""
    return tokens * w.H * (2 * (2 * w.dk + w.dv) + 2 * w.dv) + (tokens // w.L) * w.H * w.F * (w.dv + 1) * 4


def based_linear_decode_bytes(w, B: int) -> int:
    """HBM bytes of one linear-branch decode step: the fp32 state and normaliser read
    and written, q, k, v read and the bf16 output written."""
    return B * w.H * (2 * 4 * w.F * (w.dv + 1) + 2 * (2 * w.dk + w.dv) + 2 * w.dv)


def bench_based_linear(name, steps, warmup, dev, flush, peaks, sampler):
    """Prefill of the Based linear branch: out [B, L, H, dv] and the final state."""
    import torch

    import sink_aware_sliding_b200 as swa
    import workloads as wl
    w = wl.LINEAR_WORKLOADS[name]
    q, k, v = wl.make_based_linear(w, device=dev)
    out = torch.empty(w.B, w.L, w.H, w.dv, device=dev, dtype=torch.bfloat16)
    S = torch.empty(w.B, w.H, w.F, w.dv, device=dev)
    z = torch.empty(w.B, w.H, w.F, device=dev)

    def run(qq=q, kk=k, vv=v):
        swa.swa_based_linear_fwd(qq, kk, vv, out, S, z, w.scale)

    for _ in range(warmup):
        flush.fill_(1)
        run()
    torch.cuda.synchronize()
    timer = Timer(torch)
    barrier(dev)
    torch.cuda.synchronize()
    with sampler:
        for _ in range(steps):
            flush.fill_(1)
            timer(run)
        torch.cuda.synchronize()
    barrier(dev)
    ms = reduce_max(sum(timer.ms()), dev) / steps
    flops = based_linear_flops(w, w.B * w.L)
    tf = flops / (ms * 1e-3) / 1e12

    hq, hk, hv = (x.cpu().pin_memory() for x in (q, k, v))
    ho = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    dq, dk, dv = (torch.empty_like(x) for x in (q, k, v))

    def e2e_step():
        for d_, h_ in ((dq, hq), (dk, hk), (dv, hv)):
            d_.copy_(h_, non_blocking=True)
        run(dq, dk, dv)
        ho.copy_(out, non_blocking=True)

    for _ in range(3):
        e2e_step()
    torch.cuda.synchronize()
    barrier(dev)
    n_e2e = max(3, steps // 2)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(n_e2e):
        e2e_step()
    e1.record()
    torch.cuda.synchronize()
    barrier(dev)
    e2e_ms = reduce_max(e0.elapsed_time(e1), dev) / n_e2e
    # HBM-bound at the roofline: reading q, k, v and writing out and the final state
    # (93.0 MB) takes 14.2 us at the measured copy bandwidth, the FLOPs 11 us at the
    # bf16 tensor peak
    alg_bytes = based_linear_bytes(w, w.B * w.L)
    gbs = alg_bytes / (ms * 1e-3) / 1e9
    roof = {"bound": "hbm", "achieved": round(gbs, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
            "frac": round(gbs / peaks["hbm_gbs"], 4), "peak_source": peaks["source"],
            "traffic": profiled_traffic(name), "algorithmic_bytes_per_launch": alg_bytes,
            "tensor_frac": round(tf / peaks["bf16_tflops"], 4)}
    return {
        "config": w.describe(), "value": round(tf, 3), "unit": "TFLOP/s", "ms_per_step": round(ms, 5),
        "tokens_per_s": round(w.B * w.L / (ms * 1e-3), 1), "roofline": roof,
        "e2e": {"value": round(flops / (e2e_ms * 1e-3) / 1e12, 3), "unit": "TFLOP/s",
                "ms_per_step": round(e2e_ms, 4), "h2d_bytes_per_step": (q.numel() + k.numel() + v.numel()) * 2,
                "d2h_bytes_per_step": out.numel() * 2},
        "gpu_launches": steps, "l2": "flushed between steps (512 MiB write)",
    }


def bench_based_linear_decode(name, steps, warmup, dev, flush, peaks, sampler):
    """One recurrent decode step of the linear branch for a batch: reads and writes the fp32
    state (HBM-bound; the state of B=64 x H=16 heads is 72.7 MB, so L2 is flushed between steps)."""
    import torch

    import sink_aware_sliding_b200 as swa
    import workloads as wl
    w = wl.LINEAR_WORKLOADS["based_linear"]
    B = 64
    g = torch.Generator(device=dev)
    g.manual_seed(wl.SEED)
    S = torch.randn(B, w.H, w.F, w.dv, generator=g, device=dev)
    z = 100.0 + torch.rand(B, w.H, w.F, generator=g, device=dev)
    q = torch.randn(B, w.H, w.dk, generator=g, device=dev).bfloat16()
    k = torch.randn(B, w.H, w.dk, generator=g, device=dev).bfloat16()
    v = torch.randn(B, w.H, w.dv, generator=g, device=dev).bfloat16()
    out = torch.empty(B, w.H, w.dv, device=dev, dtype=torch.bfloat16)

    def run():
        swa.swa_based_linear_decode(q, k, v, S, z, out, w.scale)

    for _ in range(warmup):
        flush.fill_(1)
        run()
    torch.cuda.synchronize()
    timer = Timer(torch)
    barrier(dev)
    torch.cuda.synchronize()
    with sampler:
        for _ in range(steps):
            flush.fill_(1)
            timer(run)
        torch.cuda.synchronize()
    barrier(dev)
    ms = reduce_max(sum(timer.ms()), dev) / steps
    alg_bytes = based_linear_decode_bytes(w, B)
    gbs = alg_bytes / (ms * 1e-3) / 1e9

    hq, hk, hv = (x.cpu().pin_memory() for x in (q, k, v))
    ho = torch.empty(out.shape, dtype=out.dtype).pin_memory()

    def e2e_step():
        q.copy_(hq, non_blocking=True)
        k.copy_(hk, non_blocking=True)
        v.copy_(hv, non_blocking=True)
        run()
        ho.copy_(out, non_blocking=True)

    for _ in range(3):
        e2e_step()
    torch.cuda.synchronize()
    barrier(dev)
    n_e2e = max(3, steps // 2)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(n_e2e):
        flush.fill_(1)
        e2e_step()
    e1.record()
    torch.cuda.synchronize()
    barrier(dev)
    e2e_ms = reduce_max(e0.elapsed_time(e1), dev) / n_e2e
    roof = {"bound": "hbm", "achieved": round(gbs, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
            "frac": round(gbs / peaks["hbm_gbs"], 4), "peak_source": peaks["source"],
            "traffic": profiled_traffic(name), "algorithmic_bytes_per_launch": alg_bytes}
    return {
        "config": {"workload": name, "kind": "based_linear_decode", "B": B, "H": w.H, "dk": w.dk, "dv": w.dv,
                   "features": w.F, "state_dtype": "f32"},
        "value": round(gbs, 1), "unit": "GB/s", "ms_per_step": round(ms, 5),
        "tokens_per_s": round(B / (ms * 1e-3), 1), "roofline": roof,
        "e2e": {"value": round(alg_bytes / (e2e_ms * 1e-3) / 1e9, 1), "unit": "GB/s",
                "ms_per_step": round(e2e_ms, 4), "note": "includes an L2 flush per step",
                "h2d_bytes_per_step": (q.numel() + k.numel() + v.numel()) * 2,
                "d2h_bytes_per_step": out.numel() * 2},
        "gpu_launches": steps, "l2": "flushed between steps (512 MiB write)",
    }


def bench_hybrid_decode(name, steps, warmup, dev, flush, peaks, sampler):
    """Decode of a Based-style hybrid layer after a 2048-token prefix, one launch per
    generated token (swa_hybrid_decode): the window branch appends to its 128-slot ring
    cache and decodes over it (H=16, d=64, no sinks), and the linear branch takes its
    recurrent step on its fixed-size state (H=16, dk=16, dv=64).  B=64 sequences; the
    state (72.7 MB) and cache (33.6 MB) fit L2 together, so L2 is flushed before each step."""
    import torch

    import sink_aware_sliding_b200 as swa
    import workloads as wl
    lw = wl.LINEAR_WORKLOADS["based_linear"]
    B, H, d, W, P = 64, lw.H, 64, 128, 2048
    g = torch.Generator(device=dev)
    g.manual_seed(wl.SEED)
    z16 = dict(device=dev, dtype=torch.bfloat16)
    kc, vc = torch.empty(B, H, W, d, **z16), torch.empty(B, H, W, d, **z16)
    sk = torch.empty(B, H, 1, d, **z16)                          # unused (no sinks)
    pk = torch.randn(B, P, H, d, generator=g, device=dev).bfloat16()
    pv = torch.randn(B, P, H, d, generator=g, device=dev).bfloat16()
    swa.swa_cache_fill(pk, pv, kc, vc, sk, sk, W, 0)
    del pk, pv
    ql, kl, vl = wl.make_based_linear(lw, device=dev, B=B, L=P)
    S = torch.empty(B, H, lw.F, lw.dv, device=dev)
    zs = torch.empty(B, H, lw.F, device=dev)
    swa.swa_based_linear_fwd(ql, kl, vl, torch.empty(B, P, H, lw.dv, **z16), S, zs, lw.scale)
    del ql, kl, vl
    n = steps + warmup
    q = torch.randn(n, B, H, d, generator=g, device=dev).bfloat16()
    kn = torch.randn(n, B, H, d, generator=g, device=dev).bfloat16()
    vn = torch.randn(n, B, H, d, generator=g, device=dev).bfloat16()
    qd = torch.randn(n, B, H, lw.dk, generator=g, device=dev).bfloat16()
    kd = torch.randn(n, B, H, lw.dk, generator=g, device=dev).bfloat16()
    vd = torch.randn(n, B, H, lw.dv, generator=g, device=dev).bfloat16()
    pos = torch.arange(P, P + n, dtype=torch.int32, device=dev).view(-1, 1).expand(-1, B).contiguous()
    out_w = torch.empty(B, H, d, **z16)
    out_l = torch.empty(B, H, lw.dv, **z16)
    lse = torch.empty(B, H, device=dev, dtype=torch.float32)

    def step(i):
        swa.swa_hybrid_decode(q[i], kn[i], vn[i], pos[i], kc, vc, sk, sk, out_w, lse, W, 0,
                              qd[i], kd[i], vd[i], S, zs, out_l, scale_l=lw.scale)

    for i in range(warmup):
        flush.fill_(1)
        step(i)
    torch.cuda.synchronize()
    timer = Timer(torch)
    barrier(dev)
    torch.cuda.synchronize()
    with sampler:
        for i in range(warmup, n):
            flush.fill_(1)
            timer(lambda i=i: step(i))
        torch.cuda.synchronize()
    barrier(dev)
    ms = reduce_max(sum(timer.ms()), dev) / steps
    if swa.swa_device_error() != 0:
        raise RuntimeError("hybrid decode reported a device wait timeout")
    # HBM bytes per step: the window cache read (k and v), the appended rows, q and out
    # of the window branch, and the linear step's state and vectors
    alg_bytes = (2 * B * H * W * d * 2 + 2 * B * H * d * 2 + 2 * B * H * d * 2 + 8 * B * H
                 + based_linear_decode_bytes(lw, B))
    gbs = alg_bytes / (ms * 1e-3) / 1e9

    # end to end: the step's inputs from pinned host memory, both branches' outputs back
    host_in = [x[warmup].cpu().pin_memory() for x in (q, kn, vn, qd, kd, vd, pos)]
    dev_in = [torch.empty_like(x, device=dev) for x in host_in]
    ho_w = torch.empty(out_w.shape, dtype=out_w.dtype).pin_memory()
    ho_l = torch.empty(out_l.shape, dtype=out_l.dtype).pin_memory()

    def e2e_step():
        for dst, src in zip(dev_in, host_in):
            dst.copy_(src, non_blocking=True)
        dq_, dk_, dv_, dql, dkl, dvl, dp = dev_in
        swa.swa_hybrid_decode(dq_, dk_, dv_, dp, kc, vc, sk, sk, out_w, lse, W, 0, dql, dkl, dvl, S, zs, out_l,
                              scale_l=lw.scale)
        ho_w.copy_(out_w, non_blocking=True)
        ho_l.copy_(out_l, non_blocking=True)

    for _ in range(3):
        e2e_step()
    torch.cuda.synchronize()
    barrier(dev)
    n_e2e = max(8, steps)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(n_e2e):
        e2e_step()
    e1.record()
    torch.cuda.synchronize()
    barrier(dev)
    e2e_ms = reduce_max(e0.elapsed_time(e1), dev) / n_e2e
    h2d = sum(x.numel() * x.element_size() for x in host_in)
    d2h = ho_w.numel() * ho_w.element_size() + ho_l.numel() * ho_l.element_size()
    roof = {"bound": "hbm", "achieved": round(gbs, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
            "frac": round(gbs / peaks["hbm_gbs"], 4), "peak_source": peaks["source"],
            "traffic": profiled_traffic(name), "algorithmic_bytes_per_launch": alg_bytes}
    return {
        "config": {"workload": name, "kind": "hybrid_decode", "B": B, "H": H, "window": W, "d": d,
                   "linear_dk": lw.dk, "linear_dv": lw.dv, "prefix": P},
        "value": round(gbs, 1), "unit": "GB/s", "ms_per_step": round(ms, 5),
        "tokens_per_s": round(B / (ms * 1e-3), 1), "roofline": roof,
        "e2e": {"value": round(B / (e2e_ms * 1e-3), 1), "unit": "tokens/s", "ms_per_step": round(e2e_ms, 4),
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": steps, "l2": "flushed between steps (512 MiB write)",
    }


def bench_bwd(name, steps, warmup, dev, flush, peaks, sampler):
    """Backward pass (dq, dk, dv) of a prefill workload; FLOPs: five products of 2*d per
    visible pair and query head (S, dP, dV, dK, dQ), i.e. 2.5x the forward's."""
    import torch

    import sink_aware_sliding_b200 as swa
    import workloads as wl
    fwd_name, L = wl.BWD_WORKLOADS[name]
    w = wl.WORKLOADS[fwd_name]
    q, k, v = wl.make_prefill(w, device=dev, L=L)
    B, Lr = q.shape[0], q.shape[1]
    out = torch.empty_like(q)
    lse = torch.empty(B, w.Hq, Lr, device=dev, dtype=torch.float32)
    swa.swa_fwd(q, k, v, out, lse, w.window, w.n_sink)
    g = torch.Generator(device=dev)
    g.manual_seed(wl.SEED + 1)
    do = torch.randn(q.shape, generator=g, device=dev).bfloat16()
    dq = torch.empty(q.shape, device=dev)
    dk = torch.empty(k.shape, device=dev)
    dv = torch.empty_like(dk)

    def run():
        swa.swa_bwd(q, k, v, out, do, lse, dq, dk, dv, w.window, w.n_sink)

    for _ in range(warmup):
        flush.fill_(1)
        run()
    torch.cuda.synchronize()
    if swa.swa_device_error() != 0:
        raise RuntimeError(f"{name}: device wait timed out")
    timer = Timer(torch)
    barrier(dev)
    torch.cuda.synchronize()
    with sampler:
        for _ in range(steps):
            flush.fill_(1)
            timer(run)
        torch.cuda.synchronize()
    barrier(dev)
    ms = reduce_max(sum(timer.ms()), dev) / steps
    flops = 2.5 * prefill_flops(w, [Lr] * B)
    tflops = flops / (ms * 1e-3) / 1e12
    roof = {"bound": "tensor", "achieved": round(tflops, 1), "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
            "frac": round(tflops / peaks["bf16_tflops"], 4), "peak_source": peaks["source"],
            "flops_per_launch": flops, "traffic": profiled_traffic(name),
            "traffic_kernel": "swa_bwd_dkdv_kernel"}
    cfg = dict(w.describe(), L=Lr, workload=name, **{"pass": "backward"})
    return {"config": cfg, "value": round(tflops, 2), "unit": "TFLOP/s", "ms_per_step": round(ms, 4),
            "roofline": roof, "gpu_launches": 2 * steps, "l2": "flushed between steps (512 MiB write)"}


def bench_decode(name, steps, warmup, dev, peaks, sampler):
    """One step = one generated token for all B sequences: cache append + split-K decode + merge."""
    import torch

    import sink_aware_sliding_b200 as swa
    import workloads as wl
    w = wl.WORKLOADS[name]
    n_tok = steps                      # generated tokens timed
    di = wl.make_decode(w, device=dev, steps=n_tok + warmup)
    B, Hq, Hkv, d, W, S = w.B, w.Hq, w.Hkv, w.d, w.window, w.n_sink
    z = dict(device=dev, dtype=torch.bfloat16)
    kc, vc = torch.empty(B, Hkv, W, d, **z), torch.empty(B, Hkv, W, d, **z)
    sk, sv = torch.empty(B, Hkv, S, d, **z), torch.empty(B, Hkv, S, d, **z)
    if w.rope_base > 0:                # the prefix keys enter the cache rotated
        pp = torch.arange(w.prefix, dtype=torch.int32, device=dev).repeat(B)
        swa.swa_rope_qk(di.prefix_k, None, pp, w.rope_base)
    swa.swa_cache_fill(di.prefix_k, di.prefix_v, kc, vc, sk, sv, W, S)
    del di.prefix_k, di.prefix_v
    pos = torch.arange(w.prefix, w.prefix + n_tok + warmup, dtype=torch.int32, device=dev)
    pos = pos.view(-1, 1).expand(-1, B).contiguous()
    out = torch.empty(B, Hq, d, **z)
    lse = torch.empty(B, Hq, device=dev, dtype=torch.float32)
    ws = torch.empty(swa.swa_decode_workspace_bytes(B, Hq, Hkv, d, W, S), device=dev, dtype=torch.uint8)

    rope = w.rope_base > 0

    def append(kn, vn, p):
        if rope:
            swa.swa_rope_cache_append(kn, vn, p, kc, vc, sk, sv, W, S, w.rope_base)
        else:
            swa.swa_cache_append(kn, vn, p, kc, vc, sk, sv, W, S)

    def dec(qq, p):
        if rope:
            swa.swa_decode_rope(qq, kc, vc, sk, sv, p, out, lse, W, S, ws, w.rope_base)
        else:
            swa.swa_decode(qq, kc, vc, sk, sv, p, out, lse, W, S, ws)

    def step(i):
        append(di.k_new[i], di.v_new[i], pos[i])
        dec(di.q[i], pos[i])

    for i in range(warmup):
        step(i)
    torch.cuda.synchronize()
    barrier(dev)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with sampler:
        e0.record()
        for i in range(warmup, warmup + n_tok):
            step(i)
        e1.record()
        torch.cuda.synchronize()
    barrier(dev)
    ms = reduce_max(e0.elapsed_time(e1), dev) / n_tok
    # dominant kernel (split-K decode + merge) timed per call on the same stream
    timer = Timer(torch)
    for i in range(warmup, warmup + min(n_tok, 64)):
        timer(lambda i=i: dec(di.q[i], pos[i]))
    dec_ms = statistics.mean(timer.ms())
    p_last = w.prefix + warmup + n_tok - 1
    step_bytes = decode_step_bytes(w, p_last)
    dec_bytes = step_bytes - 2 * (2 * B * Hkv * d * 2)      # the decode call alone
    gbs = step_bytes / (ms * 1e-3) / 1e9
    tok_s = B / (ms * 1e-3)
    dec_gbs = dec_bytes / (dec_ms * 1e-3) / 1e9

    # end to end: per step copy q, k_new, v_new, pos host->device and out, lse back
    hq, hk, hv = di.q[0].cpu().pin_memory(), di.k_new[0].cpu().pin_memory(), di.v_new[0].cpu().pin_memory()
    hp = pos[warmup].cpu().pin_memory()
    ho = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    hl = torch.empty(lse.shape, dtype=lse.dtype).pin_memory()
    dq, dk, dv, dp = (torch.empty_like(t, device=dev) for t in (hq, hk, hv, hp))

    def e2e_step():
        dq.copy_(hq, non_blocking=True)
        dk.copy_(hk, non_blocking=True)
        dv.copy_(hv, non_blocking=True)
        dp.copy_(hp, non_blocking=True)
        append(dk, dv, dp)
        dec(dq, dp)
        ho.copy_(out, non_blocking=True)
        hl.copy_(lse, non_blocking=True)

    for _ in range(3):
        e2e_step()
    torch.cuda.synchronize()
    barrier(dev)
    n_e2e = max(8, n_tok // 4)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(n_e2e):
        e2e_step()
    e1.record()
    torch.cuda.synchronize()
    barrier(dev)
    e2e_ms = reduce_max(e0.elapsed_time(e1), dev) / n_e2e
    h2d = sum(t.numel() * t.element_size() for t in (hq, hk, hv, hp))
    d2h = ho.numel() * ho.element_size() + hl.numel() * hl.element_size()
    return {
        "config": w.describe(), "value": round(gbs, 1), "unit": "GB/s", "ms_per_step": round(ms, 5),
        "tokens_per_s": round(tok_s, 1), "tflops": round(decode_step_flops(w, p_last) / (ms * 1e-3) / 1e12, 2),
        "roofline": {"bound": "hbm", "achieved": round(dec_gbs, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
                     "frac": round(dec_gbs / peaks["hbm_gbs"], 4), "peak_source": peaks["source"],
                     "traffic": profiled_traffic(name), "algorithmic_bytes_per_launch": dec_bytes,
                     "kernel_ms": round(dec_ms, 5), "step_frac": round(gbs / peaks["hbm_gbs"], 4)},
        "e2e": {"value": round(B / (e2e_ms * 1e-3), 1), "unit": "tokens/s", "ms_per_step": round(e2e_ms, 4),
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": 3 * n_tok, "l2": "cache of 1.07 GB exceeds L2",
    }


# --------------------------------------------------------------------------- oracle (CPU)
def _gen_device():
    """Where the seeded inputs are drawn: on the GPU when there is one (the same values the
    GPU arm measures), else on the host (same recipe, different generator stream)."""
    import torch
    return torch.device("cuda", 0) if torch.cuda.is_available() else torch.device("cpu")


def _f64_host(x):
    import torch
    return x.detach().to("cpu").to(torch.float64).numpy()


def oracle_prefill_sample(name: str):
    """Host copies (float64) of a prefill workload's sampled query rows and of the keys and
    values they read: per sequence, all heads of the rows {0 .. s+1, w-2 .. w+s+1, the
    edges of four 128-row query blocks, the last 64 rows, 256 random rows (seed 1)}, which
    include each sequence's first row.  Returns (parts, pairs, total_pairs) with parts a
    list of (q_rows, rows, k, v) per sequence, pairs the visible (row, head) pairs the
    sample holds and total_pairs those of the whole workload."""
    import workloads as wl
    w = wl.WORKLOADS[name]
    dev = _gen_device()
    if w.kind == "varlen":
        q, k, v, cu = wl.make_varlen(w, device=dev)
        seqs = [(q[cu[i]:cu[i] + n], k[cu[i]:cu[i] + n], v[cu[i]:cu[i] + n]) for i, n in enumerate(w.seqlens)]
    else:
        q, k, v = wl.make_prefill(w, device=dev)
        seqs = [(q[b], k[b], v[b]) for b in range(w.B)]
    parts, pairs, total = [], 0, 0
    for qs, ks, vs in seqs:
        n = qs.shape[0]
        rows = wl.sample_rows(n, w.window, w.n_sink, n_random=256, seed=1)
        parts.append((_f64_host(qs[rows]), rows, _f64_host(ks), _f64_host(vs)))
        pairs += w.Hq * sum(min(t + 1, w.window) + min(max(t - w.window + 1, 0), w.n_sink) for t in rows)
        total += w.Hq * visible_pairs(n, w.window, w.n_sink)
    del q, k, v, seqs
    return parts, pairs, total


def oracle_prefill_pass(name: str, parts) -> float:
    """One pass of the oracle over a sample; returns the seconds it took."""
    import oracle
    import workloads as wl
    w = wl.WORKLOADS[name]
    t0 = time.perf_counter()
    for q_rows, rows, k, v in parts:
        oracle.swa_rows(q_rows, rows, k, v, w.window, w.n_sink, w.scale)
    return time.perf_counter() - t0


def oracle_prefill_rate(name: str, min_seconds: float = 10.0, max_seconds: float = 30.0) -> dict:
    """The fp64 oracle on the host cores over the sampled rows of a prefill workload:
    TFLOP/s on the sample's visible pairs (4 d FLOPs per pair and head), and the time
    the whole workload would take at that rate (extrapolated, not measured)."""
    import oracle
    import workloads as wl
    w = wl.WORKLOADS[name]
    parts, pairs, total = oracle_prefill_sample(name)
    secs, passes = 0.0, 0
    while True:
        secs += oracle_prefill_pass(name, parts)
        passes += 1
        if secs >= min_seconds or secs * (passes + 1) / passes > max_seconds:
            break
    flops = 4 * w.d * pairs * passes
    rate = flops / secs
    n_rows = sum(len(p[1]) for p in parts)
    return {"value": round(rate / 1e12, 6), "unit": "TFLOP/s", "cores": oracle.num_threads(), "kind": "oracle",
            "sample": (f"{n_rows} sampled query rows x {w.Hq} heads over {len(parts)} sequence(s) "
                       f"({pairs} visible pairs), {passes} passes in {secs:.1f} s; full workload "
                       f"extrapolated at the sample's per-pair rate"),
            "pairs_per_s": round(pairs * passes / secs, 1),
            "extrapolated_full_s": round(4 * w.d * total / rate, 2)}


def oracle_decode_rate(name: str, steps: int = 4) -> dict:
    """The fp64 oracle on the host cores for ``steps`` consecutive decode steps of the
    decode workload (every sequence and head), reported per step.  For each sequence the
    keys and values the steps can see (the sinks and positions prefix-w+1 .. prefix+steps-1)
    are handed to the oracle as one short sequence in which step i is row s + w - 1 + i;
    without positional terms in the scores this is the same visible set, the same
    arithmetic and the same result."""
    import torch

    import oracle
    import workloads as wl
    w = wl.WORKLOADS[name]
    if w.rope_base > 0:
        raise ValueError("the per-step oracle timing covers the decode without rotary encoding")
    dev = _gen_device()
    di = wl.make_decode(w, device=dev, steps=steps)
    P, W, S = w.prefix, w.window, w.n_sink
    secs = 0.0
    for b in range(w.B):
        k = torch.cat([di.prefix_k[b, :S], di.prefix_k[b, P - W + 1:], di.k_new[:, b]], dim=0)
        v = torch.cat([di.prefix_v[b, :S], di.prefix_v[b, P - W + 1:], di.v_new[:, b]], dim=0)
        kh, vh, qh = _f64_host(k), _f64_host(v), _f64_host(di.q[:, b])
        rows = [S + W - 1 + i for i in range(steps)]
        t0 = time.perf_counter()
        oracle.swa_rows(qh, rows, kh, vh, W, S, w.scale)
        secs += time.perf_counter() - t0
    del di
    per_step = secs / steps
    keys = min(P + 1, W) + min(max(P - W + 1, 0), S)
    return {"value": round(decode_step_bytes(w, P) / per_step / 1e9, 4), "unit": "GB/s",
            "ms_per_step": round(per_step * 1e3, 2), "tokens_per_s": round(w.B / per_step, 2),
            "cores": oracle.num_threads(), "kind": "oracle",
            "sample": (f"{steps} full decode steps (B={w.B} x {w.Hq} heads, {keys} visible keys each) "
                       f"after the {P}-token prefix, {secs:.3f} s")}


def oracle_full_rate(name: str, min_seconds: float = 5.0, max_seconds: float = 30.0) -> dict:
    """The fp64 oracle on the host cores over a whole (small) prefill workload, repeated."""
    import oracle
    import workloads as wl
    w = wl.WORKLOADS[name]
    dev = _gen_device()
    q, k, v = (_f64_host(x) for x in wl.make_prefill(w, device=dev))
    flops = prefill_flops(w, [w.L] * w.B)
    passes, t0 = 0, time.perf_counter()
    while True:
        oracle.swa_fwd(q, k, v, w.window, w.n_sink, w.scale)
        passes += 1
        dt = time.perf_counter() - t0
        if dt >= min_seconds or dt * (passes + 1) / passes > max_seconds:
            break
    return {"value": round(flops * passes / dt / 1e12, 6), "unit": "TFLOP/s", "cores": oracle.num_threads(),
            "kind": "oracle",
            "sample": f"whole workload ({w.B} sequences x {w.L} rows x {w.Hq} heads), {passes} passes in {dt:.1f} s"}


def reference_arm(args):
    """The fp64 oracle as the reference arm: each step is one pass over the headline
    workload's sampled rows (the same sample as the GPU arm's cpu_baseline)."""
    rank, world, _ = dist_env()
    if rank != 0:
        return
    import oracle
    import workloads as wl
    w = wl.WORKLOADS[HEADLINE]
    parts, pairs, total = oracle_prefill_sample(HEADLINE)
    cores = oracle.num_threads()
    for _ in range(args.warmup):
        oracle_prefill_pass(HEADLINE, parts)
    dt = sum(oracle_prefill_pass(HEADLINE, parts) for _ in range(args.steps))
    flops = 4 * w.d * pairs
    val = flops * args.steps / dt / 1e12
    n_rows = sum(len(p[1]) for p in parts)
    sample = (f"{n_rows} sampled query rows x {w.Hq} heads over {len(parts)} sequences ({pairs} visible "
              f"pairs) per step; full workload extrapolated at this rate: "
              f"{4 * w.d * total / (flops * args.steps / dt):.1f} s")
    line = {
        "impl": "reference", "metric": METRIC, "value": round(val, 6), "unit": "TFLOP/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(dt / args.steps * 1e3, 3), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded N(0,1), bf16-rounded inputs)",
        "config": dict(wl.WORKLOADS[HEADLINE].describe(), parallelism="host cores"),
        "cpu_baseline": {"value": round(val, 6), "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": round(val, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def profile_case(args):
    """Launch one workload's kernels a few times at an optional smaller size (for ncu)."""
    import torch

    import sink_aware_sliding_b200 as swa
    import workloads as wl
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    n = args.warmup + args.steps
    if args.profile_case in wl.PROJ_WORKLOADS:
        pw = wl.PROJ_WORKLOADS[args.profile_case]
        y, alpha, beta = wl.make_hadamard(pw, device=dev, T=args.L)
        z = torch.empty_like(y)
        for _ in range(n):
            swa.swa_hadamard_proj(y, alpha, beta, z)
        torch.cuda.synchronize()
        return
    if args.profile_case in wl.BWD_WORKLOADS:
        fwd_name, L = wl.BWD_WORKLOADS[args.profile_case]
        w = wl.WORKLOADS[fwd_name]
        q, k, v = wl.make_prefill(w, device=dev, L=args.L or L)
        out = torch.empty_like(q)
        lse = torch.empty(q.shape[0], w.Hq, q.shape[1], device=dev, dtype=torch.float32)
        swa.swa_fwd(q, k, v, out, lse, w.window, w.n_sink)
        do = torch.randn_like(q)
        dq = torch.empty(q.shape, device=dev)
        dk = torch.empty(k.shape, device=dev)
        dv = torch.empty_like(dk)
        for _ in range(n):
            swa.swa_bwd(q, k, v, out, do, lse, dq, dk, dv, w.window, w.n_sink)
        torch.cuda.synchronize()
        if swa.swa_device_error() != 0:
            raise SystemExit("device wait timed out")
        return
    if args.profile_case == "hybrid_decode":
        lw = wl.LINEAR_WORKLOADS["based_linear"]
        B, H, d, W = args.B or 64, lw.H, 64, 128
        z16 = dict(device=dev, dtype=torch.bfloat16)
        kc, vc = torch.randn(B, H, W, d, device=dev).bfloat16(), torch.randn(B, H, W, d, device=dev).bfloat16()
        S = torch.randn(B, H, lw.F, lw.dv, device=dev)
        zs = 100.0 + torch.rand(B, H, lw.F, device=dev)
        q, kn, vn = (torch.randn(B, H, d, device=dev).bfloat16() for _ in range(3))
        ql, kl = (torch.randn(B, H, lw.dk, device=dev).bfloat16() for _ in range(2))
        vl = torch.randn(B, H, lw.dv, device=dev).bfloat16()
        out_w, out_l = torch.empty(B, H, d, **z16), torch.empty(B, H, lw.dv, **z16)
        for i in range(n):
            pos = torch.full((B,), 4096 + i, dtype=torch.int32, device=dev)
            swa.swa_hybrid_decode(q, kn, vn, pos, kc, vc, kc, kc, out_w, None, W, 0, ql, kl, vl, S, zs, out_l,
                                  scale_l=lw.scale)
        torch.cuda.synchronize()
        return
    if args.profile_case in ("based_linear", "based_linear_decode"):
        w = wl.LINEAR_WORKLOADS["based_linear"]
        q, k, v = wl.make_based_linear(w, device=dev, B=args.B, L=args.L)
        S = torch.zeros(q.shape[0], w.H, w.F, w.dv, device=dev)
        z = torch.zeros(q.shape[0], w.H, w.F, device=dev)
        out = torch.empty(q.shape[:3] + (w.dv,), device=dev, dtype=torch.bfloat16)
        for _ in range(n):
            if args.profile_case == "based_linear":
                swa.swa_based_linear_fwd(q, k, v, out, S, z, w.scale)
            else:
                swa.swa_based_linear_decode(q[:, 0].contiguous(), k[:, 0].contiguous(), v[:, 0].contiguous(),
                                            S, z, out[:, 0].contiguous(), w.scale)
        torch.cuda.synchronize()
        return
    if args.profile_case in wl.ROPE_WORKLOADS:
        c = wl.ROPE_WORKLOADS[args.profile_case]
        T = args.L or c["T"]
        q = torch.randn(T, c["Hq"], c["d"], device=dev).bfloat16()
        k = torch.randn(T, c["Hkv"], c["d"], device=dev).bfloat16()
        pos = torch.arange(T, dtype=torch.int32, device=dev)
        for _ in range(n):
            swa.swa_rope_qk(q, k, pos, c["rope_base"])
        torch.cuda.synchronize()
        return
    w = wl.WORKLOADS[args.profile_case]
    if w.kind == "prefill":
        q, k, v = wl.make_prefill(w, device=dev, B=args.B, L=args.L)
        out = torch.empty_like(q)
        lse = torch.empty(q.shape[0], w.Hq, q.shape[1], device=dev, dtype=torch.float32)
        for _ in range(n):
            swa.swa_fwd(q, k, v, out, lse, w.window, w.n_sink)
    elif w.kind == "varlen":
        seqlens = [int(x) for x in args.seqlens.split(",")] if args.seqlens else None
        q, k, v, cu = wl.make_varlen(w, device=dev, seqlens=seqlens)
        out = torch.empty_like(q)
        lse = torch.empty(w.Hq, cu[-1], device=dev, dtype=torch.float32)
        cu_d = torch.tensor(cu, dtype=torch.int32, device=dev)
        for _ in range(n):
            swa.swa_fwd_varlen(q, k, v, out, lse, cu_d, w.window, w.n_sink)
    else:
        B = args.B or w.B
        di = wl.make_decode(w, device=dev, B=B, steps=n)
        z = dict(device=dev, dtype=torch.bfloat16)
        kc, vc = torch.empty(B, w.Hkv, w.window, w.d, **z), torch.empty(B, w.Hkv, w.window, w.d, **z)
        sk, sv = torch.empty(B, w.Hkv, w.n_sink, w.d, **z), torch.empty(B, w.Hkv, w.n_sink, w.d, **z)
        swa.swa_cache_fill(di.prefix_k, di.prefix_v, kc, vc, sk, sv, w.window, w.n_sink)
        out = torch.empty(B, w.Hq, w.d, **z)
        lse = torch.empty(B, w.Hq, device=dev, dtype=torch.float32)
        ws = torch.empty(swa.swa_decode_workspace_bytes(B, w.Hq, w.Hkv, w.d, w.window, w.n_sink),
                         device=dev, dtype=torch.uint8)
        for i in range(n):
            pos = torch.full((B,), w.prefix + i, dtype=torch.int32, device=dev)
            if w.rope_base > 0:
                swa.swa_rope_cache_append(di.k_new[i], di.v_new[i], pos, kc, vc, sk, sv, w.window,
                                          w.n_sink, w.rope_base)
                swa.swa_decode_rope(di.q[i], kc, vc, sk, sv, pos, out, lse, w.window, w.n_sink, ws,
                                    w.rope_base)
            else:
                swa.swa_cache_append(di.k_new[i], di.v_new[i], pos, kc, vc, sk, sv, w.window, w.n_sink)
                swa.swa_decode(di.q[i], kc, vc, sk, sv, pos, out, lse, w.window, w.n_sink, ws)
    torch.cuda.synchronize()
    if swa.swa_device_error() != 0:
        raise SystemExit("device wait timed out")


# --------------------------------------------------------------------------- main
def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["swa", "reference"], default="swa")
    ap.add_argument("--workloads", default="packed_long,gqa8b_prefill,based_local,decode,decode_b1,decode_rope,"
                    "rope_qk_gqa8b,hadamard_proj,bwd_based_local,bwd_gqa8b_L8192,based_linear,based_linear_decode,"
                    "hybrid_decode")
    ap.add_argument("--decode-tokens", type=int, default=1024)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--profile-case", default=None,
                    help="only launch this workload's kernels --warmup + --steps times and print "
                         "nothing (a small, self-contained case for ncu captures)")
    ap.add_argument("--L", type=int, default=None, help="with --profile-case: sequence length")
    ap.add_argument("--B", type=int, default=None, help="with --profile-case: batch")
    ap.add_argument("--seqlens", default=None, help="with --profile-case of a packed workload: its sequence lengths")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    if args.impl == "reference":
        reference_arm(args)
        return
    if args.profile_case:
        profile_case(args)
        return

    import torch
    import torch.distributed as dist
    import datetime

    rank, world, local = dist_env()
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    import sink_aware_sliding_b200 as swa
    swa.library()

    # CPU baselines first, while the GPU is idle (rank 0, one GPU only): the oracle over the
    # headline's sampled rows, and for the other prefill and decode workloads likewise.
    cpu, cpu_other = None, {}
    names = [n for n in args.workloads.split(",") if n]
    if HEADLINE not in names:
        names.insert(0, HEADLINE)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = oracle_prefill_rate(HEADLINE)
        for n in names:
            if n == "based_local":
                cpu_other[n] = oracle_full_rate(n)
            elif n == "gqa8b_prefill":
                cpu_other[n] = oracle_prefill_rate(n, min_seconds=5.0)
            elif n in ("decode", "decode_b1"):
                cpu_other[n] = oracle_decode_rate(n)
        import torch as _t
        _t.cuda.empty_cache()

    peaks = load_peaks()
    sampler = ClockSampler(dev)
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    results = {}
    for n in names:
        if n in ("decode", "decode_rope", "decode_b1"):
            results[n] = bench_decode(n, args.decode_tokens, args.warmup, dev, peaks, sampler)
        elif n.startswith("bwd_"):
            results[n] = bench_bwd(n, max(3, args.steps // 4), args.warmup, dev, flush, peaks, sampler)
        elif n == "rope_qk_gqa8b":
            results[n] = bench_rope_qk(n, args.steps, args.warmup, dev, flush, peaks, sampler)
        elif n == "hadamard_proj":
            results[n] = bench_hadamard(n, args.steps, args.warmup, dev, flush, peaks, sampler)
        elif n == "based_linear":
            results[n] = bench_based_linear(n, args.steps, args.warmup, dev, flush, peaks, sampler)
        elif n == "based_linear_decode":
            results[n] = bench_based_linear_decode(n, args.steps, args.warmup, dev, flush, peaks, sampler)
        elif n == "hybrid_decode":
            results[n] = bench_hybrid_decode(n, args.steps, args.warmup, dev, flush, peaks, sampler)
        else:
            results[n] = bench_prefill(n, args.steps, args.warmup, dev, flush, peaks, sampler)
        if n in cpu_other:
            results[n]["cpu_baseline"] = cpu_other[n]
        torch.cuda.empty_cache()

    head = results[HEADLINE]
    clocks = sampler.summary()
    if world > 1:
        dist.destroy_process_group()
    if rank != 0:
        return
    scale = world       # weak scaling: every rank ran the same work
    line = {
        "metric": METRIC,
        "value": round(head["value"] * scale, 3),
        "unit": "TFLOP/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": head["ms_per_step"],
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16", "data": "synthetic (seeded N(0,1), bf16; see workloads/__init__.py)",
        "config": dict(head["config"], parallelism=f"replicas x{world}", l2=head["l2"]),
        "roofline": head["roofline"],
        "cpu_baseline": cpu,
        "e2e": dict(head["e2e"], value=round(head["e2e"]["value"] * scale, 3)),
        "gpu_launches": sum(r["gpu_launches"] for r in results.values()),
        "clocks": clocks,
        "workloads": {n: r for n, r in results.items() if n != HEADLINE},
        "kernel_hash": kernel_source_hash(),
    }
    print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
