"""Benchmark of the QLoRA NF4 linear layer on B200.

One step = forward (Y, T saved) + backward (dX, dA, dB) of the Llama-7B-shaped
attention projection: W 4096 x 4096 NF4 (+ double quant), 4096 tokens, LoRA
r = 16, alpha = 32, synthetic seeded inputs already resident in HBM.  Metric:
algorithmic TFLOP/s, 4MNK + 6Mr(N+K) flops per step.  Two input sets are
alternated so that consecutive steps never reuse L2 (each set is ~140 MB,
over the 126 MB L2).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

--impl reference times the CPU oracle on the host instead (a bounded token
sample of the same workload).  Under torchrun every rank runs its own
replica (weak scaling) and all-reduces its adapter gradients; the time is the
max over ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

WORKLOAD = "llama7b_attn_proj_4096x4096_m4096_r16"
GEMV_WORKLOAD = "decode_gemv_28672x8192_m1"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# Kernels the library launches per step (forward: LoRA T product with its
# in-cluster reduction, dequant-GEMM; backward: U product (also converting
# the saved T), dB product, dequant-GEMM dX, dA product).
LAUNCHES_PER_STEP = 2 + 4
# ncu DRAM traffic (read + write bytes) of one dequant-GEMM launch of this
# workload, valid only for the sources it was captured on (_source_sha).
GEMM_TRAFFIC = {"source_sha": "210d254a6052a1e8", "fwd_bytes": (44.583680 + 8.124672) * 1e6,
                "dx_bytes": (44.357120 + 3.887104) * 1e6}


def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return FALLBACK_PEAKS, "fallback"


def _source_sha():
    """sha256 prefix over the sources the dequant-GEMM kernel is compiled from."""
    h = hashlib.sha256()
    for name in ("gemm_sm100.cu", "common.cuh", "kernels.cuh"):
        with open(os.path.join(ROOT, "bit_nf4_quantised_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


class Clocks:
    """SM clock and clock-event reasons, read through NVML (read-only queries)
    as fast as NVML answers by a host thread with host timestamps.  mark() brackets the
    timed region; stop() summarises the samples inside it (falling back to
    all samples, and saying so, when the region was shorter than a few
    sampling periods).  nvidia-smi reads the same counters."""
    REASONS = (("hw_slowdown", "nvmlClocksEventReasonHwSlowdown"),
               ("hw_thermal_slowdown", "nvmlClocksEventReasonHwThermalSlowdown"),
               ("sw_thermal_slowdown", "nvmlClocksEventReasonSwThermalSlowdown"),
               ("sw_power_cap", "nvmlClocksEventReasonSwPowerCap"),
               ("hw_power_brake", "nvmlClocksEventReasonHwPowerBrakeSlowdown"))

    def __init__(self, index: int):
        self.index = index
        self.samples = []          # (host time, sm MHz, reasons bitmask)
        self.window = None
        self._stop = False
        self._thread = None
        self.error = None

    def start(self):
        import threading
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nvml = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(self.index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception as e:  # no NVML: report it instead of clocks
            self.error = f"NVML unavailable: {type(e).__name__}"
            return

        def run():
            # the clock on every pass, the event reasons on every fourth (each
            # NVML query takes a sizeable fraction of a millisecond)
            nv = self._nvml
            rs, k = 0, 0
            while not self._stop:
                try:
                    mhz = nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM)
                    if k % 4 == 0:
                        rs = nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                    k += 1
                    self.samples.append((time.perf_counter(), mhz, rs))
                except Exception:
                    pass
                time.sleep(0.0001)

        self._thread = threading.Thread(target=run, daemon=True)
        self._thread.start()

    def mark(self, t0: float, t1: float):
        self.window = (t0, t1)

    def window_summary(self, t0: float, t1: float):
        """Median SM clock and the reasons seen between two host times (call
        after stop())."""
        if self.error or self._thread is None:
            return None
        sel = [x for x in self.samples if t0 <= x[0] <= t1]
        reasons = set()
        for _, _, rs in sel:
            for name, const in self.REASONS:
                bit = getattr(self._nvml, const, 0)
                if bit and (rs & bit):
                    reasons.add(name)
        return {"sm_mhz": statistics.median([m for _, m, _ in sel]) if sel else None,
                "reasons": sorted(reasons), "samples": len(sel)}

    def stop(self):
        if self.error or self._thread is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [self.error or "not started"]}
        self._stop = True
        self._thread.join(timeout=5)
        sel = self.samples
        scope = "timed region"
        if self.window is not None:
            inside = [x for x in self.samples if self.window[0] <= x[0] <= self.window[1]]
            if len(inside) >= 3:
                sel = inside
            else:
                scope = "whole measurement (timed region shorter than the sampling period)"
        reasons = set()
        for _, _, rs in sel:
            for name, const in self.REASONS:
                bit = getattr(self._nvml, const, 0)
                if bit and (rs & bit):
                    reasons.add(name)
        try:
            self._nvml.nvmlShutdown()
        except Exception:
            pass
        return {"sm_mhz": statistics.median([m for _, m, _ in sel]) if sel else None,
                "sm_max_mhz": self.max_mhz, "reasons": sorted(reasons), "samples": len(sel),
                "scope": scope}


# ------------------------------------------------------------------ GPU arm
def _setup_layer(q, syn, lin, device):
    d = syn.make_layer(lin)
    w = q.qlora_quantize(torch.from_numpy(d["W"]).to(device))
    g = {k: d[k].to(device) for k in ("X", "A", "B", "dY")}
    return d, w, g


def _step(q, lin, w, g, bufs, ws, events=None):
    """forward + backward of one layer; events = (fwd_b, fwd_e, bwd_b, bwd_e)."""
    ev_f = (events[0], events[1]) if events else None
    ev_b = (events[2], events[3]) if events else None
    q.qlora_linear_forward(g["X"], w, g["A"], g["B"], lin.gamma, Y=bufs["Y"], T_save=bufs["T"],
                           ws=ws, events=ev_f)
    q.qlora_linear_backward(g["dY"], g["X"], w, g["A"], g["B"], lin.gamma, T_saved=bufs["T"],
                            dX=bufs["dX"], dA=bufs["dA"], dB=bufs["dB"], ws=ws, events=ev_b)


def _bufs(lin, device):
    return {"Y": torch.empty(lin.M, lin.N, dtype=torch.bfloat16, device=device),
            "T": torch.empty(lin.M, lin.r, dtype=torch.float32, device=device),
            "dX": torch.empty(lin.M, lin.K, dtype=torch.bfloat16, device=device),
            "dA": torch.empty(lin.r, lin.K, dtype=torch.float32, device=device),
            "dB": torch.empty(lin.N, lin.r, dtype=torch.float32, device=device)}


def _max_over_ranks(x: float, world: int) -> float:
    if world == 1:
        return x
    dev = "cuda" if torch.distributed.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def allreduce_adapter_grads(dA: torch.Tensor, dB: torch.Tensor) -> None:
    """Data parallelism over tokens: each rank's adapter gradients are partial
    sums over its shard; the exchange is one sum over ranks."""
    torch.distributed.all_reduce(dA)
    torch.distributed.all_reduce(dB)


# hold before the short-kernel loops: their reps queue in well under this
SHORT_HOLD_MS = 20.0


def _hold_gpu(ms):
    """Occupy the current stream for about `ms` milliseconds (torch's spin
    kernel, at the maximum SM clock) so that the launches queued behind it
    run back to back; nothing of it is inside a timed region."""
    torch.cuda._sleep(int(ms * 1e-3 * 1.965e9))


def _barrier(world):
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()


def _gemv_measure(q, syn, device, reps=20):
    """Decode GEMV (M = 1, 28672 x 8192): GB/s of algorithmic bytes of the
    forward call, weights rotated over enough copies to exceed 2x L2."""
    lin = syn.WORKLOADS[GEMV_WORKLOAD].layers[0]
    d = syn.make_layer(lin, with_grad=False)
    W0 = torch.from_numpy(d["W"]).to(device)
    copies = [q.qlora_quantize(W0) for _ in range(3)]          # 3 x 121 MB stored
    del W0
    X, A, B = (d[k].to(device) for k in ("X", "A", "B"))
    Y = torch.empty(lin.M, lin.N, dtype=torch.bfloat16, device=device)
    ws = q.workspace(lin.M, lin.N, lin.K, lin.r, device)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(reps)]
    for i in range(3):
        q.qlora_linear_forward(X, copies[i % 3], A, B, lin.gamma, Y=Y, ws=ws)
    torch.cuda.synchronize()
    call_b = torch.cuda.Event(enable_timing=True)
    call_e = torch.cuda.Event(enable_timing=True)
    _hold_gpu(SHORT_HOLD_MS)
    call_b.record()
    for i in range(reps):
        q.qlora_linear_forward(X, copies[i % 3], A, B, lin.gamma, Y=Y, ws=ws, events=evs[i])
    call_e.record()
    torch.cuda.synchronize()
    kern_ms = sum(b.elapsed_time(e) for b, e in evs) / reps
    call_ms = call_b.elapsed_time(call_e) / reps
    wbytes = copies[0].nbytes
    act = lin.M * lin.K * 2 + lin.r * lin.K * 2 + lin.N * lin.r * 2 + lin.M * lin.N * 2
    # one byte count for both rates: the stored weight, X, A, B and Y
    return {"workload": GEMV_WORKLOAD, "kernel_us": kern_ms * 1e3, "call_us": call_ms * 1e3,
            "algorithmic_bytes": wbytes + act,
            "kernel_GBps": (wbytes + act) / (kern_ms * 1e-3) / 1e9,
            "call_GBps": (wbytes + act) / (call_ms * 1e-3) / 1e9}


def _quantize_measure(q, syn, device, reps=5):
    lin = syn.WORKLOADS[WORKLOAD].layers[0]
    W = torch.randn(3, lin.N, lin.K, device=device)           # 3 x 64 MiB rotated
    outs = [q.empty_nf4(lin.N, lin.K, device) for _ in range(3)]
    for i in range(3):
        q.qlora_quantize(W[i], out=outs[i], check_finite=False)
    torch.cuda.synchronize()
    b, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    _hold_gpu(SHORT_HOLD_MS)
    b.record()
    for i in range(reps):
        q.qlora_quantize(W[i % 3], out=outs[i % 3], check_finite=False)
    e.record()
    torch.cuda.synchronize()
    ms = b.elapsed_time(e) / reps
    nbytes = lin.N * lin.K * 4 + outs[0].nbytes
    return {"kernel_us": ms * 1e3, "GBps": nbytes / (ms * 1e-3) / 1e9,
            "bytes_per_call": nbytes}


def _merge_measure(q, syn, device, reps=10):
    """Merge for export on the 28672 x 8192 decode weight (r = 16): the merge
    kernel's CUDA-event time per launch, stored weights and bf16 outputs
    rotated over two copies (2 x 590 MB > 2x L2), and GB/s of algorithmic
    bytes (stored weight + adapter read, bf16 weight written); the plain
    dequantisation of the same weight beside it."""
    lin = syn.WORKLOADS[GEMV_WORKLOAD].layers[0]
    W = torch.randn(lin.N, lin.K, device=device) * lin.sigma
    ws = [q.qlora_quantize(W, check_finite=False) for _ in range(2)]
    del W
    A = (torch.randn(lin.r, lin.K, device=device) / lin.K ** 0.5).bfloat16()
    B = (torch.randn(lin.N, lin.r, device=device) * 0.01).bfloat16()
    outs = [torch.empty(lin.N, lin.K, dtype=torch.bfloat16, device=device) for _ in range(2)]

    def timed(fn):
        for i in range(3):
            fn(i)
        torch.cuda.synchronize()
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(reps)]
        _hold_gpu(SHORT_HOLD_MS)
        for i in range(reps):
            evs[i][0].record()
            fn(i)
            evs[i][1].record()
        torch.cuda.synchronize()
        return sum(b.elapsed_time(e) for b, e in evs) / reps * 1e3

    mu = timed(lambda i: q.qlora_merge(ws[i % 2], A, B, lin.gamma, out=outs[i % 2]))
    du = timed(lambda i: q.qlora_dequantize(ws[i % 2], out=outs[i % 2]))
    stored = ws[0].nbytes
    mb = stored + (lin.r * lin.K + lin.N * lin.r) * 2 + lin.N * lin.K * 2
    db = stored + lin.N * lin.K * 2
    del ws, outs
    return {"workload": f"merge_{lin.N}x{lin.K}_r{lin.r}", "kernel_us": round(mu, 2),
            "GBps": round(mb / mu / 1e3, 1), "algorithmic_bytes": mb,
            "dequantize_us": round(du, 2), "dequantize_GBps": round(db / du / 1e3, 1)}


def _adam8_measure(q, syn, device, reps=10):
    """AdamW with 8-bit state over every adapter of the 32-layer decoder
    (r = 16: 40 M parameters as one flat fp32 tensor), one launch per step
    with the bf16 copy written; GB/s of algorithmic bytes per parameter:
    p 4 + 4, g 4, two 1-byte codes read and written, bf16 copy 2 (18 B)."""
    lins = syn.WORKLOADS["llama7b_decoder_32layers_m4096_r16"].layers
    n = sum(l.r * (l.K + l.N) for l in lins)
    p = torch.randn(n, device=device) * 0.02
    g = torch.randn(n, device=device)
    pb = torch.empty(n, dtype=torch.bfloat16, device=device)
    st = q.adamw8_state(n, device)
    for _ in range(3):
        q.qlora_adamw8_step(p, g, st, 2e-4, weight_decay=0.01, p_bf16=pb)
    torch.cuda.synchronize()
    b, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    _hold_gpu(SHORT_HOLD_MS)
    b.record()
    for _ in range(reps):
        q.qlora_adamw8_step(p, g, st, 2e-4, weight_decay=0.01, p_bf16=pb)
    e.record()
    torch.cuda.synchronize()
    us = b.elapsed_time(e) / reps * 1e3
    nbytes = n * 18 + 2 * 2 * 4 * ((n + 63) // 64)
    return {"params": n, "kernel_us": round(us, 2), "GBps": round(nbytes / us / 1e3, 1),
            "bytes_per_step": nbytes}


def _format_measure(q, device, reps=10):
    """Format variants on a 28672 x 8192 weight (235 M weights, 940 MB fp32):
    quantise and bf16 dequantise throughput for NF4 / FP4 at blocksize 64 with
    FP8 scales, NF4 at 16 with fp32 scales and NF4 at 4096.  GB/s of
    algorithmic bytes (fp32 read + stored written; stored read + bf16 written).
    The codebooks are built here from their definitions: NF4 from the library,
    E2M1 FP4 as {0, 0.5, 1, 1.5, 2, 3, 4, 6}/6 with sign."""
    nf4, _ = q.nf4_build_codebook()
    mags = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
    fp4 = sorted(set([-m / 6.0 for m in mags] + [m / 6.0 for m in mags]))
    n = 28672 * 8192
    W = torch.randn(n, device=device) * 0.02
    out = torch.empty(n, dtype=torch.bfloat16, device=device)
    rows = []
    for name, codes, block, sc in (("nf4_b64_e4m3", nf4, 64, q.QLORA_SCALES_E4M3),
                                   ("fp4_b64_e4m3", fp4, 64, q.QLORA_SCALES_E4M3),
                                   ("nf4_b16_fp32", nf4, 16, q.QLORA_SCALES_FP32),
                                   ("nf4_b4096_e4m3", nf4, 4096, q.QLORA_SCALES_E4M3)):
        f = q.Format(tuple(codes), block, sc)
        p, s, m = q.qlora_quantize_fmt(W, f, check_finite=False)
        stored = p.numel() + s.numel() * s.element_size() + (m.numel() * 4 if m is not None else 0)

        def timed(fn):
            fn()
            torch.cuda.synchronize()
            b, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            _hold_gpu(SHORT_HOLD_MS)
            b.record()
            for _ in range(reps):
                fn()
            e.record()
            torch.cuda.synchronize()
            return b.elapsed_time(e) / reps * 1e3

        qu = timed(lambda: q.qlora_quantize_fmt(W, f, check_finite=False))
        du = timed(lambda: q.qlora_dequantize_fmt(p, s, m, n, f, out=out))
        rows.append({"format": name, "quantize_us": round(qu, 1),
                     "quantize_GBps": round((n * 4 + stored) / qu / 1e3, 1),
                     "dequantize_us": round(du, 1),
                     "dequantize_GBps": round((n * 2 + stored) / du / 1e3, 1)})
    del W, out
    return rows


def _gemv_sweep(q, syn, device, reps=10):
    """The decode sweep: 28672 x 8192 and 8192 x 28672 weights with 1, 4 and
    16 tokens.  Per shape the GEMV kernel's CUDA-event time (weights rotated
    over 3 stored copies, 363 MB > 2x L2) and its algorithmic bytes (stored
    weight + activations) per second."""
    out = []
    for (N, K) in ((28672, 8192), (8192, 28672)):
        lin0 = syn.WORKLOADS[f"decode_gemv_{N}x{K}_m1"].layers[0]
        W0 = syn.make_weight(lin0, np.random.default_rng(lin0.seed))
        Wd = torch.from_numpy(W0).to(device)
        copies = [q.qlora_quantize(Wd) for _ in range(3)]
        del Wd, W0
        for M in (1, 4, 16):
            lin = syn.WORKLOADS[f"decode_gemv_{N}x{K}_m{M}"].layers[0]
            d = syn.make_layer(lin, with_grad=False)
            X, A, B = (d[k].to(device) for k in ("X", "A", "B"))
            Y = torch.empty(M, N, dtype=torch.bfloat16, device=device)
            ws = q.workspace(M, N, K, lin.r, device)
            for i in range(3):
                q.qlora_linear_forward(X, copies[i % 3], A, B, lin.gamma, Y=Y, ws=ws)
            evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                   for _ in range(reps)]
            torch.cuda.synchronize()
            _hold_gpu(SHORT_HOLD_MS)
            for i in range(reps):
                q.qlora_linear_forward(X, copies[i % 3], A, B, lin.gamma, Y=Y, ws=ws,
                                       events=evs[i])
            torch.cuda.synchronize()
            us = sum(b.elapsed_time(e) for b, e in evs) / reps * 1e3
            nbytes = copies[0].nbytes + M * K * 2
            out.append({"workload": f"decode_gemv_{N}x{K}_m{M}", "kernel_us": round(us, 2),
                        "GBps": round(nbytes / (us * 1e-6) / 1e9, 1)})
        del copies
    return out


def _decoder_measure(q, syn, device, steps=2):
    """The 32-layer decoder (224 linears, 4096 tokens, r = 16): one-time
    quantise throughput over all 224 weights, then layer-by-layer forward of
    every linear followed by the backward of every linear, timed with CUDA
    events.  Weights and activations are drawn on the GPU from a seeded
    generator (N(0, 0.02^2) weights, N(0, 1) activations): the timing does not
    depend on the values, and drawing 6.5e9 weights on the host would take
    minutes.  The seven linears of a layer (q, k, v, o, gate, up, down) each
    have their own source weight and activations, shared across layers, so
    consecutive calls never find their inputs in L2."""
    lins = syn.WORKLOADS["llama7b_decoder_32layers_m4096_r16"].layers
    gen = torch.Generator(device=device)
    gen.manual_seed(5)
    kinds = {l.name.split(".")[1]: (l.N, l.K) for l in lins}
    kind = lambda l: l.name.split(".")[1]
    src = {k: torch.randn(n, kk, device=device, generator=gen) * 0.02 for k, (n, kk) in kinds.items()}
    ws = [q.empty_nf4(l.N, l.K, device) for l in lins]
    for l, w in zip(lins[:7], ws[:7]):
        q.qlora_quantize(src[kind(l)], out=w, check_finite=False)
    torch.cuda.synchronize()
    b, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    b.record()
    for l, w in zip(lins, ws):
        q.qlora_quantize(src[kind(l)], out=w, check_finite=False)
    e.record()
    torch.cuda.synchronize()
    q1_ms = b.elapsed_time(e)
    b.record()
    q.qlora_quantize_many([(src[kind(l)], w) for l, w in zip(lins, ws)], check_finite=False)
    e.record()
    torch.cuda.synchronize()
    q_ms = b.elapsed_time(e)
    params = sum(l.N * l.K for l in lins)
    q_bytes = params * 4 + sum(w.nbytes for w in ws)
    del src
    M, r = lins[0].M, lins[0].r
    act = {}
    for k, (N, K) in kinds.items():
        act[k] = {
            "X": torch.randn(M, K, device=device, generator=gen).bfloat16(),
            "dY": torch.randn(M, N, device=device, generator=gen).bfloat16(),
            "A": (torch.randn(r, K, device=device, generator=gen) / K ** 0.5).bfloat16(),
            "B": (torch.randn(N, r, device=device, generator=gen) * 0.01).bfloat16(),
            "Y": torch.empty(M, N, dtype=torch.bfloat16, device=device),
            "dX": torch.empty(M, K, dtype=torch.bfloat16, device=device),
            "dA": torch.empty(r, K, dtype=torch.float32, device=device),
            "dB": torch.empty(N, r, dtype=torch.float32, device=device)}
    Ts = [torch.empty(M, r, dtype=torch.float32, device=device) for _ in lins]
    wsp = q.workspace(M, max(n for n, _ in kinds.values()), max(kk for _, kk in kinds.values()), r,
                      device)

    def step():
        for l, w, T in zip(lins, ws, Ts):
            a = act[kind(l)]
            q.qlora_linear_forward(a["X"], w, a["A"], a["B"], l.gamma, Y=a["Y"], T_save=T, ws=wsp)
        for l, w, T in zip(reversed(lins), reversed(ws), reversed(Ts)):
            a = act[kind(l)]
            q.qlora_linear_backward(a["dY"], a["X"], w, a["A"], a["B"], l.gamma, T_saved=T,
                                    dX=a["dX"], dA=a["dA"], dB=a["dB"], ws=wsp)

    step()
    torch.cuda.synchronize()
    b.record()
    for _ in range(steps):
        step()
    e.record()
    torch.cuda.synchronize()
    ms = b.elapsed_time(e) / steps
    flops = sum(l.fwd_bwd_flops() for l in lins)
    out = {"workload": "llama7b_decoder_32layers_m4096_r16", "linears": len(lins),
           "fwd_bwd_ms": round(ms, 3), "fwd_bwd_TFLOPs": round(flops / (ms * 1e-3) / 1e12, 2),
           "quantize_ms": round(q_ms, 3), "quantize_params": params,
           "quantize_GBps": round(q_bytes / (q_ms * 1e-3) / 1e9, 1),
           "quantize_one_by_one_ms": round(q1_ms, 3),
           "quantize_one_by_one_GBps": round(q_bytes / (q1_ms * 1e-3) / 1e9, 1)}
    del Ts, wsp
    for a in act.values():
        for k in ("X", "dY", "Y", "dX", "dA", "dB"):
            del a[k]
    out["export"] = _export_measure(q, lins, ws, act, kind, device)
    return out


def _export_measure(q, lins, ws, act, kind, device, reps=3):
    """Export of the whole fine-tuned decoder: every one of the 224 stored
    weights merged with its adapter into its own slice of one bf16 buffer
    (13 GB, far beyond L2) by one qlora_merge_many call (16 weights per
    launch), timed with CUDA events, and beside it the same merges as 224
    qlora_merge calls; then the same buffer re-quantised to NF4, and, for
    comparison, the plain dequantisation of every weight.  GB/s are algorithmic bytes: the stored
    weight read, the adapter read and the bf16 weight written (merge), the
    bf16 read and the stored weight written (re-quantise: one
    qlora_quantize_many call, and 224 qlora_quantize_bf16 calls beside it)."""
    params = sum(l.N * l.K for l in lins)
    buf = torch.empty(params, dtype=torch.bfloat16, device=device)
    views, o = [], 0
    for l in lins:
        views.append(buf[o:o + l.N * l.K].view(l.N, l.K))
        o += l.N * l.K
    re_ws = [q.empty_nf4(l.N, l.K, device) for l in lins]
    stored = sum(w.nbytes for w in ws)
    adapter = sum((l.r * l.K + l.N * l.r) * 2 for l in lins)

    def timed(fn):
        fn()
        torch.cuda.synchronize()
        b, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        b.record()
        for _ in range(reps):
            fn()
        e.record()
        torch.cuda.synchronize()
        return b.elapsed_time(e) / reps

    def merge_all():
        q.qlora_merge_many([(w, act[kind(l)]["A"], act[kind(l)]["B"], l.gamma, v)
                            for l, w, v in zip(lins, ws, views)])

    def merge_each():
        for l, w, v in zip(lins, ws, views):
            a = act[kind(l)]
            q.qlora_merge(w, a["A"], a["B"], l.gamma, out=v)

    def requant_all():
        q.qlora_quantize_many(list(zip(views, re_ws)), check_finite=False)

    def requant_each():
        for w, v in zip(re_ws, views):
            q.qlora_quantize_bf16(v, out=w, check_finite=False)

    def dequant_all():
        for w, v in zip(ws, views):
            q.qlora_dequantize(w, out=v)

    m_ms = timed(merge_all)
    m1_ms = timed(merge_each)
    r_ms = timed(requant_all)
    r1_ms = timed(requant_each)
    d_ms = timed(dequant_all)
    m_bytes = stored + adapter + params * 2
    r_bytes = params * 2 + sum(w.nbytes for w in re_ws)
    d_bytes = stored + params * 2
    del buf, views, re_ws
    return {"linears": len(lins), "params": params,
            "merge_ms": round(m_ms, 3), "merge_GBps": round(m_bytes / (m_ms * 1e-3) / 1e9, 1),
            "merge_bytes": m_bytes,
            "merge_one_by_one_ms": round(m1_ms, 3),
            "merge_one_by_one_GBps": round(m_bytes / (m1_ms * 1e-3) / 1e9, 1),
            "requantize_ms": round(r_ms, 3),
            "requantize_GBps": round(r_bytes / (r_ms * 1e-3) / 1e9, 1),
            "requantize_one_by_one_ms": round(r1_ms, 3),
            "requantize_one_by_one_GBps": round(r_bytes / (r1_ms * 1e-3) / 1e9, 1),
            "dequantize_ms": round(d_ms, 3),
            "dequantize_GBps": round(d_bytes / (d_ms * 1e-3) / 1e9, 1)}


def _mlp_measure(q, syn, device, reps=6):
    """Llama-7B MLP (gate, up 4096 -> 11008, down 11008 -> 4096, 8192 tokens,
    r = 64, alpha = 16): each linear's forward + backward on its own (CUDA
    events around the step and around its two dequant-GEMM launches), and the
    chained SwiGLU block through qlora_mlp_forward / qlora_mlp_backward, whose
    backward recomputes gate and up (checkpointing).  Weights and activations
    are drawn on the GPU (timing does not depend on the values)."""
    lins = syn.WORKLOADS["llama7b_mlp_m8192_r64"].layers
    gen = torch.Generator(device=device).manual_seed(5)
    M, r, gamma = lins[0].M, lins[0].r, lins[0].gamma
    D, F = lins[0].K, lins[0].N
    store, A, B = {}, {}, {}
    for lin, name in zip(lins, ("gate", "up", "down")):
        W = torch.randn(lin.N, lin.K, device=device, generator=gen) * lin.sigma
        store[name] = q.qlora_quantize(W, check_finite=False)
        del W
        A[name] = (torch.randn(r, lin.K, device=device, generator=gen) / lin.K ** 0.5).bfloat16()
        B[name] = (torch.randn(lin.N, r, device=device, generator=gen) * 0.01).bfloat16()
    X = torch.randn(M, D, device=device, generator=gen).bfloat16()
    dY = torch.randn(M, D, device=device, generator=gen).bfloat16()
    dYf = torch.randn(M, F, device=device, generator=gen).bfloat16()
    Hin = torch.randn(M, F, device=device, generator=gen).bfloat16()
    peaks, _ = _peaks()
    rows = []
    total_flops, total_ms = 0, 0.0
    for lin, name in zip(lins, ("gate", "up", "down")):
        x = X if name != "down" else Hin
        dy = dYf if name != "down" else dY
        ws = q.workspace(M, lin.N, lin.K, r, device)
        bufs = {"Y": torch.empty(M, lin.N, dtype=torch.bfloat16, device=device),
                "T": torch.empty(M, r, dtype=torch.float32, device=device),
                "dX": torch.empty(M, lin.K, dtype=torch.bfloat16, device=device),
                "dA": torch.empty(r, lin.K, dtype=torch.float32, device=device),
                "dB": torch.empty(lin.N, r, dtype=torch.float32, device=device)}
        g = {"X": x, "A": A[name], "B": B[name], "dY": dy}
        for _ in range(3):
            _step(q, lin, store[name], g, bufs, ws)
        torch.cuda.synchronize()
        b, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        b.record()
        for _ in range(reps):
            _step(q, lin, store[name], g, bufs, ws)
        e.record()
        torch.cuda.synchronize()
        ms = b.elapsed_time(e) / reps
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(reps)]
        for i in range(reps):
            _step(q, lin, store[name], g, bufs, ws, evs[i])
        torch.cuda.synchronize()
        if q.device_error_word(ws) != 0:
            raise RuntimeError(f"device error word set in the {name} linear")
        fwd = sum(v[0].elapsed_time(v[1]) for v in evs) / reps
        dx = sum(v[2].elapsed_time(v[3]) for v in evs) / reps
        f_gemm = 2 * M * lin.N * lin.K * 2 + 2 * M * r * (lin.N + lin.K)
        flops = lin.fwd_bwd_flops()
        total_flops += flops
        total_ms += ms
        rows.append({"linear": name, "N": lin.N, "K": lin.K, "ms": round(ms, 4),
                     "TFLOPs": round(flops / (ms * 1e-3) / 1e12, 1),
                     "gemm_fwd_us": round(fwd * 1e3, 1), "gemm_dx_us": round(dx * 1e3, 1),
                     "gemm_TFLOPs": round(f_gemm / ((fwd + dx) * 1e-3) / 1e12, 1),
                     "gemm_frac_bf16": round(f_gemm / ((fwd + dx) * 1e-3) / 1e12 / peaks["bf16_tflops"], 4)})
    mlp = q.MLP(store["gate"], store["up"], store["down"], A["gate"], B["gate"], A["up"], B["up"],
                A["down"], B["down"])
    ws = q.mlp_workspace(M, mlp, device)
    Y = torch.empty(M, D, dtype=torch.bfloat16, device=device)
    dX = torch.empty(M, D, dtype=torch.bfloat16, device=device)
    grads = {}
    for lin, name in zip(lins, ("gate", "up", "down")):
        grads[f"dA_{name}"] = torch.empty(r, lin.K, dtype=torch.float32, device=device)
        grads[f"dB_{name}"] = torch.empty(lin.N, r, dtype=torch.float32, device=device)

    def chained():
        q.qlora_mlp_forward(X, mlp, gamma, Y=Y, ws=ws)
        q.qlora_mlp_backward(dY, X, mlp, gamma, dX=dX, grads=grads, ws=ws)

    for _ in range(3):
        chained()
    torch.cuda.synchronize()
    b, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    b.record()
    for _ in range(reps):
        chained()
    e.record()
    torch.cuda.synchronize()
    if q.device_error_word(ws) != 0:
        raise RuntimeError("device error word set in the chained MLP")
    cms = b.elapsed_time(e) / reps
    recompute = sum(l.fwd_flops() for l in lins[:2])
    return {"workload": "llama7b_mlp_m8192_r64", "per_linear": rows,
            "independent_ms": round(total_ms, 3),
            "independent_TFLOPs": round(total_flops / (total_ms * 1e-3) / 1e12, 1),
            "independent_frac_bf16": round(total_flops / (total_ms * 1e-3) / 1e12 / peaks["bf16_tflops"], 4),
            "chained": {"step": "forward, then backward recomputing gate(x), up(x) and h",
                        "ms": round(cms, 3), "algorithmic_flops": total_flops,
                        "recompute_flops": recompute,
                        "TFLOPs": round(total_flops / (cms * 1e-3) / 1e12, 1),
                        "TFLOPs_with_recompute": round((total_flops + recompute) / (cms * 1e-3) / 1e12, 1)}}


def run_gpu(args):
    import bit_nf4_quantised_b200 as q
    from bit_nf4_quantised_b200 import synthetic as syn

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    if world > 1:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    q.lib()
    lin = syn.WORKLOADS[WORKLOAD].layers[0]
    sets = []
    for s in range(2):                      # two input sets, alternated
        import dataclasses
        l2 = dataclasses.replace(lin, seed=lin.seed + 1000 * rank + s)
        _, w, g = _setup_layer(q, syn, l2, device)
        sets.append((w, g))
    bufs = _bufs(lin, device)
    ws = q.workspace(lin.M, lin.N, lin.K, lin.r, device)
    K = args.steps
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(K)]

    def one(i, events=None):
        w, g = sets[i % 2]
        _step(q, lin, w, g, bufs, ws, events)
        if world > 1:
            allreduce_adapter_grads(bufs["dA"], bufs["dB"])

    hw = time.perf_counter()
    for i in range(args.warmup):
        one(i)
    # hold long enough for the host to queue all K steps (from the warm-up's
    # enqueue rate, which includes first-call costs, so it errs long)
    hold_ms = min(2000.0, max(20.0, 1.5 * K * (time.perf_counter() - hw) * 1e3 / max(1, args.warmup)))
    _barrier(world)
    if q.device_error_word(ws) != 0:
        raise RuntimeError("device error word set during warm-up")
    clocks = Clocks(local)
    clocks.start()
    _barrier(world)
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    # A spin kernel holds the GPU while the host queues the steps, and the
    # timing starts after it: the timed region then measures the GPU's work
    # from a full queue, not the host's launch rate.
    _hold_gpu(hold_ms)
    h0 = time.perf_counter()
    t0.record()
    for i in range(K):
        one(i)
    t1.record()
    h_enq = time.perf_counter() - h0
    _barrier(world)
    clocks.mark(h0, time.perf_counter())
    # The GEMM kernels' own durations come from the same K steps run again
    # right after, with CUDA events recorded around the two GEMM launches on
    # the streams they run on.  They are not recorded inside the timed steps:
    # an event between the LoRA kernel and the forward GEMM would stop the
    # GEMM from starting as the LoRA kernel's programmatic dependent.
    _hold_gpu(hold_ms)
    h2 = time.perf_counter()
    for i in range(K):
        one(i, evs[i])
    h_enq_ev = time.perf_counter() - h2
    _barrier(world)
    h3 = time.perf_counter()
    clk = clocks.stop()
    gemm_clk = clocks.window_summary(h2, h3)
    ms = _max_over_ranks(t0.elapsed_time(t1), world) / K
    fwd_ms = sum(e[0].elapsed_time(e[1]) for e in evs) / K
    dx_ms = sum(e[2].elapsed_time(e[3]) for e in evs) / K

    flops = lin.fwd_bwd_flops()
    value = world * flops / (ms * 1e-3) / 1e12
    peaks, peak_kind = _peaks()
    M, N, Kd, r = lin.M, lin.N, lin.K, lin.r
    f_fwd = 2 * M * N * Kd + 2 * M * r * N          # main product + LoRA tail in the kernel
    f_dx = 2 * M * N * Kd + 2 * M * r * Kd
    achieved = (f_fwd + f_dx) / ((fwd_ms + dx_ms) * 1e-3) / 1e12
    peak = peaks["bf16_tflops"]
    sha = _source_sha()
    traffic = None
    if GEMM_TRAFFIC["source_sha"] == sha and GEMM_TRAFFIC["fwd_bytes"]:
        traffic = (GEMM_TRAFFIC["fwd_bytes"] + GEMM_TRAFFIC["dx_bytes"]) / 2
    out = {
        "metric": "QLoRA linear fwd+bwd TFLOP/s (% bf16 peak); NF4 dequant-GEMV GB/s (% HBM)",
        "value": round(value, 2), "unit": "TFLOP/s", "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": round(ms, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": WORKLOAD, "M": M, "N": N, "K": Kd, "r": r, "alpha": lin.alpha,
                   "step": "forward (Y, T) + backward (dX, dA, dB)",
                   "l2": "two input sets alternated, each ~140 MB > 126 MB L2",
                   "parallelism": f"replicas{world}" if world > 1 else "single"},
        "roofline": {"bound": "tensor", "kernel": "qlora_gemm_kernel (forward + dX launches)",
                     "achieved": round(achieved, 2), "peak": peak, "unit": "TFLOP/s",
                     "frac": round(achieved / peak, 4), "peak_source": f"{peak_kind} bf16 burst",
                     "traffic": traffic, "fwd_us": round(fwd_ms * 1e3, 2),
                     "dx_us": round(dx_ms * 1e3, 2), "clocks": gemm_clk,
                     "timing": "CUDA events around each GEMM launch, the same steps rerun "
                               "right after the timed region"},
        "host_enqueue_ms_per_step": {"timed": round(h_enq * 1e3 / K, 4),
                                     "gemm_events_pass": round(h_enq_ev * 1e3 / K, 4),
                                     "held_ms": round(hold_ms, 1)},
        "gpu_launches": LAUNCHES_PER_STEP * K,
        "clocks": clk,
    }
    if rank == 0 and world == 1:
        out["gemv"] = _gemv_measure(q, syn, device)
        out["gemv"]["frac_hbm"] = round(out["gemv"]["kernel_GBps"] / peaks["hbm_gbs"], 4)
        out["quantize"] = _quantize_measure(q, syn, device)
        out["gemv_sweep"] = _gemv_sweep(q, syn, device)
        for row in out["gemv_sweep"]:
            row["frac_hbm"] = round(row["GBps"] / peaks["hbm_gbs"], 4)
        out["decoder"] = _decoder_measure(q, syn, device)
        out["decoder"]["frac_bf16"] = round(out["decoder"]["fwd_bwd_TFLOPs"] / peak, 4)
        ex = out["decoder"]["export"]
        out["decoder"]["quantize_frac_hbm"] = round(out["decoder"]["quantize_GBps"] / peaks["hbm_gbs"], 4)
        for k in ("merge", "merge_one_by_one", "requantize", "requantize_one_by_one", "dequantize"):
            ex[f"{k}_frac_hbm"] = round(ex[f"{k}_GBps"] / peaks["hbm_gbs"], 4)
        try:
            out["merge"] = _merge_measure(q, syn, device)
            out["merge"]["frac_hbm"] = round(out["merge"]["GBps"] / peaks["hbm_gbs"], 4)
        except Exception as exc:           # an extra measurement never sinks the bench line
            out["merge"] = {"error": f"{type(exc).__name__}: {exc}"}
        try:
            out["adamw8"] = _adam8_measure(q, syn, device)
            out["adamw8"]["frac_hbm"] = round(out["adamw8"]["GBps"] / peaks["hbm_gbs"], 4)
        except Exception as exc:           # an extra measurement never sinks the bench line
            out["adamw8"] = {"error": f"{type(exc).__name__}: {exc}"}
        try:
            out["mlp"] = _mlp_measure(q, syn, device)
        except Exception as exc:           # an extra measurement never sinks the bench line
            out["mlp"] = {"error": f"{type(exc).__name__}: {exc}"}
        try:
            out["formats"] = _format_measure(q, device)
            for row in out["formats"]:
                row["dequantize_frac_hbm"] = round(row["dequantize_GBps"] / peaks["hbm_gbs"], 4)
        except Exception as exc:           # an extra measurement never sinks the bench line
            out["formats"] = {"error": f"{type(exc).__name__}: {exc}"}
        out["e2e"] = _e2e(q, syn, lin, device, max(3, K // 2))
        out["cpu_baseline"] = _cpu_baseline(seconds=args.cpu_seconds)
    else:
        out["e2e"] = _e2e(q, syn, lin, device, max(3, K // 2), world=world)
    if world > 1:
        torch.distributed.destroy_process_group()
    if rank == 0:
        print(json.dumps(out))


def _e2e(q, syn, lin, device, steps, world=1):
    """Same step through the public API with host buffers: pinned host X and
    dY copied in, Y, dX, dA, dB copied out, every step, all inside the timed
    region.  The copies run on their own streams with device inputs and
    outputs double-buffered, so that step i+1's inputs go in and step i-1's
    results come out (PCIe is full duplex) while step i computes; events order
    each buffer's reuse after its last reader."""
    d = syn.make_layer(lin)
    w = q.qlora_quantize(torch.from_numpy(d["W"]).to(device))
    host_in = {k: d[k].pin_memory() for k in ("X", "dY")}
    gs = [{k: d[k].to(device) for k in ("X", "A", "B", "dY")} for _ in range(2)]
    bufs = [_bufs(lin, device) for _ in range(2)]
    host_out = {k: torch.empty_like(v, device="cpu").pin_memory() for k, v in bufs[0].items()
                if k != "T"}
    ws = q.workspace(lin.M, lin.N, lin.K, lin.r, device)
    s_in, s_cmp, s_out = (torch.cuda.Stream(device) for _ in range(3))
    ev = lambda: torch.cuda.Event()
    in_done = [ev(), ev()]       # inputs of buffer set b landed
    cmp_done = [ev(), ev()]      # step on buffer set b finished (inputs free, outputs ready)
    out_done = [ev(), ev()]      # results of buffer set b copied out (outputs free)
    started = [False, False]

    def one(i):
        b = i % 2
        g, o = gs[b], bufs[b]
        with torch.cuda.stream(s_in):
            if started[b]:
                s_in.wait_event(cmp_done[b])          # the step that read these inputs is done
            g["X"].copy_(host_in["X"], non_blocking=True)
            g["dY"].copy_(host_in["dY"], non_blocking=True)
            in_done[b].record(s_in)
        with torch.cuda.stream(s_cmp):
            s_cmp.wait_event(in_done[b])
            if started[b]:
                s_cmp.wait_event(out_done[b])         # these outputs have been copied out
            _step(q, lin, w, g, o, ws)
            cmp_done[b].record(s_cmp)
        with torch.cuda.stream(s_out):
            s_out.wait_event(cmp_done[b])
            for k, v in host_out.items():
                v.copy_(o[k], non_blocking=True)
            out_done[b].record(s_out)
        started[b] = True

    for i in range(2):
        one(i)
    torch.cuda.synchronize()
    _barrier(world)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    cur = torch.cuda.current_stream(device)
    t0.record(cur)
    for s in (s_in, s_cmp, s_out):
        s.wait_event(t0)
    for i in range(steps):
        one(i)
    for s in (s_in, s_cmp, s_out):
        e = ev()
        e.record(s)
        cur.wait_event(e)
    t1.record(cur)
    _barrier(world)
    ms = _max_over_ranks(t0.elapsed_time(t1), world) / steps
    h2d = sum(v.numel() * v.element_size() for v in host_in.values())
    d2h = sum(v.numel() * v.element_size() for v in host_out.values())
    return {"value": round(world * lin.fwd_bwd_flops() / (ms * 1e-3) / 1e12, 2),
            "unit": "TFLOP/s", "ms_per_step": round(ms, 4), "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h,
            "overlap": "copy-in, compute and copy-out on three streams, device buffers doubled"}


# --------------------------------------------------------------- CPU oracle
def _blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else os.cpu_count()
    except Exception:
        return os.cpu_count()


class _OracleLayer:
    """The oracle's pass over a token sample of the benchmark layer."""

    def __init__(self, sample_tokens: int):
        from bit_nf4_quantised_b200 import synthetic as syn
        from oracle import nf4_oracle as o
        self.o, self.syn = o, syn
        self.lin = syn.WORKLOADS[WORKLOAD].layers[0]
        d = syn.make_layer(self.lin)
        self.store = o.quantize(d["W"])                      # the stored weight (setup)
        m = sample_tokens
        self.X, self.A, self.B, self.dY = (syn.as_f64(d[k]) for k in ("X", "A", "B", "dY"))
        self.X, self.dY = self.X[:m], self.dY[:m]
        self.m = m
        lin = self.lin
        self.flops = 4 * m * lin.N * lin.K + 6 * m * lin.r * (lin.N + lin.K)

    def step(self):
        o, lin = self.o, self.lin
        Wt = o.dequantize(*self.store, lin.N, lin.K).astype(np.float64)
        o.linear_forward(self.X, Wt, self.A, self.B, lin.gamma)
        o.linear_backward(self.dY, self.X, Wt, self.A, self.B, lin.gamma)


def _timed_passes(layer, seconds):
    n, t = 0, 0.0
    while t < seconds or n < 2:
        t0 = time.perf_counter()
        layer.step()
        t += time.perf_counter() - t0
        n += 1
    return n, t


def _cpu_shape_rates(sample_tokens: int = 128):
    """The oracle's rate on each distinct linear shape of the MLP and decoder
    workloads (one pass over a token sample, W dequantised once), and the
    times those rates give for the whole workloads, labelled extrapolated."""
    from bit_nf4_quantised_b200 import synthetic as syn
    from oracle import nf4_oracle as o
    shapes = [("mlp.gate/up", 11008, 4096, 64, 8192, 2), ("mlp.down", 4096, 11008, 64, 8192, 1),
              ("dec.qkvo", 4096, 4096, 16, 4096, 128), ("dec.gate/up", 11008, 4096, 16, 4096, 64),
              ("dec.down", 4096, 11008, 16, 4096, 32)]
    stores = {}
    rows = []
    totals = {"mlp": 0.0, "dec": 0.0}
    for name, N, K, r, M_full, count in shapes:
        lin = syn.Linear(name, sample_tokens, N, K, r, 2.0 * r, 0.02, False, N + K)
        d = syn.make_layer(lin)
        if (N, K) not in stores:
            stores[(N, K)] = o.quantize(d["W"])
        X, A, B, dY = (syn.as_f64(d[k]) for k in ("X", "A", "B", "dY"))
        t0 = time.perf_counter()
        Wt = o.dequantize(*stores[(N, K)], N, K).astype(np.float64)
        o.linear_forward(X, Wt, A, B, lin.gamma)
        o.linear_backward(dY, X, Wt, A, B, lin.gamma)
        dt = time.perf_counter() - t0
        rate = lin.fwd_bwd_flops() / dt
        full = syn.Linear(name, M_full, N, K, r, 2.0 * r).fwd_bwd_flops() * count
        totals[name.split(".")[0]] += full / rate
        rows.append({"shape": f"{N}x{K}", "r": r, "role": name, "tokens_sampled": sample_tokens,
                     "GFLOPs": round(rate / 1e9, 2)})
    return rows, {"llama7b_mlp_m8192_r64_s": round(totals["mlp"], 1),
                  "llama7b_decoder_32layers_m4096_r16_s": round(totals["dec"], 1),
                  "label": "extrapolated: workload flops divided by the per-shape rates measured "
                           f"on {sample_tokens}-token samples"}


def _cpu_baseline(seconds: float = 10.0, sample_tokens: int = 256):
    layer = _OracleLayer(sample_tokens)
    layer.step()                                               # warm
    n, t = _timed_passes(layer, seconds)
    out = {"value": round(layer.flops * n / t / 1e12, 5), "unit": "TFLOP/s",
           "cores": _blas_threads(), "kind": "oracle",
           "sample": f"{sample_tokens} of {layer.lin.M} tokens per pass, W dequantised once "
                     f"per pass, fwd+bwd in fp64 numpy; {n} passes, {t:.1f} s"}
    try:
        from threadpoolctl import threadpool_limits
        with threadpool_limits(limits=1, user_api="blas"):
            n1, t1 = _timed_passes(layer, seconds / 3)
        out["one_thread"] = {"value": round(layer.flops * n1 / t1 / 1e12, 5), "cores": 1,
                             "sample": f"the same pass on one BLAS thread; {n1} passes, {t1:.1f} s"}
    except Exception as exc:               # an extra measurement never sinks the bench line
        out["one_thread"] = {"error": f"{type(exc).__name__}: {exc}"}
    try:
        out["per_shape"], out["extrapolated"] = _cpu_shape_rates()
    except Exception as exc:
        out["per_shape"] = {"error": f"{type(exc).__name__}: {exc}"}
    return out


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    layer = _OracleLayer(sample_tokens=128)
    for _ in range(args.warmup):
        layer.step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        layer.step()
    dt = (time.perf_counter() - t0) / args.steps
    value = layer.flops / dt / 1e12
    lin = layer.lin
    out = {
        "impl": "reference",
        "metric": "QLoRA linear fwd+bwd TFLOP/s (% bf16 peak); NF4 dequant-GEMV GB/s (% HBM)",
        "value": round(value, 5), "unit": "TFLOP/s", "n_gpus": args.gpus, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(dt * 1e3, 2), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": WORKLOAD, "M": lin.M, "N": lin.N, "K": lin.K, "r": lin.r,
                   "alpha": lin.alpha, "step": "forward (Y, T) + backward (dX, dA, dB)"},
        "cpu_baseline": {"value": round(value, 5), "unit": "TFLOP/s", "kind": "oracle",
                         "cores": _blas_threads(),
                         "sample": f"{layer.m} of {lin.M} tokens per step, W dequantised once "
                                   "per step, fp64 numpy"},
        "e2e": {"value": round(value, 5), "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(out))


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    args = ap.parse_args()
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    if args.impl == "reference":
        run_reference(args)
    else:
        run_gpu(args)


if __name__ == "__main__":
    main()
