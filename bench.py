#!/usr/bin/env python3
"""Benchmark of the S + U Vᵀ hot path on one B200 (or N independent replicas).

One step = one pass of every hot-path stage over the 70B-MLP-shaped layer
(W 28672×8192 bf16, Student-t ν=3 ×0.02, seeded):
  1. magnitude top-k split at 5 % (CSR S + residual)        [split, unstructured]
  2. 2:4 split (values + in-group indices + residual)        [split, structured]
  3. pack of the 2:4 S and the rank-256 factors U, V         [pack]
  4. prefill apply, 4096 tokens                              [apply, large batch]
  5. decode apply, batch 1                                    [apply, batch 1]
Inputs are resident in HBM when the timed region starts; every input of a
stage (W 470 MB, S 264 MB, ...) is larger than the 126 MB L2, and stage 4
writes 235 MB just before stage 5 reads S, so stage 5 streams from DRAM.

`value` is the headline metric: streamed-weight GB/s of the batch-1 apply
(algorithmic bytes = 2:4 values + metadata + U + V + x + y, per call, over its
CUDA-event time).  The other stages are reported under "stages", with the
batch-1 apply also timed back to back (30 consecutive calls, median), as a
decode loop runs it.  `e2e` is the same metric through the C ABI with host X/Y
buffers (copies inside the timed region).  After the timed steps, "configs"
times every other workload the same way (each rate over its algorithmic bytes
or FLOPs, the fraction of the measured peak, and the float64 oracle timed on a
row sample of it beside it); those runs are outside the timed steps.
`--impl reference` times the float64 CPU oracle on a bounded row sample of
the headline workload.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import threading
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

M, N, R_RANK = 28672, 8192, 256
T_PREFILL = 4096
TOPK_FRAC = 0.05
SEED = 5000
METRIC = "S+UVᵀ apply: streamed-weight GB/s (batch 1) & TFLOP/s (prefill) vs roofline"
WORKLOAD = "mlp_70b_28672x8192_bf16_2to4_r256"


def decode_bytes(m=M, n=N, r=R_RANK, batch=1) -> int:
    vals = m * (n // 2) * 2
    meta = m * (n // 4) // 2          # 4 bits per group of four
    uv = (m + n) * r * 2
    return vals + meta + uv + batch * (n + m) * 2


def prefill_flops(m=M, n=N, r=R_RANK, t=T_PREFILL) -> int:
    return 2 * t * (m * (n // 2) + r * (m + n))


def split_topk_bytes(m=M, n=N, frac=TOPK_FRAC) -> int:
    k = int(np.floor(frac * m * n))
    return 2 * m * n * 2 + k * (4 + 2) + (m + 1) * 4      # read W, write R, S (i32 col + bf16 val)


def split_24_bytes(m=M, n=N) -> int:
    return 2 * m * n * 2 + m * (n // 2) * 2 + m * (n // 4)  # read W, write R, values, index bytes


def peaks() -> dict:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm": d["hbm_gbs"], "bf16": d["bf16_tflops"],
                "bf16_sustained": d.get("bf16_tflops_sustained", d["bf16_tflops"]),
                "source": "measured"}
    return {"hbm": 6650.0, "bf16": 1590.0, "bf16_sustained": 1400.0, "source": "fallback"}


DECODE_PROFILE = os.path.join(ROOT, "profiles", "decode70b_batch1_2to4.md")
DECODE_SOURCE = os.path.join(ROOT, "sparse_rank_linear_03_b200", "csrc", "apply_decode.cu")


def source_digest(path: str) -> str:
    import hashlib
    return hashlib.sha256(open(path, "rb").read()).hexdigest()[:16]


def decode_traffic():
    """DRAM bytes (read + write) of one launch of the batch-1 2:4 kernel, from the
    committed ncu summary of it, or None when the kernel's source has changed
    since that capture (the summary records the source digest it was taken on)."""
    try:
        text = open(DECODE_PROFILE).read()
    except OSError:
        return None
    vals = {}
    for line in text.splitlines():
        if ":" in line and line.strip().startswith(("dram_bytes_per_launch", "source_digest")):
            k, v = line.split(":", 1)
            vals[k.strip()] = v.strip().strip("`")
    if vals.get("source_digest") != source_digest(DECODE_SOURCE):
        return None
    try:
        return int(vals["dram_bytes_per_launch"])
    except (KeyError, ValueError):
        return None

# ------------------------------------------------------------------ clocks

class ClockSampler:
    """SM clock and clock-event reasons of one GPU, read through NVML every
    ~2 ms on a thread while the timed region runs (nvidia-smi's own sampling
    is too coarse for a region of tens of milliseconds).  `nvml` is the NVML
    module (pynvml) or a stand-in with the same calls; reading only, no
    setting of the GPU is touched."""
    REASONS = (("hw_slowdown", 0x8), ("hw_thermal_slowdown", 0x40),
               ("sw_thermal_slowdown", 0x20), ("sw_power_cap", 0x4))

    def __init__(self, gpu_uuid: str, nvml=None, period_s: float = 0.002):
        self.gpu_uuid = gpu_uuid
        self.nvml = nvml
        self.period = period_s
        self.samples = []
        self.sm_max = None
        self._stop = threading.Event()
        self._thread = None

    def _read(self):
        clk = self.nvml.nvmlDeviceGetClockInfo(self.h, self.nvml.NVML_CLOCK_SM)
        rs = self.nvml.nvmlDeviceGetCurrentClocksEventReasons(self.h)
        self.samples.append((float(clk), int(rs)))

    def _loop(self):
        while not self._stop.is_set():
            try:
                self._read()
            except Exception:
                return
            self._stop.wait(self.period)

    def __enter__(self):
        try:
            if self.nvml is None:
                import pynvml
                self.nvml = pynvml
            self.nvml.nvmlInit()
            self.h = self.nvml.nvmlDeviceGetHandleByUUID(self.gpu_uuid)
            self.sm_max = float(self.nvml.nvmlDeviceGetMaxClockInfo(self.h, self.nvml.NVML_CLOCK_SM))
            self._read()  # one sample before the region starts: the thread is live
            self.samples.clear()
            self._thread = threading.Thread(target=self._loop, daemon=True)
            self._thread.start()
        except Exception:
            self._thread = None
        return self

    def __exit__(self, *exc):
        if self._thread is not None:
            self._stop.set()
            self._thread.join(timeout=5)
            try:
                self.nvml.nvmlShutdown()
            except Exception:
                pass

    def summary(self) -> dict:
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        reasons = sorted({name for _, rs in self.samples for name, bit in self.REASONS if rs & bit})
        return {"sm_mhz": statistics.median(c for c, _ in self.samples), "sm_max_mhz": self.sm_max,
                "reasons": reasons, "samples": len(self.samples)}


# ------------------------------------------------------------------ distributed plumbing

def dist_setup(ngpus: int):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    return world, rank, local


def dist_max(x: float, world: int) -> float:
    """Max over ranks (the step time every rank reports is the slowest rank's)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    dev = "cpu" if dist.get_backend() == "gloo" else "cuda"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def replica_value(per_rank_units: float, max_seconds: float, world: int) -> float:
    """Whole-job throughput of independent replicas: all ranks' units over the
    slowest rank's time (weak scaling: every rank runs the same workload)."""
    return per_rank_units * world / max_seconds


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# ------------------------------------------------------------------ CPU oracle arm

def oracle_sample(target_s: float = 12.0, rows_cap: int = M):
    """Time the float64 oracle apply (dense Ŵ rows + product) on a row sample
    of the batch-1 workload; returns (GB/s-equivalent, rows, seconds, cores)."""
    import oracle
    from sparse_rank_linear_03_b200 import synth
    cores = len(os.sched_getaffinity(0))
    rng = np.random.default_rng(SEED + 11)
    Uf, Vf = synth.stand_in_factors(M, N, R_RANK, SEED + 2)
    U64 = oracle.bits_to_f64(synth.to_bf16_bits(Uf), "bf16")
    V64 = oracle.bits_to_f64(synth.to_bf16_bits(Vf), "bf16")
    x64 = oracle.bits_to_f64(synth.to_bf16_bits(synth.normal_f32(1, N, SEED + 1)), "bf16")

    def run(nrows):
        rows = np.sort(rng.choice(M, size=nrows, replace=False))
        Wr = synth.to_bf16_bits((0.02 * np.random.default_rng(SEED).standard_t(3, size=(nrows, N)))
                                .astype(np.float32))
        t0 = time.perf_counter()
        s = oracle.split_24(Wr, "bf16")
        S = oracle.nm24_to_dense(oracle.bits_to_f64(s["val"], "bf16"), s["idx"])
        oracle.apply_rows(rows, S, U64, V64, x64)
        return time.perf_counter() - t0

    dt = run(64)
    nrows = int(min(rows_cap, max(64, 64 * target_s / max(dt, 1e-3))))
    dt = run(nrows)
    frac = nrows / M
    gb = decode_bytes() * frac / 1e9
    return gb / dt, nrows, dt, cores


# ------------------------------------------------------------------ per-workload units

def csr_apply_bytes(nnz, m, n, r, batch, eb) -> int:
    """S values + 16-bit columns + int32 row pointers + U + V + X + Y."""
    return nnz * (eb + 2) + (m + 1) * 4 + (m + n) * r * eb + batch * (m + n) * eb


def nm24_apply_bytes(m, n, r, batch, eb=2) -> int:
    """Kept values + 4-bit metadata per group + U + V + X + Y."""
    return m * (n // 2) * eb + m * (n // 4) // 2 + (m + n) * r * eb + batch * (m + n) * eb


def topk_split_bytes(m, n, k, web, veb) -> int:
    """Read W + write R + S (int32 column + value) + int32 row pointers."""
    return 2 * m * n * web + k * (4 + veb) + (m + 1) * 4


def nm24_split_bytes(m, n, web, veb) -> int:
    """Read W + write R + kept values + one index byte per group."""
    return 2 * m * n * web + m * (n // 2) * veb + m * (n // 4)


def apply_flops(nnz, m, n, r, t) -> int:
    return 2 * t * (nnz + r * (m + n))


# ------------------------------------------------------------------ per-workload CPU leg

def oracle_layer_rate(m, n, r, fmt, dtype, frac, batch, seed, target_s):
    """The float64 oracle on a row sample of one layer: its split of the sampled
    rows, dense Ŵ rows and the product with `batch` tokens.  Returns
    (rate in the layer's apply unit per second, sample text); the unit is
    algorithmic bytes for decode batches and FLOPs for prefill batches."""
    import oracle
    from sparse_rank_linear_03_b200 import synth
    rng = np.random.default_rng(seed + 11)
    Uf, Vf = synth.stand_in_factors(m, n, r, seed + 2)
    U64 = oracle.bits_to_f64(synth.as_storage(Uf, dtype), dtype)
    V64 = oracle.bits_to_f64(synth.as_storage(Vf, dtype), dtype)
    X64 = oracle.bits_to_f64(synth.as_storage(synth.normal_f32(batch, n, seed + 1), dtype), dtype)
    eb = 4 if dtype == "f32" else 2

    def run(nrows):
        rows = np.sort(rng.choice(m, size=nrows, replace=False))
        Wr = synth.as_storage(synth.student_t_f32(nrows, n, seed), dtype)
        t0 = time.perf_counter()
        if fmt == "nm24":
            sp = oracle.split_24(Wr, dtype)
            S = oracle.nm24_to_dense(oracle.bits_to_f64(sp["val"], dtype), sp["idx"])
        else:
            sp = oracle.split_topk(Wr, frac, dtype)
            S = oracle.csr_to_dense(nrows, n, sp["row_ptr"], sp["col"],
                                    oracle.bits_to_f64(sp["val"], dtype))
        oracle.apply_rows(rows, S, U64, V64, X64)
        return time.perf_counter() - t0, nrows

    dt, nr = run(min(m, 16))
    nr = int(min(m, max(16, 16 * target_s / max(dt, 1e-3))))
    dt, nr = run(nr)
    share = nr / m
    if batch > 16:
        nnz = m * (n // 2) if fmt == "nm24" else int(np.floor(frac * m * n))
        units = apply_flops(nnz, m, n, r, batch) * share
    elif fmt == "nm24":
        units = nm24_apply_bytes(m, n, r, batch, eb) * share
    else:
        units = csr_apply_bytes(int(np.floor(frac * m * n)), m, n, r, batch, eb) * share
    return units / dt, f"{nr} of {m} rows, batch {batch}: split of the rows + dense Ŵ rows + product, {dt:.2f} s"


def oracle_split_rate(m, n, fmt, dtype, frac, seed, target_s):
    """The oracle's split (full lexsort / stable group sort) on a row block of
    W; returns (algorithmic bytes of that block per second, sample text)."""
    import oracle
    from sparse_rank_linear_03_b200 import synth

    def run(nrows):
        Wr = synth.as_storage(synth.student_t_f32(nrows, n, seed), dtype)
        t0 = time.perf_counter()
        if fmt == "nm24":
            oracle.split_24(Wr, dtype)
        else:
            oracle.split_topk(Wr, frac, dtype)
        return time.perf_counter() - t0

    dt = run(min(m, 16))
    nr = int(min(m, max(16, 16 * target_s / max(dt, 1e-3))))
    dt = run(nr)
    web = 4 if dtype == "f32" else 2
    if fmt == "nm24":
        by = nm24_split_bytes(nr, n, web, web)
    else:
        by = topk_split_bytes(nr, n, int(np.floor(frac * nr * n)), web, web)
    return by / dt, f"{nr} of {m} rows, split of the block alone, {dt:.2f} s"


def oracle_factor_rate(m, n, r, k, q, seed, target_s):
    """The oracle's randomized truncated SVD (float64) on a row block of a
    Student-t matrix; returns (FLOP/s over 2·rows·n·k·(2q + 2), sample text)."""
    import oracle
    from sparse_rank_linear_03_b200 import synth
    omega = np.random.default_rng(seed + 5).standard_normal((n, k))

    def run(nrows):
        R = synth.student_t_f32(nrows, n, seed).astype(np.float64)
        t0 = time.perf_counter()
        oracle.lowrank_randomized(R, min(r, nrows), omega[:, :min(k, nrows)], power_iters=q)
        return time.perf_counter() - t0

    nr = max(k + 1, 256)
    dt = run(nr)
    nr = int(min(m, max(nr, nr * target_s / max(dt, 1e-3))))
    dt = run(nr)
    return 2.0 * nr * n * k * (2 * q + 2) / dt, f"{nr} of {m} rows, r = {r}, k = {k}, q = {q}: {dt:.2f} s"


def oracle_rho_rate(m, n, seed, target_s):
    import oracle
    from sparse_rank_linear_03_b200 import synth

    def run(nrows):
        W = synth.to_bf16_bits(synth.student_t_f32(nrows, n, seed))
        t0 = time.perf_counter()
        oracle.concentration(W, "bf16")
        return time.perf_counter() - t0

    dt = run(64)
    nr = int(min(m, max(64, 64 * target_s / max(dt, 1e-3))))
    dt = run(nr)
    return nr * n * 2 / dt, f"{nr} of {m} rows (bf16): {dt:.2f} s"


# ------------------------------------------------------------------ per-workload GPU leg

HOLD_CYCLES = 400_000  # ~0.2 ms of device spin before each timed call


def time_calls(fn, stream, reps=20, flush=None):
    """Median CUDA-event time (ms) of `reps` calls on `stream` after 3 warm-up
    calls; with `flush` (a buffer larger than L2) written before each call,
    outside its events.  A short device spin precedes the start event, so the
    host has queued the call's launches before it records: the interval holds
    the call's kernels, not the host's time to enqueue them."""
    import torch
    for _ in range(3):
        fn()
    ts = []
    for _ in range(reps):
        if flush is not None:
            flush.fill_(1)
        torch.cuda._sleep(HOLD_CYCLES)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        fn()
        b.record(stream)
        b.synchronize()
        ts.append(a.elapsed_time(b))
    return statistics.median(ts)


def _rate(units, ms, peak, unit):
    per_s = units / (ms * 1e-3)
    if unit == "GB/s":
        v = per_s / 1e9
    else:
        v = per_s / 1e12
    return {"ms": round(ms, 5), unit: round(v, 2 if unit != "GB/s" else 1),
            "frac": round(v / peak, 4)}


def measure_configs(dev, pk, oracle_seconds: float, with_oracle: bool) -> dict:
    """Every workload other than the headline one, timed after the timed steps.

    Layers below the L2 size are timed cold: a 256 MB buffer is written before
    each call (outside its events).  The 224-matrix 7B stack (1.43 GB) is timed
    back to back.  Each rate is over the algorithmic bytes (decode, split) or
    FLOPs (prefill) and the matching measured peak (HBM copy, bf16 burst)."""
    import torch
    from sparse_rank_linear_03_b200 import hsl, synth
    from sparse_rank_linear_03_b200.configs import ATTN4096, MLP_UP_11008, PR1, STACK7B

    stream = torch.cuda.current_stream()
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    out = {}

    def cpu(fn, *a):
        if not with_oracle:
            return None
        v, sample = fn(*a)
        return v, sample

    def layer(wl, lay, split_dtype=None):
        split_dtype = split_dtype or wl.split_dtype
        Wb = synth.as_storage(synth.student_t_f32(lay.m, lay.n, lay.seed), split_dtype)
        W = synth.torch_from_storage(Wb, split_dtype, dev)
        L = hsl.Layer(lay.m, lay.n, wl.r, wl.fmt, wl.dtype)
        L.split(W, wl.frac if wl.fmt == "csr" else 0.5, None)
        Uf, Vf = synth.stand_in_factors(lay.m, lay.n, wl.r, lay.seed + 2)
        L.pack(synth.torch_from_storage(synth.as_storage(Uf, wl.dtype), wl.dtype, dev),
               synth.torch_from_storage(synth.as_storage(Vf, wl.dtype), wl.dtype, dev))
        return L, W

    def xy(wl, lay, b):
        X = synth.torch_from_storage(
            synth.as_storage(synth.normal_f32(b, lay.n, lay.seed + 1), wl.dtype), wl.dtype, dev)
        Y = torch.empty(b, lay.m, dtype=hsl.TORCH_DTYPE[wl.dtype], device=dev)
        return X, Y

    def with_cpu(rec, cpu_res, unit):
        if cpu_res is not None:
            v, sample = cpu_res
            rec["cpu_oracle"] = {"value": round(v / (1e9 if unit == "GB/s" else 1e12), 6),
                                 "unit": unit, "sample": sample}
        return rec

    # the 1024² worked-example layer (f32, CSR 5 %, r = 64) and 4096² attention (CSR 2 %, r = 128)
    for wl in (PR1, ATTN4096):
        lay = wl.layers[0]
        eb = 4 if wl.dtype == "f32" else 2
        L, W = layer(wl, lay)
        recs = {}
        for b in wl.batches:
            X, Y = xy(wl, lay, b)
            ms = time_calls(lambda: L.apply(X, Y), stream, flush=flush)
            by = csr_apply_bytes(L.nnz(), lay.m, lay.n, wl.r, b, eb)
            rec = dict(_rate(by, ms, pk["hbm"], "GB/s"), bytes=by)
            recs[f"apply_b{b}"] = with_cpu(rec, cpu(oracle_layer_rate, lay.m, lay.n, wl.r, "csr",
                                                    wl.dtype, wl.frac, b, lay.seed,
                                                    oracle_seconds / 4), "GB/s")
        if wl is ATTN4096:
            # 2048 tokens: S decompressed block by block for the dense MMA
            T = 2048
            X, Y = xy(wl, lay, T)
            ms = time_calls(lambda: L.apply(X, Y), stream, flush=flush)
            dense = 2 * T * lay.m * lay.n + 2 * T * 2 * wl.r * (lay.m + lay.n)
            rec = dict(_rate(dense, ms, pk["bf16"], "TFLOP/s"), flops_executed=dense,
                       peak="bf16 burst",
                       algorithmic_TFLOP_s=round(apply_flops(L.nnz(), lay.m, lay.n, wl.r, T)
                                                 / (ms * 1e-3) / 1e12, 2))
            recs[f"apply_T{T}"] = with_cpu(rec, cpu(oracle_layer_rate, lay.m, lay.n, wl.r, "csr",
                                                    wl.dtype, wl.frac, T, lay.seed,
                                                    oracle_seconds / 4), "TFLOP/s")
        web = 4 if wl.split_dtype == "f32" else 2
        ms = time_calls(lambda: L.split(W, wl.frac, None), stream, flush=flush)
        by = topk_split_bytes(lay.m, lay.n, L.nnz(), web, eb) - lay.m * lay.n * web  # no R
        rec = dict(_rate(by, ms, pk["hbm"], "GB/s"), bytes=by, residual=False)
        recs["split_topk"] = with_cpu(rec, cpu(oracle_split_rate, lay.m, lay.n, "csr",
                                                wl.split_dtype, wl.frac, lay.seed,
                                                oracle_seconds / 4), "GB/s")
        out[wl.name] = recs
        L.close()
        del W

    # 11008×4096 up-projection, 2:4, r = 64: batch 1 and 16 (bytes), 2048 tokens (FLOPs)
    wl = MLP_UP_11008
    lay = wl.layers[0]
    L, W = layer(wl, lay)
    recs = {}
    for b in wl.batches:
        X, Y = xy(wl, lay, b)
        ms = time_calls(lambda: L.apply(X, Y), stream, flush=flush)
        if b > 16:
            fl = apply_flops(lay.m * (lay.n // 2), lay.m, lay.n, wl.r, b)
            rec = dict(_rate(fl, ms, pk["bf16"], "TFLOP/s"), flops=fl, peak="bf16 burst")
            unit = "TFLOP/s"
        else:
            by = nm24_apply_bytes(lay.m, lay.n, wl.r, b)
            rec = dict(_rate(by, ms, pk["hbm"], "GB/s"), bytes=by)
            unit = "GB/s"
        recs[f"apply_b{b}"] = with_cpu(rec, cpu(oracle_layer_rate, lay.m, lay.n, wl.r, "nm24",
                                                "bf16", 0.5, b, lay.seed,
                                                oracle_seconds / 4), unit)
    R = torch.empty_like(W)
    ms = time_calls(lambda: L.split(W, 0.5, R), stream, flush=flush)
    by = nm24_split_bytes(lay.m, lay.n, 2, 2)
    recs["split_24"] = with_cpu(dict(_rate(by, ms, pk["hbm"], "GB/s"), bytes=by),
                                cpu(oracle_split_rate, lay.m, lay.n, "nm24", "bf16", 0.5, lay.seed,
                                    oracle_seconds / 4), "GB/s")
    out[wl.name] = recs
    L.close()
    del W, R

    # the 7B stack: 224 CSR matrices (3 %, r = 128) applied as one group at batch 1.
    # W is drawn on the device (same Student-t recipe; 6.5 G entries take minutes on the host).
    wl = STACK7B
    layers, Xs, Ys, total, nnz_all = [], [], [], 0, 0
    for lay in wl.layers:
        Wd = synth.student_t_device(lay.m, lay.n, lay.seed, dev)
        L = hsl.Layer(lay.m, lay.n, wl.r, "csr", "bf16")
        L.split(Wd, wl.frac, None)
        U, V = synth.stand_in_factors_device(lay.m, lay.n, wl.r, lay.seed + 2, dev)
        L.pack(U, V)
        del Wd
        layers.append((L, U, V))
        Xs.append(torch.randn(1, lay.n, generator=torch.Generator(device=dev).manual_seed(lay.seed + 1),
                              device=dev).to(torch.bfloat16))
        Ys.append(torch.empty(1, lay.m, dtype=torch.bfloat16, device=dev))
        total += csr_apply_bytes(L.nnz(), lay.m, lay.n, wl.r, 1, 2)
        nnz_all += L.nnz()
    gate = wl.layers[4]
    recs = {}
    for bits in (16, 8):
        if bits != 16:
            for L, U, V in layers:
                L.set_index_bits(bits)
                L.pack(U, V)
        g = hsl.Group([L for L, _, _ in layers])
        ms = time_calls(lambda: g.apply(Xs, Ys), stream)
        # 8-bit columns: 1.25 index bytes per entry instead of 2
        by = total if bits == 16 else total - nnz_all * 2 + nnz_all * 5 // 4
        rec = dict(_rate(by, ms, pk["hbm"], "GB/s"), bytes=by, matrices=len(layers),
                   column_bits=bits, timing="back to back (> L2)")
        recs["group_apply_b1" if bits == 16 else "group_apply_b1_cols8"] = with_cpu(
            rec, cpu(oracle_layer_rate, gate.m, gate.n, wl.r, "csr", "bf16", wl.frac, 1, gate.seed,
                     oracle_seconds / 4) if bits == 16 else None, "GB/s")
        g.close()
    out[wl.name] = recs
    for L, _, _ in layers:
        L.close()
    del layers
    torch.cuda.synchronize()
    return out


def measure_stage2_and_permutation(W, R24, dev, pk, oracle_seconds: float, with_oracle: bool) -> dict:
    """Stage 2 (randomized truncated SVD of the 70B layer's 2:4 residual, r = 256,
    k = 266, two power iterations) and the concentration ratio and permuted copy
    of its W, each timed with CUDA events (median of 5 after 2 warm-up calls)."""
    import torch
    from sparse_rank_linear_03_b200 import hsl
    stream = torch.cuda.current_stream()
    out = {}
    k, q = R_RANK + 10, 2
    L = hsl.Layer(M, N, R_RANK, "nm24", "bf16")
    omega = torch.randn(N, k, generator=torch.Generator(device=dev).manual_seed(SEED + 7), device=dev)
    ms = time_calls(lambda: L.factor(R24, omega, q), stream, reps=5)
    fl = 2.0 * M * N * k * (2 * q + 2)
    rec = dict(_rate(fl, ms, pk["bf16"], "TFLOP/s"), flops=fl, peak="bf16 burst",
               note="algorithmic FLOPs of the 2q+2 tall products; each runs as three bf16 "
                    "products (fp32-accurate), plus Gram matrices and Jacobi eigensolves")
    if with_oracle:
        v, sample = oracle_factor_rate(M, N, R_RANK, k, q, SEED, oracle_seconds)
        rec["cpu_oracle"] = {"value": round(v / 1e12, 6), "unit": "TFLOP/s", "sample": sample}
    out["factor_r256_k266_q2"] = rec
    L.close()
    ms = time_calls(lambda: hsl.concentration(W), stream, reps=5)
    by = M * N * 2
    rec = dict(_rate(by, ms, pk["hbm"], "GB/s"), bytes=by,
               note="includes the result's device-to-host copy and stream synchronisation")
    if with_oracle:
        v, sample = oracle_rho_rate(M, N, SEED, oracle_seconds / 2)
        rec["cpu_oracle"] = {"value": round(v / 1e9, 6), "unit": "GB/s", "sample": sample}
    out["concentration"] = rec
    g = torch.Generator(device=dev).manual_seed(SEED + 8)
    ro = torch.randperm(M, generator=g, device=dev).to(torch.int32)
    co = torch.randperm(N, generator=g, device=dev).to(torch.int32)
    dst = torch.empty_like(W)
    ms = time_calls(lambda: hsl.permute(W, ro, co, dst), stream, reps=5)
    by = 2 * M * N * 2
    out["permute"] = dict(_rate(by, ms, pk["hbm"], "GB/s"), bytes=by,
                          note="includes the host-side check of both orders")
    return out


# ------------------------------------------------------------------ GPU arm

def b2b_decode(layer, x, y, stream, calls: int) -> float:
    """Median of `calls` consecutive batch-1 applies, each bracketed by CUDA
    events on the launching stream (the weights exceed L2, so every call
    streams them from DRAM)."""
    import torch
    for _ in range(3):
        layer.apply(x, y)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(calls + 1)]
    torch.cuda.synchronize()
    ev[0].record(stream)
    for i in range(calls):
        layer.apply(x, y)
        ev[i + 1].record(stream)
    torch.cuda.synchronize()
    return statistics.median(ev[i].elapsed_time(ev[i + 1]) for i in range(calls))


def run_gpu(args, world, rank, local):
    import torch
    from sparse_rank_linear_03_b200 import hsl, synth

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream()
    pk = peaks()

    # inputs (host-generated once, resident in HBM before timing)
    W = synth.torch_from_storage(synth.to_bf16_bits(synth.student_t_f32(M, N, SEED)), "bf16", dev)
    Uf, Vf = synth.stand_in_factors(M, N, R_RANK, SEED + 2)
    U = synth.torch_from_storage(synth.to_bf16_bits(Uf), "bf16", dev)
    V = synth.torch_from_storage(synth.to_bf16_bits(Vf), "bf16", dev)
    x1 = synth.torch_from_storage(synth.to_bf16_bits(synth.normal_f32(1, N, SEED + 1)), "bf16", dev)
    Xp = torch.randn(T_PREFILL, N, generator=torch.Generator().manual_seed(SEED + 3)).to(
        torch.bfloat16).to(dev)
    y1 = torch.empty(1, M, dtype=torch.bfloat16, device=dev)
    Yp = torch.empty(T_PREFILL, M, dtype=torch.bfloat16, device=dev)
    R_csr = torch.empty_like(W)
    R_24 = torch.empty_like(W)
    csr = hsl.Layer(M, N, 0, "csr", "bf16")
    nm = hsl.Layer(M, N, R_RANK, "nm24", "bf16")

    stages = ["split_topk", "split_24", "pack", "apply_prefill", "apply_decode"]

    def step(ev=None):
        if ev:
            ev[0].record(stream)
        csr.split(W, TOPK_FRAC, R_csr)
        if ev:
            ev[1].record(stream)
        nm.split(W, 0.5, R_24)
        if ev:
            ev[2].record(stream)
        nm.pack(U, V)
        if ev:
            ev[3].record(stream)
        nm.apply(Xp, Yp)
        if ev:
            ev[4].record(stream)
        nm.apply(x1, y1)
        if ev:
            ev[5].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    csr.check()
    nm.check()

    events = [[torch.cuda.Event(enable_timing=True) for _ in range(6)] for _ in range(args.steps)]
    gpu_id = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    barrier(world)
    torch.cuda.synchronize()
    launches0 = hsl.launch_count()
    with ClockSampler(gpu_id) as clk:
        t_start = torch.cuda.Event(enable_timing=True)
        t_stop = torch.cuda.Event(enable_timing=True)
        t_start.record(stream)
        for k in range(args.steps):
            step(events[k])
        t_stop.record(stream)
        torch.cuda.synchronize()
    barrier(world)
    launches = hsl.launch_count() - launches0
    total_ms = dist_max(t_start.elapsed_time(t_stop), world)
    per = {s: [] for s in stages}
    for ev in events:
        for i, s in enumerate(stages):
            per[s].append(ev[i].elapsed_time(ev[i + 1]))
    avg = {s: dist_max(sum(v) / len(v), world) for s, v in per.items()}

    # the batch-1 apply back to back, as a decode loop runs it (the in-step call
    # above follows the prefill; here each call follows the previous one)
    b2b_ms = b2b_decode(nm, x1, y1, stream, 30)
    b2b_ms = dist_max(b2b_ms, world)

    dec_bytes = decode_bytes()
    dec_gbs = dec_bytes / (avg["apply_decode"] * 1e-3) / 1e9
    b2b_gbs = dec_bytes / (b2b_ms * 1e-3) / 1e9
    pre_tf = prefill_flops() / (avg["apply_prefill"] * 1e-3) / 1e12
    split_gbs = split_topk_bytes() / (avg["split_topk"] * 1e-3) / 1e9
    s24_gbs = split_24_bytes() / (avg["split_24"] * 1e-3) / 1e9

    # end to end through the C ABI with host buffers (pinned)
    xh = x1.cpu().pin_memory()
    yh = torch.empty(1, M, dtype=torch.bfloat16).pin_memory()
    for _ in range(3):
        nm.apply(xh, yh)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    reps = 20
    e0.record(stream)
    for _ in range(reps):
        nm.apply(xh, yh)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = dist_max(e0.elapsed_time(e1) / reps, world)
    e2e_gbs = dec_bytes / (e2e_ms * 1e-3) / 1e9 * world

    clocks = clk.summary()
    result = {
        "metric": METRIC,
        "value": round(dec_gbs * world, 1),
        "unit": "GB/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(total_ms / args.steps, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (seeded Student-t nu=3 W, N(0,1) X, Gaussian stand-in U/V)",
        "config": {"workload": WORKLOAD, "m": M, "n": N, "r": R_RANK, "decode_batch": 1,
                   "prefill_tokens": T_PREFILL, "topk_frac": TOPK_FRAC,
                   "parallelism": f"replicas{world}",
                   "l2": "inputs larger than L2 (W 470 MB, S 264 MB); prefill writes 235 MB "
                         "before the decode apply"},
        "stages": {
            "split_topk": {"ms": round(avg["split_topk"], 4), "GB/s": round(split_gbs, 1),
                           "frac_hbm": round(split_gbs / pk["hbm"], 3)},
            "split_24": {"ms": round(avg["split_24"], 4), "GB/s": round(s24_gbs, 1),
                         "frac_hbm": round(s24_gbs / pk["hbm"], 3)},
            "pack": {"ms": round(avg["pack"], 4)},
            # a ~1.7 ms kernel in a ~2.6 ms step: the burst bf16 peak applies
            "apply_prefill": {"ms": round(avg["apply_prefill"], 4), "TFLOP/s": round(pre_tf, 2),
                              "frac_tensor": round(pre_tf / pk["bf16"], 4),
                              "peak": "bf16 burst"},
            "apply_decode": {"ms": round(avg["apply_decode"], 4), "GB/s": round(dec_gbs, 1),
                             "frac_hbm": round(dec_gbs / pk["hbm"], 3)},
            "apply_decode_back_to_back": {"ms_median": round(b2b_ms, 4), "calls": 30,
                                          "GB/s": round(b2b_gbs, 1),
                                          "frac_hbm": round(b2b_gbs / pk["hbm"], 3)},
        },
        "roofline": {"bound": "hbm", "achieved": round(dec_gbs, 1), "peak": pk["hbm"],
                     "unit": "GB/s", "frac": round(dec_gbs / pk["hbm"], 4),
                     "traffic": decode_traffic(),
                     "kernel": "batch-1 2:4 apply (z, S stream and U·z in one kernel)",
                     "peak_source": pk["source"]},
        "e2e": {"value": round(e2e_gbs, 1), "unit": "GB/s", "h2d_bytes_per_step": N * 2,
                "d2h_bytes_per_step": M * 2},
        "gpu_launches": int(launches),
        "clocks": {"sm_mhz": clocks["sm_mhz"], "sm_max_mhz": clocks["sm_max_mhz"],
                   "reasons": clocks["reasons"]},
    }
    if world == 1 and not args.no_configs:
        result["stage2_and_permutation"] = measure_stage2_and_permutation(
            W, R_24, dev, pk, args.cpu_seconds / 2, not args.no_cpu_baseline)
        del W, R_csr, R_24, Xp, Yp
        csr.close()
        nm.close()
        torch.cuda.empty_cache()
        result["configs"] = measure_configs(dev, pk, oracle_seconds=args.cpu_seconds / 2,
                                            with_oracle=not args.no_cpu_baseline)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        gbs, rows, dt, cores = oracle_sample(args.cpu_seconds)
        result["cpu_baseline"] = {"value": round(gbs, 4), "unit": "GB/s", "cores": cores,
                                  "kind": "oracle",
                                  "sample": f"{rows} of {M} rows, batch 1: float64 2:4 split of "
                                            f"the rows + dense Ŵ rows + product, {dt:.1f} s"}
    return result


def run_reference(args, world, rank):
    if rank != 0:
        return None
    vals = []
    for _ in range(args.warmup):
        oracle_sample(args.cpu_seconds / 4, rows_cap=256)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        gbs, rows, dt, cores = oracle_sample(args.cpu_seconds, rows_cap=M)
        vals.append(gbs)
    wall = time.perf_counter() - t0
    v = statistics.mean(vals)
    return {"metric": METRIC, "value": round(v, 4), "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(wall / args.steps * 1e3, 1), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "impl": "reference",
            "config": {"workload": WORKLOAD, "m": M, "n": N, "r": R_RANK, "decode_batch": 1},
            "cpu_baseline": {"value": round(v, 4), "unit": "GB/s", "cores": cores, "kind": "oracle",
                             "sample": f"{rows} of {M} rows per step (float64 CPU oracle)"},
            "e2e": {"value": round(v, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="hsl", choices=["hsl", "reference"])
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-configs", action="store_true",
                    help="skip the per-workload measurements after the timed steps")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        world = int(os.environ.get("WORLD_SIZE", "1"))
        rank = int(os.environ.get("RANK", "0"))
        res = run_reference(args, world, rank)
        if res is not None:
            print(json.dumps(res, ensure_ascii=False))
        return
    world, rank, local = dist_setup(args.gpus)
    res = run_gpu(args, world, rank, local)
    if rank == 0:
        print(json.dumps(res, ensure_ascii=False))
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
