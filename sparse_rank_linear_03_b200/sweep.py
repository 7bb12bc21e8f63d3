"""Timed sweep of every workload: splits and applies, one line of JSON each.

    python -m sparse_rank_linear_03_b200.sweep [--only NAME ...] [--reps 20]

Times come from CUDA events on the launching stream around `reps` back-to-back
calls, after 3 warm-up calls; every call's operands exceed the 126 MB L2 or,
for the small layers, a 256 MB buffer is written between calls to flush L2
(the flush is outside the timed interval: each call is timed by its own pair
of events, and the median is reported).  Rates use algorithmic bytes / FLOPs:

  decode apply  bytes = S values + indices (16-bit CSR columns, 4-bit 2:4
                metadata) + row_ptr + U + V + X + Y
  prefill apply FLOPs = 2·T·(nnz + r·(m+n))
  split         bytes = read W + write residual + S (int32 col + value)

Peaks: MEASURED_PEAKS.json next to the repository root when present.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics

import numpy as np
import torch

from . import hsl, synth
from .configs import ATTN4096, MLP70B, MLP_UP_11008, PR1, STACK7B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d["hbm_gbs"], d["bf16_tflops"]
    return 6650.0, 1590.0


HBM, TC = _peaks()
_flush = None


def flush_l2():
    global _flush
    if _flush is None:
        _flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    _flush.fill_(1)


def timed(fn, reps, flush):
    for _ in range(3):
        fn()
    ts = []
    for _ in range(reps):
        if flush:
            flush_l2()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        fn()
        b.record()
        b.synchronize()
        ts.append(a.elapsed_time(b))
    return statistics.median(ts)


def _dev(bits, dt):
    return synth.torch_from_storage(bits, dt, "cuda")


def csr_bytes(nnz, m, n, r, batch, eb):
    return nnz * (eb + 2) + (m + 1) * 4 + (m + n) * r * eb + batch * (m + n) * eb


def nm24_bytes(m, n, r, batch, eb=2):
    return m * (n // 2) * eb + m * (n // 4) // 2 + (m + n) * r * eb + batch * (m + n) * eb


def layer(lay, r, fmt, dtype, split_dtype, frac):
    Wf = synth.student_t_f32(lay.m, lay.n, lay.seed)
    W = _dev(synth.as_storage(Wf, split_dtype), split_dtype)
    L = hsl.Layer(lay.m, lay.n, r, fmt, dtype)
    L.split(W, frac, None)
    U, V = synth.stand_in_factors(lay.m, lay.n, r, lay.seed + 2)
    L.pack(_dev(synth.as_storage(U, dtype), dtype), _dev(synth.as_storage(V, dtype), dtype))
    return L, W


def emit(rec):
    print(json.dumps(rec), flush=True)


def run_single(wl, reps):
    lay = wl.layers[0]
    eb = 4 if wl.dtype == "f32" else 2
    L, W = layer(lay, wl.r, wl.fmt, wl.dtype, wl.split_dtype, wl.frac)
    small = lay.m * lay.n * eb < (256 << 20)
    for b in wl.batches:
        X = _dev(synth.as_storage(synth.normal_f32(b, lay.n, lay.seed + 1), wl.dtype), wl.dtype)
        Y = torch.empty(b, lay.m, dtype=hsl.TORCH_DTYPE[wl.dtype], device="cuda")
        ms = timed(lambda: L.apply(X, Y), reps, small)
        if b >= 64 and wl.fmt == "nm24":
            fl = 2 * b * (lay.m * (lay.n // 2) + wl.r * (lay.m + lay.n))
            emit({"workload": wl.name, "op": "apply", "batch": b, "ms": ms,
                  "TFLOP/s": fl / ms / 1e9, "frac_tensor": fl / ms / 1e9 / TC})
        else:
            by = (csr_bytes(L.nnz(), lay.m, lay.n, wl.r, b, eb) if wl.fmt == "csr"
                  else nm24_bytes(lay.m, lay.n, wl.r, b, eb))
            emit({"workload": wl.name, "op": "apply", "batch": b, "ms": ms, "bytes": by,
                  "GB/s": by / ms / 1e6, "frac_hbm": by / ms / 1e6 / HBM,
                  "l2_flushed": small})
    # split
    web = 4 if wl.split_dtype == "f32" else 2
    R = torch.empty_like(W)
    frac = wl.frac if wl.fmt == "csr" else 0.5
    ms = timed(lambda: L.split(W, frac, R), reps, small)
    k = L.nnz()
    by = 2 * lay.m * lay.n * web + k * (4 + eb) if wl.fmt == "csr" else \
        2 * lay.m * lay.n * web + k * eb + lay.m * lay.n // 4
    emit({"workload": wl.name, "op": "split", "ms": ms, "bytes": by, "GB/s": by / ms / 1e6,
          "frac_hbm": by / ms / 1e6 / HBM})
    if wl.topk_frac_extra:
        C = hsl.Layer(lay.m, lay.n, 0, "csr", wl.dtype)
        ms = timed(lambda: C.split(W, wl.topk_frac_extra, R), reps, small)
        k = C.nnz()
        by = 2 * lay.m * lay.n * web + k * (4 + eb) + (lay.m + 1) * 4
        emit({"workload": wl.name, "op": "split_topk", "frac": wl.topk_frac_extra, "ms": ms,
              "bytes": by, "GB/s": by / ms / 1e6, "frac_hbm": by / ms / 1e6 / HBM})


def run_stack(reps):
    wl = STACK7B
    layers, Xs, Ys, total = [], [], [], 0
    for lay in wl.layers:
        L, W = layer(lay, wl.r, "csr", "bf16", "f32", wl.frac)
        del W
        layers.append(L)
        Xs.append(_dev(synth.to_bf16_bits(synth.normal_f32(1, lay.n, lay.seed + 1)), "bf16"))
        Ys.append(torch.empty(1, lay.m, dtype=torch.bfloat16, device="cuda"))
        total += csr_bytes(L.nnz(), lay.m, lay.n, wl.r, 1, 2)
    g = hsl.Group(layers)
    ms = timed(lambda: g.apply(Xs, Ys), reps, False)
    emit({"workload": wl.name, "op": "group_apply", "batch": 1, "matrices": len(layers),
          "ms": ms, "bytes": total, "GB/s": total / ms / 1e6, "frac_hbm": total / ms / 1e6 / HBM})


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--only", nargs="*", default=None)
    ap.add_argument("--reps", type=int, default=20)
    a = ap.parse_args()
    todo = a.only or [w.name for w in (PR1, ATTN4096, MLP_UP_11008, MLP70B, STACK7B)]
    for w in (PR1, ATTN4096, MLP_UP_11008, MLP70B):
        if w.name in todo:
            run_single(w, a.reps)
    if STACK7B.name in todo:
        run_stack(a.reps)


if __name__ == "__main__":
    main()
