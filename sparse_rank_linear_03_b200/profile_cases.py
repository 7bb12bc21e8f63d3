"""Named single-operation cases for profiler captures (ncu), not for timing.

    python -m sparse_rank_linear_03_b200.profile_cases --case decode70b --reps 3

Each case builds its layer once (split + pack), then repeats one operation
`reps` times with a device synchronisation at the end.  Cases:

  decode70b     2:4 apply, batch 1, 28672×8192 bf16, r = 256
  prefill70b    2:4 apply, 4096 tokens, same layer
  mlp16         2:4 apply, batch 16, 11008×4096 bf16, r = 64
  topk70b       top-k split at 5 % of the 28672×8192 bf16 W
  split24_70b   2:4 split of the same W
  attn4096      CSR apply, batch 1, 4096×4096 bf16 at 2 %, r = 128
  attn4096_t2048  the same layer with 2048 tokens (S decompressed for the dense MMA)
  factor70b     Stage 2 on the 70B layer's 2:4 residual (r = 256, k = 266, q = 2)
  stack7b       the 224-matrix CSR group at batch 1 (all 32 layers)
  stack7b_4     the first 4 layers of it (28 matrices, 178 MB: above L2, small
                enough for a full ncu capture)
"""
from __future__ import annotations

import argparse

import torch

from . import hsl, synth
from .configs import ATTN4096, MLP70B, MLP_UP_11008, STACK7B


def _bf(x):
    return synth.torch_from_storage(synth.to_bf16_bits(x), "bf16", "cuda")


def _layer(lay, r, fmt, frac, split_dtype="bf16"):
    Wf = synth.student_t_f32(lay.m, lay.n, lay.seed)
    W = _bf(Wf) if split_dtype == "bf16" else torch.from_numpy(Wf).cuda()
    L = hsl.Layer(lay.m, lay.n, r, fmt, "bf16")
    L.split(W, frac, None)
    U, V = synth.stand_in_factors(lay.m, lay.n, r, lay.seed + 2)
    L.pack(_bf(U), _bf(V))
    return L, W


def case(name: str):
    if name in ("decode70b", "prefill70b"):
        lay = MLP70B.layers[0]
        L, _ = _layer(lay, MLP70B.r, "nm24", 0.5)
        b = 1 if name == "decode70b" else 4096
        X = _bf(synth.normal_f32(b, lay.n, lay.seed + 1))
        Y = torch.empty(b, lay.m, dtype=torch.bfloat16, device="cuda")
        return lambda: L.apply(X, Y), (L,)
    if name == "mlp16":
        lay = MLP_UP_11008.layers[0]
        L, _ = _layer(lay, MLP_UP_11008.r, "nm24", 0.5)
        X = _bf(synth.normal_f32(16, lay.n, lay.seed + 1))
        Y = torch.empty(16, lay.m, dtype=torch.bfloat16, device="cuda")
        return lambda: L.apply(X, Y), (L,)
    if name in ("topk70b", "split24_70b"):
        lay = MLP70B.layers[0]
        W = _bf(synth.student_t_f32(lay.m, lay.n, lay.seed))
        R = torch.empty_like(W)
        if name == "topk70b":
            L = hsl.Layer(lay.m, lay.n, 0, "csr", "bf16")
            return lambda: L.split(W, MLP70B.topk_frac_extra, R), (L,)
        L = hsl.Layer(lay.m, lay.n, 0, "nm24", "bf16")
        return lambda: L.split(W, 0.5, R), (L,)
    if name in ("attn4096", "attn4096_t2048"):
        lay = ATTN4096.layers[0]
        L, _ = _layer(lay, ATTN4096.r, "csr", ATTN4096.frac, "f32")
        b = 1 if name == "attn4096" else 2048
        X = _bf(synth.normal_f32(b, lay.n, lay.seed + 1))
        Y = torch.empty(b, lay.m, dtype=torch.bfloat16, device="cuda")
        return lambda: L.apply(X, Y), (L,)
    if name == "factor70b":
        lay = MLP70B.layers[0]
        W = _bf(synth.student_t_f32(lay.m, lay.n, lay.seed))
        L = hsl.Layer(lay.m, lay.n, MLP70B.r, "nm24", "bf16")
        R = torch.empty_like(W)
        L.split(W, 0.5, R)
        del W
        omega = torch.randn(lay.n, MLP70B.r + 10, device="cuda")
        return lambda: L.factor(R, omega, 2), (L, R)
    if name in ("stack7b", "stack7b_4"):
        # W drawn on the device (6.5 G entries take minutes on the host)
        layers, Xs, Ys = [], [], []
        for lay in STACK7B.layers[:28 if name == "stack7b_4" else None]:
            W = synth.student_t_device(lay.m, lay.n, lay.seed, "cuda")
            L = hsl.Layer(lay.m, lay.n, STACK7B.r, "csr", "bf16")
            L.split(W, STACK7B.frac, None)
            del W
            L.pack(*synth.stand_in_factors_device(lay.m, lay.n, STACK7B.r, lay.seed + 2, "cuda"))
            layers.append(L)
            Xs.append(_bf(synth.normal_f32(1, lay.n, lay.seed + 1)))
            Ys.append(torch.empty(1, lay.m, dtype=torch.bfloat16, device="cuda"))
        g = hsl.Group(layers)
        return lambda: g.apply(Xs, Ys), (g, layers)
    raise SystemExit(f"unknown case {name}")


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--case", required=True)
    ap.add_argument("--reps", type=int, default=3)
    a = ap.parse_args()
    fn, keep = case(a.case)
    torch.cuda.synchronize()
    for _ in range(a.reps):
        fn()
    torch.cuda.synchronize()
    print(f"{a.case}: {a.reps} reps done, {hsl.launch_count()} launches")


if __name__ == "__main__":
    main()
