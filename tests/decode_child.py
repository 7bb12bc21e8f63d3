"""Child process of test_decode_b1_gpu: applies one seeded batch-1 bf16 2:4
layer and writes the raw output bits, so that a parent can compare the
kernels selected by different environments bit for bit."""
import sys

import numpy as np


def main(out_path: str, m: int, n: int, r: int, seed: int) -> None:
    import torch

    from sparse_rank_linear_03_b200 import hsl, synth

    W = synth.to_bf16_bits(synth.student_t_f32(m, n, seed))
    Uf, Vf = synth.stand_in_factors(m, n, r, seed + 2)
    L = hsl.Layer(m, n, r, "nm24", "bf16")
    L.split(synth.torch_from_storage(W, "bf16", "cuda"), 0.5, None)
    L.pack(synth.torch_from_storage(synth.to_bf16_bits(Uf), "bf16", "cuda"),
           synth.torch_from_storage(synth.to_bf16_bits(Vf), "bf16", "cuda"))
    X = synth.torch_from_storage(synth.to_bf16_bits(synth.normal_f32(1, n, seed + 1)), "bf16",
                                 "cuda")
    Y = L.apply(X)
    L.check()
    torch.cuda.synchronize()
    np.save(out_path, synth.storage_from_torch(Y))


if __name__ == "__main__":
    main(sys.argv[1], *(int(a) for a in sys.argv[2:6]))
