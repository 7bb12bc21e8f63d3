"""The five workloads, named by what they are.

Shapes follow the pages' LLM layers: a 1024×1024 matrix as in the worked
example of "Hierarchical Sparse + Low-Rank Compression of LLMs"
(§Two-stage compression), and Llama-7B/70B-shaped projections.
Seeds: the 1024² case uses seed 0; workload c ≥ 2 uses 1000·c + matrix index;
X uses the W seed + 1 and the stand-in factors the W seed + 2.
"""
from __future__ import annotations

from dataclasses import dataclass, field


@dataclass(frozen=True)
class Layer:
    name: str
    m: int          # output features
    n: int          # input features
    seed: int


@dataclass(frozen=True)
class Workload:
    name: str
    fmt: str                  # "csr" or "nm24"
    dtype: str                # layer dtype: "f32" or "bf16"
    split_dtype: str          # dtype the split runs on
    frac: float               # top-k fraction (0.5 for 2:4)
    r: int
    batches: tuple
    layers: tuple = field(default_factory=tuple)
    topk_frac_extra: float = 0.0   # extra unstructured split on the same W


PR1 = Workload("square1024_csr5_f32", "csr", "f32", "f32", 0.05, 64, (1,),
               (Layer("w", 1024, 1024, 0),))

ATTN4096 = Workload("attn4096_csr2_bf16", "csr", "bf16", "f32", 0.02, 128, (1, 4, 16),
                    (Layer("o_proj", 4096, 4096, 2000),))

MLP_UP_11008 = Workload("mlp_up_11008x4096_nm24_bf16", "nm24", "bf16", "bf16", 0.5, 64,
                        (1, 16, 2048), (Layer("up_proj", 11008, 4096, 3000),))

_7B_SHAPES = (("q", 4096, 4096), ("k", 4096, 4096), ("v", 4096, 4096), ("o", 4096, 4096),
              ("gate", 11008, 4096), ("up", 11008, 4096), ("down", 4096, 11008))

STACK7B = Workload("llama7b_stack_csr3_bf16", "csr", "bf16", "f32", 0.03, 128, (1,),
                   tuple(Layer(f"l{l}.{nm}", m, n, 4000 + 7 * l + i)
                         for l in range(32) for i, (nm, m, n) in enumerate(_7B_SHAPES)))

MLP70B = Workload("mlp_70b_28672x8192_nm24_bf16", "nm24", "bf16", "bf16", 0.5, 256,
                  (1, 4096), (Layer("up_proj", 28672, 8192, 5000),), topk_frac_extra=0.05)

ALL = (PR1, ATTN4096, MLP_UP_11008, STACK7B, MLP70B)
BY_NAME = {w.name: w for w in ALL}
