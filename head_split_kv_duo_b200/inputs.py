"""Seeded synthetic inputs, shared by the tests, the smoke run and the benchmark.

This module only draws random numbers and names workload shapes; it holds none of
the attention arithmetic.  Values are i.i.d. N(0, 1) drawn in float32 by a seeded
``torch.Generator`` and rounded to the working dtype.  Retrieval heads "chosen by
the seed" are the first k entries of ``randperm(kv_heads)`` per layer.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import torch


def generator(seed: int, device="cpu") -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def randn(shape, seed: int, dtype=torch.bfloat16, device="cpu") -> torch.Tensor:
    """i.i.d. N(0,1) in float32 from a seeded generator, rounded to `dtype`."""
    x = torch.randn(*shape, generator=generator(seed, device), dtype=torch.float32, device=device)
    return x.to(dtype)


def retrieval_mask(layers: int, kv_heads: int, n_retrieval: int, seed: int) -> torch.Tensor:
    """uint8 [layers][kv_heads]; per layer the first n_retrieval of a seeded permutation are 1."""
    g = generator(seed)
    m = torch.zeros(layers, kv_heads, dtype=torch.uint8)
    for l in range(layers):
        m[l, torch.randperm(kv_heads, generator=g)[:n_retrieval]] = 1
    return m


def fixed_mask(kv_heads: int, retrieval_heads) -> torch.Tensor:
    m = torch.zeros(1, kv_heads, dtype=torch.uint8)
    m[0, list(retrieval_heads)] = 1
    return m


@dataclass
class Workload:
    """Shapes of one synthetic workload (the pages' model shapes, random values)."""
    name: str
    layers: int
    q_heads: int
    kv_heads: int
    head_dim: int
    n_retrieval: int
    S: int
    W: int
    context: int
    batches: tuple = (1,)
    chunk: int = 0
    dtype: str = "bf16"
    retr_fmt: str = "same"
    retrieval_heads: tuple = field(default_factory=tuple)


WORKLOADS = {
    "tiny-mha": Workload("tiny-mha", 1, 8, 8, 64, 2, 4, 16, 256, (1,), chunk=256, dtype="fp32",
                         retrieval_heads=(1, 5)),
    "llama2-7b-mha-32k": Workload("llama2-7b-mha-32k", 1, 32, 32, 128, 8, 16, 512, 32768, (1, 8)),
    "llama3-8b-gqa-128k": Workload("llama3-8b-gqa-128k", 1, 32, 8, 128, 4, 16, 512, 131072, (1, 4)),
    "llama3-8b-gqa-prefill-256k": Workload("llama3-8b-gqa-prefill-256k", 1, 32, 8, 128, 4, 16, 512, 262144, (1,),
                                           chunk=32768),
    "llama3-8b-gqa-1m-int4-32l": Workload("llama3-8b-gqa-1m-int4-32l", 32, 32, 8, 128, 4, 16, 512, 1 << 20, (1,),
                                          retr_fmt="int4"),
}
