"""Seeded synthetic inputs shared by the tests, the bench and the CPU oracle.

This module draws random numbers and nothing else: it holds none of the
layer's arithmetic.  Every tensor is drawn in fp32 on the CPU from a seeded
``torch.Generator`` and, for the bf16 workloads, rounded to bf16
(round-to-nearest-even) before anyone sees it.  The oracle widens those
same bf16 values to fp64, which is exact, so both sides start from
identical numbers.

The five workloads follow the shapes of the pages' Megatron-style layer:
the MLP ``Z = GeLU(X@A)@B`` with ``A`` split by columns and ``B`` by rows
("图解Transformer并行计算：从矩阵乘法切分到Megatron架构设计" §2.1), a
standalone linear layer in both split modes (same page, §1.1 and §1.2),
head-wise attention with ``W_o`` split by rows (same page, §3.2), and a
layer shaped like the 175B case study (hidden 12288, 96 heads) of the
PyTorch tensor-parallel tutorial (its §5).  A sixth workload is the
vocabulary-parallel embedding and loss of the first page's §4.1-§4.2 at the
same hidden size; its token ids follow a Zipf law (frequency of the k-th
most common token proportional to 1/k), the usual shape of natural-text
token counts, with the ranks scattered over the vocabulary by a seeded
permutation so that common tokens fall in every shard.
"""
from __future__ import annotations

import dataclasses
from typing import Dict, Optional

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    """Shape and distribution recipe of one synthetic workload."""

    index: int
    name: str
    b: int
    s: int
    h: int
    f: int = 0            # MLP width (0: no MLP in this workload)
    heads: int = 0        # attention heads (0: no attention)
    t: int = 1            # logical shard count
    dtype: str = "bf16"   # "bf16" or "f32"
    w_std: float = 0.02   # weights ~ N(0, w_std^2)
    bias_std: Optional[float] = None  # None: no bias; 0.0: zero bias buffer
    n_out: int = 0        # standalone linear: output width
    vocab: int = 0        # vocabulary size V (vocabulary-parallel workload)

    @property
    def M(self) -> int:
        return self.b * self.s

    @property
    def seed(self) -> int:
        return 1234 + self.index


WORKLOADS: Dict[int, Workload] = {
    1: Workload(1, "tiny fp32 MLP", b=2, s=16, h=64, f=256, t=2, dtype="f32",
                w_std=0.02, bias_std=0.0),
    2: Workload(2, "GPT-2-small MLP", b=8, s=1024, h=768, f=3072, t=4,
                w_std=0.02, bias_std=0.01),
    3: Workload(3, "standalone linear sweep", b=1, s=8192, h=4096, n_out=16384,
                t=8, w_std=0.02),
    4: Workload(4, "head-wise attention", b=4, s=2048, h=4096, heads=32, t=8,
                w_std=0.02),
    5: Workload(5, "175B-shaped layer", b=1, s=2048, h=12288, f=49152,
                heads=96, t=8, w_std=0.006),
    6: Workload(6, "vocabulary-parallel embedding + cross-entropy", b=1, s=2048,
                h=12288, vocab=51200, t=8, w_std=0.02),
}


def _draw(gen: torch.Generator, shape, std: float, dtype: str) -> torch.Tensor:
    x = torch.randn(*shape, generator=gen, dtype=torch.float32)
    if std != 1.0:
        x.mul_(std)
    if dtype == "bf16":
        return x.to(torch.bfloat16)
    return x


def make_mlp_inputs(wl: Workload, seed: Optional[int] = None) -> Dict[str, torch.Tensor]:
    """X [M,h], A [h,f], bA [f], B [f,h], bB [h], dZ [M,h] on the CPU.

    Biases are None when the workload has none.  Order of draws is fixed:
    X, A, B, dZ, then bA, bB.
    """
    gen = torch.Generator().manual_seed(wl.seed if seed is None else seed)
    out = {
        "X": _draw(gen, (wl.M, wl.h), 1.0, wl.dtype),
        "A": _draw(gen, (wl.h, wl.f), wl.w_std, wl.dtype),
        "B": _draw(gen, (wl.f, wl.h), wl.w_std, wl.dtype),
        "dZ": _draw(gen, (wl.M, wl.h), 1.0, wl.dtype),
    }
    if wl.bias_std is None:
        out["bA"] = None
        out["bB"] = None
    else:
        out["bA"] = _draw(gen, (wl.f,), wl.bias_std, wl.dtype)
        out["bB"] = _draw(gen, (wl.h,), wl.bias_std, wl.dtype)
    return out


def make_linear_inputs(wl: Workload, seed: Optional[int] = None) -> Dict[str, torch.Tensor]:
    """X [M,K] ~ N(0,1), W [K,N] ~ N(0, w_std^2)."""
    gen = torch.Generator().manual_seed(wl.seed if seed is None else seed)
    return {
        "X": _draw(gen, (wl.M, wl.h), 1.0, wl.dtype),
        "W": _draw(gen, (wl.h, wl.n_out), wl.w_std, wl.dtype),
    }


def make_attn_inputs(wl: Workload, seed: Optional[int] = None) -> Dict[str, torch.Tensor]:
    """X [M,h], Wqkv [h,3h], Wo [h,h], dZ [M,h] on the CPU."""
    gen = torch.Generator().manual_seed((wl.seed if seed is None else seed) + 100)
    return {
        "X": _draw(gen, (wl.M, wl.h), 1.0, wl.dtype),
        "Wqkv": _draw(gen, (wl.h, 3 * wl.h), wl.w_std, wl.dtype),
        "Wo": _draw(gen, (wl.h, wl.h), wl.w_std, wl.dtype),
        "dZ": _draw(gen, (wl.M, wl.h), 1.0, wl.dtype),
    }


def zipf_ids(n: int, V: int, seed: int, exponent: float = 1.0) -> torch.Tensor:
    """n int32 token ids in [0, V): rank k (0-based) drawn with probability
    proportional to 1/(k+1)^exponent, ranks mapped to ids by a seeded
    permutation of the vocabulary."""
    gen = torch.Generator().manual_seed(seed)
    weights = torch.arange(1, V + 1, dtype=torch.float64).pow(-exponent)
    ranks = torch.multinomial(weights, n, replacement=True, generator=gen)
    perm = torch.randperm(V, generator=gen)
    return perm[ranks].to(torch.int32)


def make_vocab_inputs(wl: Workload, seed: Optional[int] = None) -> Dict[str, torch.Tensor]:
    """ids [M] int32 (Zipf), targets [M] int32 (the next token: ids shifted by
    one, the last one drawn), E [V,h] ~ N(0, w_std^2), X [M,h] ~ N(0,1) (the
    final hidden states fed to the tied output layer), dY [M,h] ~ N(0,1)."""
    s0 = (wl.seed if seed is None else seed) + 200
    stream = zipf_ids(wl.M + 1, wl.vocab, s0)
    gen = torch.Generator().manual_seed(s0 + 1)
    return {
        "ids": stream[:-1].contiguous(),
        "targets": stream[1:].contiguous(),
        "E": _draw(gen, (wl.vocab, wl.h), wl.w_std, wl.dtype),
        "X": _draw(gen, (wl.M, wl.h), 1.0, wl.dtype),
        "dY": _draw(gen, (wl.M, wl.h), 1.0, wl.dtype),
    }


def integer_tensor(shape, lo: int, hi: int, seed: int, dtype=torch.bfloat16) -> torch.Tensor:
    """Integer-valued tensor with entries uniform in [lo, hi] (exact in bf16 for |v| <= 256)."""
    gen = torch.Generator().manual_seed(seed)
    return torch.randint(lo, hi + 1, shape, generator=gen).to(dtype)


def normal_tensor(shape, std: float, seed: int, dtype: str = "bf16") -> torch.Tensor:
    """One N(0, std^2) tensor, rounded to bf16 when dtype == 'bf16'."""
    gen = torch.Generator().manual_seed(seed)
    return _draw(gen, shape, std, dtype)
