"""Seeded synthetic packed batches for packed causal attention.

This module only draws random numbers: document lengths (a packed batch is a
list of documents laid end to end, described by ``cu_seqlens``) and bf16
tensors Q, K, V, dO ~ N(0, 1).  It holds none of the attention arithmetic, so
the CPU oracle and the CUDA path can both be fed from it.

The five named workloads follow the configurations of the SAP/HSAP setting
(hybrid-context packed sequences, "Sequence-Aware Parallelism" abstract): a
tiny MHA case, and the attention shapes of Llama-3.2-1B, Llama-3.1-8B, a
512K hybrid-context batch and Llama-2-13B with many short documents.

Recipe:
  * doc lengths come from ``numpy.random.default_rng(seed)``;
  * log-uniform L = floor(exp(U(ln lo, ln hi))) clamped to [lo, hi]; docs are
    appended until their sum reaches N and the last one is truncated to fit;
  * a fixed "big" document, when the workload has one, is placed first;
  * "uniform cut points" (tiny case) draws ndocs-1 distinct cut points in
    [1, N-1] and rejects the draw until every doc has at least ``min_len``;
  * tensors are float32 N(0,1) from a seeded torch generator (CPU by default,
    or the given CUDA device for the very large cases), rounded to bf16.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import numpy as np
import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    n: int                 # packed tokens
    hq: int                # query heads
    hkv: int               # key/value heads
    d: int                 # head dim
    p: int                 # simulated sequence-parallel chunks
    backward: bool         # whether the workload runs fwd+bwd (else fwd + merge)
    docs: str              # length recipe id
    lo: int = 0
    hi: int = 0
    big: int = 0           # length of the fixed first document (0: none)
    ndocs: int = 0         # for the uniform-cut recipe
    min_len: int = 0


WORKLOADS = {
    "tiny": Workload("tiny", 1024, 4, 4, 64, 2, False, "uniform_cuts", ndocs=4, min_len=64),
    "llama32_1b_32k": Workload("llama32_1b_32k", 32768, 32, 8, 64, 8, True, "loguniform", lo=128, hi=8192),
    "llama31_8b_128k": Workload("llama31_8b_128k", 131072, 32, 8, 128, 8, True, "loguniform",
                                lo=512, hi=16384, big=65536),
    "hybrid_512k": Workload("hybrid_512k", 524288, 32, 8, 128, 16, True, "loguniform",
                            lo=1024, hi=32768, big=262144),
    "llama2_13b_64k_short": Workload("llama2_13b_64k_short", 65536, 40, 40, 128, 16, True, "uniform_int",
                                     lo=256, hi=2048),
}


def doc_lengths(w: Workload, seed: int) -> list[int]:
    """Seeded document lengths summing exactly to ``w.n``."""
    rng = np.random.default_rng(seed)
    n = w.n
    if w.docs == "uniform_cuts":
        while True:
            cuts = np.sort(rng.choice(np.arange(1, n), size=w.ndocs - 1, replace=False))
            bounds = np.concatenate([[0], cuts, [n]])
            lens = np.diff(bounds)
            if lens.min() >= w.min_len:
                return [int(x) for x in lens]
    lens: list[int] = []
    total = 0
    if w.big:
        lens.append(min(w.big, n))
        total = lens[0]
    while total < n:
        if w.docs == "loguniform":
            x = int(math.floor(math.exp(rng.uniform(math.log(w.lo), math.log(w.hi)))))
            x = max(w.lo, min(w.hi, x))
        elif w.docs == "uniform_int":
            x = int(rng.integers(w.lo, w.hi + 1))
        else:
            raise ValueError(w.docs)
        x = min(x, n - total)
        lens.append(x)
        total += x
    return lens


def cu_seqlens_from_lengths(lens) -> np.ndarray:
    cu = np.zeros(len(lens) + 1, dtype=np.int32)
    cu[1:] = np.cumsum(np.asarray(lens, dtype=np.int64))
    return cu


def randn_bf16(shape, seed: int, device: str = "cpu") -> torch.Tensor:
    g = torch.Generator(device=device).manual_seed(seed)
    return torch.randn(shape, generator=g, dtype=torch.float32, device=device).to(torch.bfloat16)


@dataclasses.dataclass
class Batch:
    workload: Workload
    seed: int
    cu_seqlens: np.ndarray      # int32 [ndocs+1], host
    q: torch.Tensor             # bf16 [N, hq, d]
    k: torch.Tensor             # bf16 [N, hkv, d]
    v: torch.Tensor             # bf16 [N, hkv, d]
    do: Optional[torch.Tensor]  # bf16 [N, hq, d] (None for forward-only workloads unless asked)


def make_batch(name_or_w, seed: int = 0, device: str = "cpu", with_do: Optional[bool] = None,
               n_override: Optional[int] = None) -> Batch:
    """Build the seeded batch of a named workload (or an explicit ``Workload``)."""
    w = WORKLOADS[name_or_w] if isinstance(name_or_w, str) else name_or_w
    if n_override is not None:
        w = dataclasses.replace(w, n=n_override)
    cu = cu_seqlens_from_lengths(doc_lengths(w, seed))
    q = randn_bf16((w.n, w.hq, w.d), seed + 1000 * 0, device)
    k = randn_bf16((w.n, w.hkv, w.d), seed + 1000 * 1, device)
    v = randn_bf16((w.n, w.hkv, w.d), seed + 1000 * 2, device)
    if with_do is None:
        with_do = w.backward
    do = randn_bf16((w.n, w.hq, w.d), seed + 1000 * 3, device) if with_do else None
    return Batch(w, seed, cu, q, k, v, do)


def custom_batch(lengths, hq: int, hkv: int, d: int, seed: int = 0, device: str = "cpu",
                 with_do: bool = True) -> Batch:
    """A batch with explicit document lengths (edge cases: ragged tails, empty docs)."""
    n = int(sum(lengths))
    w = Workload("custom", n, hq, hkv, d, 1, with_do, "explicit")
    cu = cu_seqlens_from_lengths(lengths)
    q = randn_bf16((n, hq, d), seed + 1000 * 0, device)
    k = randn_bf16((n, hkv, d), seed + 1000 * 1, device)
    v = randn_bf16((n, hkv, d), seed + 1000 * 2, device)
    do = randn_bf16((n, hq, d), seed + 1000 * 3, device) if with_do else None
    return Batch(w, seed, cu, q, k, v, do)
