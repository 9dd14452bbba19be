"""Seeded synthetic inputs for the DBSA attention engine.

This module is the only code shared by the CUDA path's tests/bench and the
CPU oracle.  It holds no arithmetic of the method: it draws demonstration
lengths, stand-in block selections (the retriever is out of scope) and
Gaussian Q/K/V tensors, with the shapes of the workloads on the paper-notes
page "Efficient Many-Shot In-Context Learning with Dynamic Block-Sparse
Attention": 50 demos per block, previous 2 blocks, 30 % retrieval
(§Configuration parameters); 30k / 90k contexts on Llama-2-7B / Llama-3.1-8B
head geometry (§Experimental setup).  The datasets themselves (TREC, NLU,
Banking-77, Clinic-150) are not used: lengths are uniform integers and the
activations are N(0, 1), cast to bf16 with round-to-nearest-even where the
workload is bf16.
"""
from __future__ import annotations

import dataclasses
from dataclasses import dataclass

import numpy as np


@dataclass(frozen=True)
class Workload:
    name: str
    index: int                      # workload number (1..5), used in seeds
    n_layers: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    dtype: str                      # "f32" or "bf16"
    rope_theta: float
    n_blocks: int
    demos_per_block: int
    demo_len_lo: int                # inclusive
    demo_len_hi: int                # inclusive
    window_j: int
    n_queries: int
    query_tokens: int               # prompt tokens of each query
    decode_steps: int               # single-token passes after the prompt pass
    retrieval_ratio: float          # fraction of blocks retrieved (plus the sink)
    n_random_blocks: int | None     # overrides the ratio when set
    order: str                      # "encoding" or "ascending" (by random score)
    n_appends: int = 0

    def n_selected_random(self) -> int:
        if self.n_random_blocks is not None:
            return min(self.n_random_blocks, self.n_blocks - 1)
        return min(int(np.floor(self.retrieval_ratio * self.n_blocks + 0.5)), self.n_blocks - 1)

    def with_(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


TINY = Workload("tiny", 1, 1, 2, 1, 64, "f32", 1e4, 8, 4, 8, 16, 2,
                1, 16, 0, 0.3, 2, "encoding")
L2_7B_30K = Workload("llama2-7b-30k", 2, 1, 32, 32, 128, "bf16", 1e4, 20, 50, 15, 45, 2,
                     1, 32, 0, 0.3, None, "encoding")
L31_8B_90K = Workload("llama3.1-8b-90k", 3, 32, 32, 8, 128, "bf16", 5e5, 60, 50, 15, 45, 2,
                      64, 40, 8, 0.3, None, "encoding")
L31_8B_APPEND = Workload("llama3.1-8b-90k-append", 4, 32, 32, 8, 128, "bf16", 5e5, 60, 50, 15, 45, 2,
                         0, 0, 0, 0.3, None, "encoding", n_appends=20)
L31_8B_128K = Workload("llama3.1-8b-128k", 5, 32, 32, 8, 128, "bf16", 5e5, 85, 50, 15, 45, 2,
                       256, 32, 0, 0.3, None, "encoding")

WORKLOADS = {w.name: w for w in (TINY, L2_7B_30K, L31_8B_90K, L31_8B_APPEND, L31_8B_128K)}


def demo_lengths(w: Workload, n_blocks: int | None = None, seed_offset: int = 0) -> np.ndarray:
    """Token length of every demonstration, uniform on [lo, hi], seeded per workload."""
    nb = w.n_blocks if n_blocks is None else n_blocks
    rng = np.random.default_rng(1000 * w.index + seed_offset)
    return rng.integers(w.demo_len_lo, w.demo_len_hi + 1, size=nb * w.demos_per_block,
                        dtype=np.int64).astype(np.int32)


def selections(w: Workload, n_blocks: int | None = None, n_queries: int | None = None,
               order: str | None = None, seed_offset: int = 0) -> list[np.ndarray]:
    """Stand-in retrieval: per query, the sink (block 0) then a seeded random
    draw (without replacement) of non-sink blocks, in encoding order or in
    ascending order of a seeded random relevance score (ties by block id)."""
    nb = w.n_blocks if n_blocks is None else n_blocks
    nq = max(w.n_queries, 1) if n_queries is None else n_queries
    order = w.order if order is None else order
    m = min(w.n_selected_random(), nb - 1)
    rng = np.random.default_rng(1000 * w.index + 7 + seed_offset)
    out = []
    for _ in range(nq):
        chosen = rng.choice(np.arange(1, nb), size=m, replace=False) if m > 0 else np.zeros(0, np.int64)
        scores = rng.random(nb)
        if order == "encoding":
            chosen = np.sort(chosen)
        elif order == "ascending":
            chosen = np.array(sorted(chosen.tolist(), key=lambda b: (scores[b], b)), dtype=np.int64)
        elif order == "reverse":
            chosen = np.sort(chosen)[::-1]
        else:
            raise ValueError(order)
        out.append(np.concatenate([[0], chosen]).astype(np.int32))
    return out


def tensor_seed(w: Workload, layer: int, role: int, step: int = 0) -> int:
    """role: 0 = Q, 1 = K, 2 = V, 3 = query/tail tokens (step = decode step)."""
    return int(w.index * 1_000_000 + layer * 1_000 + role * 100 + step)


def randn(shape, seed: int, dtype: str, device="cpu", scale: float = 1.0):
    """N(0, 1) * scale drawn in fp32 with a seeded torch generator, then cast
    (RNE) to bf16 for bf16 workloads."""
    import torch
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    x = torch.randn(tuple(shape), generator=g, device=device, dtype=torch.float32)
    if scale != 1.0:
        x = x * scale
    if dtype == "bf16":
        return x.to(torch.bfloat16)
    if dtype == "f32":
        return x
    raise ValueError(dtype)
