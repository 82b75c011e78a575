"""Seeded synthetic inputs for the indexed sparse-attention decode and prefill paths.

This module is shared by the CPU oracle's tests and by the CUDA path's tests and
benchmark. It holds the workload shapes and the random-number recipe only: it
performs none of the method's arithmetic (no group means, scores, selection,
centroids or attention). Every tensor is produced on the host with a seeded
``torch.Generator`` so that both sides see identical bits.

Recipe (shapes from the pages' workloads; values synthetic):
  * projected-key cache ``kt`` and scoring queries ``qt``: integers drawn
    uniformly from [-R, R] (R = 8, or 4 for the 1M-token hierarchical case),
    stored as bf16 (exact), so that fp32 scores are exact;
  * queries ``q`` and the K/V cache: N(0, 1), rounded to bf16;
  * "heavy hitters" (128K decode case): a seeded 1% of the positions of every
    (sequence, KV head) get both their K row and their ``kt`` row multiplied by
    4 (exact in bf16, since 4 is a power of two and |4 * kt| <= 32).

The KV budget B = 1.5625% of T at 32K follows the RULER budget of Joint Subspace
Sparse Attention for Efficient Long-Context Decoding, Fig. 3; the 128K / B=2048
setting follows its Fig. 4 and Fig. 6; the 32-query-head, 8-KV-head, d=128
shape is LLaMA-3.1-8B's (its Fig. 2 and Fig. 6 model).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field, replace

import torch

__all__ = ["Workload", "WORKLOADS", "make_decode_inputs", "make_prefill_inputs", "make_query_sets", "workload"]


@dataclass(frozen=True)
class Workload:
    """One synthetic workload (sizes, budget and value ranges)."""

    name: str
    seed: int
    batch: int
    hq: int
    hkv: int
    d: int
    T: int
    r: int
    B: int
    int_range: int = 8          # kt / qt integers uniform in [-int_range, int_range]
    heavy_frac: float = 0.0     # fraction of positions per (sequence, KV head) scaled x4
    heavy_scale: float = 4.0
    blk: int = 0                # hierarchical mode: tokens per block (0 = flat)
    keep: int = 0               # hierarchical mode: blocks kept
    nq: int = 0                 # prefill: number of query tokens (at positions T-nq .. T-1)
    extra: dict = field(default_factory=dict)

    @property
    def G(self) -> int:
        return self.hq // self.hkv

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    @property
    def n_heavy(self) -> int:
        return int(round(self.heavy_frac * self.T))

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


WORKLOADS: dict[str, Workload] = {
    # tiny decode step: one KV head, group of 4
    "tiny_4k": Workload("tiny_4k", 1001, batch=1, hq=4, hkv=1, d=128, T=4096, r=64, B=256),
    # LLaMA-3.1-8B-shaped decode layer at 32K, B = 1.5625% of T
    "llama8b_32k": Workload("llama8b_32k", 1002, batch=1, hq=32, hkv=8, d=128, T=32768, r=64, B=512),
    # 128K decode, batch 4, B = 2048, 1% heavy-hitter positions per (sequence, KV head)
    "decode_128k": Workload("decode_128k", 1003, batch=4, hq=32, hkv=8, d=128, T=131072, r=64,
                            B=2048, heavy_frac=0.01),
    # coarse-to-fine decode at 1M tokens: 64-token blocks, keep 64 blocks, then B = 2048
    "hier_1m": Workload("hier_1m", 1004, batch=1, hq=32, hkv=8, d=128, T=1048576, r=64, B=2048,
                        int_range=4, blk=64, keep=64),
    # prefill indexer + indexed attention: 4096 queries at positions T-4096 .. T-1
    "prefill_128k": Workload("prefill_128k", 1005, batch=1, hq=32, hkv=8, d=128, T=131072, r=64,
                             B=2048, nq=4096),
}


def workload(name: str) -> Workload:
    return WORKLOADS[name]


_CHUNK = 1 << 24  # elements per generation chunk (bounds the fp32 temporaries)


def _normal_bf16(shape, gen: torch.Generator) -> torch.Tensor:
    out = torch.empty(shape, dtype=torch.bfloat16)
    flat = out.view(-1)
    n = flat.numel()
    for s in range(0, n, _CHUNK):
        e = min(n, s + _CHUNK)
        flat[s:e] = torch.randn(e - s, generator=gen, dtype=torch.float32).to(torch.bfloat16)
    return out


def _int_bf16(shape, R: int, gen: torch.Generator) -> torch.Tensor:
    out = torch.empty(shape, dtype=torch.bfloat16)
    flat = out.view(-1)
    n = flat.numel()
    for s in range(0, n, _CHUNK):
        e = min(n, s + _CHUNK)
        flat[s:e] = torch.randint(-R, R + 1, (e - s,), generator=gen, dtype=torch.int32).to(torch.bfloat16)
    return out


def heavy_positions(w: Workload, gen: torch.Generator) -> torch.Tensor:
    """[batch, hkv, n_heavy] int64 positions, drawn without replacement per (b, h)."""
    n = w.n_heavy
    pos = torch.empty((w.batch, w.hkv, n), dtype=torch.int64)
    for b in range(w.batch):
        for h in range(w.hkv):
            pos[b, h] = torch.randperm(w.T, generator=gen)[:n]
    return pos


def make_decode_inputs(w: Workload, seed: int | None = None) -> dict[str, torch.Tensor]:
    """Host (CPU) bf16 tensors for one decode step.

    Returns q [batch, hq, d], qt [batch, hq, r], k / v [batch, T, hkv, d] and
    kt [batch, T, hkv, r], plus ``heavy`` ([batch, hkv, n] positions, possibly
    empty). The order of draws is fixed: qt, kt, q, k, v, heavy positions.
    """
    gen = torch.Generator().manual_seed(w.seed if seed is None else seed)
    qt = _int_bf16((w.batch, w.hq, w.r), w.int_range, gen)
    kt = _int_bf16((w.batch, w.T, w.hkv, w.r), w.int_range, gen)
    q = _normal_bf16((w.batch, w.hq, w.d), gen)
    k = _normal_bf16((w.batch, w.T, w.hkv, w.d), gen)
    v = _normal_bf16((w.batch, w.T, w.hkv, w.d), gen)
    heavy = heavy_positions(w, gen) if w.n_heavy > 0 else torch.empty((w.batch, w.hkv, 0), dtype=torch.int64)
    if heavy.numel():
        s = float(w.heavy_scale)
        for b in range(w.batch):
            for h in range(w.hkv):
                p = heavy[b, h]
                k[b, p, h, :] = (k[b, p, h, :].float() * s).to(torch.bfloat16)
                kt[b, p, h, :] = (kt[b, p, h, :].float() * s).to(torch.bfloat16)
    return {"q": q, "qt": qt, "k": k, "v": v, "kt": kt, "heavy": heavy}


def make_query_sets(w: Workload, count: int, seed: int) -> dict[str, torch.Tensor]:
    """`count` further decode queries for the same caches: q [count, batch, hq, d]
    (N(0, 1) as bf16) and qt [count, batch, hq, r] (integers in [-R, R] as bf16),
    set i drawn from seed + i in the order qt, q. Successive decode steps of a
    benchmark use different sets, so that each step selects its own K/V rows
    instead of re-reading the previous step's rows from L2."""
    q = torch.empty((count, w.batch, w.hq, w.d), dtype=torch.bfloat16)
    qt = torch.empty((count, w.batch, w.hq, w.r), dtype=torch.bfloat16)
    for i in range(count):
        gen = torch.Generator().manual_seed(seed + i)
        qt[i] = _int_bf16((w.batch, w.hq, w.r), w.int_range, gen)
        q[i] = _normal_bf16((w.batch, w.hq, w.d), gen)
    return {"q": q, "qt": qt}


def make_prefill_inputs(w: Workload, seed: int | None = None) -> dict[str, torch.Tensor]:
    """Host bf16 tensors for the prefill indexer + indexed attention.

    q [nq, hq, d] and qt [nq, hq, r] are the queries at absolute positions
    T-nq .. T-1; k / v [T, hkv, d] and kt [T, hkv, r] hold the whole cache
    (the queries' own keys included). Draw order: qt, kt, q, k, v.
    """
    assert w.batch == 1 and w.nq > 0
    gen = torch.Generator().manual_seed(w.seed if seed is None else seed)
    qt = _int_bf16((w.nq, w.hq, w.r), w.int_range, gen)
    kt = _int_bf16((w.T, w.hkv, w.r), w.int_range, gen)
    q = _normal_bf16((w.nq, w.hq, w.d), gen)
    k = _normal_bf16((w.T, w.hkv, w.d), gen)
    v = _normal_bf16((w.T, w.hkv, w.d), gen)
    return {"q": q, "qt": qt, "k": k, "v": v, "kt": kt, "q_start": w.T - w.nq}


def make_projection_inputs(seed: int, batch: int, T: int, H: int, d: int, r: int, nbases: int,
                           x_range: int | None = 3, p_range: int | None = 2) -> dict[str, torch.Tensor]:
    """Host bf16 tensors for scoring preparation: rows x [batch, T, H, d] and
    bases P [nbases, r, d]. Integer-valued when a range is given (uniform in
    [-R, R]), else x ~ N(0, 1) and P ~ N(0, 1) / sqrt(d) (an approximately
    orthonormal random basis). Draw order: x, P."""
    gen = torch.Generator().manual_seed(seed)
    x = _int_bf16((batch, T, H, d), x_range, gen) if x_range is not None else _normal_bf16((batch, T, H, d), gen)
    if p_range is not None:
        P = _int_bf16((nbases, r, d), p_range, gen)
    else:
        P = (_normal_bf16((nbases, r, d), gen).to(torch.float32) / math.sqrt(d)).to(torch.bfloat16)
    return {"x": x, "P": P}
