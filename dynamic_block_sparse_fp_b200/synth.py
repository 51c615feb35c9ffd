"""Seeded synthetic prefill inputs (Q, K, V) for the FlexPrefill hot path.

This module builds inputs only.  It holds none of the method's arithmetic
(no pooling, softmax, divergence or selection): the same tensors feed both
the CUDA path and the CPU oracle, so a mistake here cannot hide a mismatch
between the two.

The pages measure on RULER and InfiniteBench prompts run through trained
Llama-3.1-8B / GLM-4-9B weights (FlexPrefill, atlas.scime.ai summary,
"Key results" and "Experimental setup").  Neither the datasets nor the weights
exist here, so these seeded tensors stand in for them.  They copy only the
head shapes and lengths, plus two planted structures that give each head
either a query-dependent block pattern or a vertical-slash pattern:

* query-aware planting: every query block ``i`` gets its own unit vector
  ``u_i``; ``amp_qa * u_i`` is added to the queries of block ``i`` and to the
  keys of 3 key blocks drawn from ``[0, i]``;
* vertical-slash planting: one unit vector ``v`` per kv head; ``amp_vs * v`` is
  added to every query and to the sink keys 0-3 plus 8 random keys;
* configurations with GQA boost the sink keys 0-3 for every head;
* rotary embedding (rotate-half over the full head dimension) is applied to Q
  and K after planting, which gives the local (slash) diagonals.

Each kv-head group (the kv head plus its ``g`` query heads) draws from its own
generator seeded by ``(seed, kv_head)``, so any subset of groups can be
regenerated alone and bit-identically (used to time a bounded CPU sample of a
full-size workload).
"""
from __future__ import annotations

import dataclasses
import math

import torch

__all__ = ["Workload", "WORKLOADS", "make_inputs", "make_group"]


@dataclasses.dataclass(frozen=True)
class Workload:
    """One synthetic workload: shapes, method parameters and planting recipe."""

    name: str
    batch: int
    n_q_heads: int
    n_kv_heads: int
    seq_len: int
    head_dim: int
    block_size: int
    dtype: str  # "f32" or "bf16"
    gamma: float
    tau: float
    min_budget: int
    max_budget: int  # <= 0: uncapped
    rope_base: float
    p_vs: float  # probability that a kv head gets the vertical-slash planting
    seed: int
    sink_boost_all: bool  # boost sink keys 0-3 for every head
    amp_qa: float = 2.0
    amp_vs: float = 3.0
    n_random_vs_keys: int = 8
    n_planted_blocks: int = 3
    fixed_kinds: tuple | None = None  # per kv head: "qa" / "vs" (overrides p_vs)
    qa_mode: int = 0  # query-aware heads: 0 flattened map, 1 query-wise rows
    vs_mode: int = 0  # vertical-slash heads: 0 token lines, 1 block-pooled lines

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)

    @property
    def n_blocks(self) -> int:
        return -(-self.seq_len // self.block_size)  # ceil: a partial last block counts


WORKLOADS: dict[str, Workload] = {
    # Tiny CPU-checkable case: 2 heads (one of each planting), fp32, d=64.
    "tiny_n1024": Workload(
        name="tiny_n1024", batch=1, n_q_heads=2, n_kv_heads=2, seq_len=1024,
        head_dim=64, block_size=64, dtype="f32", gamma=0.95, tau=0.1,
        min_budget=256, max_budget=0, rope_base=10000.0, p_vs=0.5, seed=0,
        sink_boost_all=False, fixed_kinds=("qa", "vs")),
    # Llama-3.1-8B-shaped layer (32 q / 8 kv heads, d=128) at 8k, 32k, 128k.
    "llama8b_n8192": Workload(
        name="llama8b_n8192", batch=1, n_q_heads=32, n_kv_heads=8, seq_len=8192,
        head_dim=128, block_size=128, dtype="bf16", gamma=0.95, tau=0.1,
        min_budget=1024, max_budget=0, rope_base=500000.0, p_vs=0.5, seed=1,
        sink_boost_all=True),
    "llama8b_n32768": Workload(
        name="llama8b_n32768", batch=1, n_q_heads=32, n_kv_heads=8, seq_len=32768,
        head_dim=128, block_size=128, dtype="bf16", gamma=0.95, tau=0.1,
        min_budget=1024, max_budget=0, rope_base=500000.0, p_vs=0.5, seed=2,
        sink_boost_all=True),
    "llama8b_n131072": Workload(
        name="llama8b_n131072", batch=1, n_q_heads=32, n_kv_heads=8, seq_len=131072,
        head_dim=128, block_size=128, dtype="bf16", gamma=0.95, tau=0.1,
        min_budget=1024, max_budget=0, rope_base=500000.0, p_vs=0.5, seed=3,
        sink_boost_all=True),
    # GLM-4-9B-shaped layer (32 q / 2 kv heads), 75% vertical-slash heads.
    "glm9b_n65536_b128": Workload(
        name="glm9b_n65536_b128", batch=1, n_q_heads=32, n_kv_heads=2, seq_len=65536,
        head_dim=128, block_size=128, dtype="bf16", gamma=0.95, tau=0.1,
        min_budget=1024, max_budget=32768, rope_base=500000.0, p_vs=0.75, seed=4,
        sink_boost_all=True),
    "glm9b_n65536_b64": Workload(
        name="glm9b_n65536_b64", batch=1, n_q_heads=32, n_kv_heads=2, seq_len=65536,
        head_dim=128, block_size=64, dtype="bf16", gamma=0.95, tau=0.1,
        min_budget=1024, max_budget=32768, rope_base=500000.0, p_vs=0.75, seed=4,
        sink_boost_all=True),
}


def _unit(gen: torch.Generator, d: int) -> torch.Tensor:
    u = torch.randn(d, generator=gen, dtype=torch.float32)
    return u / u.norm()


def _rope_tables(n: int, d: int, base: float, positions_from: int = 0):
    half = d // 2
    inv = base ** (-torch.arange(0, half, dtype=torch.float64) * 2.0 / d)
    pos = torch.arange(positions_from, positions_from + n, dtype=torch.float64)
    ang = pos[:, None] * inv[None, :]
    return torch.cos(ang).float(), torch.sin(ang).float()


def _apply_rope_(x: torch.Tensor, cos: torch.Tensor, sin: torch.Tensor) -> None:
    """In-place rotate-half rotary embedding over the last dim of x [..., n, d]."""
    half = x.shape[-1] // 2
    x1 = x[..., :half].clone()
    x2 = x[..., half:]
    x[..., :half] = x1 * cos - x2 * sin
    x[..., half:] = x2 * cos + x1 * sin


def group_kind(w: Workload, b: int, kv: int) -> str:
    """Planting kind ("qa" or "vs") of kv head ``kv`` in batch item ``b``."""
    if w.fixed_kinds is not None:
        return w.fixed_kinds[kv]
    gen = torch.Generator().manual_seed(_group_seed(w, b, kv) ^ 0x5A5A)
    return "vs" if torch.rand(1, generator=gen).item() < w.p_vs else "qa"


def _group_seed(w: Workload, b: int, kv: int) -> int:
    return (w.seed * 1_000_003 + b * 10_007 + kv * 101 + 7) & 0x7FFFFFFF


def make_group(w: Workload, b: int, kv: int):
    """Q [g,N,d], K [N,d], V [N,d] (fp32, before the dtype cast) for one kv group."""
    g = w.n_q_heads // w.n_kv_heads
    n, d, bs = w.seq_len, w.head_dim, w.block_size
    nb = -(-n // bs)  # a partial last block is planted like the others
    gen = torch.Generator().manual_seed(_group_seed(w, b, kv))
    q = torch.randn(g, n, d, generator=gen, dtype=torch.float32)
    k = torch.randn(n, d, generator=gen, dtype=torch.float32)
    v = torch.randn(n, d, generator=gen, dtype=torch.float32)
    kind = group_kind(w, b, kv)
    if kind == "qa":
        for i in range(nb):
            u = _unit(gen, d)
            avail = i + 1
            m = min(w.n_planted_blocks, avail)
            blocks = torch.randperm(avail, generator=gen)[:m]
            q[:, i * bs:(i + 1) * bs, :] += w.amp_qa * u
            for j in blocks.tolist():
                k[j * bs:(j + 1) * bs, :] += w.amp_qa * u
    if kind == "vs" or w.sink_boost_all:
        vv = _unit(gen, d)
        sinks = list(range(min(4, n)))
        if kind == "vs":
            extra = (torch.randperm(max(n - 4, 0), generator=gen)[: w.n_random_vs_keys]
                     + 4).tolist()
            sinks = sinks + extra
        for t in sinks:
            k[t, :] += w.amp_vs * vv
        q += w.amp_vs * vv
    cos, sin = _rope_tables(n, d, w.rope_base)
    _apply_rope_(q, cos, sin)
    _apply_rope_(k, cos, sin)
    return q, k, v, kind


def make_inputs(w: Workload, kv_heads=None):
    """Build Q [Bt,Hq,N,d], K/V [Bt,Hkv',N,d] on the CPU.

    ``kv_heads`` (optional list) restricts the result to those kv groups; the
    q-head axis then holds their ``g`` query heads each, in order.  Returns a
    dict with torch tensors in the workload dtype (fp32 or bf16) and the
    per-kv-head planting kinds.
    """
    kvs = list(range(w.n_kv_heads)) if kv_heads is None else list(kv_heads)
    g = w.n_q_heads // w.n_kv_heads
    dt = torch.float32 if w.dtype == "f32" else torch.bfloat16
    n, d = w.seq_len, w.head_dim
    q = torch.empty(w.batch, g * len(kvs), n, d, dtype=dt)
    k = torch.empty(w.batch, len(kvs), n, d, dtype=dt)
    v = torch.empty(w.batch, len(kvs), n, d, dtype=dt)
    kinds = []
    for b in range(w.batch):
        row = []
        for a, kv in enumerate(kvs):
            qg, kg, vg, kind = make_group(w, b, kv)
            q[b, a * g:(a + 1) * g] = qg.to(dt)
            k[b, a] = kg.to(dt)
            v[b, a] = vg.to(dt)
            row.append(kind)
        kinds.append(row)
    return {"q": q, "k": k, "v": v, "kinds": kinds, "kv_heads": kvs}
