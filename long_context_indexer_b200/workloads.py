"""Seeded synthetic workloads for the sparse-attention index pipeline.

This module only draws random numbers and lays them out; it contains none of
the pipeline's arithmetic (no scoring, no selection, no attention, no block
compression). Both the CUDA path and the CPU oracle consume the exact bytes it
produces.

Workload shapes follow the five configurations the library is measured on
(one-layer slices of a million-token MoE model's sparse attention, as described
in "Day-0 Inference Adaptation of Ultra-Large-Scale MoE Models on Domestic AI
Accelerators", section 4.1, and "Day-0 Adaptation for Trillion-Parameter MoE
Models", section IV):

* indexer inputs (``q_c``, ``k_c`` and the per-token indexer keys ``k_idx``)
  are integers k/16 with k uniform in [-32, 32], i.e. multiples of 1/16 in
  [-2, 2]. Every product and partial sum of the block score is then a multiple
  of 2^-8 below 2^21 ulps, so fp32 accumulation is exact in any order;
* attention inputs ``q``, ``k_pool``, ``v_pool`` are N(0, 1);
* the paged KV pool holds ``B * NB`` referenced pages plus ``spare_pages``
  unreferenced pages filled with NaN, so any wrong gather poisons the output;
* the block table is a seeded random permutation of the pool's pages.

Layouts (row-major, innermost last):
  q_c    [B, S, H_i, d_c]          k_c   [B, NB, H_i, d_c]
  k_idx  [B, ctx, H_i, d_c]        (only where k_c is produced by block compression)
  q      [B, S, H_q, hd]           k_pool, v_pool [P, H_kv, bs, hd]
  block_table [B, NB] int32        ctx_len [B] int32, q_start [B] int32
"""
from __future__ import annotations

import dataclasses
from typing import Dict, Optional

import torch

__all__ = ["Config", "CONFIGS", "generate", "grid_values", "ScanConfig", "SCAN_CONFIGS",
           "generate_scan"]


@dataclasses.dataclass(frozen=True)
class Config:
    name: str
    dtype: str          # "f32" or "bf16": storage type of every floating input
    B: int              # sequences
    S: int              # queries per sequence
    ctx: int            # tokens in the cache of every sequence
    q_start: int        # absolute position of query 0 (same for every sequence)
    bs: int             # tokens per KV block (page)
    H_i: int            # indexer heads
    d_c: int            # indexer dim
    topk: int           # blocks selected per query
    H_q: int            # attention query heads
    H_kv: int           # attention KV heads
    hd: int             # attention head dim
    seed: int
    spare_pages: int = 64
    compress: bool = False   # k_c comes from block-mean compression of k_idx

    @property
    def NB(self) -> int:
        return (self.ctx + self.bs - 1) // self.bs

    @property
    def num_pages(self) -> int:
        return self.B * self.NB + self.spare_pages

    @property
    def torch_dtype(self) -> torch.dtype:
        return torch.float32 if self.dtype == "f32" else torch.bfloat16

    def replace(self, **kw) -> "Config":
        return dataclasses.replace(self, **kw)


# The five measured configurations. The 1M-token configuration is one cache
# with two query sets (a decode step and a 4096-token chunk at the end of the
# context); both use seed 4 so they share the same cache bytes.
CONFIGS: Dict[str, Config] = {
    "tiny": Config("tiny", "f32", B=1, S=256, ctx=256, q_start=0, bs=16, H_i=1, d_c=64,
                   topk=4, H_q=4, H_kv=4, hd=64, seed=0, spare_pages=4, compress=True),
    "decode": Config("decode", "bf16", B=32, S=1, ctx=32768, q_start=32767, bs=64, H_i=8,
                     d_c=128, topk=32, H_q=16, H_kv=1, hd=128, seed=1),
    "prefill": Config("prefill", "bf16", B=1, S=8192, ctx=8192, q_start=0, bs=64, H_i=8,
                      d_c=128, topk=32, H_q=16, H_kv=1, hd=128, seed=2),
    "long": Config("long", "bf16", B=8, S=1, ctx=262144, q_start=262143, bs=64, H_i=8,
                   d_c=128, topk=64, H_q=32, H_kv=2, hd=128, seed=3),
    "1m_decode": Config("1m_decode", "bf16", B=1, S=1, ctx=1048576, q_start=1048575, bs=128,
                        H_i=8, d_c=128, topk=16, H_q=16, H_kv=1, hd=128, seed=4),
    "1m_chunk": Config("1m_chunk", "bf16", B=1, S=4096, ctx=1048576, q_start=1048576 - 4096,
                       bs=128, H_i=8, d_c=128, topk=16, H_q=16, H_kv=1, hd=128, seed=4),
}


def grid_values(shape, gen: torch.Generator, dtype: torch.dtype, lo: int = -32,
                hi: int = 32, denom: float = 16.0) -> torch.Tensor:
    """Integers uniform in [lo, hi] divided by ``denom`` (exact in bf16 and fp32)."""
    k = torch.randint(lo, hi + 1, shape, generator=gen, dtype=torch.int32)
    return (k.to(torch.float32) / denom).to(dtype)


def _randn_chunked(shape, gen: torch.Generator, dtype: torch.dtype,
                   rows_per_chunk: int = 4096) -> torch.Tensor:
    """N(0,1) values drawn chunk by chunk along dim 0 (bounded fp32 temporaries)."""
    out = torch.empty(shape, dtype=dtype)
    for r0 in range(0, shape[0], rows_per_chunk):
        r1 = min(shape[0], r0 + rows_per_chunk)
        out[r0:r1] = torch.randn((r1 - r0,) + tuple(shape[1:]), generator=gen,
                                 dtype=torch.float32).to(dtype)
    return out


def generate(cfg: Config, seed: Optional[int] = None, with_kv: bool = True,
             with_indexer: bool = True) -> Dict[str, torch.Tensor]:
    """Draw one workload on the CPU. Returns contiguous CPU tensors.

    The block table, the indexer keys, the KV pool and the query side each draw
    from their own generator; the cache draws do not depend on S, so two
    configurations that share a seed and the cache shapes (the 1M decode step
    and the 1M chunk) share the cache bytes.
    """
    seed = cfg.seed if seed is None else seed
    dt = cfg.torch_dtype
    B, S, NB = cfg.B, cfg.S, cfg.NB
    P = cfg.num_pages
    out: Dict[str, torch.Tensor] = {}

    # One generator per component, so skipping a component never shifts the
    # draws of another.
    tgen = torch.Generator().manual_seed(seed * 16 + 1)
    perm = torch.randperm(P, generator=tgen).to(torch.int32)
    out["block_table"] = perm[: B * NB].reshape(B, NB).contiguous()

    if with_indexer:
        igen = torch.Generator().manual_seed(seed * 16 + 2)
        if cfg.compress:
            out["k_idx"] = grid_values((B, cfg.ctx, cfg.H_i, cfg.d_c), igen, dt)
        else:
            out["k_c"] = grid_values((B, NB, cfg.H_i, cfg.d_c), igen, dt)

    if with_kv:
        kgen = torch.Generator().manual_seed(seed * 16 + 3)
        k_pool = _randn_chunked((P, cfg.H_kv, cfg.bs, cfg.hd), kgen, dt)
        v_pool = _randn_chunked((P, cfg.H_kv, cfg.bs, cfg.hd), kgen, dt)
        spare = perm[B * NB:].long()
        if spare.numel():
            k_pool[spare] = float("nan")
            v_pool[spare] = float("nan")
        out["k_pool"] = k_pool
        out["v_pool"] = v_pool

    # Query side: a separate generator stream keyed by the query shape so that
    # the cache draw above does not depend on S.
    qgen = torch.Generator().manual_seed(seed * 1000003 + S)
    if with_indexer:
        out["q_c"] = grid_values((B, S, cfg.H_i, cfg.d_c), qgen, dt)
    out["q"] = torch.randn((B, S, cfg.H_q, cfg.hd), generator=qgen, dtype=torch.float32).to(dt)
    out["ctx_len"] = torch.full((B,), cfg.ctx, dtype=torch.int32)
    out["q_start"] = torch.full((B,), cfg.q_start, dtype=torch.int32)
    return out



# ---------------------------------------------------------------- state scan

@dataclasses.dataclass(frozen=True)
class ScanConfig:
    """A chunked gated state scan workload: B sequences of T tokens, H heads,
    dk = dv = d, chunks of C tokens."""
    name: str
    B: int
    T: int
    H: int
    d: int
    C: int
    seed: int
    gate_lo: float = 0.9     # gates uniform in [gate_lo, 1)

    @property
    def nchunks(self) -> int:
        return (self.T + self.C - 1) // self.C

    def replace(self, **kw) -> "ScanConfig":
        return dataclasses.replace(self, **kw)


# 9 sequences x 16 heads = 144 (sequence, head) scans of 16384 tokens: one per SM
SCAN_CONFIGS: Dict[str, ScanConfig] = {
    "scan": ScanConfig("scan", B=9, T=16384, H=16, d=128, C=128, seed=5),
    "scan_small": ScanConfig("scan_small", B=2, T=300, H=3, d=128, C=128, seed=6),
}


def generate_scan(cfg: ScanConfig, seed: Optional[int] = None) -> Dict[str, torch.Tensor]:
    """q, k, v ~ N(0, 1/d) in bf16 (unit-norm scale for the dot products), gates
    uniform in [gate_lo, 1) (fp32), initial state ~ N(0, 1) (fp32). CPU tensors."""
    seed = cfg.seed if seed is None else seed
    g = torch.Generator().manual_seed(seed * 7919 + 17)
    s = cfg.d ** -0.5
    shape = (cfg.B, cfg.T, cfg.H, cfg.d)
    out = {
        "q": (_randn_chunked(shape, g, torch.float32) * s).to(torch.bfloat16),
        "k": (_randn_chunked(shape, g, torch.float32) * s).to(torch.bfloat16),
        "v": _randn_chunked(shape, g, torch.bfloat16),
        "gate": cfg.gate_lo + (1 - cfg.gate_lo) * torch.rand((cfg.B, cfg.H, cfg.nchunks),
                                                             generator=g),
        "state": torch.randn((cfg.B, cfg.H, cfg.d, cfg.d), generator=g),
    }
    return out
