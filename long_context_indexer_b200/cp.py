"""Context parallelism: one long sequence's cache split by block range over
ranks (one process per GPU), with the exchange steps of [AI-acc] §3
(communication libraries for multi-card inference) and [Hetero] §VII
(communication overlap).

Rank r holds blocks [j_lo, j_hi) of every sequence: their block keys
``k_c_local [B, j_hi - j_lo, H_i, d_c]`` and their KV pages, addressed by a
rank-local block table. One step for a batch of queries:

1. ``local_select``: the rank's exact top-k over its visible blocks (the
   library's index selection with positions shifted by ``-j_lo * bs``), the
   ids made global, and their scores.
2. an all-gather of (scores, ids) over the ranks, then ``merge_select``: the
   global top-k, the same on every rank and equal to the one-GPU ranking (the
   global top-k lies in the union of the ranks' top-k lists).
3. ``local_attend``: attention over the selected blocks the rank holds, as a
   normalised partial output with its log-sum-exp.
4. an all-gather of the partials, then ``merge_attend``: their exact
   log-sum-exp combination.

Every computation runs in the library's kernels; this module only prepares
arguments and calls ``torch.distributed`` for the two all-gathers (NCCL over
NVLink between GPUs). The exchanged bytes per query row are
``ranks * topk * 8`` for the selection and ``ranks * H_q * (2 * hd + 4)`` for
the partials.
"""
from __future__ import annotations

import dataclasses
from typing import List, Optional, Tuple

import torch

from . import lci

_I32_MIN, _I32_MAX = -(2 ** 31), 2 ** 31 - 1


def shard_ranges(nb: int, world: int) -> List[Tuple[int, int]]:
    """Contiguous block ranges [j_lo, j_hi) of near-equal size, one per rank."""
    if nb <= 0 or world <= 0:
        raise ValueError("shard_ranges: sizes must be positive")
    base, extra = divmod(nb, world)
    out, lo = [], 0
    for r in range(world):
        hi = lo + base + (1 if r < extra else 0)
        out.append((lo, hi))
        lo = hi
    return out


@dataclasses.dataclass
class ContextShard:
    """The part of a paged cache one rank holds: blocks [j_lo, j_hi)."""
    j_lo: int
    j_hi: int
    block_size: int
    k_c: torch.Tensor              # [B, j_hi - j_lo, H_i, d_c]
    table: lci.BlockTable          # local block -> local page
    k_pool: torch.Tensor           # [P_local, H_kv, bs, hd]
    v_pool: torch.Tensor

    def shifted(self, pos: torch.Tensor) -> torch.Tensor:
        """Positions in the shard's frame: pos - j_lo * block_size."""
        return lci.ids_shift(pos, _I32_MIN, _I32_MAX, -self.j_lo * self.block_size)


def local_select(shard: ContextShard, q_c: torch.Tensor, ctx_len: torch.Tensor,
                 q_start: torch.Tensor, topk: int, phase: str = "auto"):
    """Step 1: (scores, global ids) [B, S, topk] of the shard's top-k blocks."""
    ids = lci.index_select(q_c, shard.k_c, shard.block_size, shard.shifted(ctx_len),
                           shard.shifted(q_start), topk, phase=phase)
    scores = lci.block_scores_at(q_c, shard.k_c, ids)
    return scores, lci.ids_shift(ids, 0, shard.j_hi - shard.j_lo, shard.j_lo)


def merge_select(scores_all: torch.Tensor, ids_all: torch.Tensor) -> torch.Tensor:
    """Step 2: the global top-k [B, S, topk] from every rank's [R, B, S, topk] lists."""
    return lci.topk_merge(scores_all, ids_all)


def local_attend(shard: ContextShard, q: torch.Tensor, ids: torch.Tensor, ctx_len: torch.Tensor,
                 q_start: torch.Tensor, scale: float = 0.0, phase: str = "auto"):
    """Step 3: the partial (out [B, S, H_q, hd], lse [B, S, H_q]) over the
    selected blocks this shard holds."""
    local = lci.ids_shift(ids, shard.j_lo, shard.j_hi, -shard.j_lo)
    return lci.sparse_attn_partial(q, shard.k_pool, shard.v_pool, shard.table, local,
                                   shard.shifted(ctx_len), shard.shifted(q_start), scale=scale,
                                   phase=phase)


def merge_attend(o_all: torch.Tensor, lse_all: torch.Tensor) -> torch.Tensor:
    """Step 4: combine [R, B, S, H_q, hd] partials by their [R, B, S, H_q] lse."""
    return lci.attn_merge(o_all, lse_all)


def all_gather(x: torch.Tensor, group=None) -> torch.Tensor:
    """[R, *x.shape]: x of every rank, in rank order (x alone without a group)."""
    import torch.distributed as dist
    if group is None and not (dist.is_available() and dist.is_initialized()):
        return x.unsqueeze(0)
    world = dist.get_world_size(group)
    x = x.contiguous().reshape((-1,) + tuple(x.shape[1:])) if x.dim() else x.reshape(1)
    out = torch.empty((world * x.shape[0],) + tuple(x.shape[1:]), dtype=x.dtype, device=x.device)
    dist.all_gather_into_tensor(out, x, group=group)
    return out.reshape((world,) + tuple(x.shape))


def step(shard: ContextShard, q_c: torch.Tensor, q: torch.Tensor, ctx_len: torch.Tensor,
         q_start: torch.Tensor, topk: int, group=None, scale: float = 0.0,
         phase: str = "auto") -> Tuple[torch.Tensor, torch.Tensor]:
    """One context-parallel step on this rank: (global ids, out), identical on
    every rank of the group."""
    scores, ids = local_select(shard, q_c, ctx_len, q_start, topk, phase)
    ids = merge_select(all_gather(scores, group), all_gather(ids, group))
    o, lse = local_attend(shard, q, ids, ctx_len, q_start, scale, phase)
    return ids, merge_attend(all_gather(o, group), all_gather(lse, group))


def make_shard(j_lo: int, j_hi: int, k_c: torch.Tensor, block_table: torch.Tensor,
               k_pool: torch.Tensor, v_pool: torch.Tensor,
               device: Optional[torch.device] = None) -> ContextShard:
    """The shard of a one-GPU cache that holds blocks [j_lo, j_hi): its block
    keys and its pages, copied into rank-local tensors (local pages numbered in
    block order)."""
    device = k_c.device if device is None else device
    B = k_c.shape[0]
    n = j_hi - j_lo
    pages = block_table[:, j_lo:j_hi].reshape(-1).long().to(k_pool.device)
    kp = k_pool.index_select(0, pages).to(device).contiguous()
    vp = v_pool.index_select(0, pages).to(device).contiguous()
    local_table = torch.arange(B * n, dtype=torch.int32, device=device).reshape(B, n)
    bt = lci.create_block_table(local_table, kp)
    return ContextShard(j_lo, j_hi, kp.shape[2], k_c[:, j_lo:j_hi].contiguous().to(device), bt,
                        kp, vp)
