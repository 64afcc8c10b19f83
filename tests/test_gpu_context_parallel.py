"""Context parallelism (GPU), with the ranks emulated one after another on one
GPU: each shard's steps run on its own block range, and the all-gathers are
replaced by stacking the shards' results in rank order. Block ids must equal
the oracle's one-GPU ranking bit for bit; outputs must be within the bf16
tolerance of the oracle.
"""
import pytest
import torch

from long_context_indexer_b200 import cp
from long_context_indexer_b200.workloads import CONFIGS, generate
import oracle
from tests.gpu_common import assert_out_close

pytestmark = pytest.mark.gpu


def _emulate(cfg, w, world, rows=None):
    d = {k: v.cuda() for k, v in w.items()}
    shards = [cp.make_shard(lo, hi, d["k_c"], d["block_table"], d["k_pool"], d["v_pool"])
              for lo, hi in cp.shard_ranges(cfg.NB, world)]
    sel = [cp.local_select(sh, d["q_c"], d["ctx_len"], d["q_start"], cfg.topk) for sh in shards]
    ids = cp.merge_select(torch.stack([s for s, _ in sel]), torch.stack([i for _, i in sel]))
    part = [cp.local_attend(sh, d["q"], ids, d["ctx_len"], d["q_start"]) for sh in shards]
    out = cp.merge_attend(torch.stack([o for o, _ in part]), torch.stack([l for _, l in part]))
    torch.cuda.synchronize()
    import long_context_indexer_b200 as lci
    lci.get_device_status()
    return ids, out


@pytest.mark.parametrize("name,world", [("1m_decode", 4), ("1m_decode", 3), ("decode", 2),
                                        ("long", 8)])
def test_context_parallel_decode_matches_one_gpu_oracle(name, world):
    cfg = CONFIGS[name]
    w = generate(cfg)
    ids, out = _emulate(cfg, w, world)
    ref_ids = oracle.index_select(w["q_c"], w["k_c"], cfg.bs, w["ctx_len"], w["q_start"], cfg.topk)
    assert torch.equal(ids.cpu().reshape(-1, cfg.topk), ref_ids)
    ref = oracle.sparse_attn(w["q"], w["k_pool"], w["v_pool"], w["block_table"], ref_ids,
                             w["ctx_len"], w["q_start"], 1.0 / cfg.hd ** 0.5)
    assert_out_close(out.reshape(-1, cfg.H_q, cfg.hd), ref, torch.bfloat16, name)


def test_context_parallel_prefill_chunk_matches_one_gpu_oracle():
    cfg = CONFIGS["1m_chunk"].replace(S=512, q_start=(1 << 20) - 512)
    w = generate(cfg)
    ids, out = _emulate(cfg, w, 4)
    ref_ids = oracle.index_select(w["q_c"], w["k_c"], cfg.bs, w["ctx_len"], w["q_start"], cfg.topk)
    assert torch.equal(ids.cpu().reshape(-1, cfg.topk), ref_ids)
    rows = list(range(0, 512, 7))
    ref = oracle.sparse_attn(w["q"], w["k_pool"], w["v_pool"], w["block_table"], ref_ids[rows],
                             w["ctx_len"], w["q_start"], 1.0 / cfg.hd ** 0.5, rows=rows)
    assert_out_close(out.reshape(-1, cfg.H_q, cfg.hd)[rows], ref, torch.bfloat16, "cp chunk")


def test_context_parallel_with_ragged_short_sequences():
    """Sequences whose cache ends before some shards' ranges begin: those
    shards select nothing for them and contribute no partial."""
    cfg = CONFIGS["decode"].replace(B=3, ctx=4096, q_start=4095, topk=8, spare_pages=4)
    w = generate(cfg)
    w["ctx_len"] = torch.tensor([4096, 700, 1], dtype=torch.int32)
    w["q_start"] = torch.tensor([4095, 699, 0], dtype=torch.int32)
    ids, out = _emulate(cfg, w, 4)
    ref_ids = oracle.index_select(w["q_c"], w["k_c"], cfg.bs, w["ctx_len"], w["q_start"], cfg.topk)
    assert torch.equal(ids.cpu().reshape(-1, cfg.topk), ref_ids)
    ref = oracle.sparse_attn(w["q"], w["k_pool"], w["v_pool"], w["block_table"], ref_ids,
                             w["ctx_len"], w["q_start"], 1.0 / cfg.hd ** 0.5)
    assert_out_close(out.reshape(-1, cfg.H_q, cfg.hd), ref, torch.bfloat16, "ragged cp")
