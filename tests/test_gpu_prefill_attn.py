"""Tensor-core prefill attention (GPU) against the oracle and against the
one-row-at-a-time decode attention kernel on the same block ids.

The prefill kernel computes a tile of 128 MMA rows (several queries times the
query heads of one KV head) over the union of the blocks those queries
selected, masking per row. These cases stress what that schedule adds: unions
that leave a stage half empty, pages of 128 tokens (two units per block),
queries past the end of the sequence, -1 entries, rows that select nothing,
and logits whose maximum grows by far more than the lazy-rescale margin from
one stage to the next.
"""
import math

import pytest
import torch

import long_context_indexer_b200 as lci
import oracle
from long_context_indexer_b200.workloads import CONFIGS, generate
from tests.gpu_common import TOL, assert_out_close, oracle_rows, upload

pytestmark = pytest.mark.gpu

BASE = CONFIGS["prefill"].replace(name="pfa", spare_pages=8)


def _attn(cfg, d, ids, phase, scale=0.0):
    bt = lci.create_block_table(d["block_table"], d["k_pool"])
    out = lci.sparse_attn(d["q"], d["k_pool"], d["v_pool"], bt, ids, d["ctx_len"], d["q_start"],
                          scale=scale, phase=phase)
    torch.cuda.synchronize()
    lci.get_device_status()
    return out


def _oracle(cfg, w, ids, scale=None):
    scale = 1.0 / math.sqrt(cfg.hd) if scale is None else scale
    return oracle.sparse_attn(w["q"], w["k_pool"], w["v_pool"], w["block_table"],
                              ids.cpu().reshape(-1, ids.shape[-1]), w["ctx_len"], w["q_start"],
                              scale)


@pytest.mark.parametrize("S,q0,ctx,bs,topk,H_q,H_kv", [
    (77, 300, 377, 64, 5, 16, 1),      # ragged last tile, odd unions
    (40, 2000, 2040, 128, 7, 16, 1),   # 128-token pages: two units per block
    (33, 0, 33, 64, 3, 8, 1),          # 16 queries per tile, first block partial
    (50, 600, 700, 64, 9, 16, 2),      # two KV heads
    (64, 960, 1024, 64, 64, 16, 1),    # 512 selected blocks per tile
])
def test_prefill_kernel_matches_oracle_and_decode_kernel(S, q0, ctx, bs, topk, H_q, H_kv):
    cfg = BASE.replace(B=2, S=S, q_start=q0, ctx=ctx, bs=bs, topk=topk, H_q=H_q, H_kv=H_kv)
    w = generate(cfg)
    w["ctx_len"] = torch.tensor([ctx, max(1, ctx - 150)], dtype=torch.int32)
    d = upload(w)
    ids = lci.index_select(d["q_c"], d["k_c"], cfg.bs, d["ctx_len"], d["q_start"], cfg.topk)
    out_p = _attn(cfg, d, ids, "prefill")
    out_d = _attn(cfg, d, ids, "decode")
    ref = _oracle(cfg, w, ids)
    assert_out_close(out_p.reshape(-1, cfg.H_q, cfg.hd), ref, torch.bfloat16, "prefill kernel")
    assert (out_p.float() - out_d.float()).abs().max().item() <= TOL[torch.bfloat16]


def test_prefill_kernel_with_holes_and_empty_rows():
    """-1 entries anywhere in a row, rows with no block at all, and a block
    whose tokens all lie after the query."""
    cfg = BASE.replace(B=1, S=24, q_start=500, ctx=524, topk=6)
    w = generate(cfg)
    d = upload(w)
    ids = lci.index_select(d["q_c"], d["k_c"], cfg.bs, d["ctx_len"], d["q_start"], cfg.topk)
    ids = ids.clone()
    ids[0, 0, 2] = -1
    ids[0, 3, 0] = -1
    ids[0, 5, :] = -1                     # selects nothing: zero output
    ids[0, 7, :] = torch.tensor([8, -1, 0, -1, 3, -1], dtype=torch.int32)  # block 8 starts at 512 > 507
    out = _attn(cfg, d, ids, "prefill")
    ref = _oracle(cfg, w, ids)
    assert_out_close(out.reshape(-1, cfg.H_q, cfg.hd), ref, torch.bfloat16, "holes")
    assert (out[0, 5] == 0).all()


def test_prefill_kernel_rescales_when_the_maximum_jumps():
    """A softmax scale of 1 (about 11x the default) makes the logits' maximum
    grow by far more than the lazy margin between stages, so the running
    output is rescaled in TMEM many times."""
    cfg = BASE.replace(B=1, S=64, q_start=3000, ctx=3064, topk=24)
    w = generate(cfg)
    d = upload(w)
    ids = lci.index_select(d["q_c"], d["k_c"], cfg.bs, d["ctx_len"], d["q_start"], cfg.topk)
    out = _attn(cfg, d, ids, "prefill", scale=1.0)
    ref = _oracle(cfg, w, ids, scale=1.0)
    assert_out_close(out.reshape(-1, cfg.H_q, cfg.hd), ref, torch.bfloat16, "rescale")


def test_prefill_kernel_nan_tail_and_bad_ids_are_contained():
    """Cache slots past ctx_len hold NaN; an out-of-range block id is skipped
    and reported without disturbing the other rows."""
    cfg = BASE.replace(B=1, S=20, q_start=980, ctx=1000, topk=4)
    w = generate(cfg)
    last_block = (cfg.ctx - 1) // cfg.bs
    page = int(w["block_table"][0, last_block])
    w["k_pool"][page, :, cfg.ctx % cfg.bs:] = float("nan")
    w["v_pool"][page, :, cfg.ctx % cfg.bs:] = float("nan")
    d = upload(w)
    ids = lci.index_select(d["q_c"], d["k_c"], cfg.bs, d["ctx_len"], d["q_start"], cfg.topk)
    ref_ids, ref = oracle_rows(cfg, w)
    assert torch.equal(ids.cpu().reshape(-1, cfg.topk), ref_ids)
    out = _attn(cfg, d, ids, "prefill")
    assert_out_close(out.reshape(-1, cfg.H_q, cfg.hd), ref, torch.bfloat16, "nan tail")
    bad = ids.clone()
    bad[0, 4, 1] = cfg.NB + 3
    bt = lci.create_block_table(d["block_table"], d["k_pool"])
    lci.sparse_attn(d["q"], d["k_pool"], d["v_pool"], bt, bad, d["ctx_len"], d["q_start"],
                    phase="prefill")
    with pytest.raises(lci.LciError) as e:
        lci.get_device_status()
    assert e.value.status == 5
