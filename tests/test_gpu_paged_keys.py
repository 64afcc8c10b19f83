"""Block keys kept per page of the paged cache (GPU): the online producer
against the oracle's block compression, and index selection through the block
table against the oracle's ranking on the dense keys.

Indexer keys are multiples of 1/16 in [-2, 2], so the fp32 running sums are
exact and every key must match the oracle's mean rounded once to bf16, bit for
bit, after any sequence of appends (a prefill chunk, single decode tokens, a
chunk that starts inside a block).
"""
import pytest
import torch

import long_context_indexer_b200 as lci
import oracle
from long_context_indexer_b200.workloads import CONFIGS, generate, grid_values

pytestmark = pytest.mark.gpu


def _table(B, NB, P, seed):
    perm = torch.randperm(P, generator=torch.Generator().manual_seed(seed)).to(torch.int32)
    return perm[: B * NB].reshape(B, NB).contiguous()


def _gathered(keys, table, nb):
    """[B, nb, H_i, d_c] keys of the first nb blocks of every sequence (CPU)."""
    kc = keys.kc.cpu()
    return kc[table[:, :nb].long()]


@pytest.mark.parametrize("dtype,bs", [(torch.bfloat16, 64), (torch.float32, 16), (torch.bfloat16, 48)])
def test_online_keys_match_block_compression_after_every_kind_of_append(dtype, bs):
    B, H_i, d_c, ctx = 3, 2, 64, 260
    NB = (ctx + bs - 1) // bs
    P = B * NB + 7
    gen = torch.Generator().manual_seed(11)
    k_idx = grid_values((B, ctx, H_i, d_c), gen, dtype)
    table = _table(B, NB, P, 12)
    dummy_pool = torch.zeros((P, 1, bs, 32), dtype=dtype, device="cuda")
    bt = lci.create_block_table(table.cuda(), dummy_pool)
    keys = lci.PagedKeys(P, H_i, d_c, dtype, "cuda")
    keys.kc.fill_(float("nan"))  # pages are written only by the producer
    d_k = k_idx.cuda()
    # prefill chunk of 70, single tokens to 130, a chunk of 37 starting inside a
    # block, then single tokens to the end
    plan = [(0, 70)] + [(t, 1) for t in range(70, 130)] + [(130, 37)] + \
           [(t, 1) for t in range(167, ctx)]
    checkpoints = {130, 167, ctx}
    for p0, T in plan:
        start = torch.full((B,), p0, dtype=torch.int32, device="cuda")
        keys.update(d_k[:, p0:p0 + T].contiguous(), start, bt)
        n = p0 + T
        if n in checkpoints:
            torch.cuda.synchronize()
            lci.get_device_status()
            nb = (n + bs - 1) // bs
            ref = oracle.block_compress(k_idx[:, :n], bs).to(dtype)
            got = _gathered(keys, table, nb)
            assert torch.equal(got, ref), f"keys differ after {n} tokens"


def test_online_keys_flag_blocks_past_the_table():
    B, H_i, d_c, bs = 1, 1, 16, 16
    table = _table(B, 2, 4, 3)
    bt = lci.create_block_table(table.cuda(), torch.zeros((4, 1, bs, 32), device="cuda"))
    keys = lci.PagedKeys(4, H_i, d_c, torch.float32, "cuda")
    k = torch.ones((B, 1, H_i, d_c), device="cuda")
    keys.update(k, torch.tensor([2 * bs], dtype=torch.int32, device="cuda"), bt)  # block 2 of 2
    with pytest.raises(lci.LciError) as e:
        lci.get_device_status()
    assert e.value.status == 5
    assert (keys.kc == 0).all()


def _paged_from_dense(cfg, w):
    """Scatter the dense block keys into a page pool through the block table;
    pages no sequence references hold NaN."""
    P = cfg.num_pages
    kc = torch.full((P, cfg.H_i, cfg.d_c), float("nan"), dtype=cfg.torch_dtype)
    kc[w["block_table"].reshape(-1).long()] = w["k_c"].reshape(-1, cfg.H_i, cfg.d_c)
    return kc


@pytest.mark.parametrize("name,phase", [("decode", "auto"), ("long", "auto"),
                                        ("prefill", "auto"), ("prefill", "decode")])
def test_paged_index_select_matches_oracle(name, phase):
    cfg = CONFIGS[name]
    if name == "prefill" and phase == "decode":
        cfg = cfg.replace(S=1024, ctx=5000, q_start=5000 - 1024)
    w = generate(cfg, with_kv=False)
    kc = _paged_from_dense(cfg, w).cuda()
    d = {k: v.cuda() for k, v in w.items()}
    bt = lci.create_block_table(d["block_table"],
                                torch.zeros((cfg.num_pages, 1, cfg.bs, 32), dtype=cfg.torch_dtype,
                                            device="cuda"))
    ids = lci.index_select_paged(d["q_c"], kc, bt, d["ctx_len"], d["q_start"], cfg.topk,
                                 phase=phase)
    torch.cuda.synchronize()
    lci.get_device_status()
    ref = oracle.index_select(w["q_c"], w["k_c"], cfg.bs, w["ctx_len"], w["q_start"], cfg.topk)
    assert torch.equal(ids.cpu().reshape(-1, cfg.topk), ref)
    dense = lci.index_select(d["q_c"], d["k_c"], cfg.bs, d["ctx_len"], d["q_start"], cfg.topk,
                             phase=phase)
    assert torch.equal(ids, dense)
