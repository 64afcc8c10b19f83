"""CUDA path (through the C ABI) against the CPU oracle, element by element.

Block ids must match bit for bit (order and -1 padding included); outputs must
match within max-abs 2e-2 (bf16) or 1e-4 (fp32). The five measured
configurations run at full size, with the oracle computing every id row where
that takes seconds and sampled rows (first, last, block boundaries, random)
where it does not.
"""
import random

import pytest
import torch

import long_context_indexer_b200 as lci
import oracle
from long_context_indexer_b200.workloads import CONFIGS, generate
from tests.gpu_common import TOL, assert_out_close, oracle_k_c, oracle_rows, run_gpu, upload

pytestmark = pytest.mark.gpu


def _sample_rows(cfg, n_random=24, seed=0):
    S, B = cfg.S, cfg.B
    rows = set()
    for b in range(B):
        for s in (0, 1, cfg.bs - 1, cfg.bs, cfg.bs + 1, S // 2, S - 2, S - 1):
            if 0 <= s < S:
                rows.add(b * S + s)
    rng = random.Random(seed)
    rows.update(rng.randrange(B * S) for _ in range(n_random))
    return sorted(rows)


# ------------------------------------------------------------ full configs

def test_tiny_fp32_end_to_end():
    cfg = CONFIGS["tiny"]
    w = generate(cfg)
    k_c, ids, out = run_gpu(cfg, upload(w))
    assert torch.equal(k_c.cpu().double(), oracle.block_compress(w["k_idx"], cfg.bs))
    ref_ids, ref_out = oracle_rows(cfg, w)
    assert torch.equal(ids.cpu().reshape(-1, cfg.topk), ref_ids)
    assert_out_close(out.reshape(-1, cfg.H_q, cfg.hd), ref_out, torch.float32, "tiny")


@pytest.mark.parametrize("name", ["decode", "long", "1m_decode"])
def test_decode_configs_all_rows(name):
    cfg = CONFIGS[name]
    w = generate(cfg)
    _, ids, out = run_gpu(cfg, upload(w))
    ref_ids, ref_out = oracle_rows(cfg, w)
    assert torch.equal(ids.cpu().reshape(-1, cfg.topk), ref_ids)
    assert_out_close(out.reshape(-1, cfg.H_q, cfg.hd), ref_out, torch.bfloat16, name)


def _rows_per_tile(cfg, per_tile, tile=128, seed=0):
    """Flat query rows spread over every tile of `tile` consecutive queries of
    every sequence: the first and last row of each tile plus random ones."""
    rng = random.Random(seed)
    rows = set()
    for b in range(cfg.B):
        for t0 in range(0, cfg.S, tile):
            t1 = min(cfg.S, t0 + tile)
            picks = {t0, t1 - 1}
            while len(picks) < min(per_tile, t1 - t0):
                picks.add(rng.randrange(t0, t1))
            rows.update(b * cfg.S + s for s in picks)
    return sorted(rows)


def test_prefill_config():
    cfg = CONFIGS["prefill"]
    w = generate(cfg)
    _, ids, out = run_gpu(cfg, upload(w))
    # every id row (8192 x 128 blocks) ...
    ref_ids = oracle.index_select(w["q_c"], w["k_c"], cfg.bs, w["ctx_len"], w["q_start"], cfg.topk)
    assert torch.equal(ids.cpu().reshape(-1, cfg.topk), ref_ids)
    # ... and the attention output on 8 rows of each of the 64 tiles of 128
    # queries, plus the block boundaries
    rows = sorted(set(_rows_per_tile(cfg, 8)) | set(_sample_rows(cfg, 0)))
    assert len(rows) >= 512
    _, ref_out = oracle_rows(cfg, w, rows=rows)
    got = out.reshape(-1, cfg.H_q, cfg.hd)[rows]
    assert_out_close(got, ref_out, torch.bfloat16, "prefill")
    assert torch.isfinite(out).all()


def test_1m_chunk_config():
    cfg = CONFIGS["1m_chunk"]
    w = generate(cfg)
    _, ids, out = run_gpu(cfg, upload(w))
    # every id row: 4096 queries x 8192 visible blocks, against the oracle's
    # full ranking (this is the shape on which the tensor-core indexer splits
    # each m-tile's blocks over CTAs and merges their lists)
    ref_ids = oracle.index_select(w["q_c"], w["k_c"], cfg.bs, w["ctx_len"], w["q_start"], cfg.topk)
    assert torch.equal(ids.cpu().reshape(-1, cfg.topk), ref_ids)
    # the attention output on 16 rows of each of the 32 tiles of 128 queries
    rows = _rows_per_tile(cfg, 16)
    assert len(rows) >= 512
    ref_out = oracle.sparse_attn(w["q"], w["k_pool"], w["v_pool"], w["block_table"], ref_ids[rows],
                                 w["ctx_len"], w["q_start"], 1.0 / cfg.hd ** 0.5, rows=rows)
    assert_out_close(out.reshape(-1, cfg.H_q, cfg.hd)[rows], ref_out, torch.bfloat16, "1m_chunk")
    assert torch.isfinite(out).all()


# ------------------------------------------------------------ small cases, edges

SMALL = CONFIGS["decode"].replace(name="small", B=3, S=1, ctx=1000, q_start=999, bs=64, topk=4,
                                  H_q=8, H_kv=2, hd=128, H_i=2, d_c=64, spare_pages=5)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("S,q0,ctx,topk", [(1, 999, 1000, 4), (37, 950, 1000, 3), (70, 0, 70, 2),
                                           (5, 1200, 1000, 32), (300, 10, 900, 1)])
def test_small_ragged_cases(dtype, S, q0, ctx, topk):
    cfg = SMALL.replace(dtype=dtype, S=S, q_start=q0, ctx=ctx, topk=topk)
    w = generate(cfg)
    # ragged per-sequence lengths and start positions
    w["ctx_len"] = torch.tensor([ctx, max(1, ctx // 2), 1], dtype=torch.int32)[: cfg.B]
    w["q_start"] = torch.tensor([q0, max(0, q0 - 333), 0], dtype=torch.int32)[: cfg.B]
    _, ids, out = run_gpu(cfg, upload(w))
    ref_ids, ref_out = oracle_rows(cfg, w)
    assert torch.equal(ids.cpu().reshape(-1, topk), ref_ids)
    assert_out_close(out.reshape(-1, cfg.H_q, cfg.hd), ref_out, cfg.torch_dtype, "ragged")


def test_empty_context_gives_no_ids_and_zero_output():
    cfg = SMALL
    w = generate(cfg)
    w["ctx_len"] = torch.tensor([0, 0, 5], dtype=torch.int32)
    _, ids, out = run_gpu(cfg, upload(w))
    assert (ids[:2] == -1).all()
    assert (out[:2] == 0).all()
    assert ids[2, 0, 0].item() == 0 and (ids[2, 0, 1:] == -1).all()


def test_ties_break_to_lower_block_id():
    cfg = SMALL.replace(S=4, q_start=996)
    w = generate(cfg)
    w["q_c"].zero_()
    _, ids, _ = run_gpu(cfg, upload(w))
    assert (ids.cpu() == torch.arange(cfg.topk, dtype=torch.int32)).all()
    # partial ties: only a few distinct score values
    w = generate(cfg)
    w["q_c"] = (w["q_c"] > 1).to(w["q_c"].dtype) * 0.0625
    w["k_c"] = (w["k_c"] > 0).to(w["k_c"].dtype) * 0.0625
    _, ids, _ = run_gpu(cfg, upload(w))
    ref_ids, _ = oracle_rows(cfg, w)
    assert torch.equal(ids.cpu().reshape(-1, cfg.topk), ref_ids)


@pytest.mark.parametrize("ctx,topk,mode", [
    (32768, 200, "grid"),    # k above the sorted-list pass: radix select over 512 blocks
    (262144, 200, "grid"),   # the same over 4096 blocks
    (262144, 64, "zero"),    # all scores equal: every chunk survives pruning -> radix select
    (262144, 64, "few"),     # few distinct scores: ties at the pruning bound
    (70400, 128, "grid"),    # 1100 blocks, k at the sorted pass's limit, pruned
    (8192, 128, "grid"),     # k == n: all 128 visible blocks, in rank order
    (65536, 1, "grid"),      # k == 1 over 1024 blocks (one sorted-list pass, 4 per lane)
    (16384, 9, "grid"),      # 256 blocks: one composite per lane
])
def test_select_paths(ctx, topk, mode):
    """Every branch of the CTA top-k: one sorted-list pass (32, 64 or 128
    composites per warp), pruning by chunk maxima then a sorted-list pass, and
    the exact radix select for large k or candidate sets that ties inflate."""
    cfg = CONFIGS["decode"].replace(name="sel", B=2, ctx=ctx, q_start=ctx - 1, topk=topk)
    w = generate(cfg, with_kv=False)
    dt = w["q_c"].dtype
    if mode == "zero":
        w["q_c"].zero_()
    elif mode == "few":
        w["q_c"] = (w["q_c"] > 1).to(dt) * 0.0625
        w["k_c"] = (w["k_c"] > 0).to(dt) * 0.0625
    d = upload(w)
    ids = lci.index_select(d["q_c"], d["k_c"], cfg.bs, d["ctx_len"], d["q_start"], topk)
    torch.cuda.synchronize()
    lci.get_device_status()
    ref = oracle.index_select(w["q_c"], w["k_c"], cfg.bs, w["ctx_len"], w["q_start"], topk)
    assert torch.equal(ids.cpu().reshape(-1, topk), ref.reshape(-1, topk))
    if mode == "zero":
        assert (ids.cpu().reshape(-1, topk) == torch.arange(topk, dtype=torch.int32)).all()


def test_extreme_grid_values_are_exact():
    cfg = SMALL.replace(H_i=8, d_c=128, topk=6, S=2, q_start=998)
    w = generate(cfg)
    w["q_c"].fill_(2.0)
    sign = torch.where(torch.rand(w["k_c"].shape, generator=torch.Generator().manual_seed(5)) < 0.5,
                       -2.0, 2.0)
    w["k_c"] = sign.to(w["k_c"].dtype)
    _, ids, _ = run_gpu(cfg, upload(w))
    ref_ids, _ = oracle_rows(cfg, w)
    assert torch.equal(ids.cpu().reshape(-1, cfg.topk), ref_ids)


def test_decode_matches_prefill_rows():
    """The shared representation: decode at position p equals prefill row p."""
    cfg = SMALL.replace(S=48, q_start=900, ctx=948, B=2)
    w = generate(cfg)
    d = upload(w)
    _, ids_p, out_p = run_gpu(cfg, d, phase="prefill")
    for s in (0, 17, 47):
        d1 = dict(d)
        d1["q_c"] = d["q_c"][:, s:s + 1].contiguous()
        d1["q"] = d["q"][:, s:s + 1].contiguous()
        d1["q_start"] = d["q_start"] + s
        _, ids_d, out_d = run_gpu(cfg.replace(S=1), d1, phase="decode")
        assert torch.equal(ids_d[:, 0], ids_p[:, s])
        assert (out_d[:, 0].float() - out_p[:, s].float()).abs().max().item() <= TOL[torch.bfloat16]


def test_phases_agree_and_runs_are_deterministic():
    cfg = SMALL.replace(S=40, q_start=500)
    d = upload(generate(cfg))
    res = [run_gpu(cfg, d, phase=ph) for ph in ("auto", "prefill", "decode", "auto")]
    for r in res[1:]:
        assert torch.equal(r[1], res[0][1])
    assert torch.equal(res[3][2], res[0][2])


def test_page_permutation_gives_identical_output():
    cfg = SMALL.replace(S=3, q_start=990)
    w = generate(cfg)
    d = upload(w)
    _, ids, out = run_gpu(cfg, d)
    P = cfg.num_pages
    perm = torch.randperm(P, generator=torch.Generator().manual_seed(7))
    k2 = torch.empty_like(w["k_pool"])
    v2 = torch.empty_like(w["v_pool"])
    k2[perm] = w["k_pool"]
    v2[perm] = w["v_pool"]
    d2 = dict(d, k_pool=k2.cuda(), v_pool=v2.cuda(),
              block_table=perm[w["block_table"].long()].to(torch.int32).cuda())
    _, ids2, out2 = run_gpu(cfg, d2)
    assert torch.equal(ids, ids2)
    assert torch.equal(out, out2)


def test_explicit_scale():
    cfg = SMALL.replace(S=2, q_start=998)
    w = generate(cfg)
    _, _, out = run_gpu(cfg, upload(w), scale=0.02)
    _, ref = oracle_rows(cfg, w, scale=0.02)
    assert_out_close(out.reshape(-1, cfg.H_q, cfg.hd), ref, torch.bfloat16, "scale")


def test_device_bounds_checks_report_without_trapping():
    cfg = SMALL
    w = generate(cfg)
    d = upload(w)
    bt = lci.create_block_table(d["block_table"], d["k_pool"])
    bad_ids = torch.tensor([[[0, cfg.NB, -1, 3]], [[-5, 1, 2, -1]], [[0, 1, 2, 3]]],
                           dtype=torch.int32, device="cuda")
    lci.sparse_attn(d["q"], d["k_pool"], d["v_pool"], bt, bad_ids, d["ctx_len"], d["q_start"])
    with pytest.raises(lci.LciError) as e:
        lci.get_device_status()
    assert e.value.status == 5
    lci.get_device_status()  # cleared
    bad_table = d["block_table"].clone()
    bad_table[1, 3] = cfg.num_pages
    bt2 = lci.create_block_table(bad_table, d["k_pool"])
    bt2.validate()
    with pytest.raises(lci.LciError):
        lci.get_device_status()
    ok_ids = torch.tensor([[[0, 1, 2, 3]]] * 3, dtype=torch.int32, device="cuda")
    lci.sparse_attn(d["q"], d["k_pool"], d["v_pool"], bt2, ok_ids, d["ctx_len"], d["q_start"])
    with pytest.raises(lci.LciError):
        lci.get_device_status()


@pytest.mark.parametrize("S,q0", [(1, 999), (24, 976)])
def test_unwritten_cache_slots_never_reach_the_output(S, q0):
    """Pool slots past ctx_len (unwritten cache memory) are loaded with their
    64-token tile but masked; NaN there must not leak into the output."""
    cfg = SMALL.replace(S=S, q_start=q0, ctx=1000)
    w = generate(cfg)
    bs = cfg.bs
    for b in range(cfg.B):
        last_block = (cfg.ctx - 1) // bs
        page = int(w["block_table"][b, last_block])
        w["k_pool"][page, :, cfg.ctx % bs:] = float("nan")
        w["v_pool"][page, :, cfg.ctx % bs:] = float("nan")
    _, ids, out = run_gpu(cfg, upload(w))
    ref_ids, ref_out = oracle_rows(cfg, w)
    assert torch.equal(ids.cpu().reshape(-1, cfg.topk), ref_ids)
    assert_out_close(out.reshape(-1, cfg.H_q, cfg.hd), ref_out, torch.bfloat16, "nan-tail")


@pytest.mark.parametrize("persistent", [False, True])
@pytest.mark.parametrize("name", ["decode", "small", "small_f32", "1m_decode"])
def test_fused_decode_step_matches_two_calls_and_oracle(name, persistent):
    """lci_sparse_decode (rows attended as soon as they are selected) gives the
    block ids and outputs of index_select + sparse_attn, call after call."""
    cfg = {"decode": CONFIGS["decode"], "1m_decode": CONFIGS["1m_decode"], "small": SMALL,
           "small_f32": SMALL.replace(dtype="f32")}[name]
    if persistent and name.startswith("small"):
        pytest.skip("the one-launch step takes 1024-feature bf16 keys")
    w = generate(cfg)
    d = upload(w)
    _, ids2, out2 = run_gpu(cfg, d)
    bt = lci.create_block_table(d["block_table"], d["k_pool"])
    first = None
    for _ in range(3):  # the per-call state must reset between calls
        ids, out = lci.sparse_decode(d["q_c"], d["k_c"], d["ctx_len"], d["q_start"], cfg.topk,
                                     d["q"], d["k_pool"], d["v_pool"], bt, persistent=persistent)
        torch.cuda.synchronize()
        lci.get_device_status()
        assert torch.equal(ids, ids2)
        # the one-launch step splits and combines the attention its own way:
        # within the tolerance of the two-call result, and run to run identical
        assert (out.float() - out2.float()).abs().max().item() <= TOL[cfg.torch_dtype]
        first = out.clone() if first is None else first
        assert torch.equal(out, first)
    ref_ids, ref_out = oracle_rows(cfg, w)
    assert torch.equal(ids.cpu().reshape(-1, cfg.topk), ref_ids)
    assert_out_close(out.reshape(-1, cfg.H_q, cfg.hd), ref_out, cfg.torch_dtype, name)


@pytest.mark.parametrize("topk", [48, 64])
def test_prefill_tensor_core_long_lists_split_tiles(topk):
    """The tensor-core indexer with lists longer than 32 (one epilogue warp per
    TMEM lane quarter) and each row's n-tiles split over two CTAs whose lists
    the last CTA merges."""
    cfg = SMALL.replace(B=1, S=256, ctx=20000, q_start=20000 - 256, topk=topk)
    assert cfg.NB > 256  # two 256-block n-tiles
    w = generate(cfg)
    _, ids, out = run_gpu(cfg, upload(w), phase="prefill")
    ref_ids, ref_out = oracle_rows(cfg, w)
    assert torch.equal(ids.cpu().reshape(-1, topk), ref_ids)
    assert_out_close(out.reshape(-1, cfg.H_q, cfg.hd), ref_out, cfg.torch_dtype, "long lists")


@pytest.mark.parametrize("B,H_kv", [(20, 2), (60, 1)])
def test_decode_attention_deep_ring_uneven_splits(B, H_kv):
    """Decode shapes whose (row, KV head) pairs fill the SMs with 3- or 2-CTA
    clusters: the 6-stage ring, with units split unevenly over the cluster."""
    cfg = CONFIGS["decode"].replace(name="deep", B=B, H_kv=H_kv, ctx=6000, q_start=5999,
                                    topk=11, spare_pages=8)
    w = generate(cfg)
    d = upload(w)
    _, ids, out = run_gpu(cfg, d)
    ref_ids, ref_out = oracle_rows(cfg, w)
    assert torch.equal(ids.cpu().reshape(-1, cfg.topk), ref_ids)
    assert_out_close(out.reshape(-1, cfg.H_q, cfg.hd), ref_out, cfg.torch_dtype, "deep ring")
    bt = lci.create_block_table(d["block_table"], d["k_pool"])
    for persistent in (False, True):
        ids_f, out_f = lci.sparse_decode(d["q_c"], d["k_c"], d["ctx_len"], d["q_start"], cfg.topk,
                                         d["q"], d["k_pool"], d["v_pool"], bt,
                                         persistent=persistent)
        torch.cuda.synchronize()
        assert torch.equal(ids_f, ids)
        assert_out_close(out_f.reshape(-1, cfg.H_q, cfg.hd), ref_out, cfg.torch_dtype, "one call")


@pytest.mark.parametrize("B,H_kv,topk", [(300, 1, 3), (150, 1, 4), (100, 1, 4), (40, 1, 4),
                                         (50, 1, 7), (40, 1, 9), (1, 1, 5), (3, 2, 5), (1, 1, 6),
                                         (1, 1, 7), (2, 1, 9)])
def test_decode_attention_every_cluster_size(B, H_kv, topk):
    """Decode shapes that split each (row, KV head) pair over 1 to 8 CTAs of a
    cluster (the split count follows from the pairs and the units per pair):
    300 pairs run one CTA each, 150, 100 and 40 pairs two-CTA-per-SM clusters
    of 2, 3 and 4; 50 and 40 pairs with 7 and 9 units one-CTA-per-SM clusters
    of 2 and 3 (two consumer groups on alternate tiles, odd unit counts), and
    single rows with 5, 6, 7 or 9 units clusters of 5 to 8, whose output slices
    are uneven. H_kv = 2 leaves half of the 16 MMA rows unused."""
    cfg = CONFIGS["decode"].replace(name="splits", B=B, H_kv=H_kv, ctx=1000, q_start=999,
                                    topk=topk, spare_pages=4)
    w = generate(cfg)
    _, ids, out = run_gpu(cfg, upload(w))
    ref_ids, ref_out = oracle_rows(cfg, w)
    assert torch.equal(ids.cpu().reshape(-1, cfg.topk), ref_ids)
    assert_out_close(out.reshape(-1, cfg.H_q, cfg.hd), ref_out, cfg.torch_dtype, "cluster splits")


@pytest.mark.parametrize("name", ["decode", "long", "1m_decode"])
def test_one_launch_decode_step_over_many_calls(name):
    """The one-launch decode step (persistent CTAs claiming scoring chunks, then
    attention splits) keeps its per-call counters and epoch in the workspace:
    ten calls in a row on one workspace, interleaved with calls of another
    size on another workspace, give the oracle's ids and outputs every time."""
    cfg = CONFIGS[name]
    w = generate(cfg)
    d = upload(w)
    bt = lci.create_block_table(d["block_table"], d["k_pool"])
    other = SMALL.replace(H_i=8, d_c=128, S=3, q_start=997)
    wo = generate(other)
    do = upload(wo)
    bto = lci.create_block_table(do["block_table"], do["k_pool"])
    ref_ids, ref_out = oracle_rows(cfg, w)
    ref_ids_o, ref_out_o = oracle_rows(other, wo)
    for _ in range(10):
        ids, out = lci.sparse_decode(d["q_c"], d["k_c"], d["ctx_len"], d["q_start"], cfg.topk,
                                     d["q"], d["k_pool"], d["v_pool"], bt, persistent=True)
        ids_o, out_o = lci.sparse_decode(do["q_c"], do["k_c"], do["ctx_len"], do["q_start"],
                                         other.topk, do["q"], do["k_pool"], do["v_pool"], bto,
                                         persistent=True)
    torch.cuda.synchronize()
    lci.get_device_status()
    assert torch.equal(ids.cpu().reshape(-1, cfg.topk), ref_ids)
    assert_out_close(out.reshape(-1, cfg.H_q, cfg.hd), ref_out, torch.bfloat16, name)
    assert torch.equal(ids_o.cpu().reshape(-1, other.topk), ref_ids_o)
    assert_out_close(out_o.reshape(-1, other.H_q, other.hd), ref_out_o, torch.bfloat16, "other")


def test_prepared_decode_step_matches_the_plain_call():
    """SparseDecodeStep takes its pointers once and launches with them every
    call; after the inputs are overwritten in place it sees the new values."""
    cfg = CONFIGS["decode"].replace(B=8, ctx=8192, q_start=8191, spare_pages=8)
    w = generate(cfg)
    d = upload(w)
    bt = lci.create_block_table(d["block_table"], d["k_pool"])
    step = lci.SparseDecodeStep(d["q_c"], d["k_c"], d["ctx_len"], d["q_start"], cfg.topk, d["q"],
                                d["k_pool"], d["v_pool"], bt)
    for seed in (0, 1):
        if seed:
            d["q_c"].copy_(torch.flip(d["q_c"], dims=[0]))
            d["q"].copy_(torch.flip(d["q"], dims=[0]))
        step()
        ids, out = lci.sparse_decode(d["q_c"], d["k_c"], d["ctx_len"], d["q_start"], cfg.topk,
                                     d["q"], d["k_pool"], d["v_pool"], bt)
        torch.cuda.synchronize()
        lci.get_device_status()
        assert torch.equal(step.ids, ids)
        assert torch.equal(step.out, out)


def test_prepared_decode_step_graph_with_transfers():
    """SparseDecodeStep.capture: host-to-device copies of the inputs, the step
    and device-to-host copies of ids and out, replayed as one CUDA graph; each
    replay sees the host inputs' current contents and matches the plain call."""
    cfg = CONFIGS["decode"].replace(B=8, ctx=8192, q_start=8191, spare_pages=8)
    w = generate(cfg)
    d = upload(w)
    bt = lci.create_block_table(d["block_table"], d["k_pool"])
    h_qc = w["q_c"].clone().pin_memory()
    h_q = w["q"].clone().pin_memory()
    step = lci.SparseDecodeStep(d["q_c"], d["k_c"], d["ctx_len"], d["q_start"], cfg.topk, d["q"],
                                d["k_pool"], d["v_pool"], bt)
    h_ids = torch.empty(step.ids.shape, dtype=step.ids.dtype).pin_memory()
    h_out = torch.empty(step.out.shape, dtype=step.out.dtype).pin_memory()
    step()
    g = step.capture(h2d=[(d["q_c"], h_qc), (d["q"], h_q)], d2h=[(h_ids, step.ids), (h_out, step.out)])
    for flip in (False, True):
        if flip:
            h_qc.copy_(torch.flip(w["q_c"], dims=[0]))
            h_q.copy_(torch.flip(w["q"], dims=[0]))
        g.replay()
        torch.cuda.synchronize()
        ids, out = lci.sparse_decode(h_qc.cuda(), d["k_c"], d["ctx_len"], d["q_start"], cfg.topk,
                                     h_q.cuda(), d["k_pool"], d["v_pool"], bt)
        torch.cuda.synchronize()
        lci.get_device_status()
        assert torch.equal(h_ids, ids.cpu())
        assert torch.equal(h_out, out.cpu())
    with pytest.raises(ValueError):
        step.capture(h2d=[(d["q_c"], w["q_c"])])  # pageable host memory


def test_both_decode_forms_share_one_workspace():
    """The two-kernel and the one-launch decode forms alternate on one
    workspace: neither takes the other's publication flags for its own."""
    cfg = CONFIGS["decode"].replace(B=20, H_kv=2, ctx=6000, q_start=5999, topk=11, spare_pages=8)
    w = generate(cfg)
    d = upload(w)
    ref_ids, ref_out = oracle_rows(cfg, w)
    bt = lci.create_block_table(d["block_table"], d["k_pool"])
    need = lci.sparse_decode_workspace_size(cfg.B, cfg.S, cfg.H_i, cfg.d_c, cfg.topk, cfg.H_q, bt)
    ws = torch.zeros(need, dtype=torch.uint8, device="cuda")
    for persistent in (False, True, True, False, True):
        ids = torch.full((cfg.B, 1, cfg.topk), 12345, dtype=torch.int32, device="cuda")
        ids, out = lci.sparse_decode(d["q_c"], d["k_c"], d["ctx_len"], d["q_start"], cfg.topk,
                                     d["q"], d["k_pool"], d["v_pool"], bt, ids=ids, ws=ws,
                                     persistent=persistent)
        torch.cuda.synchronize()
        lci.get_device_status()
        assert torch.equal(ids.cpu().reshape(-1, cfg.topk), ref_ids), persistent
        assert_out_close(out.reshape(-1, cfg.H_q, cfg.hd), ref_out, cfg.torch_dtype,
                         f"persistent={persistent}")


def test_one_workspace_serves_every_schedule_dtype_and_topk():
    """Calls with the same (batch, S) share one workspace without clearing it:
    the tensor-core schedule with split candidate lists (bf16, two topk
    values) and the row-wise schedule (f32, and bf16 with phase 'decode')
    alternate on it, and every call's ids match the oracle."""
    base = SMALL.replace(S=37, q_start=950, ctx=1000)
    calls = [("bf16", 3, "prefill"), ("f32", 3, "auto"), ("bf16", 16, "prefill"),
             ("bf16", 5, "decode"), ("bf16", 3, "prefill"), ("f32", 16, "auto")]
    need = max(lci.index_select_workspace_size(base.B, base.S, base.H_i, base.d_c, base.NB, k, ph)
               for _, k, ph in calls)
    ws = torch.zeros(need + 256, dtype=torch.uint8, device="cuda")
    off = (-ws.data_ptr()) % 256
    ws = ws[off:off + need]
    for dtype, topk, phase in calls:
        cfg = base.replace(dtype=dtype, topk=topk)
        w = generate(cfg, with_kv=False)
        w["ctx_len"] = torch.tensor([1000, 500, 1], dtype=torch.int32)
        w["q_start"] = torch.tensor([950, 617, 0], dtype=torch.int32)
        d = upload(w)
        ids = lci.index_select(d["q_c"], d["k_c"], cfg.bs, d["ctx_len"], d["q_start"], topk,
                               phase=phase, ws=ws)
        torch.cuda.synchronize()
        lci.get_device_status()
        ref = oracle.index_select(w["q_c"], w["k_c"], cfg.bs, w["ctx_len"], w["q_start"], topk)
        assert torch.equal(ids.cpu().reshape(-1, topk), ref), (dtype, topk, phase)


@pytest.mark.parametrize("topk", [32, 64])
def test_prefill_indexer_column_windows(topk):
    """Every m-tile has a single 256-block n-tile, so its CTAs (four here) split
    the tile's visible columns into windows of whole 32-column groups, the last
    window ragged, and the last CTA merges the windows' lists."""
    cfg = SMALL.replace(B=1, S=2560, ctx=12800, q_start=12800 - 2560, topk=topk)
    assert cfg.NB == 200
    w = generate(cfg, with_kv=False)
    d = upload(w)
    ids = lci.index_select(d["q_c"], d["k_c"], cfg.bs, d["ctx_len"], d["q_start"], topk,
                           phase="prefill")
    torch.cuda.synchronize()
    lci.get_device_status()
    ref = oracle.index_select(w["q_c"], w["k_c"], cfg.bs, w["ctx_len"], w["q_start"], topk)
    assert torch.equal(ids.cpu().reshape(-1, topk), ref)


def test_prefill_indexer_sequence_without_context():
    """The tensor-core schedule with a sequence whose context is empty (no
    visible block in any of its m-tiles, every CTA's window empty) beside one
    whose m-tiles split their columns: the empty one gets -1 everywhere."""
    cfg = SMALL.replace(B=2, S=256, ctx=3000, q_start=3000 - 256, topk=8)
    w = generate(cfg, with_kv=False)
    w["ctx_len"] = torch.tensor([3000, 0], dtype=torch.int32)
    w["q_start"] = torch.tensor([3000 - 256, 0], dtype=torch.int32)
    d = upload(w)
    ids = lci.index_select(d["q_c"], d["k_c"], cfg.bs, d["ctx_len"], d["q_start"], cfg.topk,
                           phase="prefill")
    torch.cuda.synchronize()
    lci.get_device_status()
    ref = oracle.index_select(w["q_c"], w["k_c"], cfg.bs, w["ctx_len"], w["q_start"], cfg.topk)
    got = ids.cpu().reshape(-1, cfg.topk)
    assert torch.equal(got, ref)
    assert (got[cfg.S:] == -1).all()
