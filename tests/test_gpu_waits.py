"""Bounded device waits (GPU): a wait that runs out is reported as
LCI_ERR_TIMEOUT, the kernel returns, and the context stays usable.

The pipelined attention entry point starts each query row when the caller's
producer publishes it. Here nothing ever publishes (the flags stay zero) and the
wait limit is 1 ms: every row must give up, produce a zero row, and the status
must read LCI_ERR_TIMEOUT. No GPU fault is involved: the wait is a polling loop
with a time limit, and the kernel skips its loads for a row that never came.
"""
import pytest
import torch

import long_context_indexer_b200 as lci
from long_context_indexer_b200.workloads import CONFIGS, generate
from tests.gpu_common import run_gpu, upload

pytestmark = pytest.mark.gpu

LCI_ERR_TIMEOUT = 6
SMALL = CONFIGS["decode"].replace(name="small", B=3, S=1, ctx=1000, q_start=999, bs=64, topk=4,
                                  H_q=8, H_kv=2, hd=128, H_i=2, d_c=64, spare_pages=5)


def test_pipelined_attention_with_published_rows_matches_sparse_attn():
    cfg = SMALL.replace(S=5, q_start=995)
    d = upload(generate(cfg))
    _, ids, out = run_gpu(cfg, d)
    bt = lci.create_block_table(d["block_table"], d["k_pool"])
    ready = torch.ones((cfg.B, cfg.S), dtype=torch.int32, device="cuda")
    got = lci.sparse_attn_pipelined(d["q"], d["k_pool"], d["v_pool"], bt, ids, d["ctx_len"],
                                    d["q_start"], ready)
    torch.cuda.synchronize()
    lci.get_device_status()
    assert torch.equal(got, out)


def test_unpublished_rows_time_out_and_report_timeout():
    cfg = SMALL.replace(S=2, q_start=998)
    d = upload(generate(cfg))
    _, ids, out_ref = run_gpu(cfg, d)
    bt = lci.create_block_table(d["block_table"], d["k_pool"])
    ready = torch.zeros((cfg.B, cfg.S), dtype=torch.int32, device="cuda")
    ready[1, 0] = 1  # one row is published, the others never are
    default = lci.get_wait_limit_ns()
    assert default == 2_000_000_000
    lci.set_wait_limit_ns(1_000_000)  # 1 ms
    try:
        assert lci.get_wait_limit_ns() == 1_000_000
        out = torch.full_like(d["q"], 7.0)
        lci.sparse_attn_pipelined(d["q"], d["k_pool"], d["v_pool"], bt, ids, d["ctx_len"],
                                  d["q_start"], ready, out=out)
        with pytest.raises(lci.LciError) as e:
            lci.get_device_status()
        assert e.value.status == LCI_ERR_TIMEOUT
        assert "timed out" in str(e.value)
        lci.get_device_status()  # the sticky word was cleared
    finally:
        lci.set_wait_limit_ns(default)
    # rows whose flag never came are zero; the published row is attended
    assert (out[0] == 0).all() and (out[2] == 0).all() and (out[1, 1] == 0).all()
    assert torch.equal(out[1, 0], out_ref[1, 0])
    # the context is still usable: a plain call gives the usual result
    _, ids2, out2 = run_gpu(cfg, d)
    assert torch.equal(ids2, ids) and torch.equal(out2, out_ref)


def test_two_kernel_decode_after_a_timed_out_consumer():
    """After a consumer gave up, the two-kernel form of the one-call decode
    step (block keys of 512 features, which the one-launch kernel does not
    take) on a workspace whose flags were left set still waits for this call's
    own publications."""
    cfg = CONFIGS["decode"].replace(H_i=4)
    d = upload(generate(cfg))
    _, ids_ref, out_ref = run_gpu(cfg, d)
    bt = lci.create_block_table(d["block_table"], d["k_pool"])
    need = lci.sparse_decode_workspace_size(cfg.B, cfg.S, cfg.H_i, cfg.d_c, cfg.topk, cfg.H_q, bt)
    ws = torch.zeros(need, dtype=torch.uint8, device="cuda")
    # Every publication flag left set, as after a consumer that gave up while
    # its producer published late. The arrival counters (the first 256 bytes,
    # one per row) are the only part that must start at zero; the rest of the
    # scratch is overwritten by every call.
    ws.fill_(1)
    ws[:256].zero_()
    for _ in range(2):
        ids = torch.full_like(ids_ref, -1)
        ids, out = lci.sparse_decode(d["q_c"], d["k_c"], d["ctx_len"], d["q_start"], cfg.topk,
                                     d["q"], d["k_pool"], d["v_pool"], bt, ids=ids, ws=ws)
        torch.cuda.synchronize()
        lci.get_device_status()
        assert torch.equal(ids, ids_ref)
        assert torch.equal(out, out_ref)
