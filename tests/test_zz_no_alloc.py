"""lci_index_select_noalloc against lci_index_select (GPU).

The allocation-free entry point is for callers that may not allocate device
memory or keep a workspace of their own (code inside a host framework that owns
every device allocation). It must return exactly the block ids of the regular
entry point, call after call, even though every call reuses the same built-in
scratch array, which keeps the previous call's contents. This file sorts last
so that a run stopping at the first failure has already run every other test.
"""
import ctypes
import os
import re

import pytest
import torch

from long_context_indexer_b200 import lci
from long_context_indexer_b200.workloads import CONFIGS, generate

pytestmark = pytest.mark.gpu

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include",
                      "lci.h")


def _scratch_limit():
    """LCI_NOALLOC_SCRATCH_BYTES as the public header defines it."""
    m = re.search(r"#define\s+LCI_NOALLOC_SCRATCH_BYTES\s+\((\d+)u\s*<<\s*(\d+)\)",
                  open(HEADER).read())
    assert m, "LCI_NOALLOC_SCRATCH_BYTES not found in the header"
    return int(m.group(1)) << int(m.group(2))


NOALLOC_BYTES = _scratch_limit()


def _inputs(cfg):
    w = generate(cfg, with_kv=False)
    return {k: v.cuda() for k, v in w.items()}


def _both(cfg):
    d = _inputs(cfg)
    ref = lci.index_select(d["q_c"], d["k_c"], cfg.bs, d["ctx_len"], d["q_start"], cfg.topk)
    got = torch.full_like(ref, -7)
    status = lci.load_library().lci_index_select_noalloc(
        ctypes.c_void_p(d["q_c"].data_ptr()), ctypes.c_void_p(d["k_c"].data_ptr()), lci.LCI_BF16,
        cfg.B, cfg.S, cfg.H_i, cfg.d_c, cfg.bs, cfg.NB, ctypes.c_void_p(d["ctx_len"].data_ptr()),
        ctypes.c_void_p(d["q_start"].data_ptr()), cfg.topk, 0, ctypes.c_void_p(got.data_ptr()),
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert status == 0, lci.load_library().lci_last_error()
    torch.cuda.synchronize()
    lci.get_device_status()
    return ref, got


def test_noalloc_matches_workspace_entry_point_on_consecutive_calls():
    first = CONFIGS["decode"]                                   # 32 rows x 512 blocks
    second = CONFIGS["decode"].replace(B=5, S=40, ctx=5000, q_start=4900, topk=12,
                                       spare_pages=0)           # 200 rows x 79 blocks
    for cfg in (first, second, first):
        ref, got = _both(cfg)
        assert torch.equal(got, ref), cfg
        assert (got >= 0).any()


def test_noalloc_binding_with_prefill_phase_matches_tensor_core_schedule():
    """The Python wrapper, with phase='prefill' on a shape the tensor-core
    schedule takes: the allocation-free call runs the row-wise kernel and must
    still give the tensor-core schedule's block ids."""
    cfg = CONFIGS["prefill"].replace(S=512, ctx=4096, q_start=4096 - 512, topk=32)
    d = _inputs(cfg)
    ref = lci.index_select(d["q_c"], d["k_c"], cfg.bs, d["ctx_len"], d["q_start"], cfg.topk,
                           phase="prefill")
    for _ in range(2):
        got = lci.index_select_noalloc(d["q_c"], d["k_c"], cfg.bs, d["ctx_len"], d["q_start"],
                                       cfg.topk, phase="prefill")
        torch.cuda.synchronize()
        lci.get_device_status()
        assert torch.equal(got, ref)
    with pytest.raises(ValueError):  # the wrapper checks dtypes before any call
        lci.index_select_noalloc(d["q_c"], d["k_c"].float(), cfg.bs, d["ctx_len"], d["q_start"],
                                 cfg.topk)


def test_noalloc_accepts_every_size_within_its_scratch():
    """The largest batch whose decode-schedule workspace fits the built-in
    scratch is accepted; that workspace size bounds what the call needs."""
    # narrow block keys (H_i*d_c = 8) keep the inputs small next to the scratch
    cfg = CONFIGS["decode"].replace(H_i=1, d_c=8)
    B = 1
    while lci.index_select_workspace_size(B + 1, 1, cfg.H_i, cfg.d_c, cfg.NB, cfg.topk,
                                          "decode") <= NOALLOC_BYTES:
        B += 1
    big = cfg.replace(B=B, spare_pages=0)
    ref, got = _both(big)
    assert torch.equal(got, ref)


def test_noalloc_rejects_sizes_beyond_its_scratch():
    cfg = CONFIGS["prefill"].replace(S=4096, ctx=1 << 20, q_start=(1 << 20) - 4096, bs=128,
                                     topk=16)  # 4096 rows x 8192 blocks: 128 MiB of scores
    lib = lci.load_library()
    fake = ctypes.c_void_p(0x7F0000000000)
    rc = lib.lci_index_select_noalloc(fake, fake, lci.LCI_BF16, cfg.B, cfg.S, cfg.H_i, cfg.d_c,
                                      cfg.bs, cfg.NB, fake, fake, cfg.topk, 0, fake, None)
    assert rc == 3  # LCI_ERR_WORKSPACE, returned before anything is launched
    assert b"scratch" in lib.lci_last_error()
    assert cfg.B * cfg.S * cfg.NB * 4 > NOALLOC_BYTES
