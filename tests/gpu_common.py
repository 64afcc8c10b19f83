"""Shared helpers of the GPU parity tests: run the CUDA path through the C ABI
and the oracle on the same seeded CPU bytes."""
from __future__ import annotations

import math

import torch

import long_context_indexer_b200 as lci
import oracle

TOL = {torch.float32: 1e-4, torch.bfloat16: 2e-2}


def upload(w):
    return {k: v.cuda() for k, v in w.items()}


def run_gpu(cfg, d, phase="auto", topk=None, scale=0.0):
    """index_select + sparse_attn on device tensors d; returns (k_c, ids, out)."""
    topk = cfg.topk if topk is None else topk
    k_c = lci.block_compress(d["k_idx"], cfg.bs) if "k_idx" in d else d["k_c"]
    ids = lci.index_select(d["q_c"], k_c, cfg.bs, d["ctx_len"], d["q_start"], topk, phase=phase)
    bt = lci.create_block_table(d["block_table"], d["k_pool"])
    out = lci.sparse_attn(d["q"], d["k_pool"], d["v_pool"], bt, ids, d["ctx_len"], d["q_start"],
                          scale=scale, phase=phase)
    torch.cuda.synchronize()
    lci.get_device_status()
    return k_c, ids, out


def oracle_k_c(cfg, w):
    """The oracle's k_c in the workload dtype (exact for grid inputs and bs a power of 2)."""
    if "k_idx" in w:
        return oracle.block_compress(w["k_idx"], cfg.bs).to(cfg.torch_dtype)
    return w["k_c"]


def oracle_rows(cfg, w, rows=None, topk=None, scale=None):
    """Oracle ids [n, topk] and out [n, H_q, hd] (fp64) for the given flat rows."""
    topk = cfg.topk if topk is None else topk
    scale = 1.0 / math.sqrt(cfg.hd) if scale is None else scale
    k_c = oracle_k_c(cfg, w)
    ids = oracle.index_select(w["q_c"], k_c, cfg.bs, w["ctx_len"], w["q_start"], topk, rows=rows)
    out = oracle.sparse_attn(w["q"], w["k_pool"], w["v_pool"], w["block_table"], ids,
                             w["ctx_len"], w["q_start"], scale, rows=rows)
    return ids, out


def assert_out_close(got, ref, dtype, what=""):
    got = got.double().cpu()
    assert torch.isfinite(got).all(), f"{what}: non-finite output"
    err = (got - ref).abs().max().item()
    assert err <= TOL[dtype], f"{what}: max-abs error {err:.3e} above {TOL[dtype]:.0e}"
    return err
