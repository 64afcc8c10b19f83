"""CPU oracle of the sparse-attention index pipeline (test infrastructure).

Only the tests, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline leg
use this package. It loads ``liblci_oracle.so`` (plain C, fp64, built from
``lci_oracle.c`` by :func:`build`) and marshals torch CPU tensors into it. It
shares no code with the CUDA library and never imports it.

Every function takes the workload's raw bytes (fp32 or bf16, widened exactly in
C) and returns float64 / int32 torch tensors.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional, Sequence

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "lci_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liblci_oracle.so")
_lib = None

_F32, _BF16, _F64 = 0, 1, 2
_ERRORS = {1: "bad argument", 2: "block id or page out of range", 3: "out of memory"}


def build(force: bool = False) -> str:
    """Compile lci_oracle.c with gcc (-O2 -fopenmp, no fast-math) into the package."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared", "-Wall", "-Wextra",
               "-o", _LIB_PATH, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        # LCI_ORACLE_LIB names a deliberately broken build of this oracle; only
        # the mutation test sets it, to show that the pins catch such slips.
        path = os.environ.get("LCI_ORACLE_LIB")
        if not path:
            path = build()
        lib = ctypes.CDLL(path)
        i64, vp = ctypes.c_int64, ctypes.c_void_p
        lib.orc_block_compress.argtypes = [vp, ctypes.c_int, i64, i64, i64, i64, i64, vp]
        lib.orc_block_scores.argtypes = [vp, vp, ctypes.c_int, i64, i64, i64, i64, i64, i64,
                                         vp, vp, vp, i64, vp]
        lib.orc_index_select.argtypes = [vp, vp, ctypes.c_int, i64, i64, i64, i64, i64, i64,
                                         vp, vp, i64, vp, i64, vp]
        attn = [vp, vp, vp, ctypes.c_int, i64, i64, i64, i64, i64, i64, i64, vp, i64, vp, i64,
                vp, vp, ctypes.c_double, vp, i64, vp]
        lib.orc_sparse_attn.argtypes = attn
        lib.orc_dense_masked.argtypes = attn
        for f in (lib.orc_block_compress, lib.orc_block_scores, lib.orc_index_select,
                  lib.orc_sparse_attn, lib.orc_dense_masked):
            f.restype = ctypes.c_int
        lib.orc_gated_state_scan.argtypes = [vp, vp, vp, ctypes.c_int, vp, vp, i64, i64, i64,
                                             i64, i64, i64, vp]
        lib.orc_gated_state_scan.restype = ctypes.c_int
        lib.orc_num_threads.restype = ctypes.c_int
        lib.orc_set_num_threads.argtypes = [ctypes.c_int]
        _lib = lib
    return _lib


def num_threads() -> int:
    return _load().orc_num_threads()


def set_num_threads(n: int) -> None:
    _load().orc_set_num_threads(int(n))


def _dt(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return _F32
    if t.dtype == torch.bfloat16:
        return _BF16
    if t.dtype == torch.float64:
        return _F64
    raise TypeError(f"oracle: unsupported dtype {t.dtype}")


def _cpu(t: torch.Tensor) -> torch.Tensor:
    t = t.detach()
    if t.device.type != "cpu":
        t = t.cpu()
    return t.contiguous()


def _i32(t) -> torch.Tensor:
    return _cpu(torch.as_tensor(t)).to(torch.int32).contiguous()


def _rows(rows: Optional[Sequence[int]], total: int):
    if rows is None:
        return None, total
    r = torch.as_tensor(list(rows) if not isinstance(rows, torch.Tensor) else rows,
                        dtype=torch.int64).contiguous()
    return r, r.numel()


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _check(rc: int, what: str) -> None:
    if rc != 0:
        raise ValueError(f"oracle {what}: {_ERRORS.get(rc, rc)}")


def block_compress(k_idx: torch.Tensor, bs: int) -> torch.Tensor:
    """A0: mean of the per-token indexer keys of each block. [B,T,H,D] -> [B,NB,H,D] fp64."""
    k_idx = _cpu(k_idx)
    B, T, H, D = k_idx.shape
    NB = (T + bs - 1) // bs
    out = torch.empty((B, NB, H, D), dtype=torch.float64)
    _check(_load().orc_block_compress(_ptr(k_idx), _dt(k_idx), B, T, H, D, bs, _ptr(out)),
           "block_compress")
    return out


def block_scores(q_c, k_c, bs, ctx_len, q_start, rows=None) -> torch.Tensor:
    """A1: scores [nrows, NB] fp64, -inf for blocks that are not causal-visible."""
    q_c, k_c = _cpu(q_c), _cpu(k_c)
    if q_c.dtype != k_c.dtype:
        raise TypeError("oracle: q_c and k_c must share a dtype")
    B, S, H, D = q_c.shape
    NB = k_c.shape[1]
    ctx_len, q_start = _i32(ctx_len), _i32(q_start)
    r, n = _rows(rows, B * S)
    out = torch.empty((n, NB), dtype=torch.float64)
    _check(_load().orc_block_scores(_ptr(q_c), _ptr(k_c), _dt(q_c), B, S, H, D, NB, bs,
                                    _ptr(ctx_len), _ptr(q_start), _ptr(r), n, _ptr(out)),
           "block_scores")
    return out


def index_select(q_c, k_c, bs, ctx_len, q_start, topk, rows=None) -> torch.Tensor:
    """A1+A2: ids [nrows, topk] int32 in rank order, -1 padded."""
    q_c, k_c = _cpu(q_c), _cpu(k_c)
    if q_c.dtype != k_c.dtype:
        raise TypeError("oracle: q_c and k_c must share a dtype")
    B, S, H, D = q_c.shape
    NB = k_c.shape[1]
    ctx_len, q_start = _i32(ctx_len), _i32(q_start)
    r, n = _rows(rows, B * S)
    ids = torch.empty((n, topk), dtype=torch.int32)
    _check(_load().orc_index_select(_ptr(q_c), _ptr(k_c), _dt(q_c), B, S, H, D, NB, bs,
                                    _ptr(ctx_len), _ptr(q_start), topk, _ptr(r), n, _ptr(ids)),
           "index_select")
    return ids


def _attn(fn, q, k_pool, v_pool, block_table, ids, ctx_len, q_start, scale, rows):
    q, k_pool, v_pool = _cpu(q), _cpu(k_pool), _cpu(v_pool)
    if not (q.dtype == k_pool.dtype == v_pool.dtype):
        raise TypeError("oracle: q, k_pool and v_pool must share a dtype")
    B, S, H_q, hd = q.shape
    P, H_kv, bs, hd2 = k_pool.shape
    if hd2 != hd or tuple(v_pool.shape) != tuple(k_pool.shape):
        raise ValueError("oracle: pool shape mismatch")
    block_table = _i32(block_table)
    NB = block_table.shape[1]
    r, n = _rows(rows, B * S)
    ids = _i32(ids).reshape(n, -1).contiguous()
    topk = ids.shape[1]
    ctx_len, q_start = _i32(ctx_len), _i32(q_start)
    out = torch.empty((n, H_q, hd), dtype=torch.float64)
    rc = fn(_ptr(q), _ptr(k_pool), _ptr(v_pool), _dt(q), B, S, H_q, H_kv, hd, P, bs,
            _ptr(block_table), NB, _ptr(ids), topk, _ptr(ctx_len), _ptr(q_start),
            float(scale), _ptr(r), n, _ptr(out))
    _check(rc, "attention")
    return out


def sparse_attn(q, k_pool, v_pool, block_table, ids, ctx_len, q_start, scale, rows=None):
    """A3+A4: exact softmax attention over the selected blocks' tokens. [nrows,H_q,hd] fp64.

    ``ids`` holds one row per requested query row ([nrows, topk] or [B,S,topk]
    when ``rows`` is None).
    """
    return _attn(_load().orc_sparse_attn, q, k_pool, v_pool, block_table, ids, ctx_len,
                 q_start, scale, rows)


def dense_masked(q, k_pool, v_pool, block_table, ids, ctx_len, q_start, scale, rows=None):
    """Full causal attention with non-selected positions masked to -inf. [nrows,H_q,hd] fp64."""
    return _attn(_load().orc_dense_masked, q, k_pool, v_pool, block_table, ids, ctx_len,
                 q_start, scale, rows)


def gated_state_scan(q, k, v, gate, state, C):
    """N4: chunked gated state scan. q, k [B,T,H,dk], v [B,T,H,dv], gate
    [B,H,nchunks], state [B,H,dk,dv]. Returns (out [B,T,H,dv], final state)
    in fp64; the input state is not modified."""
    q, k, v = _cpu(q), _cpu(k), _cpu(v)
    if not (q.dtype == k.dtype == v.dtype):
        raise TypeError("oracle: q, k and v must share a dtype")
    B, T, H, dk = q.shape
    dv = v.shape[3]
    if tuple(k.shape) != (B, T, H, dk) or tuple(v.shape[:3]) != (B, T, H):
        raise ValueError("oracle: q, k, v shapes disagree")
    nchunks = (T + C - 1) // C
    gate = _cpu(gate).to(torch.float64).contiguous()
    if tuple(gate.shape) != (B, H, nchunks):
        raise ValueError("oracle: gate must be [B, H, nchunks]")
    st = _cpu(state).to(torch.float64).clone().contiguous()
    if tuple(st.shape) != (B, H, dk, dv):
        raise ValueError("oracle: state must be [B, H, dk, dv]")
    out = torch.empty((B, T, H, dv), dtype=torch.float64)
    _check(_load().orc_gated_state_scan(_ptr(q), _ptr(k), _ptr(v), _dt(q), _ptr(gate), _ptr(st),
                                        B, T, H, dk, dv, C, _ptr(out)), "gated_state_scan")
    return out, st
