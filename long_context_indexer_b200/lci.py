"""Thin Python binding of liblci.so (include/lci.h).

Argument marshalling only: every function checks the torch tensors it is given
(device, dtype, contiguity, shapes), takes their device pointers and the
current CUDA stream, and calls the C entry point of the same name. Outputs and
workspaces are torch allocations; the computation runs entirely in the
library's CUDA kernels. There is no fallback: if liblci.so is missing or fails
to load, every call raises.
"""
from __future__ import annotations

import ctypes
import os
import threading
from typing import Dict, Optional, Tuple

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "liblci.so")

LCI_OK = 0
STATUS_NAMES = {0: "LCI_OK", 1: "LCI_ERR_INVALID_ARG", 2: "LCI_ERR_UNSUPPORTED",
                3: "LCI_ERR_WORKSPACE", 4: "LCI_ERR_CUDA", 5: "LCI_ERR_DEVICE_BOUNDS",
                6: "LCI_ERR_TIMEOUT"}
LCI_F32, LCI_BF16 = 0, 1
PHASES = {"auto": 0, "prefill": 1, "decode": 2}

# Every entry point of include/lci.h: name -> (restype, argtypes)
_vp, _i32, _sz, _f32 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_size_t, ctypes.c_float
_st = ctypes.c_int
SIGNATURES = {
    "lci_version": (ctypes.c_char_p, []),
    "lci_status_string": (ctypes.c_char_p, [_st]),
    "lci_last_error": (ctypes.c_char_p, []),
    "lci_create_block_table": (_st, [_vp, _i32, _i32, _i32, _i32, _i32, _i32, _st,
                                     ctypes.POINTER(_vp)]),
    "lci_destroy_block_table": (_st, [_vp]),
    "lci_validate_block_table": (_st, [_vp, _vp]),
    "lci_block_compress": (_st, [_vp, _st, _i32, _i32, _i32, _i32, _i32, _vp, _vp]),
    "lci_index_select_workspace_size": (_st, [_i32, _i32, _i32, _i32, _i32, _i32, _st,
                                              ctypes.POINTER(_sz)]),
    "lci_index_select": (_st, [_vp, _vp, _st, _i32, _i32, _i32, _i32, _i32, _i32, _vp, _vp, _i32,
                               _st, _vp, _vp, _sz, _vp]),
    "lci_sparse_attn_workspace_size": (_st, [_i32, _i32, _i32, _i32, _vp, _st,
                                             ctypes.POINTER(_sz)]),
    "lci_sparse_attn": (_st, [_vp, _i32, _i32, _i32, _vp, _vp, _vp, _vp, _i32, _vp, _vp, _f32,
                              _st, _vp, _vp, _sz, _vp]),
    "lci_get_device_status": (_st, [_vp]),
    "lci_sparse_decode_workspace_size": (_st, [_i32, _i32, _i32, _i32, _i32, _i32, _vp,
                                               ctypes.POINTER(_sz)]),
    "lci_sparse_decode": (_st, [_vp, _vp, _st, _i32, _i32, _i32, _i32, _i32, _vp, _vp, _i32, _vp,
                                _i32, _vp, _vp, _vp, _f32, _vp, _vp, _vp, _sz, _vp]),
    "lci_index_select_noalloc": (_st, [_vp, _vp, _st, _i32, _i32, _i32, _i32, _i32, _i32, _vp, _vp,
                                       _i32, _st, _vp, _vp]),
    "lci_sparse_attn_pipelined": (_st, [_vp, _i32, _i32, _i32, _vp, _vp, _vp, _vp, _i32, _vp, _vp,
                                        _f32, _vp, _vp, _vp]),
    "lci_set_wait_limit_ns": (_st, [ctypes.c_uint64]),
    "lci_sparse_decode_persistent": (_st, [_vp, _vp, _st, _i32, _i32, _i32, _i32, _i32, _vp, _vp,
                                           _i32, _vp, _i32, _vp, _vp, _vp, _f32, _vp, _vp, _vp,
                                           _sz, _vp]),
    "lci_gated_state_scan": (_st, [_vp, _vp, _vp, _st, _vp, _vp, _vp, _i32, _i32, _i32, _i32, _i32,
                                   _i32, _vp, _vp]),
    "lci_block_scores_at": (_st, [_vp, _vp, _st, _i32, _i32, _i32, _i32, _i32, _vp, _i32, _vp,
                                  _vp]),
    "lci_ids_shift": (_st, [_vp, ctypes.c_int64, _i32, _i32, _i32, _vp, _vp]),
    "lci_topk_merge": (_st, [_vp, _vp, _i32, ctypes.c_int64, _i32, _vp, _vp]),
    "lci_sparse_attn_partial": (_st, [_vp, _i32, _i32, _i32, _vp, _vp, _vp, _vp, _i32, _vp, _vp,
                                      _f32, _st, _vp, _vp, _vp]),
    "lci_attn_merge": (_st, [_vp, _vp, _st, _i32, ctypes.c_int64, _i32, _vp, _vp]),
    "lci_kc_update": (_st, [_vp, _st, _i32, _i32, _i32, _i32, _vp, _vp, _vp, _vp, _vp]),
    "lci_index_select_paged_workspace_size": (_st, [_i32, _i32, _i32, _i32, _i32, _vp, _st, _st,
                                                    ctypes.POINTER(_sz)]),
    "lci_index_select_paged": (_st, [_vp, _vp, _st, _i32, _i32, _i32, _i32, _vp, _vp, _vp, _i32,
                                     _st, _vp, _vp, _sz, _vp]),
    "lci_get_wait_limit_ns": (_st, [ctypes.POINTER(ctypes.c_uint64)]),
}

_lib = None
_lock = threading.Lock()


class LciError(RuntimeError):
    def __init__(self, status: int, where: str, message: str):
        self.status = status
        super().__init__(f"{where}: {STATUS_NAMES.get(status, status)}: {message}")


def load_library() -> ctypes.CDLL:
    """Load liblci.so (built by long_context_indexer_b200.build); raise if absent."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise RuntimeError(f"liblci.so not found at {LIB_PATH}; build it with "
                                   "`python -m long_context_indexer_b200.build`")
            lib = ctypes.CDLL(LIB_PATH)
            for name, (res, args) in SIGNATURES.items():
                fn = getattr(lib, name)
                fn.restype = res
                fn.argtypes = args
            _lib = lib
    return _lib


def _check(status: int, where: str) -> None:
    if status != LCI_OK:
        msg = load_library().lci_last_error().decode(errors="replace")
        raise LciError(status, where, msg)


def version() -> str:
    return load_library().lci_version().decode()


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return LCI_F32
    if t.dtype == torch.bfloat16:
        return LCI_BF16
    raise TypeError(f"lci: unsupported dtype {t.dtype} (float32 or bfloat16)")


def _dev(t: torch.Tensor, name: str, dtype: Optional[torch.dtype] = None, ndim: Optional[int] = None):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"lci: {name} must be a torch.Tensor")
    if t.device.type != "cuda":
        raise ValueError(f"lci: {name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"lci: {name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"lci: {name} must be {dtype}, got {t.dtype}")
    if ndim is not None and t.dim() != ndim:
        raise ValueError(f"lci: {name} must have {ndim} dims, got {t.dim()}")
    return ctypes.c_void_p(t.data_ptr())


# ---------------------------------------------------------------- workspaces

_ws: Dict[Tuple[int, str], torch.Tensor] = {}


def workspace(device: torch.device, nbytes: int, tag: str) -> torch.Tensor:
    """A zero-initialised, 256-byte aligned device buffer of at least nbytes.

    Workspaces hold arrival counters that the library leaves at zero after
    every call, but only in the layout of the shape they were used with. So a
    cached buffer is keyed by ``tag``, which callers make unique per layout
    (entry point and the sizes the layout depends on), and is zero-filled once
    when first allocated.
    """
    key = (torch.device(device).index or 0, tag)
    buf = _ws.get(key)
    if buf is None or buf.numel() < nbytes:
        buf = torch.zeros(max(nbytes, 256), dtype=torch.uint8, device=device)
        _ws[key] = buf
    return buf


# ---------------------------------------------------------------- block table

class BlockTable:
    """Owns an lci_block_table handle; keeps the table tensor alive."""

    def __init__(self, table: torch.Tensor, num_pages: int, block_size: int, num_kv_heads: int,
                 head_dim: int, dtype: torch.dtype):
        ptr = _dev(table, "block_table", torch.int32, 2)
        self.table = table
        self.batch, self.max_blocks = table.shape
        self.num_pages, self.block_size = int(num_pages), int(block_size)
        self.num_kv_heads, self.head_dim = int(num_kv_heads), int(head_dim)
        self.dtype = dtype
        handle = ctypes.c_void_p()
        lib = load_library()
        _check(lib.lci_create_block_table(ptr, self.batch, self.max_blocks, self.num_pages,
                                          self.block_size, self.num_kv_heads, self.head_dim,
                                          _dtype_code(torch.empty(0, dtype=dtype)),
                                          ctypes.byref(handle)), "lci_create_block_table")
        self._handle = handle
        self._lib = lib

    @property
    def handle(self) -> ctypes.c_void_p:
        return self._handle

    def validate(self, stream=None) -> None:
        _check(self._lib.lci_validate_block_table(self._handle, _stream(stream)),
               "lci_validate_block_table")

    def close(self) -> None:
        if getattr(self, "_handle", None):
            self._lib.lci_destroy_block_table(self._handle)
            self._handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def create_block_table(table: torch.Tensor, k_pool: torch.Tensor) -> BlockTable:
    """Block table over pools shaped [num_pages, H_kv, block_size, head_dim]."""
    P, H_kv, bs, hd = k_pool.shape
    return BlockTable(table, P, bs, H_kv, hd, k_pool.dtype)


# ---------------------------------------------------------------- entry points

def block_compress(k_idx: torch.Tensor, block_size: int, out: Optional[torch.Tensor] = None,
                   stream=None) -> torch.Tensor:
    """A0: [B, T, H, D] per-token indexer keys -> [B, ceil(T/bs), H, D] block means."""
    B, T, H, D = k_idx.shape
    NB = (T + block_size - 1) // block_size
    if out is None:
        out = torch.empty((B, NB, H, D), dtype=k_idx.dtype, device=k_idx.device)
    _check(load_library().lci_block_compress(_dev(k_idx, "k_idx", None, 4), _dtype_code(k_idx), B, T,
                                             H, D, block_size, _dev(out, "out", k_idx.dtype, 4),
                                             _stream(stream)), "lci_block_compress")
    return out


def index_select_workspace_size(B, S, H_i, d_c, nb_max, topk, phase="auto") -> int:
    n = ctypes.c_size_t()
    _check(load_library().lci_index_select_workspace_size(B, S, H_i, d_c, nb_max, topk,
                                                          PHASES[phase], ctypes.byref(n)),
           "lci_index_select_workspace_size")
    return n.value


def index_select(q_c: torch.Tensor, k_c: torch.Tensor, block_size: int, ctx_len: torch.Tensor,
                 q_start: torch.Tensor, topk: int, phase: str = "auto",
                 ids: Optional[torch.Tensor] = None, ws: Optional[torch.Tensor] = None,
                 stream=None) -> torch.Tensor:
    """A1+A2: ids [B, S, topk] int32, ranked (score desc, id asc), -1 padded."""
    B, S, H_i, d_c = q_c.shape
    nb_max = k_c.shape[1]
    if k_c.shape[0] != B or k_c.shape[2:] != q_c.shape[2:] or k_c.dtype != q_c.dtype:
        raise ValueError("lci: k_c must be [B, nb_max, H_i, d_c] with q_c's dtype")
    if ids is None:
        ids = torch.empty((B, S, topk), dtype=torch.int32, device=q_c.device)
    need = index_select_workspace_size(B, S, H_i, d_c, nb_max, topk, phase)
    if ws is None:
        ws = workspace(q_c.device, need, f"index_select:{B}x{S}x{nb_max}:{H_i * d_c}")
    _check(load_library().lci_index_select(
        _dev(q_c, "q_c", None, 4), _dev(k_c, "k_c", q_c.dtype, 4), _dtype_code(q_c), B, S, H_i, d_c,
        block_size, nb_max, _dev(ctx_len, "ctx_len", torch.int32, 1),
        _dev(q_start, "q_start", torch.int32, 1), topk, PHASES[phase],
        _dev(ids, "ids", torch.int32, 3), _dev(ws, "workspace"), ws.numel() * ws.element_size(),
        _stream(stream)), "lci_index_select")
    return ids


def index_select_noalloc(q_c: torch.Tensor, k_c: torch.Tensor, block_size: int,
                         ctx_len: torch.Tensor, q_start: torch.Tensor, topk: int,
                         phase: str = "auto", ids: Optional[torch.Tensor] = None,
                         stream=None) -> torch.Tensor:
    """index_select through lci_index_select_noalloc: no workspace, no device
    allocation inside the library (its scratch is a fixed array in liblci.so)."""
    B, S, H_i, d_c = q_c.shape
    nb_max = k_c.shape[1]
    if k_c.shape[0] != B or k_c.shape[2:] != q_c.shape[2:] or k_c.dtype != q_c.dtype:
        raise ValueError("lci: k_c must be [B, nb_max, H_i, d_c] with q_c's dtype")
    if ids is None:
        ids = torch.empty((B, S, topk), dtype=torch.int32, device=q_c.device)
    _check(load_library().lci_index_select_noalloc(
        _dev(q_c, "q_c", None, 4), _dev(k_c, "k_c", q_c.dtype, 4), _dtype_code(q_c), B, S, H_i, d_c,
        block_size, nb_max, _dev(ctx_len, "ctx_len", torch.int32, 1),
        _dev(q_start, "q_start", torch.int32, 1), topk, PHASES[phase],
        _dev(ids, "ids", torch.int32, 3), _stream(stream)), "lci_index_select_noalloc")
    return ids


def sparse_attn_workspace_size(B, S, H_q, topk, table: BlockTable, phase="auto") -> int:
    n = ctypes.c_size_t()
    _check(load_library().lci_sparse_attn_workspace_size(B, S, H_q, topk, table.handle,
                                                         PHASES[phase], ctypes.byref(n)),
           "lci_sparse_attn_workspace_size")
    return n.value


def sparse_attn(q: torch.Tensor, k_pool: torch.Tensor, v_pool: torch.Tensor, table: BlockTable,
                ids: torch.Tensor, ctx_len: torch.Tensor, q_start: torch.Tensor,
                scale: float = 0.0, phase: str = "auto", out: Optional[torch.Tensor] = None,
                ws: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """A3+A4: exact softmax attention over the selected blocks. out [B, S, H_q, hd]."""
    B, S, H_q, hd = q.shape
    topk = ids.shape[-1]
    if tuple(ids.shape) != (B, S, topk):
        raise ValueError("lci: ids must be [B, S, topk]")
    if tuple(k_pool.shape) != (table.num_pages, table.num_kv_heads, table.block_size,
                               table.head_dim) or v_pool.shape != k_pool.shape:
        raise ValueError("lci: pools do not match the block table")
    if q.dtype != table.dtype or k_pool.dtype != q.dtype or v_pool.dtype != q.dtype:
        raise TypeError("lci: q and the pools must share the block table's dtype")
    if hd != table.head_dim:
        raise ValueError("lci: q's head_dim differs from the block table's")
    if out is None:
        out = torch.empty_like(q)
    need = sparse_attn_workspace_size(B, S, H_q, topk, table, phase)
    if ws is None:
        ws = workspace(q.device, need, f"sparse_attn:{B}x{S}x{H_q}x{topk}:{table.max_blocks}:"
                                       f"{table.num_kv_heads}x{table.block_size}")
    _check(load_library().lci_sparse_attn(
        _dev(q, "q", None, 4), B, S, H_q, _dev(k_pool, "k_pool"), _dev(v_pool, "v_pool"),
        table.handle, _dev(ids, "ids", torch.int32, 3), topk, _dev(ctx_len, "ctx_len", torch.int32, 1),
        _dev(q_start, "q_start", torch.int32, 1), float(scale), PHASES[phase],
        _dev(out, "out", q.dtype, 4), _dev(ws, "workspace"), ws.numel() * ws.element_size(),
        _stream(stream)), "lci_sparse_attn")
    return out


_decode_ws_sizes: Dict[Tuple[int, ...], int] = {}


def sparse_decode_workspace_size(B, S, H_i, d_c, topk, H_q, table: BlockTable) -> int:
    key = (B, S, H_i, d_c, topk, H_q, table.max_blocks, table.num_kv_heads, table.block_size,
           table.head_dim, str(table.dtype))
    n = _decode_ws_sizes.get(key)
    if n is None:
        c = ctypes.c_size_t()
        _check(load_library().lci_sparse_decode_workspace_size(B, S, H_i, d_c, topk, H_q,
                                                               table.handle, ctypes.byref(c)),
               "lci_sparse_decode_workspace_size")
        n = _decode_ws_sizes[key] = c.value
    return n


def sparse_decode(q_c: torch.Tensor, k_c: torch.Tensor, ctx_len: torch.Tensor,
                  q_start: torch.Tensor, topk: int, q: torch.Tensor, k_pool: torch.Tensor,
                  v_pool: torch.Tensor, table: BlockTable, scale: float = 0.0,
                  ids: Optional[torch.Tensor] = None, out: Optional[torch.Tensor] = None,
                  ws: Optional[torch.Tensor] = None, stream=None, persistent: bool = False):
    """index_select + sparse_attn in one call (rows attended as they are selected).

    Returns (ids [B, S, topk] int32, out [B, S, H_q, hd])."""
    B, S, H_i, d_c = q_c.shape
    nb_max = k_c.shape[1]
    H_q = q.shape[2]
    if tuple(q.shape[:2]) != (B, S):
        raise ValueError("lci: q must be [B, S, H_q, hd] with q_c's B and S")
    if tuple(k_pool.shape) != (table.num_pages, table.num_kv_heads, table.block_size,
                               table.head_dim) or v_pool.shape != k_pool.shape:
        raise ValueError("lci: pools do not match the block table")
    if ids is None:
        ids = torch.empty((B, S, topk), dtype=torch.int32, device=q_c.device)
    if out is None:
        out = torch.empty_like(q)
    need = sparse_decode_workspace_size(B, S, H_i, d_c, topk, H_q, table)
    if ws is None:
        ws = workspace(q_c.device, need, f"sparse_decode:{B}x{S}x{nb_max}:{H_i * d_c}:{topk}:"
                                         f"{H_q}x{table.num_kv_heads}x{table.block_size}")
    name = "lci_sparse_decode_persistent" if persistent else "lci_sparse_decode"
    _check(getattr(load_library(), name)(
        _dev(q_c, "q_c", None, 4), _dev(k_c, "k_c", q_c.dtype, 4), _dtype_code(q_c), B, S, H_i,
        d_c, nb_max, _dev(ctx_len, "ctx_len", torch.int32, 1),
        _dev(q_start, "q_start", torch.int32, 1), topk, _dev(q, "q", q_c.dtype, 4), H_q,
        _dev(k_pool, "k_pool", q_c.dtype), _dev(v_pool, "v_pool", q_c.dtype), table.handle,
        float(scale), _dev(ids, "ids", torch.int32, 3), _dev(out, "out", q_c.dtype, 4),
        _dev(ws, "workspace"), ws.numel() * ws.element_size(), _stream(stream)), name)
    return ids, out


class PagedKeys:
    """Block keys stored per page of a paged KV cache (one key per page), with
    the fp32 running sums the online producer extends."""

    def __init__(self, num_pages: int, H_i: int, d_c: int, dtype: torch.dtype, device):
        self.kc = torch.zeros((num_pages, H_i, d_c), dtype=dtype, device=device)
        self.kc_sum = torch.zeros((num_pages, H_i * d_c), dtype=torch.float32, device=device)

    def update(self, k_idx: torch.Tensor, start: torch.Tensor, table: BlockTable,
               stream=None) -> None:
        """Append k_idx [B, T, H_i, d_c] at positions start[b] .. start[b]+T-1."""
        B, T, H_i, d_c = k_idx.shape
        if k_idx.dtype != self.kc.dtype or tuple(self.kc.shape[1:]) != (H_i, d_c):
            raise ValueError("lci: k_idx must match the paged keys' dtype and [H_i, d_c]")
        if self.kc.shape[0] != table.num_pages:
            raise ValueError("lci: paged keys and block table differ in page count")
        _check(load_library().lci_kc_update(
            _dev(k_idx, "k_idx", None, 4), _dtype_code(k_idx), B, T, H_i, d_c,
            _dev(start, "start", torch.int32, 1), table.handle, _dev(self.kc_sum, "kc_sum"),
            _dev(self.kc, "kc"), _stream(stream)), "lci_kc_update")


def index_select_paged(q_c: torch.Tensor, keys: "PagedKeys", table: BlockTable,
                       ctx_len: torch.Tensor, q_start: torch.Tensor, topk: int,
                       phase: str = "auto", ids: Optional[torch.Tensor] = None,
                       ws: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """index_select with block keys read from the paged pool through the table."""
    B, S, H_i, d_c = q_c.shape
    kc = keys.kc if isinstance(keys, PagedKeys) else keys
    if kc.dtype != q_c.dtype or tuple(kc.shape[1:]) != (H_i, d_c):
        raise ValueError("lci: paged keys must be [num_pages, H_i, d_c] with q_c's dtype")
    if ids is None:
        ids = torch.empty((B, S, topk), dtype=torch.int32, device=q_c.device)
    lib = load_library()
    n = ctypes.c_size_t()
    _check(lib.lci_index_select_paged_workspace_size(B, S, H_i, d_c, topk, table.handle,
                                                     _dtype_code(q_c), PHASES[phase],
                                                     ctypes.byref(n)),
           "lci_index_select_paged_workspace_size")
    if ws is None:
        ws = workspace(q_c.device, n.value,
                       f"index_select_paged:{B}x{S}x{table.max_blocks}:{H_i * d_c}:{phase}")
    _check(lib.lci_index_select_paged(
        _dev(q_c, "q_c", None, 4), _dev(kc, "kc", q_c.dtype, 3), _dtype_code(q_c), B, S, H_i, d_c,
        table.handle, _dev(ctx_len, "ctx_len", torch.int32, 1),
        _dev(q_start, "q_start", torch.int32, 1), topk, PHASES[phase],
        _dev(ids, "ids", torch.int32, 3), _dev(ws, "workspace"), ws.numel() * ws.element_size(),
        _stream(stream)), "lci_index_select_paged")
    return ids


def block_scores_at(q_c: torch.Tensor, k_c: torch.Tensor, ids: torch.Tensor,
                    out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """scores [B, S, topk] fp32 of the given block ids (-inf for -1)."""
    B, S, H_i, d_c = q_c.shape
    topk = ids.shape[-1]
    if tuple(ids.shape) != (B, S, topk):
        raise ValueError("lci: ids must be [B, S, topk]")
    if out is None:
        out = torch.empty((B, S, topk), dtype=torch.float32, device=q_c.device)
    _check(load_library().lci_block_scores_at(
        _dev(q_c, "q_c", None, 4), _dev(k_c, "k_c", q_c.dtype, 4), _dtype_code(q_c), B, S, H_i, d_c,
        k_c.shape[1], _dev(ids, "ids", torch.int32, 3), topk, _dev(out, "scores", torch.float32, 3),
        _stream(stream)), "lci_block_scores_at")
    return out


def ids_shift(ids: torch.Tensor, lo: int, hi: int, offset: int,
              out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """(lo <= id < hi) ? id + offset : -1, elementwise."""
    if out is None:
        out = torch.empty_like(ids)
    _check(load_library().lci_ids_shift(_dev(ids, "ids", torch.int32), ids.numel(), int(lo),
                                        int(hi), int(offset), _dev(out, "out", torch.int32),
                                        _stream(stream)), "lci_ids_shift")
    return out


def topk_merge(scores: torch.Tensor, ids: torch.Tensor, out: Optional[torch.Tensor] = None,
               stream=None) -> torch.Tensor:
    """Merge [L, ..., topk] ranked lists into the top-k [..., topk] of their union."""
    L, topk = ids.shape[0], ids.shape[-1]
    if scores.shape != ids.shape:
        raise ValueError("lci: scores and ids must have the same shape")
    rows = ids[0].numel() // topk
    if out is None:
        out = torch.empty(ids.shape[1:], dtype=torch.int32, device=ids.device)
    _check(load_library().lci_topk_merge(_dev(scores, "scores", torch.float32),
                                         _dev(ids, "ids", torch.int32), L, rows, topk,
                                         _dev(out, "out", torch.int32), _stream(stream)),
           "lci_topk_merge")
    return out


def sparse_attn_partial(q: torch.Tensor, k_pool: torch.Tensor, v_pool: torch.Tensor,
                        table: BlockTable, ids: torch.Tensor, ctx_len: torch.Tensor,
                        q_start: torch.Tensor, scale: float = 0.0, phase: str = "auto",
                        out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
                        stream=None):
    """sparse_attn plus the base-2 log-sum-exp [B, S, H_q] of each row's logits."""
    B, S, H_q, hd = q.shape
    topk = ids.shape[-1]
    if tuple(ids.shape) != (B, S, topk):
        raise ValueError("lci: ids must be [B, S, topk]")
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, S, H_q), dtype=torch.float32, device=q.device)
    _check(load_library().lci_sparse_attn_partial(
        _dev(q, "q", table.dtype, 4), B, S, H_q, _dev(k_pool, "k_pool", table.dtype),
        _dev(v_pool, "v_pool", table.dtype), table.handle, _dev(ids, "ids", torch.int32, 3), topk,
        _dev(ctx_len, "ctx_len", torch.int32, 1), _dev(q_start, "q_start", torch.int32, 1),
        float(scale), PHASES[phase], _dev(out, "out", q.dtype, 4),
        _dev(lse, "lse", torch.float32, 3), _stream(stream)), "lci_sparse_attn_partial")
    return out, lse


def attn_merge(o: torch.Tensor, lse: torch.Tensor, out: Optional[torch.Tensor] = None,
               stream=None) -> torch.Tensor:
    """Combine partials o [L, ..., hd] with lse [L, ...] into out [..., hd]."""
    L, hd = o.shape[0], o.shape[-1]
    if tuple(lse.shape) != tuple(o.shape[:-1]):
        raise ValueError("lci: lse must be o's shape without the last dim")
    if out is None:
        out = torch.empty(o.shape[1:], dtype=o.dtype, device=o.device)
    _check(load_library().lci_attn_merge(_dev(o, "o", None), _dev(lse, "lse", torch.float32),
                                         _dtype_code(o), L, lse[0].numel(), hd,
                                         _dev(out, "out", o.dtype), _stream(stream)),
           "lci_attn_merge")
    return out


def gated_state_scan(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, gate: torch.Tensor,
                     state: torch.Tensor, chunk: int = 128, out: Optional[torch.Tensor] = None,
                     state_out: Optional[torch.Tensor] = None, stream=None):
    """N4: chunked gated state scan. q, k [B, T, H, dk], v [B, T, H, dv] (bf16),
    gate [B, H, ceil(T/chunk)] and state [B, H, dk, dv] (fp32). Returns
    (out [B, T, H, dv] fp32, final state); state_out=state updates in place."""
    B, T, H, dk = q.shape
    dv = v.shape[3]
    if tuple(k.shape) != (B, T, H, dk) or tuple(v.shape[:3]) != (B, T, H):
        raise ValueError("lci: q, k, v shapes disagree")
    if tuple(gate.shape) != (B, H, -(-T // chunk)) or tuple(state.shape) != (B, H, dk, dv):
        raise ValueError("lci: gate must be [B, H, nchunks] and state [B, H, dk, dv]")
    if out is None:
        out = torch.empty((B, T, H, dv), dtype=torch.float32, device=q.device)
    if state_out is None:
        state_out = torch.empty_like(state)
    _check(load_library().lci_gated_state_scan(
        _dev(q, "q", None, 4), _dev(k, "k", q.dtype, 4), _dev(v, "v", q.dtype, 4), _dtype_code(q),
        _dev(gate, "gate", torch.float32, 3), _dev(state, "state", torch.float32, 4),
        _dev(state_out, "state_out", torch.float32, 4), B, T, H, dk, dv, chunk,
        _dev(out, "out", torch.float32, 4), _stream(stream)), "lci_gated_state_scan")
    return out, state_out


def sparse_attn_pipelined(q: torch.Tensor, k_pool: torch.Tensor, v_pool: torch.Tensor,
                          table: BlockTable, ids: torch.Tensor, ctx_len: torch.Tensor,
                          q_start: torch.Tensor, ready: torch.Tensor, scale: float = 0.0,
                          out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """sparse_attn whose query rows each start once ready[row] (uint32 as int32,
    [B, S]) is published nonzero by the caller's producer."""
    B, S, H_q, hd = q.shape
    topk = ids.shape[-1]
    if tuple(ids.shape) != (B, S, topk) or tuple(ready.shape) != (B, S):
        raise ValueError("lci: ids must be [B, S, topk] and ready [B, S]")
    if tuple(k_pool.shape) != (table.num_pages, table.num_kv_heads, table.block_size,
                               table.head_dim) or v_pool.shape != k_pool.shape:
        raise ValueError("lci: pools do not match the block table")
    if out is None:
        out = torch.empty_like(q)
    _check(load_library().lci_sparse_attn_pipelined(
        _dev(q, "q", table.dtype, 4), B, S, H_q, _dev(k_pool, "k_pool", table.dtype),
        _dev(v_pool, "v_pool", table.dtype), table.handle, _dev(ids, "ids", torch.int32, 3), topk,
        _dev(ctx_len, "ctx_len", torch.int32, 1), _dev(q_start, "q_start", torch.int32, 1),
        float(scale), _dev(ready, "ready", torch.int32, 2), _dev(out, "out", q.dtype, 4),
        _stream(stream)), "lci_sparse_attn_pipelined")
    return out


def set_wait_limit_ns(ns: int) -> None:
    """Limit of every bounded device wait on the current device (nanoseconds)."""
    _check(load_library().lci_set_wait_limit_ns(int(ns)), "lci_set_wait_limit_ns")


def get_wait_limit_ns() -> int:
    v = ctypes.c_uint64()
    _check(load_library().lci_get_wait_limit_ns(ctypes.byref(v)), "lci_get_wait_limit_ns")
    return v.value


class SparseDecodeStep:
    """A decode step prepared once, for a loop that calls it every step: the
    tensors are checked and their device pointers taken here, the workspace is
    allocated, and each call makes only the lci_sparse_decode C call on the
    given stream (the caller updates the buffers' contents between calls, e.g.
    by copying the new tokens' queries into q_c and q)."""

    def __init__(self, q_c: torch.Tensor, k_c: torch.Tensor, ctx_len: torch.Tensor,
                 q_start: torch.Tensor, topk: int, q: torch.Tensor, k_pool: torch.Tensor,
                 v_pool: torch.Tensor, table: BlockTable, scale: float = 0.0,
                 ids: Optional[torch.Tensor] = None, out: Optional[torch.Tensor] = None,
                 ws: Optional[torch.Tensor] = None, stream=None, persistent: bool = False):
        B, S, H_i, d_c = q_c.shape
        nb_max = k_c.shape[1]
        H_q = q.shape[2]
        if tuple(q.shape[:2]) != (B, S):
            raise ValueError("lci: q must be [B, S, H_q, hd] with q_c's B and S")
        if tuple(k_pool.shape) != (table.num_pages, table.num_kv_heads, table.block_size,
                                   table.head_dim) or v_pool.shape != k_pool.shape:
            raise ValueError("lci: pools do not match the block table")
        self.ids = torch.empty((B, S, topk), dtype=torch.int32, device=q_c.device) \
            if ids is None else ids
        self.out = torch.empty_like(q) if out is None else out
        need = sparse_decode_workspace_size(B, S, H_i, d_c, topk, H_q, table)
        self.ws = torch.zeros(max(need, 256), dtype=torch.uint8, device=q_c.device) \
            if ws is None else ws
        if self.ws.numel() * self.ws.element_size() < need:
            raise ValueError("lci: workspace too small")
        self._keep = (q_c, k_c, ctx_len, q_start, q, k_pool, v_pool, table)
        self._name = "lci_sparse_decode_persistent" if persistent else "lci_sparse_decode"
        self._fn = getattr(load_library(), self._name)
        self._stream = _stream(stream)
        self._args = (
            _dev(q_c, "q_c", None, 4), _dev(k_c, "k_c", q_c.dtype, 4), _dtype_code(q_c), B, S, H_i,
            d_c, nb_max, _dev(ctx_len, "ctx_len", torch.int32, 1),
            _dev(q_start, "q_start", torch.int32, 1), topk, _dev(q, "q", q_c.dtype, 4), H_q,
            _dev(k_pool, "k_pool", q_c.dtype), _dev(v_pool, "v_pool", q_c.dtype), table.handle,
            ctypes.c_float(scale), _dev(self.ids, "ids", torch.int32, 3),
            _dev(self.out, "out", q_c.dtype, 4), _dev(self.ws, "workspace"),
            ctypes.c_size_t(self.ws.numel() * self.ws.element_size()), self._stream)

    def __call__(self, stream=None) -> None:
        """Launch the step on its stream, or on `stream` if given (e.g. the
        stream a CUDA graph is being captured on)."""
        args = self._args if stream is None else self._args[:-1] + (_stream(stream),)
        rc = self._fn(*args)
        if rc != LCI_OK:
            _check(rc, self._name)

    def capture(self, h2d=(), d2h=()) -> "torch.cuda.CUDAGraph":
        """The step with its transfers as one CUDA graph, for a serving loop
        that replays it every step: the copies ``dst.copy_(src)`` of ``h2d``
        (device tensors filled from pinned host tensors), this step, then the
        copies of ``d2h`` (pinned host tensors filled from device tensors). The
        graph reads and writes the same buffers on every replay; the caller
        refills the host inputs and reads the host outputs between replays
        (after synchronising). Call the step once before capturing it."""
        for dst, src in list(h2d) + list(d2h):
            host = dst if dst.device.type == "cpu" else src
            if not host.is_pinned():
                raise ValueError("lci: graph transfers need pinned host tensors")
        g = torch.cuda.CUDAGraph()
        torch.cuda.synchronize()
        with torch.cuda.graph(g):
            for dst, src in h2d:
                dst.copy_(src, non_blocking=True)
            self(torch.cuda.current_stream())  # the capturing stream
            for dst, src in d2h:
                dst.copy_(src, non_blocking=True)
        torch.cuda.synchronize()
        return g


def get_device_status(stream=None) -> None:
    """Synchronise the stream; raise LciError (LCI_ERR_TIMEOUT or
    LCI_ERR_DEVICE_BOUNDS) if a device wait ran out or a bounds check fired."""
    _check(load_library().lci_get_device_status(_stream(stream)), "lci_get_device_status")
