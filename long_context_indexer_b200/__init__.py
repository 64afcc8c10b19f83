"""lci -- B200-native sparse-attention index pipeline.

The CUDA library is ``liblci.so`` (C ABI in ``include/lci.h``); ``lci`` is its
thin ctypes binding and ``workloads`` the seeded synthetic input generator.
Importing the package loads nothing; the library is loaded on first use.
"""
from .lci import (BlockTable, LciError, PagedKeys, SparseDecodeStep, block_compress,
                  create_block_table,
                  gated_state_scan, get_device_status,
                  get_wait_limit_ns, index_select, index_select_noalloc, index_select_paged,
                  index_select_workspace_size, load_library, set_wait_limit_ns, sparse_attn,
                  sparse_attn_pipelined, sparse_attn_workspace_size, sparse_decode,
                  sparse_decode_workspace_size, version)

__all__ = ["BlockTable", "LciError", "PagedKeys", "SparseDecodeStep", "block_compress",
           "create_block_table",
           "gated_state_scan", "get_device_status",
           "get_wait_limit_ns", "index_select", "index_select_noalloc", "index_select_paged",
           "index_select_workspace_size", "load_library", "set_wait_limit_ns", "sparse_attn",
           "sparse_attn_pipelined", "sparse_attn_workspace_size", "sparse_decode",
           "sparse_decode_workspace_size", "version"]
