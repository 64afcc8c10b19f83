"""The C ABI library loads, exports every declared entry point, and rejects bad
arguments on the host before launching anything (CPU only: no CUDA call is
reached in these tests)."""
import ctypes
import os
import re

import pytest

import long_context_indexer_b200 as lci
from long_context_indexer_b200 import lci as binding
from long_context_indexer_b200.build import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "lci.h")

INVALID, UNSUPPORTED, WORKSPACE = 1, 2, 3
FAKE = ctypes.c_void_p(0x7F0000000000)  # 256-byte aligned, never dereferenced


def declared_entry_points():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"^LCI_API\s+[\w\s\*]+?\b(lci_\w+)\s*\(", text, flags=re.M)))


@pytest.fixture(scope="module")
def lib():
    build()
    return lci.load_library()


def test_every_declared_symbol_is_exported(lib):
    names = declared_entry_points()
    assert len(names) >= 12
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(binding.SIGNATURES), "binding and header disagree"


def test_version_and_status_strings(lib):
    assert lci.version().count(".") == 2
    for code in range(7):
        assert lib.lci_status_string(code)


def _index_select(lib, **kw):
    a = dict(q_c=FAKE, k_c=FAKE, dtype=1, B=2, S=1, H_i=8, d_c=128, bs=64, nb_max=512,
             ctx=FAKE, q0=FAKE, topk=32, phase=0, ids=FAKE, ws=None, ws_bytes=0)
    a.update(kw)
    return lib.lci_index_select(a["q_c"], a["k_c"], a["dtype"], a["B"], a["S"], a["H_i"], a["d_c"],
                                a["bs"], a["nb_max"], a["ctx"], a["q0"], a["topk"], a["phase"],
                                a["ids"], a["ws"], a["ws_bytes"], None)


def test_index_select_host_checks(lib):
    assert _index_select(lib, q_c=None) == INVALID
    assert _index_select(lib, ids=None) == INVALID
    assert _index_select(lib, B=0) == INVALID
    assert _index_select(lib, topk=0) == INVALID
    assert _index_select(lib, bs=0) == INVALID
    assert _index_select(lib, dtype=7) == INVALID
    assert _index_select(lib, phase=9) == INVALID
    assert _index_select(lib, topk=257) == UNSUPPORTED
    assert _index_select(lib, nb_max=1 << 20) == UNSUPPORTED
    assert _index_select(lib, H_i=1, d_c=127) == UNSUPPORTED   # H_i*d_c not a multiple of 8
    assert _index_select(lib, q_c=ctypes.c_void_p(0x7F0000000002)) == INVALID  # misaligned
    assert _index_select(lib) == WORKSPACE                      # no workspace
    need = binding.index_select_workspace_size(2, 1, 8, 128, 512, 32)
    assert need > 0
    assert _index_select(lib, ws=FAKE, ws_bytes=need - 1) == WORKSPACE
    # a prefill-shaped call (tensor-core schedule) asks for its own, larger workspace
    need_p = binding.index_select_workspace_size(2, 512, 8, 128, 512, 32, "prefill")
    assert _index_select(lib, S=512, phase=1, ws=FAKE, ws_bytes=need_p - 1) == WORKSPACE
    assert _index_select(lib, ws=ctypes.c_void_p(0x7F0000000010), ws_bytes=need) == WORKSPACE
    assert b"workspace" in lib.lci_last_error()


def test_block_table_lifecycle_and_attn_host_checks(lib):
    h = ctypes.c_void_p()
    assert lib.lci_create_block_table(None, 2, 4, 8, 64, 1, 128, 1, ctypes.byref(h)) == INVALID
    assert lib.lci_create_block_table(FAKE, 2, 0, 8, 64, 1, 128, 1, ctypes.byref(h)) == INVALID
    assert lib.lci_create_block_table(FAKE, 2, 4, 8, 64, 2, 128, 1, ctypes.byref(h)) == 0
    try:
        def attn(**kw):
            a = dict(q=FAKE, B=2, S=1, H_q=16, kp=FAKE, vp=FAKE, t=h, ids=FAKE, topk=4, ctx=FAKE,
                     q0=FAKE, scale=0.0, phase=0, out=FAKE)
            a.update(kw)
            return lib.lci_sparse_attn(a["q"], a["B"], a["S"], a["H_q"], a["kp"], a["vp"], a["t"],
                                       a["ids"], a["topk"], a["ctx"], a["q0"], a["scale"],
                                       a["phase"], a["out"], None, 0, None)
        assert attn(q=None) == INVALID
        assert attn(t=None) == INVALID
        assert attn(H_q=15) == INVALID        # not a multiple of the 2 KV heads
        assert attn(B=3) == INVALID           # more sequences than the table has rows
        assert attn(topk=0) == INVALID
        assert attn(topk=300) == UNSUPPORTED
        assert attn(phase=5) == INVALID
        n = ctypes.c_size_t()
        assert lib.lci_sparse_attn_workspace_size(2, 1, 16, 4, h, 0, ctypes.byref(n)) == 0
    finally:
        assert lib.lci_destroy_block_table(h) == 0
    h2 = ctypes.c_void_p()
    assert lib.lci_create_block_table(FAKE, 1, 4, 8, 64, 1, 48, 1, ctypes.byref(h2)) == 0
    try:
        assert lib.lci_sparse_attn(FAKE, 1, 1, 1, FAKE, FAKE, h2, FAKE, 4, FAKE, FAKE, 0.0, 0,
                                   FAKE, None, 0, None) == UNSUPPORTED  # head_dim 48
    finally:
        lib.lci_destroy_block_table(h2)
    assert lib.lci_destroy_block_table(None) == 0


def test_block_compress_host_checks(lib):
    assert lib.lci_block_compress(None, 0, 1, 16, 1, 64, 16, FAKE, None) == INVALID
    assert lib.lci_block_compress(FAKE, 0, 1, 0, 1, 64, 16, FAKE, None) == INVALID
    assert lib.lci_block_compress(FAKE, 3, 1, 16, 1, 64, 16, FAKE, None) == INVALID


def test_binding_rejects_cpu_tensors():
    import torch
    with pytest.raises(ValueError):
        binding._dev(torch.zeros(4), "x")


def test_sparse_decode_host_checks(lib):
    h = ctypes.c_void_p()
    # bf16 table: 2 sequences x 8 blocks of 64 tokens, 1 KV head of dim 128, 20 pages
    assert lib.lci_create_block_table(FAKE, 2, 8, 20, 64, 1, 128, 1, ctypes.byref(h)) == 0
    try:
        need = ctypes.c_size_t()
        assert lib.lci_sparse_decode_workspace_size(2, 1, 8, 128, 4, 16, h, ctypes.byref(need)) == 0
        assert need.value > 0
        assert lib.lci_sparse_decode_workspace_size(2, 1, 8, 128, 4, 16, h, None) == INVALID
        assert lib.lci_sparse_decode_workspace_size(2, 1, 8, 128, 4, 16, None, ctypes.byref(need)) == INVALID

        def dec(**kw):
            a = dict(q_c=FAKE, k_c=FAKE, dtype=1, B=2, S=1, H_i=8, d_c=128, nb_max=8, ctx=FAKE,
                     q0=FAKE, topk=4, q=FAKE, H_q=16, kp=FAKE, vp=FAKE, t=h, scale=0.0, ids=FAKE,
                     out=FAKE, ws=FAKE, ws_bytes=need.value)
            a.update(kw)
            return lib.lci_sparse_decode(a["q_c"], a["k_c"], a["dtype"], a["B"], a["S"], a["H_i"],
                                         a["d_c"], a["nb_max"], a["ctx"], a["q0"], a["topk"],
                                         a["q"], a["H_q"], a["kp"], a["vp"], a["t"], a["scale"],
                                         a["ids"], a["out"], a["ws"], a["ws_bytes"], None)
        assert dec(q_c=None) == INVALID
        assert dec(out=None) == INVALID
        assert dec(t=None) == INVALID
        assert dec(nb_max=7) == INVALID                 # differs from the table's 8 blocks
        assert dec(dtype=0) == INVALID                  # fp32 indexer with a bf16 cache
        assert dec(B=3) == INVALID                      # more sequences than the table
        assert dec(q_c=ctypes.c_void_p(FAKE.value + 8)) == INVALID  # not 16-byte aligned
        assert dec(ws=None) == WORKSPACE
        assert dec(ws_bytes=256) == WORKSPACE           # far below either schedule's need
        assert dec(ws=ctypes.c_void_p(FAKE.value + 16)) == WORKSPACE  # not 256-byte aligned
        assert dec(scale=float("inf")) == INVALID
        assert dec(topk=0) == INVALID
    finally:
        assert lib.lci_destroy_block_table(h) == 0


def test_index_select_noalloc_host_checks(lib):
    def na(**kw):
        a = dict(q_c=FAKE, k_c=FAKE, dtype=1, B=2, S=1, H_i=8, d_c=128, bs=64, nb_max=512,
                 ctx=FAKE, q0=FAKE, topk=32, phase=0, ids=FAKE)
        a.update(kw)
        return lib.lci_index_select_noalloc(a["q_c"], a["k_c"], a["dtype"], a["B"], a["S"],
                                            a["H_i"], a["d_c"], a["bs"], a["nb_max"], a["ctx"],
                                            a["q0"], a["topk"], a["phase"], a["ids"], None)
    assert na(k_c=None) == INVALID
    assert na(bs=0) == INVALID
    assert na(phase=9) == INVALID
    assert na(k_c=ctypes.c_void_p(FAKE.value + 4)) == INVALID
    # 256 rows x 16384 blocks of fp32 scores alone exceed the built-in scratch
    assert na(B=256, nb_max=16384) == WORKSPACE
    assert b"scratch" in lib.lci_last_error()


def test_wait_limit_and_pipelined_attention_host_checks(lib):
    # limits outside [1 ns, 60 s] are rejected before any CUDA call
    assert lib.lci_set_wait_limit_ns(0) == INVALID
    assert lib.lci_set_wait_limit_ns(61 * 10**9) == INVALID
    assert b"wait_limit" in lib.lci_last_error()
    assert lib.lci_get_wait_limit_ns(None) == INVALID
    h = ctypes.c_void_p()
    assert lib.lci_create_block_table(FAKE, 2, 8, 20, 64, 1, 128, 1, ctypes.byref(h)) == 0
    hf = ctypes.c_void_p()
    assert lib.lci_create_block_table(FAKE, 2, 8, 20, 64, 1, 128, 0, ctypes.byref(hf)) == 0
    try:
        def pip(**kw):
            a = dict(q=FAKE, B=2, S=1, H_q=16, kp=FAKE, vp=FAKE, t=h, ids=FAKE, topk=4, ctx=FAKE,
                     q0=FAKE, scale=0.0, ready=FAKE, out=FAKE)
            a.update(kw)
            return lib.lci_sparse_attn_pipelined(a["q"], a["B"], a["S"], a["H_q"], a["kp"],
                                                 a["vp"], a["t"], a["ids"], a["topk"], a["ctx"],
                                                 a["q0"], a["scale"], a["ready"], a["out"], None)
        assert pip(ready=None) == INVALID
        assert pip(out=None) == INVALID
        assert pip(t=None) == INVALID
        assert pip(B=3) == INVALID
        assert pip(H_q=32) == UNSUPPORTED                  # 32 query heads per KV head
        assert pip(t=hf) == UNSUPPORTED                    # fp32 pools
        assert pip(kp=ctypes.c_void_p(FAKE.value + 2)) == UNSUPPORTED  # misaligned pool
        assert pip(scale=float("inf")) == INVALID
    finally:
        lib.lci_destroy_block_table(h)
        lib.lci_destroy_block_table(hf)


def test_device_status_names_timeouts():
    assert binding.STATUS_NAMES[6] == "LCI_ERR_TIMEOUT"
    text = open(HEADER).read()
    assert "reserved" not in text.split("LCI_ERR_TIMEOUT = 6", 1)[1].split("\n", 1)[0]


def test_paged_key_entry_points_host_checks(lib):
    h = ctypes.c_void_p()
    # bf16 table: 2 sequences x 8 blocks of 64 tokens, 20 pages
    assert lib.lci_create_block_table(FAKE, 2, 8, 20, 64, 1, 128, 1, ctypes.byref(h)) == 0
    try:
        upd = lambda **kw: lib.lci_kc_update(  # noqa: E731
            kw.get("k", FAKE), kw.get("dtype", 1), kw.get("B", 2), kw.get("T", 1), 8, 128,
            kw.get("start", FAKE), kw.get("t", h), kw.get("sum", FAKE), kw.get("kc", FAKE), None)
        assert upd(k=None) == INVALID
        assert upd(t=None) == INVALID
        assert upd(sum=None) == INVALID
        assert upd(T=0) == INVALID
        assert upd(B=3) == INVALID          # more sequences than the table
        assert upd(dtype=5) == INVALID
        n = ctypes.c_size_t()
        assert lib.lci_index_select_paged_workspace_size(2, 1, 8, 128, 32, h, 1, 0,
                                                         ctypes.byref(n)) == 0
        assert n.value > 0
        assert lib.lci_index_select_paged_workspace_size(2, 1, 8, 128, 32, None, 1, 0,
                                                         ctypes.byref(n)) == INVALID

        def sel(**kw):
            a = dict(q_c=FAKE, kc=FAKE, dtype=1, B=2, S=1, H_i=8, d_c=128, t=h, ctx=FAKE, q0=FAKE,
                     topk=32, phase=0, ids=FAKE, ws=FAKE, ws_bytes=n.value)
            a.update(kw)
            return lib.lci_index_select_paged(a["q_c"], a["kc"], a["dtype"], a["B"], a["S"],
                                              a["H_i"], a["d_c"], a["t"], a["ctx"], a["q0"],
                                              a["topk"], a["phase"], a["ids"], a["ws"],
                                              a["ws_bytes"], None)
        assert sel(kc=None) == INVALID
        assert sel(t=None) == INVALID
        assert sel(B=3) == INVALID
        assert sel(phase=7) == INVALID
        assert sel(topk=300) == UNSUPPORTED
        assert sel(kc=ctypes.c_void_p(FAKE.value + 8)) == INVALID
        assert sel(ws=None) == WORKSPACE
        assert sel(ws_bytes=n.value - 1) == WORKSPACE
    finally:
        lib.lci_destroy_block_table(h)
