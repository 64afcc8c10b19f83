"""Host-side pieces of bench.py that need no GPU: the staging buffers of the
end-to-end step and the source digest that ties reported DRAM traffic to the
kernels an ncu capture ran on."""
import torch

import bench


def test_packed_buffer_segments_are_aligned_disjoint_and_round_trip():
    tensors = {
        "q_c": torch.randn(3, 1, 8, 128).to(torch.bfloat16),
        "q": torch.randn(3, 1, 16, 128).to(torch.bfloat16),
        "ctx_len": torch.tensor([5, 6, 7], dtype=torch.int32),
        "q_start": torch.tensor([4, 5, 6], dtype=torch.int32),
    }
    buf, views = bench.packed_buffer(tensors, "cpu")
    base = buf.data_ptr()
    spans = []
    for k, t in tensors.items():
        v = views[k]
        assert v.dtype == t.dtype and v.shape == t.shape and v.is_contiguous()
        off = v.data_ptr() - base
        assert off % 256 == 0
        spans.append((off, off + t.numel() * t.element_size()))
        v.copy_(t)
    spans.sort()
    assert all(a[1] <= b[0] for a, b in zip(spans, spans[1:]))
    assert spans[-1][1] <= buf.numel()
    for k, t in tensors.items():
        assert torch.equal(views[k], t)


def test_code_only_drops_comments_and_whitespace_but_not_code():
    a = "int x = 1;  // one\n/* block\n comment */ int y = 2;\n"
    b = "int x = 1;\n\n   int y = 2; // two"
    c = "int x = 1; int y = 3;"
    assert bench._code_only(a) == bench._code_only(b)
    assert bench._code_only(a) != bench._code_only(c)


def test_profiled_traffic_is_reported_only_for_the_captured_sources(monkeypatch):
    key = ("decode", "index_select")
    nbytes, digest = bench.PROFILED_TRAFFIC[key]
    monkeypatch.setattr(bench, "sources_digest", lambda: digest)
    assert bench.profiled_traffic(*key) == nbytes
    monkeypatch.setattr(bench, "sources_digest", lambda: "0" * 16)
    assert bench.profiled_traffic(*key) is None
    assert bench.profiled_traffic("decode", "no_such_kernel") is None


def test_config_entry_rates_and_fractions():
    cfg = bench.CONFIGS["1m_chunk"]
    r = {"t_step_ms": 0.5, "t_index_ms": 0.1, "t_attn_ms": 0.4,
         "alg": {"index_bytes": 2e8, "index_flops": 6e10, "attn_bytes": 8e8, "attn_flops": 4e10}}
    pk = {"hbm_gbs": 8000.0, "bf16_tflops": 2000.0}
    e = bench.config_entry(cfg, r, pk)
    assert abs(e["tokens_per_s"] - cfg.B * cfg.S / 5e-4) < 1e-6
    assert abs(e["index_gbs"] - 2000.0) < 1e-9 and abs(e["index_frac_hbm"] - 0.25) < 1e-12
    assert abs(e["index_tflops"] - 600.0) < 1e-9 and abs(e["index_frac_bf16"] - 0.3) < 1e-12
    assert abs(e["attn_gbs"] - 2000.0) < 1e-9 and abs(e["attn_frac_bf16"] - 0.05) < 1e-12
