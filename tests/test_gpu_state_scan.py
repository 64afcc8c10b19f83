"""Chunked gated state scan (GPU) against the oracle.

The state stays in fp32; the readout multiplies the bf16 queries by the state
split into two bf16 parts (hi + lo, each element within about 2^-17 of the
fp32 state). Over a 128-term dot product that bounds the readout error by
about 128 * 2^-17 * max|q| * max|S|, below 1e-3 * max|out| for these inputs,
and the fp32 accumulation of the update adds far less. Outputs and the final
state are compared with the fp64 oracle at max-abs 2e-4 of the output's (or
state's) largest magnitude.
"""
import pytest
import torch

import long_context_indexer_b200 as lci
import oracle
from long_context_indexer_b200.workloads import SCAN_CONFIGS, generate_scan

pytestmark = pytest.mark.gpu

REL = 2e-4


def _close(got, ref, what):
    got = got.double().cpu()
    assert torch.isfinite(got).all(), what
    scale = max(1.0, ref.abs().max().item())
    err = (got - ref).abs().max().item()
    assert err <= REL * scale, f"{what}: max-abs error {err:.3e} above {REL * scale:.3e}"


def _run(w, chunk=128, in_place=False):
    d = {k: v.cuda() for k, v in w.items()}
    st = d["state"].clone()
    out, st_out = lci.gated_state_scan(d["q"], d["k"], d["v"], d["gate"], st, chunk,
                                       state_out=st if in_place else None)
    torch.cuda.synchronize()
    lci.get_device_status()
    return out, st_out


@pytest.mark.parametrize("T", [300, 128, 1, 129])
def test_state_scan_matches_oracle(T):
    cfg = SCAN_CONFIGS["scan_small"].replace(T=T)
    w = generate_scan(cfg)
    out, st = _run(w)
    ref_out, ref_st = oracle.gated_state_scan(w["q"], w["k"], w["v"], w["gate"], w["state"], cfg.C)
    _close(out, ref_out, f"out T={T}")
    _close(st, ref_st, f"state T={T}")


@pytest.mark.parametrize("gate", [0.0, 1.0])
def test_state_scan_extreme_gates_in_place(gate):
    cfg = SCAN_CONFIGS["scan_small"].replace(T=520)
    w = generate_scan(cfg)
    w["gate"].fill_(gate)
    out, st = _run(w, in_place=True)
    ref_out, ref_st = oracle.gated_state_scan(w["q"], w["k"], w["v"], w["gate"], w["state"], cfg.C)
    _close(out, ref_out, f"out gate={gate}")
    _close(st, ref_st, f"state gate={gate}")


def test_state_scan_full_size_sampled_heads():
    cfg = SCAN_CONFIGS["scan"]
    w = generate_scan(cfg)
    out, st = _run(w)
    for b, h in ((0, 0), (4, 7), (8, 15)):
        sl = {k: (v[b:b + 1, :, h:h + 1].contiguous() if k in ("q", "k", "v")
                  else v[b:b + 1, h:h + 1].contiguous()) for k, v in w.items()}
        ref_out, ref_st = oracle.gated_state_scan(sl["q"], sl["k"], sl["v"], sl["gate"],
                                                  sl["state"], cfg.C)
        _close(out[b:b + 1, :, h:h + 1], ref_out, f"out ({b},{h})")
        _close(st[b:b + 1, h:h + 1], ref_st, f"state ({b},{h})")


def test_state_scan_rejects_unsupported_shapes():
    cfg = SCAN_CONFIGS["scan_small"]
    d = {k: v.cuda() for k, v in generate_scan(cfg).items()}
    with pytest.raises(lci.LciError) as e:
        lci.gated_state_scan(d["q"], d["k"], d["v"], d["gate"].repeat(1, 1, 2)[:, :, :5].contiguous(),
                             d["state"], chunk=64)
    assert e.value.status == 2
