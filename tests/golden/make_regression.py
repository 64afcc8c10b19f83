"""Write tests/golden/oracle_regression.json from the CPU oracle alone.

The pages print no worked example for the index pipeline, so the stored values
here are a regression set of the oracle itself (section 6 of "Day-0 Inference Adaptation of Ultra-Large-Scale MoE Models on
Domestic AI Accelerators" recommends turning problems met into reusable test
cases): small seeded cases whose block ids and a digest of
the attention output must not change unless the oracle's definition changes.
Run from the repository root:  python tests/golden/make_regression.py
"""
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
from long_context_indexer_b200.workloads import CONFIGS, generate  # noqa: E402

CASES = [
    ("tiny", {}),
    ("small_decode", dict(B=3, S=1, ctx=640, q_start=639, bs=64, topk=4, H_q=4, H_kv=1, hd=32,
                          H_i=2, d_c=16, spare_pages=2, dtype="bf16", compress=False)),
    ("small_prefill", dict(B=1, S=40, ctx=200, q_start=160, bs=16, topk=3, H_q=4, H_kv=2, hd=16,
                           H_i=2, d_c=8, spare_pages=2, dtype="bf16", compress=False)),
]


def run_case(name, over):
    cfg = CONFIGS["tiny"].replace(name=name, **over) if over else CONFIGS["tiny"]
    w = generate(cfg)
    k_c = oracle.block_compress(w["k_idx"], cfg.bs).to(cfg.torch_dtype) if cfg.compress else w["k_c"]
    ids = oracle.index_select(w["q_c"], k_c, cfg.bs, w["ctx_len"], w["q_start"], cfg.topk)
    out = oracle.sparse_attn(w["q"], w["k_pool"], w["v_pool"], w["block_table"], ids,
                             w["ctx_len"], w["q_start"], cfg.hd ** -0.5)
    return {
        "config": {k: getattr(cfg, k) for k in ("B", "S", "ctx", "q_start", "bs", "topk", "H_q",
                                                "H_kv", "hd", "H_i", "d_c", "spare_pages",
                                                "dtype", "compress", "seed")},
        "ids": ids.tolist(),
        "out_sum": float(out.sum()),
        "out_abs_sum": float(out.abs().sum()),
        "out_first_row": out.reshape(out.shape[0], -1)[0, :8].tolist(),
    }


def main():
    data = {"source": "written by tests/golden/make_regression.py from oracle/ only",
            "cases": {name: run_case(name, over) for name, over in CASES}}
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "oracle_regression.json")
    with open(path, "w") as f:
        json.dump(data, f, indent=0)
        f.write("\n")


if __name__ == "__main__":
    main()
