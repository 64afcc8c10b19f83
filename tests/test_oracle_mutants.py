"""The oracle's pins must catch plausible slips (CPU only).

Each case plants one mistake in a copy of the oracle's C source (a dropped term,
an off-by-one, a reversed order, a wrong index), builds it into a scratch
directory, and runs the pin suite against that build in a subprocess. The
suite must fail for every mutant; the unmodified oracle passes it (the pin
tests themselves).
"""
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "lci_oracle.c")

# (name, original text, planted mistake)
MUTANTS = [
    ("score drops all heads but one",
     "            for (int64_t h = 0; h < H; ++h)\n                for (int64_t d = 0; d < D; ++d)\n                    acc +=",
     "            for (int64_t h = 0; h < 1; ++h)\n                for (int64_t d = 0; d < D; ++d)\n                    acc +="),
    ("score reads the query row of the sequence, not of the query",
     "ld(q_c, dt, (row * H + h) * D + d)", "ld(q_c, dt, (b * H + h) * D + d)"),
    ("query's own block not visible", "int64_t v = last / bs + 1;", "int64_t v = last / bs;"),
    ("ties keep the higher id", "return (x->id > y->id) - (x->id < y->id);",
     "return (x->id < y->id) - (x->id > y->id);"),
    ("ascending scores", "if (x->score > y->score) return -1;\n    if (x->score < y->score) return 1;",
     "if (x->score < y->score) return -1;\n    if (x->score > y->score) return 1;"),
    ("query's own token masked", "if (t > last) break;", "if (t >= last) break;"),
    ("kv head chosen modulo instead of by group", "            int64_t g = h / G;\n            double* o = out + (r * H_q + h) * hd;\n            for (int64_t d = 0; d < hd; ++d) o[d] = 0.0;\n            if (n == 0) continue;",
     "            int64_t g = h % H_kv;\n            double* o = out + (r * H_q + h) * hd;\n            for (int64_t d = 0; d < hd; ++d) o[d] = 0.0;\n            if (n == 0) continue;"),
    ("pool slot and head transposed", "return ((page * H_kv + g) * bs + u) * hd + d;",
     "return ((page * bs + u) * H_kv + g) * hd + d;"),
    ("scale dropped", "                logit[t] = scale * dot;\n                if (logit[t] > m) m = logit[t];\n            }\n            double den",
     "                logit[t] = dot;\n                if (logit[t] > m) m = logit[t];\n            }\n            double den"),
    ("block mean divides by the block size", "sum / (double)(t1 - t0)", "sum / (double)bs"),
    ("bf16 widened with the wrong shift", "<< 16;", "<< 15;"),
    ("block table row stride ignored", "int64_t page = block_table[b * nb_max + j];\n            for (int64_t u = 0; u < bs; ++u) {",
     "int64_t page = block_table[j];\n            for (int64_t u = 0; u < bs; ++u) {"),
    ("visibility ignores the context length",
     "    int64_t last = p < ctx - 1 ? p : ctx - 1;\n    if (last < 0) return 0;",
     "    int64_t last = p;\n    if (last < 0) return 0;"),
    ("attention ignores the context length",
     "        int64_t last = p < ctx - 1 ? p : ctx - 1;\n        double* logit = (double*)malloc(sizeof(double) * (size_t)(topk * bs));",
     "        int64_t last = p;\n        double* logit = (double*)malloc(sizeof(double) * (size_t)(topk * bs));"),
    ("unused slots padded with block 0", "ids[r * topk + i] = i < k ? (int32_t)cand[i].id : -1;",
     "ids[r * topk + i] = i < k ? (int32_t)cand[i].id : 0;"),
    ("softmax normaliser dropped",
     "            for (int64_t d = 0; d < hd; ++d) o[d] /= den;\n        }\n        free(logit); free(tok_page); free(tok_slot);",
     "        }\n        free(logit); free(tok_page); free(tok_slot);"),
    ("dense reference ignores the selection", "if (!selected) { logit[t] = -INFINITY; continue; }",
     "if (0) { logit[t] = -INFINITY; continue; }"),
    ("last visible block left out of the ranking", "qsort(cand, (size_t)vis, sizeof(scored_block), rank_cmp);",
     "qsort(cand, (size_t)(vis > 0 ? vis - 1 : 0), sizeof(scored_block), rank_cmp);"),
    ("attention reads the sequence's query, not the row's",
     "dot += ld(q, dt, (row * H_q + h) * hd + d) *\n                           ld(k_pool, dt, pool_off(tok_page[t], g, tok_slot[t], d, H_kv, bs, hd));",
     "dot += ld(q, dt, (b * H_q + h) * hd + d) *\n                           ld(k_pool, dt, pool_off(tok_page[t], g, tok_slot[t], d, H_kv, bs, hd));"),
    ("token slot off by one", "tok_slot[n] = u;", "tok_slot[n] = u > 0 ? u - 1 : 0;"),
    ("state scan reads out before the chunk's update",
     "                for (int64_t t = t0; t < t1; ++t)\n                    for (int64_t i = 0; i < dk; ++i) {\n                        const double ki",
     "                for (int64_t t = t1; t < t1; ++t)\n                    for (int64_t i = 0; i < dk; ++i) {\n                        const double ki"),
    ("state scan gate dropped", "for (int64_t i = 0; i < dk * dv; ++i) S[i] *= g;",
     "for (int64_t i = 0; i < dk * dv; ++i) S[i] *= 1.0;"),
    ("state scan k and v swapped in the update",
     "S[i * dv + j] += ki * ld(v, dt, ((b * T + t) * H + h) * dv + j);",
     "S[i * dv + j] += ki * ld(v, dt, ((b * T + t) * H + h) * dv + (j + i) % dv);"),
    ("state scan gate index off by one chunk", "const double g = gate[(b * H + h) * nchunks + c];",
     "const double g = gate[(b * H + h) * nchunks + (c > 0 ? c - 1 : 0)];"),
    ("state scan chunk end ignores T",
     "const int64_t t0 = c * C, t1 = (c + 1) * C < T ? (c + 1) * C : T;",
     "const int64_t t0 = c * C, t1 = (c + 1) * C < T ? (c + 1) * C : T - 1;"),
]


@pytest.mark.parametrize("name,orig,bad", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_pins_catch_mutant(name, orig, bad, tmp_path):
    src = open(SRC).read()
    assert src.count(orig) == 1, f"mutation site not unique: {name}"
    mut_c = tmp_path / "mutant.c"
    mut_c.write_text(src.replace(orig, bad))
    mut_so = tmp_path / "libmutant.so"
    subprocess.run(["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared", "-o", str(mut_so),
                    str(mut_c), "-lm"], check=True)
    env = dict(os.environ, LCI_ORACLE_LIB=str(mut_so), OMP_NUM_THREADS="2")
    res = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                          os.path.join(ROOT, "tests", "test_oracle_pins.py")],
                         cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert res.returncode != 0, f"pins did not catch: {name}\n{res.stdout[-2000:]}"
