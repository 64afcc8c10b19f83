/*
 * lci_oracle.c -- plain, slow CPU oracle of the sparse-attention index pipeline.
 *
 * TEST INFRASTRUCTURE ONLY. This file is the definition the CUDA library is
 * checked against. Only the tests, the smoke check and the benchmark's CPU
 * baseline load it; the library never calls it and shares no code with it.
 *
 * What it computes (one layer, one step):
 *
 *   A0  block compression   k_c[b,j,h,:] = mean over the tokens t of block j of
 *                           k_idx[b,t,h,:]  ("query/key representation
 *                           generation", the first of the three stages in
 *                           "Day-0 Inference Adaptation for Ultra-Large MoE
 *                           Models on Domestic GPUs", section "Adapting Sparse
 *                           Attention"; mean pooling is the plainest compressor
 *                           and the one the measured tiny workload names).
 *   A1  block scoring       score[b,s,j] = sum_h sum_d q_c[b,s,h,d] * k_c[b,j,h,d]
 *                           (the score of compressed queries against compressed
 *                           keys, "Day-0 Inference Adaptation of Ultra-Large-Scale
 *                           MoE Models on Domestic AI Accelerators", section 4.1,
 *                           summed over the indexer heads).
 *   A2  masked top-k        ids[b,s,:] = the min(topk, vis) causal-visible blocks
 *                           with the largest scores, ranked by (score desc, block
 *                           id asc), padded with -1 (same page, section 4.1;
 *                           the score/top-k/mask combination of page 1's
 *                           section "Operatorizing Index Selection").
 *   N4  gated state scan    the chunked gated state update and readout of the
 *                           linear-attention family (orc_gated_state_scan below).
 *   A3+A4 sparse attention  exact softmax attention of each query head over the
 *                           tokens of the selected blocks only, gathered from a
 *                           paged KV pool through a block table (page 2 section
 *                           4.1, attention restricted to the chosen positions;
 *                           "Day-0 Adaptation for Trillion-Parameter MoE Models"
 *                           section IV, KV pages and the page table).
 *
 * Readings where the pages are silent (each is also listed in the design notes):
 *   - Query position p = q_start[b] + s. The last attendable token is
 *     last = min(p, ctx_len[b] - 1). A block j is visible when it holds a token
 *     t <= last, i.e. j <= last / bs; vis = min(nb_max, last / bs + 1), 0 when
 *     last < 0. The query's own partial block is a candidate on equal terms.
 *   - Inside a selected block only tokens t <= last take part.
 *   - An empty token set gives an all-zero output row.
 *   - Query head h reads KV head g = h / (H_q / H_kv) (grouped-query attention).
 *   - The softmax scale is given by the caller (the pages name none; the
 *     library's default is 1/sqrt(hd)).
 *
 * Arithmetic is IEEE fp64 throughout; bf16 and fp32 inputs are widened exactly.
 * No blocking, fusion or reordering beyond the definition: each function is a
 * loop nest over its definition. Rows are independent and run under OpenMP.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

enum { ORC_F32 = 0, ORC_BF16 = 1, ORC_F64 = 2 };
enum { ORC_OK = 0, ORC_BAD_ARG = 1, ORC_BAD_ID = 2, ORC_NOMEM = 3 };

/* Element i of a floating array of type dt, widened exactly to double. */
static double ld(const void* p, int dt, int64_t i) {
    if (dt == ORC_F32) return (double)((const float*)p)[i];
    if (dt == ORC_BF16) {
        uint32_t u = ((uint32_t)((const uint16_t*)p)[i]) << 16;
        float f;
        memcpy(&f, &u, sizeof f);
        return (double)f;
    }
    return ((const double*)p)[i];
}

int orc_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

void orc_set_num_threads(int n) {
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

/* Number of causal-visible blocks for a query at absolute position p. */
static int64_t visible_blocks(int64_t p, int64_t ctx, int64_t bs, int64_t nb_max) {
    int64_t last = p < ctx - 1 ? p : ctx - 1;
    if (last < 0) return 0;
    int64_t v = last / bs + 1;
    return v < nb_max ? v : nb_max;
}

/*
 * A0. k_c[b][j][h][d] = (1/n_j) * sum_{t in block j} k_idx[b][t][h][d], where
 * block j holds tokens [j*bs, min(T, (j+1)*bs)) and n_j is their count.
 */
int orc_block_compress(const void* k_idx, int dt, int64_t B, int64_t T, int64_t H,
                       int64_t D, int64_t bs, double* k_c) {
    if (!k_idx || !k_c || B < 0 || T < 0 || H <= 0 || D <= 0 || bs <= 0) return ORC_BAD_ARG;
    int64_t NB = (T + bs - 1) / bs;
    for (int64_t b = 0; b < B; ++b)
        for (int64_t j = 0; j < NB; ++j) {
            int64_t t0 = j * bs, t1 = (j + 1) * bs < T ? (j + 1) * bs : T;
            for (int64_t h = 0; h < H; ++h)
                for (int64_t d = 0; d < D; ++d) {
                    double sum = 0.0;
                    for (int64_t t = t0; t < t1; ++t)
                        sum += ld(k_idx, dt, ((b * T + t) * H + h) * D + d);
                    k_c[((b * NB + j) * H + h) * D + d] = sum / (double)(t1 - t0);
                }
        }
    return ORC_OK;
}

/* Row r of the flattened [B*S] query rows: the r-th entry of rows[], or r. */
static int64_t row_at(const int64_t* rows, int64_t r) { return rows ? rows[r] : r; }

/*
 * A1. score[r][j] for j < vis(p) (the dot product summed over indexer heads),
 * -INFINITY for blocks that are not causal-visible.
 */
int orc_block_scores(const void* q_c, const void* k_c, int dt, int64_t B, int64_t S,
                     int64_t H, int64_t D, int64_t nb_max, int64_t bs,
                     const int32_t* ctx_len, const int32_t* q_start,
                     const int64_t* rows, int64_t nrows, double* scores) {
    if (!q_c || !k_c || !ctx_len || !q_start || !scores || bs <= 0 || H <= 0 || D <= 0)
        return ORC_BAD_ARG;
    if (!rows) nrows = B * S;
    int bad = 0;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t r = 0; r < nrows; ++r) {
        int64_t row = row_at(rows, r);
        if (row < 0 || row >= B * S) { bad = 1; continue; }
        int64_t b = row / S, s = row % S;
        int64_t p = (int64_t)q_start[b] + s;
        int64_t vis = visible_blocks(p, ctx_len[b], bs, nb_max);
        for (int64_t j = 0; j < nb_max; ++j) {
            if (j >= vis) { scores[r * nb_max + j] = -INFINITY; continue; }
            double acc = 0.0;
            for (int64_t h = 0; h < H; ++h)
                for (int64_t d = 0; d < D; ++d)
                    acc += ld(q_c, dt, (row * H + h) * D + d) *
                           ld(k_c, dt, ((b * nb_max + j) * H + h) * D + d);
            scores[r * nb_max + j] = acc;
        }
    }
    return bad ? ORC_BAD_ARG : ORC_OK;
}

typedef struct { double score; int64_t id; } scored_block;

/* Rank order: larger score first; equal scores keep the lower block id first. */
static int rank_cmp(const void* a, const void* b) {
    const scored_block* x = (const scored_block*)a;
    const scored_block* y = (const scored_block*)b;
    if (x->score > y->score) return -1;
    if (x->score < y->score) return 1;
    return (x->id > y->id) - (x->id < y->id);
}

/*
 * A1+A2. ids[r][i] for i < min(topk, vis): the i-th block in rank order among
 * the visible blocks; the rest of the row is -1.
 */
int orc_index_select(const void* q_c, const void* k_c, int dt, int64_t B, int64_t S,
                     int64_t H, int64_t D, int64_t nb_max, int64_t bs,
                     const int32_t* ctx_len, const int32_t* q_start, int64_t topk,
                     const int64_t* rows, int64_t nrows, int32_t* ids) {
    if (topk <= 0 || !ids || nb_max <= 0) return ORC_BAD_ARG;
    if (!rows) nrows = B * S;
    double* scores = (double*)malloc(sizeof(double) * (size_t)(nrows > 0 ? nrows : 1) * (size_t)nb_max);
    if (!scores) return ORC_NOMEM;
    int rc = orc_block_scores(q_c, k_c, dt, B, S, H, D, nb_max, bs, ctx_len, q_start, rows,
                              nrows, scores);
    if (rc != ORC_OK) { free(scores); return rc; }
    int nomem = 0;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t r = 0; r < nrows; ++r) {
        int64_t row = row_at(rows, r);
        int64_t b = row / S, s = row % S;
        int64_t p = (int64_t)q_start[b] + s;
        int64_t vis = visible_blocks(p, ctx_len[b], bs, nb_max);
        scored_block* cand = (scored_block*)malloc(sizeof(scored_block) * (size_t)(vis > 0 ? vis : 1));
        if (!cand) { nomem = 1; continue; }
        for (int64_t j = 0; j < vis; ++j) {
            cand[j].score = scores[r * nb_max + j];
            cand[j].id = j;
        }
        qsort(cand, (size_t)vis, sizeof(scored_block), rank_cmp);
        int64_t k = topk < vis ? topk : vis;
        for (int64_t i = 0; i < topk; ++i)
            ids[r * topk + i] = i < k ? (int32_t)cand[i].id : -1;
        free(cand);
    }
    free(scores);
    return nomem ? ORC_NOMEM : ORC_OK;
}

/* Offset of K/V element (page, kv head g, slot u, dim d) in a [P][H_kv][bs][hd] pool. */
static int64_t pool_off(int64_t page, int64_t g, int64_t u, int64_t d, int64_t H_kv,
                        int64_t bs, int64_t hd) {
    return ((page * H_kv + g) * bs + u) * hd + d;
}

/*
 * Shared argument check of the two attention oracles: every id is -1 or a
 * block below nb_max, and every referenced table entry names a pool page.
 */
static int check_ids(const int32_t* ids, int64_t topk, const int32_t* table, int64_t nb_max,
                     int64_t num_pages, int64_t B, int64_t S, const int64_t* rows, int64_t nrows) {
    for (int64_t r = 0; r < nrows; ++r) {
        int64_t row = row_at(rows, r);
        if (row < 0 || row >= B * S) return ORC_BAD_ARG;
        int64_t b = row / S;
        for (int64_t i = 0; i < topk; ++i) {
            int32_t j = ids[r * topk + i];
            if (j == -1) continue;
            if (j < 0 || j >= nb_max) return ORC_BAD_ID;
            int32_t page = table[b * nb_max + j];
            if (page < 0 || page >= num_pages) return ORC_BAD_ID;
        }
    }
    return ORC_OK;
}

/*
 * A3+A4. For every row r and query head h:
 *   T    = { t : block(t) is one of ids[r][*], t <= last }
 *   l_t  = scale * <q[row][h], K[block_table[b][block(t)]][g][t mod bs]>
 *   out  = sum_{t in T} exp(l_t - m) v_t / sum_{t in T} exp(l_t - m),  m = max_t l_t
 * with g = h / (H_q / H_kv); out = 0 when T is empty. ids rows (ids[r] for the
 * r-th requested row) may be in any order and must not repeat a block.
 */
int orc_sparse_attn(const void* q, const void* k_pool, const void* v_pool, int dt,
                    int64_t B, int64_t S, int64_t H_q, int64_t H_kv, int64_t hd,
                    int64_t num_pages, int64_t bs, const int32_t* block_table, int64_t nb_max,
                    const int32_t* ids, int64_t topk, const int32_t* ctx_len,
                    const int32_t* q_start, double scale, const int64_t* rows, int64_t nrows,
                    double* out) {
    if (!q || !k_pool || !v_pool || !block_table || !ids || !ctx_len || !q_start || !out ||
        H_q <= 0 || H_kv <= 0 || H_q % H_kv != 0 || hd <= 0 || bs <= 0 || topk <= 0)
        return ORC_BAD_ARG;
    if (!rows) nrows = B * S;
    int rc = check_ids(ids, topk, block_table, nb_max, num_pages, B, S, rows, nrows);
    if (rc != ORC_OK) return rc;
    int64_t G = H_q / H_kv;
    int nomem = 0;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t r = 0; r < nrows; ++r) {
        int64_t row = row_at(rows, r);
        int64_t b = row / S, s = row % S;
        int64_t p = (int64_t)q_start[b] + s;
        int64_t ctx = ctx_len[b];
        int64_t last = p < ctx - 1 ? p : ctx - 1;
        double* logit = (double*)malloc(sizeof(double) * (size_t)(topk * bs));
        int64_t* tok_page = (int64_t*)malloc(sizeof(int64_t) * (size_t)(topk * bs));
        int64_t* tok_slot = (int64_t*)malloc(sizeof(int64_t) * (size_t)(topk * bs));
        if (!logit || !tok_page || !tok_slot) {
            nomem = 1;
            free(logit); free(tok_page); free(tok_slot);
            continue;
        }
        /* The token set T of this row (shared by all heads). */
        int64_t n = 0;
        for (int64_t i = 0; i < topk; ++i) {
            int32_t j = ids[r * topk + i];
            if (j < 0) continue;
            int64_t page = block_table[b * nb_max + j];
            for (int64_t u = 0; u < bs; ++u) {
                int64_t t = (int64_t)j * bs + u;
                if (t > last) break;
                tok_page[n] = page;
                tok_slot[n] = u;
                ++n;
            }
        }
        for (int64_t h = 0; h < H_q; ++h) {
            int64_t g = h / G;
            double* o = out + (r * H_q + h) * hd;
            for (int64_t d = 0; d < hd; ++d) o[d] = 0.0;
            if (n == 0) continue;
            double m = -INFINITY;
            for (int64_t t = 0; t < n; ++t) {
                double dot = 0.0;
                for (int64_t d = 0; d < hd; ++d)
                    dot += ld(q, dt, (row * H_q + h) * hd + d) *
                           ld(k_pool, dt, pool_off(tok_page[t], g, tok_slot[t], d, H_kv, bs, hd));
                logit[t] = scale * dot;
                if (logit[t] > m) m = logit[t];
            }
            double den = 0.0;
            for (int64_t t = 0; t < n; ++t) {
                double w = exp(logit[t] - m);
                den += w;
                for (int64_t d = 0; d < hd; ++d)
                    o[d] += w * ld(v_pool, dt, pool_off(tok_page[t], g, tok_slot[t], d, H_kv, bs, hd));
            }
            for (int64_t d = 0; d < hd; ++d) o[d] /= den;
        }
        free(logit); free(tok_page); free(tok_slot);
    }
    return nomem ? ORC_NOMEM : ORC_OK;
}

/*
 * Full dense attention over every token t <= last of the sequence, with the
 * logits of tokens whose block is not among ids[r][*] set to -infinity before
 * the softmax. For distinct ids this is the same function as orc_sparse_attn,
 * written the long way round: page 3 section IV asks that the sparse path be
 * checked against full attention.
 */
int orc_dense_masked(const void* q, const void* k_pool, const void* v_pool, int dt,
                     int64_t B, int64_t S, int64_t H_q, int64_t H_kv, int64_t hd,
                     int64_t num_pages, int64_t bs, const int32_t* block_table, int64_t nb_max,
                     const int32_t* ids, int64_t topk, const int32_t* ctx_len,
                     const int32_t* q_start, double scale, const int64_t* rows, int64_t nrows,
                     double* out) {
    if (!q || !k_pool || !v_pool || !block_table || !ids || !ctx_len || !q_start || !out ||
        H_q <= 0 || H_kv <= 0 || H_q % H_kv != 0 || hd <= 0 || bs <= 0 || topk <= 0)
        return ORC_BAD_ARG;
    if (!rows) nrows = B * S;
    int rc = check_ids(ids, topk, block_table, nb_max, num_pages, B, S, rows, nrows);
    if (rc != ORC_OK) return rc;
    int64_t G = H_q / H_kv;
    int nomem = 0;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t r = 0; r < nrows; ++r) {
        int64_t row = row_at(rows, r);
        int64_t b = row / S, s = row % S;
        int64_t p = (int64_t)q_start[b] + s;
        int64_t ctx = ctx_len[b];
        int64_t last = p < ctx - 1 ? p : ctx - 1;
        int64_t ntok = last + 1 > 0 ? last + 1 : 0;
        if (ntok > nb_max * bs) ntok = nb_max * bs;
        double* logit = (double*)malloc(sizeof(double) * (size_t)(ntok > 0 ? ntok : 1));
        if (!logit) { nomem = 1; continue; }
        for (int64_t h = 0; h < H_q; ++h) {
            int64_t g = h / G;
            double* o = out + (r * H_q + h) * hd;
            double m = -INFINITY;
            for (int64_t t = 0; t < ntok; ++t) {
                int64_t j = t / bs, u = t % bs;
                int selected = 0;
                for (int64_t i = 0; i < topk; ++i)
                    if (ids[r * topk + i] == j) selected = 1;
                if (!selected) { logit[t] = -INFINITY; continue; }
                int64_t page = block_table[b * nb_max + j];
                double dot = 0.0;
                for (int64_t d = 0; d < hd; ++d)
                    dot += ld(q, dt, (row * H_q + h) * hd + d) *
                           ld(k_pool, dt, pool_off(page, g, u, d, H_kv, bs, hd));
                logit[t] = scale * dot;
                if (logit[t] > m) m = logit[t];
            }
            for (int64_t d = 0; d < hd; ++d) o[d] = 0.0;
            if (m == -INFINITY) continue; /* no selected token: zero row */
            double den = 0.0;
            for (int64_t t = 0; t < ntok; ++t) {
                double w = exp(logit[t] - m); /* exp(-inf) = 0 for masked tokens */
                if (w == 0.0) continue;
                int64_t j = t / bs, u = t % bs;
                int64_t page = block_table[b * nb_max + j];
                den += w;
                for (int64_t d = 0; d < hd; ++d)
                    o[d] += w * ld(v_pool, dt, pool_off(page, g, u, d, H_kv, bs, hd));
            }
            for (int64_t d = 0; d < hd; ++d) o[d] /= den;
        }
        free(logit);
    }
    return nomem ? ORC_NOMEM : ORC_OK;
}

/*
 * N4. Chunked gated state scan ("Day-0 Adaptation for Trillion-Parameter MoE
 * Models", section III, the gated incremental state update of the linear
 * attention family: the sequence is scanned in chunks of C tokens and a state
 * matrix is carried from chunk to chunk). For every sequence b and head h, with
 * the state S [dk][dv] starting at state[b][h] and chunk c holding tokens
 * [c*C, min(T, (c+1)*C)):
 *     S        = gate[b][h][c] * S + sum_{t in chunk c} k_t^T v_t
 *     out[t]   = q_t S                       for every t in chunk c
 * (the readout uses the state after the chunk's own update). On return
 * state[b][h] holds the final S.
 *   q, k [B][T][H][dk]; v [B][T][H][dv] (type dt); gate [B][H][nchunks];
 *   state [B][H][dk][dv] (in/out); out [B][T][H][dv].
 */
int orc_gated_state_scan(const void* q, const void* k, const void* v, int dt, const double* gate,
                         double* state, int64_t B, int64_t T, int64_t H, int64_t dk, int64_t dv,
                         int64_t C, double* out) {
    if (!q || !k || !v || !gate || !state || !out || B < 0 || T < 0 || H <= 0 || dk <= 0 ||
        dv <= 0 || C <= 0)
        return ORC_BAD_ARG;
    const int64_t nchunks = (T + C - 1) / C;
    int nomem = 0;
#pragma omp parallel for collapse(2) schedule(dynamic)
    for (int64_t b = 0; b < B; ++b)
        for (int64_t h = 0; h < H; ++h) {
            double* S = state + (b * H + h) * dk * dv;
            for (int64_t c = 0; c < nchunks; ++c) {
                const int64_t t0 = c * C, t1 = (c + 1) * C < T ? (c + 1) * C : T;
                const double g = gate[(b * H + h) * nchunks + c];
                for (int64_t i = 0; i < dk * dv; ++i) S[i] *= g;
                for (int64_t t = t0; t < t1; ++t)
                    for (int64_t i = 0; i < dk; ++i) {
                        const double ki = ld(k, dt, ((b * T + t) * H + h) * dk + i);
                        for (int64_t j = 0; j < dv; ++j)
                            S[i * dv + j] += ki * ld(v, dt, ((b * T + t) * H + h) * dv + j);
                    }
                for (int64_t t = t0; t < t1; ++t)
                    for (int64_t j = 0; j < dv; ++j) {
                        double acc = 0.0;
                        for (int64_t i = 0; i < dk; ++i)
                            acc += ld(q, dt, ((b * T + t) * H + h) * dk + i) * S[i * dv + j];
                        out[((b * T + t) * H + h) * dv + j] = acc;
                    }
            }
        }
    return nomem ? ORC_NOMEM : ORC_OK;
}
