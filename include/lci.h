/*
 * lci.h -- C ABI of the B200 sparse-attention index pipeline (liblci.so).
 *
 * The library implements one layer of index-selected sparse attention for long
 * contexts, as described by three web pages:
 *   [GPU-stack] "Day-0 Inference Adaptation for Ultra-Large MoE Models on
 *               Domestic GPUs: A Software Stack Perspective"
 *   [AI-acc]    "Day-0 Inference Adaptation of Ultra-Large-Scale MoE Models on
 *               Domestic AI Accelerators"
 *   [Hetero]    "Day-0 Adaptation for Trillion-Parameter MoE Models: A
 *               Comprehensive Guide to Heterogeneous Compute Deployment"
 *
 * Pipeline: compressed block keys k_c are scored against compressed queries
 * q_c (summed over indexer heads), every query keeps the top-k causal-visible
 * blocks, and exact softmax attention runs over the tokens of those blocks,
 * gathered from a paged KV pool through a block table. Prefill (many queries
 * per sequence) and decode (one query per sequence) share one representation:
 * int32 block ids in rank order plus the block table.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * - Pointers named d_* and all tensor arguments are DEVICE pointers on the
 *   current CUDA device; the caller allocates and owns them. The library keeps
 *   no reference to them after a call returns (except the block table object,
 *   which records the table pointer it is given; see below).
 * - Layouts are dense row-major, innermost index last, with no padding.
 *   Floating tensors of one call share one element type (lci_dtype).
 * - `stream` is a cudaStream_t passed as void*; NULL is the legacy default
 *   stream. Every launch is asynchronous on it. No entry point synchronises,
 *   except lci_get_device_status.
 * - Host-detectable argument errors return a status before anything is
 *   launched; lci_last_error() then describes the problem. Launch calls make
 *   no device allocation: scratch memory is the caller's workspace.
 * - Device-side checks (block ids outside [-1, nb_max), table entries outside
 *   [0, num_pages)) never trap: the offending item is skipped, a sticky device
 *   status word is set, and lci_get_device_status reports it.
 * - Every device-side wait (a copy landing in shared memory, a row published
 *   by a producer) is bounded by a wait limit (lci_set_wait_limit_ns, 2 s by
 *   default). A wait that runs out skips its work, sets the sticky status word
 *   and lets the kernel return; lci_get_device_status then reports
 *   LCI_ERR_TIMEOUT. No kernel of the library can wait forever.
 * - Query position: p = d_q_start[b] + s for query s of sequence b. The last
 *   attendable token is last = min(p, d_ctx_len[b] - 1). Block j is causal-
 *   visible when j * block_size <= last (so vis = min(nb_max, last/bs + 1)).
 */
#ifndef LCI_H
#define LCI_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define LCI_API __attribute__((visibility("default")))
#else
#define LCI_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    LCI_OK = 0,
    LCI_ERR_INVALID_ARG = 1,   /* null pointer, bad size or inconsistent shapes */
    LCI_ERR_UNSUPPORTED = 2,   /* valid arguments outside what the kernels cover */
    LCI_ERR_WORKSPACE = 3,     /* workspace missing, misaligned or too small */
    LCI_ERR_CUDA = 4,          /* a CUDA runtime call failed (see lci_last_error) */
    LCI_ERR_DEVICE_BOUNDS = 5, /* a device-side bounds check fired (sticky word) */
    LCI_ERR_TIMEOUT = 6        /* a bounded device wait gave up (sticky word) */
} lci_status;

typedef enum { LCI_F32 = 0, LCI_BF16 = 1 } lci_dtype;

/* Which kernel family runs. AUTO: DECODE when S == 1, PREFILL otherwise.
 * Both produce identical block ids for identical inputs ([GPU-stack],
 * "Separate Paths for Prefill and Decode": two schedules, one representation). */
typedef enum { LCI_PHASE_AUTO = 0, LCI_PHASE_PREFILL = 1, LCI_PHASE_DECODE = 2 } lci_phase;

typedef struct lci_block_table lci_block_table; /* opaque, host-side */

/* Library version string ("major.minor.patch"). */
LCI_API const char* lci_version(void);

/* Static description of a status code. */
LCI_API const char* lci_status_string(lci_status status);

/* Message of the last failing call on this host thread ("" when none). */
LCI_API const char* lci_last_error(void);

/*
 * Block table of a paged KV cache ([GPU-stack] "Reorganizing KV Cache Layout";
 * [Hetero] §II and §IV, KV pages addressed through a page table).
 *
 *   d_table      [batch][max_blocks] int32, device. Entry (b, j) is the pool
 *                page that holds logical block j (tokens j*block_size ..
 *                (j+1)*block_size-1) of sequence b. The object records this
 *                pointer without copying; the caller keeps the memory alive and
 *                may update its contents between calls.
 *   num_pages    pages in each KV pool.
 *   block_size   tokens per page.
 *   num_kv_heads, head_dim, kv_dtype: shape and type of the pools
 *                K, V = [num_pages][num_kv_heads][block_size][head_dim].
 * Allocates only the host object. Returns LCI_ERR_INVALID_ARG on a null
 * pointer or a non-positive size.
 */
LCI_API lci_status lci_create_block_table(const int32_t* d_table, int32_t batch, int32_t max_blocks,
                                  int32_t num_pages, int32_t block_size, int32_t num_kv_heads,
                                  int32_t head_dim, lci_dtype kv_dtype, lci_block_table** out);

/* Frees the host object (never the caller's table memory). NULL is a no-op. */
LCI_API lci_status lci_destroy_block_table(lci_block_table* table);

/*
 * Bounds-checks every table entry against [0, num_pages) on the device.
 * Violations set the sticky device status word (see lci_get_device_status).
 */
LCI_API lci_status lci_validate_block_table(const lci_block_table* table, void* stream);

/*
 * A0 -- block compression ([GPU-stack] "Adapting Sparse Attention", the
 * representation-generation stage; [AI-acc] §4.1, k_comp):
 *   k_c[b][j][h][d] = mean over the tokens t of block j of k_idx[b][t][h][d]
 * with block j = tokens [j*block_size, min(tokens, (j+1)*block_size)).
 *   k_idx  [batch][tokens][heads][dim], device, dtype
 *   k_c    [batch][ceil(tokens/block_size)][heads][dim], device, dtype (output)
 * Sums in fp32, divides by the token count, rounds once to dtype.
 */
LCI_API lci_status lci_block_compress(const void* k_idx, lci_dtype dtype, int32_t batch, int32_t tokens,
                              int32_t heads, int32_t dim, int32_t block_size, void* k_c,
                              void* stream);

/*
 * Workspace bytes lci_index_select needs for these sizes, for either dtype
 * (0 is possible). With LCI_PHASE_DECODE it is the scratch of the
 * one-row-at-a-time schedule alone, which lci_index_select_noalloc uses.
 */
LCI_API lci_status lci_index_select_workspace_size(int32_t batch, int32_t S, int32_t H_i, int32_t d_c,
                                           int32_t nb_max, int32_t topk, lci_phase phase,
                                           size_t* bytes);

/*
 * A1 + A2 -- block scoring fused with the causal-masked top-k
 * ([GPU-stack] "Operatorizing Index Selection": scoring, top-k and masking in
 * one operator; [AI-acc] §4.1, matmul of compressed queries and keys followed
 * by an on-device top-k that avoids a full sort):
 *   score[b][s][j] = sum_h sum_d q_c[b][s][h][d] * k_c[b][j][h][d]   (j < vis)
 *   d_ids[b][s][0 .. min(topk, vis)) = visible block ids ranked by
 *       (score descending, block id ascending); the rest of the row is -1.
 *   q_c        [batch][S][H_i][d_c], device, dtype
 *   k_c        [batch][nb_max][H_i][d_c], device, dtype
 *   d_ctx_len  [batch] int32, d_q_start [batch] int32, device
 *   d_ids      [batch][S][topk] int32, device (output)
 *   workspace  >= lci_index_select_workspace_size bytes, 256-byte aligned.
 *              It starts with arrival counters and per-row selection bounds
 *              whose position depends on (batch, S) alone; scratch follows.
 *              Zero-fill a workspace before its first call; every successful
 *              call leaves that prefix at zero again, so later calls with the
 *              same (batch, S) need no clearing, whatever their dtype, topk,
 *              nb_max or phase (the workspace must still be large enough).
 *              Zero it again before using it with another (batch, S), and
 *              after a call that failed on the device. Calls that share a
 *              workspace must not overlap in time.
 * Scores are accumulated in fp32. Limits: 1 <= topk <= 256,
 * nb_max <= 16384, H_i*d_c <= 8192 and a multiple of 8 (bf16) or 4 (f32).
 */
LCI_API lci_status lci_index_select(const void* q_c, const void* k_c, lci_dtype dtype, int32_t batch,
                            int32_t S, int32_t H_i, int32_t d_c, int32_t block_size,
                            int32_t nb_max, const int32_t* d_ctx_len, const int32_t* d_q_start,
                            int32_t topk, lci_phase phase, int32_t* d_ids, void* workspace,
                            size_t workspace_bytes, void* stream);

/*
 * A0 online, over a paged pool ([GPU-stack] "Adapting Sparse Attention": the
 * representation-generation stage; [GPU-stack] "Reorganizing KV Cache
 * Layout": block-level caching shared between prefill and decode). The block
 * keys live beside the KV pages, one per page, addressed through the same
 * block table:
 *   kc     [num_pages][H_i][d_c], dtype   (the key of the block held by a page)
 *   kc_sum [num_pages][H_i*d_c] fp32      (running sum of the block's tokens)
 * T new tokens of every sequence b, at positions d_start[b] .. d_start[b]+T-1,
 * enter the cache with indexer keys k_idx [batch][T][H_i][d_c] (device,
 * dtype). Every block they touch, at page table[b][block], gets
 *   kc_sum[page] = (the block's earlier tokens' sum if it already held tokens
 *                   before d_start[b], else 0) + the new tokens' sum
 *   kc[page]     = kc_sum[page] / (tokens of the block now present)
 * (fp32 sums, the quotient formed in fp64 and rounded once to dtype). T = 1
 * is the decode step; a chunk of T tokens is prefill. After any sequence of
 * calls that fills positions 0..n-1 in order, kc equals lci_block_compress of
 * those n tokens (exactly, for inputs whose fp32 sums are exact, such as
 * multiples of 1/16 of magnitude <= 2 in blocks of up to 2^17 tokens).
 * A block index >= max_blocks or a page outside [0, num_pages) is skipped and
 * sets the device status word. Calls for the same sequence must be in order.
 */
LCI_API lci_status lci_kc_update(const void* k_idx, lci_dtype dtype, int32_t batch, int32_t T,
                                 int32_t H_i, int32_t d_c, const int32_t* d_start,
                                 const lci_block_table* table, float* kc_sum, void* kc,
                                 void* stream);

/*
 * Workspace bytes lci_index_select_paged needs for these sizes.
 */
LCI_API lci_status lci_index_select_paged_workspace_size(int32_t batch, int32_t S, int32_t H_i,
                                                         int32_t d_c, int32_t topk,
                                                         const lci_block_table* table,
                                                         lci_dtype dtype, lci_phase phase,
                                                         size_t* bytes);

/*
 * lci_index_select with the block keys read from the paged pool kc
 * [num_pages][H_i][d_c] through the block table: block j of sequence b is
 * scored with kc[table[b][j]] (nb_max and block_size are the table's). Same
 * results as lci_index_select on the gathered dense keys. The decode schedule
 * reads each block's key at its page directly; the tensor-core prefill
 * schedule first gathers the keys of cached blocks into the workspace.
 * Workspace: lci_index_select_paged_workspace_size bytes, 256-byte aligned,
 * with lci_index_select's zero-fill rule.
 */
LCI_API lci_status lci_index_select_paged(const void* q_c, const void* kc, lci_dtype dtype,
                                          int32_t batch, int32_t S, int32_t H_i, int32_t d_c,
                                          const lci_block_table* table, const int32_t* d_ctx_len,
                                          const int32_t* d_q_start, int32_t topk, lci_phase phase,
                                          int32_t* d_ids, void* workspace, size_t workspace_bytes,
                                          void* stream);

/*
 * Workspace bytes lci_sparse_attn needs for these sizes (0 is possible).
 */
LCI_API lci_status lci_sparse_attn_workspace_size(int32_t batch, int32_t S, int32_t H_q, int32_t topk,
                                          const lci_block_table* table, lci_phase phase,
                                          size_t* bytes);

/*
 * A3 + A4 -- paged gather and exact sparse attention ([AI-acc] §4.1, exact
 * attention over the selected positions only; [Hetero] §IV, gather of the
 * selected KV pages, then a compute-heavy prefill or memory-heavy decode
 * kernel). For query head h (KV head g = h / (H_q / num_kv_heads)):
 *   T   = { t : t / block_size is one of d_ids[b][s][*], t <= last }
 *   out = sum_{t in T} softmax_t(scale * q . K_t) V_t ,  K_t, V_t read at
 *         pool[table[b][t / block_size]][g][t % block_size][:]
 * An empty T gives a zero row. Rows of d_ids may be in any order, may hold -1
 * entries anywhere, and must not repeat a block.
 *   q        [batch][S][H_q][head_dim], device, dtype = the table's kv_dtype
 *   k_pool, v_pool  [num_pages][num_kv_heads][block_size][head_dim], device
 *   d_ids    [batch][S][topk] int32, device
 *   scale    softmax scale; <= 0 selects 1/sqrt(head_dim)
 *   out      [batch][S][H_q][head_dim], device, dtype (output)
 *   workspace >= lci_sparse_attn_workspace_size bytes, 256-byte aligned; the
 *             same zero-fill rule as lci_index_select (per set of sizes).
 * Softmax and accumulation are fp32; bf16 inputs feed the tensor cores.
 * Limits: H_q a multiple of num_kv_heads, head_dim a multiple of 32 and
 * <= 256, topk <= 256.
 */
LCI_API lci_status lci_sparse_attn(const void* q, int32_t batch, int32_t S, int32_t H_q,
                           const void* k_pool, const void* v_pool, const lci_block_table* table,
                           const int32_t* d_ids, int32_t topk, const int32_t* d_ctx_len,
                           const int32_t* d_q_start, float scale, lci_phase phase, void* out,
                           void* workspace, size_t workspace_bytes, void* stream);

/*
 * Context parallelism: one long context split into block ranges over several
 * GPUs ([AI-acc] §3: communication libraries for multi-card inference;
 * [Hetero] §VII: communication overlap). Each rank holds the block keys and
 * KV pages of its range [j_lo, j_hi) and runs the steps below; the caller
 * exchanges the small per-query results between ranks (an all-gather).
 *
 * 1. lci_index_select on the rank's keys with positions shifted by -j_lo*bs
 *    (q_start - j_lo*bs, ctx_len - j_lo*bs): the rank's local top-k.
 *    lci_ids_shift(lo=0, hi=j_hi-j_lo, offset=+j_lo) makes the ids global and
 *    lci_block_scores_at gives their scores.
 * 2. After gathering every rank's (scores, ids), lci_topk_merge yields the
 *    global top-k, identical on every rank and equal to the one-GPU result:
 *    the global top-k lies in the union of the local ones.
 * 3. lci_ids_shift(lo=j_lo, hi=j_hi, offset=-j_lo) keeps the selected blocks
 *    the rank holds; lci_sparse_attn_partial attends over them and returns the
 *    normalised output and its log-sum-exp.
 * 4. After gathering every rank's (out, lse), lci_attn_merge combines them.
 */

/*
 * scores[b][s][i] = sum_h sum_d q_c[b][s][h][d] * k_c[b][ids[b][s][i]][h][d]
 * (fp32), -inf where the id is -1. Layouts as lci_index_select; d_scores
 * [batch][S][topk] float, device (output). An id outside [-1, nb_max) is
 * scored -inf and sets the device status word.
 */
LCI_API lci_status lci_block_scores_at(const void* q_c, const void* k_c, lci_dtype dtype,
                                       int32_t batch, int32_t S, int32_t H_i, int32_t d_c,
                                       int32_t nb_max, const int32_t* d_ids, int32_t topk,
                                       float* d_scores, void* stream);

/*
 * d_out[i] = (lo <= d_ids[i] < hi) ? d_ids[i] + offset : -1 for i < n
 * (device arrays of int32; in place is allowed).
 */
LCI_API lci_status lci_ids_shift(const int32_t* d_ids, int64_t n, int32_t lo, int32_t hi,
                                 int32_t offset, int32_t* d_out, void* stream);

/*
 * Top-k of nlists ranked lists per row. d_scores, d_ids [nlists][rows][topk]
 * (device): list r of a row holds block ids in rank order (score descending,
 * id ascending), ended by -1. d_out [rows][topk] int32 (device): the best topk
 * ids of the union by the same order, -1 padded. nlists <= 64.
 */
LCI_API lci_status lci_topk_merge(const float* d_scores, const int32_t* d_ids, int32_t nlists,
                                  int64_t rows, int32_t topk, int32_t* d_out, void* stream);

/*
 * lci_sparse_attn that also returns, per query row and head, the log2 of the
 * sum of 2^(scale*log2(e)*q.k) over the attended tokens (the log-sum-exp of
 * the scaled logits in base 2): d_lse [batch][S][H_q] float (device), -inf
 * where no token is attended (the output row is then zero). Supported shape:
 * bf16 pools, head_dim 128, block_size a multiple of 64, at most 16 query
 * heads per KV head (else LCI_ERR_UNSUPPORTED). Needs no workspace.
 */
LCI_API lci_status lci_sparse_attn_partial(const void* q, int32_t batch, int32_t S, int32_t H_q,
                                           const void* k_pool, const void* v_pool,
                                           const lci_block_table* table, const int32_t* d_ids,
                                           int32_t topk, const int32_t* d_ctx_len,
                                           const int32_t* d_q_start, float scale, lci_phase phase,
                                           void* out, float* d_lse, void* stream);

/*
 * Exact combination of nlists partial attention results:
 *   out[x][:] = sum_r w_r o[r][x][:] / sum_r w_r,  w_r = 2^(lse[r][x] - max_r lse[r][x])
 * for every (row, head) x; zero where every lse is -inf.
 *   d_o   [nlists][rows_heads][head_dim], dtype (device)
 *   d_lse [nlists][rows_heads] float (device)
 *   d_out [rows_heads][head_dim], dtype (device, output)
 */
LCI_API lci_status lci_attn_merge(const void* d_o, const float* d_lse, lci_dtype dtype,
                                  int32_t nlists, int64_t rows_heads, int32_t head_dim,
                                  void* d_out, void* stream);

/*
 * lci_index_select without any device allocation. The reference pages have no
 * counterpart; this entry point exists for callers that are not allowed to
 * allocate device memory or to hold a workspace of their own: for example code
 * running inside a host framework that owns every device allocation (a plugin
 * or an engine with a pre-planned memory arena) and so cannot call cudaMalloc
 * or keep a separate scratch buffer per call site.
 *
 * Same arguments, layouts, results and limits as lci_index_select, minus the
 * workspace; it always runs the one-row-at-a-time kernel (the decode schedule)
 * whatever the phase. Its scratch is one fixed array of
 * LCI_NOALLOC_SCRATCH_BYTES bytes inside the library, which every GPU that
 * loads the library holds until the process exits. The scratch a call needs is
 *   align256(4*batch*ceil(S/128)) + align256(4*rows) + align256(4*rows*nb_max)
 *   + align256(4*rows*nchunks)
 * bytes (rows = batch*S; nchunks <= nb_max, the chunks a row is scored in),
 * which is exactly what lci_index_select_workspace_size returns for the same
 * sizes with LCI_PHASE_DECODE. Sizes whose scratch exceeds the array return
 * LCI_ERR_WORKSPACE before anything is launched.
 * Every call looks up the array's device address for the current device (the
 * first lookup on a device may load the library's device code: make the first
 * call on each device before any stream capture). Each call
 * clears the array's arrival counters on `stream` before its kernel runs (the
 * array keeps the previous call's contents otherwise). All calls on a device
 * share the one array: calls that may overlap on the GPU (other streams, other
 * host threads) race and corrupt each other's results. The caller still passes
 * and owns all inputs and outputs. No cudaMalloc or cudaFree is ever called.
 */
#define LCI_NOALLOC_SCRATCH_BYTES (8u << 20)
LCI_API lci_status lci_index_select_noalloc(const void* q_c, const void* k_c, lci_dtype dtype,
                                            int32_t batch, int32_t S, int32_t H_i, int32_t d_c,
                                            int32_t block_size, int32_t nb_max,
                                            const int32_t* d_ctx_len, const int32_t* d_q_start,
                                            int32_t topk, lci_phase phase, int32_t* d_ids,
                                            void* stream);

/*
 * Workspace bytes lci_sparse_decode needs for these sizes and this block table
 * (nb_max is the table's max_blocks).
 */
LCI_API lci_status lci_sparse_decode_workspace_size(int32_t batch, int32_t S, int32_t H_i,
                                                    int32_t d_c, int32_t topk, int32_t H_q,
                                                    const lci_block_table* table, size_t* bytes);

/*
 * One decode step in one call: lci_index_select (one-row-at-a-time schedule)
 * followed by lci_sparse_attn, with identical block ids and outputs within the
 * attention tolerance. [GPU-stack] "Separate Paths for Prefill and Decode" asks
 * that decode pipeline index prefetching with incremental aggregation; [Hetero]
 * §IV that index retrieval and attention be pipelined to hide retrieval
 * latency. The indexer publishes each query row as soon as its block ids are
 * final, and the attention kernel, launched behind it (programmatic dependent
 * launch), starts on a row as soon as that row is published, while later rows
 * are still being scored. For 2 KiB block keys (H_i*d_c*element size = 2048)
 * a row is published as its picks, (block id, page) pairs in the workspace
 * that the attention's producer polls one by one and turns straight into tile
 * loads; for other key sizes as a flag per row.
 * Arguments are those of the two calls; k_c's nb_max must equal the table's
 * max_blocks and all floating inputs share one dtype. The workspace holds the
 * scratch, the per-row publications and the per-call counters: zero-fill it
 * before its first call and again before using it with other sizes or after a
 * call that failed on the device; every successful call leaves it ready for
 * the next. A publication left by an earlier call is never taken for a new
 * one (the indexer resets it before the attention kernel can start). Calls
 * sharing a workspace must not overlap in time.
 */
LCI_API lci_status lci_sparse_decode(const void* q_c, const void* k_c, lci_dtype dtype,
                                     int32_t batch, int32_t S, int32_t H_i, int32_t d_c,
                                     int32_t nb_max, const int32_t* d_ctx_len,
                                     const int32_t* d_q_start, int32_t topk, const void* q,
                                     int32_t H_q, const void* k_pool, const void* v_pool,
                                     const lci_block_table* table, float scale, int32_t* d_ids,
                                     void* out, void* workspace, size_t workspace_bytes,
                                     void* stream);

/*
 * A3 + A4 with the attention of each query row started as soon as a producer
 * publishes that row ([Hetero] §IV: index retrieval and attention should be
 * pipelined so that retrieval latency is hidden; [GPU-stack] "Separate Paths
 * for Prefill and Decode": decode as a pipeline of index prefetching and
 * incremental aggregation). This is the consumer half of lci_sparse_decode for
 * callers that produce the block ids themselves, in a kernel running on
 * another stream or earlier on this one.
 *   d_ready  [batch][S] uint32, device. The producer writes row r of d_ids,
 *            then sets d_ready[r] to a nonzero value with release semantics
 *            (st.release.gpu, or a __threadfence() before a plain store). The
 *            library only reads d_ready; the caller clears it between calls.
 * Other arguments, layouts and results are those of lci_sparse_attn. A row
 * whose flag stays zero for the wait limit (lci_set_wait_limit_ns) gets a
 * zero output row, and lci_get_device_status reports LCI_ERR_TIMEOUT.
 * Supported shape (else LCI_ERR_UNSUPPORTED): bf16 pools, head_dim 128,
 * block_size a multiple of 64, at most 16 query heads per KV head.
 */
LCI_API lci_status lci_sparse_attn_pipelined(const void* q, int32_t batch, int32_t S, int32_t H_q,
                                             const void* k_pool, const void* v_pool,
                                             const lci_block_table* table, const int32_t* d_ids,
                                             int32_t topk, const int32_t* d_ctx_len,
                                             const int32_t* d_q_start, float scale,
                                             const uint32_t* d_ready, void* out, void* stream);

/*
 * Limit, in nanoseconds of GPU global time, of every bounded device wait of
 * the library on the current device (default 2 s; 1 ns .. 60 s, else
 * LCI_ERR_INVALID_ARG). Takes effect for kernels launched after the call;
 * not for use during stream capture.
 */
LCI_API lci_status lci_set_wait_limit_ns(uint64_t ns);
LCI_API lci_status lci_get_wait_limit_ns(uint64_t* ns);

/*
 * N4 -- chunked gated state scan of the linear-attention family ([Hetero]
 * §II: gated incremental state updates maintained across strides; §III: the
 * state scanned over the sequence in chunks, updated by the gate and k^T v,
 * read out by q). For every sequence b and head h, with S [dk][dv] starting
 * at state_in[b][h] and chunk c holding tokens [c*chunk, min(T, (c+1)*chunk)):
 *   S      = gate[b][h][c] * S + sum_{t in chunk c} k[b][t][h]^T v[b][t][h]
 *   out[b][t][h] = q[b][t][h] S            for every t in chunk c
 * (the readout sees the chunk's own update); state_out[b][h] = the final S.
 *   q, k   [batch][T][H][dk], v [batch][T][H][dv], dtype (device)
 *   d_gate [batch][H][ceil(T/chunk)] float (device)
 *   d_state_in, d_state_out [batch][H][dk][dv] float (device; may be the same
 *          array: the update is then in place)
 *   d_out  [batch][T][H][dv] float (device, output)
 * The state stays in fp32 in TMEM; the readout multiplies q by the state split
 * into two bf16 parts (hi + lo, relative error about 2^-17). Supported: bf16,
 * dk = dv = 128, chunk = 128 (else LCI_ERR_UNSUPPORTED).
 */
LCI_API lci_status lci_gated_state_scan(const void* q, const void* k, const void* v,
                                        lci_dtype dtype, const float* d_gate,
                                        const float* d_state_in, float* d_state_out,
                                        int32_t batch, int32_t T, int32_t H, int32_t dk,
                                        int32_t dv, int32_t chunk, float* d_out, void* stream);

/*
 * Synchronises `stream`, then returns and clears the sticky device status
 * word of the current device: LCI_OK; LCI_ERR_TIMEOUT when a bounded device
 * wait ran out since the last call; otherwise LCI_ERR_DEVICE_BOUNDS when a
 * device bounds check fired. lci_last_error() lists every flag that was set.
 */
/*
 * The same decode step as lci_sparse_decode in ONE persistent launch: about
 * one CTA per SM claims work items from a global counter, first the scoring
 * chunks of the query rows (the last chunk of a row to finish selects the
 * row's blocks and publishes it), then attention splits of (row, KV head)
 * pairs whose rows are published, while later rows are still being scored;
 * the last split of a pair to finish combines the splits. A CTA claims
 * attention work only after every scoring item has been claimed by a running
 * CTA, and scoring never waits, so the launch completes whatever the
 * residency. Same arguments, results (ids identical, outputs within the
 * attention tolerance) and workspace as lci_sparse_decode; the workspace also
 * keeps the per-call counters and an epoch, which every call leaves ready for
 * the next. Supported (else LCI_ERR_UNSUPPORTED): bf16, H_i*d_c = 1024,
 * head_dim 128, block_size a multiple of 64, at most 16 query heads per KV
 * head, 16-byte aligned pools.
 */
LCI_API lci_status lci_sparse_decode_persistent(const void* q_c, const void* k_c, lci_dtype dtype,
                                                int32_t batch, int32_t S, int32_t H_i,
                                                int32_t d_c, int32_t nb_max,
                                                const int32_t* d_ctx_len, const int32_t* d_q_start,
                                                int32_t topk, const void* q, int32_t H_q,
                                                const void* k_pool, const void* v_pool,
                                                const lci_block_table* table, float scale,
                                                int32_t* d_ids, void* out, void* workspace,
                                                size_t workspace_bytes, void* stream);

LCI_API lci_status lci_get_device_status(void* stream);

#ifdef __cplusplus
}
#endif

#endif /* LCI_H */
