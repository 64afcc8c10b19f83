// lci.cu -- C ABI of the sparse-attention index pipeline (see include/lci.h).
//
// Host side only: argument checks, workspace layout, kernel selection and
// launches. Every step of the computation runs in the kernels included below.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <mutex>
#include <new>
#include <string>

#include "../../include/lci.h"
#include "attn_decode.cuh"
#include "attn_prefill.cuh"
#include "attn_simt.cuh"
#include "common.cuh"
#include "compress.cuh"
#include "cp_merge.cuh"
#include "decode_fused.cuh"
#include "index_gemv.cuh"
#include "index_prefill.cuh"
#include "state_scan.cuh"
#include "topk_select.cuh"

struct lci_block_table {
    const int32_t* d_table;
    int32_t batch, max_blocks, num_pages, block_size, num_kv_heads, head_dim;
    lci_dtype dtype;
    // TMA descriptors of the last pool pair the table was used with: a decode
    // loop calls with the same pools every step, so they are encoded once
    std::mutex map_mu;
    const void* map_k_pool = nullptr;
    const void* map_v_pool = nullptr;
    CUtensorMap map_k, map_v;
};

namespace {

thread_local std::string t_last_error;

lci_status fail(lci_status st, const char* fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof buf, fmt, ap);
    va_end(ap);
    t_last_error = buf;
    return st;
}

lci_status ok() {
    t_last_error.clear();
    return LCI_OK;
}

lci_status check_launch(const char* what) {
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return fail(LCI_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
    return ok();
}

constexpr size_t kAlign = 256;
constexpr uint64_t kMaxWaitLimitNs = 60ull * 1000000000ull;  // 60 s
size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

bool dtype_ok(lci_dtype d) { return d == LCI_F32 || d == LCI_BF16; }
size_t dtype_size(lci_dtype d) { return d == LCI_F32 ? 4 : 2; }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

lci_phase resolve_phase(lci_phase ph, int32_t S) {
    if (ph == LCI_PHASE_AUTO) return S == 1 ? LCI_PHASE_DECODE : LCI_PHASE_PREFILL;
    return ph;
}

// ------------------------------------------------------------ index_select

constexpr int kIndexThreads = 256;
constexpr int kMaxNbMax = 16384;
constexpr int kMaxIndexK = 8192;
constexpr int kIndexMaxSmem = 65536 + 1024;

struct IndexPlan {
    int chunk_blocks, nchunks;
    bool qreg;  // 2 KiB block keys: query slice in registers
    // 2 KiB block keys take the streaming kernel: chunk maxima every s_chunk
    // blocks, s_nchunks per row (never more than the layout holds)
    bool stream;
    int s_chunk, s_nchunks;
    size_t off_counters, off_scores, off_chunk_max, bytes;
    size_t smem;
};

// Blocks per chunk: at most 32 blocks and 32 KiB of block keys, halved while
// the grid would not cover the 148 SMs about four times.
int index_chunk(long long rows, int32_t K, int32_t nb_max, size_t esz) {
    const size_t row_bytes = (size_t)K * esz;
    int chunk = 32;
    while (chunk > 1 && (size_t)chunk * row_bytes > 32768) chunk >>= 1;
    while (chunk > 4 && rows * ((nb_max + chunk - 1) / chunk) < 4 * 148) chunk >>= 1;
    return chunk;
}

// Every index_select schedule keeps the state that must start at zero (arrival
// counters, per-row selection bounds) in one prefix of the workspace whose
// size depends on (batch, S) alone, and its scratch after it. Each schedule
// leaves its own zero state at zero after a successful call and writes no
// scratch inside the prefix, so a workspace serves calls of any dtype, topk
// or schedule for the same (batch, S) without clearing.
size_t index_zero_prefix(int32_t batch, int32_t S) {
    const long long m_tiles = (S + lci::pre::kBM - 1) / lci::pre::kBM;
    return align_up((size_t)batch * m_tiles * sizeof(unsigned int)) +
           align_up((size_t)batch * S * sizeof(unsigned int));
}

IndexPlan plan_index(int32_t batch, int32_t S, int32_t K, int32_t nb_max, size_t esz) {
    IndexPlan pl{};
    const long long rows = (long long)batch * S;
    const size_t row_bytes = (size_t)K * esz;
    const int chunk = index_chunk(rows, K, nb_max, esz);
    pl.chunk_blocks = chunk;
    pl.nchunks = (nb_max + chunk - 1) / chunk;
    // The layout is sized for the smaller fp32 chunk, so that one workspace
    // size serves both element types.
    const int nchunks_alloc = (nb_max + index_chunk(rows, K, nb_max, 4) - 1) / index_chunk(rows, K, nb_max, 4);
    pl.off_counters = 0;  // rows counters, inside the zero prefix
    pl.off_scores = index_zero_prefix(batch, S);
    pl.off_chunk_max = pl.off_scores + align_up((size_t)rows * nb_max * sizeof(float));
    pl.bytes = pl.off_chunk_max + align_up((size_t)rows * nchunks_alloc * sizeof(uint32_t));
    pl.qreg = row_bytes == 2048;
    pl.stream = row_bytes == 2048;
    pl.s_chunk = std::max(8, index_chunk(rows, K, nb_max, 4));
    while ((nb_max + pl.s_chunk - 1) / pl.s_chunk > lci::kMaxChunks) pl.s_chunk *= 2;
    pl.s_nchunks = (nb_max + pl.s_chunk - 1) / pl.s_chunk;
    const size_t stage = (size_t)chunk * row_bytes + (pl.qreg ? 0 : (size_t)K * sizeof(float));
    const size_t sel = sizeof(lci::SelectSmem);
    pl.smem = stage > sel ? stage : sel;
    return pl;
}

lci_status check_index_args(int32_t batch, int32_t S, int32_t H_i, int32_t d_c, int32_t nb_max,
                            int32_t topk, lci_dtype dtype) {
    if (batch <= 0 || S <= 0 || H_i <= 0 || d_c <= 0 || nb_max <= 0)
        return fail(LCI_ERR_INVALID_ARG, "index_select: sizes must be positive "
                    "(batch=%d S=%d H_i=%d d_c=%d nb_max=%d)", batch, S, H_i, d_c, nb_max);
    if (topk <= 0) return fail(LCI_ERR_INVALID_ARG, "index_select: topk must be positive (%d)", topk);
    if (!dtype_ok(dtype)) return fail(LCI_ERR_INVALID_ARG, "index_select: unknown dtype %d", (int)dtype);
    if (topk > lci::kMaxTopk)
        return fail(LCI_ERR_UNSUPPORTED, "index_select: topk %d above %d", topk, lci::kMaxTopk);
    if (nb_max > kMaxNbMax)
        return fail(LCI_ERR_UNSUPPORTED, "index_select: nb_max %d above %d", nb_max, kMaxNbMax);
    const long long K = (long long)H_i * d_c;
    const int vec = dtype == LCI_BF16 ? 8 : 4;
    if (K > kMaxIndexK || K % vec != 0)
        return fail(LCI_ERR_UNSUPPORTED, "index_select: H_i*d_c=%lld must be <= %d and a multiple "
                    "of %d", K, kMaxIndexK, vec);
    return LCI_OK;
}

// CTAs of the streaming index kernel the device holds at once.
template <typename T>
int index_stream_slots() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 0;
    static std::mutex mu;
    static int slots[64] = {0};
    std::lock_guard<std::mutex> lock(mu);
    if (dev < 0 || dev >= 64) return 0;
    if (slots[dev] == 0) {
        int sms = 0, per_sm = 0;
        if (cudaFuncSetAttribute(lci::index_stream_select_kernel<T, kIndexThreads>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 lci::ixs::smem_bytes<kIndexThreads>()) != cudaSuccess ||
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
            cudaOccupancyMaxActiveBlocksPerMultiprocessor(
                &per_sm, lci::index_stream_select_kernel<T, kIndexThreads>, kIndexThreads,
                lci::ixs::smem_bytes<kIndexThreads>()) != cudaSuccess)
            return 0;
        slots[dev] = sms * std::max(1, per_sm);
    }
    return slots[dev];
}

template <typename T>
lci_status launch_index_stream(const void* q_c, const void* k_c, int32_t batch, int32_t S,
                               int32_t bs, int32_t nb_max, const int32_t* ctx_len,
                               const int32_t* q_start, int32_t topk, int32_t* ids, void* ws,
                               const IndexPlan& pl, cudaStream_t st, unsigned int* ready,
                               const int32_t* page_table, int32_t num_pages, const int32_t* table,
                               unsigned long long* picks) {
    const long long rows = (long long)batch * S;
    const int slots = index_stream_slots<T>();
    if (slots <= 0) return fail(LCI_ERR_CUDA, "index_select: device query failed");
    // Blocks per CTA: whole chunks, as few as keep every CTA resident at once,
    // and at most 64 chunks (the chunk maxima one CTA records).
    const long long per_row = std::max(1ll, slots / rows);
    const long long units = (nb_max + pl.s_chunk - 1) / pl.s_chunk;
    long long cta_units = (units + per_row - 1) / per_row;
    cta_units = std::min(std::max(cta_units, 1ll), 64ll);
    const int cta_blocks = (int)(cta_units * pl.s_chunk);
    const int ncta = (nb_max + cta_blocks - 1) / cta_blocks;
    const long long grid = rows * ncta;
    if (grid >= (1ll << 31)) return fail(LCI_ERR_UNSUPPORTED, "index_select: grid too large");
    char* w = static_cast<char*>(ws);
    lci::index_stream_select_kernel<T, kIndexThreads>
        <<<(unsigned)grid, kIndexThreads, lci::ixs::smem_bytes<kIndexThreads>(), st>>>(
            static_cast<const T*>(q_c), static_cast<const T*>(k_c), S, nb_max, bs, ctx_len, q_start,
            topk, pl.s_chunk, cta_blocks, ncta, pl.s_nchunks,
            reinterpret_cast<float*>(w + pl.off_scores), reinterpret_cast<uint32_t*>(w + pl.off_chunk_max),
            reinterpret_cast<unsigned int*>(w + pl.off_counters), ids, ready, page_table, num_pages,
            table, picks);
    return check_launch("index_select");
}

template <typename T>
lci_status launch_index_gemv(const void* q_c, const void* k_c, int32_t batch, int32_t S, int32_t K,
                             int32_t bs, int32_t nb_max, const int32_t* ctx_len,
                             const int32_t* q_start, int32_t topk, int32_t* ids, void* ws,
                             const IndexPlan& pl, cudaStream_t st, unsigned int* ready = nullptr,
                             const int32_t* page_table = nullptr, int32_t num_pages = 0,
                             const int32_t* table = nullptr, unsigned long long* picks = nullptr) {
    if (pl.stream)
        return launch_index_stream<T>(q_c, k_c, batch, S, bs, nb_max, ctx_len, q_start, topk, ids,
                                      ws, pl, st, ready, page_table, num_pages, table, picks);
    constexpr int KV = 2048 / (16 * 32);
    auto kern = pl.qreg ? lci::index_gemv_select_kernel<T, kIndexThreads, KV>
                        : lci::index_gemv_select_kernel<T, kIndexThreads, 0>;
    // Largest dynamic shared memory any plan asks for: 32 KiB of block keys
    // plus an 8192-float query row.
    static std::once_flag once;
    static cudaError_t attr_err = cudaSuccess;
    std::call_once(once, [] {
        attr_err = cudaFuncSetAttribute(lci::index_gemv_select_kernel<T, kIndexThreads, KV>,
                                        cudaFuncAttributeMaxDynamicSharedMemorySize, kIndexMaxSmem);
        if (attr_err == cudaSuccess)
            attr_err = cudaFuncSetAttribute(lci::index_gemv_select_kernel<T, kIndexThreads, 0>,
                                            cudaFuncAttributeMaxDynamicSharedMemorySize,
                                            kIndexMaxSmem);
    });
    if (attr_err != cudaSuccess)
        return fail(LCI_ERR_CUDA, "index_select: %s", cudaGetErrorString(attr_err));
    if (pl.smem > (size_t)kIndexMaxSmem)
        return fail(LCI_ERR_UNSUPPORTED, "index_select: needs %zu bytes of shared memory", pl.smem);
    char* w = static_cast<char*>(ws);
    const long long nblk = (long long)batch * S * pl.nchunks;
    if (nblk >= (1ll << 31)) return fail(LCI_ERR_UNSUPPORTED, "index_select: grid too large");
    kern<<<(unsigned)nblk, kIndexThreads, pl.smem, st>>>(
        static_cast<const T*>(q_c), static_cast<const T*>(k_c), S, K, nb_max, bs, ctx_len, q_start,
        topk, pl.chunk_blocks, pl.nchunks, reinterpret_cast<float*>(w + pl.off_scores),
        reinterpret_cast<uint32_t*>(w + pl.off_chunk_max),
        reinterpret_cast<unsigned int*>(w + pl.off_counters), ids, ready, page_table, num_pages);
    return check_launch("index_select");
}

// ------------------------------------------------------------ sparse_attn

lci_status check_attn_args(int32_t batch, int32_t S, int32_t H_q, const lci_block_table* t,
                           int32_t topk) {
    if (!t) return fail(LCI_ERR_INVALID_ARG, "sparse_attn: null block table");
    if (batch <= 0 || S <= 0 || H_q <= 0 || topk <= 0)
        return fail(LCI_ERR_INVALID_ARG, "sparse_attn: sizes must be positive (batch=%d S=%d H_q=%d "
                    "topk=%d)", batch, S, H_q, topk);
    if (batch > t->batch)
        return fail(LCI_ERR_INVALID_ARG, "sparse_attn: batch %d exceeds the table's %d", batch,
                    t->batch);
    if (H_q % t->num_kv_heads != 0)
        return fail(LCI_ERR_INVALID_ARG, "sparse_attn: H_q %d not a multiple of num_kv_heads %d",
                    H_q, t->num_kv_heads);
    if (topk > lci::kMaxTopk)
        return fail(LCI_ERR_UNSUPPORTED, "sparse_attn: topk %d above %d", topk, lci::kMaxTopk);
    if (t->head_dim % 32 != 0 || t->head_dim > 32 * lci::kSimtMaxHdPerLane)
        return fail(LCI_ERR_UNSUPPORTED, "sparse_attn: head_dim %d must be a multiple of 32 and "
                    "<= %d", t->head_dim, 32 * lci::kSimtMaxHdPerLane);
    return LCI_OK;
}

template <typename T>
lci_status launch_attn_simt(const void* q, int32_t batch, int32_t S, int32_t H_q,
                            const void* k_pool, const void* v_pool, const lci_block_table* t,
                            const int32_t* ids, int32_t topk, const int32_t* ctx_len,
                            const int32_t* q_start, float scale, void* out, cudaStream_t st) {
    const int G = H_q / t->num_kv_heads;
    const int warps = G < 16 ? G : 16;
    dim3 grid((unsigned)(batch * S), (unsigned)t->num_kv_heads);
    const float scale_log2 = scale * 1.4426950408889634f;
    lci::sparse_attn_simt_kernel<T><<<grid, warps * 32, 0, st>>>(
        static_cast<const T*>(q), static_cast<const T*>(k_pool), static_cast<const T*>(v_pool),
        t->d_table, t->max_blocks, t->num_pages, t->num_kv_heads, t->block_size, t->head_dim, S,
        H_q, ids, topk, ctx_len, q_start, scale_log2, static_cast<T*>(out));
    return check_launch("sparse_attn");
}

// ---- TMA tensor maps (driver entry point fetched through the runtime) ----

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

// A KV pool [P][H_kv][bs][128] bf16 seen as a 2D tensor of P*H_kv*bs rows of
// 128 elements, read in 64x64 boxes with the 128-byte swizzle.
lci_status encode_pool_map(CUtensorMap* map, const void* pool, long long rows) {
    auto enc = tensor_map_encoder();
    if (!enc) return fail(LCI_ERR_CUDA, "sparse_attn: cuTensorMapEncodeTiled unavailable");
    cuuint64_t dims[2] = {(cuuint64_t)lci::dec::kHD, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)lci::dec::kHD * 2};
    cuuint32_t box[2] = {64, 64};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(pool), dims,
                     strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(LCI_ERR_CUDA, "sparse_attn: tensor map encode failed (%d)", (int)r);
    return LCI_OK;
}

// The pools' tensor maps, from the table's cache when the pools are the ones
// it last saw.
lci_status pool_maps(const lci_block_table* t, const void* k_pool, const void* v_pool,
                     CUtensorMap* tm_k, CUtensorMap* tm_v) {
    lci_block_table* mt = const_cast<lci_block_table*>(t);
    std::lock_guard<std::mutex> lock(mt->map_mu);
    if (mt->map_k_pool != k_pool || mt->map_v_pool != v_pool) {
        const long long rows = (long long)t->num_pages * t->num_kv_heads * t->block_size;
        lci_status s = encode_pool_map(&mt->map_k, k_pool, rows);
        if (s != LCI_OK) return s;
        s = encode_pool_map(&mt->map_v, v_pool, rows);
        if (s != LCI_OK) {
            mt->map_k_pool = mt->map_v_pool = nullptr;
            return s;
        }
        mt->map_k_pool = k_pool;
        mt->map_v_pool = v_pool;
    }
    *tm_k = mt->map_k;
    *tm_v = mt->map_v;
    return LCI_OK;
}

// Tensor-core schedule for many queries per sequence (index_prefill.cuh).
struct PrefillPlan {
    int m_tiles, n_split, kt, ksteps;
    size_t off_counters, off_key, off_id, off_bound, bytes;
};

PrefillPlan plan_prefill(int32_t batch, int32_t S, int32_t K, int32_t nb_max, int32_t topk) {
    PrefillPlan pl{};
    pl.m_tiles = (S + lci::pre::kBM - 1) / lci::pre::kBM;
    pl.ksteps = K / lci::pre::kBK;
    pl.kt = topk <= 16 ? 16 : (topk <= 32 ? 32 : 64);
    const int n_tiles = (nb_max + lci::pre::kBN - 1) / lci::pre::kBN;
    // about one CTA per SM; the merge copies n_split * topk candidates per row
    // of a 128-row tile into the stage memory. The CTAs of an m-tile split its
    // n-tiles, or with a single n-tile its visible columns.
    long long split = 148 / ((long long)batch * pl.m_tiles);
    split = split < 1 ? 1 : split;
    split = split > 8 ? 8 : split;
    const int split_max = n_tiles == 1 ? lci::pre::kBN / 64 : n_tiles;  // windows of >= 64 columns
    split = split > split_max ? split_max : split;
    while (split > 1 &&
           (long long)lci::pre::kBM * split * topk * 8 > (long long)lci::pre::kStages * lci::pre::kStageBytes)
        --split;
    pl.n_split = (int)split;
    const long long cand = (long long)batch * pl.m_tiles * lci::pre::kBM * pl.n_split * topk;
    // counters and row bounds in the zero prefix, then the split lists
    pl.off_counters = 0;
    pl.off_bound = align_up((size_t)batch * pl.m_tiles * sizeof(unsigned int));
    pl.off_key = index_zero_prefix(batch, S);
    pl.off_id = pl.off_key + align_up((size_t)cand * sizeof(uint32_t));
    pl.bytes = pl.off_id + align_up((size_t)cand * sizeof(int32_t));
    return pl;
}

bool prefill_path(lci_dtype dtype, lci_phase phase, int32_t S, int32_t K, int32_t topk,
                  const void* q_c, const void* k_c) {
    const lci_phase ph = resolve_phase(phase, S);
    const bool wants = phase == LCI_PHASE_PREFILL || (ph == LCI_PHASE_PREFILL && S >= 32);
    return wants && dtype == LCI_BF16 && K % lci::pre::kBK == 0 && topk <= 64 && aligned16(q_c) &&
           aligned16(k_c);  // (null pointers count as aligned: size queries pass them)
}

lci_status encode_rows_map(CUtensorMap* map, const void* base, long long rows, int K, int box_rows) {
    auto enc = tensor_map_encoder();
    if (!enc) return fail(LCI_ERR_CUDA, "index_select: cuTensorMapEncodeTiled unavailable");
    cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)K * 2};
    cuuint32_t box[2] = {(cuuint32_t)lci::pre::kBK, (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims,
                     strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(LCI_ERR_CUDA, "index_select: tensor map encode failed (%d)", (int)r);
    return LCI_OK;
}

template <int KT>
lci_status launch_prefill_kt(const CUtensorMap& tq, const CUtensorMap& tk, int32_t batch, int32_t S,
                             int32_t nb_max, int32_t bs, const int32_t* ctx_len,
                             const int32_t* q_start, int32_t topk, const PrefillPlan& pl,
                             char* ws, int32_t* ids, cudaStream_t st) {
    auto kern = lci::index_prefill_tc_kernel<KT>;
    static std::once_flag once;
    static cudaError_t attr_err = cudaSuccess;
    std::call_once(once, [kern] {
        attr_err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        lci::pre::kSmemBytes);
    });
    if (attr_err != cudaSuccess)
        return fail(LCI_ERR_CUDA, "index_select: %s", cudaGetErrorString(attr_err));
    dim3 grid((unsigned)pl.n_split, (unsigned)pl.m_tiles, (unsigned)batch);
    kern<<<grid, lci::pre::Cfg<KT>::kThreads, lci::pre::kSmemBytes, st>>>(
        tq, tk, S, nb_max, bs, ctx_len, q_start, topk, pl.ksteps, pl.m_tiles, pl.n_split,
        reinterpret_cast<uint32_t*>(ws + pl.off_key), reinterpret_cast<int32_t*>(ws + pl.off_id),
        reinterpret_cast<unsigned int*>(ws + pl.off_counters),
        reinterpret_cast<unsigned int*>(ws + pl.off_bound), ids);
    return check_launch("index_select");
}

lci_status launch_index_prefill(const void* q_c, const void* k_c, int32_t batch, int32_t S,
                                int32_t K, int32_t bs, int32_t nb_max, const int32_t* ctx_len,
                                const int32_t* q_start, int32_t topk, int32_t* ids, void* ws,
                                const PrefillPlan& pl, cudaStream_t st) {
    CUtensorMap tq, tk;
    lci_status s = encode_rows_map(&tq, q_c, (long long)batch * S, K, lci::pre::kBM);
    if (s != LCI_OK) return s;
    s = encode_rows_map(&tk, k_c, (long long)batch * nb_max, K, lci::pre::kBN);
    if (s != LCI_OK) return s;
    char* w = static_cast<char*>(ws);
    if (pl.kt == 16)
        return launch_prefill_kt<16>(tq, tk, batch, S, nb_max, bs, ctx_len, q_start, topk, pl, w, ids, st);
    if (pl.kt == 32)
        return launch_prefill_kt<32>(tq, tk, batch, S, nb_max, bs, ctx_len, q_start, topk, pl, w, ids, st);
    return launch_prefill_kt<64>(tq, tk, batch, S, nb_max, bs, ctx_len, q_start, topk, pl, w, ids, st);
}

bool decode_kernel_fits(const lci_block_table* t, int32_t H_q, const void* k_pool,
                        const void* v_pool) {
    const int G = H_q / t->num_kv_heads;
    const long long rows = (long long)t->num_pages * t->num_kv_heads * t->block_size;
    return t->dtype == LCI_BF16 && t->head_dim == lci::dec::kHD && t->block_size % 64 == 0 &&
           G <= lci::dec::kRows && aligned16(k_pool) && aligned16(v_pool) && rows < (1ll << 31);
}

struct DecodeShape {
    int nsplit;  // CTAs (one cluster) per (row, KV head) pair
    bool deep;   // one CTA per SM with the deep ring
};

DecodeShape decode_shape(long long pairs, int units) {
    // When the pairs fill the SMs with clusters of 2-4 CTAs, give each SM one
    // CTA with the deep ring (and two consumer groups); otherwise two shallow
    // CTAs per SM and up to 8 splits.
    const long long per_sm = 148 / pairs;
    if (per_sm >= 2 && per_sm <= 4 && units >= 2 * per_sm) return {(int)per_sm, true};
    long long want = (2 * 148 + pairs - 1) / pairs;
    if (want > lci::dec::kMaxSplit) want = lci::dec::kMaxSplit;
    if (want > units) want = units;
    return {want < 1 ? 1 : (int)want, false};
}

template <int ST, int GR>
cudaError_t decode_kernel_attr() {
    static std::once_flag once;
    static cudaError_t err = cudaSuccess;
    std::call_once(once, [] {
        err = cudaFuncSetAttribute(lci::sparse_attn_decode_kernel<ST, GR>,
                                   cudaFuncAttributeMaxDynamicSharedMemorySize,
                                   lci::dec::smem_bytes(ST));
    });
    return err;
}

// The deep ring runs one CTA per SM with two consumer groups, the shallow one
// two CTAs per SM with one group each.
constexpr int kDeepGroups = 2, kShallowGroups = 1;

lci_status launch_attn_decode(const void* q, int32_t batch, int32_t S, int32_t H_q,
                              const void* k_pool, const void* v_pool, const lci_block_table* t,
                              const int32_t* ids, int32_t topk, const int32_t* ctx_len,
                              const int32_t* q_start, float scale, void* out, cudaStream_t st,
                              const unsigned int* ready = nullptr, bool early_start = true,
                              float* lse = nullptr, const unsigned long long* picks = nullptr) {
    CUtensorMap tm_k, tm_v;
    lci_status s = pool_maps(t, k_pool, v_pool, &tm_k, &tm_v);
    if (s != LCI_OK) return s;
    const long long pairs = (long long)batch * S * t->num_kv_heads;
    const int units = topk * (t->block_size / 64);
    const DecodeShape shape = decode_shape(pairs, units);
    const int nsplit = shape.nsplit;
    const int stages = shape.deep ? lci::dec::kStagesDeep : lci::dec::kStagesShallow;
    const cudaError_t attr_err =
        shape.deep ? decode_kernel_attr<lci::dec::kStagesDeep, kDeepGroups>()
                   : decode_kernel_attr<lci::dec::kStagesShallow, kShallowGroups>();
    if (attr_err != cudaSuccess)
        return fail(LCI_ERR_CUDA, "sparse_attn: %s", cudaGetErrorString(attr_err));
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)pairs, (unsigned)nsplit, 1);
    cfg.blockDim = dim3(lci::dec::threads(shape.deep ? kDeepGroups : kShallowGroups), 1, 1);
    cfg.dynamicSmemBytes = lci::dec::smem_bytes(stages);
    cfg.stream = st;
    cudaLaunchAttribute attrs[2];
    int na = 0;
    if (nsplit > 1) {
        attrs[na].id = cudaLaunchAttributeClusterDimension;
        attrs[na].val.clusterDim.x = 1;
        attrs[na].val.clusterDim.y = (unsigned)nsplit;
        attrs[na].val.clusterDim.z = 1;
        ++na;
    }
    if (early_start) {  // may start under the previous kernel on the stream
        attrs[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attrs[na].val.programmaticStreamSerializationAllowed = 1;
        ++na;
    }
    cfg.attrs = attrs;
    cfg.numAttrs = na;
    const float scale_log2 = scale * 1.4426950408889634f;
    auto kern = shape.deep ? lci::sparse_attn_decode_kernel<lci::dec::kStagesDeep, kDeepGroups>
                           : lci::sparse_attn_decode_kernel<lci::dec::kStagesShallow, kShallowGroups>;
    cudaError_t e = cudaLaunchKernelEx(
        &cfg, kern, tm_k, tm_v, static_cast<const __nv_bfloat16*>(q),
        t->d_table, t->max_blocks, t->num_pages, t->num_kv_heads, t->block_size, S, H_q, ids, topk,
        ctx_len, q_start, scale_log2, static_cast<__nv_bfloat16*>(out), nsplit, ready, lse, picks);
    if (e != cudaSuccess) return fail(LCI_ERR_CUDA, "sparse_attn: %s", cudaGetErrorString(e));
    return check_launch("sparse_attn");
}

// The tensor-core prefill schedule (attn_prefill.cuh): the decode kernel's
// shape limits, 4, 8 or 16 query heads per KV head (32, 16 or 8 queries per
// 128-row tile), at most 16384 blocks per sequence and 1024 selected blocks per
// tile, token positions below 2^31.
bool prefill_attn_fits(const lci_block_table* t, int32_t H_q, int32_t topk, const void* k_pool,
                       const void* v_pool) {
    if (!decode_kernel_fits(t, H_q, k_pool, v_pool)) return false;
    const int G = H_q / t->num_kv_heads;
    return (G == 4 || G == 8 || G == 16) && t->max_blocks <= 32 * lci::pfa::kMaxWords &&
           (long long)t->max_blocks * t->block_size < (1LL << 31) &&
           (long long)(lci::pfa::kRows / G) * topk <= lci::pfa::kMaxUnion;
}

// Which attention kernel a call runs: the tensor-core tile schedule when asked
// for (LCI_PHASE_PREFILL) and it fits, or, under LCI_PHASE_AUTO, for many
// queries per sequence whose selections are likely to share blocks (at most
// four times as many blocks as a tile's queries select in all); otherwise the
// one-row-at-a-time kernel, which gathers each query's blocks on its own.
bool use_prefill_attn(const lci_block_table* t, int32_t S, int32_t H_q, int32_t topk,
                      lci_phase phase, const void* k_pool, const void* v_pool) {
    if (phase == LCI_PHASE_DECODE || !prefill_attn_fits(t, H_q, topk, k_pool, v_pool)) return false;
    if (phase == LCI_PHASE_PREFILL) return true;
    const int QT = lci::pfa::kRows / (H_q / t->num_kv_heads);
    return S >= 16 && (long long)t->max_blocks <= 4ll * QT * topk;
}

lci_status launch_attn_prefill(const void* q, int32_t batch, int32_t S, int32_t H_q,
                               const void* k_pool, const void* v_pool, const lci_block_table* t,
                               const int32_t* ids, int32_t topk, const int32_t* ctx_len,
                               const int32_t* q_start, float scale, void* out, cudaStream_t st,
                               float* lse = nullptr) {
    CUtensorMap tm_k, tm_v;
    lci_status s = pool_maps(t, k_pool, v_pool, &tm_k, &tm_v);
    if (s != LCI_OK) return s;
    static std::once_flag once;
    static cudaError_t attr_err = cudaSuccess;
    std::call_once(once, [] {
        attr_err = cudaFuncSetAttribute(lci::sparse_attn_prefill_kernel,
                                        cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        lci::pfa::kSmemBytes);
    });
    if (attr_err != cudaSuccess)
        return fail(LCI_ERR_CUDA, "sparse_attn: %s", cudaGetErrorString(attr_err));
    const int G = H_q / t->num_kv_heads;
    const int QT = lci::pfa::kRows / G;
    const int q_tiles = (S + QT - 1) / QT;
    const long long tiles = (long long)batch * q_tiles * t->num_kv_heads;
    if (tiles >= (1ll << 31)) return fail(LCI_ERR_UNSUPPORTED, "sparse_attn: grid too large");
    const float scale_log2 = scale * 1.4426950408889634f;
    lci::sparse_attn_prefill_kernel<<<(unsigned)tiles, lci::pfa::kThreads, lci::pfa::kSmemBytes, st>>>(
        tm_k, tm_v, static_cast<const __nv_bfloat16*>(q), t->d_table, t->max_blocks, t->num_pages,
        t->num_kv_heads, t->block_size, S, H_q, ids, topk, ctx_len, q_start, scale_log2,
        static_cast<__nv_bfloat16*>(out), q_tiles, lse);
    return check_launch("sparse_attn");
}

__global__ void validate_table_kernel(const int32_t* __restrict__ table, long long n,
                                      int num_pages) {
    for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n;
         i += (long long)gridDim.x * blockDim.x) {
        const int v = table[i];
        if (v < 0 || v >= num_pages) lci::raise_status(lci::kStatusBadPage);
    }
}

}  // namespace

extern "C" {

const char* lci_version(void) { return "0.1.0"; }

const char* lci_status_string(lci_status s) {
    switch (s) {
        case LCI_OK: return "ok";
        case LCI_ERR_INVALID_ARG: return "invalid argument";
        case LCI_ERR_UNSUPPORTED: return "unsupported configuration";
        case LCI_ERR_WORKSPACE: return "workspace missing or too small";
        case LCI_ERR_CUDA: return "CUDA error";
        case LCI_ERR_DEVICE_BOUNDS: return "device bounds check fired";
        case LCI_ERR_TIMEOUT: return "device wait timed out";
    }
    return "unknown status";
}

const char* lci_last_error(void) { return t_last_error.c_str(); }

lci_status lci_create_block_table(const int32_t* d_table, int32_t batch, int32_t max_blocks,
                                  int32_t num_pages, int32_t block_size, int32_t num_kv_heads,
                                  int32_t head_dim, lci_dtype kv_dtype, lci_block_table** out) {
    if (!out) return fail(LCI_ERR_INVALID_ARG, "create_block_table: null output pointer");
    *out = nullptr;
    if (!d_table) return fail(LCI_ERR_INVALID_ARG, "create_block_table: null table pointer");
    if (batch <= 0 || max_blocks <= 0 || num_pages <= 0 || block_size <= 0 || num_kv_heads <= 0 ||
        head_dim <= 0)
        return fail(LCI_ERR_INVALID_ARG, "create_block_table: sizes must be positive");
    if (!dtype_ok(kv_dtype)) return fail(LCI_ERR_INVALID_ARG, "create_block_table: unknown dtype");
    lci_block_table* t = new (std::nothrow) lci_block_table;
    if (!t) return fail(LCI_ERR_INVALID_ARG, "create_block_table: host allocation failed");
    t->d_table = d_table;
    t->batch = batch;
    t->max_blocks = max_blocks;
    t->num_pages = num_pages;
    t->block_size = block_size;
    t->num_kv_heads = num_kv_heads;
    t->head_dim = head_dim;
    t->dtype = kv_dtype;
    *out = t;
    return ok();
}

lci_status lci_destroy_block_table(lci_block_table* table) {
    delete table;
    return ok();
}

lci_status lci_validate_block_table(const lci_block_table* t, void* stream) {
    if (!t) return fail(LCI_ERR_INVALID_ARG, "validate_block_table: null table");
    const long long n = (long long)t->batch * t->max_blocks;
    const int blocks = (int)((n + 255) / 256 < 1184 ? (n + 255) / 256 : 1184);
    validate_table_kernel<<<blocks, 256, 0, static_cast<cudaStream_t>(stream)>>>(t->d_table, n,
                                                                                  t->num_pages);
    return check_launch("validate_block_table");
}

lci_status lci_block_compress(const void* k_idx, lci_dtype dtype, int32_t batch, int32_t tokens,
                              int32_t heads, int32_t dim, int32_t block_size, void* k_c,
                              void* stream) {
    if (!k_idx || !k_c) return fail(LCI_ERR_INVALID_ARG, "block_compress: null pointer");
    if (batch <= 0 || tokens <= 0 || heads <= 0 || dim <= 0 || block_size <= 0)
        return fail(LCI_ERR_INVALID_ARG, "block_compress: sizes must be positive");
    if (!dtype_ok(dtype)) return fail(LCI_ERR_INVALID_ARG, "block_compress: unknown dtype");
    const int NB = (tokens + block_size - 1) / block_size;
    const int HD = heads * dim;
    const long long total = (long long)batch * NB * HD;
    const int threads = 256;
    const long long want = (total + threads - 1) / threads;
    const int blocks = (int)(want < 148 * 16 ? want : 148 * 16);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (dtype == LCI_F32)
        lci::block_compress_kernel<float><<<blocks, threads, 0, st>>>(
            static_cast<const float*>(k_idx), batch, tokens, HD, block_size, NB,
            static_cast<float*>(k_c));
    else
        lci::block_compress_kernel<__nv_bfloat16><<<blocks, threads, 0, st>>>(
            static_cast<const __nv_bfloat16*>(k_idx), batch, tokens, HD, block_size, NB,
            static_cast<__nv_bfloat16*>(k_c));
    return check_launch("block_compress");
}

lci_status lci_index_select_workspace_size(int32_t batch, int32_t S, int32_t H_i, int32_t d_c,
                                           int32_t nb_max, int32_t topk, lci_phase phase,
                                           size_t* bytes) {
    if (!bytes) return fail(LCI_ERR_INVALID_ARG, "index_select_workspace_size: null output");
    lci_status st = check_index_args(batch, S, H_i, d_c, nb_max, topk, LCI_BF16);
    if (st != LCI_OK && st != LCI_ERR_UNSUPPORTED) return st;
    (void)phase;
    // the schedule a bf16 call with these sizes takes (fp32 always runs row-wise)
    const int K = H_i * d_c;
    const bool tc = prefill_path(LCI_BF16, phase, S, K, topk, nullptr, nullptr);
    const size_t g = plan_index(batch, S, K, nb_max, 2).bytes;  // same for both types
    *bytes = tc ? std::max(g, plan_prefill(batch, S, K, nb_max, topk).bytes) : g;
    return ok();
}

lci_status lci_index_select(const void* q_c, const void* k_c, lci_dtype dtype, int32_t batch,
                            int32_t S, int32_t H_i, int32_t d_c, int32_t block_size,
                            int32_t nb_max, const int32_t* d_ctx_len, const int32_t* d_q_start,
                            int32_t topk, lci_phase phase, int32_t* d_ids, void* workspace,
                            size_t workspace_bytes, void* stream) {
    if (!q_c || !k_c || !d_ctx_len || !d_q_start || !d_ids)
        return fail(LCI_ERR_INVALID_ARG, "index_select: null pointer argument");
    if (block_size <= 0) return fail(LCI_ERR_INVALID_ARG, "index_select: block_size must be positive");
    lci_status st = check_index_args(batch, S, H_i, d_c, nb_max, topk, dtype);
    if (st != LCI_OK) return st;
    if (phase != LCI_PHASE_AUTO && phase != LCI_PHASE_PREFILL && phase != LCI_PHASE_DECODE)
        return fail(LCI_ERR_INVALID_ARG, "index_select: unknown phase %d", (int)phase);
    if (!aligned16(q_c) || !aligned16(k_c))
        return fail(LCI_ERR_INVALID_ARG, "index_select: q_c and k_c must be 16-byte aligned");
    const int K = H_i * d_c;
    const IndexPlan pl = plan_index(batch, S, K, nb_max, dtype_size(dtype));
    if (!workspace || workspace_bytes < pl.bytes ||
        (reinterpret_cast<uintptr_t>(workspace) & (kAlign - 1)) != 0)
        return fail(LCI_ERR_WORKSPACE, "index_select: workspace needs %zu bytes, 256-byte aligned "
                    "(got %zu at %p)", pl.bytes, workspace_bytes, workspace);
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    if (prefill_path(dtype, phase, S, K, topk, q_c, k_c)) {
        const PrefillPlan pp = plan_prefill(batch, S, K, nb_max, topk);
        if (workspace_bytes < pp.bytes)
            return fail(LCI_ERR_WORKSPACE, "index_select: workspace needs %zu bytes", pp.bytes);
        return launch_index_prefill(q_c, k_c, batch, S, K, block_size, nb_max, d_ctx_len, d_q_start,
                                    topk, d_ids, workspace, pp, cs);
    }
    if (dtype == LCI_F32)
        return launch_index_gemv<float>(q_c, k_c, batch, S, K, block_size, nb_max, d_ctx_len,
                                        d_q_start, topk, d_ids, workspace, pl, cs);
    return launch_index_gemv<__nv_bfloat16>(q_c, k_c, batch, S, K, block_size, nb_max, d_ctx_len,
                                            d_q_start, topk, d_ids, workspace, pl, cs);
}

// ---- paged block keys (online producer, paged index selection) ----

lci_status lci_kc_update(const void* k_idx, lci_dtype dtype, int32_t batch, int32_t T, int32_t H_i,
                         int32_t d_c, const int32_t* d_start, const lci_block_table* table,
                         float* kc_sum, void* kc, void* stream) {
    if (!k_idx || !d_start || !table || !kc_sum || !kc)
        return fail(LCI_ERR_INVALID_ARG, "kc_update: null pointer argument");
    if (batch <= 0 || T <= 0 || H_i <= 0 || d_c <= 0)
        return fail(LCI_ERR_INVALID_ARG, "kc_update: sizes must be positive");
    if (!dtype_ok(dtype)) return fail(LCI_ERR_INVALID_ARG, "kc_update: unknown dtype");
    if (batch > table->batch)
        return fail(LCI_ERR_INVALID_ARG, "kc_update: batch %d exceeds the table's %d", batch,
                    table->batch);
    const long long HD = (long long)H_i * d_c;
    const long long slots = ((long long)T + table->block_size - 1) / table->block_size + 1;
    const long long total = (long long)batch * slots * HD;
    const int threads = 256;
    const long long want = (total + threads - 1) / threads;
    const int blocks = (int)(want < 148 * 16 ? want : 148 * 16);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (dtype == LCI_F32)
        lci::kc_update_kernel<float><<<blocks, threads, 0, st>>>(
            static_cast<const float*>(k_idx), batch, T, (int)HD, table->block_size, d_start,
            table->d_table, table->max_blocks, table->num_pages, (int)slots, kc_sum,
            static_cast<float*>(kc));
    else
        lci::kc_update_kernel<__nv_bfloat16><<<blocks, threads, 0, st>>>(
            static_cast<const __nv_bfloat16*>(k_idx), batch, T, (int)HD, table->block_size, d_start,
            table->d_table, table->max_blocks, table->num_pages, (int)slots, kc_sum,
            static_cast<__nv_bfloat16*>(kc));
    return check_launch("kc_update");
}

namespace {
struct PagedPlan {
    bool tc;             // tensor-core schedule over a dense gather of the keys
    size_t off_dense;    // [batch][nb_max][K] gathered keys (tc only)
    size_t off_rest;     // the schedule's own workspace
    size_t bytes;
    PrefillPlan pp;
    IndexPlan ip;
};

PagedPlan plan_paged(lci_dtype dtype, int32_t batch, int32_t S, int32_t K, int32_t nb_max,
                     int32_t topk, lci_phase phase, const void* q_c, const void* kc) {
    PagedPlan pl{};
    pl.tc = prefill_path(dtype, phase, S, K, topk, q_c, kc);
    pl.ip = plan_index(batch, S, K, nb_max, dtype_size(dtype));
    if (pl.tc) {
        pl.pp = plan_prefill(batch, S, K, nb_max, topk);
        pl.off_dense = 0;
        pl.off_rest = align_up((size_t)batch * nb_max * K * dtype_size(dtype));
        pl.bytes = pl.off_rest + pl.pp.bytes;
    } else {
        pl.off_rest = 0;
        pl.bytes = pl.ip.bytes;
    }
    return pl;
}
}  // namespace

lci_status lci_index_select_paged_workspace_size(int32_t batch, int32_t S, int32_t H_i,
                                                 int32_t d_c, int32_t topk,
                                                 const lci_block_table* table, lci_dtype dtype,
                                                 lci_phase phase, size_t* bytes) {
    if (!bytes || !table)
        return fail(LCI_ERR_INVALID_ARG, "index_select_paged_workspace_size: null argument");
    lci_status st = check_index_args(batch, S, H_i, d_c, table->max_blocks, topk, dtype);
    if (st != LCI_OK) return st;
    *bytes = plan_paged(dtype, batch, S, H_i * d_c, table->max_blocks, topk, phase, nullptr,
                        nullptr).bytes;
    return ok();
}

lci_status lci_index_select_paged(const void* q_c, const void* kc, lci_dtype dtype, int32_t batch,
                                  int32_t S, int32_t H_i, int32_t d_c,
                                  const lci_block_table* table, const int32_t* d_ctx_len,
                                  const int32_t* d_q_start, int32_t topk, lci_phase phase,
                                  int32_t* d_ids, void* workspace, size_t workspace_bytes,
                                  void* stream) {
    if (!q_c || !kc || !table || !d_ctx_len || !d_q_start || !d_ids)
        return fail(LCI_ERR_INVALID_ARG, "index_select_paged: null pointer argument");
    const int32_t nb_max = table->max_blocks;
    lci_status st = check_index_args(batch, S, H_i, d_c, nb_max, topk, dtype);
    if (st != LCI_OK) return st;
    if (batch > table->batch)
        return fail(LCI_ERR_INVALID_ARG, "index_select_paged: batch %d exceeds the table's %d",
                    batch, table->batch);
    if (phase != LCI_PHASE_AUTO && phase != LCI_PHASE_PREFILL && phase != LCI_PHASE_DECODE)
        return fail(LCI_ERR_INVALID_ARG, "index_select_paged: unknown phase %d", (int)phase);
    if (!aligned16(q_c) || !aligned16(kc))
        return fail(LCI_ERR_INVALID_ARG, "index_select_paged: q_c and kc must be 16-byte aligned");
    const int K = H_i * d_c;
    const PagedPlan pl = plan_paged(dtype, batch, S, K, nb_max, topk, phase, q_c, kc);
    if (!workspace || workspace_bytes < pl.bytes ||
        (reinterpret_cast<uintptr_t>(workspace) & (kAlign - 1)) != 0)
        return fail(LCI_ERR_WORKSPACE, "index_select_paged: workspace needs %zu bytes, 256-byte "
                    "aligned (got %zu at %p)", pl.bytes, workspace_bytes, workspace);
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    char* w = static_cast<char*>(workspace);
    if (pl.tc) {
        // gather the visible blocks' keys through the table, then the dense
        // tensor-core schedule
        const int vec = (int)(K * dtype_size(dtype) / 16);
        const long long total = (long long)batch * nb_max * vec;
        const long long want = (total + 255) / 256;
        const int blocks = (int)(want < 148 * 16 ? want : 148 * 16);
        lci::kc_gather_kernel<<<blocks, 256, 0, cs>>>(
            static_cast<const uint4*>(kc), table->d_table, d_ctx_len, batch, nb_max,
            table->block_size, table->num_pages, vec, reinterpret_cast<uint4*>(w + pl.off_dense));
        st = check_launch("index_select_paged");
        if (st != LCI_OK) return st;
        return launch_index_prefill(q_c, w + pl.off_dense, batch, S, K, table->block_size, nb_max,
                                    d_ctx_len, d_q_start, topk, d_ids, w + pl.off_rest, pl.pp, cs);
    }
    if (dtype == LCI_F32)
        return launch_index_gemv<float>(q_c, kc, batch, S, K, table->block_size, nb_max, d_ctx_len,
                                        d_q_start, topk, d_ids, w + pl.off_rest, pl.ip, cs, nullptr,
                                        table->d_table, table->num_pages);
    return launch_index_gemv<__nv_bfloat16>(q_c, kc, batch, S, K, table->block_size, nb_max,
                                            d_ctx_len, d_q_start, topk, d_ids, w + pl.off_rest,
                                            pl.ip, cs, nullptr, table->d_table, table->num_pages);
}

lci_status lci_sparse_attn_workspace_size(int32_t batch, int32_t S, int32_t H_q, int32_t topk,
                                          const lci_block_table* table, lci_phase phase,
                                          size_t* bytes) {
    if (!bytes) return fail(LCI_ERR_INVALID_ARG, "sparse_attn_workspace_size: null output");
    lci_status st = check_attn_args(batch, S, H_q, table, topk);
    if (st != LCI_OK) return st;
    (void)phase;
    *bytes = 0;
    return ok();
}

lci_status lci_sparse_attn(const void* q, int32_t batch, int32_t S, int32_t H_q,
                           const void* k_pool, const void* v_pool, const lci_block_table* table,
                           const int32_t* d_ids, int32_t topk, const int32_t* d_ctx_len,
                           const int32_t* d_q_start, float scale, lci_phase phase, void* out,
                           void* workspace, size_t workspace_bytes, void* stream) {
    if (!q || !k_pool || !v_pool || !d_ids || !d_ctx_len || !d_q_start || !out)
        return fail(LCI_ERR_INVALID_ARG, "sparse_attn: null pointer argument");
    lci_status st = check_attn_args(batch, S, H_q, table, topk);
    if (st != LCI_OK) return st;
    if (phase != LCI_PHASE_AUTO && phase != LCI_PHASE_PREFILL && phase != LCI_PHASE_DECODE)
        return fail(LCI_ERR_INVALID_ARG, "sparse_attn: unknown phase %d", (int)phase);
    if (!(scale > 0.f)) scale = 1.0f / std::sqrt((float)table->head_dim);
    if (!std::isfinite(scale)) return fail(LCI_ERR_INVALID_ARG, "sparse_attn: non-finite scale");
    (void)workspace;
    (void)workspace_bytes;
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    if (use_prefill_attn(table, S, H_q, topk, phase, k_pool, v_pool))
        return launch_attn_prefill(q, batch, S, H_q, k_pool, v_pool, table, d_ids, topk, d_ctx_len,
                                   d_q_start, scale, out, cs);
    if (decode_kernel_fits(table, H_q, k_pool, v_pool))
        return launch_attn_decode(q, batch, S, H_q, k_pool, v_pool, table, d_ids, topk, d_ctx_len,
                                  d_q_start, scale, out, cs);
    if (table->dtype == LCI_F32)
        return launch_attn_simt<float>(q, batch, S, H_q, k_pool, v_pool, table, d_ids, topk,
                                       d_ctx_len, d_q_start, scale, out, cs);
    return launch_attn_simt<__nv_bfloat16>(q, batch, S, H_q, k_pool, v_pool, table, d_ids, topk,
                                           d_ctx_len, d_q_start, scale, out, cs);
}

// ---- context parallelism: partial results and their exact combination ----

lci_status lci_sparse_attn_partial(const void* q, int32_t batch, int32_t S, int32_t H_q,
                                   const void* k_pool, const void* v_pool,
                                   const lci_block_table* table, const int32_t* d_ids,
                                   int32_t topk, const int32_t* d_ctx_len,
                                   const int32_t* d_q_start, float scale, lci_phase phase,
                                   void* out, float* lse, void* stream) {
    if (!q || !k_pool || !v_pool || !d_ids || !d_ctx_len || !d_q_start || !out || !lse)
        return fail(LCI_ERR_INVALID_ARG, "sparse_attn_partial: null pointer argument");
    lci_status st = check_attn_args(batch, S, H_q, table, topk);
    if (st != LCI_OK) return st;
    if (phase != LCI_PHASE_AUTO && phase != LCI_PHASE_PREFILL && phase != LCI_PHASE_DECODE)
        return fail(LCI_ERR_INVALID_ARG, "sparse_attn_partial: unknown phase %d", (int)phase);
    if (!decode_kernel_fits(table, H_q, k_pool, v_pool))
        return fail(LCI_ERR_UNSUPPORTED, "sparse_attn_partial: needs bf16 pools, head_dim 128, "
                    "block_size a multiple of 64, at most 16 query heads per KV head and "
                    "16-byte aligned pools");
    if (!(scale > 0.f)) scale = 1.0f / std::sqrt((float)table->head_dim);
    if (!std::isfinite(scale)) return fail(LCI_ERR_INVALID_ARG, "sparse_attn_partial: non-finite scale");
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    if (use_prefill_attn(table, S, H_q, topk, phase, k_pool, v_pool))
        return launch_attn_prefill(q, batch, S, H_q, k_pool, v_pool, table, d_ids, topk, d_ctx_len,
                                   d_q_start, scale, out, cs, lse);
    return launch_attn_decode(q, batch, S, H_q, k_pool, v_pool, table, d_ids, topk, d_ctx_len,
                              d_q_start, scale, out, cs, nullptr, true, lse);
}

lci_status lci_block_scores_at(const void* q_c, const void* k_c, lci_dtype dtype, int32_t batch,
                               int32_t S, int32_t H_i, int32_t d_c, int32_t nb_max,
                               const int32_t* d_ids, int32_t topk, float* d_scores, void* stream) {
    if (!q_c || !k_c || !d_ids || !d_scores)
        return fail(LCI_ERR_INVALID_ARG, "block_scores_at: null pointer argument");
    lci_status st = check_index_args(batch, S, H_i, d_c, nb_max, topk, dtype);
    if (st != LCI_OK) return st;
    if (!aligned16(q_c) || !aligned16(k_c))
        return fail(LCI_ERR_INVALID_ARG, "block_scores_at: q_c and k_c must be 16-byte aligned");
    const long long pairs = (long long)batch * S * topk;
    const long long want = (pairs + 7) / 8;  // 8 warps per CTA
    const int blocks = (int)(want < 148 * 32 ? want : 148 * 32);
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    const int K = H_i * d_c;
    if (dtype == LCI_F32)
        lci::block_scores_at_kernel<float><<<blocks, 256, 0, cs>>>(
            static_cast<const float*>(q_c), static_cast<const float*>(k_c), S, K, nb_max, d_ids,
            topk, pairs, d_scores);
    else
        lci::block_scores_at_kernel<__nv_bfloat16><<<blocks, 256, 0, cs>>>(
            static_cast<const __nv_bfloat16*>(q_c), static_cast<const __nv_bfloat16*>(k_c), S, K,
            nb_max, d_ids, topk, pairs, d_scores);
    return check_launch("block_scores_at");
}

lci_status lci_ids_shift(const int32_t* d_ids, int64_t n, int32_t lo, int32_t hi, int32_t offset,
                         int32_t* d_out, void* stream) {
    if (!d_ids || !d_out) return fail(LCI_ERR_INVALID_ARG, "ids_shift: null pointer argument");
    if (n < 0) return fail(LCI_ERR_INVALID_ARG, "ids_shift: negative count");
    if (n == 0) return ok();
    const long long want = (n + 255) / 256;
    const int blocks = (int)(want < 148 * 16 ? want : 148 * 16);
    lci::ids_shift_kernel<<<blocks, 256, 0, static_cast<cudaStream_t>(stream)>>>(d_ids, n, lo, hi,
                                                                                 offset, d_out);
    return check_launch("ids_shift");
}

lci_status lci_topk_merge(const float* d_scores, const int32_t* d_ids, int32_t nlists, int64_t rows,
                          int32_t topk, int32_t* d_out, void* stream) {
    if (!d_scores || !d_ids || !d_out)
        return fail(LCI_ERR_INVALID_ARG, "topk_merge: null pointer argument");
    if (nlists <= 0 || rows <= 0 || topk <= 0)
        return fail(LCI_ERR_INVALID_ARG, "topk_merge: sizes must be positive");
    if (nlists > lci::kMaxLists)
        return fail(LCI_ERR_UNSUPPORTED, "topk_merge: %d lists above %d", nlists, lci::kMaxLists);
    const long long blocks = (rows + 127) / 128;
    if (blocks >= (1ll << 31)) return fail(LCI_ERR_UNSUPPORTED, "topk_merge: too many rows");
    lci::topk_merge_kernel<<<(unsigned)blocks, 128, 0, static_cast<cudaStream_t>(stream)>>>(
        d_scores, d_ids, nlists, rows, topk, d_out);
    return check_launch("topk_merge");
}

lci_status lci_attn_merge(const void* d_o, const float* d_lse, lci_dtype dtype, int32_t nlists,
                          int64_t rows_heads, int32_t head_dim, void* d_out, void* stream) {
    if (!d_o || !d_lse || !d_out) return fail(LCI_ERR_INVALID_ARG, "attn_merge: null pointer argument");
    if (nlists <= 0 || rows_heads <= 0 || head_dim <= 0)
        return fail(LCI_ERR_INVALID_ARG, "attn_merge: sizes must be positive");
    if (!dtype_ok(dtype)) return fail(LCI_ERR_INVALID_ARG, "attn_merge: unknown dtype");
    const long long total = rows_heads * head_dim;
    const long long want = (total + 255) / 256;
    const int blocks = (int)(want < 148 * 16 ? want : 148 * 16);
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    if (dtype == LCI_F32)
        lci::attn_merge_kernel<float><<<blocks, 256, 0, cs>>>(
            static_cast<const float*>(d_o), d_lse, nlists, rows_heads, head_dim,
            static_cast<float*>(d_out));
    else
        lci::attn_merge_kernel<__nv_bfloat16><<<blocks, 256, 0, cs>>>(
            static_cast<const __nv_bfloat16*>(d_o), d_lse, nlists, rows_heads, head_dim,
            static_cast<__nv_bfloat16*>(d_out));
    return check_launch("attn_merge");
}

}  // extern "C"

// ---- chunked gated state scan ----

namespace {
// [B][T][H][128] bf16 as a 4-D tensor (d, h, t, b), read in 64 x 1 x 128 x 1
// boxes with the 128-byte swizzle; tokens past T read as zero.
lci_status encode_bthd_map(CUtensorMap* map, const void* base, int32_t B, int32_t T, int32_t H) {
    auto enc = tensor_map_encoder();
    if (!enc) return fail(LCI_ERR_CUDA, "gated_state_scan: cuTensorMapEncodeTiled unavailable");
    cuuint64_t dims[4] = {128, (cuuint64_t)H, (cuuint64_t)T, (cuuint64_t)B};
    cuuint64_t strides[3] = {256, (cuuint64_t)H * 256, (cuuint64_t)T * H * 256};
    cuuint32_t box[4] = {64, 1, 128, 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims,
                     strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS)
        return fail(LCI_ERR_CUDA, "gated_state_scan: tensor map encode failed (%d)", (int)r);
    return LCI_OK;
}
}  // namespace

extern "C" lci_status lci_gated_state_scan(const void* q, const void* k, const void* v,
                                           lci_dtype dtype, const float* d_gate,
                                           const float* d_state_in, float* d_state_out,
                                           int32_t batch, int32_t T, int32_t H, int32_t dk,
                                           int32_t dv, int32_t chunk, float* d_out, void* stream) {
    if (!q || !k || !v || !d_gate || !d_state_in || !d_state_out || !d_out)
        return fail(LCI_ERR_INVALID_ARG, "gated_state_scan: null pointer argument");
    if (batch <= 0 || T <= 0 || H <= 0 || dk <= 0 || dv <= 0 || chunk <= 0)
        return fail(LCI_ERR_INVALID_ARG, "gated_state_scan: sizes must be positive");
    if (!dtype_ok(dtype)) return fail(LCI_ERR_INVALID_ARG, "gated_state_scan: unknown dtype");
    if (dtype != LCI_BF16 || dk != lci::gss::kD || dv != lci::gss::kD || chunk != lci::gss::kC)
        return fail(LCI_ERR_UNSUPPORTED, "gated_state_scan: supports bf16 q/k/v with dk = dv = %d "
                    "and chunks of %d tokens", lci::gss::kD, lci::gss::kC);
    if (!aligned16(q) || !aligned16(k) || !aligned16(v))
        return fail(LCI_ERR_INVALID_ARG, "gated_state_scan: q, k and v must be 16-byte aligned");
    if ((long long)batch * H >= (1ll << 31))
        return fail(LCI_ERR_UNSUPPORTED, "gated_state_scan: grid too large");
    CUtensorMap tq, tk, tv;
    lci_status s = encode_bthd_map(&tq, q, batch, T, H);
    if (s == LCI_OK) s = encode_bthd_map(&tk, k, batch, T, H);
    if (s == LCI_OK) s = encode_bthd_map(&tv, v, batch, T, H);
    if (s != LCI_OK) return s;
    static std::once_flag once;
    static cudaError_t attr_err = cudaSuccess;
    std::call_once(once, [] {
        attr_err = cudaFuncSetAttribute(lci::gated_state_scan_kernel,
                                        cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        lci::gss::kSmemBytes);
    });
    if (attr_err != cudaSuccess)
        return fail(LCI_ERR_CUDA, "gated_state_scan: %s", cudaGetErrorString(attr_err));
    const int nchunks = (T + chunk - 1) / chunk;
    lci::gated_state_scan_kernel<<<(unsigned)(batch * H), lci::gss::kThreads, lci::gss::kSmemBytes,
                                   static_cast<cudaStream_t>(stream)>>>(
        tq, tk, tv, d_gate, d_state_in, d_state_out, T, H, nchunks, d_out);
    return check_launch("gated_state_scan");
}

// ---- index selection without device allocation ----
//
// The scratch of lci_index_select_noalloc: one file-scope device array per GPU
// that loads the library. Host code never passes its name to a kernel (on the
// host it is only a stand-in symbol); the device address comes from
// cudaGetSymbolAddress, looked up on every call with the caller's device
// current (a host-side lookup once the module is loaded).
static __device__ __align__(256) unsigned char g_noalloc_scratch[LCI_NOALLOC_SCRATCH_BYTES];

namespace {
lci_status noalloc_scratch(void** out) {
    cudaError_t e = cudaGetSymbolAddress(out, g_noalloc_scratch);
    if (e != cudaSuccess)
        return fail(LCI_ERR_CUDA, "index_select_noalloc: scratch address lookup failed: %s",
                    cudaGetErrorString(e));
    return LCI_OK;
}
}  // namespace

extern "C" lci_status lci_index_select_noalloc(const void* q_c, const void* k_c, lci_dtype dtype,
                                               int32_t batch, int32_t S, int32_t H_i, int32_t d_c,
                                               int32_t block_size, int32_t nb_max,
                                               const int32_t* d_ctx_len, const int32_t* d_q_start,
                                               int32_t topk, lci_phase phase, int32_t* d_ids,
                                               void* stream) {
    if (!q_c || !k_c || !d_ctx_len || !d_q_start || !d_ids)
        return fail(LCI_ERR_INVALID_ARG, "index_select_noalloc: null pointer argument");
    if (block_size <= 0)
        return fail(LCI_ERR_INVALID_ARG, "index_select_noalloc: block_size must be positive");
    lci_status st = check_index_args(batch, S, H_i, d_c, nb_max, topk, dtype);
    if (st != LCI_OK) return st;
    if (phase != LCI_PHASE_AUTO && phase != LCI_PHASE_PREFILL && phase != LCI_PHASE_DECODE)
        return fail(LCI_ERR_INVALID_ARG, "index_select_noalloc: unknown phase %d", (int)phase);
    if (!aligned16(q_c) || !aligned16(k_c))
        return fail(LCI_ERR_INVALID_ARG, "index_select_noalloc: q_c and k_c must be 16-byte aligned");
    const int K = H_i * d_c;
    const IndexPlan pl = plan_index(batch, S, K, nb_max, dtype_size(dtype));
    if (pl.bytes > (size_t)LCI_NOALLOC_SCRATCH_BYTES)
        return fail(LCI_ERR_WORKSPACE, "index_select_noalloc: these sizes need %zu bytes of scratch; "
                    "the built-in scratch holds %u", pl.bytes, (unsigned)LCI_NOALLOC_SCRATCH_BYTES);
    void* scratch = nullptr;
    st = noalloc_scratch(&scratch);
    if (st != LCI_OK) return st;
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    // The arrival counters must start at zero; the array holds the last call's data.
    cudaError_t e = cudaMemsetAsync(static_cast<char*>(scratch) + pl.off_counters, 0,
                                    (size_t)batch * S * sizeof(unsigned int), cs);
    if (e != cudaSuccess) return fail(LCI_ERR_CUDA, "index_select_noalloc: %s", cudaGetErrorString(e));
    if (dtype == LCI_F32)
        return launch_index_gemv<float>(q_c, k_c, batch, S, K, block_size, nb_max, d_ctx_len,
                                        d_q_start, topk, d_ids, scratch, pl, cs);
    return launch_index_gemv<__nv_bfloat16>(q_c, k_c, batch, S, K, block_size, nb_max, d_ctx_len,
                                            d_q_start, topk, d_ids, scratch, pl, cs);
}

extern "C" {

// ---- fused decode step ----

struct DecodePlan {
    IndexPlan ix;
    bool fused;                 // the one-launch persistent kernel
    int nsplit;                 // attention splits per (row, KV head) pair (fused)
    size_t off_ready;           // publication flags of the two-kernel form (0 / 1)
    size_t off_picks;           // published (block id, page) picks of the two-kernel form
    size_t off_pready;          // publication flags of the one-launch form (call epochs)
    size_t off_split, off_sync, off_part, bytes;
};

// The one-launch kernel covers bf16 keys of 1024 features (2 KiB per block)
// over the decode attention kernel's shapes.
bool fused_decode_fits(lci_dtype dtype, int32_t K, const lci_block_table* t, int32_t H_q,
                       const void* k_pool, const void* v_pool) {
    return dtype == LCI_BF16 && K == 1024 && decode_kernel_fits(t, H_q, k_pool, v_pool);
}

DecodePlan plan_decode(int32_t batch, int32_t S, int32_t K, int32_t nb_max, size_t esz,
                       int32_t topk, const lci_block_table* t, int32_t H_q, bool fused) {
    DecodePlan d{};
    d.ix = plan_index(batch, S, K, nb_max, esz);
    d.fused = fused;
    const size_t rows = (size_t)batch * S;
    d.off_ready = align_up(d.ix.bytes);
    d.off_picks = d.off_ready + align_up(rows * sizeof(unsigned int));
    size_t end = d.off_picks + align_up(rows * (size_t)topk * sizeof(unsigned long long));
    if (fused) {
        // splits: about two attention items per SM, at least two 64-token tiles each
        const long long pairs = (long long)rows * t->num_kv_heads;
        const int nunits = topk * (t->block_size / 64);
        long long want = (2 * 148 + pairs - 1) / pairs;
        if (want > 32) want = 32;
        if (want > nunits / 2) want = nunits / 2;
        if (want < 1) want = 1;
        const int per = (int)((nunits + want - 1) / want);
        d.nsplit = (nunits + per - 1) / per;
        // the one-launch form keeps its own flags: the two-kernel form leaves
        // its flags at 1, which is an epoch value the one-launch form waits for
        d.off_pready = end;
        d.off_split = d.off_pready + align_up(rows * sizeof(unsigned int));
        d.off_sync = d.off_split + align_up((size_t)pairs * sizeof(unsigned int));
        d.off_part = d.off_sync + kAlign;
        end = d.off_part + align_up((size_t)pairs * d.nsplit * lci::fdec::kPartFloats * sizeof(float));
    }
    (void)H_q;
    d.bytes = end;
    return d;
}

lci_status lci_sparse_decode_workspace_size(int32_t batch, int32_t S, int32_t H_i, int32_t d_c,
                                            int32_t topk, int32_t H_q,
                                            const lci_block_table* table, size_t* bytes) {
    if (!bytes || !table)
        return fail(LCI_ERR_INVALID_ARG, "sparse_decode_workspace_size: null argument");
    lci_status st = check_index_args(batch, S, H_i, d_c, table->max_blocks, topk, LCI_BF16);
    if (st != LCI_OK && st != LCI_ERR_UNSUPPORTED) return st;
    st = check_attn_args(batch, S, H_q, table, topk);
    if (st != LCI_OK) return st;
    const int K = H_i * d_c;
    // enough for either schedule (the fused one is chosen when the call fits it)
    const bool fused = table->dtype == LCI_BF16 && K == 1024 &&
                       fused_decode_fits(LCI_BF16, K, table, H_q, nullptr, nullptr);
    *bytes = plan_decode(batch, S, K, table->max_blocks, 2, topk, table, H_q, fused).bytes;
    return ok();
}

lci_status launch_decode_fused(const void* q_c, const void* k_c, int32_t batch, int32_t S,
                               int32_t nb_max, const int32_t* ctx_len, const int32_t* q_start,
                               int32_t topk, const void* q, int32_t H_q, const void* k_pool,
                               const void* v_pool, const lci_block_table* t, float scale,
                               int32_t* ids, void* out, char* w, const DecodePlan& pl,
                               cudaStream_t st) {
    if ((long long)pl.ix.chunk_blocks * 2048 > lci::fdec::kChunkBytes)
        return fail(LCI_ERR_UNSUPPORTED, "sparse_decode: chunk of %d blocks too large",
                    pl.ix.chunk_blocks);
    CUtensorMap tm_k, tm_v;
    lci_status s = pool_maps(t, k_pool, v_pool, &tm_k, &tm_v);
    if (s != LCI_OK) return s;
    static std::once_flag once;
    static cudaError_t attr_err = cudaSuccess;
    static int num_sms = 148;
    std::call_once(once, [] {
        attr_err = cudaFuncSetAttribute(lci::sparse_decode_fused_kernel,
                                        cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        lci::fdec::kSmemBytes);
        int dev = 0;
        if (attr_err == cudaSuccess) attr_err = cudaGetDevice(&dev);
        if (attr_err == cudaSuccess)
            attr_err = cudaDeviceGetAttribute(&num_sms, cudaDevAttrMultiProcessorCount, dev);
    });
    if (attr_err != cudaSuccess)
        return fail(LCI_ERR_CUDA, "sparse_decode: %s", cudaGetErrorString(attr_err));
    const int rows = batch * S;
    const long long items = (long long)rows * pl.ix.nchunks +
                            (long long)rows * t->num_kv_heads * pl.nsplit;
    if (items >= (1ll << 31)) return fail(LCI_ERR_UNSUPPORTED, "sparse_decode: too many work items");
    const int grid = (int)std::min<long long>(num_sms, items);
    const float scale_log2 = scale * 1.4426950408889634f;
    lci::sparse_decode_fused_kernel<<<grid, lci::fdec::kThreads, lci::fdec::kSmemBytes, st>>>(
        static_cast<const __nv_bfloat16*>(q_c), static_cast<const __nv_bfloat16*>(k_c), S, nb_max,
        t->block_size, ctx_len, q_start, topk, pl.ix.chunk_blocks, pl.ix.nchunks,
        reinterpret_cast<float*>(w + pl.ix.off_scores), reinterpret_cast<uint32_t*>(w + pl.ix.off_chunk_max),
        reinterpret_cast<unsigned int*>(w + pl.ix.off_counters), ids, tm_k, tm_v,
        static_cast<const __nv_bfloat16*>(q), t->d_table, t->num_pages, t->num_kv_heads, H_q,
        scale_log2, static_cast<__nv_bfloat16*>(out), pl.nsplit,
        reinterpret_cast<float*>(w + pl.off_part), reinterpret_cast<unsigned int*>(w + pl.off_split),
        reinterpret_cast<unsigned int*>(w + pl.off_pready), reinterpret_cast<unsigned int*>(w + pl.off_sync),
        rows);
    return check_launch("sparse_decode");
}

static lci_status sparse_decode_impl(const void* q_c, const void* k_c, lci_dtype dtype,
                                     int32_t batch, int32_t S, int32_t H_i, int32_t d_c,
                                     int32_t nb_max, const int32_t* d_ctx_len,
                                     const int32_t* d_q_start, int32_t topk, const void* q,
                                     int32_t H_q, const void* k_pool, const void* v_pool,
                                     const lci_block_table* table, float scale, int32_t* d_ids,
                                     void* out, void* workspace, size_t workspace_bytes,
                                     void* stream, bool one_launch) {
    if (!q_c || !k_c || !d_ctx_len || !d_q_start || !d_ids || !q || !k_pool || !v_pool || !out)
        return fail(LCI_ERR_INVALID_ARG, "sparse_decode: null pointer argument");
    lci_status st = check_index_args(batch, S, H_i, d_c, nb_max, topk, dtype);
    if (st != LCI_OK) return st;
    st = check_attn_args(batch, S, H_q, table, topk);
    if (st != LCI_OK) return st;
    if (table->max_blocks != nb_max)
        return fail(LCI_ERR_INVALID_ARG, "sparse_decode: nb_max %d differs from the table's %d",
                    nb_max, table->max_blocks);
    if (dtype != table->dtype)
        return fail(LCI_ERR_INVALID_ARG, "sparse_decode: q_c/k_c and the pools differ in dtype");
    if (!aligned16(q_c) || !aligned16(k_c))
        return fail(LCI_ERR_INVALID_ARG, "sparse_decode: q_c and k_c must be 16-byte aligned");
    const int K = H_i * d_c;
    const bool fused = one_launch;
    if (one_launch && !fused_decode_fits(dtype, K, table, H_q, k_pool, v_pool))
        return fail(LCI_ERR_UNSUPPORTED, "sparse_decode_persistent: needs bf16 keys of H_i*d_c = "
                    "1024, bf16 pools of head_dim 128, block_size a multiple of 64, at most 16 "
                    "query heads per KV head and 16-byte aligned pools");
    const DecodePlan pl = plan_decode(batch, S, K, nb_max, dtype_size(dtype), topk, table, H_q,
                                      fused);
    if (!workspace || workspace_bytes < pl.bytes ||
        (reinterpret_cast<uintptr_t>(workspace) & (kAlign - 1)) != 0)
        return fail(LCI_ERR_WORKSPACE, "sparse_decode: workspace needs %zu bytes, 256-byte aligned "
                    "(got %zu at %p)", pl.bytes, workspace_bytes, workspace);
    if (!(scale > 0.f)) scale = 1.0f / std::sqrt((float)table->head_dim);
    if (!std::isfinite(scale)) return fail(LCI_ERR_INVALID_ARG, "sparse_decode: non-finite scale");
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    char* w = static_cast<char*>(workspace);
    if (pl.fused)
        return launch_decode_fused(q_c, k_c, batch, S, nb_max, d_ctx_len, d_q_start, topk, q, H_q,
                                   k_pool, v_pool, table, scale, d_ids, out, w, pl, cs);
    if (dtype == LCI_BF16 && decode_kernel_fits(table, H_q, k_pool, v_pool)) {
        // rows are published one by one and attended as soon as they are ready:
        // as (block id, page) picks from the streaming index kernel, else as a
        // flag per row
        if (pl.ix.stream) {
            unsigned long long* picks = reinterpret_cast<unsigned long long*>(w + pl.off_picks);
            st = launch_index_gemv<__nv_bfloat16>(q_c, k_c, batch, S, K, table->block_size, nb_max,
                                                  d_ctx_len, d_q_start, topk, d_ids, workspace,
                                                  pl.ix, cs, nullptr, nullptr, 0, table->d_table,
                                                  picks);
            if (st != LCI_OK) return st;
            return launch_attn_decode(q, batch, S, H_q, k_pool, v_pool, table, d_ids, topk,
                                      d_ctx_len, d_q_start, scale, out, cs, nullptr, true, nullptr,
                                      picks);
        }
        unsigned int* ready = reinterpret_cast<unsigned int*>(w + pl.off_ready);
        st = launch_index_gemv<__nv_bfloat16>(q_c, k_c, batch, S, K, table->block_size, nb_max,
                                              d_ctx_len, d_q_start, topk, d_ids, workspace, pl.ix,
                                              cs, ready);
        if (st != LCI_OK) return st;
        return launch_attn_decode(q, batch, S, H_q, k_pool, v_pool, table, d_ids, topk, d_ctx_len,
                                  d_q_start, scale, out, cs, ready, true);
    }
    // other shapes: the two calls in sequence
    st = dtype == LCI_F32
             ? launch_index_gemv<float>(q_c, k_c, batch, S, K, table->block_size, nb_max, d_ctx_len,
                                        d_q_start, topk, d_ids, workspace, pl.ix, cs)
             : launch_index_gemv<__nv_bfloat16>(q_c, k_c, batch, S, K, table->block_size, nb_max,
                                                d_ctx_len, d_q_start, topk, d_ids, workspace, pl.ix,
                                                cs);
    if (st != LCI_OK) return st;
    if (table->dtype == LCI_F32)
        return launch_attn_simt<float>(q, batch, S, H_q, k_pool, v_pool, table, d_ids, topk,
                                       d_ctx_len, d_q_start, scale, out, cs);
    if (decode_kernel_fits(table, H_q, k_pool, v_pool))
        return launch_attn_decode(q, batch, S, H_q, k_pool, v_pool, table, d_ids, topk, d_ctx_len,
                                  d_q_start, scale, out, cs);
    return launch_attn_simt<__nv_bfloat16>(q, batch, S, H_q, k_pool, v_pool, table, d_ids, topk,
                                           d_ctx_len, d_q_start, scale, out, cs);
}

lci_status lci_sparse_decode(const void* q_c, const void* k_c, lci_dtype dtype, int32_t batch,
                             int32_t S, int32_t H_i, int32_t d_c, int32_t nb_max,
                             const int32_t* d_ctx_len, const int32_t* d_q_start, int32_t topk,
                             const void* q, int32_t H_q, const void* k_pool, const void* v_pool,
                             const lci_block_table* table, float scale, int32_t* d_ids, void* out,
                             void* workspace, size_t workspace_bytes, void* stream) {
    return sparse_decode_impl(q_c, k_c, dtype, batch, S, H_i, d_c, nb_max, d_ctx_len, d_q_start,
                              topk, q, H_q, k_pool, v_pool, table, scale, d_ids, out, workspace,
                              workspace_bytes, stream, false);
}

lci_status lci_sparse_decode_persistent(const void* q_c, const void* k_c, lci_dtype dtype,
                                        int32_t batch, int32_t S, int32_t H_i, int32_t d_c,
                                        int32_t nb_max, const int32_t* d_ctx_len,
                                        const int32_t* d_q_start, int32_t topk, const void* q,
                                        int32_t H_q, const void* k_pool, const void* v_pool,
                                        const lci_block_table* table, float scale, int32_t* d_ids,
                                        void* out, void* workspace, size_t workspace_bytes,
                                        void* stream) {
    return sparse_decode_impl(q_c, k_c, dtype, batch, S, H_i, d_c, nb_max, d_ctx_len, d_q_start,
                              topk, q, H_q, k_pool, v_pool, table, scale, d_ids, out, workspace,
                              workspace_bytes, stream, true);
}

lci_status lci_get_device_status(void* stream) {
    cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return fail(LCI_ERR_CUDA, "get_device_status: %s", cudaGetErrorString(e));
    unsigned int v = 0, zero = 0;
    e = cudaMemcpyFromSymbol(&v, lci::g_device_status, sizeof v);
    if (e == cudaSuccess) e = cudaMemcpyToSymbol(lci::g_device_status, &zero, sizeof zero);
    if (e != cudaSuccess) return fail(LCI_ERR_CUDA, "get_device_status: %s", cudaGetErrorString(e));
    if (v == 0) return ok();
    const lci_status code = (v & lci::kStatusTimeout) ? LCI_ERR_TIMEOUT : LCI_ERR_DEVICE_BOUNDS;
    return fail(code, "device status flags 0x%x:%s%s%s", v,
                (v & lci::kStatusBadBlockId) ? " block id out of range" : "",
                (v & lci::kStatusBadPage) ? " page out of range" : "",
                (v & lci::kStatusTimeout) ? " bounded wait timed out" : "");
}

lci_status lci_set_wait_limit_ns(uint64_t ns) {
    if (ns == 0 || ns > kMaxWaitLimitNs)
        return fail(LCI_ERR_INVALID_ARG, "set_wait_limit_ns: %llu outside [1, %llu]",
                    (unsigned long long)ns, (unsigned long long)kMaxWaitLimitNs);
    const unsigned long long v = ns;
    cudaError_t e = cudaMemcpyToSymbol(lci::g_wait_limit_ns, &v, sizeof v);
    if (e != cudaSuccess) return fail(LCI_ERR_CUDA, "set_wait_limit_ns: %s", cudaGetErrorString(e));
    return ok();
}

lci_status lci_get_wait_limit_ns(uint64_t* ns) {
    if (!ns) return fail(LCI_ERR_INVALID_ARG, "get_wait_limit_ns: null output");
    unsigned long long v = 0;
    cudaError_t e = cudaMemcpyFromSymbol(&v, lci::g_wait_limit_ns, sizeof v);
    if (e != cudaSuccess) return fail(LCI_ERR_CUDA, "get_wait_limit_ns: %s", cudaGetErrorString(e));
    *ns = v;
    return ok();
}

lci_status lci_sparse_attn_pipelined(const void* q, int32_t batch, int32_t S, int32_t H_q,
                                     const void* k_pool, const void* v_pool,
                                     const lci_block_table* table, const int32_t* d_ids,
                                     int32_t topk, const int32_t* d_ctx_len,
                                     const int32_t* d_q_start, float scale,
                                     const uint32_t* d_ready, void* out, void* stream) {
    if (!q || !k_pool || !v_pool || !d_ids || !d_ctx_len || !d_q_start || !d_ready || !out)
        return fail(LCI_ERR_INVALID_ARG, "sparse_attn_pipelined: null pointer argument");
    lci_status st = check_attn_args(batch, S, H_q, table, topk);
    if (st != LCI_OK) return st;
    if (!decode_kernel_fits(table, H_q, k_pool, v_pool))
        return fail(LCI_ERR_UNSUPPORTED, "sparse_attn_pipelined: needs bf16 pools, head_dim 128, "
                    "block_size a multiple of 64, at most 16 query heads per KV head and "
                    "16-byte aligned pools");
    if (!(scale > 0.f)) scale = 1.0f / std::sqrt((float)table->head_dim);
    if (!std::isfinite(scale)) return fail(LCI_ERR_INVALID_ARG, "sparse_attn_pipelined: non-finite scale");
    return launch_attn_decode(q, batch, S, H_q, k_pool, v_pool, table, d_ids, topk, d_ctx_len,
                              d_q_start, scale, out, static_cast<cudaStream_t>(stream),
                              reinterpret_cast<const unsigned int*>(d_ready), false);
}

}  // extern "C"
