// index_gemv.cuh -- block scoring fused with the causal-masked top-k, one query
// row at a time (the decode schedule; also the generic path for any S).
//
// Grid rows x chunks (1-D, chunk fastest). Each CTA scores one chunk of the row's causal-visible
// blocks: k_c rows stream from HBM with 16-byte loads, every warp dots them
// against the query row staged in shared memory and reduces with shuffles. The
// fp32 scores go to the workspace (L2-resident, 4 bytes per 2 KiB block key).
// The last CTA of the row to arrive (atomic counter, no spin-wait) runs the
// exact CTA radix select over the row's scores and writes the block ids, then
// resets the counter for the next call.
#pragma once

#include "common.cuh"
#include "ptx.cuh"
#include "topk_select.cuh"

namespace lci {

template <typename T> struct ElemsPer16B;
template <> struct ElemsPer16B<float> { static constexpr int v = 4; };
template <> struct ElemsPer16B<__nv_bfloat16> { static constexpr int v = 8; };

__device__ __forceinline__ float dot_chunk(const uint4& raw, const float* q, float) {
    return __uint_as_float(raw.x) * q[0] + __uint_as_float(raw.y) * q[1] +
           __uint_as_float(raw.z) * q[2] + __uint_as_float(raw.w) * q[3];
}

__device__ __forceinline__ float dot_chunk(const uint4& raw, const float* q, __nv_bfloat16) {
    const float2 a = bf16x2_to_f32(raw.x), b = bf16x2_to_f32(raw.y);
    const float2 c = bf16x2_to_f32(raw.z), d = bf16x2_to_f32(raw.w);
    return a.x * q[0] + a.y * q[1] + b.x * q[2] + b.y * q[3] + c.x * q[4] + c.y * q[5] +
           d.x * q[6] + d.y * q[7];
}

// Dot product of 16 bytes of a key with 16 bytes of the query, both packed.
__device__ __forceinline__ float dot16(const uint4& k, const uint4& q, float) {
    return __uint_as_float(k.x) * __uint_as_float(q.x) + __uint_as_float(k.y) * __uint_as_float(q.y) +
           __uint_as_float(k.z) * __uint_as_float(q.z) + __uint_as_float(k.w) * __uint_as_float(q.w);
}

__device__ __forceinline__ float dot16(const uint4& k, const uint4& q, __nv_bfloat16) {
    const float2 a = bf16x2_to_f32(k.x), b = bf16x2_to_f32(k.y);
    const float2 c = bf16x2_to_f32(k.z), d = bf16x2_to_f32(k.w);
    const float2 qa = bf16x2_to_f32(q.x), qb = bf16x2_to_f32(q.y);
    const float2 qc = bf16x2_to_f32(q.z), qd = bf16x2_to_f32(q.w);
    return a.x * qa.x + a.y * qa.y + b.x * qb.x + b.y * qb.y + c.x * qc.x + c.y * qc.y +
           d.x * qd.x + d.y * qd.y;
}

// KV > 0: every block key is KV*32 16-byte chunks (2 KiB for KV = 4) and lane l
// always owns chunks l + 32*c, so its slice of the query row lives in
// registers. KV == 0: any size, query row staged in shared memory.
template <typename T, int NT, int KV>
__global__ void __launch_bounds__(NT) index_gemv_select_kernel(
    const T* __restrict__ q_c, const T* __restrict__ k_c, int S, int K, int nb_max, int bs,
    const int32_t* __restrict__ ctx_len, const int32_t* __restrict__ q_start, int topk,
    int chunk_blocks, int nchunks, float* __restrict__ scores,
    uint32_t* __restrict__ chunk_max, unsigned int* __restrict__ counters,
    int32_t* __restrict__ ids, unsigned int* __restrict__ ready,
    const int32_t* __restrict__ page_table, int num_pages) {
    // Dynamic shared memory: [k_c chunk: chunk_blocks * K * sizeof(T)]
    // [query row: K floats, only when KV == 0]; the last CTA of a row reuses it
    // for the select's scratch.
    extern __shared__ __align__(128) unsigned char dyn_smem[];
    __shared__ uint64_t bar;
    __shared__ int s_last;
    __shared__ uint32_t s_max;
    constexpr int NW = NT / 32;
    constexpr int E = ElemsPer16B<T>::v;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    // chunk fastest: a row's CTAs are dispatched together, so rows complete (and
    // are selected) one after another instead of all at the end
    const int row = blockIdx.x / nchunks, chunk = blockIdx.x - row * nchunks;
    // Publication flags (one per row) start every call cleared: the row's first
    // CTA clears its flag before this CTA lets the dependent grid launch, so a
    // flag left set by an earlier call (say one whose consumer gave up waiting)
    // can never be taken for this call's publication. The row's publishing CTA
    // arrives on the row counter after this CTA, so it stores after the clear.
    if (ready != nullptr && chunk == 0) {
        if (tid == 0) {
            ready[row] = 0u;
            __threadfence();
        }
        __syncthreads();
    }
    // Let the attention kernel that follows on the stream start its prologue;
    // it waits for this grid's results (or its row's flag) before reading ids.
    pdl_trigger();
    const int b = row / S, s = row - b * S;
    const long long p = (long long)__ldg(&q_start[b]) + s;
    const int vis = visible_blocks(p, __ldg(&ctx_len[b]), bs, nb_max);
    const int j0 = chunk * chunk_blocks;
    const int j1 = min(j0 + chunk_blocks, vis);
    const size_t row_bytes = (size_t)K * sizeof(T);
    float* row_scores = scores + (size_t)row * nb_max;

    if (tid == 0) s_max = 0u;  // below every real key
    if (j0 < j1) {
        unsigned char* tile = dyn_smem;
        if (tid == 0) {
            mbar_init(&bar, 1);
            fence_mbar_init();
            const uint32_t bytes = (uint32_t)((j1 - j0) * row_bytes);
            mbar_arrive_expect_tx(&bar, bytes);
            if (page_table == nullptr) {
                // The chunk's block keys are one contiguous range of k_c.
                const unsigned char* src =
                    reinterpret_cast<const unsigned char*>(k_c + ((size_t)b * nb_max + j0) * K);
                for (uint32_t off = 0; off < bytes; off += 16384u)
                    bulk_load(tile + off, src + off, min(16384u, bytes - off), &bar);
            } else {
                // Paged block keys: one row per block, at the block's page.
                for (int j = j0; j < j1; ++j) {
                    int page = page_table[(size_t)b * nb_max + j];
                    if (page < 0 || page >= num_pages) {
                        raise_status(kStatusBadPage);
                        page = 0;  // keep the copy in bounds; the result is flagged
                    }
                    bulk_load(tile + (size_t)(j - j0) * row_bytes,
                              reinterpret_cast<const unsigned char*>(k_c + (size_t)page * K),
                              (uint32_t)row_bytes, &bar);
                }
            }
        }
        const T* qrow = q_c + (size_t)row * K;
        if constexpr (KV > 0) {
            // this lane's query slice: chunks lane + 32*c, E elements each
            float qv[KV][E];
#pragma unroll
            for (int c = 0; c < KV; ++c) {
                const uint4 raw = *reinterpret_cast<const uint4*>(qrow + (lane + 32 * c) * E);
                const T* e8 = reinterpret_cast<const T*>(&raw);
#pragma unroll
                for (int e = 0; e < E; ++e) qv[c][e] = to_f32(e8[e]);
            }
            __syncthreads();
            const bool ok = mbar_wait(&bar, 0);
            for (int j = j0 + warp; ok && j < j1; j += NW) {
                const uint4* kr = reinterpret_cast<const uint4*>(tile + (size_t)(j - j0) * row_bytes);
                float acc = 0.f;
#pragma unroll
                for (int c = 0; c < KV; ++c) acc += dot_chunk(kr[lane + 32 * c], qv[c], T());
                acc = warp_sum(acc);
                if (lane == 0) {
                    row_scores[j] = acc;
                    atomicMax(&s_max, score_key(acc));
                }
            }
        } else {
            float* qs = reinterpret_cast<float*>(dyn_smem + (size_t)chunk_blocks * row_bytes);
            for (int i = tid; i < K; i += NT) qs[i] = to_f32(qrow[i]);
            __syncthreads();
            const bool ok = mbar_wait(&bar, 0);
            const int nvec = K / E;
            for (int j = j0 + warp; ok && j < j1; j += NW) {
                const uint4* kr = reinterpret_cast<const uint4*>(tile + (size_t)(j - j0) * row_bytes);
                float acc = 0.f;
                for (int c = lane; c < nvec; c += 32) acc += dot_chunk(kr[c], qs + c * E, T());
                acc = warp_sum(acc);
                if (lane == 0) {
                    row_scores[j] = acc;
                    atomicMax(&s_max, score_key(acc));
                }
            }
        }
    }
    __syncthreads();
    if (tid == 0 && j0 < j1) chunk_max[(size_t)row * nchunks + chunk] = s_max;
    __threadfence();
    __syncthreads();
    if (tid == 0) {
        const unsigned prev = atomicAdd(&counters[row], 1u);
        s_last = (prev == (unsigned)(nchunks - 1));
    }
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    if (tid == 0) counters[row] = 0u;
    SelectSmem& sel = *reinterpret_cast<SelectSmem*>(dyn_smem);
    cta_topk_select<NT>(row_scores, chunk_max + (size_t)row * nchunks, vis, chunk_blocks, topk,
                        ids + (size_t)row * topk, sel);
    if (ready != nullptr) {  // publish the row to a consumer running concurrently
        __syncthreads();
        if (tid == 0) {
            __threadfence();
            st_release_gpu(ready + row, 1u);
        }
    }
}

// Streaming form for 2 KiB block keys (K = 1024 bf16 or 512 fp32), the decode
// schedule. Grid rows x ncta (ncta fastest), sized by the host so that every
// CTA is resident at once: CTA `part` of a row scores blocks
// [part*cta_blocks, +cta_blocks) of the visible range, streaming them through
// a two-stage ring of NW blocks (one per warp) filled by bulk copies, so its
// loads stay in flight back to back instead of waiting for a later wave. It
// records the maximum key of every `chunk_blocks` blocks (cta_blocks is a
// multiple of chunk_blocks); the last CTA of the row selects as above.
namespace ixs {
constexpr int kStages = 2;
constexpr int kRowBytes = 2048;
template <int NT> constexpr int smem_bytes() {
    return kStages * (NT / 32) * kRowBytes > (int)sizeof(SelectSmem) ? kStages * (NT / 32) * kRowBytes
                                                                      : (int)sizeof(SelectSmem);
}
}  // namespace ixs

//
// With `picks` (and the KV cache's block `table`), the row's selection is also
// published for an attention kernel running concurrently: picks[row][r] is
// (block id << 32 | page) of rank r, -1 for both past the selection, and
// kPickPending until written (the row's first CTA resets it every call).
template <typename T, int NT>
__global__ void __launch_bounds__(NT) index_stream_select_kernel(
    const T* __restrict__ q_c, const T* __restrict__ k_c, int S, int nb_max, int bs,
    const int32_t* __restrict__ ctx_len, const int32_t* __restrict__ q_start, int topk,
    int chunk_blocks, int cta_blocks, int ncta, int nchunks, float* __restrict__ scores,
    uint32_t* __restrict__ chunk_max, unsigned int* __restrict__ counters,
    int32_t* __restrict__ ids, unsigned int* __restrict__ ready,
    const int32_t* __restrict__ page_table, int num_pages,
    const int32_t* __restrict__ table, unsigned long long* __restrict__ picks) {
    constexpr int NW = NT / 32;
    constexpr int KV = ixs::kRowBytes / (16 * 32);  // 16-byte pieces per lane of a key
    constexpr int kStageBytes = NW * ixs::kRowBytes;
    constexpr int kMaxUnits = 64;  // chunk maxima one CTA records
    extern __shared__ __align__(128) unsigned char dyn_smem[];
    __shared__ uint64_t bars[ixs::kStages];
    __shared__ uint32_t s_umax[kMaxUnits];
    __shared__ int s_last;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int row = blockIdx.x / ncta, part = blockIdx.x - row * ncta;
    const int b = row / S, s = row - b * S;
    const int qs = __ldg(&q_start[b]), cl = __ldg(&ctx_len[b]);  // in flight during the clear
    // The row's publication flag (or picks) starts every call cleared (see the
    // kernel above).
    if (part == 0 && (ready != nullptr || picks != nullptr)) {
        if (ready != nullptr && tid == 0) ready[row] = 0u;
        if (picks != nullptr)
            for (int r = tid; r < topk; r += NT) picks[(size_t)row * topk + r] = kPickPending;
        __threadfence();
        __syncthreads();
    }
    pdl_trigger();
    const int vis = visible_blocks((long long)qs + s, cl, bs, nb_max);
    const int j0 = part * cta_blocks;
    const int j1 = min(j0 + cta_blocks, vis);
    const int nst = j0 < j1 ? (j1 - j0 + NW - 1) / NW : 0;  // stages of work
    float* row_scores = scores + (size_t)row * nb_max;
    const unsigned char* kbase = reinterpret_cast<const unsigned char*>(k_c);
    // Stage `it` covers blocks j0 + it*NW .. +NW: one contiguous copy of k_c, or
    // one copy per block at the block's page.
    auto issue = [&](int it) {
        const int a = j0 + it * NW, e = min(a + NW, j1);
        unsigned char* dst = dyn_smem + (it % ixs::kStages) * kStageBytes;
        uint64_t* bar = &bars[it % ixs::kStages];
        mbar_arrive_expect_tx(bar, (uint32_t)((e - a) * ixs::kRowBytes));
        if (page_table == nullptr) {
            bulk_load(dst, kbase + ((size_t)b * nb_max + a) * ixs::kRowBytes,
                      (uint32_t)((e - a) * ixs::kRowBytes), bar);
        } else {
            for (int j = a; j < e; ++j) {
                int page = page_table[(size_t)b * nb_max + j];
                if (page < 0 || page >= num_pages) {
                    raise_status(kStatusBadPage);
                    page = 0;  // keep the copy in bounds; the result is flagged
                }
                bulk_load(dst + (j - a) * ixs::kRowBytes, kbase + (size_t)page * ixs::kRowBytes,
                          ixs::kRowBytes, bar);
            }
        }
    };
    if (tid == 0) {
        for (int i = 0; i < ixs::kStages; ++i) mbar_init(&bars[i], 1);
        fence_mbar_init();
        for (int it = 0; it < nst && it < ixs::kStages; ++it) issue(it);
    }
    for (int u = tid; u < kMaxUnits; u += NT) s_umax[u] = 0u;  // below every real key
    // this lane's slice of the query row: pieces lane + 32*c, kept packed
    uint4 qv[KV];
    const uint4* qrow = reinterpret_cast<const uint4*>(q_c + (size_t)row * (ixs::kRowBytes / sizeof(T)));
#pragma unroll
    for (int c = 0; c < KV; ++c) qv[c] = __ldg(qrow + lane + 32 * c);
    __syncthreads();
    bool ok = true;
    for (int it = 0; it < nst; ++it) {
        const int st = it % ixs::kStages;
        ok = ok && mbar_wait(&bars[st], (uint32_t)((it / ixs::kStages) & 1));
        const int j = j0 + it * NW + warp;
        if (ok && j < j1) {
            const uint4* kr = reinterpret_cast<const uint4*>(dyn_smem + st * kStageBytes +
                                                             warp * ixs::kRowBytes);
            float acc = 0.f;
#pragma unroll
            for (int c = 0; c < KV; ++c) acc += dot16(kr[lane + 32 * c], qv[c], T());
            acc = warp_sum(acc);
            if (lane == 0) {
                row_scores[j] = acc;
                atomicMax(&s_umax[(j - j0) / chunk_blocks], score_key(acc));
            }
        }
        __syncthreads();  // stage st is read: refill it
        if (tid == 0 && ok && it + ixs::kStages < nst) issue(it + ixs::kStages);
    }
    if (j0 < j1) {
        const int u0 = j0 / chunk_blocks, nu = (j1 - j0 + chunk_blocks - 1) / chunk_blocks;
        for (int u = tid; u < nu; u += NT) chunk_max[(size_t)row * nchunks + u0 + u] = s_umax[u];
    }
    __syncthreads();  // this CTA's scores and chunk maxima are written
    if (tid == 0) {
        // the arrival releases them; the row's last arrival acquires every
        // earlier arrival's (the CTA barriers carry both to the other threads)
        const unsigned prev = atom_add_acq_rel_gpu(&counters[row], 1u);
        s_last = (prev == (unsigned)(ncta - 1));
    }
    __syncthreads();
    if (!s_last) return;
    if (tid == 0) counters[row] = 0u;
    SelectSmem& sel = *reinterpret_cast<SelectSmem*>(dyn_smem);
    int32_t* row_ids = ids + (size_t)row * topk;
    if (picks != nullptr) {
        // the table row is warm in L2 by the time the ranks are known
        const int32_t* trow = table + (size_t)b * nb_max;
        for (int l = tid * 32; l < nb_max; l += NT * 32) prefetch_l2(trow + l);
        unsigned long long* row_picks = picks + (size_t)row * topk;
        cta_topk_select<NT>(
            row_scores, chunk_max + (size_t)row * nchunks, vis, chunk_blocks, topk,
            [=](int rank, int id) {
                row_ids[rank] = id;
                const int page = id >= 0 ? __ldg(trow + id) : -1;
                row_picks[rank] = ((unsigned long long)(unsigned)id << 32) | (unsigned)page;
            },
            sel);
        return;
    }
    cta_topk_select<NT>(row_scores, chunk_max + (size_t)row * nchunks, vis, chunk_blocks, topk,
                        row_ids, sel);
    if (ready != nullptr) {  // publish the row to a consumer running concurrently
        __syncthreads();      // every id is written
        if (tid == 0) st_release_gpu(ready + row, 1u);
    }
}

}  // namespace lci
