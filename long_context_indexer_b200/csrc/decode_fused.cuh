// decode_fused.cuh -- one decode step (A1 + A2 + A3 + A4) in one persistent
// launch ([GPU-stack] "Separate Paths for Prefill and Decode": decode as a
// pipeline of index prefetching and incremental aggregation; [Hetero] §IV:
// index retrieval and attention computation pipelined so that retrieval
// latency is hidden).
//
// About one CTA per SM. Every CTA claims work items from one global counter,
// in order:
//   items [0, rows*nchunks)      scoring: one chunk of a query row's block keys
//                                (bulk copies, up to kBufs chunks in flight per
//                                CTA), scores to the workspace; the last chunk
//                                of a row to finish runs the exact top-k select
//                                and publishes the row (release store of the
//                                call's epoch in ready[row])
//   items [.., + pairs*nsplit)   attention: a split of one (row, KV head) pair's
//                                selected 64-token tiles, TMA-fed, mma.sync with
//                                online softmax; the split's partial (m, l, o) goes
//                                to the workspace and the last split of the pair
//                                to finish combines them into the output
// A CTA takes an attention item only after every scoring item has been claimed
// by a running CTA, and scoring never waits on anything, so every row it waits
// for is published: the launch cannot deadlock, whatever the residency. Rows
// are claimed in order, so the attention of early rows overlaps the scoring of
// later ones.
//
// Per-call state (claim and exit counters, the epoch) lives in the workspace:
// the last CTA to exit resets the counters and advances the epoch, so a zeroed
// workspace serves every later call of the same sizes.
#pragma once

#include "attn_decode.cuh"
#include "common.cuh"
#include "index_gemv.cuh"
#include "ptx.cuh"
#include "topk_select.cuh"

namespace lci {

namespace fdec {
constexpr int kThreads = 256;        // 8 warps: all score; 4 consume + 1 produce in attention
constexpr int kStages = 6;           // attention ring, 32 KiB per stage
constexpr int kBufs = 4;             // scoring chunks in flight, 32 KiB each
constexpr int kChunkBytes = 32768;
constexpr int kRingBytes = kStages * dec::kStageBytes;  // 192 KiB
constexpr int kOffSel = kRingBytes;
constexpr int kOffBar = kOffSel + (int)((sizeof(SelectSmem) + 1023) / 1024 * 1024);
constexpr int kSmemBytes = kOffBar + 512 + 1024;
constexpr int kPartFloats = 2 * dec::kRows + dec::kRows * dec::kHD;  // m, l, o[16][128]
// sync words in the workspace
enum { kEpoch = 0, kClaim = 1, kExit = 2 };
}  // namespace fdec

__global__ void __launch_bounds__(fdec::kThreads, 1) sparse_decode_fused_kernel(
    // index selection
    const __nv_bfloat16* __restrict__ q_c, const __nv_bfloat16* __restrict__ k_c, int S, int nb_max,
    int bs, const int32_t* __restrict__ ctx_len, const int32_t* __restrict__ q_start, int topk,
    int chunk_blocks, int nchunks, float* __restrict__ scores, uint32_t* __restrict__ chunk_max,
    unsigned int* __restrict__ row_counter, int32_t* __restrict__ ids,
    // attention
    const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
    const __nv_bfloat16* __restrict__ q, const int32_t* __restrict__ table, int num_pages,
    int H_kv, int H_q, float scale_log2, __nv_bfloat16* __restrict__ out, int nsplit,
    float* __restrict__ part, unsigned int* __restrict__ split_counter,
    // protocol
    unsigned int* __restrict__ ready, unsigned int* __restrict__ sync_words, int rows) {
    using namespace dec;
    constexpr int K = 1024;          // H_i * d_c: 2 KiB bf16 block keys
    constexpr int KV = 4;            // 16-byte chunks of a key per lane
    constexpr int NW = fdec::kThreads / 32;
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char* smem = reinterpret_cast<unsigned char*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    SelectSmem& sel = *reinterpret_cast<SelectSmem*>(smem + fdec::kOffSel);
    uint64_t* abar = reinterpret_cast<uint64_t*>(smem + fdec::kOffBar);  // [kBufs]
    uint64_t* full_bar = abar + fdec::kBufs;                             // [kStages]
    uint64_t* empty_bar = full_bar + fdec::kStages;                      // [kStages]
    int* info = reinterpret_cast<int*>(empty_bar + fdec::kStages);      // [kStages]
    int* s_item = info + fdec::kStages;                                  // [kBufs]
    int* s_ctl = s_item + fdec::kBufs;                                   // [8] broadcasts
    uint32_t* s_max = reinterpret_cast<uint32_t*>(s_ctl + 8);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int items_a = rows * nchunks;
    const int pairs = rows * H_kv;
    const int items_total = items_a + pairs * nsplit;
    const int G = H_q / H_kv;
    const int tiles_per_block = bs / kTile;
    const unsigned int epoch = ld_relaxed_gpu(sync_words + fdec::kEpoch) + 1u;

    if (tid == 0) {
        for (int i = 0; i < fdec::kBufs; ++i) mbar_init(&abar[i], 1);
        for (int i = 0; i < fdec::kStages; ++i) {
            mbar_init(&full_bar[i], 1);
            mbar_init(&empty_bar[i], kConsumers);
        }
        fence_mbar_init();
    }
    if (warp == kConsumers && lane == 0) {
        prefetch_tensormap(&tm_k);
        prefetch_tensormap(&tm_v);
    }
    __syncthreads();

    // ======================= scoring (A1 + A2) =======================
    // s_ctl[0]: items claimed and loading (tail), s_ctl[1]: the first claimed
    // attention item (or items_total), s_ctl[2]: the select flag
    int head = 0, tail = 0;
    bool more = true;
    int first_b = items_total;
    auto chunk_range = [&](int w, int& row, int& chunk, int& j0, int& j1, int& vis) {
        row = w / nchunks;
        chunk = w - row * nchunks;
        const int b = row / S, s = row - b * S;
        vis = visible_blocks((long long)__ldg(&q_start[b]) + s, __ldg(&ctx_len[b]), bs, nb_max);
        j0 = chunk * chunk_blocks;
        j1 = min(j0 + chunk_blocks, vis);
    };
    for (;;) {
        if (tid == 0) {
            while (more && tail - head < fdec::kBufs) {
                const int w = (int)atomicAdd(sync_words + fdec::kClaim, 1u);
                if (w >= items_a) {
                    more = false;
                    first_b = w;
                    break;
                }
                const int slot = tail % fdec::kBufs;
                s_item[slot] = w;
                int row, chunk, j0, j1, vis;
                chunk_range(w, row, chunk, j0, j1, vis);
                if (j0 < j1) {
                    const uint32_t bytes = (uint32_t)(j1 - j0) * (uint32_t)(K * 2);
                    const unsigned char* src = reinterpret_cast<const unsigned char*>(
                        k_c + ((size_t)(row / S) * nb_max + j0) * K);
                    unsigned char* dst = smem + slot * fdec::kChunkBytes;
                    mbar_arrive_expect_tx(&abar[slot], bytes);
                    for (uint32_t off = 0; off < bytes; off += 16384u)
                        bulk_load(dst + off, src + off, min(16384u, bytes - off), &abar[slot]);
                } else {
                    mbar_arrive(&abar[slot]);
                }
                ++tail;
            }
            s_ctl[0] = tail;
            s_ctl[1] = more ? -1 : first_b;
        }
        __syncthreads();
        tail = s_ctl[0];
        if (s_ctl[1] >= 0) {
            more = false;
            first_b = s_ctl[1];
        }
        if (head == tail) break;
        const int slot = head % fdec::kBufs;
        const int w = s_item[slot];
        int row, chunk, j0, j1, vis;
        chunk_range(w, row, chunk, j0, j1, vis);
        if (tid == 0) *s_max = 0u;
        const bool ok = mbar_wait(&abar[slot], (head / fdec::kBufs) & 1);
        __syncthreads();  // s_max cleared before any update
        float* row_scores = scores + (size_t)row * nb_max;
        if (ok && j0 < j1) {
            const __nv_bfloat16* qrow = q_c + (size_t)row * K;
            float qv[KV][8];
#pragma unroll
            for (int c = 0; c < KV; ++c) {
                const uint4 raw = *reinterpret_cast<const uint4*>(qrow + (lane + 32 * c) * 8);
                const __nv_bfloat16* e8 = reinterpret_cast<const __nv_bfloat16*>(&raw);
#pragma unroll
                for (int e = 0; e < 8; ++e) qv[c][e] = __bfloat162float(e8[e]);
            }
            const unsigned char* tile = smem + slot * fdec::kChunkBytes;
            for (int j = j0 + warp; j < j1; j += NW) {
                const uint4* kr = reinterpret_cast<const uint4*>(tile + (size_t)(j - j0) * K * 2);
                float acc = 0.f;
#pragma unroll
                for (int c = 0; c < KV; ++c) acc += dot_chunk(kr[lane + 32 * c], qv[c], __nv_bfloat16());
                acc = warp_sum(acc);
                if (lane == 0) {
                    row_scores[j] = acc;
                    atomicMax(s_max, score_key(acc));
                }
            }
        }
        __syncthreads();  // the buffer is read; the chunk maximum is final
        ++head;
        if (tid == 0) {
            if (j0 < j1) chunk_max[(size_t)row * nchunks + chunk] = *s_max;
            __threadfence();
            const unsigned prev = atomicAdd(&row_counter[row], 1u);
            s_ctl[2] = prev == (unsigned)(nchunks - 1);
        }
        __syncthreads();
        if (s_ctl[2]) {
            // the row's last chunk: select its blocks and publish the row
            __threadfence();
            if (tid == 0) row_counter[row] = 0u;
            cta_topk_select<fdec::kThreads>(row_scores, chunk_max + (size_t)row * nchunks, vis,
                                            chunk_blocks, topk, ids + (size_t)row * topk, sel);
            __syncthreads();
            if (tid == 0) {
                __threadfence();
                st_release_gpu(ready + row, epoch);
            }
        }
    }

    // ======================= attention (A3 + A4) =======================
    // The scoring buffers were read by generic loads; the ring is written by
    // TMA (async proxy) from here on.
    fence_proxy_async_smem();
    __syncthreads();
    const int g8 = lane >> 2, q4 = lane & 3;
    int it_base = 0;  // ring iterations so far (phases continue across items)
    int w = first_b;
    float* wo = reinterpret_cast<float*>(smem);           // combine scratch (ring is idle)
    constexpr int kSlots = 64, kElems = kSlots * 32;
    float* wm = wo + kConsumers * kElems;
    float* wl = wm + kConsumers * kRows;
    float* wf = wl + kConsumers * kRows;
    float* cm = wf + kConsumers * kRows;
    float* cl = cm + kRows;
    while (w < items_total) {
        // claim the next item now: the atomic's round trip overlaps this item
        int next_w = 0;
        if (tid == 0) next_w = (int)atomicAdd(sync_words + fdec::kClaim, 1u);
        const int wb = w - items_a;
        const int pair = wb / nsplit, split = wb - pair * nsplit;
        const int row = pair / H_kv, g = pair - row * H_kv;
        const int b = row / S, s = row - b * S;
        const int nunits = topk * tiles_per_block;
        const int per = (nunits + nsplit - 1) / nsplit;
        const int u0 = split * per;
        const int u1 = min(nunits, u0 + per);
        const long long p = (long long)__ldg(&q_start[b]) + s;
        const long long ctx = __ldg(&ctx_len[b]);
        const long long last = p < ctx - 1 ? p : ctx - 1;
        if (tid == 0) {
            bool alive = ld_acquire_gpu(ready + row) == epoch;
            if (!alive) {  // bounded wait for the row's publication
                const unsigned long long t0 = global_ns();
                const unsigned long long limit = g_wait_limit_ns;
                unsigned int sleep_ns = 32;
                while (!alive) {
                    __nanosleep(sleep_ns);
                    alive = ld_acquire_gpu(ready + row) == epoch;
                    if (!alive && global_ns() - t0 > limit) {
                        raise_status(kStatusTimeout);
                        break;
                    }
                    sleep_ns = sleep_ns < 512 ? 2 * sleep_ns : 512;
                }
            }
            s_ctl[3] = alive;
        }
        __syncthreads();
        const bool alive = s_ctl[3] != 0;

        float m_a = -INFINITY, m_b = -INFINITY, l_a = 0.f, l_b = 0.f;
        float o[2][8][4];
#pragma unroll
        for (int hh = 0; hh < 2; ++hh)
#pragma unroll
            for (int i = 0; i < 8; ++i)
#pragma unroll
                for (int e = 0; e < 4; ++e) o[hh][i][e] = 0.f;

        if (warp == kConsumers) {
            // ---------------- producer ----------------
            const int32_t* row_ids = ids + (size_t)row * topk;
            for (int base = u0; base < u1; base += 32) {
                const int u = base + lane;
                int t0 = -1, y = 0;
                if (u < u1 && alive) {
                    const int i = u / tiles_per_block, sub = u - i * tiles_per_block;
                    const int j = __ldcg(row_ids + i);
                    if (j >= 0 && j < nb_max) {
                        const int page = table[(size_t)b * nb_max + j];
                        if (page < 0 || page >= num_pages) {
                            raise_status(kStatusBadPage);
                        } else if ((long long)j * bs + sub * kTile <= last) {
                            t0 = j * bs + sub * kTile;
                            y = (page * H_kv + g) * bs + sub * kTile;
                        }
                    } else if (j != -1) {
                        raise_status(kStatusBadBlockId);
                    }
                }
                const int n = min(32, u1 - base);
                for (int k = 0; k < n; ++k) {
                    const int tk = __shfl_sync(0xffffffffu, t0, k);
                    const int yk = __shfl_sync(0xffffffffu, y, k);
                    const int it = it_base + base - u0 + k;
                    const int st = it % fdec::kStages;
                    if (lane == 0) {
                        if (it >= fdec::kStages)
                            mbar_wait(&empty_bar[st], ((it / fdec::kStages) - 1) & 1);
                        info[st] = tk;
                        if (tk < 0) {
                            mbar_arrive(&full_bar[st]);
                        } else {
                            unsigned char* dst = smem + st * kStageBytes;
                            mbar_arrive_expect_tx(&full_bar[st], kStageBytes);
                            tma_load_2d(dst, &tm_k, 0, yk, &full_bar[st]);
                            tma_load_2d(dst + kBox, &tm_k, 64, yk, &full_bar[st]);
                            tma_load_2d(dst + 2 * kBox, &tm_v, 0, yk, &full_bar[st]);
                            tma_load_2d(dst + 3 * kBox, &tm_v, 64, yk, &full_bar[st]);
                        }
                    }
                    __syncwarp();
                }
            }
        } else if (warp < kConsumers) {
            // ---------------- consumers ----------------
            uint4 qa[4], qb[4];
            const int ha = g8, hb = g8 + 8;
            const __nv_bfloat16* qrow = q + ((size_t)row * H_q + (size_t)g * G) * kHD;
#pragma unroll
            for (int sl = 0; sl < 4; ++sl) {
                const int d0 = 32 * sl + 8 * q4;
                qa[sl] = ha < G ? *reinterpret_cast<const uint4*>(qrow + (size_t)ha * kHD + d0)
                                : make_uint4(0, 0, 0, 0);
                qb[sl] = hb < G ? *reinterpret_cast<const uint4*>(qrow + (size_t)hb * kHD + d0)
                                : make_uint4(0, 0, 0, 0);
            }
            for (int u = u0; u < u1; ++u) {
                const int it = it_base + u - u0;
                const int st = it % fdec::kStages;
                const bool ok = mbar_wait(&full_bar[st], (it / fdec::kStages) & 1);
                const int t0 = info[st];
                if (ok && t0 >= 0)
                    dec_consume_tile(smem_u32(smem + st * kStageBytes), warp, g8, q4, t0, last,
                                     scale_log2, qa, qb, m_a, m_b, l_a, l_b, o);
                __syncwarp();
                if (lane == 0) mbar_arrive(&empty_bar[st]);
            }
        }
        it_base += u1 - u0;
        __syncthreads();  // every stage of the item consumed: the ring is idle

        // ---- the four consumer warps' partials -> this split's (m, l, o) ----
        if (warp < kConsumers) {
            l_a += __shfl_xor_sync(0xffffffffu, l_a, 1);
            l_a += __shfl_xor_sync(0xffffffffu, l_a, 2);
            l_b += __shfl_xor_sync(0xffffffffu, l_b, 1);
            l_b += __shfl_xor_sync(0xffffffffu, l_b, 2);
            if (q4 == 0) {
                wm[warp * kRows + g8] = m_a;
                wm[warp * kRows + g8 + 8] = m_b;
                wl[warp * kRows + g8] = l_a;
                wl[warp * kRows + g8 + 8] = l_b;
            }
            float* dst = wo + warp * kElems + lane;
#pragma unroll
            for (int hh = 0; hh < 2; ++hh)
#pragma unroll
                for (int i = 0; i < 8; ++i)
#pragma unroll
                    for (int e = 0; e < 4; ++e) dst[(32 * hh + 4 * i + e) * 32] = o[hh][i][e];
        }
        __syncthreads();
        if (tid < kRows) {
            float M = -INFINITY;
#pragma unroll
            for (int w2 = 0; w2 < kConsumers; ++w2) M = fmaxf(M, wm[w2 * kRows + tid]);
            const float base = M == -INFINITY ? 0.f : M;
            float L = 0.f;
#pragma unroll
            for (int w2 = 0; w2 < kConsumers; ++w2) {
                const float f = exp2f(wm[w2 * kRows + tid] - base);
                wf[w2 * kRows + tid] = f;
                L += f * wl[w2 * kRows + tid];
            }
            cm[tid] = M;
            cl[tid] = L;
        }
        __syncthreads();
        __nv_bfloat16* orow = out + ((size_t)row * H_q + (size_t)g * G) * kHD;
        float* pp = part + ((size_t)pair * nsplit + split) * fdec::kPartFloats;
        if (nsplit > 1 && tid < kRows) {
            pp[tid] = cm[tid];
            pp[kRows + tid] = cl[tid];
        }
        for (int sidx = tid; sidx < kElems; sidx += fdec::kThreads) {
            const int ln = sidx & 31, oi = sidx >> 5, e = oi & 3;
            const int hd_row = (ln >> 2) + 8 * (e >> 1);
            const int dim = 64 * (oi >> 5) + 16 * (ln & 3) + 8 * (e & 1) + ((oi >> 2) & 7);
            float acc = 0.f;
#pragma unroll
            for (int w2 = 0; w2 < kConsumers; ++w2)
                acc += wf[w2 * kRows + hd_row] * wo[w2 * kElems + sidx];
            if (nsplit == 1) {
                if (hd_row < G) {
                    const float L = cl[hd_row];
                    orow[hd_row * kHD + dim] = __float2bfloat16_rn(L > 0.f ? acc / L : 0.f);
                }
            } else {
                pp[2 * kRows + hd_row * kHD + dim] = acc;
            }
        }
        if (nsplit > 1) {
            // ---- the pair's last split combines every split's partial ----
            __threadfence();
            __syncthreads();
            if (tid == 0) {
                const unsigned prev = atomicAdd(&split_counter[pair], 1u);
                s_ctl[4] = prev == (unsigned)(nsplit - 1);
            }
            __syncthreads();
            if (s_ctl[4]) {
                __threadfence();
                const float* p0 = part + (size_t)pair * nsplit * fdec::kPartFloats;
                if (tid < kRows) {
                    float M = -INFINITY;
                    for (int c = 0; c < nsplit; ++c)
                        M = fmaxf(M, __ldcg(p0 + (size_t)c * fdec::kPartFloats + tid));
                    const float base = M == -INFINITY ? 0.f : M;
                    float L = 0.f;
                    for (int c = 0; c < nsplit; ++c) {
                        const float* pc = p0 + (size_t)c * fdec::kPartFloats;
                        L += exp2f(__ldcg(pc + tid) - base) * __ldcg(pc + kRows + tid);
                    }
                    cm[tid] = base;
                    cl[tid] = L > 0.f ? 1.f / L : 0.f;
                }
                __syncthreads();
                for (int x = tid; x < G * kHD; x += fdec::kThreads) {
                    const int hd_row = x / kHD;
                    float acc = 0.f;
                    for (int c = 0; c < nsplit; ++c) {
                        const float* pc = p0 + (size_t)c * fdec::kPartFloats;
                        acc += exp2f(__ldcg(pc + hd_row) - cm[hd_row]) * __ldcg(pc + 2 * kRows + x);
                    }
                    orow[x] = __float2bfloat16_rn(acc * cl[hd_row]);
                }
                if (tid == 0) split_counter[pair] = 0u;
            }
        }
        // the combine scratch is the ring: async-proxy writes come next
        fence_proxy_async_smem();
        __syncthreads();
        if (tid == 0) s_ctl[5] = next_w;
        __syncthreads();
        w = s_ctl[5];
    }

    // ---- the last CTA out resets the counters and advances the epoch ----
    __syncthreads();
    if (tid == 0) {
        __threadfence();
        const unsigned n = atomicAdd(sync_words + fdec::kExit, 1u);
        if (n == gridDim.x - 1) {
            sync_words[fdec::kClaim] = 0u;
            sync_words[fdec::kExit] = 0u;
            __threadfence();
            sync_words[fdec::kEpoch] = epoch;
        }
    }
}

}  // namespace lci
