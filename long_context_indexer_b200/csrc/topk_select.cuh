// topk_select.cuh -- exact CTA-wide top-k of block scores without a full sort.
//
// [GPU-stack] "Operatorizing Index Selection" and [AI-acc] §4.1 ask for a top-k
// that prunes candidates coarsely and then selects exactly, instead of sorting
// every score. Scores become order-preserving uint32 keys (larger score, larger
// key; -0.0 folded onto +0.0), and a key with its block id forms a 64-bit
// composite (key << 32 | ~id) whose order is the selection order: key
// descending, then block id ascending. A row's blocks are scored in chunks,
// and every chunk also reports its maximum key.
//
//  1. Chunk pruning (when the row has more blocks than one pass holds). The
//     k-th largest chunk maximum M is a lower bound of the k-th largest score:
//     the k chunks whose maxima are >= M hold k distinct scores >= M. So a
//     chunk whose maximum is below M holds no winner, and only the chunks with
//     maximum >= M are kept. Lossless, and so is any lower bound of M in its
//     place (used when there are many chunks: the k-th largest of the maxima
//     of groups of 4 chunk maxima).
//  2. Exact selection of at most 1024 candidates, in two barrier-free steps
//     joined by one CTA barrier: every warp sorts its share of the candidates
//     (32, 64 or 128 composites, bitonic network over registers and shuffles)
//     into shared memory; then the rank of each of a warp's best min(k, share)
//     is the number of candidates above it, the sum of one binary search per
//     warp list (unrolled, the eight searches interleave). Ranks are unique
//     (ids are), so the composites of rank < k are exactly the top k.
// Rows whose candidates still exceed one pass (long runs of equal scores), and
// k above 128, take an exact four-pass radix select over all scores read from
// global memory instead.
#pragma once

#include "common.cuh"

namespace lci {

constexpr int kMaxTopk = 256;
constexpr int kSortMaxK = 128;     // k handled by the sorted-list pass
constexpr int kSortMaxN = 1024;    // candidates per sorted-list pass (8 warps x 128)
constexpr int kMaxChunks = 1024;   // chunk maxima the pruning step ranks

struct SelectSmem {
    union {
        uint64_t lists[kSortMaxN];  // per-warp sorted composites
        struct {
            unsigned int hist[256];
            uint32_t win_key[kMaxTopk];
            int32_t win_id[kMaxTopk];
        } rad;                      // the radix fallback
    };
    int32_t surv[kMaxChunks];       // chunks kept by the pruning step
    int warp_tot[32];
    int bcast[8];
};

__device__ __forceinline__ uint32_t load_key(const float* scores, int i) {
    return score_key(__ldcg(scores + i));
}

// Composite of a key and a block id (id >= 0): larger key first, then lower
// id. 0 is below every composite of a real element and marks padding.
__device__ __forceinline__ uint64_t compose(uint32_t key, int id) {
    return ((uint64_t)key << 32) | (uint64_t)(0xFFFFFFFFu - (uint32_t)id);
}
__device__ __forceinline__ int composite_id(uint64_t c) {
    return (int)(0xFFFFFFFFu - (uint32_t)(c & 0xFFFFFFFFull));
}
__device__ __forceinline__ uint32_t composite_key(uint64_t c) { return (uint32_t)(c >> 32); }

__device__ __forceinline__ uint64_t shfl_xor_u64(uint64_t v, int m) {
    const uint32_t lo = __shfl_xor_sync(0xffffffffu, (uint32_t)v, m);
    const uint32_t hi = __shfl_xor_sync(0xffffffffu, (uint32_t)(v >> 32), m);
    return ((uint64_t)hi << 32) | lo;
}

// Bitonic sort of the warp's 32*E composites into descending order. Element
// index lane*E + r lives in register c[r] of that lane: index bits below
// log2(E) pair registers of one lane, higher bits pair lanes (shuffles).
template <int E>
__device__ __forceinline__ void warp_sort_desc(uint64_t (&c)[E]) {
    constexpr int N = 32 * E;
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int size = 2; size <= N; size <<= 1) {
#pragma unroll
        for (int d = size >> 1; d > 0; d >>= 1) {
            if (d < E) {
#pragma unroll
                for (int r = 0; r < E; ++r) {
                    const int p = r ^ d;
                    if (p > r) {
                        // blocks whose index has the `size` bit clear end descending
                        const bool desc = ((lane * E + r) & size) == 0;
                        const uint64_t a = c[r], b = c[p];
                        const bool swap = desc ? (a < b) : (a > b);
                        c[r] = swap ? b : a;
                        c[p] = swap ? a : b;
                    }
                }
            } else {
#pragma unroll
                for (int r = 0; r < E; ++r) {
                    const int idx = lane * E + r;
                    const uint64_t o = shfl_xor_u64(c[r], d / E);
                    const bool lower = (idx & d) == 0;
                    const bool desc = (idx & size) == 0;
                    const bool keep_max = lower == desc;
                    c[r] = keep_max ? (c[r] > o ? c[r] : o) : (c[r] < o ? c[r] : o);
                }
            }
        }
    }
}

// Top k (k <= kSortMaxK) of the m <= NT/32*32*E composites get(0..m): calls
// emit(rank, composite) once for each of the k best, rank 0 first. All NT
// threads call it; it ends with the list memory still in use (callers that
// reuse it synchronise first).
template <int NT, int E, typename Get, typename Emit>
__device__ __forceinline__ void sorted_topk_e(int m, int k, Get get, uint64_t* lists, Emit emit) {
    constexpr int NW = NT / 32, N = 32 * E;
    static_assert(NW * N <= kSortMaxN, "lists hold every warp's share");
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    uint64_t c[E];
#pragma unroll
    for (int r = 0; r < E; ++r) {
        const int i = warp * N + lane * E + r;
        c[r] = i < m ? get(i) : 0ull;
    }
    warp_sort_desc<E>(c);
    const int len = k < N ? k : N;
#pragma unroll
    for (int r = 0; r < E; ++r) lists[warp * N + lane * E + r] = c[r];
    __syncthreads();
    for (int e = threadIdx.x; e < NW * len; e += NT) {
        const int w = e / len, p = e - w * len;
        const uint64_t x = lists[w * N + p];
        if (x == 0ull) continue;  // padding
        int q[NW];
#pragma unroll
        for (int w2 = 0; w2 < NW; ++w2) q[w2] = 0;
#pragma unroll
        for (int s = N; s > 0; s >>= 1) {
#pragma unroll
            for (int w2 = 0; w2 < NW; ++w2) {
                const int idx = min(q[w2] + s - 1, N - 1);
                q[w2] += (q[w2] + s <= N && lists[w2 * N + idx] > x) ? s : 0;
            }
        }
        int rank = 0;
#pragma unroll
        for (int w2 = 0; w2 < NW; ++w2) rank += q[w2];
        if (rank < k) emit(rank, x);
    }
}

template <int NT, typename Get, typename Emit>
__device__ __forceinline__ void sorted_topk(int m, int k, Get get, uint64_t* lists, Emit emit) {
    constexpr int NW = NT / 32;
    if (m <= NW * 32)
        sorted_topk_e<NT, 1>(m, k, get, lists, emit);
    else if (m <= NW * 64)
        sorted_topk_e<NT, 2>(m, k, get, lists, emit);
    else
        sorted_topk_e<NT, 4>(m, k, get, lists, emit);
}

// Lower bound of the k-th largest of the m composites get(0..m) (k <= NW*32,
// m <= NW*32*E): each lane keeps the largest of its E elements, and the k-th
// largest lane maximum is returned (k lanes hold an element at least that
// large, so the k-th largest element is at least that large). All NT threads
// call it and get the value.
template <int NT, int E, typename Get>
__device__ __forceinline__ uint64_t sorted_bound_e(int m, int k, Get get, uint64_t* lists, int* bcast) {
    constexpr int NW = NT / 32;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    uint64_t c[1];
    c[0] = 0ull;
#pragma unroll
    for (int r = 0; r < E; ++r) {
        const int i = warp * 32 * E + lane * E + r;
        const uint64_t v = i < m ? get(i) : 0ull;
        c[0] = v > c[0] ? v : c[0];
    }
    warp_sort_desc<1>(c);
    lists[warp * 32 + lane] = c[0];
    __syncthreads();
    const int len = k < 32 ? k : 32;
    for (int e = threadIdx.x; e < NW * len; e += NT) {
        const int w = e / len, p = e - w * len;
        const uint64_t x = lists[w * 32 + p];
        if (x == 0ull) continue;
        int q[NW];
#pragma unroll
        for (int w2 = 0; w2 < NW; ++w2) q[w2] = 0;
#pragma unroll
        for (int s = 32; s > 0; s >>= 1) {
#pragma unroll
            for (int w2 = 0; w2 < NW; ++w2) {
                const int idx = min(q[w2] + s - 1, 31);
                q[w2] += (q[w2] + s <= 32 && lists[w2 * 32 + idx] > x) ? s : 0;
            }
        }
        int rank = 0;
#pragma unroll
        for (int w2 = 0; w2 < NW; ++w2) rank += q[w2];
        if (rank == k - 1) {
            bcast[0] = (int)(uint32_t)(x >> 32);
        }
    }
    __syncthreads();
    return (uint64_t)(uint32_t)bcast[0] << 32;
}

// Exact four-pass radix select over all n scores read from global memory: the
// fallback when the candidates do not fit one sorted-list pass. Leaves the k
// winners, unordered, in rad.win_key / rad.win_id.
template <int NT>
__device__ void radix_select_global(const float* scores, int n, int k, SelectSmem& sm) {
    constexpr int NW = NT / 32;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    uint32_t prefix = 0, mask = 0;
    int remaining = k;
    for (int shift = 24; shift >= 0; shift -= 8) {
        for (int i = tid; i < 256; i += NT) sm.rad.hist[i] = 0u;
        __syncthreads();
        for (int i = tid; i < n; i += NT) {
            const uint32_t u = load_key(scores, i);
            if ((u & mask) == prefix) atomicAdd(&sm.rad.hist[(u >> shift) & 255u], 1u);
        }
        __syncthreads();
        if (warp == 0) {
            int c[8], lsum = 0;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                c[i] = (int)sm.rad.hist[255 - 8 * lane - i];
                lsum += c[i];
            }
            int incl = lsum;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int t = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += t;
            }
            const int excl = incl - lsum;
            if (excl < remaining && remaining <= incl) {
                int cum = excl;
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    if (cum + c[i] >= remaining) {
                        sm.bcast[0] = 255 - 8 * lane - i;
                        sm.bcast[1] = cum;
                        break;
                    }
                    cum += c[i];
                }
            }
        }
        __syncthreads();
        remaining -= sm.bcast[1];
        prefix |= (uint32_t)sm.bcast[0] << shift;
        mask |= 255u << shift;
        __syncthreads();
    }
    const uint32_t T = prefix;
    const int n_gt = k - remaining;
    if (tid == 0) sm.bcast[2] = 0;
    __syncthreads();
    for (int i = tid; i < n; i += NT) {
        const uint32_t u = load_key(scores, i);
        if (u > T) {
            const int slot = atomicAdd(&sm.bcast[2], 1);
            if (slot < kMaxTopk) {  // always true: fewer than k keys lie above T
                sm.rad.win_key[slot] = u;
                sm.rad.win_id[slot] = i;
            }
        }
    }
    int taken = 0;  // keys equal to T, lowest index first
    for (int base = 0; base < n && taken < remaining; base += NT) {
        const int i = base + tid;
        const bool f = (i < n) && load_key(scores, i) == T;
        const unsigned bal = __ballot_sync(0xffffffffu, f);
        const int lpre = __popc(bal & ((1u << lane) - 1u));
        if (lane == 0) sm.warp_tot[warp] = __popc(bal);
        __syncthreads();
        int woff = 0, tot = 0;
#pragma unroll
        for (int w = 0; w < NW; ++w) {
            const int c = sm.warp_tot[w];
            woff += (w < warp) ? c : 0;
            tot += c;
        }
        const int pos = taken + woff + lpre;
        if (f && pos < remaining && n_gt + pos < kMaxTopk) {
            sm.rad.win_key[n_gt + pos] = T;
            sm.rad.win_id[n_gt + pos] = i;
        }
        taken += tot;
        __syncthreads();
    }
    __syncthreads();
}

// Rank of every winner among the k winners by (key desc, id asc), one warp
// per winner (lanes compare 32 at once, a ballot counts those ahead); writes
// out[rank] = id.
template <int NT, typename Pick>
__device__ __forceinline__ void rank_winners(const uint32_t* keys, const int32_t* ids, int k,
                                             Pick pick) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    for (int e = warp; e < k; e += NT / 32) {
        const uint32_t ke = keys[e];
        const int ie = ids[e];
        int rank = 0;
        for (int base = 0; base < k; base += 32) {
            const int j = base + lane;
            bool ahead = false;
            if (j < k) {
                const uint32_t kj = keys[j];
                ahead = (kj > ke) || (kj == ke && ids[j] < ie);
            }
            rank += __popc(__ballot_sync(0xffffffffu, ahead));
        }
        if (lane == 0) pick(rank, ie);
    }
}

// All NT (<= 256) threads of the CTA call this. scores[0..n) are the row's
// scores and chunk_max[0..ceil(n/chunk)) the maximum key of every chunk of
// `chunk` consecutive blocks, both in global memory (L2). Calls pick(rank, id)
// once for every rank in [0, topk): the selected block ids in rank order,
// then -1. Requires topk <= kMaxTopk.
template <int NT, typename Pick>
__device__ void cta_topk_select(const float* scores, const uint32_t* chunk_max, int n, int chunk,
                                int topk, Pick pick, SelectSmem& sm) {
    static_assert(NT % 32 == 0 && NT <= 256, "up to 8 warps");
    constexpr int NW = NT / 32;
    constexpr int kPass = NW * 128;  // candidates one sorted-list pass holds
    const int tid = threadIdx.x;
    const int k = n < topk ? n : topk;
    for (int i = k + tid; i < topk; i += NT) pick(i, -1);
    if (k <= 0) return;
    auto emit_id = [&](int rank, uint64_t x) { pick(rank, composite_id(x)); };
    if (k <= kSortMaxK && n <= kPass) {
        sorted_topk<NT>(n, k, [&](int i) { return compose(load_key(scores, i), i); }, sm.lists,
                        emit_id);
        return;
    }
    const int nch = (n + chunk - 1) / chunk;
    if (k <= kSortMaxK && k <= nch && nch <= kMaxChunks && nch <= kPass) {
        // 1. the k-th largest chunk maximum, or a lower bound of it, bounds the
        //    k-th largest score from below
        if (tid == 0) sm.bcast[6] = 0;
        auto getc = [&](int c) { return compose(__ldcg(chunk_max + c), c); };
        uint32_t kth;
        if (nch > NW * 64 && k <= 32) {
            // many chunks, small k: the bound from the lanes' maxima of 4 chunk
            // maxima costs one 32-element sort per warp instead of a 128-element one
            kth = composite_key(sorted_bound_e<NT, 4>(nch, k, getc, sm.lists, sm.bcast + 5));
        } else {
            sorted_topk<NT>(nch, k, getc, sm.lists, [&](int rank, uint64_t x) {
                if (rank == k - 1) sm.bcast[5] = (int)composite_key(x);
            });
            __syncthreads();
            kth = (uint32_t)sm.bcast[5];
        }
        // surviving chunks: maximum >= kth (at least the k chunks ranked above)
        for (int c = tid; c < nch; c += NT) {
            if (__ldcg(chunk_max + c) >= kth) sm.surv[atomicAdd(&sm.bcast[6], 1)] = c;
        }
        __syncthreads();
        const int nsurv = sm.bcast[6];
        if ((long long)nsurv * chunk <= kPass) {
            // every surviving chunk takes `chunk` slots; slots past the end of
            // the row are padding
            sorted_topk<NT>(
                nsurv * chunk, k,
                [&](int i) {
                    const int t = i / chunk, e = i - t * chunk;
                    const int j = sm.surv[t] * chunk + e;
                    return j < n ? compose(load_key(scores, j), j) : 0ull;
                },
                sm.lists, emit_id);
            return;
        }
        __syncthreads();  // the radix pass reuses the list memory
    }
    radix_select_global<NT>(scores, n, k, sm);
    rank_winners<NT>(sm.rad.win_key, sm.rad.win_id, k, pick);
}

// The common case: write the ids to out[0..topk).
template <int NT>
__device__ __forceinline__ void cta_topk_select(const float* scores, const uint32_t* chunk_max,
                                                int n, int chunk, int topk, int32_t* out,
                                                SelectSmem& sm) {
    cta_topk_select<NT>(scores, chunk_max, n, chunk, topk, [=](int rank, int id) { out[rank] = id; },
                        sm);
}

}  // namespace lci
