// topk_select.cuh -- exact CTA-wide top-k of block scores without a full sort.
//
// [GPU-stack] "Operatorizing Index Selection" and [AI-acc] §4.1 ask for a top-k
// that prunes candidates coarsely and then selects exactly, instead of sorting
// every score. Scores become order-preserving uint32 keys (larger score, larger
// key; -0.0 folded onto +0.0). A row's blocks are scored in chunks, and every
// chunk also reports its maximum key.
//
//  1. Chunk pruning (when the row has more chunks than k). The k-th largest
//     chunk maximum M is a lower bound of the k-th largest score: the k chunks
//     whose maxima are >= M hold k distinct scores >= M. So a chunk whose
//     maximum is below M holds no winner, and only the chunks with maximum
//     >= M are gathered. Lossless.
//  2. Exact selection among the gathered candidates: one histogram pass over
//     the top 11 key bits (2048 bins) finds the bin holding the k-th largest
//     key; keys in higher bins are in; keys of that boundary bin are ranked
//     exactly (key desc, block id asc) among themselves.
//  3. The k winners are ranked and written in order, padded with -1.
// Ranks are computed a warp per element: 32 lanes compare at once and a
// ballot counts the elements ranked ahead.
// If the candidates overflow the shared buffers (long rows of equal scores), a
// four-pass radix select over all scores, read from global memory, takes over.
#pragma once

#include "common.cuh"

namespace lci {

constexpr int kMaxTopk = 256;
constexpr int kSelBins = 2048;      // top 11 bits of the key
constexpr int kSelShift = 21;
constexpr int kCandCap = 1024;         // candidates held in shared memory
constexpr int kMaxBoundary = kCandCap;  // boundary-bin keys resolved by rank (all may tie)

struct SelectSmem {
    unsigned int hist[kSelBins];
    uint32_t cand_key[kCandCap];
    int32_t cand_id[kCandCap];
    uint32_t bnd_key[kMaxBoundary];
    int32_t bnd_id[kMaxBoundary];
    uint32_t win_key[kMaxTopk];
    int32_t win_id[kMaxTopk];
    int warp_tot[32];
    int bcast[8];
};

__device__ __forceinline__ uint32_t load_key(const float* scores, int i) {
    return score_key(__ldcg(scores + i));
}

// Block-wide inclusive scan of one int per thread (NT threads).
template <int NT>
__device__ __forceinline__ int block_incl_scan(int v, int* warp_tot) {
    constexpr int NW = NT / 32;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int t = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += t;
    }
    if (lane == 31) warp_tot[warp] = v;
    __syncthreads();
    int off = 0;
#pragma unroll
    for (int w = 0; w < NW; ++w) off += (w < warp) ? warp_tot[w] : 0;
    __syncthreads();
    return v + off;
}

// Rank of every element e of keys/ids[0..m) among the same m elements, by
// (key desc, id asc): one warp per element, lanes compare 32 elements at once
// and a ballot counts the ones ranked ahead. Calls f(e, rank) from lane 0.
template <int NT, typename F>
__device__ __forceinline__ void warp_ranks(const uint32_t* keys, const int32_t* ids, int m, F f) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    for (int e = warp; e < m; e += NT / 32) {
        const uint32_t ke = keys[e];
        const int ie = ids[e];
        int rank = 0;
        for (int base = 0; base < m; base += 32) {
            const int j = base + lane;
            bool ahead = false;
            if (j < m) {
                const uint32_t kj = keys[j];
                ahead = (kj > ke) || (kj == ke && ids[j] < ie);
            }
            rank += __popc(__ballot_sync(0xffffffffu, ahead));
        }
        if (lane == 0) f(e, rank);
    }
}

// Top k of the m candidates cand_key/cand_id[0..m) (k <= m, k <= kMaxTopk,
// m <= kCandCap). Leaves the k winners, unordered, in win_key/win_id.
template <int NT>
__device__ void select_candidates(int m, int k, SelectSmem& sm) {
    const int tid = threadIdx.x;
    for (int i = tid; i < kSelBins; i += NT) sm.hist[i] = 0u;
    if (tid < 8) sm.bcast[tid] = 0;
    __syncthreads();
    for (int i = tid; i < m; i += NT) atomicAdd(&sm.hist[sm.cand_key[i] >> kSelShift], 1u);
    __syncthreads();
    // thread t owns bins 2047-8t .. 2040-8t (descending)
    int c[8], lsum = 0;
#pragma unroll
    for (int q = 0; q < 8; ++q) {
        c[q] = (int)sm.hist[kSelBins - 1 - 8 * tid - q];
        lsum += c[q];
    }
    const int incl = block_incl_scan<NT>(lsum, sm.warp_tot);
    const int excl = incl - lsum;
    if (excl < k && k <= incl) {
        int cum = excl;
#pragma unroll
        for (int q = 0; q < 8; ++q) {
            if (cum + c[q] >= k) {
                sm.bcast[0] = kSelBins - 1 - 8 * tid - q;  // boundary bin
                sm.bcast[1] = cum;                        // keys above it
                break;
            }
            cum += c[q];
        }
    }
    __syncthreads();
    const uint32_t dstar = (uint32_t)sm.bcast[0];
    const int above = sm.bcast[1];
    const int need = k - above;
    for (int i = tid; i < m; i += NT) {
        const uint32_t u = sm.cand_key[i];
        const uint32_t bin = u >> kSelShift;
        if (bin > dstar) {
            const int slot = atomicAdd(&sm.bcast[3], 1);
            if (slot < kMaxTopk) {  // always true: `above` < k keys
                sm.win_key[slot] = u;
                sm.win_id[slot] = sm.cand_id[i];
            }
        } else if (bin == dstar) {
            const int slot = atomicAdd(&sm.bcast[4], 1);
            if (slot < kMaxBoundary) {
                sm.bnd_key[slot] = u;
                sm.bnd_id[slot] = sm.cand_id[i];
            }
        }
    }
    __syncthreads();
    const int nb = min(sm.bcast[4], kMaxBoundary);  // never clipped: nb <= m <= kCandCap
    warp_ranks<NT>(sm.bnd_key, sm.bnd_id, nb, [&](int e, int rank) {
        if (rank < need && above + rank < kMaxTopk) {
            sm.win_key[above + rank] = sm.bnd_key[e];
            sm.win_id[above + rank] = sm.bnd_id[e];
        }
    });
    __syncthreads();
}

// Exact four-pass radix select over all n scores read from global memory: the
// fallback when the candidates do not fit. Leaves the k winners in win_*.
template <int NT>
__device__ void radix_select_global(const float* scores, int n, int k, SelectSmem& sm) {
    constexpr int NW = NT / 32;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    uint32_t prefix = 0, mask = 0;
    int remaining = k;
    for (int shift = 24; shift >= 0; shift -= 8) {
        for (int i = tid; i < 256; i += NT) sm.hist[i] = 0u;
        __syncthreads();
        for (int i = tid; i < n; i += NT) {
            const uint32_t u = load_key(scores, i);
            if ((u & mask) == prefix) atomicAdd(&sm.hist[(u >> shift) & 255u], 1u);
        }
        __syncthreads();
        if (warp == 0) {
            int c[8], lsum = 0;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                c[i] = (int)sm.hist[255 - 8 * lane - i];
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
                sm.win_key[slot] = u;
                sm.win_id[slot] = i;
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
            sm.win_key[n_gt + pos] = T;
            sm.win_id[n_gt + pos] = i;
        }
        taken += tot;
        __syncthreads();
    }
    __syncthreads();
}

// All NT threads of the CTA call this. scores[0..n) are the row's scores and
// chunk_max[0..ceil(n/chunk)) the maximum key of every chunk of `chunk`
// consecutive blocks, both in global memory (L2). Writes out[0..topk): the
// selected block ids in rank order, then -1. Requires topk <= kMaxTopk.
template <int NT>
__device__ void cta_topk_select(const float* scores, const uint32_t* chunk_max, int n, int chunk,
                                int topk, int32_t* out, SelectSmem& sm) {
    static_assert(NT == 256, "one thread per 8 histogram bins");
    const int tid = threadIdx.x;
    const int k = n < topk ? n : topk;
    const int nch = (n + chunk - 1) / chunk;
    int m = -1;  // candidates gathered; -1: fall back to the global radix select
    if (n <= kCandCap) {
#pragma unroll 8
        for (int i = tid; i < n; i += NT) {
            sm.cand_key[i] = load_key(scores, i);
            sm.cand_id[i] = i;
        }
        m = n;
    } else if (k > 0 && nch <= kCandCap && k <= nch) {
        // 1. the k-th largest chunk maximum bounds the k-th largest score
#pragma unroll 8
        for (int c = tid; c < nch; c += NT) {
            sm.cand_key[c] = __ldcg(chunk_max + c);
            sm.cand_id[c] = c;
        }
        __syncthreads();
        select_candidates<NT>(nch, k, sm);
        uint32_t kth = 0xffffffffu;
        for (int e = 0; e < k; ++e) kth = min(kth, sm.win_key[e]);
        if (tid == 0) sm.bcast[7] = 0;
        __syncthreads();
        // surviving chunks: maximum >= kth (at least the k winners)
        for (int c = tid; c < nch; c += NT) {
            if (sm.cand_key[c] >= kth) {
                const int t = atomicAdd(&sm.bcast[7], 1);
                if (t < kMaxBoundary) sm.bnd_id[t] = c;
            }
        }
        __syncthreads();
        const int nsurv = sm.bcast[7];
        if (nsurv <= kMaxBoundary && (long long)nsurv * chunk <= kCandCap) {
            // every surviving chunk takes `chunk` slots; slots past the end of
            // the row hold key 0, below every real key, so they never win
            m = nsurv * chunk;
#pragma unroll 8
            for (int idx = tid; idx < m; idx += NT) {
                const int t = idx / chunk, e = idx - t * chunk;
                const int j = sm.bnd_id[t] * chunk + e;
                sm.cand_key[idx] = j < n ? load_key(scores, j) : 0u;
                sm.cand_id[idx] = j < n ? j : -1;
            }
        }
    }
    __syncthreads();
    if (m >= 0)
        select_candidates<NT>(m, k, sm);
    else
        radix_select_global<NT>(scores, n, k, sm);
    // 3. rank the k winners (key desc, id asc) and write them in order
    warp_ranks<NT>(sm.win_key, sm.win_id, k, [&](int e, int rank) { out[rank] = sm.win_id[e]; });
    for (int i = k + tid; i < topk; i += NT) out[i] = -1;
}

}  // namespace lci
