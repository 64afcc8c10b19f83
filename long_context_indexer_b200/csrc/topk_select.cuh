// topk_select.cuh -- exact CTA-wide top-k of block scores without a full sort.
//
// [GPU-stack] "Operatorizing Index Selection" and [AI-acc] §4.1 ask for a top-k
// that avoids sorting every candidate. This one is a most-significant-digit
// radix select over order-preserving uint32 keys: four 8-bit histogram passes
// find the k-th largest key T, the keys above T are taken as they come, the
// keys equal to T are taken lowest block id first (an ordered compaction), and
// only the k survivors are ranked (key desc, id asc).
#pragma once

#include "common.cuh"

namespace lci {

constexpr int kMaxTopk = 256;

struct SelectSmem {
    unsigned int hist[256];
    uint32_t cand_key[kMaxTopk];
    int32_t cand_id[kMaxTopk];
    int warp_cnt[32];
    int bcast[4];
};

// All NT threads of the CTA call this. keys[0..n) lives in shared memory and
// is not modified. Writes out[0..topk): the selected indices in rank order,
// then -1. Requires topk <= kMaxTopk.
template <int NT>
__device__ void cta_topk_from_keys(const uint32_t* keys, int n, int topk, int32_t* out,
                                   SelectSmem& sm) {
    constexpr int NW = NT / 32;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int k = n < topk ? n : topk;
    int ncand;
    if (n <= k) {
        // Every visible block is selected; only the ranking remains.
        for (int i = tid; i < n; i += NT) {
            sm.cand_key[i] = keys[i];
            sm.cand_id[i] = i;
        }
        ncand = n;
    } else {
        uint32_t prefix = 0, mask = 0;
        int remaining = k;  // how many of the keys matching `prefix` are still to take
        for (int shift = 24; shift >= 0; shift -= 8) {
            for (int i = tid; i < 256; i += NT) sm.hist[i] = 0u;
            __syncthreads();
            for (int i = tid; i < n; i += NT) {
                const uint32_t u = keys[i];
                if ((u & mask) == prefix) atomicAdd(&sm.hist[(u >> shift) & 255u], 1u);
            }
            __syncthreads();
            if (warp == 0) {
                // Lane l owns digits 255-8l .. 248-8l (descending). A warp
                // scan gives how many keys lie above each lane's digits.
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
            const uint32_t d = (uint32_t)sm.bcast[0];
            remaining -= sm.bcast[1];
            prefix |= d << shift;
            mask |= 255u << shift;
            __syncthreads();
        }
        const uint32_t T = prefix;       // the k-th largest key
        const int n_gt = k - remaining;  // keys strictly above T
        if (tid == 0) sm.bcast[2] = 0;
        __syncthreads();
        for (int i = tid; i < n; i += NT) {
            const uint32_t u = keys[i];
            if (u > T) {
                const int slot = atomicAdd(&sm.bcast[2], 1);
                if (slot < kMaxTopk) {  // always true: fewer than k keys lie above T
                    sm.cand_key[slot] = u;
                    sm.cand_id[slot] = i;
                }
            }
        }
        // Keys equal to T, lowest index first, until `remaining` are taken.
        int taken = 0;
        for (int base = 0; base < n && taken < remaining; base += NT) {
            const int i = base + tid;
            const bool f = (i < n) && keys[i] == T;
            const unsigned bal = __ballot_sync(0xffffffffu, f);
            const int lpre = __popc(bal & ((1u << lane) - 1u));
            if (lane == 0) sm.warp_cnt[warp] = __popc(bal);
            __syncthreads();
            int woff = 0, tot = 0;
#pragma unroll
            for (int w = 0; w < NW; ++w) {
                const int c = sm.warp_cnt[w];
                woff += (w < warp) ? c : 0;
                tot += c;
            }
            const int pos = taken + woff + lpre;
            if (f && pos < remaining && n_gt + pos < kMaxTopk) {
                sm.cand_key[n_gt + pos] = T;
                sm.cand_id[n_gt + pos] = i;
            }
            taken += tot;
            __syncthreads();
        }
        ncand = k;
    }
    __syncthreads();
    for (int e = tid; e < ncand; e += NT) {
        const uint32_t ke = sm.cand_key[e];
        const int ie = sm.cand_id[e];
        int rank = 0;
        for (int f = 0; f < ncand; ++f) {
            const uint32_t kf = sm.cand_key[f];
            rank += (kf > ke) || (kf == ke && sm.cand_id[f] < ie);
        }
        out[rank] = ie;
    }
    for (int i = ncand + tid; i < topk; i += NT) out[i] = -1;
}

}  // namespace lci
