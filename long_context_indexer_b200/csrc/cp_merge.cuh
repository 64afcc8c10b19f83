// cp_merge.cuh -- the exchange steps of context parallelism: a long context
// split into block ranges over several GPUs ([AI-acc] §3, communication
// libraries for multi-card inference; [Hetero] §VII, communication overlap).
//
// Every rank selects the top-k of its own visible blocks; the global top-k of
// a query is contained in the union of the ranks' lists (a block outside its
// rank's top-k has k better blocks on that rank alone), so merging the lists
// by (score desc, block id asc) is exact. Every rank then attends over the
// selected blocks it holds and emits a partial: its normalised output and the
// log2-sum-exp2 of its scaled logits; the partials combine exactly as
//   out = sum_r 2^(lse_r - M) o_r / sum_r 2^(lse_r - M),  M = max_r lse_r.
#pragma once

#include "common.cuh"

namespace lci {

// scores[row][i] = q_c[row] . k_c[b][ids[row][i]] (fp32), -inf for id -1.
// One warp per (row, i); lanes stride the H_i*d_c features in 16-byte vectors.
template <typename T>
__global__ void block_scores_at_kernel(const T* __restrict__ q_c, const T* __restrict__ k_c, int S,
                                       int K, int nb_max, const int32_t* __restrict__ ids,
                                       int topk, long long pairs, float* __restrict__ scores) {
    constexpr int E = 16 / sizeof(T);
    const int lane = threadIdx.x & 31;
    const long long warps = (long long)gridDim.x * (blockDim.x >> 5);
    for (long long w = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); w < pairs;
         w += warps) {
        const long long row = w / topk;
        const int b = (int)(row / S);
        const int j = ids[w];
        float acc = 0.f;
        if (j >= 0 && j < nb_max) {
            const uint4* qr = reinterpret_cast<const uint4*>(q_c + (size_t)row * K);
            const uint4* kr = reinterpret_cast<const uint4*>(k_c + ((size_t)b * nb_max + j) * K);
            for (int c = lane; c < K / E; c += 32) {
                const uint4 a = qr[c], k = kr[c];
                const T* ae = reinterpret_cast<const T*>(&a);
                const T* ke = reinterpret_cast<const T*>(&k);
#pragma unroll
                for (int e = 0; e < E; ++e) acc += to_f32(ae[e]) * to_f32(ke[e]);
            }
        } else if (j != -1 && lane == 0) {
            raise_status(kStatusBadBlockId);
        }
        acc = warp_sum(acc);
        if (lane == 0) scores[w] = (j >= 0 && j < nb_max) ? acc : -INFINITY;
    }
}

// out = (lo <= id < hi) ? id + offset : -1, elementwise.
__global__ void ids_shift_kernel(const int32_t* __restrict__ ids, long long n, int lo, int hi,
                                 int offset, int32_t* __restrict__ out) {
    for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n;
         i += (long long)gridDim.x * blockDim.x) {
        const int j = ids[i];
        out[i] = (j >= lo && j < hi) ? j + offset : -1;
    }
}

constexpr int kMaxLists = 64;

// Per row: the top-k of `nlists` ranked lists (score desc, id asc; -1 marks
// the end of a list), ranked the same way. One thread per row.
__global__ void topk_merge_kernel(const float* __restrict__ scores, const int32_t* __restrict__ ids,
                                  int nlists, long long rows, int topk,
                                  int32_t* __restrict__ out) {
    const long long row = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (row >= rows) return;
    int head[kMaxLists];
    for (int r = 0; r < nlists; ++r) head[r] = 0;
    for (int i = 0; i < topk; ++i) {
        int best = -1;
        uint32_t bk = 0u;
        int32_t bi = 0;
        for (int r = 0; r < nlists; ++r) {
            if (head[r] >= topk) continue;
            const size_t at = ((size_t)r * rows + row) * topk + head[r];
            const int32_t id = ids[at];
            if (id < 0) continue;
            const uint32_t key = score_key(scores[at]);
            if (best < 0 || key > bk || (key == bk && id < bi)) {
                best = r;
                bk = key;
                bi = id;
            }
        }
        out[(size_t)row * topk + i] = best < 0 ? -1 : bi;
        if (best >= 0) ++head[best];
    }
}

// out[row][h][:] = combination of the partial outputs o[r][row][h][:] by
// their log2-sum-exp2 weights; zero when no partial holds a token.
template <typename T>
__global__ void attn_merge_kernel(const T* __restrict__ o, const float* __restrict__ lse,
                                  int nlists, long long rows_heads, int hd, T* __restrict__ out) {
    const long long total = rows_heads * hd;
    for (long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x; idx < total;
         idx += (long long)gridDim.x * blockDim.x) {
        const long long rh = idx / hd;
        float M = -INFINITY;
        for (int r = 0; r < nlists; ++r) M = fmaxf(M, lse[(size_t)r * rows_heads + rh]);
        float num = 0.f, den = 0.f;
        if (M > -INFINITY) {
            for (int r = 0; r < nlists; ++r) {
                const float lr = lse[(size_t)r * rows_heads + rh];
                if (lr == -INFINITY) continue;
                const float w = exp2f(lr - M);
                num += w * to_f32(o[(size_t)r * total + idx]);
                den += w;
            }
        }
        out[idx] = from_f32<T>(den > 0.f ? num / den : 0.f);
    }
}

}  // namespace lci
