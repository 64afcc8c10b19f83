// compress.cuh -- A0, block compression of per-token indexer keys into one key
// per KV block: k_c[b][j][:] = mean of k_idx[b][t][:] over the tokens t of
// block j ([GPU-stack] "Adapting Sparse Attention", representation stage).
#pragma once

#include "common.cuh"

namespace lci {

// One thread per output element; consecutive threads take consecutive
// feature indices, so every token row is read coalesced.
template <typename T>
__global__ void block_compress_kernel(const T* __restrict__ k_idx, int B, int tokens, int HD,
                                      int bs, int NB, T* __restrict__ k_c) {
    const long long total = (long long)B * NB * HD;
    for (long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x; idx < total;
         idx += (long long)gridDim.x * blockDim.x) {
        const int e = (int)(idx % HD);
        const long long bj = idx / HD;
        const int j = (int)(bj % NB);
        const long long b = bj / NB;
        const int t0 = j * bs;
        const int t1 = min(tokens, t0 + bs);
        float sum = 0.f;
        for (int t = t0; t < t1; ++t) sum += to_f32(k_idx[(b * tokens + t) * HD + e]);
        k_c[idx] = from_f32<T>(sum / (float)(t1 - t0));
    }
}

}  // namespace lci

namespace lci {

__device__ __forceinline__ float from_f64_to(double x, float) { return (float)x; }
__device__ __forceinline__ __nv_bfloat16 from_f64_to(double x, __nv_bfloat16) {
    return __double2bfloat16(x);
}

// Online form of the block compression over a paged pool. T new tokens of
// sequence b, at positions start[b] .. start[b]+T-1, enter the cache; every
// block they touch gets its running fp32 sum (kc_sum[page]) extended by them
// and its key rewritten as kc[page] = sum / (tokens now in the block), with
// page = table[b][block]. A block that already held tokens before this call
// (a partly filled last block) continues from its stored sum; a block the
// call starts restarts it. One thread per (sequence, touched block, feature);
// the quotient is formed in fp64 and rounded once to the key's type.
template <typename T>
__global__ void kc_update_kernel(const T* __restrict__ k_idx, int B, int T_new, int HD, int bs,
                                 const int32_t* __restrict__ start, const int32_t* __restrict__ table,
                                 int nb_max, int num_pages, int slots, float* __restrict__ kc_sum,
                                 T* __restrict__ kc) {
    const long long total = (long long)B * slots * HD;
    for (long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x; idx < total;
         idx += (long long)gridDim.x * blockDim.x) {
        const int e = (int)(idx % HD);
        const long long bs_idx = idx / HD;
        const int slot = (int)(bs_idx % slots);
        const int b = (int)(bs_idx / slots);
        const long long p0 = start[b];
        if (p0 < 0) {
            if (slot == 0 && e == 0) raise_status(kStatusBadBlockId);
            continue;
        }
        const long long p1 = p0 + T_new;  // one past the last new token
        const long long j = p0 / bs + slot;
        if (j * bs >= p1) continue;       // this sequence touches fewer blocks
        if (j >= nb_max) {
            if (e == 0) raise_status(kStatusBadBlockId);
            continue;
        }
        const int page = table[(size_t)b * nb_max + j];
        if (page < 0 || page >= num_pages) {
            if (e == 0) raise_status(kStatusBadPage);
            continue;
        }
        const long long t_lo = p0 > j * bs ? p0 : j * bs;
        const long long t_hi = p1 < (j + 1) * bs ? p1 : (j + 1) * bs;
        float* sum_p = kc_sum + (size_t)page * HD + e;
        float sum = t_lo > j * bs ? *sum_p : 0.f;
        for (long long t = t_lo; t < t_hi; ++t)
            sum += to_f32(k_idx[((size_t)b * T_new + (size_t)(t - p0)) * HD + e]);
        *sum_p = sum;
        kc[(size_t)page * HD + e] = from_f64_to((double)sum / (double)(t_hi - j * bs), T());
    }
}

// Gather of paged block keys into the dense [B][nb_max][HD] layout of the
// indexer (one 16-byte vector per thread). Only blocks holding cached tokens
// (j * bs < ctx_len[b]) are read through the table; the other rows are zero
// and are never visible to a query.
__global__ void kc_gather_kernel(const uint4* __restrict__ kc, const int32_t* __restrict__ table,
                                 const int32_t* __restrict__ ctx_len, int B, int nb_max, int bs,
                                 int num_pages, int vec_per_row, uint4* __restrict__ dense) {
    const long long total = (long long)B * nb_max * vec_per_row;
    for (long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x; idx < total;
         idx += (long long)gridDim.x * blockDim.x) {
        const long long bj = idx / vec_per_row;
        const int v = (int)(idx - bj * vec_per_row);
        const int b = (int)(bj / nb_max), j = (int)(bj - (long long)b * nb_max);
        uint4 x = make_uint4(0, 0, 0, 0);
        if ((long long)j * bs < ctx_len[b]) {
            const int page = table[bj];
            if (page >= 0 && page < num_pages)
                x = kc[(size_t)page * vec_per_row + v];
            else if (v == 0)
                raise_status(kStatusBadPage);
        }
        dense[idx] = x;
    }
}

}  // namespace lci
