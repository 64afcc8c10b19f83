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
