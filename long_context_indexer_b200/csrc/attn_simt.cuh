// attn_simt.cuh -- generic sparse attention on CUDA cores (fp32 math).
//
// One CTA per (query row, KV head); one warp per query head of the group. The
// warp walks the row's selected blocks through the block table, and for every
// causal-valid token computes the logit (lanes split head_dim, shuffle
// reduction) and folds it into an online softmax (running max, running sum,
// rescaled accumulator), all in fp32 with exp2. Serves fp32 inputs and any
// shape the tensor-core kernels do not cover.
#pragma once

#include "common.cuh"

namespace lci {

constexpr int kSimtMaxHdPerLane = 8;  // head_dim <= 256

template <typename T>
__global__ void __launch_bounds__(512) sparse_attn_simt_kernel(
    const T* __restrict__ q, const T* __restrict__ k_pool, const T* __restrict__ v_pool,
    const int32_t* __restrict__ table, int nb_max, int num_pages, int H_kv, int bs, int hd,
    int S, int H_q, const int32_t* __restrict__ ids, int topk,
    const int32_t* __restrict__ ctx_len, const int32_t* __restrict__ q_start, float scale_log2,
    T* __restrict__ out) {
    const int row = blockIdx.x, g = blockIdx.y;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
    const int G = H_q / H_kv;
    const int b = row / S, s = row - b * S;
    const long long p = (long long)q_start[b] + s;
    const long long ctx = ctx_len[b];
    const long long last = p < ctx - 1 ? p : ctx - 1;
    const int per_lane = hd >> 5;
    const int32_t* row_ids = ids + (size_t)row * topk;

    for (int hl = warp; hl < G; hl += nwarps) {
        const int h = g * G + hl;
        const T* qh = q + ((size_t)row * H_q + h) * hd;
        float qv[kSimtMaxHdPerLane], o[kSimtMaxHdPerLane];
#pragma unroll
        for (int e = 0; e < kSimtMaxHdPerLane; ++e) {
            qv[e] = e < per_lane ? to_f32(qh[lane + 32 * e]) * scale_log2 : 0.f;
            o[e] = 0.f;
        }
        float m = -INFINITY, l = 0.f;
        for (int i = 0; i < topk; ++i) {
            const int j = row_ids[i];
            if (j == -1) continue;
            if (j < -1 || j >= nb_max) {
                if (lane == 0) raise_status(kStatusBadBlockId);
                continue;
            }
            const int page = table[(size_t)b * nb_max + j];
            if (page < 0 || page >= num_pages) {
                if (lane == 0) raise_status(kStatusBadPage);
                continue;
            }
            const long long first = (long long)j * bs;
            if (first > last) continue;
            const int ntok = (int)min((long long)bs, last - first + 1);
            const size_t base = ((size_t)page * H_kv + g) * bs * hd;
            for (int u = 0; u < ntok; ++u) {
                const T* kr = k_pool + base + (size_t)u * hd;
                const T* vr = v_pool + base + (size_t)u * hd;
                float dot = 0.f;
#pragma unroll
                for (int e = 0; e < kSimtMaxHdPerLane; ++e)
                    if (e < per_lane) dot += qv[e] * to_f32(kr[lane + 32 * e]);
                dot = warp_sum(dot);
                const float m_new = fmaxf(m, dot);
                const float corr = exp2f(m - m_new);
                const float pw = exp2f(dot - m_new);
                l = l * corr + pw;
#pragma unroll
                for (int e = 0; e < kSimtMaxHdPerLane; ++e)
                    if (e < per_lane) o[e] = o[e] * corr + pw * to_f32(vr[lane + 32 * e]);
                m = m_new;
            }
        }
        const float inv = l > 0.f ? 1.f / l : 0.f;
        T* oh = out + ((size_t)row * H_q + h) * hd;
#pragma unroll
        for (int e = 0; e < kSimtMaxHdPerLane; ++e)
            if (e < per_lane) oh[lane + 32 * e] = from_f32<T>(o[e] * inv);
    }
}

}  // namespace lci
