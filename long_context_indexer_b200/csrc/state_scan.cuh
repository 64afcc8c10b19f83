// state_scan.cuh -- chunked gated state scan of the linear-attention family
// on the 5th-generation tensor cores ([Hetero] §II and §III: a gated
// incremental state update scanned over the sequence in chunks, a state
// tensor carried from chunk to chunk and read out by the queries):
//
//   for each chunk c of C = 128 tokens:   S   = gate[c] * S + K_c^T V_c
//                                          out = Q_c S          (rows of chunk c)
//
// One CTA per (sequence, head), dk = dv = 128. The state is kept transposed
// in TMEM, S^T [dv lanes x dk columns] fp32, so that both products are
// 128 x 128 x 128 tcgen05 MMAs with the state as the accumulator or as A:
//   update   S^T  += V_c^T K_c   A = V_c (MN-major), B = K_c (MN-major), D = S^T
//   readout  O^T   = S^T Q_c^T   A = S^T from TMEM as bf16 (hi and lo halves,
//                                 S = hi + lo to about 2^-17), B = Q_c (K-major)
// The gate is applied by the state warps (two threads per TMEM lane = dv row,
// 64 dk columns each) when they split S^T for the readout, so it never waits
// on memory. The output goes through two TMEM buffers: output warps write
// chunk c while the state warps split the state of chunk c+1.
// Q, K and V chunks stream in by TMA (4-D tensor maps over [B][T][H][128],
// zero fill past T) through a two-stage ring; the output is written in fp32.
#pragma once

#include "attn_prefill.cuh"
#include "common.cuh"
#include "index_prefill.cuh"
#include "ptx.cuh"

namespace lci {

namespace gss {
constexpr int kC = 128;              // tokens per chunk
constexpr int kD = 128;              // dk = dv
constexpr int kHalf = 128 * 128;     // 128 rows x 64 columns of bf16: 16 KiB
constexpr int kTile = 2 * kHalf;     // 128 x 128 bf16: 32 KiB
constexpr int kStages = 2;
constexpr int kStageBytes = 3 * kTile;  // Q, K, V
// warps: 0 TMA, 1 MMA, 2..9 state (two per TMEM lane quarter, 64 dk columns
// each), 10..13 output (one per lane quarter)
constexpr int kStateWarps = 8, kOutWarps = 4;
constexpr int kThreads = 64 + 32 * (kStateWarps + kOutWarps);
// TMEM columns: S^T fp32, its bf16 hi and lo halves, two output buffers
constexpr int kColS = 0, kColHi = 128, kColLo = 192, kColO = 256, kTmemCols = 512;
constexpr int kOffBar = kStages * kStageBytes;
constexpr int kSmemBytes = kOffBar + 256 + 1024;
// D fp32, A and B bf16, M = N = 128; the update reads both operands MN-major
constexpr uint32_t kIdescRead = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(128 >> 3) << 17) |
                                ((uint32_t)(128 >> 4) << 24);
constexpr uint32_t kIdescUpd = kIdescRead | (1u << 15) | (1u << 16);
}  // namespace gss

// 4-D tiled TMA load: coordinates (x innermost .. w outermost).
__device__ __forceinline__ void tma_load_4d(void* dst, const CUtensorMap* map, int x, int y, int z,
                                            int w, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3, %4, %5}], [%6];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(w), "r"(smem_u32(bar))
        : "memory");
}

__global__ void __launch_bounds__(gss::kThreads, 1) gated_state_scan_kernel(
    const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
    const __grid_constant__ CUtensorMap tm_v, const float* __restrict__ gate,
    const float* __restrict__ state_in, float* __restrict__ state_out, int T, int H, int nchunks,
    float* __restrict__ out) {
    using namespace gss;
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char* smem = reinterpret_cast<unsigned char*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + kOffBar);  // [kStages]
    uint64_t* empty = full + kStages;                                // [kStages]
    uint64_t* s0ready = empty + kStages;   // initial state in TMEM (state warps)
    uint64_t* upd_done = s0ready + 1;      // update MMAs of a chunk completed
    uint64_t* cdone = upd_done + 1;        // hi/lo written and S^T gated (state warps)
    uint64_t* out_ready = cdone + 1;       // [2] readout MMAs into output buffer b completed
    uint64_t* ofree = out_ready + 2;       // [2] output buffer b read out (output warps)
    uint64_t* drain = ofree + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
    volatile int* s_abort = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int bh = blockIdx.x;
    const int b = bh / H, h = bh - b * H;
    const float* g_row = gate + (size_t)bh * nchunks;

    if (tid == 0) {
        for (int i = 0; i < kStages; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], 1);
        }
        mbar_init(s0ready, kStateWarps);
        mbar_init(upd_done, 1);
        mbar_init(cdone, kStateWarps);
        for (int i = 0; i < 2; ++i) {
            mbar_init(&out_ready[i], 1);
            mbar_init(&ofree[i], kOutWarps);
        }
        mbar_init(drain, 1);
        *s_abort = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32(tmem_slot)),
                     "r"(kTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    if (warp == 0 && lane == 0) {
        prefetch_tensormap(&tm_q);
        prefetch_tensormap(&tm_k);
        prefetch_tensormap(&tm_v);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    if (warp == 0) {
        // ---------------- TMA producer ----------------
        if (lane == 0) {
            for (int c = 0; c < nchunks; ++c) {
                const int st = c % kStages;
                if (*s_abort) break;
                if (c >= kStages && !mbar_wait(&empty[st], ((c / kStages) - 1) & 1)) {
                    *s_abort = 1;
                    break;
                }
                unsigned char* base = smem + st * kStageBytes;
                mbar_arrive_expect_tx(&full[st], kStageBytes);
                const int t0 = c * kC;
                for (int half = 0; half < 2; ++half) {
                    tma_load_4d(base + half * kHalf, &tm_q, half * 64, h, t0, b, &full[st]);
                    tma_load_4d(base + kTile + half * kHalf, &tm_k, half * 64, h, t0, b, &full[st]);
                    tma_load_4d(base + 2 * kTile + half * kHalf, &tm_v, half * 64, h, t0, b,
                                &full[st]);
                }
            }
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer ----------------
        if (lane == 0) {
            auto update = [&](int c) -> bool {
                const int st = c % kStages;
                if (!mbar_wait(&full[st], (c / kStages) & 1)) return false;
                tc_fence_after();
                const uint32_t base = smem_u32(smem + st * kStageBytes);
                const uint32_t kb = base + kTile, vb = base + 2 * kTile;
#pragma unroll
                for (int kt = 0; kt < kC / 16; ++kt)  // 16 tokens per MMA
                    tc_mma(tmem_base + kColS, sw128_desc_mn(vb + kt * 2048, kHalf),
                           sw128_desc_mn(kb + kt * 2048, kHalf), kIdescUpd, 1u);
                tc_commit(upd_done);
                return true;
            };
            bool fine = nchunks == 0 || (mbar_wait(s0ready, 0) && update(0));
            for (int c = 0; c < nchunks && fine; ++c) {
                if (*s_abort || !mbar_wait(cdone, c & 1) ||
                    (c >= 2 && !mbar_wait(&ofree[c & 1], ((c >> 1) - 1) & 1))) {
                    fine = false;
                    break;
                }
                tc_fence_after();
                const int st = c % kStages;
                const uint32_t qb = smem_u32(smem + st * kStageBytes);
                // O^T = S^T Q^T with S^T = hi + lo, A from TMEM (8 columns per K = 16)
#pragma unroll
                for (int part = 0; part < 2; ++part) {
                    const uint32_t a = tmem_base + (part ? kColLo : kColHi);
#pragma unroll
                    for (int kk = 0; kk < kD / 16; ++kk) {
                        const uint32_t off = (kk >> 2) * kHalf;
                        tc_mma_tmem_a(tmem_base + kColO + (c & 1) * 128, a + kk * 8,
                                      sw128_desc(qb + off) + 2 * (kk & 3), kIdescRead,
                                      (part | kk) != 0 ? 1u : 0u);
                    }
                }
                tc_commit(&out_ready[c & 1]);
                tc_commit(&empty[st]);
                if (c + 1 < nchunks) fine = update(c + 1);
            }
            if (!fine) *s_abort = 1;
            tc_commit(drain);
            mbar_wait(drain, 0);
        }
    } else {
        const int quarter = warp & 3;
        const int i = quarter * 32 + lane;  // dv index = TMEM lane
        const uint32_t lane_addr = tmem_base + ((uint32_t)(quarter * 32) << 16);
        const size_t st_base = (size_t)bh * kD * kD;
        if (warp < 2 + kStateWarps) {
            // ---------------- state warps: dk columns 64*hf .. 64*hf+63 of row i ----------------
            const int hf = (warp - 2) >> 2;
            {   // S^T[i][:] = gate[0] * S0[:][i]
                const float g0 = nchunks > 0 ? g_row[0] : 1.f;
#pragma unroll
                for (int ch = 0; ch < 2; ++ch) {
                    uint32_t v[32];
                    const int d0 = hf * 64 + ch * 32;
#pragma unroll
                    for (int e = 0; e < 32; ++e)
                        v[e] = __float_as_uint(g0 * state_in[st_base + (size_t)(d0 + e) * kD + i]);
                    tmem_st32(lane_addr + kColS + d0, v);
                }
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(s0ready);
            }
            for (int c = 0; c < nchunks; ++c) {
                const bool w1 = mbar_wait(upd_done, c & 1);
                if (!__all_sync(0xffffffffu, w1 && !*s_abort)) {
                    *s_abort = 1;
                    break;
                }
                tc_fence_after();
                const bool last = c + 1 == nchunks;
                const float gn = last ? 1.f : g_row[c + 1];
#pragma unroll
                for (int ch = 0; ch < 2; ++ch) {
                    const int d0 = hf * 64 + ch * 32;
                    uint32_t v[32];
                    tmem_ld32(lane_addr + kColS + d0, v);
                    uint32_t hi[16], lo[16];
#pragma unroll
                    for (int e = 0; e < 16; ++e) {
                        const float x0 = __uint_as_float(v[2 * e]), x1 = __uint_as_float(v[2 * e + 1]);
                        const __nv_bfloat162 hp = __floats2bfloat162_rn(x0, x1);
                        const float2 hf2 = __bfloat1622float2(hp);
                        hi[e] = *reinterpret_cast<const uint32_t*>(&hp);
                        lo[e] = pack_bf16x2(x0 - hf2.x, x1 - hf2.y);
                    }
                    tmem_st16(lane_addr + kColHi + d0 / 2, hi);
                    tmem_st16(lane_addr + kColLo + d0 / 2, lo);
                    if (last) {
                        // the final state, S[:][i]
#pragma unroll
                        for (int e = 0; e < 32; ++e)
                            state_out[st_base + (size_t)(d0 + e) * kD + i] = __uint_as_float(v[e]);
                    } else {
#pragma unroll
                        for (int e = 0; e < 32; ++e) v[e] = __float_as_uint(gn * __uint_as_float(v[e]));
                        tmem_st32(lane_addr + kColS + d0, v);
                    }
                }
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(cdone);
            }
        } else {
            // ---------------- output warps: O^T[i][t] -> out[b][t][h][i] ----------------
            for (int c = 0; c < nchunks; ++c) {
                const bool w2 = mbar_wait(&out_ready[c & 1], (c >> 1) & 1);
                if (!__all_sync(0xffffffffu, w2 && !*s_abort)) {
                    *s_abort = 1;
                    break;
                }
                tc_fence_after();
                const int t0 = c * kC;
                float* ob = out + (((size_t)b * T + t0) * H + h) * kD + i;
                const size_t tstride = (size_t)H * kD;
#pragma unroll
                for (int ch = 0; ch < 4; ++ch) {
                    uint32_t v[32];
                    tmem_ld32(lane_addr + kColO + (c & 1) * 128 + ch * 32, v);
#pragma unroll
                    for (int e = 0; e < 32; ++e) {
                        const int t = ch * 32 + e;
                        if (t0 + t < T) ob[(size_t)t * tstride] = __uint_as_float(v[e]);
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&ofree[c & 1]);
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                     "r"(kTmemCols)
                     : "memory");
    }
}

}  // namespace lci
