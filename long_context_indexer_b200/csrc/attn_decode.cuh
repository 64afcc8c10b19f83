// attn_decode.cuh -- paged gather + exact sparse attention on tensor cores
// (bf16 in, fp32 softmax and accumulation), head_dim 128, up to 16 query heads
// per KV head, block_size a multiple of 64.
//
// Work: one "pair" = (query row, KV head g). Its selected blocks are cut into
// 64-token tiles ("units"); the units of a pair are split over `nsplit` CTAs
// that form one thread-block cluster.
//
// Per CTA: one producer warp walks the CTA's units, resolves block id -> page
// through the block table and issues TMA tensor loads of the K and V tiles
// (two 64x64 boxes each, 128-byte swizzle) into a 3-stage shared-memory ring
// guarded by mbarriers. Four consumer warps each take 16 tokens of every tile:
// S = Q K^T with mma.m16n8k16 (the 16 rows are the query heads of the group),
// an online softmax in fp32 (exp2, running max and sum), then O += P V.
//
// Fragment layout: the head-dim order inside each 32-dim slice is permuted
// identically for Q and K, the token order inside each 8-token group is the
// permutation pi(x) = x ^ (4 * (x & 1)) for both the S columns and the V rows,
// and the output columns of P V are permuted so that each thread ends with 16
// contiguous dims. Together with the swizzle this makes every 16-byte shared
// load bank-conflict free and needs no ldmatrix.
//
// Combine: the four warps merge through shared memory into a CTA partial
// (max, sum, unnormalised O) held in registers; the CTAs of a cluster then
// store each slice of their partial into the CTA that finishes that slice
// (distributed shared memory), so one cluster barrier separates the exchange
// from the final merge. No global workspace and no atomics.
#pragma once

#include <cooperative_groups.h>

#include "common.cuh"
#include "ptx.cuh"

namespace lci {

namespace dec {
constexpr int kHD = 128;           // head dim
constexpr int kTile = 64;          // tokens per unit
// shared-memory ring depth: 3 stages let two CTAs share an SM; 6 stages fill
// one SM when the grid has about one CTA per SM
constexpr int kStagesShallow = 3;
constexpr int kStagesDeep = 6;
constexpr int kConsumers = 4;      // consumer warps of a group, 16 tokens each
constexpr int kThreads = (kConsumers + 1) * 32;  // one group and the producer
__host__ __device__ constexpr int threads(int groups) { return (kConsumers * groups + 1) * 32; }
constexpr int kBox = 64 * 64 * 2;  // one 64x64 bf16 box = 8 KiB
constexpr int kStageBytes = 4 * kBox;  // K: 2 boxes, V: 2 boxes
constexpr int kMaxSplit = 8;
constexpr int kRows = 16;          // query heads per MMA (padded)
constexpr int kSlots = 64;         // fp32 accumulators per consumer thread
constexpr int kMetaBytes = 256;    // barriers and unit info after the ring
// Slots of one cluster CTA's slice of the output (a multiple of 4), and the
// padded per-lane pitch of a received slice (4 mod 8 floats: 16-byte
// accesses of 8 consecutive lanes hit distinct banks).
__host__ __device__ constexpr int slice_slots(int nsplit) {
    return ((kSlots + nsplit - 1) / nsplit + 3) & ~3;
}
__host__ __device__ constexpr int slice_pitch(int sp) { return sp + ((12 - (sp & 7)) & 7); }
constexpr int recv_floats() {
    int m = 0;
    for (int n = 2; n <= kMaxSplit; ++n) {
        const int f = n * 32 * slice_pitch(slice_slots(n));
        m = f > m ? f : m;
    }
    return m;
}
constexpr int kRecvFloats = recv_floats();  // slices received from the cluster
// shared memory: ring stages, barriers and metadata, received slices and the
// sources' (max, sum) per head
constexpr int smem_bytes(int stages) {
    return stages * kStageBytes + 1024 /*align*/ + kMetaBytes +
           (kRecvFloats + kMaxSplit * kRows * 2) * 4;
}

}  // namespace dec

__device__ __forceinline__ int tok_perm(int x) { return x ^ ((x & 1) << 2); }

// N (2 or 4) consecutive bf16 outputs: one 4- or 8-byte store when the output
// allows it, else N 2-byte stores.
template <int N>
__device__ __forceinline__ void store_bf16_run(__nv_bfloat16* p, const float (&v)[N], bool vec) {
    if constexpr (N == 4) {
        if (vec) {
            uint2 w;
            w.x = pack_bf16x2(v[0], v[1]);
            w.y = pack_bf16x2(v[2], v[3]);
            *reinterpret_cast<uint2*>(p) = w;
            return;
        }
    } else if constexpr (N == 2) {
        if (vec) {
            *reinterpret_cast<uint32_t*>(p) = pack_bf16x2(v[0], v[1]);
            return;
        }
    }
#pragma unroll
    for (int j = 0; j < N; ++j) p[j] = __float2bfloat16_rn(v[j]);
}

// Byte offset of (row r, 16-byte chunk c of the 128-dim row) inside one K or V
// tile stored as two 64x64 boxes with the 128-byte swizzle.
__device__ __forceinline__ uint32_t tile_off(int r, int c) {
    return (uint32_t)((c >> 3) * dec::kBox + r * 128 + (((c & 7) ^ (r & 7)) << 4));
}

// One 64-token K/V tile (two 64x64 boxes of K then of V, 128-byte swizzle, at
// shared address kbase) for consumer warp w, which takes tokens 16w..16w+15:
// S = Q K^T with mma.m16n8k16, the online softmax update of (m, l) for the
// fragment's two head rows, and O += P V for NH of the two 64-dim halves of the
// output, starting at half h0. t0 is the tile's first token; tokens after
// `last` are masked (their V is never read into the MMA).
template <int NH>
__device__ __forceinline__ void dec_consume_tile(uint32_t kbase, int w, int g8, int q4, int t0,
                                                 long long last, float scale_log2,
                                                 const uint4 (&qa)[4], const uint4 (&qb)[4],
                                                 float& m_a, float& m_b, float& l_a, float& l_b,
                                                 float (&o)[NH][8][4], int h0 = 0) {
    using namespace dec;
    const long long wt0 = (long long)t0 + 16 * w;  // first token of this warp
    if (wt0 <= last) {
        const uint32_t vbase = kbase + 2 * kBox;
        // S = Q K^T over this warp's 16 tokens (two n-tiles of 8)
        float sacc[2][4];
#pragma unroll
        for (int j = 0; j < 2; ++j) {
#pragma unroll
            for (int e = 0; e < 4; ++e) sacc[j][e] = 0.f;
            const int tr = 16 * w + 8 * j + tok_perm(g8);
#pragma unroll
            for (int sl = 0; sl < 4; ++sl) {
                const uint4 kk = lds128(kbase + tile_off(tr, 4 * sl + q4));
                mma_bf16_16816(sacc[j], qa[sl].x, qb[sl].x, qa[sl].y, qb[sl].y, kk.x, kk.y);
                mma_bf16_16816(sacc[j], qa[sl].z, qb[sl].z, qa[sl].w, qb[sl].w, kk.z, kk.w);
            }
        }
        // tokens of the C-fragment columns: n = 2*q4, 2*q4+1 of each n-tile
        const int c0 = tok_perm(2 * q4), c1 = tok_perm(2 * q4 + 1);
        const bool partial = wt0 + 15 > last;
        float x[2][4];
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            const long long ta = wt0 + 8 * j + c0, tb = wt0 + 8 * j + c1;
            x[j][0] = (partial && ta > last) ? -INFINITY : sacc[j][0] * scale_log2;
            x[j][1] = (partial && tb > last) ? -INFINITY : sacc[j][1] * scale_log2;
            x[j][2] = (partial && ta > last) ? -INFINITY : sacc[j][2] * scale_log2;
            x[j][3] = (partial && tb > last) ? -INFINITY : sacc[j][3] * scale_log2;
        }
        float mx_a = fmaxf(fmaxf(x[0][0], x[0][1]), fmaxf(x[1][0], x[1][1]));
        float mx_b = fmaxf(fmaxf(x[0][2], x[0][3]), fmaxf(x[1][2], x[1][3]));
        mx_a = fmaxf(mx_a, __shfl_xor_sync(0xffffffffu, mx_a, 1));
        mx_a = fmaxf(mx_a, __shfl_xor_sync(0xffffffffu, mx_a, 2));
        mx_b = fmaxf(mx_b, __shfl_xor_sync(0xffffffffu, mx_b, 1));
        mx_b = fmaxf(mx_b, __shfl_xor_sync(0xffffffffu, mx_b, 2));
        const float mn_a = fmaxf(m_a, mx_a), mn_b = fmaxf(m_b, mx_b);
        const float base_a = mn_a == -INFINITY ? 0.f : mn_a;
        const float base_b = mn_b == -INFINITY ? 0.f : mn_b;
        const float corr_a = exp2f(m_a - base_a), corr_b = exp2f(m_b - base_b);
        m_a = mn_a;
        m_b = mn_b;
        float pr[2][4];
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            pr[j][0] = exp2f(x[j][0] - base_a);
            pr[j][1] = exp2f(x[j][1] - base_a);
            pr[j][2] = exp2f(x[j][2] - base_b);
            pr[j][3] = exp2f(x[j][3] - base_b);
        }
        l_a = l_a * corr_a + (pr[0][0] + pr[0][1] + pr[1][0] + pr[1][1]);
        l_b = l_b * corr_b + (pr[0][2] + pr[0][3] + pr[1][2] + pr[1][3]);
#pragma unroll
        for (int h = 0; h < NH; ++h)
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                o[h][i][0] *= corr_a;
                o[h][i][1] *= corr_a;
                o[h][i][2] *= corr_b;
                o[h][i][3] *= corr_b;
            }
        const uint32_t pa0 = pack_bf16x2(pr[0][0], pr[0][1]);
        const uint32_t pa1 = pack_bf16x2(pr[0][2], pr[0][3]);
        const uint32_t pa2 = pack_bf16x2(pr[1][0], pr[1][1]);
        const uint32_t pa3 = pack_bf16x2(pr[1][2], pr[1][3]);
        // V rows of the k positions 2q4, 2q4+1, 2q4+8, 2q4+9
        const int r0 = 16 * w + c0, r1 = 16 * w + c1, r2 = r0 + 8, r3 = r1 + 8;
        // masked tokens must not reach the MMA (their V may be unset memory)
        const bool z0 = partial && wt0 + c0 > last, z1 = partial && wt0 + c1 > last;
        const bool z2 = partial && wt0 + 8 + c0 > last, z3 = partial && wt0 + 8 + c1 > last;
#pragma unroll
        for (int hh = 0; hh < NH; ++hh) {
            const int h = h0 + hh;
            uint4 va = lds128(vbase + tile_off(r0, 8 * h + g8));
            uint4 vb = lds128(vbase + tile_off(r1, 8 * h + g8));
            uint4 vc = lds128(vbase + tile_off(r2, 8 * h + g8));
            uint4 vd = lds128(vbase + tile_off(r3, 8 * h + g8));
            if (z0) va = make_uint4(0, 0, 0, 0);
            if (z1) vb = make_uint4(0, 0, 0, 0);
            if (z2) vc = make_uint4(0, 0, 0, 0);
            if (z3) vd = make_uint4(0, 0, 0, 0);
            const uint32_t wa[4] = {va.x, va.y, va.z, va.w}, wb[4] = {vb.x, vb.y, vb.z, vb.w};
            const uint32_t wc[4] = {vc.x, vc.y, vc.z, vc.w}, wd[4] = {vd.x, vd.y, vd.z, vd.w};
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const uint32_t sel = (i & 1) ? 0x7632u : 0x5410u;
                const uint32_t b0 = __byte_perm(wa[i >> 1], wb[i >> 1], sel);
                const uint32_t b1 = __byte_perm(wc[i >> 1], wd[i >> 1], sel);
                mma_bf16_16816(o[hh][i], pa0, pa1, pa2, pa3, b0, b1);
            }
        }
    }
}

// kGroups consumer groups of kConsumers warps take alternate ring stages, each
// with its own softmax state (two groups when the CTA has an SM to itself: the
// latency of one tile's MMA and softmax chain hides under the other's).
template <int kStages, int kGroups>
__global__ void __launch_bounds__(dec::threads(kGroups)) sparse_attn_decode_kernel(
    const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
    const __nv_bfloat16* __restrict__ q, const int32_t* __restrict__ table, int nb_max,
    int num_pages, int H_kv, int bs, int S, int H_q, const int32_t* __restrict__ ids, int topk,
    const int32_t* __restrict__ ctx_len, const int32_t* __restrict__ q_start, float scale_log2,
    __nv_bfloat16* __restrict__ out, int nsplit, const unsigned int* __restrict__ ready,
    float* __restrict__ lse, const unsigned long long* __restrict__ picks) {
    using namespace dec;
    namespace cg = cooperative_groups;
    constexpr int kCW = kConsumers * kGroups;    // consumer warps; warp kCW produces
    constexpr int kWoS = kSlots + 4;             // partial row pitch (4 mod 8 floats: no conflicts)
    constexpr int kSlotsPer = kSlots / kCW;      // accumulator slots each thread merges
    constexpr int kNT = threads(kGroups);
    static_assert(kGroups == 1 || kGroups == 2, "one or two groups");
    static_assert(kCW * (32 * kWoS + 2 * kRows) * 4 <= kStages * kStageBytes,
                  "warp partials fit in the ring");
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char* smem = reinterpret_cast<unsigned char*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* full_bar = reinterpret_cast<uint64_t*>(smem + kStages * kStageBytes);
    uint64_t* empty_bar = full_bar + kStages;
    int* info = reinterpret_cast<int*>(empty_bar + kStages);  // t0 of the unit, or -1

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int pair = blockIdx.x, split = blockIdx.y;
    const int row = pair / H_kv, g = pair - row * H_kv;
    const int G = H_q / H_kv;
    const int b = row / S, s = row - b * S;
    const int tiles_per_block = bs / kTile;
    const int nunits = topk * tiles_per_block;
    const int per = (nunits + nsplit - 1) / nsplit;
    const int u0 = split * per;
    const int u1 = min(nunits, u0 + per);

    if (tid == 0) {
        for (int i = 0; i < kStages; ++i) {
            mbar_init(&full_bar[i], 1);
            mbar_init(&empty_bar[i], kConsumers);
        }
        fence_mbar_init();
    }
    if (warp == kCW && lane == 0) {
        prefetch_tensormap(&tm_k);
        prefetch_tensormap(&tm_v);
    }
    __syncthreads();
    // first half of the barrier that guarantees every CTA of the cluster runs
    // before any distributed shared memory store (the wait is at the combine)
    if (nsplit > 1) cluster_arrive_relaxed();

    // Per-thread fragment coordinates.
    const int g8 = lane >> 2, q4 = lane & 3;

    // Query rows of this pair (independent of the previous kernel's output).
    uint4 qa[4], qb[4];
    if (warp < kCW) {
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
    }

    // Positions and the block table are inputs of the step; warm the table row
    // into L2 so the page lookups after the wait hit it.
    const long long p = (long long)q_start[b] + s;
    const long long ctx = ctx_len[b];
    const long long last = p < ctx - 1 ? p : ctx - 1;
    if (warp == kCW) {
        const int32_t* trow = table + (size_t)b * nb_max;
        const int nlines = min(nb_max, 8192) / 32;  // 128-byte lines of the row
        for (int l = lane; l < nlines; l += 32) prefetch_l2(trow + l * 32);
    }
    // Block ids come from a producer: either the previous kernel on the stream
    // (programmatic dependent launch: wait for that whole grid), or a producer
    // that publishes rows one by one by a release store of a nonzero ready[row]
    // after writing the row's ids (bounded wait on this row's flag only). The
    // library's producer clears its flags itself before this grid can start. A
    // row whose flag never comes is skipped (zero output, time-out status).
    // A producer may instead publish each pick as (block id, page) in
    // picks[row][rank] (kPickPending until written): the producer warp then
    // polls exactly the picks it needs, with no flag, id or table round trip.
    __shared__ int s_alive;
    if (picks == nullptr) {
        if (ready == nullptr) {
            pdl_wait();
        } else {
            if (tid == 0) s_alive = wait_flag_set(ready + row) ? 1 : 0;
            __syncthreads();
        }
    }
    const bool alive = picks != nullptr || ready == nullptr || s_alive != 0;

    float m_a = -INFINITY, m_b = -INFINITY, l_a = 0.f, l_b = 0.f;
    float o[2][8][4];
#pragma unroll
    for (int h = 0; h < 2; ++h)
#pragma unroll
        for (int i = 0; i < 8; ++i)
#pragma unroll
            for (int e = 0; e < 4; ++e) o[h][i][e] = 0.f;

    if (warp == kCW) {
        // ---------------- producer ----------------
        // Lanes resolve 32 units at a time (block id -> page -> TMA row), so the
        // dependent id and table loads overlap; lane 0 then issues the copies.
        const int32_t* row_ids = ids + (size_t)row * topk;
        bool running = true;
        for (int base = u0; base < u1 && running; base += 32) {
            const int u = base + lane;
            int t0 = -1, y = 0;
            if (u < u1 && alive) {
                const int i = u / tiles_per_block, sub = u - i * tiles_per_block;
                int j, page = -1;
                if (picks != nullptr) {
                    const unsigned long long v =
                        wait_slot(picks + (size_t)row * topk + i, kPickPending, ~0ull);
                    j = (int)(unsigned)(v >> 32);
                    page = (int)(unsigned)(v & 0xffffffffull);
                } else {
                    j = __ldcg(row_ids + i);
                    if (j >= 0 && j < nb_max) page = table[(size_t)b * nb_max + j];
                }
                if (j >= 0 && j < nb_max) {
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
                const int it = base - u0 + k;
                const int st = it % kStages;
                int ok = 1;
                if (lane == 0) {
                    if (it >= kStages) ok = mbar_wait(&empty_bar[st], ((it / kStages) - 1) & 1);
                    if (ok) {
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
                }
                if (!__shfl_sync(0xffffffffu, ok, 0)) {
                    running = false;
                    break;
                }
            }
        }
    } else {
        // ---------------- consumers ----------------
        // group grp takes the stages it = grp, grp + kGroups, ...; warp w of
        // the group takes tokens 16w..16w+15 of each tile
        const int grp = warp / kConsumers, w = warp - grp * kConsumers;
        for (int u = u0 + grp, it = grp; u < u1; u += kGroups, it += kGroups) {
            const int st = it % kStages;
            const bool ok = mbar_wait(&full_bar[st], (it / kStages) & 1);
            const int t0 = info[st];
            if (ok && t0 >= 0)
                dec_consume_tile(smem_u32(smem + st * kStageBytes), w, g8, q4, t0, last,
                                 scale_log2, qa, qb, m_a, m_b, l_a, l_b, o);
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty_bar[st]);
        }
    }
    __syncthreads();  // every stage consumed: the ring memory is free

    // ---------------- combine ----------------
    // Accumulator slot o = 32*h + 4*i + e of lane l holds head (l>>2) + 8*(e>>1),
    // dim 64*h + 16*(l&3) + 8*(e&1) + i (the mma C-fragment layout).
    // 1. Each consumer warp leaves (max, sum, unnormalised O) in the free ring
    //    memory; consumer thread (w, l) then merges slots 16w..16w+15 of lane l
    //    over the four warps into the CTA partial, in registers.
    // 2. A lone CTA normalises and writes the output. In a cluster, each CTA
    //    stores every slice of its partial into the CTA owning that slice
    //    (distributed shared memory), one cluster barrier publishes the stores,
    //    and every owner merges its slice over the cluster from its own memory.
    float* wo = reinterpret_cast<float*>(smem);             // [warp][lane][kWoS]
    float* wm = wo + kCW * 32 * kWoS;                       // [warp][16] running max
    float* wl = wm + kCW * kRows;                           // [warp][16] running sum
    float* ro = reinterpret_cast<float*>(smem + kStages * kStageBytes + kMetaBytes);
    float* rml = ro + kRecvFloats;                          // [source CTA][16][max, sum]
    __nv_bfloat16* orow = out + ((size_t)row * H_q + (size_t)g * G) * kHD;
    const bool vec_out = (reinterpret_cast<uintptr_t>(out) & 7u) == 0u;
    if (warp < kCW) {
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
        float4* dst = reinterpret_cast<float4*>(wo + (warp * 32 + lane) * kWoS);
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
            for (int i = 0; i < 8; ++i)
                dst[8 * h + i] = make_float4(o[h][i][0], o[h][i][1], o[h][i][2], o[h][i][3]);
    }
    __syncthreads();
    const int sp = slice_slots(nsplit), pitch = slice_pitch(sp);
    if (nsplit > 1) cluster_wait();  // every CTA of the cluster has started
    if (warp < kCW) {
        // heads of this lane's slots: e = 0, 1 -> ha; e = 2, 3 -> hb
        constexpr int NJ = kSlotsPer / 4;  // float4 groups this thread merges
        const int ha = g8, hb = g8 + 8;
        float Ma = -INFINITY, Mb = -INFINITY;
#pragma unroll
        for (int w2 = 0; w2 < kCW; ++w2) {
            Ma = fmaxf(Ma, wm[w2 * kRows + ha]);
            Mb = fmaxf(Mb, wm[w2 * kRows + hb]);
        }
        const float ba = Ma == -INFINITY ? 0.f : Ma, bb = Mb == -INFINITY ? 0.f : Mb;
        float fa[kCW], fb[kCW], La = 0.f, Lb = 0.f;
#pragma unroll
        for (int w2 = 0; w2 < kCW; ++w2) {
            fa[w2] = exp2f(wm[w2 * kRows + ha] - ba);
            fb[w2] = exp2f(wm[w2 * kRows + hb] - bb);
            La += fa[w2] * wl[w2 * kRows + ha];
            Lb += fb[w2] * wl[w2 * kRows + hb];
        }
        float4 acc[NJ];
#pragma unroll
        for (int j = 0; j < NJ; ++j) acc[j] = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int w2 = 0; w2 < kCW; ++w2) {
            const float4* src =
                reinterpret_cast<const float4*>(wo + (w2 * 32 + lane) * kWoS) + NJ * warp;
#pragma unroll
            for (int j = 0; j < NJ; ++j) {
                const float4 v = src[j];
                acc[j].x += fa[w2] * v.x;
                acc[j].y += fa[w2] * v.y;
                acc[j].z += fb[w2] * v.z;
                acc[j].w += fb[w2] * v.w;
            }
        }
        if (nsplit == 1) {
            // slots kSlotsPer*warp + 4j + e: h = slot >> 5, i = (slot >> 2) & 7,
            // so group j of component e lands on dim 64h + 16*q4 + 8*(e&1) + i0 + j
            const float ia = La > 0.f ? 1.f / La : 0.f, ib = Lb > 0.f ? 1.f / Lb : 0.f;
            const int slot0 = kSlotsPer * warp;
            const int d0 = 64 * (slot0 >> 5) + 16 * q4 + ((slot0 >> 2) & 7);
            if (ha < G) {
                float vx[NJ], vy[NJ];
#pragma unroll
                for (int j = 0; j < NJ; ++j) {
                    vx[j] = acc[j].x * ia;
                    vy[j] = acc[j].y * ia;
                }
                store_bf16_run<NJ>(orow + ha * kHD + d0, vx, vec_out);
                store_bf16_run<NJ>(orow + ha * kHD + d0 + 8, vy, vec_out);
            }
            if (hb < G) {
                float vz[NJ], vw[NJ];
#pragma unroll
                for (int j = 0; j < NJ; ++j) {
                    vz[j] = acc[j].z * ib;
                    vw[j] = acc[j].w * ib;
                }
                store_bf16_run<NJ>(orow + hb * kHD + d0, vz, vec_out);
                store_bf16_run<NJ>(orow + hb * kHD + d0 + 8, vw, vec_out);
            }
            // log2-sum-exp2 of the scaled logits, for combining partial results
            if (lse != nullptr && warp == 0 && q4 == 0) {
                float* lrow = lse + (size_t)row * H_q + (size_t)g * G;
                if (ha < G) lrow[ha] = La > 0.f ? Ma + log2f(La) : -INFINITY;
                if (hb < G) lrow[hb] = Lb > 0.f ? Mb + log2f(Lb) : -INFINITY;
            }
        } else {
            namespace cg = cooperative_groups;
            cg::cluster_group cluster = cg::this_cluster();
#pragma unroll
            for (int j = 0; j < NJ; ++j) {
                const int slot = kSlotsPer * warp + 4 * j;
                const int owner = slot / sp;
                float* dst = cluster.map_shared_rank(ro, owner) +
                             (size_t)(split * 32 + lane) * pitch + (slot - owner * sp);
                *reinterpret_cast<float4*>(dst) = acc[j];
            }
            if (warp == 0 && q4 == 0) {
                for (int c = 0; c < nsplit; ++c) {
                    float* d = cluster.map_shared_rank(rml, c) + split * 2 * kRows;
                    *reinterpret_cast<float2*>(d + 2 * ha) = make_float2(Ma, La);
                    *reinterpret_cast<float2*>(d + 2 * hb) = make_float2(Mb, Lb);
                }
            }
        }
    }
    if (nsplit == 1) return;
    cluster_arrive();
    cluster_wait();
    // This CTA owns slots [split*sp, split*sp + sp) of every lane.
    const int s0 = split * sp;
    const int ngroups = s0 < kSlots ? (min(kSlots, s0 + sp) - s0) / 4 : 0;
    for (int e = tid; e < ngroups * 32; e += kNT) {
        const int ln = e & 31, gq = e >> 5;
        const int slot = s0 + 4 * gq;
        const int ha = ln >> 2, hb = ha + 8;
        float Ma = -INFINITY, Mb = -INFINITY;
#pragma unroll
        for (int r = 0; r < kMaxSplit; ++r) {
            if (r < nsplit) {
                Ma = fmaxf(Ma, rml[(r * kRows + ha) * 2]);
                Mb = fmaxf(Mb, rml[(r * kRows + hb) * 2]);
            }
        }
        const float ba = Ma == -INFINITY ? 0.f : Ma, bb = Mb == -INFINITY ? 0.f : Mb;
        float La = 0.f, Lb = 0.f;
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int r = 0; r < kMaxSplit; ++r) {
            if (r < nsplit) {
                const float2 xa = *reinterpret_cast<const float2*>(rml + (r * kRows + ha) * 2);
                const float2 xb = *reinterpret_cast<const float2*>(rml + (r * kRows + hb) * 2);
                const float fa = exp2f(xa.x - ba), fb = exp2f(xb.x - bb);
                La += fa * xa.y;
                Lb += fb * xb.y;
                const float4 v = *reinterpret_cast<const float4*>(ro + (size_t)(r * 32 + ln) * pitch + 4 * gq);
                acc.x += fa * v.x;
                acc.y += fa * v.y;
                acc.z += fb * v.z;
                acc.w += fb * v.w;
            }
        }
        const float ia = La > 0.f ? 1.f / La : 0.f, ib = Lb > 0.f ? 1.f / Lb : 0.f;
        const int d = 64 * (slot >> 5) + 16 * (ln & 3) + ((slot >> 2) & 7);
        if (ha < G) {
            orow[ha * kHD + d] = __float2bfloat16_rn(acc.x * ia);
            orow[ha * kHD + d + 8] = __float2bfloat16_rn(acc.y * ia);
        }
        if (hb < G) {
            orow[hb * kHD + d] = __float2bfloat16_rn(acc.z * ib);
            orow[hb * kHD + d + 8] = __float2bfloat16_rn(acc.w * ib);
        }
    }
    if (lse != nullptr && split == 0 && tid < G) {
        float M = -INFINITY;
        for (int r = 0; r < nsplit; ++r) M = fmaxf(M, rml[(r * kRows + tid) * 2]);
        const float base = M == -INFINITY ? 0.f : M;
        float L = 0.f;
        for (int r = 0; r < nsplit; ++r)
            L += exp2f(rml[(r * kRows + tid) * 2] - base) * rml[(r * kRows + tid) * 2 + 1];
        lse[(size_t)row * H_q + (size_t)g * G + tid] = L > 0.f ? M + log2f(L) : -INFINITY;
    }
}

}  // namespace lci
