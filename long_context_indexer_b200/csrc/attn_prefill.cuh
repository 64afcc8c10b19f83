// attn_prefill.cuh -- paged gather + exact sparse attention for many queries
// per sequence on the 5th-generation tensor cores (tcgen05 + TMEM), bf16 in,
// fp32 softmax and accumulation, head_dim 128, block_size a multiple of 64.
//
// [Hetero] §IV asks for a compute-heavy prefill path next to the memory-bound
// decode path; [GPU-stack] "Separate Paths for Prefill and Decode" asks for
// batched fused operators in prefill. The work here is organised so that a
// gathered K/V tile serves many rows of one MMA:
//
// Tile. A CTA owns 128 MMA rows: QT = 128 / G consecutive queries of one
// sequence times the G query heads of one KV head g (row r = query r / G,
// head r % G). It walks the union of the blocks its QT queries selected, in
// block order, in stages of 128 tokens (two 64-token units: two blocks of 64,
// or one block of 128). For every stage:
//   S  = Q K^T            tcgen05.mma, M=128 rows, N=128 tokens, K=128 dims
//   P  = exp2(S*c - m)    rows whose query did not select the unit's block, and
//                         tokens after the query's position, get P = 0
//   O += P V              tcgen05.mma with A = P read from TMEM, B = V read
//                         MN-major from shared memory (S = Q K^T reads Q from
//                         TMEM too)
// Q (as bf16 pairs, the MMA's A operand), S (two buffers, each also holding
// its stage's P once read) and O live in TMEM; shared memory holds only the
// K and V rings (three stages each). Rows of one
// MMA belong to different queries, so a K/V tile is read once per tile instead
// of once per query.
//
// Warps: 0 TMA producer (K and V rings, 128-byte swizzle), 1 MMA issuer (one
// thread), 2..9 softmax: two threads per MMA row (TMEM lane), each taking one
// 64-token unit of a stage and 64 of the output dims. The softmax is online
// with a lazy rescale: a row's reference maximum m moves only when a stage's
// maximum exceeds it by more than 8 (log2 units), so P <= 2^8 and O is
// rescaled in TMEM only then (after the previous P V has completed). The
// final O / l is exact whatever m is.
//
// V rows of tokens at or past the sequence's context length (a partly filled
// last page: unwritten cache memory) and of absent units are zeroed in shared
// memory before the P V MMA reads them, so such memory never reaches O even as
// 0 * NaN.
#pragma once

#include "common.cuh"
#include "index_prefill.cuh"
#include "ptx.cuh"

namespace lci {

namespace pfa {
constexpr int kHD = 128;
constexpr int kRows = 128;             // MMA rows per tile
constexpr int kStageTok = 128;         // tokens per stage (two 64-token units)
constexpr int kHalf = 128 * 128;       // one 64-dim half of a 128-row tile: 16 KiB
constexpr int kTileBytes = 2 * kHalf;  // 128 rows x 128 dims bf16: 32 KiB
constexpr int kKStages = 3, kVStages = 3;
constexpr int kMaxWords = 512;         // block bitmap words: nb_max <= 16384
constexpr int kMaxUnion = 1024;        // distinct blocks per tile (QT * topk)
constexpr int kSoftWarps = 8;            // two threads per MMA row
constexpr int kVWarp = 2 + kSoftWarps;     // V producer (warp 0 produces K)
constexpr int kThreads = 64 + 32 * kSoftWarps + 32;
// TMEM columns: O [128 rows x 128 dims] fp32, two S buffers [128 x 128 tokens]
// fp32 whose first 64 columns then hold the stage's P as bf16 pairs, and Q
// [128 x 128 dims] as bf16 pairs (the A operand of S = Q K^T)
constexpr int kColO = 0, kColS = 128, kColQ = 384, kTmemCols = 512;
constexpr float kLazy = 8.0f;          // rescale when the maximum grows past m + 8
// shared memory layout (offsets from a 1024-byte aligned base)
constexpr int kOffK = 0;
constexpr int kOffV = kOffK + kKStages * kTileBytes;
constexpr int kOffUnion = kOffV + kVStages * kTileBytes;
constexpr int kUnionBytes = 2 * kMaxWords * 4 + 3 * kMaxUnion * 4;
constexpr int kOffBar = kOffUnion + kUnionBytes;
// exchange between a row's two threads: [3][2][128] floats (two stage buffers
// of row maxima, then the row sums) and [2][2][128] ints (wait outcomes)
constexpr int kOffXchg = kOffBar + 256;
constexpr int kSmemBytes = kOffXchg + 3 * 2 * 128 * 4 + 2 * 2 * 128 * 4 + 1024 /*alignment slack*/;
// instruction descriptors: D fp32, A and B bf16, M = 128, N = 128;
// S = Q K^T with both operands K-major, O += P V with V (B) MN-major
constexpr uint32_t kIdescQK = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(128 >> 3) << 17) |
                              ((uint32_t)(128 >> 4) << 24);
constexpr uint32_t kIdescPV = kIdescQK | (1u << 16);
}  // namespace pfa

// Shared-memory descriptor of an MN-major operand written by TMA with the
// 128-byte swizzle: 64-element rows of 128 bytes along MN, 8 rows (along K)
// per 1024-byte swizzle atom; `lbo` bytes to the next 64 elements along MN,
// 1024 bytes to the next 8 rows along K.
__device__ __forceinline__ uint64_t sw128_desc_mn(uint32_t smem_addr, uint32_t lbo) {
    return (uint64_t)((smem_addr >> 4) & 0x3fff) | ((uint64_t)((lbo >> 4) & 0x3fff) << 16) |
           ((uint64_t)(1024 >> 4) << 32) | ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}

// D (+)= A B with A read from TMEM (M lanes x K/2 columns of bf16 pairs).
__device__ __forceinline__ void tc_mma_tmem_a(uint32_t tmem_d, uint32_t tmem_a, uint64_t b,
                                              uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(tmem_d),
        "r"(tmem_a), "l"(b), "r"(idesc), "r"(accumulate));
}

// 16 consecutive 32-bit columns of this thread's TMEM lane <- r.
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,"
        "%13,%14,%15,%16};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
        "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
        "r"(r[15])
        : "memory");
}

// 32 consecutive 32-bit columns of this thread's TMEM lane <- r.
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,"
        "%13,%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(
            taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
        "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
        "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]),
        "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]),
        "r"(r[29]), "r"(r[30]), "r"(r[31])
        : "memory");
}

__device__ __forceinline__ void tmem_wait_st() {
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// 64 consecutive 32-bit columns of this thread's TMEM lane, one load.
__device__ __forceinline__ void tmem_ld64(uint32_t taddr, uint32_t (&r)[64]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x64.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32,%33,%34,%35,%36,%37,%38,%39,%40,%41,%42,%43,%44,%45,%46,%47,%48,%49,%50,%51,%52,%53,%54,%55,%56,%57,%58,%59,%60,%61,%62,%63}, [%64];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31]), "=r"(r[32]), "=r"(r[33]), "=r"(r[34]), "=r"(r[35]), "=r"(r[36]), "=r"(r[37]), "=r"(r[38]), "=r"(r[39]), "=r"(r[40]), "=r"(r[41]), "=r"(r[42]), "=r"(r[43]), "=r"(r[44]), "=r"(r[45]), "=r"(r[46]), "=r"(r[47]), "=r"(r[48]), "=r"(r[49]), "=r"(r[50]), "=r"(r[51]), "=r"(r[52]), "=r"(r[53]), "=r"(r[54]), "=r"(r[55]), "=r"(r[56]), "=r"(r[57]), "=r"(r[58]), "=r"(r[59]), "=r"(r[60]), "=r"(r[61]), "=r"(r[62]), "=r"(r[63])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;"
                 : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]), "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]), "+r"(r[15]), "+r"(r[16]), "+r"(r[17]), "+r"(r[18]), "+r"(r[19]), "+r"(r[20]), "+r"(r[21]), "+r"(r[22]), "+r"(r[23]), "+r"(r[24]), "+r"(r[25]), "+r"(r[26]), "+r"(r[27]), "+r"(r[28]), "+r"(r[29]), "+r"(r[30]), "+r"(r[31]), "+r"(r[32]), "+r"(r[33]), "+r"(r[34]), "+r"(r[35]), "+r"(r[36]), "+r"(r[37]), "+r"(r[38]), "+r"(r[39]), "+r"(r[40]), "+r"(r[41]), "+r"(r[42]), "+r"(r[43]), "+r"(r[44]), "+r"(r[45]), "+r"(r[46]), "+r"(r[47]), "+r"(r[48]), "+r"(r[49]), "+r"(r[50]), "+r"(r[51]), "+r"(r[52]), "+r"(r[53]), "+r"(r[54]), "+r"(r[55]), "+r"(r[56]), "+r"(r[57]), "+r"(r[58]), "+r"(r[59]), "+r"(r[60]), "+r"(r[61]), "+r"(r[62]), "+r"(r[63])
                 :
                 : "memory");
}

// Byte offset of (row r, 16-byte chunk c of its 128 dims) in a 128-row tile
// stored as two 64-dim halves with the 128-byte swizzle.
__device__ __forceinline__ uint32_t pfa_off(int r, int c) {
    return (uint32_t)((c >> 3) * pfa::kHalf + r * 128 + (((c & 7) ^ (r & 7)) << 4));
}

__global__ void __launch_bounds__(pfa::kThreads, 1) sparse_attn_prefill_kernel(
    const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
    const __nv_bfloat16* __restrict__ q, const int32_t* __restrict__ table, int nb_max,
    int num_pages, int H_kv, int bs, int S, int H_q, const int32_t* __restrict__ ids, int topk,
    const int32_t* __restrict__ ctx_len, const int32_t* __restrict__ q_start, float scale_log2,
    __nv_bfloat16* __restrict__ out, int q_tiles, float* __restrict__ lse) {
    using namespace pfa;
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char* smem = reinterpret_cast<unsigned char*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint32_t* bitmap = reinterpret_cast<uint32_t*>(smem + kOffUnion);  // [kMaxWords]
    uint32_t* wpre = bitmap + kMaxWords;                                // [kMaxWords]
    int* ublk = reinterpret_cast<int*>(wpre + kMaxWords);              // [kMaxUnion]
    int* upage = ublk + kMaxUnion;                                      // [kMaxUnion]
    uint32_t* umask = reinterpret_cast<uint32_t*>(upage + kMaxUnion);  // [kMaxUnion]
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kOffBar);
    uint64_t* kfull = bars;                  // [kKStages]
    uint64_t* kempty = kfull + kKStages;     // [kKStages]
    uint64_t* vfull = kempty + kKStages;     // [kVStages]
    uint64_t* vempty = vfull + kVStages;     // [kVStages]
    uint64_t* sfull = vempty + kVStages;     // [2] S buffer written
    uint64_t* pfull = sfull + 2;             // [2] P buffer written (4 softmax warps)
    uint64_t* obar = pfull + 2;              // every P V completed, in order
    uint64_t* ofin = obar + 1;               // the tile's last P V completed
    uint64_t* drain = ofin + 1;              // every MMA of the tile completed
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
    int* s_nunion = reinterpret_cast<int*>(tmem_slot + 1);
    // set by any role whose bounded wait ran out: every role then stops
    volatile int* s_abort = s_nunion + 1;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int G = H_q / H_kv;
    const int QT = kRows / G;
    // heaviest tiles (latest queries: most visible blocks) first
    const int tile = (int)(gridDim.x - 1 - blockIdx.x);
    const int g = tile % H_kv;
    const int qt = (tile / H_kv) % q_tiles;
    const int b = tile / (H_kv * q_tiles);
    const int s0 = qt * QT;
    const int nwords = (nb_max + 31) >> 5;
    const int upb = bs / 64;  // 64-token units per block

    if (tid == 0) {
        for (int i = 0; i < kKStages; ++i) {
            mbar_init(&kfull[i], 1);
            mbar_init(&kempty[i], 1);
        }
        for (int i = 0; i < kVStages; ++i) {
            mbar_init(&vfull[i], 1);
            mbar_init(&vempty[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&sfull[i], 1);
            mbar_init(&pfull[i], kSoftWarps);
        }
        mbar_init(obar, 1);
        mbar_init(ofin, 1);
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
        prefetch_tensormap(&tm_k);
        prefetch_tensormap(&tm_v);
    }
    // ---------------- the union of the tile's selected blocks ----------------
    for (int w = tid; w < nwords; w += kThreads) bitmap[w] = 0u;
    const int nent = QT * topk;
    for (int e = tid; e < nent; e += kThreads) umask[e] = 0u;
    __syncthreads();
    for (int e = tid; e < nent; e += kThreads) {
        const int qi = e / topk;
        const int s = s0 + qi;
        if (s < S) {
            const int j = ids[((size_t)b * S + s) * topk + (e - qi * topk)];
            if (j >= 0 && j < nb_max)
                atomicOr(&bitmap[j >> 5], 1u << (j & 31));
            else if (j != -1)
                raise_status(kStatusBadBlockId);
        }
    }
    __syncthreads();
    if (warp == 0) {  // exclusive prefix of the words' population counts
        const int per = (nwords + 31) / 32;
        int sum = 0;
        for (int k = 0; k < per; ++k) {
            const int w = lane * per + k;
            if (w < nwords) sum += __popc(bitmap[w]);
        }
        int incl = sum;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int t = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += t;
        }
        int run = incl - sum;
        for (int k = 0; k < per; ++k) {
            const int w = lane * per + k;
            if (w < nwords) {
                wpre[w] = (uint32_t)run;
                run += __popc(bitmap[w]);
            }
        }
        if (lane == 31) *s_nunion = incl;
    }
    __syncthreads();
    for (int e = tid; e < nent; e += kThreads) {
        const int qi = e / topk;
        const int s = s0 + qi;
        if (s < S) {
            const int j = ids[((size_t)b * S + s) * topk + (e - qi * topk)];
            if (j >= 0 && j < nb_max) {
                const int pos = (int)wpre[j >> 5] + __popc(bitmap[j >> 5] & ((1u << (j & 31)) - 1u));
                ublk[pos] = j;
                atomicOr(&umask[pos], 1u << qi);
            }
        }
    }
    __syncthreads();
    const int nunion = *s_nunion;
    for (int u = tid; u < nunion; u += kThreads) {
        const int page = table[(size_t)b * nb_max + ublk[u]];
        if (page < 0 || page >= num_pages) {
            raise_status(kStatusBadPage);
            upage[u] = -1;
        } else {
            upage[u] = page;
        }
    }
    const int nunits = nunion * upb;
    const int nstages = (nunits + 1) / 2;
    const long long ctx = ctx_len[b];

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    // ---------------- Q tile -> TMEM (the A operand of S = Q K^T) ----------------
    // The softmax warps store their row halves (bf16 pairs: column c holds dims
    // 2c, 2c+1); the MMA warp waits for them on named barrier 5. The producer
    // starts its loads meanwhile.
    constexpr int kQBarrier = 5, kQThreads = 32 + 32 * kSoftWarps;
    if (warp >= 2 && warp < kVWarp) {
        const int quarter = warp & 3, hf = (warp - 2) >> 2;
        const int r = quarter * 32 + lane;
        const int qi = r / G, s = s0 + qi;
        const uint4* src = reinterpret_cast<const uint4*>(
            q + (((size_t)b * S + s) * H_q + (size_t)g * G + (r - qi * G)) * kHD);
        uint32_t qv[32];
#pragma unroll
        for (int c = 0; c < 8; ++c) {
            const uint4 v = s < S ? src[8 * hf + c] : make_uint4(0, 0, 0, 0);
            qv[4 * c] = v.x;
            qv[4 * c + 1] = v.y;
            qv[4 * c + 2] = v.z;
            qv[4 * c + 3] = v.w;
        }
        tmem_st32(tmem_base + ((uint32_t)(quarter * 32) << 16) + kColQ + hf * 32, qv);
        tmem_wait_st();
        tc_fence_before();
        named_barrier_sync(kQBarrier, kQThreads);
    } else if (warp == 1) {
        named_barrier_sync(kQBarrier, kQThreads);
        tc_fence_after();
    }

    if (warp == 0 || warp == kVWarp) {
        // ---------------- TMA producers: K (warp 0) and V (the last warp) ----------------
        // Separate producers let K run ahead of the V ring, whose slots free
        // only after the softmax and P V of their stage.
        const bool is_k = warp == 0;
        const int nst = is_k ? kKStages : kVStages;
        uint64_t* fullb = is_k ? kfull : vfull;
        uint64_t* emptyb = is_k ? kempty : vempty;
        const CUtensorMap* tm = is_k ? &tm_k : &tm_v;
        unsigned char* ring = smem + (is_k ? kOffK : kOffV);
        if (lane == 0) {
            for (int i = 0; i < nstages; ++i) {
                const int st = i % nst;
                int ys[2];
                int nload = 0;
                for (int c = 0; c < 2; ++c) {
                    const int u = 2 * i + c;
                    ys[c] = -1;
                    if (u < nunits) {
                        const int blk = u / upb, sub = u - blk * upb;
                        const int page = upage[blk];
                        if (page >= 0) {
                            ys[c] = (page * H_kv + g) * bs + sub * 64;
                            ++nload;
                        }
                    }
                }
                const uint32_t bytes = (uint32_t)nload * 2u * 8192u;
                if (*s_abort) break;
                if (i >= nst && !mbar_wait(&emptyb[st], ((i / nst) - 1) & 1)) {
                    *s_abort = 1;
                    break;
                }
                unsigned char* dst = ring + st * kTileBytes;
                if (bytes) {
                    mbar_arrive_expect_tx(&fullb[st], bytes);
                    for (int c = 0; c < 2; ++c)
                        if (ys[c] >= 0) {
                            tma_load_2d(dst + c * 8192, tm, 0, ys[c], &fullb[st]);
                            tma_load_2d(dst + kHalf + c * 8192, tm, 64, ys[c], &fullb[st]);
                        }
                } else {
                    mbar_arrive(&fullb[st]);
                }
            }
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer ----------------
        if (lane == 0) {
            auto pv = [&](int j) -> bool {
                const int vs = j % kVStages;
                if (!mbar_wait(&pfull[j & 1], (j >> 1) & 1) ||
                    !mbar_wait(&vfull[vs], (j / kVStages) & 1)) {
                    *s_abort = 1;
                    return false;
                }
                tc_fence_after();
                const uint32_t vb = smem_u32(smem + kOffV + vs * kTileBytes);
#pragma unroll
                for (int kt = 0; kt < kStageTok / 16; ++kt)  // 16 tokens per MMA
                    tc_mma_tmem_a(tmem_base + kColO, tmem_base + kColS + (j & 1) * 128 + kt * 8,
                                  sw128_desc_mn(vb + kt * 2048, kHalf), kIdescPV,
                                  (j > 0 || kt > 0) ? 1u : 0u);
                tc_commit(&vempty[vs]);
                tc_commit(obar);
                return true;
            };
            bool fine = true;
            for (int i = 0; i < nstages && fine; ++i) {
                const int ks = i % kKStages;
                if (*s_abort || !mbar_wait(&kfull[ks], (i / kKStages) & 1)) {
                    *s_abort = 1;
                    fine = false;
                    break;
                }
                tc_fence_after();
                const uint32_t kb = smem_u32(smem + kOffK + ks * kTileBytes);
                const uint32_t d = tmem_base + kColS + (i & 1) * 128;
#pragma unroll
                for (int kk = 0; kk < kHD / 16; ++kk) {  // 16 dims per MMA
                    const uint32_t off = (kk >> 2) * kHalf;
                    tc_mma_tmem_a(d, tmem_base + kColQ + kk * 8, sw128_desc(kb + off) + 2 * (kk & 3),
                                  kIdescQK, kk > 0 ? 1u : 0u);
                }
                tc_commit(&kempty[ks]);
                tc_commit(&sfull[i & 1]);
                if (i > 0) fine = pv(i - 1);
            }
            if (fine && nstages > 0 && pv(nstages - 1)) tc_commit(ofin);
            // nothing of this thread may still run on the tensor core when the
            // TMEM is released
            tc_commit(drain);
            mbar_wait(drain, 0);
        }
    } else {
        // ---------------- softmax and epilogue: two threads per MMA row ----------------
        // Thread (r, hf) owns row r's tokens of unit slot hf (stage columns
        // 64*hf .. 64*hf+63) and output dims 64*hf .. 64*hf+63. The two halves
        // of a row agree on its maximum through shared memory and a named
        // barrier of their two warps (ids 1..4, one per TMEM lane quarter).
        const int quarter = warp & 3;
        const int hf = (warp - 2) >> 2;
        const int r = quarter * 32 + lane;
        const int bar_id = 1 + quarter;
        const int qi = r / G, s = s0 + qi;
        const long long p = (long long)q_start[b] + s;
        const long long last = s < S ? (p < ctx - 1 ? p : ctx - 1) : -1;
        // 32-bit copies for the per-stage tests (token positions fit 31 bits)
        const int last32 = (int)(last < 0x7fffffffLL ? last : 0x7fffffffLL);
        const int ctx32 = (int)(ctx < 0x7fffffffLL ? ctx : 0x7fffffffLL);
        const uint32_t qbit = 1u << qi;
        const uint32_t lane_addr = tmem_base + ((uint32_t)(quarter * 32) << 16);
        float* xchg = reinterpret_cast<float*>(smem + kOffXchg);  // [3][2][128]
        int* xok = reinterpret_cast<int*>(xchg + 3 * 2 * 128);      // [2][2][128]
        float m_ref = -INFINITY;  // reference maximum (log2 units), the same in both halves
        float l = 0.f;            // this half's share of the row sum
        // The stage's two 64-token units (c = 0, 1) come from the union
        // entries (page, block, query mask) of blocks nb and nb + 1, loaded one
        // stage ahead so that their shared-memory latency hides behind the
        // previous stage; (nb, nsub) walk the units in order without a division
        // by the units per block. Token positions fit 31 bits (nb_max * bs <
        // 2^31); an entry past the union is read (in bounds) but not used.
        int nb = 0, nsub = 0;
        int pg0, bl0, pg1, bl1;
        uint32_t mk0, mk1;
        auto fetch = [&]() {
            const int b0 = min(nb, kMaxUnion - 1), b1 = min(nb + 1, kMaxUnion - 1);
            pg0 = upage[b0];
            bl0 = ublk[b0];
            mk0 = umask[b0];
            pg1 = upage[b1];
            bl1 = ublk[b1];
            mk1 = umask[b1];
        };
        fetch();
        for (int i = 0; i < nstages; ++i) {
            // each unit's first token (-1: past the union or an absent page)
            const bool same = nsub + 1 < upb;  // unit 1 in the same block as unit 0
            const int pgb = same ? pg0 : pg1, blb = same ? bl0 : bl1;
            const uint32_t mkb = same ? mk0 : mk1;
            const int ut0a = 2 * i < nunits && pg0 >= 0 ? bl0 * bs + nsub * 64 : -1;
            const int ut0b = 2 * i + 1 < nunits && pgb >= 0 ? blb * bs + (same ? nsub + 1 : 0) * 64 : -1;
            // this half's unit: whether the row takes it, and how many of its
            // 64 tokens the row may see
            const int t0 = hf ? ut0b : ut0a;
            int nval = 0;
            if (t0 >= 0 && ((hf ? mkb : mk0) & qbit) != 0u && t0 <= last32)
                nval = last32 - t0 >= 63 ? 64 : last32 - t0 + 1;
            nsub += 2;
            while (nsub >= upb) {
                nsub -= upb;
                ++nb;
            }
            fetch();  // the next stage's entries
            const bool waited = mbar_wait(&sfull[i & 1], (i >> 1) & 1);
            const int my_ok = waited && !*s_abort;
            tc_fence_after();
            uint32_t sv[64];
            float mx = -INFINITY;
            const bool warp_any = __any_sync(0xffffffffu, nval > 0);
            if (warp_any) {
                tmem_ld64(lane_addr + kColS + (i & 1) * 128 + hf * 64, sv);
                if (nval < 64) {
#pragma unroll
                    for (int e = 0; e < 64; ++e)
                        sv[e] = e < nval ? sv[e] : __float_as_uint(-INFINITY);
                }
                // eight independent running maxima, two new values per
                // three-input max, then a tree
                float pm[8];
#pragma unroll
                for (int k = 0; k < 8; ++k) pm[k] = __uint_as_float(sv[k]);
#pragma unroll
                for (int e = 8; e < 64; e += 2)
                    pm[(e >> 1) & 7] = fmax3(pm[(e >> 1) & 7], __uint_as_float(sv[e]),
                                             __uint_as_float(sv[e + 1]));
                mx = fmax3(fmax3(pm[0], pm[1], pm[2]), fmax3(pm[3], pm[4], pm[5]),
                           fmaxf(pm[6], pm[7]));
            }
            // the row maximum of the stage (raw scores; the scale is positive),
            // and whether both halves may go on: one decision for the pair of
            // warps, so their named barriers always match
            float* xm = xchg + (i & 1) * 256;
            int* xo = xok + (i & 1) * 256;
            xm[hf * 128 + r] = mx;
            xo[hf * 128 + r] = my_ok;
            tc_fence_before();  // this half's S loads are ordered before the partner's P stores
            named_barrier_sync(bar_id, 64);
            tc_fence_after();
            if (!__all_sync(0xffffffffu, my_ok && xo[(hf ^ 1) * 128 + r])) {
                *s_abort = 1;
                break;
            }
            const float mrow = fmaxf(mx, xm[(hf ^ 1) * 128 + r]) * scale_log2;
            // lazy reference: move m only when the stage's maximum passes m + 8
            float corr = 1.f;
            if (mrow > m_ref + kLazy) {
                corr = m_ref > -INFINITY ? fast_exp2(m_ref - mrow) : 1.f;
                m_ref = mrow;
            }
            // P = 2^(s*c - m) as bf16 pairs; it overwrites the S buffer's first
            // 64 columns (both halves have read their S columns: the barrier above)
            const float neg_m = -m_ref;
            uint32_t pk[32];
            if (nval > 0) {
                // the scale and shift, and the row sum, on packed fp32 pairs:
                // one instruction for two tokens
                const float2 sc2 = make_float2(scale_log2, scale_log2);
                const float2 nm2 = make_float2(neg_m, neg_m);
                float2 ps[4];
#pragma unroll
                for (int k = 0; k < 4; ++k) ps[k] = make_float2(0.f, 0.f);
#pragma unroll
                for (int e = 0; e < 32; ++e) {
                    // masked entries hold -inf: 2^-inf = 0
                    const float2 x = ffma2(
                        make_float2(__uint_as_float(sv[2 * e]), __uint_as_float(sv[2 * e + 1])), sc2, nm2);
                    const float2 pe = make_float2(fast_exp2(x.x), fast_exp2(x.y));
                    ps[e & 3] = fadd2(ps[e & 3], pe);
                    pk[e] = pack_bf16x2(pe.x, pe.y);
                }
                const float2 s01 = fadd2(ps[0], ps[1]), s23 = fadd2(ps[2], ps[3]);
                const float2 st = fadd2(s01, s23);
                l = fmaf(l, corr, st.x + st.y);
            } else {
#pragma unroll
                for (int e = 0; e < 32; ++e) pk[e] = 0u;
                l *= corr;
            }
            tmem_st32(lane_addr + kColS + (i & 1) * 128 + hf * 32, pk);
            if (__any_sync(0xffffffffu, corr != 1.f)) {
                // O holds earlier stages of this row: rescale this half's
                // columns once the previous P V has landed (after P, so that
                // the S registers are free and the wait comes as late as it can)
                if (!mbar_wait(obar, (i - 1) & 1)) *s_abort = 1;
                tc_fence_after();
#pragma unroll 1  // one 32-column chunk in registers at a time
                for (int ch = 0; ch < 2; ++ch) {
                    uint32_t ov[32];
                    tmem_ld32(lane_addr + kColO + hf * 64 + ch * 32, ov);
#pragma unroll
                    for (int e = 0; e < 32; ++e) ov[e] = __float_as_uint(__uint_as_float(ov[e]) * corr);
                    tmem_st32(lane_addr + kColO + hf * 64 + ch * 32, ov);
                }
            }
            tmem_wait_st();
            // V rows of an absent unit and of tokens past the context length
            // must be zero before the P V MMA reads them (this thread: token row
            // r of the stage, dims 64*hf .. 64*hf+63)
            const bool stage_tail =  // the same for every thread
                ut0a < 0 || ut0b < 0 || ut0a > ctx32 - 64 || ut0b > ctx32 - 64;
            if (stage_tail) {
                const int vs = i % kVStages;
                if (!mbar_wait(&vfull[vs], (i / kVStages) & 1)) *s_abort = 1;
                const int mine_t0 = (r >> 6) ? ut0b : ut0a;
                if (mine_t0 < 0 || mine_t0 + (r & 63) >= ctx32) {
                    unsigned char* vt = smem + kOffV + vs * kTileBytes;
#pragma unroll
                    for (int cc = 8 * hf; cc < 8 * hf + 8; ++cc)
                        *reinterpret_cast<uint4*>(vt + pfa_off(r, cc)) = make_uint4(0, 0, 0, 0);
                }
                fence_proxy_async_smem();
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&pfull[i & 1]);
        }
        // ---------------- epilogue: O / l -> bf16 ----------------
        float* xl = xchg + 2 * 256;
        xl[hf * 128 + r] = l;
        named_barrier_sync(bar_id, 64);
        const float ltot = l + xl[(hf ^ 1) * 128 + r];
        if (nstages > 0 && !*s_abort) {
            if (!mbar_wait(ofin, 0)) *s_abort = 1;
            tc_fence_after();
        }
        const float inv = ltot > 0.f ? 1.f / ltot : 0.f;
        // log2-sum-exp2 of the scaled logits, for combining partial results
        if (lse != nullptr && s < S && hf == 0)
            lse[((size_t)b * S + s) * H_q + (size_t)g * G + (r - qi * G)] =
                ltot > 0.f ? m_ref + __log2f(ltot) : -INFINITY;
        __nv_bfloat16* orow = out + (((size_t)b * S + s) * H_q + (size_t)g * G + (r - qi * G)) * kHD;
#pragma unroll
        for (int ch = 0; ch < 2; ++ch) {
            uint32_t ov[32];
            if (nstages > 0) {
                tmem_ld32(lane_addr + kColO + hf * 64 + ch * 32, ov);
            } else {
#pragma unroll
                for (int e = 0; e < 32; ++e) ov[e] = 0u;
            }
            if (s < S) {
                uint32_t pk[16];
#pragma unroll
                for (int e = 0; e < 16; ++e)
                    pk[e] = pack_bf16x2(__uint_as_float(ov[2 * e]) * inv,
                                        __uint_as_float(ov[2 * e + 1]) * inv);
                uint4* dst = reinterpret_cast<uint4*>(orow + hf * 64 + ch * 32);
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    dst[e] = make_uint4(pk[4 * e], pk[4 * e + 1], pk[4 * e + 2], pk[4 * e + 3]);
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
