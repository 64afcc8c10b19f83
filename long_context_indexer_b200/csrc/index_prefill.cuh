// index_prefill.cuh -- block scoring fused with the causal-masked top-k on the
// 5th-generation tensor cores (tcgen05 + TMEM), for many queries per sequence.
//
// score[s, j] = q_c[s, :] . k_c[j, :] is a dense [S x NB] GEMM over
// K = H_i * d_c ([AI-acc] §4.1, matmul of compressed queries and keys). Each
// CTA owns a 128-query m-tile and a range of 256-block n-tiles:
//
//   warp 0      TMA producer: 64-wide K slices of q_c (128 rows) and k_c
//               (256 rows), 128-byte swizzle, into a 4-stage ring;
//   warp 1      one thread issues tcgen05.mma (M=128, N=256, K=16, bf16 ->
//               fp32) into one of two TMEM accumulators (2 x 256 columns) and
//               commits stage releases / accumulator-ready signals;
//   warps 2..   epilogue (4 warps, or 8 for k <= 32): a thread owns one query
//               row (TMEM lane) and, with two warps per lane quarter, every
//               other 32-column group of each tile. It reads 32 scores per
//               tcgen05.ld, drops blocks that are not causal-visible, appends
//               the scores above its threshold to a shared-memory buffer, and
//               inserts the buffer into a running exact top-k in registers
//               when some lane's buffer nears full. Scores never reach global
//               memory ([GPU-stack] "Operatorizing Index Selection": scoring,
//               top-k and masking fused in one pass).
//
// Every list (a row's part inside one CTA) publishes its k-th best key to a
// per-row bound in the workspace (atomicMax) and filters against the best bound
// any list of the row has published: a list's k-th best is a lower bound on the
// row's final k-th best, so a score below the bound cannot be selected. As the
// lists of a row grow at the same time, the bound runs only a little ahead of
// each list's own threshold.
//
// n-tiles beyond the last visible block of the m-tile are skipped. An m-tile
// may be split over several CTAs: by n-tiles, or, when it has a single n-tile,
// by windows of that tile's visible columns. Each CTA then writes its per-row
// candidates (key, id) to the workspace and the last CTA to arrive (atomic
// counter, no spin-wait) merges them. Ties break to the lower block id.
#pragma once

#include "common.cuh"
#include "ptx.cuh"

namespace lci {

namespace pre {
constexpr int kBM = 128, kBN = 256, kBK = 64;
constexpr int kStages = 4;
constexpr int kChunk = 8;                // columns between checks of the candidate buffers
constexpr int kABytes = kBM * kBK * 2;   // 16 KiB
constexpr int kBBytes = kBN * kBK * 2;   // 32 KiB
constexpr int kStageBytes = kABytes + kBBytes;
constexpr int kTmemCols = 2 * kBN;       // two accumulators
constexpr int kCandBytes = 32 * 1024;            // per-thread candidate buffers (score, id)
static_assert(64 * kBM * 4 <= kCandBytes, "the staged output rows (topk <= 64) fit the candidate area");
constexpr int kSmemBytes = kStages * kStageBytes + kCandBytes + 1024 /*align*/ + 256 /*barriers*/;
// Epilogue warps: kParts per TMEM lane quarter, each taking every kParts-th
// 32-column group of every tile with its own list. More parts hide more
// latency; the register budget (65536 / threads) bounds them by the list
// length KT.
template <int KT> struct Epi { static constexpr int kParts = KT <= 32 ? 2 : 1; };
template <int KT> struct Cfg { static constexpr int kThreads = 64 + 128 * Epi<KT>::kParts; };
// instruction descriptor: D fp32, A/B bf16, both K-major, M = 128, N = n (a
// multiple of 16 up to 256: the first n rows of the B tile)
__host__ __device__ constexpr uint32_t idesc_n(int n) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(n >> 3) << 17) |
           ((uint32_t)(kBM >> 4) << 24);
}
}  // namespace pre

// Shared-memory matrix descriptor of a K-major tile written by TMA with the
// 128-byte swizzle: 8-row groups 1024 bytes apart, sm_100 descriptor version.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t smem_addr) {
    return (uint64_t)((smem_addr >> 4) & 0x3fff) | ((uint64_t)1 << 16) /* LBO (unused) */ |
           ((uint64_t)(1024 >> 4) << 32) /* SBO */ | ((uint64_t)1 << 46) /* version */ |
           ((uint64_t)2 << 61) /* SWIZZLE_128B */;
}

__device__ __forceinline__ void tc_mma(uint32_t tmem_d, uint64_t a, uint64_t b, uint32_t idesc,
                                       uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
        "l"(a), "l"(b), "r"(idesc), "r"(accumulate));
}

__device__ __forceinline__ void tc_commit(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     smem_u32(bar))
                 : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// 32 consecutive fp32 columns of this thread's TMEM lane.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,"
        "%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
          "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
          "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
          "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;"
                 : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]),
                   "+r"(r[6]), "+r"(r[7]), "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]),
                   "+r"(r[12]), "+r"(r[13]), "+r"(r[14]), "+r"(r[15]), "+r"(r[16]), "+r"(r[17]),
                   "+r"(r[18]), "+r"(r[19]), "+r"(r[20]), "+r"(r[21]), "+r"(r[22]), "+r"(r[23]),
                   "+r"(r[24]), "+r"(r[25]), "+r"(r[26]), "+r"(r[27]), "+r"(r[28]), "+r"(r[29]),
                   "+r"(r[30]), "+r"(r[31])
                 :
                 : "memory");
}

// Running top-KT of one row, sorted by key descending, in registers. Entries
// start as (key 0, id -1), below every real key. A new element with a key equal
// to an entry comes later in block order, so it ranks behind it: it enters
// only when its key is strictly above the last entry. The insertion is a
// shift network: every position updates from its own and its predecessor's
// old values, so the KT updates are independent of one another.
template <int KT>
struct RowTopK {
    uint32_t key[KT];
    int32_t id[KT];
    __device__ __forceinline__ void init() {
#pragma unroll
        for (int i = 0; i < KT; ++i) {
            key[i] = 0u;
            id[i] = -1;
        }
        thr_f = -INFINITY;
    }
    float thr_f;  // score of the last entry once the list is full
    __device__ __forceinline__ uint32_t threshold() const { return key[KT - 1]; }
    __device__ __forceinline__ bool full() const { return id[KT - 1] >= 0; }
    __device__ __forceinline__ void insert(uint32_t k, int32_t j) {
        // c[i]: the new key beats entry i. Keys move with unsigned min/max
        // (the list is sorted), ids follow the same decisions.
        bool c[KT];
#pragma unroll
        for (int i = 0; i < KT; ++i) c[i] = k > key[i];
#pragma unroll
        for (int i = KT - 1; i > 0; --i) {
            id[i] = c[i - 1] ? id[i - 1] : (c[i] ? j : id[i]);
            key[i] = min(key[i - 1], max(k, key[i]));
        }
        id[0] = c[0] ? j : id[0];
        key[0] = max(k, key[0]);
        // back from key to score: the inverse of score_key
        const uint32_t w = key[KT - 1];
        thr_f = __uint_as_float((w & 0x80000000u) ? (w & 0x7fffffffu) : ~w);
    }
};

// The score of a nonzero key (the inverse of score_key).
__device__ __forceinline__ float key_score(uint32_t w) {
    return __uint_as_float((w & 0x80000000u) ? (w & 0x7fffffffu) : ~w);
}
// The largest float below a finite x: "s > below(x)" is "s >= x" for finite s
// (with -0.0 == +0.0).
__device__ __forceinline__ float float_below(float x) {
    if (x == 0.f) return __uint_as_float(0x80000001u);
    const uint32_t u = __float_as_uint(x);
    return __uint_as_float(x > 0.f ? u - 1u : u + 1u);
}

// Best of N composites c[base .. base+N) by a tournament (depth log2 N):
// the winner's value and index.
template <int N> struct Tournament {
    static __device__ __forceinline__ void run(const uint64_t* c, int base, uint64_t& best,
                                               int& at) {
        uint64_t c1;
        int a1;
        Tournament<N / 2>::run(c, base, best, at);
        Tournament<N - N / 2>::run(c, base + N / 2, c1, a1);
        const bool t = c1 > best;
        best = t ? c1 : best;
        at = t ? a1 : at;
    }
};
template <> struct Tournament<1> {
    static __device__ __forceinline__ void run(const uint64_t* c, int base, uint64_t& best,
                                               int& at) {
        best = c[base];
        at = base;
    }
};

// k-way merge of one row's NS sorted lists into its best `nout` entries. The
// lists sit in shared memory from (shared-window) addresses keys / ids: entry
// (list q, rank h) at byte offset q * list_bytes + h * pre::kBM * 4, each list
// `len` long. An entry's composite (key << 32 | ~id) orders key desc then id
// asc, and an empty entry (key 0, id -1) composes to 0, below every real one;
// emit(i, composite) receives output rank i (an empty one as 0). Each list's
// head entry is held in a register, so a step is one tournament and one
// refill of the winner's list.
template <int NS, typename Emit>
__device__ __forceinline__ void merge_sorted_lists(uint32_t keys, uint32_t ids,
                                                   uint32_t list_bytes, int len, int nout,
                                                   Emit emit) {
    constexpr uint32_t kRank = pre::kBM * 4;
    uint64_t cur[NS];
    int head[NS];
#pragma unroll
    for (int q = 0; q < NS; ++q) {
        head[q] = 0;
        const uint32_t off = (uint32_t)q * list_bytes;
        cur[q] = ((uint64_t)lds32(keys + off) << 32) | (uint32_t)~lds32(ids + off);
    }
    for (int i = 0; i < nout; ++i) {
        uint64_t bc;
        int best;
        Tournament<NS>::run(cur, 0, bc, best);
        emit(i, bc);
        int h = 0;
#pragma unroll
        for (int q = 0; q < NS; ++q) h = q == best ? head[q] : h;
        ++h;  // the winner's next entry (an exhausted list stays at composite 0)
        const uint32_t off = (uint32_t)best * list_bytes + (uint32_t)min(h, len - 1) * kRank;
        const uint64_t next =
            h < len ? ((uint64_t)lds32(keys + off) << 32) | (uint32_t)~lds32(ids + off) : 0ull;
#pragma unroll
        for (int q = 0; q < NS; ++q) {
            head[q] = q == best ? h : head[q];
            cur[q] = q == best ? next : cur[q];
        }
    }
}

template <int KT>
__global__ void __launch_bounds__(pre::Cfg<KT>::kThreads, 1) index_prefill_tc_kernel(
    const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k, int S,
    int nb_max, int bs, const int32_t* __restrict__ ctx_len, const int32_t* __restrict__ q_start,
    int topk, int ksteps, int m_tiles, int n_split, uint32_t* __restrict__ part_key,
    int32_t* __restrict__ part_id, unsigned int* __restrict__ counters,
    unsigned int* __restrict__ row_bound, int32_t* __restrict__ ids) {
    using namespace pre;
    constexpr int kParts = Epi<KT>::kParts;        // epilogue warps per TMEM lane quarter
    constexpr int kEW = 4 * kParts;                // epilogue warps
    constexpr int kGroup = 32;                    // TMEM columns per load
    constexpr int kGroupsPerPart = kBN / kGroup / kParts;
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char* smem = reinterpret_cast<unsigned char*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint32_t* cand = reinterpret_cast<uint32_t*>(smem + kStages * kStageBytes);  // [32][kBM] keys, then ids
    uint64_t* full_bar = reinterpret_cast<uint64_t*>(smem + kStages * kStageBytes + kCandBytes);
    uint64_t* empty_bar = full_bar + kStages;
    uint64_t* tfull_bar = empty_bar + kStages;
    uint64_t* tempty_bar = tfull_bar + 2;
    uint64_t* merge_bar = tempty_bar + 2;    // the split lists' bulk copies
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(merge_bar + 1);
    int* s_last = reinterpret_cast<int*>(tmem_slot + 1);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int ns = blockIdx.x, mt = blockIdx.y, b = blockIdx.z;
    const int row0 = mt * kBM;

    // Visible n-tiles of this m-tile (causal), and this CTA's share of them.
    const long long ctx = ctx_len[b];
    const long long p_last = (long long)q_start[b] + min(S - 1, row0 + kBM - 1);
    const int vis_max = visible_blocks(p_last, ctx, bs, nb_max);
    const int n_tiles = (vis_max + kBN - 1) / kBN;
    // Several n-tiles: the CTAs of the m-tile split them. One n-tile: every
    // CTA computes it and takes a window [c_lo, c_hi) of its visible columns
    // (whole 32-column groups) into its list.
    int t_lo = 0, t_hi = 0, c_lo = 0, c_hi = kBN;
    if (n_tiles == 1 && n_split > 1) {
        const int cols = ((vis_max + n_split - 1) / n_split + 31) & ~31;
        c_lo = ns * cols;
        c_hi = min(kBN, c_lo + cols);
        t_hi = c_lo < vis_max ? 1 : 0;
    } else {
        const int per = (n_tiles + n_split - 1) / n_split;
        t_lo = ns * per;
        t_hi = min(n_tiles, t_lo + per);
    }
    const int my_tiles = max(0, t_hi - t_lo);

    if (tid == 0) {
        for (int i = 0; i < kStages; ++i) {
            mbar_init(&full_bar[i], 1);
            mbar_init(&empty_bar[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&tfull_bar[i], 1);
            mbar_init(&tempty_bar[i], kEW);  // one arrive per epilogue warp
        }
        mbar_init(merge_bar, 1);
        fence_mbar_init();
    }
    if (warp == 1) {  // the whole warp allocates the two accumulators
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32(tmem_slot)),
                     "r"(kTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    if (warp == 0 && lane == 0) {
        prefetch_tensormap(&tm_q);
        prefetch_tensormap(&tm_k);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    // The m-tile's output rows are staged in the candidate area once the
    // epilogue is done with it, entry (rank i, row r) at out_slot(i, r): the
    // row index XOR the rank keeps both the per-row writes (32 rows, one
    // rank) and the row-major copy-out (one row, consecutive ranks) free of
    // bank conflicts. The copy-out then writes the tile's contiguous
    // rows x topk ids with coalesced stores.
    int32_t* out_s = reinterpret_cast<int32_t*>(cand);
    auto out_slot = [&](int i, int r) { return i * kBM + (r ^ (i & 31)); };
    auto store_rows = [&](int t0, int nt) {
        const int n = min(kBM, S - row0) * topk;
        int32_t* dst = ids + ((size_t)b * S + row0) * topk;
        // entry j is (row j / topk, rank j % topk), stepped without a division
        const int drow = nt / topk, drank = nt - drow * topk;
        int rr = t0 / topk, i = t0 - rr * topk;
        for (int j = t0; j < n; j += nt) {
            dst[j] = out_s[out_slot(i, rr)];
            rr += drow;
            i += drank;
            if (i >= topk) {
                i -= topk;
                ++rr;
            }
        }
    };

    if (warp == 0) {
        // ---------------- TMA producer ----------------
        if (lane == 0) {
            int it = 0;
            for (int t = 0; t < my_tiles; ++t) {
                const int n0 = (t_lo + t) * kBN;
                for (int ks = 0; ks < ksteps; ++ks, ++it) {
                    const int st = it % kStages;
                    if (it >= kStages && !mbar_wait(&empty_bar[st], ((it / kStages) - 1) & 1)) break;
                    unsigned char* a = smem + st * kStageBytes;
                    mbar_arrive_expect_tx(&full_bar[st], kStageBytes);
                    tma_load_2d(a, &tm_q, ks * kBK, b * S + row0, &full_bar[st]);
                    tma_load_2d(a + kABytes, &tm_k, ks * kBK, b * nb_max + n0, &full_bar[st]);
                }
            }
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer ----------------
        if (lane == 0) {
            int it = 0;
            bool ok = true;
            for (int t = 0; t < my_tiles && ok; ++t) {
                const int buf = t & 1;
                if (t >= 2) ok = mbar_wait(&tempty_bar[buf], ((t >> 1) - 1) & 1);
                tc_fence_after();
                const uint32_t d = tmem_base + (uint32_t)(buf * kBN);
                // only the tile's visible columns (and none past the CTA's
                // window): the epilogue never reads the others
                const int ncols = min(min(kBN, vis_max - (t_lo + t) * kBN), c_hi);
                const uint32_t idesc = idesc_n(max(16, (ncols + 15) & ~15));
                for (int ks = 0; ks < ksteps && ok; ++ks, ++it) {
                    const int st = it % kStages;
                    ok = mbar_wait(&full_bar[st], (it / kStages) & 1);
                    tc_fence_after();
                    const uint32_t a = smem_u32(smem + st * kStageBytes);
                    const uint64_t ad = sw128_desc(a), bd = sw128_desc(a + kABytes);
#pragma unroll
                    for (int kk = 0; kk < kBK / 16; ++kk)  // +32 bytes per K=16 step
                        tc_mma(d, ad + 2 * kk, bd + 2 * kk, idesc, (ks | kk) != 0);
                    tc_commit(&empty_bar[st]);  // the stage is free once these MMAs finish
                }
                tc_commit(&tfull_bar[buf]);  // accumulator ready
            }
        }
    } else {
        // ---------------- epilogue: kParts threads per query row ----------------
        const int ew = warp - 2;                // 0 .. kEW-1
        const int quarter = warp & 3;           // TMEM lanes 32*quarter .. +31
        const int part = ew >> 2;               // which chunks of every tile
        const int r = quarter * 32 + lane;
        const int s = row0 + r;
        const long long p = (long long)q_start[b] + s;
        const int vis = s < S ? visible_blocks(p, ctx, bs, nb_max) : 0;
        const int et = ew * 32 + lane;          // epilogue thread index
        // Candidates that beat the threshold are appended to this
        // thread's buffer (entry q at cbuf[q * kEpiThreads]); the insertion
        // network runs only when some lane's buffer is about to fill. A warp
        // then pays for the network once per buffered candidate of its busiest
        // lane, instead of once per chunk in which any of its 32 rows passed.
        constexpr int kEpiThreads = 32 * kEW;
        constexpr int kBuf = kCandBytes / (8 * kEpiThreads);
        static_assert(kBuf >= 2 * kChunk, "candidate buffer too small");
        uint2* cbuf = reinterpret_cast<uint2*>(cand) + et;
        int nc = 0;
        RowTopK<KT> top;
        top.init();
        // the row's shared bound: gk is the best key seen (own or published),
        // gthr the float filter it implies (-inf while there is none)
        unsigned int* bound = s < S ? row_bound + (size_t)b * S + s : nullptr;
        uint32_t gk = 0u;
        float gthr = -INFINITY;
        auto flush = [&]() {
            // Branch-free: a lane past its own candidates inserts key 0, and a
            // key at or below the list's last entry changes nothing either
            // (the network moves an entry only for a strictly larger key).
            const int m = __reduce_max_sync(0xffffffffu, nc);
            uint2 e = cbuf[0];
            for (int q = 0; q < m; ++q) {
                const uint2 next = cbuf[min(q + 1, kBuf - 1) * kEpiThreads];  // loaded ahead
                top.insert(q < nc ? score_key(__uint_as_float(e.x)) : 0u, (int32_t)e.y);
                e = next;
            }
            nc = 0;
            if (top.full() && top.threshold() > gk && bound != nullptr) {
                gk = top.threshold();
                gthr = fmaxf(gthr, float_below(key_score(gk)));
                atomicMax(bound, gk);
            }
        };
        // this part's groups c (columns (c * kParts + part) * kGroup ..) inside
        // the CTA's column window: c_begin <= c < c_end
        const int c_begin = (c_lo / kGroup - part + kParts - 1) / kParts;
        const int c_end = (c_hi / kGroup - part + kParts - 1) / kParts;
        for (int t = 0; t < my_tiles; ++t) {
            const int buf = t & 1;
            const bool ok = mbar_wait(&tfull_bar[buf], (t >> 1) & 1);
            tc_fence_after();
            const int n0 = (t_lo + t) * kBN;
            if (ok) {
                const uint32_t lane_base =
                    tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(buf * kBN);
                if (t == 0 && c_hi == kBN && __all_sync(0xffffffffu, n0 + kBN <= vis)) {
                    // First tile, empty list, every column visible to the warp's
                    // rows (and computed: no column window): a lower bound of this part's KT-th
                    // best score from the tile itself. Its columns fall into KT
                    // runs of kSub; every run's maximum is a score of the part, so
                    // with L the smallest run maximum, KT scores are >= L and a
                    // score below L never enters the list.
                    constexpr int kSub = kBN / kParts / KT;
                    static_assert(kSub >= 1 && kGroup % kSub == 0, "runs tile a group");
                    float lmin = INFINITY;
#pragma unroll 1
                    for (int c = 0; c < kGroupsPerPart; ++c) {
                        const int col = (c * kParts + part) * kGroup;
                        uint32_t raw[kGroup];
                        __syncwarp();
                        tmem_ld32(lane_base + (uint32_t)col, raw);
#pragma unroll
                        for (int g0 = 0; g0 < kGroup; g0 += kSub) {
                            float mrun = -INFINITY;
#pragma unroll
                            for (int i = 0; i < kSub; ++i)
                                if (n0 + col + g0 + i < vis) mrun = fmaxf(mrun, __uint_as_float(raw[g0 + i]));
                            lmin = fminf(lmin, mrun);
                        }
                    }
                    if (lmin > -INFINITY && lmin < INFINITY) gthr = fmaxf(gthr, float_below(lmin));
                }
#pragma unroll 1
                for (int c = c_begin; c < c_end; ++c) {
                    const int col = (c * kParts + part) * kGroup;  // parts interleave groups
                    // the row's bound as published so far, used from the next group on
                    const uint32_t gk_next = bound != nullptr ? ld_relaxed_gpu(bound) : 0u;
                    uint32_t raw[kGroup];
                    __syncwarp();  // reconverge before the warp-collective TMEM load
                    tmem_ld32(lane_base + (uint32_t)col, raw);
#pragma unroll
                    for (int sc = 0; sc < kGroup / kChunk; ++sc) {
                        const int jb = n0 + col + sc * kChunk;
                        if (jb < vis) {
                            // exact order test on the raw fp32 scores (finite, and
                            // -0.0 == +0.0); equal scores come later in block order
                            // and so never enter a full list
                            const float thr = fmaxf(top.full() ? top.thr_f : -INFINITY, gthr);
#pragma unroll
                            for (int i = 0; i < kChunk; ++i) {
                                // a store only for a passing score: shared-memory
                                // bandwidth is shared with the TMA writes and the
                                // MMA operand reads
                                const uint32_t v = raw[sc * kChunk + i];
                                if ((jb + i < vis) && __uint_as_float(v) > thr) {
                                    cbuf[nc * kEpiThreads] = make_uint2(v, (uint32_t)(jb + i));
                                    ++nc;
                                }
                            }
                        }
                        __syncwarp();
                        if (__any_sync(0xffffffffu, nc > kBuf - kChunk)) flush();
                    }
                    if (gk_next > gk) {
                        gk = gk_next;
                        gthr = fmaxf(gthr, float_below(key_score(gk)));
                    }
                }
                __syncwarp();
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&tempty_bar[buf]);
        }
        flush();
        // ---------------- merge the parts, write in rank order ----------------
        // (the stage memory is idle: every MMA and copy has completed)
        uint32_t* xk = reinterpret_cast<uint32_t*>(smem);                  // [part][i][row]
        int32_t* xi = reinterpret_cast<int32_t*>(smem) + kParts * KT * kBM;
#pragma unroll
        for (int i = 0; i < KT; ++i) {
            xk[(part * KT + i) * kBM + r] = top.key[i];
            xi[(part * KT + i) * kBM + r] = top.id[i];
        }
        named_barrier_sync(1, 32 * kEW);
        // every list of the row is final: with one CTA per row range the bound
        // is reset here, otherwise by the CTA that merges the splits
        if (n_split == 1 && part == 0 && bound != nullptr) *bound = 0u;
        if (part == 0) {
            // split lists of the m-tile: [split][rank][row], rows fastest (the
            // stores of a warp are contiguous, and so are the merge's reads)
            const size_t pbase = (((size_t)b * m_tiles + mt) * n_split + ns) * topk * kBM + r;
            const uint32_t ko = smem_u32(out_s);
            auto emit = [&](int i, uint64_t c) {
                if (n_split == 1) {
                    sts32(ko + 4u * (uint32_t)out_slot(i, r), ~(uint32_t)c);
                } else {
                    part_key[pbase + (size_t)i * kBM] = (uint32_t)(c >> 32);
                    part_id[pbase + (size_t)i * kBM] = (int32_t)~(uint32_t)c;
                }
            };
            merge_sorted_lists<kParts>(smem_u32(xk + r), smem_u32(xi + r),
                                       (uint32_t)(KT * kBM * 4), KT, topk, emit);
        }
        if (n_split == 1) {
            named_barrier_sync(1, 32 * kEW);
            store_rows(et, 32 * kEW);
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
    if (n_split == 1) return;

    // ---------------- merge the split candidates (last CTA of the m-tile) ----------------
    __syncthreads();  // this CTA's lists are written
    if (tid == 0) {
        // the arrival releases them; the m-tile's last arrival acquires the others'
        unsigned int* ctr = counters + (size_t)b * m_tiles + mt;
        const unsigned prev = atom_add_acq_rel_gpu(ctr, 1u);
        *s_last = prev == (unsigned)(n_split - 1);
        if (*s_last) *ctr = 0u;  // ready for the next call
    }
    __syncthreads();
    if (!*s_last) return;
    // Copy the m-tile's candidate lists [n_split][topk][128 rows] (keys, then
    // ids: two contiguous ranges) into the idle stage memory with two bulk
    // copies, then merge per row.
    const int per_row = n_split * topk;
    const size_t base = ((size_t)b * m_tiles + mt) * kBM * per_row;
    uint32_t* mk = reinterpret_cast<uint32_t*>(smem);
    int32_t* mi = reinterpret_cast<int32_t*>(smem) + kBM * per_row;
    if (tid == 0) {
        const uint32_t bytes = (uint32_t)(kBM * per_row * 4);
        fence_proxy_async_global();  // the acquired lists, then the copies that read them
        fence_proxy_async_smem();    // this CTA's earlier reads of the stage memory, then the copies
        mbar_arrive_expect_tx(merge_bar, 2u * bytes);
        bulk_load(mk, part_key + base, bytes, merge_bar);
        bulk_load(mi, part_id + base, bytes, merge_bar);
    }
    // (the barrier makes a time-out, which raises the status, a decision of
    // the whole CTA: the rows' ids are then left unwritten)
    if (!__syncthreads_and(mbar_wait(merge_bar, 0))) return;
    const int r = (warp & 3) * 32 + lane;
    const int s = row0 + r;
    if (warp >= 2 && warp < 6 && s < S) {  // one thread per row merges
        row_bound[(size_t)b * S + s] = 0u;  // every CTA of the m-tile has finished with it
        const uint32_t kk = smem_u32(mk + r), ki = smem_u32(mi + r), ko = smem_u32(out_s);
        const uint32_t lb = (uint32_t)(topk * kBM * 4);
        auto emit = [&](int i, uint64_t c) {
            sts32(ko + 4u * (uint32_t)out_slot(i, r), ~(uint32_t)c);  // id, -1 when empty
        };
        switch (n_split) {
            case 2: merge_sorted_lists<2>(kk, ki, lb, topk, topk, emit); break;
            case 3: merge_sorted_lists<3>(kk, ki, lb, topk, topk, emit); break;
            case 4: merge_sorted_lists<4>(kk, ki, lb, topk, topk, emit); break;
            case 5: merge_sorted_lists<5>(kk, ki, lb, topk, topk, emit); break;
            case 6: merge_sorted_lists<6>(kk, ki, lb, topk, topk, emit); break;
            case 7: merge_sorted_lists<7>(kk, ki, lb, topk, topk, emit); break;
            default: merge_sorted_lists<8>(kk, ki, lb, topk, topk, emit); break;
        }
    }
    __syncthreads();
    store_rows(tid, Cfg<KT>::kThreads);
}

}  // namespace lci
