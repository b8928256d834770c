// rr_select_tc.cu -- full routing and the relay layer on the tensor cores.
//
// Method: "RouteRelay: Event-Triggered Cross-Layer Route Reuse for Efficient
// Dynamic Sparse Attention" (arXiv 2609.07306), cited as RouteRelay §x.
//
// Full routing of a row (§2.1 Eq. 1-2, §3.1 items 1-2) takes two kernels:
//
//   route_select_kernel  (one CTA = one head x 128 query rows, the machinery
//       of rr_tc.cuh with the query tile in TMEM as the MMA's A operand and
//       two accumulators) scores the row block against the head's key tiles
//       twice:
//         pass 0  per row, the largest score of each of 128 column groups
//                 (group = column mod 128); T = the (k+m)-th largest of these
//                 maxima, found by a bit search on their 16-bit order keys
//                 (floor), is at most the row's (k+m)-th best score since
//                 that many distinct valid scores reach it;
//         pass 1  every valid score >= T is kept: the thread owning (row,
//                 quarter of the columns) stores it in its slots in shared
//                 memory (two quarters share a region, one filling it from
//                 the bottom, the other from the top) and records the kept
//                 columns of each tile in a 32-bit mask held in TMEM.
//       Each thread then turns its kept scores into (score, chunk) sort keys
//       and the row's keys go to its record in device memory.
//   route_finish_kernel  (one warp per row) orders the keys (score desc,
//       chunk asc) by a counting sort over 128 bins with exact ranking inside
//       a bin, writes route | near-miss and alpha (the k-th score), draws the
//       random sentinels and adds the global ones.  Rows whose kept scores
//       overflow their slots go to a retry list and are routed exactly on
//       the CUDA cores (route_rows_kernel, rr_route_simt.cu).
//
// The relay layer (§3.2 Eq. 5-8, §4.1-4.2) runs the same two kernels over
// every row and takes the relay decision in route_finish_kernel from the
// kept scores: a candidate chunk of the old ledger row whose score is kept
// has that exact score; one that is not kept scores below T.  So alpha (min
// over the route, Eq. 6) is exact when every route chunk is kept, beta (max
// over the sentinels, Eq. 7) is exact when at least one sentinel is kept,
// and Eq. 8 can often be settled with one side bounded by T.  A stable row
// keeps its ids and stores alpha; a challenged row is rebuilt from the same
// kept scores at this layer.  Rows the bound cannot settle are rescored
// exactly (relay_exact_kernel, candidate key rows gathered) and, if
// challenged, rebuilt there from their kept scores.  On B200 the dense score tiles cost
// less than the per-score work of the test, so one pass that both tests and
// re-routes is cheaper than a rescoring pass followed by a re-route pass;
// the ledger that comes out is the one the pages' two-stage procedure
// defines, and the counters follow the pages' counting rule (c candidates per
// relay row plus the valid keys of every refreshed row).
#include <algorithm>

#include "rr_tc.cuh"

namespace rr {
namespace tc {

constexpr int kSelEpiWarps = 16;
constexpr int kSelThreads = 32 * (2 + kSelEpiWarps);
constexpr int kSelAcc = 2;                       // accumulators (TMEM columns 0..255)
constexpr uint32_t kQCol = kSelAcc * 128;        // query tile (A operand): 96 columns at most
constexpr uint32_t kMaskCol = kQCol + 96;        // kept-column masks: [quarter][tile], 128 columns
constexpr int kMaskTiles = 32;                   // blocks with more key tiles keep masks in device memory
constexpr int kPairCap = 92;                     // kept-score slots shared by two quarters of a row
constexpr int kValStride = kRows + 1;            // padded (slot, row) grid of the kept scores
constexpr int kRowCap = 128;                     // kept scores per row (the record; 4 per lane)
constexpr int kKeysPerLane = kRowCap / 32;
constexpr int kTopWords = 65;                    // u32 words per row of 16-bit group maxima
constexpr int kChunkStride = kRows + 2;          // u16 (slot, row) grid of the kept scores' chunks
constexpr int kHalf = 16;                        // columns per capacity check in pass 1

struct SelLayout {
    uint32_t k, vals, rows, thr, cnt, bars, misc, total;
    int stages;
    __host__ __device__ CtaLayout cta() const { return CtaLayout{0u, k, rows, bars, misc, stages}; }
};

constexpr uint32_t kRingBytes = 128 * 1024;

// k (key ring, 128 KB: as many stages of 128 key rows x dk bf16 as fit, at
// most 8; after pass 1 the chunk grid [2][kPairCap][kChunkStride] u16) |
// vals [2][kPairCap][kValStride] f32
// (before pass 1 the group maxima [kRows][kTopWords] u32) | rows | thr | cnt
// | barriers | misc.  dk: bf16 elements per key row (d, or 3 d for split fp32).
__host__ __device__ inline SelLayout sel_layout(int dk) {
    SelLayout s;
    s.stages = (int)(kRingBytes / (uint32_t)(kKeys * dk * 2));
    if (s.stages > kMaxStages) s.stages = kMaxStages;
    uint32_t o = 0;
    s.k = o;    o = up(o + kRingBytes, 1024);
    s.vals = o; o = up(o + 2 * kPairCap * kValStride * 4, 16);
    s.rows = o; o = up(o + kRows * 4, 16);
    s.thr = o;  o = up(o + kRows * 4, 16);
    s.cnt = o;  o = up(o + kRows * 4, 16);
    s.bars = o; o = up(o + 8 * kNumBars, 16);
    s.misc = o; o = up(o + 16, 16);
    s.total = o + 1024;   // slack for aligning the dynamic base to 1024
    return s;
}
static_assert(kRingBytes >= 2 * kPairCap * kChunkStride * 2, "the key ring holds the chunk grid");

__device__ __forceinline__ void tc_st16(uint32_t taddr, const uint32_t *r) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
        "%11, %12, %13, %14, %15, %16};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
        "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
        : "memory");
}
__device__ __forceinline__ void tc_st8(uint32_t taddr, const uint32_t *r) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
        : "memory");
}
__device__ __forceinline__ void tc_st1(uint32_t taddr, uint32_t v) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x1.b32 [%0], {%1};" ::"r"(taddr), "r"(v) : "memory");
}
__device__ __forceinline__ void tc_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// Pass 1's step for column J of a thread's 32: if v >= T, store v at the
// shared address `addr`, advance `addr` by `step` bytes and set bit J of
// `mask` (one comparison and three predicated instructions).
template <int J>
__device__ __forceinline__ void keep_if(float v, float T, uint32_t &addr, int32_t step, uint32_t &mask) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ge.f32 p, %2, %3;\n\t"
        "@p st.shared.f32 [%0], %2;\n\t"
        "@p add.s32 %0, %0, %4;\n\t"
        "@p or.b32 %1, %1, %5;\n\t}"
        : "+r"(addr), "+r"(mask)
        : "f"(v), "f"(T), "r"(step), "n"(1u << J)
        : "memory");
}
template <int J0, int N>
__device__ __forceinline__ void keep_run(const float *v, float T, uint32_t &addr, int32_t step, uint32_t &mask) {
    if constexpr (N > 0) {
        keep_if<J0>(v[J0], T, addr, step, mask);
        keep_run<J0 + 1, N - 1>(v, T, addr, step, mask);
    }
}

// Larger key = better: score desc, then chunk asc (-0 counts as +0).
__device__ __forceinline__ uint64_t sel_key(float v, int j) {
    const float z = v == 0.0f ? 0.0f : v;
    return ((uint64_t)ord32(z) << 32) | (uint32_t)(0xffffu - (uint32_t)j);
}
__device__ __forceinline__ int sel_key_chunk(uint64_t key) { return (int)(0xffffu - (uint32_t)(key & 0xffffu)); }
__device__ __forceinline__ float sel_key_score(uint64_t key) { return unord32((uint32_t)(key >> 32)); }

// x = hi + mid + lo with each part a bf16 (round to nearest even at every
// step; each remainder is exact in fp32, and the third part takes the last
// 8 significant bits).  Bits of hi, mid, lo in b[0..2].
__device__ __forceinline__ void split3_bf16(float x, uint32_t *b) {
    const __nv_bfloat16 h = __float2bfloat16_rn(x);
    const float r1 = x - __bfloat162float(h);
    const __nv_bfloat16 m = __float2bfloat16_rn(r1);
    const float r2 = r1 - __bfloat162float(m);
    const __nv_bfloat16 l = __float2bfloat16_rn(r2);
    b[0] = (uint32_t)__bfloat16_as_ushort(h);
    b[1] = (uint32_t)__bfloat16_as_ushort(m);
    b[2] = (uint32_t)__bfloat16_as_ushort(l);
}

// MMA issuer of the selection kernel (the whole warp; one elected lane
// issues): A (the query tile) from TMEM.
template <int kSteps>
__device__ __forceinline__ void sel_mma_tile(uint32_t d_tmem, uint32_t a_tmem, uint64_t kdesc) {
#pragma unroll
    for (int kk = 0; kk < kSteps; ++kk) {
        const uint64_t off16 = (uint64_t)((kk >> 2) * (kSubTileBytes >> 4) + (kk & 3) * 2);
        tc_mma_bf16_ts_elect(d_tmem, a_tmem + (uint32_t)(kk * 8), kdesc + off16, kIdesc, kk > 0 ? 1u : 0u);
    }
}

// Split fp32 (d = 64): the query row is [q_hi | q_mid | q_lo] in TMEM (32
// columns per part) and the key row [k_hi | k_mid | k_lo] in three 64-wide
// sub-tiles; the score is the sum of the six part products whose orders add
// up to at most two (hi = order 0), smallest first: mid.mid, hi.lo, lo.hi,
// hi.mid, mid.hi, hi.hi.  With |mid| <= 2^-8 |x| and |lo| <= 2^-16 |x|,
// the dropped products mid.lo and lo.mid are each at most 2^-24 |q_t| |k_t|
// and lo.lo at most 2^-32 |q_t| |k_t|: together at most 2^-23 |q| |k| per
// score, below the fp32 rounding of the sum itself.
__device__ __forceinline__ void sel_mma_tile_split(uint32_t d_tmem, uint32_t a_tmem, uint64_t kdesc) {
    constexpr int kPa[6] = {1, 0, 2, 0, 1, 0};
    constexpr int kPb[6] = {1, 2, 0, 1, 0, 0};
#pragma unroll
    for (int p = 0; p < 6; ++p) {
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
            const uint64_t off16 = (uint64_t)(kPb[p] * (kSubTileBytes >> 4) + kk * 2);
            tc_mma_bf16_ts_elect(d_tmem, a_tmem + (uint32_t)(kPa[p] * 32 + kk * 8), kdesc + off16, kIdesc,
                                 (p > 0 || kk > 0) ? 1u : 0u);
        }
    }
}

__device__ __forceinline__ void sel_mma_issuer(Cta &c, int dk, int split) {
    const int total = 2 * c.ntiles;
    const uint32_t k_addr = saddr(c.k_s);
    const uint32_t stage_bytes = (uint32_t)(kKeys * dk * 2);
    const uint32_t tmem = __shfl_sync(kFull, c.tmem_base, 0);
    const uint32_t a_tmem = tmem + kQCol;
    for (int g = 0; g < total; ++g) {
        const int s = g % c.stages, a = g % kSelAcc;
        if (!mbar_wait_warp(&c.full[s], (g / c.stages) & 1, c.abort_flag)) break;
        if (!mbar_wait_warp(&c.acc_empty[a], ((g / kSelAcc) & 1) ^ 1, c.abort_flag)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem + (uint32_t)(a * kKeys);
        const uint64_t kdesc = sw128_desc(k_addr + (uint32_t)s * stage_bytes);
        if (split) sel_mma_tile_split(d_tmem, a_tmem, kdesc);
        else if (dk == 128) sel_mma_tile<8>(d_tmem, a_tmem, kdesc);
        else sel_mma_tile<4>(d_tmem, a_tmem, kdesc);
        tc_commit_elect(&c.empty[s]);
        tc_commit_elect(&c.acc_full[a]);
    }
    tc_commit_elect(c.mma_done);
    const long long t0 = clock64();
    while (!mbar_test(c.mma_done, 0) && clock64() - t0 < kSpinLimit) {
    }
}

// ---- selection kernel ------------------------------------------------------------
__global__ void __launch_bounds__(kSelThreads, 1)
route_select_kernel(LedgerDev L, const void *__restrict__ Qv,
                    const __grid_constant__ CUtensorMap tmap_k, int use_list) {
    extern __shared__ __align__(1024) unsigned char smem_dyn[];
    unsigned char *smem = align_smem_1024(smem_dyn);
    const int d = L.d, ksel = L.ksel;
    const int split = L.split;
    const int dk = split ? 3 * d : d;   // bf16 elements per key row in the ring
    const SelLayout lay = sel_layout(dk);
    const __nv_bfloat16 *Q = static_cast<const __nv_bfloat16 *>(Qv);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int h = blockIdx.y;

    // Each epilogue thread starts loading its quarter of its query row (the
    // row the set-up below will list for it) before the set-up, so that the
    // loads are in flight while barriers and TMEM are prepared: 64 bytes
    // (d = 128 bf16, or 16 fp32 elements of a split row), or 32 (d = 64 bf16).
    uint4 qpre[4];
    if (warp >= 2) {
        const int qt = (warp - 2) >> 2, r = (warp & 3) * 32 + lane;
        const int count = use_list ? L.head_count[h] : L.nq;
        const int rp = blockIdx.x * kRows + r;
        const int row = rp < count ? (use_list ? L.list[(size_t)h * L.nq + rp] : rp) : -1;
        const size_t base = ((size_t)h * L.nq + (row >= 0 ? row : 0)) * d;
        const uint4 *src = split ? reinterpret_cast<const uint4 *>(static_cast<const float *>(Qv) + base + qt * 16)
                                 : reinterpret_cast<const uint4 *>(Q + base + qt * (d >> 2));
        const int n16 = (split || d == 128) ? 4 : 2;
#pragma unroll
        for (int i = 0; i < 4; ++i) qpre[i] = (row >= 0 && i < n16) ? src[i] : make_uint4(0u, 0u, 0u, 0u);
    }
    Cta c;
    if (!cta_setup(c, smem, lay.cta(), L, Q, L.list, L.head_count, use_list, /*q_to_smem=*/false))
        return;

    // The producer starts at once; the MMA warp waits until the epilogue
    // warps have put the query tile into TMEM (barrier q_ready).
    if (warp == 0) {
        producer(c, &tmap_k, dk, h, 2);
    } else if (warp == 1) {
        if (mbar_wait_warp(c.q_ready, 0, c.abort_flag)) {
            tc_fence_after();
            sel_mma_issuer(c, dk, split);
        }
    } else {
        // the query tile into TMEM columns kQCol.. (row r in lane r, two
        // bf16 per column): epilogue warp (sub-partition sub, quarter qt)
        // writes a quarter of the row's elements for its 32 rows
        {
            const int ew = warp - 2, sub = warp & 3, qt = ew >> 2;
            const uint32_t taddr =
                c.tmem_base + ((uint32_t)(sub * 32) << 16) + kQCol + (uint32_t)(qt * (d >> 3));
            uint32_t w[16];
            if (split) {
                // fp32 elements 16 qt .. 16 qt + 15, each split into bf16
                // hi + mid + lo (x = hi + mid + lo exactly); part p goes to
                // columns 32 p + 8 qt .. 32 p + 8 qt + 7
                uint32_t part[3][8];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const float x[4] = {__uint_as_float(qpre[i].x), __uint_as_float(qpre[i].y),
                                        __uint_as_float(qpre[i].z), __uint_as_float(qpre[i].w)};
#pragma unroll
                    for (int e = 0; e < 4; e += 2) {
                        uint32_t b0[3], b1[3];
                        split3_bf16(x[e], b0);
                        split3_bf16(x[e + 1], b1);
#pragma unroll
                        for (int p = 0; p < 3; ++p) part[p][2 * i + (e >> 1)] = b0[p] | (b1[p] << 16);
                    }
                }
#pragma unroll
                for (int p = 0; p < 3; ++p)
                    tc_st8(c.tmem_base + ((uint32_t)(sub * 32) << 16) + kQCol + (uint32_t)(p * 32 + qt * 8),
                           part[p]);
            } else if (d == 128) {
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    w[4 * i] = qpre[i].x; w[4 * i + 1] = qpre[i].y; w[4 * i + 2] = qpre[i].z; w[4 * i + 3] = qpre[i].w;
                }
                tc_st16(taddr, w);
            } else {
#pragma unroll
                for (int i = 0; i < 2; ++i) {
                    w[4 * i] = qpre[i].x; w[4 * i + 1] = qpre[i].y; w[4 * i + 2] = qpre[i].z; w[4 * i + 3] = qpre[i].w;
                }
                tc_st8(taddr, w);
            }
            tc_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(c.q_ready);
        }
        // Four warps per TMEM sub-partition: quarter qt reads columns
        // 32*qt..32*qt+31 of every tile.  The epilogue threads meet at named
        // barrier 1 between phases (every one of them reaches every barrier,
        // also after a timeout, so none can be left waiting).
        const int ew = warp - 2;
        const int sub = warp & 3;
        const int qt = ew >> 2;
        const int r = sub * 32 + lane;
        const int row = c.rows_s[r];
        const int n_valid = row >= 0 ? valid_keys(row, L.nk, L.causal) : 0;
        const uint32_t lane_base = c.tmem_base + ((uint32_t)(sub * 32) << 16) + (uint32_t)(qt * 32);
        const int nt = c.ntiles;
        const long long wait_limit = L.wait_budget > 0 ? L.wait_budget : kSpinLimit;
        bool ok = true;
        auto epi_sync = [] { asm volatile("bar.sync 1, %0;" ::"n"(kSelEpiWarps * 32) : "memory"); };

        // pass 0: the largest valid score of each column group (this
        // quarter's 32 columns of every tile; group = column mod 128)
        float m[32];
#pragma unroll
        for (int q = 0; q < 32; ++q) m[q] = -INFINITY;
        for (int i = 0; i < nt && ok; ++i) {
            if (!(ok = acc_wait<kSelAcc>(c, i, wait_limit))) break;
            float v[32];
            tc_ld32(lane_base + (uint32_t)((i % kSelAcc) * kKeys), v);
            acc_release<kSelAcc>(c, i);   // the scores are in registers: the MMA may reuse the accumulator
            const int col0 = i * kKeys + qt * 32;
            if (col0 + 32 <= n_valid) {
#pragma unroll
                for (int q = 0; q < 32; ++q) m[q] = fmaxf(m[q], v[q]);
            } else {
#pragma unroll
                for (int q = 0; q < 32; ++q) m[q] = fmaxf(m[q], col0 + q < n_valid ? v[q] : -INFINITY);
            }
        }
        // the row's 128 maxima as 16-bit order keys (the top half of the
        // order-preserving key: a floor), [r][kTopWords] words
        uint32_t *tops = reinterpret_cast<uint32_t *>(smem + lay.vals);
#pragma unroll
        for (int p = 0; p < 16; ++p)
            tops[r * kTopWords + qt * 16 + p] = (ord32(m[2 * p]) >> 16) | (ord32(m[2 * p + 1]) & 0xFFFF0000u);
        epi_sync();

        // threshold of each row (kRows / kSelEpiWarps rows per warp): the
        // largest 16-bit key K that at least k + m of the row's 128 maxima
        // reach; T = the float of key K << 16.  Each lane holds 4 maxima; with
        // j = ceil((k + m) / 32), the answer lies between the smallest and the
        // largest of the lanes' j-th largest maxima (the lanes' top j values
        // are 32 j >= k + m values above the first; above the second each
        // lane has fewer than j, so fewer than k + m in all), and the bit
        // search starts below the bits those two share.  Rows with at most
        // k + m valid keys keep all of them (T = -inf).
        float *thr_s = reinterpret_cast<float *>(smem + lay.thr);
        {
            constexpr int kRowsPerWarp = kRows / kSelEpiWarps;
            const uint16_t *tops16 = reinterpret_cast<const uint16_t *>(tops);
            const int jsel = (ksel + 31) >> 5;   // 1..2 (k + m <= 64)
            uint32_t key[kRowsPerWarp][4], K[kRowsPerWarp];
            int hb[kRowsPerWarp];
            int hbmax = -1;
#pragma unroll
            for (int k2 = 0; k2 < kRowsPerWarp; ++k2) {
                const int rr = ew * kRowsPerWarp + k2;
#pragma unroll
                for (int i = 0; i < 4; ++i) key[k2][i] = tops16[rr * (2 * kTopWords) + i * 32 + lane];
                // the lane's largest and second largest of its four keys
                const uint32_t a0 = max(key[k2][0], key[k2][1]), b0 = min(key[k2][0], key[k2][1]);
                const uint32_t a1 = max(key[k2][2], key[k2][3]), b1 = min(key[k2][2], key[k2][3]);
                const uint32_t top1 = max(a0, a1);
                const uint32_t top2 = max(min(a0, a1), max(b0, b1));
                const uint32_t u = jsel == 1 ? top1 : top2;
                const uint32_t kmx = __reduce_max_sync(kFull, u);
                const uint32_t kmn = __reduce_min_sync(kFull, u);
                const uint32_t x = kmx ^ kmn;
                hb[k2] = x ? 31 - __clz(x) : -1;
                K[k2] = hb[k2] >= 0 ? (kmx & ~((2u << hb[k2]) - 1u)) : kmx;
                hbmax = max(hbmax, hb[k2]);
            }
            for (int bit = hbmax; bit >= 0; --bit) {
#pragma unroll
                for (int k2 = 0; k2 < kRowsPerWarp; ++k2) {
                    const uint32_t cand = K[k2] | (1u << bit);
                    const unsigned mine = (key[k2][0] >= cand ? 1u : 0u) + (key[k2][1] >= cand ? 1u : 0u) +
                                          (key[k2][2] >= cand ? 1u : 0u) + (key[k2][3] >= cand ? 1u : 0u);
                    const unsigned tot = __reduce_add_sync(kFull, mine);
                    if (bit <= hb[k2] && (int)tot >= ksel) K[k2] = cand;
                }
            }
#pragma unroll
            for (int k2 = 0; k2 < kRowsPerWarp; ++k2) {
                const int rr = ew * kRowsPerWarp + k2;
                const int rowr = c.rows_s[rr];
                const int nv = rowr >= 0 ? valid_keys(rowr, L.nk, L.causal) : 0;
                float t = unord32(K[k2] << 16);
                if (nv <= ksel || t != t) t = -INFINITY;
                if (lane == k2) thr_s[rr] = t;
            }
        }
        epi_sync();
        const float T = thr_s[r];

        // pass 1: keep every valid score >= T (tiles backwards: the first
        // ones were loaded last).  Quarters 2p and 2p+1 of row r share the
        // slots p*kPairCap.. of column r of the vals grid: the even quarter
        // fills them upwards, the odd one downwards, so they collide only
        // when together they keep more than kPairCap scores (the row is then
        // redone).  A 16-column half takes the unchecked path while 16 more
        // slots of this thread's own count are free.  The tile's kept columns
        // go to TMEM column kMaskCol + 32*qt + t (device memory for blocks of
        // more than kMaskTiles tiles).
        const int pair = qt >> 1;
        const bool down = (qt & 1) != 0;
        float *vals = reinterpret_cast<float *>(smem + lay.vals);
        float *pv = vals + (pair * kPairCap + (down ? kPairCap - 1 : 0)) * kValStride + r;
        const int step = down ? -kValStride : kValStride;
        int cur = 0;
        const size_t blk = (size_t)blockIdx.y * gridDim.x + blockIdx.x;
        const bool masks_in_tmem = nt <= kMaskTiles;
        const uint32_t mask_tmem = c.tmem_base + ((uint32_t)(sub * 32) << 16) + kMaskCol + (uint32_t)(qt * 32);
        uint32_t *gmask = L.cand_masks + (blk * (size_t)L.mt * 4 + qt) * kRows + r;
        for (int i = 0; i < nt && ok; ++i) {
            const int g = nt + i;
            const int t = nt - 1 - i;
            if (!(ok = acc_wait<kSelAcc>(c, g, wait_limit))) break;
            float v[32];
            tc_ld32(lane_base + (uint32_t)((g % kSelAcc) * kKeys), v);
            acc_release<kSelAcc>(c, g);
            const int lim = n_valid - (t * kKeys + qt * 32);   // columns jj < lim are valid
            uint32_t mask = 0u;
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
                if (lim >= 32 && cur <= kPairCap - kHalf) {
                    uint32_t mh = 0u;
                    uint32_t addr = saddr(pv);
                    if (hf == 0) keep_run<0, kHalf>(v, T, addr, step * 4, mh);
                    else keep_run<kHalf, kHalf>(v, T, addr, step * 4, mh);
                    const int n = __popc(mh);
                    pv += n * step;
                    cur += n;
                    mask |= mh;
                } else {
#pragma unroll
                    for (int jj = hf * kHalf; jj < (hf + 1) * kHalf; ++jj) {
                        if (jj < lim && v[jj] >= T) {
                            if (cur < kPairCap) {
                                *pv = v[jj];
                                pv += step;
                                mask |= 1u << jj;
                            }
                            ++cur;
                        }
                    }
                }
            }
            if (masks_in_tmem) tc_st1(mask_tmem + (uint32_t)t, mask);
            else gmask[(size_t)t * 4 * kRows] = mask;
        }
        tc_wait_st();
        // kept count per quarter, one byte each (0xFF: the row is redone)
        reinterpret_cast<uint8_t *>(smem + lay.cnt)[r * 4 + qt] = (uint8_t)(cur <= kPairCap ? cur : 0xFF);
        epi_sync();   // every count is written and every MMA (the key ring's last reader) is done

        // sort keys.  First each thread pairs its kept scores, in the order
        // they were stored (tiles descending, columns ascending), with their
        // chunks by walking its tile masks, and writes the chunks beside the
        // scores (chunk grid [2][kPairCap][kChunkStride] u16 in the idle key
        // ring).  Then one warp per row turns (score, chunk) into sort keys,
        // quarters in order, and stores them to the row's record.
        const bool cta_ok = *c.abort_flag == 0;
        const uint32_t *cnt_s = reinterpret_cast<const uint32_t *>(smem + lay.cnt);
        uint16_t *chunks_s = reinterpret_cast<uint16_t *>(smem + lay.k);
        auto row_total = [&](int rr, int *cq) {
            const uint32_t cw = cnt_s[rr];
            int tot = 0;
            bool bad = !cta_ok;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                cq[q] = (int)((cw >> (8 * q)) & 0xFFu);
                bad |= cq[q] > kPairCap;
                tot += cq[q];
            }
            bad |= cq[0] + cq[1] > kPairCap || cq[2] + cq[3] > kPairCap || tot > kRowCap;
            return bad ? -1 : tot;
        };
        {
            int cq[4];
            const int total = row_total(r, cq);
            const int own = (qt == 0 ? cq[0] : qt == 1 ? cq[1] : qt == 2 ? cq[2] : cq[3]);
            const bool walk = row >= 0 && total >= 0 && own > 0;
            uint16_t *cp = chunks_s + (pair * kPairCap + (down ? kPairCap - 1 : 0)) * kChunkStride + r;
            const int cstep = down ? -kChunkStride : kChunkStride;
            if (masks_in_tmem) {
                // the thread's tile masks in registers (a warp-wide load),
                // walked tiles descending, columns ascending
                uint32_t mk[kMaskTiles];
                tc_ld32(mask_tmem, reinterpret_cast<float *>(mk));
                if (walk) {
#pragma unroll
                    for (int t = kMaskTiles - 1; t >= 0; --t) {
                        if (t < nt) {
                            uint32_t m = mk[t];
                            const int base = t * kKeys + qt * 32;
                            while (m != 0u) {
                                *cp = (uint16_t)(base + __ffs(m) - 1);
                                cp += cstep;
                                m &= m - 1u;
                            }
                        }
                    }
                }
            } else if (walk) {
                for (int t = nt - 1; t >= 0; --t) {
                    uint32_t m = gmask[(size_t)t * 4 * kRows];
                    const int base = t * kKeys + qt * 32;
                    while (m != 0u) {
                        *cp = (uint16_t)(base + __ffs(m) - 1);
                        cp += cstep;
                        m &= m - 1u;
                    }
                }
            }
        }
        epi_sync();

        // hand-off: each row's keys to its record (one warp per row), with
        // the count and the threshold
        for (int k2 = 0; k2 < kRows / kSelEpiWarps; ++k2) {
            const int rr = ew * (kRows / kSelEpiWarps) + k2;
            if (c.rows_s[rr] < 0) continue;   // warp-uniform
            int cq[4];
            const int total = row_total(rr, cq);
            const size_t slot = blk * kRows + rr;
            uint64_t *rec = L.cand_keys + slot * kRowCap;
            const int c01 = cq[0] + cq[1], c012 = c01 + cq[2];
#pragma unroll
            for (int i = 0; i < kKeysPerLane; ++i) {
                // key e: quarter q, its kk-th score (quarter pair region, upwards
                // for even quarters, downwards for odd ones)
                const int e = lane + 32 * i;
                if (e < total) {
                    const int q = e < cq[0] ? 0 : e < c01 ? 1 : e < c012 ? 2 : 3;
                    const int kk = e - (q == 0 ? 0 : q == 1 ? cq[0] : q == 2 ? c01 : c012);
                    const int s = (q >> 1) * kPairCap + ((q & 1) ? kPairCap - 1 - kk : kk);
                    rec[e] = sel_key(vals[s * kValStride + rr], (int)chunks_s[s * kChunkStride + rr]);
                }
            }
            if (lane == 0) L.cand_meta[slot] = make_uint2(total >= 0 ? (uint32_t)total : 0xFFFFFFFFu,
                                                          __float_as_uint(thr_s[rr]));
        }
    }
    cta_teardown(c, L);
}

// ---- row finishing ---------------------------------------------------------------
constexpr int kFinWarps = 8;
constexpr int kFinThreads = 32 * kFinWarps;
constexpr int kFinSub = 4;                     // finishing CTAs per selection row block
constexpr int kFinRows = kRows / kFinSub;      // rows per finishing CTA (4 per warp)
constexpr int kBins = 128;
static_assert(kBins == 4 * 32, "four bins per lane in the finishing sort");
constexpr int kBitsWords = 128;        // membership bitmaps: rows with <= 4096 valid keys

struct FinScratch {
    uint64_t keys[kRowCap];            // kept keys in bin order
    alignas(16) uint32_t hist[kBins];  // bin counts, then bin starts (4 per lane)
    uint32_t bits[kBitsWords];         // selected and accepted chunks
    uint32_t cbits[2 * kBitsWords];    // relay: chunks of the old route (bit 0) and sentinels (bit 1)
    int32_t acc[32];                   // accepted random sentinels, in order
};

struct FinCounts {
    unsigned long long rows = 0, pairs = 0, full = 0;
};

// What a warp reads from device memory for one row, loaded one row ahead
// so that the loads of row i+1 are in flight while row i is finished.
struct RowIn {
    int row;
    size_t slot;
    uint2 meta;
    uint64_t key[kKeysPerLane];   // the record's first kRowCap slots (those past the count unused)
    int32_t id[3];                // relay: the old ledger row, ids lane, lane + 32, lane + 64 (c <= 96)
};

template <bool kRelay>
__device__ __forceinline__ void load_row(const LedgerDev &L, int h, int row, size_t slot, int lane, RowIn &in) {
    in.row = row;
    in.slot = slot;
    in.meta = L.cand_meta[slot];
    const uint64_t *rec = L.cand_keys + slot * kRowCap;
    const int total = (int)in.meta.x;   // -1 (all ones): the row is redone, nothing to read
#pragma unroll
    for (int i = 0; i < kKeysPerLane; ++i) in.key[i] = lane + 32 * i < total ? rec[lane + 32 * i] : 0ull;
    if (kRelay) {
        const int32_t *idr = L.ids + ((size_t)h * L.nq + row) * L.c;
#pragma unroll
        for (int i = 0; i < 3; ++i) {
            const int e = lane + 32 * i;
            in.id[i] = e < L.c ? idr[e] : -1;
        }
    }
}

// One warp finishes one row from its sort keys.  Returns with nothing
// written when the row is handed on: its kept scores overflowed (anchor:
// retry list; relay: exact rescoring), or (relay) the test keeps the old
// route or needs exact scores.
template <bool kRelay>
__device__ __forceinline__ void finish_one(const LedgerDev &L, int layer, int h, const RowIn &in,
                                           FinScratch &w, int lane, FinCounts &cnt) {
    const int row = in.row;
    const int n_valid = valid_keys(row, L.nk, L.causal);
    const size_t grow = (size_t)h * L.nq + row;
    const uint32_t lt_mask = (1u << lane) - 1u;
    const uint2 meta = in.meta;
    const float T = __uint_as_float(meta.y);
    const int total = (int)meta.x;   // kept keys, or -1: redo the row
    if (total < 0 || total > kRowCap || total < min(L.ksel, n_valid)) {
        if (lane == 0) {
            if (kRelay) {
                L.und_list[atomicAdd(L.und_count, 1)] = (int)grow;   // flags: set by the exact rescoring
            } else {
                const int pos = atomicAdd(&L.retry_count[h], 1);
                L.retry_list[(size_t)h * L.nq + pos] = row;
                atomicAdd(&L.counters[10], 1ULL);
            }
        }
        return;
    }
    uint64_t key[kKeysPerLane];
    bool live[kKeysPerLane];
    bool bad_key = false;
#pragma unroll
    for (int i = 0; i < kKeysPerLane; ++i) {
        const int e = lane + 32 * i;
        live[i] = e < total;
        key[i] = live[i] ? in.key[i] : 0ull;
        bad_key |= live[i] && sel_key_chunk(key[i]) >= n_valid;
    }
    if (__any_sync(kFull, bad_key)) {   // never expected: a record that does not match the row
        if (lane == 0) {
            atomicOr(&L.counters[2], 4ULL);
            if (kRelay) {
                L.und_list[atomicAdd(L.und_count, 1)] = (int)grow;   // flags: set by the exact rescoring
            } else {
                const int pos = atomicAdd(&L.retry_count[h], 1);
                L.retry_list[(size_t)h * L.nq + pos] = row;
                atomicAdd(&L.counters[10], 1ULL);
            }
        }
        return;
    }

    if constexpr (kRelay) {
        // relay test of the old ledger row (§3.2 Eq. 5-8) from the kept scores
        if (n_valid > 32 * kBitsWords) {   // no bitmap for such rows: rescore exactly
            if (lane == 0) {
                L.und_list[atomicAdd(L.und_count, 1)] = (int)grow;   // flags: set by the exact rescoring
            }
            return;
        }
        // the old row's chunks, two bits each in cbits (bit 0: route, bit 1:
        // sentinel; 16 chunks per word).  cbits is all zero here: cleared when
        // the warp starts and, after every row, at the words that row set.
        int rt = 0, st = 0;
        bool bad = false;
#pragma unroll
        for (int i = 0; i < 3; ++i) {
            const int e = lane + 32 * i;
            const int j = in.id[i];
            const bool valid = j >= 0 && j < n_valid;
            bad |= j >= n_valid || j < -1;
            const bool route = e < L.k;
            if (valid) atomicOr(&w.cbits[j >> 4], (route ? 1u : 2u) << ((j & 15) << 1));
            rt += valid && route ? 1 : 0;
            st += valid && !route ? 1 : 0;
        }
        rt = (int)__reduce_add_sync(kFull, (unsigned)rt);
        st = (int)__reduce_add_sync(kFull, (unsigned)st);
        if (__any_sync(kFull, bad) && lane == 0) atomicOr(&L.counters[2], 1ULL);
        __syncwarp();
        // alpha and beta as order keys of the scores (the sort keys' top
        // words), reduced across the warp as unsigned integers
        uint32_t amin_k = 0xFFFFFFFFu, bmax_k = 0u;
        int rf = 0, sf = 0;
#pragma unroll
        for (int i = 0; i < kKeysPerLane; ++i) {
            if (!live[i]) continue;
            const int j = sel_key_chunk(key[i]);
            const uint32_t cb = (w.cbits[j >> 4] >> ((j & 15) << 1)) & 3u;
            const uint32_t ok = (uint32_t)(key[i] >> 32);
            if (cb & 1u) { amin_k = min(amin_k, ok); ++rf; }   // Eq. 6
            if (cb & 2u) { bmax_k = max(bmax_k, ok); ++sf; }   // Eq. 7
        }
        __syncwarp();   // every lane has looked its keys up: clear the words this row set
#pragma unroll
        for (int i = 0; i < 3; ++i) {
            const int j = in.id[i];
            if (j >= 0 && j < n_valid) w.cbits[j >> 4] = 0u;
        }
        __syncwarp();
        amin_k = __reduce_min_sync(kFull, amin_k);
        bmax_k = __reduce_max_sync(kFull, bmax_k);
        rf = (int)__reduce_add_sync(kFull, (unsigned)rf);
        sf = (int)__reduce_add_sync(kFull, (unsigned)sf);
        const float amin = rf > 0 ? unord32(amin_k) : INFINITY;
        const float bmax = sf > 0 ? unord32(bmax_k) : -INFINITY;
        // alpha is exact when every route chunk was kept; beta when a
        // sentinel was kept (the others score below T) or there is none
        const bool aexact = rf == rt;
        const bool bexact = sf > 0 || st == 0;
        // the decision of relay_decide, with one side bounded by T where the
        // kept scores do not give it exactly
        const bool marked = L.gamma_h > 0.0f && (L.flags[grow] & 2u) != 0u;
        int dec = -1;            // 0 keep, 1 refresh, 2 rescore exactly
        uint8_t keep_flag = 0;   // flags byte of a kept row
        if (L.max_age > 0 || L.min_reuse > 0) {   // the ledger's age rules
            const int age = layer - L.anchor_layer[grow];
            if (L.max_age > 0 && age >= L.max_age) {
                dec = 1;
            } else if (L.min_reuse > 0 && age <= L.min_reuse) {
                dec = aexact ? 0 : 2;
                keep_flag = marked ? 2u : 0u;   // no test: the mark stays
            }
        }
        if (dec < 0) {
            float g = L.gamma_rows ? L.gamma_rows[grow] : L.gamma;
            if (marked && L.gamma_h > g) g = L.gamma_h;            // hysteresis margin
            if (aexact && bexact) dec = (amin > bmax + g) ? 0 : 1;   // Eq. 8
            else if (aexact) dec = (amin > T + g) ? 0 : 2;        // beta < T
            else if (sf > 0) dec = 1;                             // alpha < T <= beta
            else dec = 2;
        }
        if (dec == 0) {
            if (lane == 0) {
                L.alpha[grow] = amin;
                L.flags[grow] = keep_flag;
            }
            cnt.pairs += (unsigned long long)(rt + st);
            return;
        }
        if (dec == 2) {   // the exact rescoring writes the row's flags byte
            if (lane == 0) L.und_list[atomicAdd(L.und_count, 1)] = (int)grow;
            return;
        }
        cnt.pairs += (unsigned long long)(rt + st + n_valid);
        cnt.rows += 1;
        cnt.full += (unsigned long long)n_valid;
    }

    // order: counting sort of the kept keys over 128 bins of their score key
    // (larger key = lower bin; bin = (largest key - key) >> shift, the shift
    // putting the key range in 64..128 bins), then each key's rank among the
    // keys of its bin
    uint32_t hmx = 0u, hmn = 0xFFFFFFFFu;
#pragma unroll
    for (int i = 0; i < kKeysPerLane; ++i) {
        if (!live[i]) continue;
        const uint32_t hi = (uint32_t)(key[i] >> 32);
        hmx = max(hmx, hi);
        hmn = min(hmn, hi);
    }
    hmx = __reduce_max_sync(kFull, hmx);
    hmn = __reduce_min_sync(kFull, hmn);
    const int shift = max(0, 25 - __clz(hmx - hmn));   // (hmx - hmn) >> shift < 128
    reinterpret_cast<uint4 *>(w.hist)[lane] = make_uint4(0u, 0u, 0u, 0u);
    __syncwarp();
    int bin[kKeysPerLane];
    uint32_t in_bin[kKeysPerLane];
#pragma unroll
    for (int i = 0; i < kKeysPerLane; ++i) {
        bin[i] = (int)min((uint32_t)(kBins - 1), (hmx - (uint32_t)(key[i] >> 32)) >> shift);
        in_bin[i] = live[i] ? atomicAdd(&w.hist[bin[i]], 1u) : 0u;
    }
    __syncwarp();
    {
        const uint4 hv = reinterpret_cast<const uint4 *>(w.hist)[lane];
        uint32_t incl = hv.x + hv.y + hv.z + hv.w;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t x = __shfl_up_sync(kFull, incl, o);
            if (lane >= o) incl += x;
        }
        const uint32_t excl = incl - (hv.x + hv.y + hv.z + hv.w);
        __syncwarp();
        reinterpret_cast<uint4 *>(w.hist)[lane] =
            make_uint4(excl, excl + hv.x, excl + hv.x + hv.y, excl + hv.x + hv.y + hv.z);
    }
    __syncwarp();
    int start[kKeysPerLane];
#pragma unroll
    for (int i = 0; i < kKeysPerLane; ++i) {
        start[i] = (int)w.hist[bin[i]];
        if (live[i]) w.keys[start[i] + (int)in_bin[i]] = key[i];
    }
    __syncwarp();
    const int nr = min(L.k, n_valid);
    const int nm = min(L.m, n_valid - nr);
    const int nsel = nr + nm;
    int32_t *out = L.ids + grow * L.c;
    bool sel[kKeysPerLane];
    int jc[kKeysPerLane];
#pragma unroll
    for (int i = 0; i < kKeysPerLane; ++i) {
        sel[i] = false;
        jc[i] = live[i] ? sel_key_chunk(key[i]) : -1;
        // a key with nsel or more keys in the bins above it is not selected:
        // no rank needed (these are the lowest, most crowded bins)
        if (!live[i] || start[i] >= nsel) continue;
        const int end = bin[i] + 1 < kBins ? (int)w.hist[bin[i] + 1] : total;
        int rank = 0;
        for (int p = start[i]; p < end; ++p) rank += w.keys[p] > key[i] ? 1 : 0;
        const int pos = start[i] + rank;
        if (pos < nsel) {
            sel[i] = true;
            out[pos < nr ? pos : L.k + (pos - nr)] = jc[i];
            if (pos == nr - 1) L.alpha[grow] = sel_key_score(key[i]);
        }
    }
    if (nsel < L.k + L.m) {   // padding of short rows
        for (int sl = lane; sl < L.k + L.m; sl += 32)
            if (sl < L.k ? sl >= nr : sl - L.k >= nm) out[sl] = -1;
    }

    // random sentinels (§3.1 item 2, §3.4): Philox4x32-10 words keyed
    // (seed; global head, row, layer, t/4), chunk = (word * n_valid) >> 32,
    // repeats and route / near-miss / global members rejected, accepted in
    // draw order; a pool of at most r chunks is taken whole in ascending
    // order, and a row that exhausts max_draws is completed in ascending order
    const bool use_bits = n_valid <= 32 * kBitsWords;
    if (use_bits) {
        const int words = (n_valid + 31) >> 5;
        for (int q = lane; q < words; q += 32) w.bits[q] = 0u;
        __syncwarp();
#pragma unroll
        for (int i = 0; i < kKeysPerLane; ++i)
            if (sel[i]) atomicOr(&w.bits[jc[i] >> 5], 1u << (jc[i] & 31));
        __syncwarp();
    }
    int acc = 0;
    auto in_sel_or_acc = [&](int j) -> bool {
        if (use_bits) return ((w.bits[j >> 5] >> (j & 31)) & 1u) != 0u;
        bool hit = false;
        for (int src = 0; src < 32; ++src) {
#pragma unroll
            for (int i = 0; i < kKeysPerLane; ++i) {
                const int cj = __shfl_sync(kFull, sel[i] ? jc[i] : -1, src);
                hit |= cj == j;
            }
        }
        for (int a = 0; a < acc; ++a) hit |= w.acc[a] == j;
        return hit;
    };
    // mandatory global sentinels (§3.1 item 3; g <= 32): lane t examines
    // candidate t; they follow the random block and leave the random pool
    const int g = L.g_sink + L.g_recent;
    int n_glob = 0;
    if (g > 0) {
        const int jg = lane < g ? global_cand(L, row, lane) : -1;
        const bool listable = lane < g && global_cand_listable(L, lane, jg, n_valid);
        const bool in_rn = in_sel_or_acc(listable ? jg : 0);   // nothing accepted yet
        const bool keep = listable && !in_rn;
        const uint32_t km = __ballot_sync(kFull, keep);
        n_glob = __popc(km);
        int32_t *gout = out + L.k + L.m + L.r;
        if (keep) gout[__popc(km & lt_mask)] = jg;
        if (lane >= n_glob && lane < g) gout[lane] = -1;
    }
    auto taken = [&](int j) -> bool {
        const bool hit = in_sel_or_acc(j);   // every lane calls it (it may shuffle)
        return hit || is_global_cand(L, row, n_valid, j);
    };
    auto accept = [&](bool is_free, int j) {
        const uint32_t fm = __ballot_sync(kFull, is_free);
        const int idx = acc + __popc(fm & lt_mask);
        if (is_free && idx < L.r) {
            w.acc[idx] = j;
            if (use_bits) atomicOr(&w.bits[j >> 5], 1u << (j & 31));
        }
        acc = min(L.r, acc + __popc(fm));
        __syncwarp();
    };
    if (L.r > 0) {
        if (n_valid - nsel - n_glob > L.r) {
            for (int t0 = 0; acc < L.r && t0 < L.max_draws; t0 += 32) {
                const int t = t0 + lane;
                const PhiloxOut o = philox4x32_10((uint32_t)(L.bh_offset + h), (uint32_t)row,
                                                  (uint32_t)layer, (uint32_t)(t >> 2), L.seed_lo, L.seed_hi);
                const int q = t & 3;
                const uint32_t word = q == 0 ? o.w[0] : q == 1 ? o.w[1] : q == 2 ? o.w[2] : o.w[3];
                const int j = (int)__umulhi(word, (uint32_t)n_valid);
                const bool tk = taken(j);
                const bool ok_t = t < L.max_draws && !tk;
                const uint32_t same = __match_any_sync(kFull, j) & __ballot_sync(kFull, ok_t);
                accept(ok_t && (same & lt_mask) == 0u, j);
            }
            if (acc < L.r && lane == 0) atomicAdd(&L.counters[7], 1ULL);
        }
        for (int j0 = 0; acc < L.r && j0 < n_valid; j0 += 32) {
            const int j = j0 + lane;
            const bool tk = taken(min(j, n_valid - 1));
            accept(j < n_valid && !tk, j);
        }
    }
    __syncwarp();
    if (lane < L.r) out[L.k + L.m + lane] = lane < acc ? w.acc[lane] : -1;
    if (lane == 0) {
        L.anchor_layer[grow] = layer;
        L.flags[grow] = L.rebuild_flag;
    }
}

template <bool kRelay>
__global__ void __launch_bounds__(kFinThreads, 4)
route_finish_kernel(LedgerDev L, int layer, int use_list) {
    __shared__ FinScratch scr[kFinWarps];
    __shared__ unsigned long long red_cnt[kFinWarps][3];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int h = blockIdx.y;
    const int count = use_list ? L.head_count[h] : L.nq;
    // CTA (x, h) finishes rows 32 (x % 4) .. 32 (x % 4) + 31 of the
    // selection kernel's row block x / 4 of head h
    const int bsel = blockIdx.x / kFinSub, part = blockIdx.x % kFinSub;
    const int row0 = bsel * kRows + part * kFinRows;
    if (row0 >= count) return;
    const int n_rows = min(kFinRows, count - row0);
    const size_t blk = (size_t)h * ((L.nq + kRows - 1) / kRows) + bsel;
    const size_t slot0 = blk * kRows + (size_t)part * kFinRows;
    FinCounts cnt;
    constexpr int kPerWarp = kFinRows / kFinWarps;
    const int rr0 = warp * kPerWarp;
    auto row_at = [&](int rr) { return use_list ? L.list[(size_t)h * L.nq + row0 + rr] : row0 + rr; };
    if (kRelay) {   // the relay test's chunk map starts clear (each row clears what it sets)
        for (int q = lane; q < 2 * kBitsWords; q += 32) scr[warp].cbits[q] = 0u;
        __syncwarp();
    }
    for (int k2 = 0; k2 < kPerWarp; ++k2) {
        const int rr = rr0 + k2;
        if (rr >= n_rows) break;   // warp-uniform
        RowIn cur;
        load_row<kRelay>(L, h, row_at(rr), slot0 + rr, lane, cur);
        finish_one<kRelay>(L, layer, h, cur, scr[warp], lane, cnt);
        __syncwarp();
    }
    if (kRelay) {
        if (lane == 0) {
            red_cnt[warp][0] = cnt.rows;
            red_cnt[warp][1] = cnt.pairs;
            red_cnt[warp][2] = cnt.full;
        }
        __syncthreads();
        if (tid < 3) {
            unsigned long long s = 0;
            for (int i = 0; i < kFinWarps; ++i) s += red_cnt[i][tid];
            const int slot_of = tid == 0 ? 0 : tid == 1 ? 1 : 8;   // rows, pairs, full-routing pairs
            if (s) atomicAdd(&L.counters[slot_of], s);
        }
    }
}

// ---- exact rescoring of the relay rows the kept scores leave open ------------------
// One warp per listed row: alpha and beta from the row's candidate key rows
// (Eq. 5-7, fp32 products of the inputs), the decision of Eq. 8 with the
// ledger's age rules; a challenged row is rebuilt by the same warp from its
// kept scores (the finishing step of an anchor row), or, when its record
// overflowed, goes to the retry list.
constexpr int kExactWarps = 8;

// The candidate's score, fp32 products of the inputs (bf16 rows: 8 elements
// per 16-byte load; fp32 rows: 4).
template <int D>
__device__ __forceinline__ float exact_dot(const float *qv, const __nv_bfloat16 *krow) {
    const uint4 *kp = reinterpret_cast<const uint4 *>(krow);
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 4
    for (int c8 = 0; c8 < D / 8; ++c8) {
        const uint4 kv = __ldg(kp + c8);
        const float *q8 = qv + c8 * 8;
        acc[0] = fmaf(q8[0], __uint_as_float(kv.x << 16), acc[0]);
        acc[1] = fmaf(q8[1], __uint_as_float(kv.x & 0xffff0000u), acc[1]);
        acc[2] = fmaf(q8[2], __uint_as_float(kv.y << 16), acc[2]);
        acc[3] = fmaf(q8[3], __uint_as_float(kv.y & 0xffff0000u), acc[3]);
        acc[0] = fmaf(q8[4], __uint_as_float(kv.z << 16), acc[0]);
        acc[1] = fmaf(q8[5], __uint_as_float(kv.z & 0xffff0000u), acc[1]);
        acc[2] = fmaf(q8[6], __uint_as_float(kv.w << 16), acc[2]);
        acc[3] = fmaf(q8[7], __uint_as_float(kv.w & 0xffff0000u), acc[3]);
    }
    return (acc[0] + acc[1]) + (acc[2] + acc[3]);
}
template <int D>
__device__ __forceinline__ float exact_dot(const float *qv, const float *krow) {
    const float4 *kp = reinterpret_cast<const float4 *>(krow);
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 4
    for (int c4 = 0; c4 < D / 4; ++c4) {
        const float4 kv = __ldg(kp + c4);
        const float *q4 = qv + c4 * 4;
        acc[0] = fmaf(q4[0], kv.x, acc[0]);
        acc[1] = fmaf(q4[1], kv.y, acc[1]);
        acc[2] = fmaf(q4[2], kv.z, acc[2]);
        acc[3] = fmaf(q4[3], kv.w, acc[3]);
    }
    return (acc[0] + acc[1]) + (acc[2] + acc[3]);
}
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }
__device__ __forceinline__ float to_f32(float x) { return x; }

template <int D, typename T>
__global__ void __launch_bounds__(32 * kExactWarps)
relay_exact_kernel(LedgerDev L, const T *__restrict__ Q, const T *__restrict__ K, int layer) {
    __shared__ __align__(16) float qs[kExactWarps][D];
    __shared__ FinScratch fin[kExactWarps];
    __shared__ unsigned long long red_cnt[kExactWarps][3];
    const size_t slots_per_head = (size_t)((L.nq + kRows - 1) / kRows) * kRows;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n = *L.und_count;
    unsigned long long crow = 0, cpair = 0, cfull = 0;
    for (int u = blockIdx.x * kExactWarps + warp; u < n; u += gridDim.x * kExactWarps) {
        const int grow = L.und_list[u];
        const int h = grow / L.nq, i = grow - h * L.nq;
        const int n_valid = valid_keys(i, L.nk, L.causal);
        for (int t = lane; t < D; t += 32) qs[warp][t] = to_f32(Q[(size_t)grow * D + t]);
        __syncwarp();
        const int32_t *idr = L.ids + (size_t)grow * L.c;
        const T *Kh = K + (size_t)h * L.nk * D;
        float amin = INFINITY, bmax = -INFINITY;
        int ncand = 0;
        bool bad = false;
        for (int e0 = 0; e0 < L.c; e0 += 32) {
            const int e = e0 + lane;
            const int j = e < L.c ? idr[e] : -1;
            const bool valid = j >= 0 && j < n_valid;
            bad |= j >= n_valid || j < -1;
            if (valid) {
                const float sc = exact_dot<D>(qs[warp], Kh + (size_t)j * D);
                if (e < L.k) amin = fminf(amin, sc);   // Eq. 6
                else bmax = fmaxf(bmax, sc);           // Eq. 7
                ++ncand;
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            amin = fminf(amin, __shfl_xor_sync(kFull, amin, o));
            bmax = fmaxf(bmax, __shfl_xor_sync(kFull, bmax, o));
            ncand += __shfl_xor_sync(kFull, ncand, o);
        }
        const bool any_bad = __any_sync(kFull, bad);
        uint32_t fl = 0u;
        if (lane == 0) fl = relay_decide(L, (size_t)grow, layer, amin, bmax);   // Eq. 8
        fl = __shfl_sync(kFull, fl, 0);
        const bool refresh = (fl & 1u) != 0u;
        if (lane == 0) {
            if (!refresh) {
                L.flags[grow] = (uint8_t)fl;
                L.alpha[grow] = amin;
            }
            if (any_bad) atomicOr(&L.counters[2], 1ULL);
            cpair += (unsigned long long)ncand;
            if (refresh) {
                crow += 1;
                cpair += (unsigned long long)n_valid;
                cfull += (unsigned long long)n_valid;
            }
        }
        if (refresh) {
            // the row is rebuilt at this layer from the same kept scores (its
            // record from the selection kernel); a record that overflowed
            // goes to the retry list
            RowIn in;
            load_row<false>(L, h, i, (size_t)h * slots_per_head + i, lane, in);
            FinCounts unused;
            finish_one<false>(L, layer, h, in, fin[warp], lane, unused);
        }
        __syncwarp();
    }
    if (lane == 0) {
        red_cnt[warp][0] = crow;
        red_cnt[warp][1] = cpair;
        red_cnt[warp][2] = cfull;
    }
    __syncthreads();
    if (threadIdx.x < 3) {
        unsigned long long s = 0;
        for (int w = 0; w < kExactWarps; ++w) s += red_cnt[w][threadIdx.x];
        const int slot_of[3] = {0, 1, 8};
        if (s) atomicAdd(&L.counters[slot_of[threadIdx.x]], s);
    }
}

// Kc fp32 [rows, d] -> bf16 parts [rows, 3 d] = [hi | mid | lo] per row
// (the split of split3_bf16), four elements per thread.
__global__ void __launch_bounds__(256) split_keys_kernel(const float4 *__restrict__ K, uint16_t *__restrict__ out,
                                                         size_t n4, int d4) {
    for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n4; i += (size_t)gridDim.x * blockDim.x) {
        const float4 v = __ldg(K + i);
        const size_t row = i / (size_t)d4;
        const int t = (int)(i - row * (size_t)d4) * 4;
        const float x[4] = {v.x, v.y, v.z, v.w};
        uint32_t b[4][3];
#pragma unroll
        for (int e = 0; e < 4; ++e) split3_bf16(x[e], b[e]);
        uint16_t *dst = out + row * (size_t)(12 * d4) + t;
#pragma unroll
        for (int p = 0; p < 3; ++p)
            *reinterpret_cast<uint2 *>(dst + p * 4 * d4) =
                make_uint2(b[0][p] | (b[1][p] << 16), b[2][p] | (b[3][p] << 16));
    }
}

}  // namespace tc

bool route_select_split_supported(const LedgerDev &L, int dtype) {
    return dtype == kF32 && L.d == 64 && L.ksel <= 64 && L.r <= 32 && L.nk <= 65535 && L.c <= 96 &&
           L.g_sink + L.g_recent <= 32 && route_select_smem_bytes(L) <= 232448;
}

CandSizes route_select_candidate_sizes(const LedgerDev &L, int dtype) {
    CandSizes z{0, 0, 0, 0, 0};
    const bool split = route_select_split_supported(L, dtype);
    if (!route_rows_tc_supported(L, dtype) && !split) return z;
    const size_t blocks = (size_t)L.bh * ((L.nq + tc::kRows - 1) / tc::kRows);
    const size_t mt = (size_t)((L.nk + tc::kKeys - 1) / tc::kKeys);
    z.keys = blocks * tc::kRows * tc::kRowCap * sizeof(uint64_t);
    z.masks = mt > (size_t)tc::kMaskTiles ? blocks * mt * 4 * tc::kRows * sizeof(uint32_t) : 0;
    z.meta = blocks * tc::kRows * sizeof(uint2);
    z.und = (size_t)L.bh * L.nq * sizeof(int32_t);
    if (split) z.ksplit = (size_t)L.bh * L.nk * 3 * L.d * sizeof(uint16_t);
    return z;
}

size_t route_select_smem_bytes(const LedgerDev &L) { return tc::sel_layout(L.d).total; }

cudaError_t route_select_prepare() {
    cudaError_t e = cudaFuncSetAttribute(tc::route_select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)tc::sel_layout(128).total);
    return e;
}

cudaError_t launch_route_select(const LedgerDev &L, const void *q, const CUtensorMap &map, int layer,
                                bool use_list, SelectMode mode, cudaStream_t s) {
    dim3 grid((L.nq + tc::kRows - 1) / tc::kRows, L.bh);
    tc::route_select_kernel<<<grid, tc::kSelThreads, tc::sel_layout(L.split ? 3 * L.d : L.d).total, s>>>(
        L, q, map, use_list ? 1 : 0);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    dim3 fgrid(grid.x * tc::kFinSub, L.bh);
    if (mode == SelectMode::kRelay)
        tc::route_finish_kernel<true><<<fgrid, tc::kFinThreads, 0, s>>>(L, layer, 0);
    else
        tc::route_finish_kernel<false><<<fgrid, tc::kFinThreads, 0, s>>>(L, layer, use_list ? 1 : 0);
    return cudaGetLastError();
}

namespace {

// Kc of an fp32 problem into its three bf16 parts, and the tensor map of
// the part rows.
cudaError_t split_keys(const LedgerDev &L, const void *k, CUtensorMap *map, cudaStream_t s) {
    const size_t n4 = (size_t)L.bh * L.nk * (L.d / 4);
    const unsigned blocks = (unsigned)std::min<size_t>((n4 + 255) / 256, (size_t)148 * 16);
    tc::split_keys_kernel<<<blocks, 256, 0, s>>>(static_cast<const float4 *>(k), L.ksplit, n4, L.d / 4);
    cudaError_t e = cudaGetLastError();
    if (e == cudaSuccess) e = tc::key_rows_tensor_map(L.ksplit, 3 * L.d, L.nk, L.bh, map);
    return e;
}

}  // namespace

// Rows whose kept scores overflowed (retry lists) are rebuilt exactly on the
// CUDA cores.  The lists are short (usually empty), so the grid is narrow:
// about four CTAs per SM over all heads, each striding over its head's list.
cudaError_t launch_retry_rows_simt(const LedgerDev &L, const void *q, const void *k, int layer,
                                   cudaStream_t s) {
    LedgerDev R = L;
    R.list = L.retry_list;
    R.head_count = L.retry_count;
    const int max_tiles = std::max(1, (4 * 148 + L.bh - 1) / L.bh);
    return launch_route_rows_simt(R, L.split ? kF32 : kBF16, q, k, layer, true, s, max_tiles);
}

cudaError_t launch_route_rows_split(const LedgerDev &L, const void *q, const void *k, int layer,
                                    bool use_list, cudaStream_t s) {
    CUtensorMap map;
    cudaError_t e = split_keys(L, k, &map, s);
    if (e == cudaSuccess) e = cudaMemsetAsync(L.retry_count, 0, (size_t)L.bh * sizeof(int32_t), s);
    if (e == cudaSuccess) e = launch_route_select(L, q, map, layer, use_list, SelectMode::kAnchor, s);
    if (e != cudaSuccess) return e;
    return launch_retry_rows_simt(L, q, k, layer, s);
}

cudaError_t launch_relay_oneshot(const LedgerDev &L, const void *q, const void *k, int layer,
                                 cudaStream_t s) {
    CUtensorMap map;
    cudaError_t e = L.split ? split_keys(L, k, &map, s) : tc::key_tensor_map(L, k, &map);
    if (e == cudaSuccess) e = cudaMemsetAsync(L.retry_count, 0, (size_t)L.bh * sizeof(int32_t), s);
    if (e == cudaSuccess) e = cudaMemsetAsync(L.und_count, 0, sizeof(int32_t), s);
    if (e == cudaSuccess) e = launch_route_select(L, q, map, layer, false, SelectMode::kRelay, s);
    if (e != cudaSuccess) return e;
    const unsigned grid = 148 * 2;   // grid-stride over the open rows (usually none)
    if (L.split) {
        tc::relay_exact_kernel<64, float><<<grid, 32 * tc::kExactWarps, 0, s>>>(
            L, static_cast<const float *>(q), static_cast<const float *>(k), layer);
    } else {
        const auto *Q = static_cast<const __nv_bfloat16 *>(q);
        const auto *K = static_cast<const __nv_bfloat16 *>(k);
        if (L.d == 128)
            tc::relay_exact_kernel<128, __nv_bfloat16><<<grid, 32 * tc::kExactWarps, 0, s>>>(L, Q, K, layer);
        else
            tc::relay_exact_kernel<64, __nv_bfloat16><<<grid, 32 * tc::kExactWarps, 0, s>>>(L, Q, K, layer);
    }
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    return launch_retry_rows_simt(L, q, k, layer, s);
}

}  // namespace rr
