// rr_route_tc.cu -- full routing on the Blackwell tensor cores (tcgen05 + TMEM).
//
// Method: "RouteRelay: Event-Triggered Cross-Layer Route Reuse for Efficient
// Dynamic Sparse Attention" (arXiv 2609.07306), cited as RouteRelay §x.
//
// Computes, for 128 query rows of one head at a time, the score rows S = Qc
// Kc^T (§2.1 Eq. 1) tile by tile on the tensor cores and selects each row's
// k + m best key chunks (§2.1 Eq. 2 and §3.1 item 1) without writing S to
// memory; then draws the random sentinels (§3.1 item 2) and writes the
// ledger row (§3.1 Eq. 4).  Serves the anchor layer (all rows) and the
// refresh of the compacted unstable rows (§4.2, rows taken from the
// per-head list).  The relay rescoring on the same tiles
// (relay_rescore_tc_kernel, §3.2 Eq. 5-8) sits at the end of the file.
//
// CTA layout (one CTA = one head x 128 query rows):
//   warp 0     TMA producer: 128-key x d tiles of Kc (bf16, 128-byte
//              swizzle) into a ring of shared-memory stages.
//   warp 1     allocates 512 TMEM columns (four 128x128 fp32 accumulators);
//              one lane issues tcgen05.mma (M=128, N=128, K=16 per op) for
//              every key tile and commits to mbarriers.
//   warps 2-   epilogue, reading the score tile with tcgen05.ld; a warp may
//              only read the 32 TMEM lanes (= query rows) of its sub-partition
//              (warp index mod 4).  The heap kernel runs 4 such warps, one
//              thread per row; the two-pass kernel and the rescoring kernel
//              run 16, the four warps of a sub-partition each taking a
//              quarter of every tile's columns.
// The query tile is gathered by row index into the layout a 128-byte
// swizzled TMA load would produce, so anchor and refresh share one path.
//
// Selection (route_rows_tc_kernel).  The tensor cores are cheap next to the
// per-score work of an exact top-(k+m), so the key tiles are streamed twice
// and the MMA recomputed:
//   pass 0  per row: the two largest valid scores of each of 64 column
//           groups; T = the (k+m)-th largest of these 128 values (a lower
//           bound of the row's (k+m)-th best score, since that many distinct
//           scores reach it);
//   pass 1  per row: every valid score >= T is appended to the row's buffer
//           (on Gaussian-like rows about 10% more than k+m).
// The kept scores are then ordered (score desc, chunk asc) and the row's
// ledger entry written by one warp per row (finish_row): in a separate
// kernel reading the kept scores from global memory, or by the same CTA.  A
// row whose kept scores do not fit the buffer (kCap) is appended to a retry
// list and routed by route_rows_tc_heap_kernel, which keeps a per-row
// min-heap of the k+m best over one pass; results are exact either way.
//
// Every wait is bounded; a timeout sets bit 1 of the error word and the CTA
// drains its copies, frees its TMEM and returns.
#include "rr_tc.cuh"

namespace rr {
namespace tc {

constexpr int kHeapThreads = 32 * (2 + 4);     // heap kernel: 4 epilogue warps (one per row)
constexpr int kEpiWarps = 16;                  // two-pass kernel: epilogue warps (four per row)
constexpr int kPassThreads = 32 * (2 + kEpiWarps);
// two-pass selection
constexpr int kGroups = 16;                // column groups per quarter row (four quarters per row)
constexpr int kTops = 8 * kGroups;         // group top-2 values per row
constexpr int kTopStride = kTops + 1;      // padded row of the group tops in shared memory
constexpr int kCap = 120;                  // kept scores per row
constexpr int kBufStride = kRows + 1;      // padded row of the append buffers (slot-major)
constexpr int kStageCols = 16;             // columns per staging round of the collect pass
constexpr int kThrLowBit = 16;             // threshold search stops at this key bit
// heap selection (retry path)
constexpr int kBuf = 32;

// Stages of the key ring (what the shared memory left by the selection
// buffers allows).
__host__ __device__ inline int stages_for(int d, bool two_pass) {
    if (two_pass) return d == 64 ? 4 : 2;
    return 2;
}

struct Layout {
    uint32_t q, k, sel, bufv, bufi, stg, rows, red, bars, misc, total;
    int stages;
    __host__ __device__ CtaLayout cta() const { return CtaLayout{q, k, rows, bars, misc, stages}; }
};

// two_pass: q | k | sel (91 KB: the group tops [kRows][kTopStride] f32 after
//           pass 0, then bufv [kCap][kBufStride] f32 | bufi [kCap][kBufStride]
//           u16, padded so that one row's slots fall in distinct banks) |
//           stg [epilogue threads][kStageCols] f32 | rows | red (threshold
//           and kept count per row)
// heap:     q | k | heap [ksel][kRows] u64 | bufv [kBuf][kRows] f32 | bufi [kBuf][kRows] i32
__host__ __device__ inline Layout layout_of(int d, int ksel, bool two_pass) {
    Layout s;
    s.stages = stages_for(d, two_pass);
    uint32_t o = 0;
    s.q = o;    o = up(o + kRows * d * 2, 1024);
    s.k = o;    o = up(o + s.stages * kKeys * d * 2, 1024);
    s.sel = o;
    if (two_pass) {
        s.bufv = o; o = up(o + kCap * kBufStride * 4, 16);
        s.bufi = o; o = up(o + kCap * kBufStride * 2, 16);
        o = up(s.sel + (kRows * kTopStride * 4 > o - s.sel ? kRows * kTopStride * 4 : o - s.sel), 16);
        s.stg = o;  o = up(o + kEpiWarps * 32 * kStageCols * 4, 16);
    } else {
        s.stg = 0;
        o = up(o + kRows * ksel * 8, 16);   // the heap, at sel
        s.bufv = o; o = up(o + kRows * kBuf * 4, 16);
        s.bufi = o; o = up(o + kRows * kBuf * 4, 16);
    }
    s.rows = o; o = up(o + kRows * 4, 16);
    s.red = o;  o = up(o + (two_pass ? 2 * kRows * 4 : 0), 16);
    s.bars = o; o = up(o + 8 * kNumBars, 16);
    s.misc = o; o = up(o + 16, 16);
    s.total = o + 1024;   // slack for aligning the dynamic base to 1024
    return s;
}

// Random sentinels (RouteRelay §3.1 item 2, §3.4) of one row, one thread:
// Philox4x32-10 draws keyed (seed; head, row, layer, t/4), chunk = (word *
// n_valid) >> 32, rejecting repeats and route / near-miss members
// (`in_excl`); a pool of at most r chunks is taken whole in ascending order,
// and a row that exhausts max_draws is completed in ascending order.
// Accepted chunks go to acc_at(0..); with a membership bitmap (`bits`,
// words at stride kRows, already holding route and near-miss) they are also
// marked there, which makes in_excl cover them.
template <typename Excl, typename Acc>
__device__ __forceinline__ int random_sentinels(const LedgerDev &L, int ghead, int row, int layer,
                                                int n_valid, int nsel, Excl in_excl, Acc acc_at,
                                                int32_t *out, uint32_t *bits) {
    int acc = 0;
    auto taken = [&](int j) {
        if (in_excl(j)) return true;
        if (bits) return false;
        for (int e = 0; e < acc; ++e)
            if ((int)acc_at(e) == j) return true;
        return false;
    };
    auto accept = [&](int j) {
        acc_at(acc) = j;
        ++acc;
        if (bits) bits[(j >> 5) * kRows] |= 1u << (j & 31);
    };
    if (L.r > 0) {
        const int np = n_valid - nsel;
        if (np > L.r) {
            uint32_t w4[4] = {0u, 0u, 0u, 0u};
            for (int t = 0; acc < L.r && t < L.max_draws; ++t) {
                if ((t & 3) == 0) {
                    const PhiloxOut o = philox4x32_10((uint32_t)ghead, (uint32_t)row, (uint32_t)layer,
                                                      (uint32_t)(t >> 2), L.seed_lo, L.seed_hi);
                    w4[0] = o.w[0]; w4[1] = o.w[1]; w4[2] = o.w[2]; w4[3] = o.w[3];
                }
                const int sel = t & 3;
                const uint32_t w = sel == 0 ? w4[0] : sel == 1 ? w4[1] : sel == 2 ? w4[2] : w4[3];
                const int j = (int)__umulhi(w, (uint32_t)n_valid);
                if (!taken(j)) accept(j);
            }
            if (acc < L.r) atomicAdd(&L.counters[7], 1ULL);
        }
        for (int j = 0; acc < L.r && j < n_valid; ++j)
            if (!taken(j)) accept(j);
    }
    for (int e = 0; e < L.r; ++e) out[e] = e < acc ? (int)acc_at(e) : -1;
    return acc;
}

// ---- per-row keys for the heap path ---------------------------------------------
// Keys order (score, chunk) pairs: larger key = higher score, then smaller chunk.
__device__ __forceinline__ uint64_t make_key(float s, int j) {
    return ((uint64_t)ord32(s) << 32) | (uint32_t)(~(uint32_t)j);
}
__device__ __forceinline__ int key_chunk(uint64_t key) { return (int)(~(uint32_t)key); }
__device__ __forceinline__ float key_score(uint64_t key) { return unord32((uint32_t)(key >> 32)); }

// Min-heap of n keys for one row; element e lives at H[e * kRows] (rows are
// interleaved so that 32 threads touching the same e hit distinct banks).
__device__ __forceinline__ void heap_sift(uint64_t *H, int n, uint64_t K) {
    int i = 0;
    while (true) {
        const int l = 2 * i + 1;
        if (l >= n) break;
        const uint64_t kl = H[l * kRows];
        const uint64_t kr = (l + 1 < n) ? H[(l + 1) * kRows] : ~0ull;
        const bool right = kr < kl;
        const uint64_t kc = right ? kr : kl;
        if (kc >= K) break;
        H[i * kRows] = kc;
        i = right ? l + 1 : l;
    }
    H[i * kRows] = K;
}

// ---- heap kernel: one pass, per-row min-heap (the retry path) --------------------
__global__ void __launch_bounds__(kHeapThreads, 1)
route_rows_tc_heap_kernel(LedgerDev L, const __nv_bfloat16 *__restrict__ Q,
                          const __grid_constant__ CUtensorMap tmap_k, int layer, int use_list) {
    extern __shared__ __align__(1024) unsigned char smem_dyn[];
    unsigned char *smem = align_smem_1024(smem_dyn);
    const int d = L.d, ksel = L.ksel;
    const Layout lay = layout_of(d, ksel, false);
    Cta c;
    if (!cta_setup(c, smem, lay.cta(), L, Q, L.list, L.head_count, use_list)) return;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int h = blockIdx.y;

    if (warp == 0) {
        producer(c, &tmap_k, d, h, 1);
    } else if (warp == 1) {
        mma_issuer(c, d, 1);
    } else {
        const int sub = warp & 3;
        const int r = sub * 32 + lane;
        const int row = c.rows_s[r];
        const int n_valid = row >= 0 ? valid_keys(row, L.nk, L.causal) : 0;
        uint64_t *H = reinterpret_cast<uint64_t *>(smem + lay.sel) + r;
        float *bv = reinterpret_cast<float *>(smem + lay.bufv) + r;
        int *bi = reinterpret_cast<int *>(smem + lay.bufi) + r;
        for (int e = 0; e < ksel; ++e) H[e * kRows] = 0ull;
        float thr = -INFINITY;
        bool ok = true;
        for (int t = 0; t < c.ntiles && ok; ++t) {
            if (!(ok = acc_wait(c, t))) break;
            const uint32_t tbase = c.tmem_base + ((uint32_t)(sub * 32) << 16) + (uint32_t)((t % kAcc) * kKeys);
#pragma unroll 1
            for (int ch = 0; ch < kKeys / 32; ++ch) {
                float v[32];
                tc_ld32(tbase + (uint32_t)(ch * 32), v);
                const int col0 = t * kKeys + ch * 32;
                int cnt = 0;
#pragma unroll
                for (int jj = 0; jj < 32; ++jj) {
                    if (col0 + jj < n_valid && v[jj] >= thr) {
                        bv[cnt * kRows] = v[jj];
                        bi[cnt * kRows] = col0 + jj;
                        ++cnt;
                    }
                }
                for (int e = 0; e < cnt; ++e) {
                    const uint64_t key = make_key(bv[e * kRows], bi[e * kRows]);
                    if (key > H[0]) heap_sift(H, ksel, key);
                }
                const uint64_t root = H[0];
                thr = root == 0ull ? -INFINITY : key_score(root);
            }
            acc_release(c, t);
        }
        if (ok && row >= 0) {
            // best-first order: repeatedly move the heap minimum to the end
            for (int end = ksel - 1; end > 0; --end) {
                const uint64_t top = H[0];
                const uint64_t last = H[end * kRows];
                H[end * kRows] = top;
                heap_sift(H, end, last);
            }
            const int nr = min(L.k, n_valid);
            const int nm = min(L.m, n_valid - nr);
            const int nsel = nr + nm;
            const size_t grow = (size_t)h * L.nq + row;
            int32_t *out = L.ids + grow * L.c;
            for (int e = 0; e < L.k; ++e) out[e] = e < nr ? key_chunk(H[e * kRows]) : -1;
            for (int e = 0; e < L.m; ++e) out[L.k + e] = e < nm ? key_chunk(H[(nr + e) * kRows]) : -1;
            auto in_rn = [&](int j) {
                for (int e = 0; e < nsel; ++e)
                    if (key_chunk(H[e * kRows]) == j) return true;
                return false;
            };
            // mandatory global sentinels, after the random block
            const int g = L.g_sink + L.g_recent;
            int n_glob = 0;
            int32_t *gout = out + L.k + L.m + L.r;
            for (int t = 0; t < g; ++t) {
                const int j = global_cand(L, row, t);
                if (global_cand_listable(L, t, j, n_valid) && !in_rn(j)) gout[n_glob++] = j;
            }
            for (int t = n_glob; t < g; ++t) gout[t] = -1;
            random_sentinels(
                L, L.bh_offset + h, row, layer, n_valid, nsel + n_glob,
                [&](int j) { return in_rn(j) || is_global_cand(L, row, n_valid, j); },
                [&](int e) -> int & { return bi[e * kRows]; }, out + L.k + L.m, nullptr);
            L.alpha[grow] = key_score(H[(nr - 1) * kRows]);
            L.anchor_layer[grow] = layer;
            L.flags[grow] = L.rebuild_flag;
        }
    }
    cta_teardown(c, L);
}

// ---- finishing a row from its kept scores (one warp per row) ---------------------
// The ledger row of one query row from its kept scores (a superset of its
// k + m best): route | near-miss in best-first order (score desc, chunk asc),
// alpha (the k-th score) and the random sentinels (RouteRelay §3.1 items
// 1-2).
//
// Order: the kept scores are binned over their own range (128 bins, larger
// score = lower bin, ties share a bin), placed by bin, and each one's final
// position is its bin's start plus the number of better keys in its bin.
// Sentinels: 32 draws at a time, one per lane (the same Philox words,
// rejection rule and ascending completion as random_sentinels above); a draw
// is accepted if its chunk is not selected, not accepted earlier and not
// drawn by an earlier lane of the round (warp match), in draw order.
constexpr int kFinBins = 128;
constexpr int kFinBitsWords = 128;   // membership bitmap: rows with <= 4096 valid keys

struct FinWarp {
    uint64_t keys[kCap];             // kept scores placed by bin
    uint32_t hist[kFinBins];         // counts, then start offsets
    uint32_t bits[kFinBitsWords];    // selected and accepted chunks
    int32_t acc[32];                 // accepted sentinels, in order
};

// Larger key = better: score desc, then chunk asc (-0 counts as +0).
__device__ __forceinline__ uint64_t cand_key(float v, int j) {
    const float z = v == 0.0f ? 0.0f : v;
    return ((uint64_t)ord32(z) << 32) | (uint32_t)(0xffffu - (uint32_t)j);
}

// One warp, every lane with the same arguments.  The row's `run` kept scores
// are read through getv(e) / geti(e), e < run <= kCap; they include the
// row's min(k + m, valid keys) best.
template <typename GetV, typename GetI>
__device__ __forceinline__ void finish_row(const LedgerDev &L, int layer, int h, int row, int run,
                                           GetV getv, GetI geti, FinWarp &w, int lane) {
    const int n_valid = valid_keys(row, L.nk, L.causal);
    const uint32_t lt_mask = (1u << lane) - 1u;

    float v[4];
    int jc[4];
    bool live[4];
    float mx = -INFINITY, mn = INFINITY;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int e = lane + 32 * i;
        live[i] = e < run;
        v[i] = 0.f;
        jc[i] = -1;
        if (live[i]) {
            v[i] = getv(e);
            jc[i] = geti(e);
            mx = fmaxf(mx, v[i]);
            mn = fminf(mn, v[i]);
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, o));
        mn = fminf(mn, __shfl_xor_sync(kFull, mn, o));
    }
    const float inv = mx > mn ? (float)kFinBins / (mx - mn) : 0.f;
    const float neg_inv = -inv, hi_inv = mx * inv;

    // counting sort by bin
#pragma unroll
    for (int q = 0; q < kFinBins / 32; ++q) w.hist[lane + 32 * q] = 0u;
    __syncwarp();
    int bin[4];
    uint32_t in_bin[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        bin[i] = min((int)fmaxf(fmaf(v[i], neg_inv, hi_inv), 0.f), kFinBins - 1);
        in_bin[i] = live[i] ? atomicAdd(&w.hist[bin[i]], 1u) : 0u;
    }
    __syncwarp();
    {
        uint32_t hc[kFinBins / 32], tot = 0;
#pragma unroll
        for (int q = 0; q < kFinBins / 32; ++q) { hc[q] = w.hist[lane * (kFinBins / 32) + q]; tot += hc[q]; }
        uint32_t incl = tot;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t x = __shfl_up_sync(kFull, incl, o);
            if (lane >= o) incl += x;
        }
        uint32_t run_start = incl - tot;
        __syncwarp();
#pragma unroll
        for (int q = 0; q < kFinBins / 32; ++q) {
            w.hist[lane * (kFinBins / 32) + q] = run_start;
            run_start += hc[q];
        }
    }
    __syncwarp();
    uint64_t key[4];
    int start[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        key[i] = cand_key(v[i], jc[i] < 0 ? 0 : jc[i]);
        start[i] = (int)w.hist[bin[i]];
        if (live[i]) w.keys[start[i] + (int)in_bin[i]] = key[i];
    }
    __syncwarp();
    const int nr = min(L.k, n_valid);
    const int nm = min(L.m, n_valid - nr);
    const int nsel = nr + nm;
    const size_t grow = (size_t)h * L.nq + row;
    int32_t *out = L.ids + grow * L.c;
    bool sel[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        sel[i] = false;
        if (!live[i]) continue;
        const int end = bin[i] + 1 < kFinBins ? (int)w.hist[bin[i] + 1] : run;
        int rank = 0;
        for (int p = start[i]; p < end; ++p) rank += w.keys[p] > key[i] ? 1 : 0;
        const int pos = start[i] + rank;
        if (pos < nsel) {
            sel[i] = true;
            out[pos < nr ? pos : L.k + (pos - nr)] = jc[i];
            if (pos == nr - 1) L.alpha[grow] = v[i];
        }
    }
    for (int sl = lane; sl < L.k + L.m; sl += 32) {   // padding of short rows
        if (sl < L.k ? sl >= nr : sl - L.k >= nm) out[sl] = -1;
    }

    // random sentinels
    const bool use_bits = n_valid <= 32 * kFinBitsWords;
    if (use_bits) {
        const int words = (n_valid + 31) >> 5;
        for (int q = lane; q < words; q += 32) w.bits[q] = 0u;
        __syncwarp();
#pragma unroll
        for (int i = 0; i < 4; ++i)
            if (sel[i]) atomicOr(&w.bits[jc[i] >> 5], 1u << (jc[i] & 31));
        __syncwarp();
    }
    int acc = 0;
    // chunk j in route U near-miss, or accepted as a random sentinel (this
    // lane's j; accepted ones are in the bitmap, or in w.acc[0..acc))
    auto in_sel_or_acc = [&](int j) -> bool {
        if (use_bits) return ((w.bits[j >> 5] >> (j & 31)) & 1u) != 0u;
        bool hit = false;
        for (int src = 0; src < 32; ++src) {
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int cj = __shfl_sync(kFull, sel[i] ? jc[i] : -1, src);
                hit |= cj == j;
            }
        }
        for (int a = 0; a < acc; ++a) hit |= w.acc[a] == j;
        return hit;
    };
    // mandatory global sentinels (g <= 32): lane t examines candidate t; they
    // are written after the random block and leave the random pool
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
    // accept this round's free lanes in lane order, up to r in total
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
                                                  (uint32_t)layer, (uint32_t)(t >> 2), L.seed_lo,
                                                  L.seed_hi);
                const int q = t & 3;
                const uint32_t word = q == 0 ? o.w[0] : q == 1 ? o.w[1] : q == 2 ? o.w[2] : o.w[3];
                const int j = (int)__umulhi(word, (uint32_t)n_valid);
                const bool tk = taken(j);   // every lane calls it (it may shuffle)
                const bool ok_t = t < L.max_draws && !tk;
                // first draw of its chunk among this round's free draws
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

// ---- two-pass kernel with in-CTA row finishing ---------------------------------
// The allocation-free entry point's full routing: the epilogue warps finish
// their rows themselves (one warp per row, from the kept scores in shared
// memory), so the kernel needs no candidate buffers in device memory.
__global__ void __launch_bounds__(kPassThreads, 1)
route_rows_tc_kernel(LedgerDev L, const __nv_bfloat16 *__restrict__ Q,
                     const __grid_constant__ CUtensorMap tmap_k, int layer, int use_list) {
    extern __shared__ __align__(1024) unsigned char smem_dyn[];
    unsigned char *smem = align_smem_1024(smem_dyn);
    const int d = L.d, ksel = L.ksel;
    const Layout lay = layout_of(d, ksel, true);
    Cta c;
    if (!cta_setup(c, smem, lay.cta(), L, Q, L.list, L.head_count, use_list)) return;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int h = blockIdx.y;

    if (warp == 0) {
        producer(c, &tmap_k, d, h, 2);
    } else if (warp == 1) {
        mma_issuer(c, d, 2);
    } else {
        // Four warps per TMEM sub-partition: quarter qt reads columns
        // 32*qt..32*qt+31 of every tile.  The epilogue threads meet at named
        // barrier 1 between phases (every one of them reaches every barrier,
        // also after a timeout, so none can be left waiting).
        const int ew = warp - 2;   // epilogue warp 0..kEpiWarps-1
        const int sub = warp & 3;
        const int qt = ew >> 2;
        const int r = sub * 32 + lane;
        const int row = c.rows_s[r];
        const int n_valid = row >= 0 ? valid_keys(row, L.nk, L.causal) : 0;
        const uint32_t lane_base = c.tmem_base + ((uint32_t)(sub * 32) << 16) + (uint32_t)(qt * 32);
        const int nt = c.ntiles;
        bool ok = true;
        int g = 0;
        auto epi_sync = [] { asm volatile("bar.sync 1, %0;" ::"n"(kEpiWarps * 32) : "memory"); };
        int *rowcnt = reinterpret_cast<int *>(smem + lay.red) + kRows;   // [kRows] kept per row

        // pass 0: the two largest valid scores of each column group (this
        // quarter's columns, group = column mod 16)
        float m1[kGroups], m2[kGroups];
#pragma unroll
        for (int q = 0; q < kGroups; ++q) { m1[q] = -INFINITY; m2[q] = -INFINITY; }
        for (int i = 0; i < nt && ok; ++i, ++g) {
            if (!(ok = acc_wait(c, g))) break;
            float v[32];
            tc_ld32(lane_base + (uint32_t)((g % kAcc) * kKeys), v);
            acc_release(c, g);   // the scores are in registers: the MMA may reuse the accumulator
            const int col0 = i * kKeys + qt * 32;
            if (col0 + 32 <= n_valid) {
#pragma unroll
                for (int jj = 0; jj < 32; ++jj) {
                    const int q = jj & (kGroups - 1);
                    m2[q] = fmaxf(m2[q], fminf(m1[q], v[jj]));
                    m1[q] = fmaxf(m1[q], v[jj]);
                }
            } else {
#pragma unroll
                for (int jj = 0; jj < 32; ++jj) {
                    const int q = jj & (kGroups - 1);
                    const float x = col0 + jj < n_valid ? v[jj] : -INFINITY;
                    m2[q] = fmaxf(m2[q], fminf(m1[q], x));
                    m1[q] = fmaxf(m1[q], x);
                }
            }
        }
        // the row's 128 group tops: [r][kTopStride], this quarter at qt * 32
        float *tops = reinterpret_cast<float *>(smem + lay.sel);
#pragma unroll
        for (int q = 0; q < kGroups; ++q) {
            tops[r * kTopStride + qt * 2 * kGroups + q] = m1[q];
            tops[r * kTopStride + qt * 2 * kGroups + kGroups + q] = m2[q];
        }
        if (qt == 0) rowcnt[r] = 0;
        epi_sync();

        // threshold T of each row (kRows / kEpiWarps rows per warp): the
        // largest key K, a multiple of 2^kThrLowBit, that at least k + m of
        // the group tops' order-preserving keys reach.  At least k + m
        // distinct valid scores are >= T, so T is at most the row's (k + m)-th
        // best score.  Rows with at most k + m valid keys keep all of them
        // (T = -inf).
        float *thr_s = reinterpret_cast<float *>(smem + lay.red);   // [kRows]
        {
            constexpr int kRowsPerWarp = kRows / kEpiWarps;
            uint32_t key[kRowsPerWarp][4], K[kRowsPerWarp];
#pragma unroll
            for (int k2 = 0; k2 < kRowsPerWarp; ++k2) {
                const int rr = ew * kRowsPerWarp + k2;
#pragma unroll
                for (int i = 0; i < 4; ++i) key[k2][i] = ord32(tops[rr * kTopStride + i * 32 + lane]);
                K[k2] = 0u;
            }
            // the rows' searches interleaved (independent chains)
            for (int bit = 31; bit >= kThrLowBit; --bit) {
#pragma unroll
                for (int k2 = 0; k2 < kRowsPerWarp; ++k2) {
                    const uint32_t cand = K[k2] | (1u << bit);
                    const unsigned mine = (key[k2][0] >= cand ? 1u : 0u) + (key[k2][1] >= cand ? 1u : 0u) +
                                          (key[k2][2] >= cand ? 1u : 0u) + (key[k2][3] >= cand ? 1u : 0u);
                    if ((int)__reduce_add_sync(kFull, mine) >= ksel) K[k2] = cand;
                }
            }
#pragma unroll
            for (int k2 = 0; k2 < kRowsPerWarp; ++k2) {
                const int rr = ew * kRowsPerWarp + k2;
                const int rowr = c.rows_s[rr];
                const int nv = rowr >= 0 ? valid_keys(rowr, L.nk, L.causal) : 0;
                float t = unord32(K[k2]);
                if (nv <= ksel || t != t) t = -INFINITY;
                if (lane == k2) thr_s[rr] = t;
            }
        }
        epi_sync();
        const float T = thr_s[r];

        // pass 1: keep every valid score >= T.  Each thread builds a bit mask
        // of its kept columns for a round of 16, stages the round's scores
        // in shared memory (16-byte chunks swizzled by lane, so the stores do
        // not collide), claims that many slots of the row's buffer with one
        // atomic and appends the kept ones; no slot leaves the buffer.
        float *bv = reinterpret_cast<float *>(smem + lay.bufv) + r;
        uint16_t *bi = reinterpret_cast<uint16_t *>(smem + lay.bufi) + r;
        float *stg = reinterpret_cast<float *>(smem + lay.stg) + (ew * 32 + lane) * kStageCols;
        const int sw = (lane >> 1) & 3;   // 8 lanes of a 64-byte row stride: 8 distinct bank groups
        for (int i = 0; i < nt && ok; ++i, ++g) {
            if (!(ok = acc_wait(c, g))) break;
            const int t = tile_of(g, nt);
            float v[32];
            tc_ld32(lane_base + (uint32_t)((g % kAcc) * kKeys), v);
            acc_release(c, g);
            const int col0 = t * kKeys + qt * 32;
            const int lim = n_valid - col0;   // columns jj < lim are valid
#pragma unroll
            for (int hq = 0; hq < 32 / kStageCols; ++hq) {
                const int o = hq * kStageCols;
                // four independent partial masks (short dependency chains)
                uint32_t mk[4] = {0u, 0u, 0u, 0u};
                if (lim >= 32) {
#pragma unroll
                    for (int jj = 0; jj < kStageCols; ++jj)
                        mk[jj & 3] |= v[o + jj] >= T ? (1u << jj) : 0u;
                } else {
#pragma unroll
                    for (int jj = 0; jj < kStageCols; ++jj)
                        mk[jj & 3] |= (o + jj < lim && v[o + jj] >= T) ? (1u << jj) : 0u;
                }
                uint32_t mask = (mk[0] | mk[1]) | (mk[2] | mk[3]);
#pragma unroll
                for (int c4 = 0; c4 < kStageCols / 4; ++c4)
                    *reinterpret_cast<float4 *>(stg + ((c4 ^ sw) << 2)) =
                        make_float4(v[o + 4 * c4], v[o + 4 * c4 + 1], v[o + 4 * c4 + 2], v[o + 4 * c4 + 3]);
                if (mask != 0u) {
                    int sl = atomicAdd(&rowcnt[r], __popc(mask));
                    const int colo = col0 + o;
                    do {
                        const int jj = __ffs(mask) - 1;
                        mask &= mask - 1u;
                        if (sl < kCap) {
                            bv[sl * kBufStride] = stg[(((jj >> 2) ^ sw) << 2) + (jj & 3)];
                            bi[sl * kBufStride] = (uint16_t)(colo + jj);
                        }
                        ++sl;
                    } while (mask != 0u);
                }
            }
        }
        epi_sync();

        // A row is finished from its buffer when every wait succeeded, its
        // kept scores fit the buffer, and at least min(k + m, valid keys) were
        // kept; other rows go to the retry list (exact heap selection).
        const bool cta_ok = *c.abort_flag == 0;
        auto row_good = [&](int rw, int nv, int kept) {
            return cta_ok && rw >= 0 && kept <= kCap && (nv <= ksel ? kept == nv : kept >= ksel);
        };
        const int kept = rowcnt[r];
        const bool good = row_good(row, n_valid, kept);
        if (qt == 0 && ok && row >= 0 && !good) {
            const int pos = atomicAdd(&L.retry_count[h], 1);
            L.retry_list[(size_t)h * L.nq + pos] = row;
            atomicAdd(&L.counters[10], 1ULL);
        }

        // finish the rows here (kRows / kEpiWarps per warp), the warps'
        // scratch in the query/key buffers (every MMA is done)
        FinWarp &fw = reinterpret_cast<FinWarp *>(smem + lay.q)[ew];
        const float *bvb = reinterpret_cast<const float *>(smem + lay.bufv);
        const uint16_t *bib = reinterpret_cast<const uint16_t *>(smem + lay.bufi);
        for (int k2 = 0; k2 < kRows / kEpiWarps; ++k2) {
            const int rr = ew * (kRows / kEpiWarps) + k2;
            const int rowr = c.rows_s[rr];
            const int nv = rowr >= 0 ? valid_keys(rowr, L.nk, L.causal) : 0;
            const int kr = rowcnt[rr];
            if (!row_good(rowr, nv, kr)) continue;   // warp-uniform
            finish_row(
                L, layer, h, rowr, kr, [&](int e) { return bvb[e * kBufStride + rr]; },
                [&](int e) { return (int)bib[e * kBufStride + rr]; }, fw, lane);
        }
    }
    cta_teardown(c, L);
}

// ---- relay rescoring on the tensor cores ---------------------------------------
// The relay test of RouteRelay §3.2 (Eq. 5-8) for every row of a head: alpha =
// min over the row's route ids of s_ij, beta = max over its sentinel ids
// (near-miss and random), flag = !(alpha > beta + gamma); a stable row keeps
// its ids and stores alpha.  The candidates' scores are read from dense
// 128 x 128 score tiles (one MMA pass over the row block's key tiles): on
// B200 the tensor cores score a whole tile in about the time it takes to
// gather the 80 candidate key rows of a few query rows.  Each row's
// candidates are marked in two bitmaps (route, sentinel) of one 2048-column
// segment at a time; the epilogue folds every marked score of a tile into the
// row's running min / max.
constexpr int kSegCols = 2048;                  // key columns per bitmap segment
constexpr int kSegWords = kSegCols / 32;
constexpr int kSegStride = kSegWords + 1;       // padded row: distinct banks across rows
constexpr int kRescoreIdsPerThread = (64 + kBuf + 3) / 4;   // ledger ids per quarter thread (c <= 96)

__host__ __device__ inline Layout rescore_layout(int d) {
    Layout s;
    s.stages = d == 64 ? 4 : 3;
    uint32_t o = 0;
    s.q = o;    o = up(o + kRows * d * 2, 1024);
    s.k = o;    o = up(o + s.stages * kKeys * d * 2, 1024);
    s.sel = o;  o = up(o + 2 * kRows * kSegStride * 4, 16);   // route bits | sentinel bits
    s.bufv = s.bufi = s.stg = 0;
    s.rows = o; o = up(o + kRows * 4, 16);
    s.red = o;  o = up(o + 3 * 4 * kRows * 4, 16);   // per quarter: alpha, beta, candidates | bad
    s.bars = o; o = up(o + 8 * (2 * kMaxStages + 2 * kAcc + 1), 16);
    s.misc = o; o = up(o + 16, 16);
    s.total = o + 1024;
    return s;
}

__global__ void __launch_bounds__(kPassThreads, 1)
relay_rescore_tc_kernel(LedgerDev L, const __nv_bfloat16 *__restrict__ Q,
                        const __grid_constant__ CUtensorMap tmap_k, int layer) {
    extern __shared__ __align__(1024) unsigned char smem_dyn[];
    unsigned char *smem = align_smem_1024(smem_dyn);
    const int d = L.d;
    const Layout lay = rescore_layout(d);
    Cta c;
    if (!cta_setup(c, smem, lay.cta(), L, Q, L.list, L.head_count, 0)) return;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int h = blockIdx.y;

    if (warp == 0) {
        producer(c, &tmap_k, d, h, 1);
    } else if (warp == 1) {
        mma_issuer(c, d, 1);
    } else {
        const int ew = warp - 2;
        const int sub = warp & 3;
        const int qt = ew >> 2;   // quarter of the tile's columns
        const int r = sub * 32 + lane;
        const int row = c.rows_s[r];
        const int n_valid = row >= 0 ? valid_keys(row, L.nk, L.causal) : 0;
        const uint32_t lane_base = c.tmem_base + ((uint32_t)(sub * 32) << 16) + (uint32_t)(qt * 32);
        const int nt = c.ntiles;
        auto epi_sync = [] { asm volatile("bar.sync 1, %0;" ::"n"(kEpiWarps * 32) : "memory"); };
        uint32_t *rbits = reinterpret_cast<uint32_t *>(smem + lay.sel);   // [kRows][kSegStride]
        uint32_t *sbits = rbits + kRows * kSegStride;
        const int32_t *idr = L.ids + ((size_t)h * L.nq + (row >= 0 ? row : 0)) * L.c;

        // this quarter's share of the row's ids (slots qt, qt+4, ...), loaded
        // once: count the valid candidates (Eq. 5) and flag out-of-range ids;
        // invalid slots become -1
        int jid[kRescoreIdsPerThread];
        int ncand = 0;
        bool bad = false;
#pragma unroll
        for (int i = 0; i < kRescoreIdsPerThread; ++i) {
            const int e = qt + 4 * i;
            const int j = (row >= 0 && e < L.c) ? idr[e] : -1;
            const bool valid = j >= 0 && j < n_valid;
            ncand += valid ? 1 : 0;
            bad |= j >= n_valid || j < -1;
            jid[i] = valid ? j : -1;
        }
        float amin = INFINITY, bmax = -INFINITY;
        bool ok = true;
        int g = 0;
        const int nseg = (nt * kKeys + kSegCols - 1) / kSegCols;
        for (int sg = 0; sg < nseg; ++sg) {
            for (int w = qt; w < kSegWords; w += 4) {
                rbits[r * kSegStride + w] = 0u;
                sbits[r * kSegStride + w] = 0u;
            }
            epi_sync();
#pragma unroll
            for (int i = 0; i < kRescoreIdsPerThread; ++i) {
                const int j = jid[i];
                if (j >= 0 && j / kSegCols == sg) {
                    const int jj = j - sg * kSegCols;
                    atomicOr(&(qt + 4 * i < L.k ? rbits : sbits)[r * kSegStride + (jj >> 5)],
                             1u << (jj & 31));
                }
            }
            epi_sync();
            const int t_end = min(nt, (sg + 1) * (kSegCols / kKeys));
            for (; g < t_end && ok; ++g) {   // one pass: tile index = g
                if (!(ok = acc_wait(c, g))) break;
                float v[32];
                tc_ld32(lane_base + (uint32_t)((g % kAcc) * kKeys), v);
                acc_release(c, g);
                const int wi = (g * kKeys + qt * 32 - sg * kSegCols) >> 5;
                const uint32_t rw = rbits[r * kSegStride + wi];
                const uint32_t sw = sbits[r * kSegStride + wi];
#pragma unroll
                for (int jj = 0; jj < 32; ++jj) {
                    amin = fminf(amin, ((rw >> jj) & 1u) ? v[jj] : INFINITY);   // Eq. 6
                    bmax = fmaxf(bmax, ((sw >> jj) & 1u) ? v[jj] : -INFINITY);  // Eq. 7
                }
            }
            epi_sync();   // the segment's bitmaps are no longer read
        }

        float *red_a = reinterpret_cast<float *>(smem + lay.red);   // [4][kRows]
        float *red_b = red_a + 4 * kRows;
        int *red_n = reinterpret_cast<int *>(red_b + 4 * kRows);
        red_a[qt * kRows + r] = amin;
        red_b[qt * kRows + r] = bmax;
        red_n[qt * kRows + r] = ncand | (bad ? (1 << 30) : 0);
        epi_sync();
        const bool cta_ok = *c.abort_flag == 0;
        unsigned pairs = 0;
        if (qt == 0) {
            float a = red_a[r], b = red_b[r];
            int n = red_n[r];
            for (int q = 1; q < 4; ++q) {
                a = fminf(a, red_a[q * kRows + r]);
                b = fmaxf(b, red_b[q * kRows + r]);
                n |= red_n[q * kRows + r] & (1 << 30);
                n += red_n[q * kRows + r] & ((1 << 30) - 1);
            }
            if (cta_ok && row >= 0) {
                const size_t grow = (size_t)h * L.nq + row;
                const uint8_t fl = relay_decide(L, grow, layer, a, b);   // Eq. 8
                const bool refresh = (fl & 1u) != 0u;
                L.flags[grow] = fl;
                if (!refresh) L.alpha[grow] = a;
                if (n & (1 << 30)) atomicOr(&L.counters[2], 1ULL);
                pairs = (unsigned)(n & ((1 << 30) - 1));
            } else if (row >= 0) {
                // a wait timed out (bit 1 of the error word): the row's scores
                // are unknown, so it is flagged and the refresh rebuilds it
                // rather than keeping a route no test confirmed
                L.flags[(size_t)h * L.nq + row] = 1;
            }
            const unsigned wsum = __reduce_add_sync(kFull, pairs);
            if (lane == 0 && wsum) atomicAdd(&L.counters[1], (unsigned long long)wsum);
        }
    }
    cta_teardown(c, L);
}

// ---- host side -----------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static bool tried = false;
    if (!tried) {
        tried = true;
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    }
    return fn;
}

cudaError_t key_tensor_map(const LedgerDev &L, const void *k, CUtensorMap *map) {
    return key_rows_tensor_map(k, L.d, L.nk, L.bh, map);
}

cudaError_t key_rows_tensor_map(const void *k, int row_elems, int nk, int bh, CUtensorMap *map) {
    EncodeTiledFn enc = encode_fn();
    if (!enc || row_elems % 64 != 0) return cudaErrorNotSupported;
    const cuuint64_t dims[3] = {(cuuint64_t)row_elems, (cuuint64_t)nk, (cuuint64_t)bh};
    const cuuint64_t strides[2] = {(cuuint64_t)row_elems * 2, (cuuint64_t)nk * row_elems * 2};
    const cuuint32_t box[3] = {64u, (cuuint32_t)kKeys, 1u};
    const cuuint32_t estr[3] = {1u, 1u, 1u};
    const CUresult cr = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(k), dims,
                            strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return cr == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

}  // namespace tc

bool route_rows_tc_supported(const LedgerDev &L, int dtype) {
    if (!(dtype == kBF16 && (L.d == 64 || L.d == 128) && L.ksel <= 64 && L.r <= tc::kBuf &&
          L.nk <= 65535 && L.c <= 4 * tc::kRescoreIdsPerThread))
        return false;
    // the fused kernel finishes its rows with per-warp scratch in the
    // query/key buffers
    const tc::Layout lay = tc::layout_of(L.d, L.ksel, true);
    const tc::Layout layh = tc::layout_of(L.d, L.ksel, false);
    return lay.total <= 232448 && layh.total <= 232448 && tc::rescore_layout(L.d).total <= 232448 &&
           lay.sel - lay.q >= (uint32_t)(tc::kEpiWarps * sizeof(tc::FinWarp)) &&
           route_select_smem_bytes(L) <= 232448;
}

cudaError_t route_rows_tc_prepare() {
    // the kernels may be launched with up to their largest layout
    const int big = (int)tc::layout_of(128, 64, true).total;
    const int big_heap = (int)tc::layout_of(128, 64, false).total;
    cudaError_t e = cudaFuncSetAttribute(tc::route_rows_tc_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, big);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(tc::route_rows_tc_heap_kernel,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, big_heap);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(tc::relay_rescore_tc_kernel,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)tc::rescore_layout(128).total);
    if (e == cudaSuccess) e = route_select_prepare();
    return e;
}

cudaError_t launch_relay_rescore_tc(const LedgerDev &L, const void *q, const void *k, int layer,
                                    cudaStream_t s) {
    CUtensorMap map;
    cudaError_t e = tc::key_tensor_map(L, k, &map);
    if (e != cudaSuccess) return e;
    dim3 grid((L.nq + tc::kRows - 1) / tc::kRows, L.bh);
    tc::relay_rescore_tc_kernel<<<grid, tc::kPassThreads, tc::rescore_layout(L.d).total, s>>>(
        L, static_cast<const __nv_bfloat16 *>(q), map, layer);
    return cudaGetLastError();
}

cudaError_t launch_route_rows_tc(const LedgerDev &L, const void *q, const void *k, int layer,
                                 bool use_list, cudaStream_t s) {
    CUtensorMap map;
    cudaError_t e = tc::key_tensor_map(L, k, &map);
    if (e != cudaSuccess) return e;
    e = cudaMemsetAsync(L.retry_count, 0, (size_t)L.bh * sizeof(int32_t), s);
    if (e != cudaSuccess) return e;
    dim3 grid((L.nq + tc::kRows - 1) / tc::kRows, L.bh);
    if (L.cand_keys) {
        // selection kernel + row finishing (rr_select_tc.cu); overflowed rows
        // on the CUDA cores
        e = launch_route_select(L, q, map, layer, use_list, SelectMode::kAnchor, s);
        if (e != cudaSuccess) return e;
        return launch_retry_rows_simt(L, q, k, layer, s);
    } else {
        const size_t smem2 = tc::layout_of(L.d, L.ksel, true).total;
        tc::route_rows_tc_kernel<<<grid, tc::kPassThreads, smem2, s>>>(
            L, static_cast<const __nv_bfloat16 *>(q), map, layer, use_list ? 1 : 0);
        e = cudaGetLastError();
    }
    if (e != cudaSuccess) return e;
    return launch_route_retry(L, q, map, layer, s);
}

cudaError_t launch_route_retry(const LedgerDev &L, const void *q, const CUtensorMap &map, int layer,
                               cudaStream_t s) {
    // rows the two-pass kernels could not finish: exact heap selection
    LedgerDev R = L;
    R.list = L.retry_list;
    R.head_count = L.retry_count;
    dim3 grid((L.nq + tc::kRows - 1) / tc::kRows, L.bh);
    const size_t smemh = tc::layout_of(L.d, L.ksel, false).total;
    tc::route_rows_tc_heap_kernel<<<grid, tc::kHeapThreads, smemh, s>>>(
        R, static_cast<const __nv_bfloat16 *>(q), map, layer, 1);
    return cudaGetLastError();
}

}  // namespace rr
