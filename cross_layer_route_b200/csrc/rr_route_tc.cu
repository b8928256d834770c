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
// per-head list).
//
// CTA layout (one CTA = one head x 128 query rows; 6 warps):
//   warp 0   TMA producer: 128-key x d tiles of Kc (bf16, 128-byte swizzle)
//            into a 2-stage shared-memory ring.
//   warp 1   allocates 256 TMEM columns (two 128x128 fp32 accumulators) and
//            one lane issues tcgen05.mma (M=128, N=128, K=16 per op) for
//            every key tile, committing to mbarriers.
//   warps 2-5  epilogue, one thread per query row (= TMEM lane): reads its
//            row's 128 scores of a tile with tcgen05.ld, keeps those at or
//            above the row's running threshold in a small append buffer, and
//            folds the buffer into a per-row min-heap of the k + m best (the
//            heap's root is the threshold).  Finally heap-sorts, draws the
//            random sentinels and writes the ledger row.
// The query tile is gathered by row index into the same swizzled layout
// the TMA would produce, so anchor and refresh share one code path.
// Every wait is bounded; a timeout sets bit 1 of the error word and the CTA
// drains its copies, frees its TMEM and returns.
#include <cuda.h>
#include <float.h>
#include <limits.h>

#include "rr_device.cuh"
#include "rr_internal.h"

namespace rr {
namespace tc {

constexpr int kRows = 128;
constexpr int kKeys = 128;
constexpr int kStages = 2;
constexpr int kEpiWarps = 4;
constexpr int kThreads = 32 * (2 + kEpiWarps);
constexpr int kBuf = 32;
constexpr int kTmemCols = 256;
constexpr int kSubTileBytes = 128 * 128;   // 128 rows x 64 bf16 (one 128-byte swizzle span)
constexpr long long kSpinLimit = 1ll << 31;

struct Layout {
    uint32_t q, k, heap, bufv, bufi, rows, bars, misc, total;
};

__host__ __device__ inline uint32_t up(uint32_t x, uint32_t a) { return (x + a - 1) / a * a; }

__host__ __device__ inline Layout layout_of(int d, int ksel) {
    Layout s;
    uint32_t o = 0;
    s.q = o;    o = up(o + kRows * d * 2, 1024);
    s.k = o;    o = up(o + kStages * kKeys * d * 2, 1024);
    s.heap = o; o = up(o + kRows * ksel * 8, 16);
    s.bufv = o; o = up(o + kRows * kBuf * 4, 16);
    s.bufi = o; o = up(o + kRows * kBuf * 4, 16);
    s.rows = o; o = up(o + kRows * 4, 16);
    s.bars = o; o = up(o + 8 * (2 * kStages + 5), 16);
    s.misc = o; o = up(o + 16, 16);
    s.total = o + 1024;   // slack for aligning the dynamic base to 1024
    return s;
}

// ---- PTX wrappers (forms from the PTX ISA for sm_100a) -----------------------
__device__ __forceinline__ uint32_t saddr(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void mbar_init(uint64_t *b, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(saddr(b)), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint64_t *b, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(saddr(b)), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t *b) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(saddr(b)) : "memory");
}
__device__ __forceinline__ bool mbar_test(uint64_t *b, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(saddr(b)), "r"(parity)
        : "memory");
    return ok != 0;
}
// Bounded wait for the phase of the given parity.  Returns false on timeout
// (and raises the CTA's abort flag) or when another role already aborted.
__device__ __forceinline__ bool mbar_wait(uint64_t *b, uint32_t parity, volatile int *abort_flag) {
    if (mbar_test(b, parity)) return true;
    const long long t0 = clock64();
    while (!mbar_test(b, parity)) {
        if (*abort_flag) return false;
        if (clock64() - t0 > kSpinLimit) {
            *abort_flag = 1;
            return false;
        }
    }
    return true;
}
__device__ __forceinline__ void tma_load_3d(void *dst, const CUtensorMap *map, uint64_t *bar, int c0,
                                            int c1, int c2) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(saddr(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(saddr(bar)), "r"(c0), "r"(c1), "r"(c2)
        : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_commit(uint64_t *bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     saddr(bar))
                 : "memory");
}
__device__ __forceinline__ void tc_mma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                            uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}
// 32 lanes x 32 consecutive fp32 columns; thread t gets its lane's 32 values.
__device__ __forceinline__ void tc_ld32(uint32_t taddr, float *v) {
    uint32_t r[32];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, "
        "%12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, "
        "%30, %31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
          "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
          "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
          "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

// Shared-memory matrix descriptor of a K-major operand stored as 128-byte
// swizzled rows (8-row groups 1024 bytes apart): start address >> 4, leading
// byte offset 16 B, stride byte offset 1024 B, descriptor version 1,
// layout "128-byte swizzle".
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr_bytes) {
    return (uint64_t)((saddr_bytes >> 4) & 0x3FFFu) | ((uint64_t)1u << 16) |
           ((uint64_t)(1024u >> 4) << 32) | ((uint64_t)1u << 46) | ((uint64_t)2u << 61);
}
// Instruction descriptor: fp32 accumulator, bf16 A and B, both K-major,
// N = 128 (bits 17..22 hold N/8), M = 128 (bits 24..28 hold M/16).
constexpr uint32_t kIdesc = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(kKeys >> 3) << 17) |
                            ((uint32_t)(kRows >> 4) << 24);

// ---- per-row selection (one thread per row) ------------------------------------
// Keys order (score, chunk) pairs: larger key = higher score, then smaller chunk.
__device__ __forceinline__ uint32_t ord32(float f) {
    const uint32_t u = __float_as_uint(f);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float unord32(uint32_t o) {
    return __uint_as_float((o & 0x80000000u) ? (o & 0x7FFFFFFFu) : ~o);
}
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

__device__ __forceinline__ bool in_keys(const uint64_t *H, int n, int j) {
    for (int e = 0; e < n; ++e)
        if (key_chunk(H[e * kRows]) == j) return true;
    return false;
}
__device__ __forceinline__ bool in_ints(const int *B, int n, int j) {
    for (int e = 0; e < n; ++e)
        if (B[e * kRows] == j) return true;
    return false;
}

__global__ void __launch_bounds__(kThreads, 1)
route_rows_tc_kernel(LedgerDev L, const __nv_bfloat16 *__restrict__ Q,
                     const __grid_constant__ CUtensorMap tmap_k, int layer, int use_list) {
    extern __shared__ __align__(1024) unsigned char smem_dyn[];
    unsigned char *smem = reinterpret_cast<unsigned char *>(
        (reinterpret_cast<uintptr_t>(smem_dyn) + 1023) & ~uintptr_t(1023));
    const int d = L.d;
    const int ksel = L.ksel;
    const Layout lay = layout_of(d, ksel);
    unsigned char *q_s = smem + lay.q;
    unsigned char *k_s = smem + lay.k;
    uint64_t *heap_all = reinterpret_cast<uint64_t *>(smem + lay.heap);
    float *bufv_all = reinterpret_cast<float *>(smem + lay.bufv);
    int *bufi_all = reinterpret_cast<int *>(smem + lay.bufi);
    int *rows_s = reinterpret_cast<int *>(smem + lay.rows);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + lay.bars);
    uint64_t *full = bars;                  // [kStages]
    uint64_t *empty = bars + kStages;       // [kStages]
    uint64_t *acc_full = bars + 2 * kStages;       // [2]
    uint64_t *acc_empty = bars + 2 * kStages + 2;  // [2]
    uint64_t *mma_done = bars + 2 * kStages + 4;   // [1]
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + lay.misc);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + lay.misc + 4);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int h = blockIdx.y;
    const int nq = L.nq, nk = L.nk;
    const int count = use_list ? L.head_count[h] : nq;
    const int row0 = blockIdx.x * kRows;
    if (row0 >= count) return;
    const int n_rows = min(kRows, count - row0);

    if (tid < kRows) {
        int row = -1;
        if (tid < n_rows) row = use_list ? L.list[(size_t)h * nq + row0 + tid] : row0 + tid;
        rows_s[tid] = row;
    }
    if (tid == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&acc_full[a], 1);
            mbar_init(&acc_empty[a], kEpiWarps);
        }
        mbar_init(mma_done, 1);
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         saddr(tmem_slot)),
                     "r"(kTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    __syncthreads();

    // query tile: gather rows by index into the 128-byte-swizzled K-major
    // layout (row r, 16-byte chunk c of its 64-element half kb lands at
    // kb*16KB + r*128 + ((c ^ (r & 7)) * 16)).
    const int c16 = d >> 3;  // 16-byte chunks per row
    for (int e = tid; e < kRows * c16; e += kThreads) {
        const int r = e / c16, c = e - r * c16;
        const int row = rows_s[r];
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        if (row >= 0) v = *reinterpret_cast<const uint4 *>(Q + ((size_t)h * nq + row) * d + c * 8);
        const int kb = c >> 3, cc = c & 7;
        *reinterpret_cast<uint4 *>(q_s + kb * kSubTileBytes + r * 128 + ((cc ^ (r & 7)) << 4)) = v;
    }
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    int max_row = -1;
    for (int e = 0; e < n_rows; ++e) max_row = max(max_row, rows_s[e]);
    const int kend = L.causal ? min(nk, max_row + 1) : nk;
    const int ntiles = (kend + kKeys - 1) / kKeys;
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    if (warp == 0) {
        // ---------------- TMA producer ----------------
        if (lane == 0) {
            asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmap_k))
                         : "memory");
            int issued = 0;
            for (int t = 0; t < ntiles; ++t) {
                const int s = t % kStages;
                if (!mbar_wait(&empty[s], ((t / kStages) & 1) ^ 1, abort_flag)) break;
                mbar_expect_tx(&full[s], (uint32_t)(kKeys * d * 2));
                for (int kb = 0; kb < (d >> 6); ++kb)
                    tma_load_3d(k_s + s * (kKeys * d * 2) + kb * kSubTileBytes, &tmap_k, &full[s],
                                kb * 64, t * kKeys, h);
                ++issued;
            }
            // drain: every issued stage must have landed before the CTA exits
            for (int t = max(0, issued - kStages); t < issued; ++t) {
                const int s = t % kStages;
                const long long t0 = clock64();
                while (!mbar_test(&full[s], (t / kStages) & 1) && clock64() - t0 < kSpinLimit) {
                }
            }
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer ----------------
        if (lane == 0) {
            const uint32_t q_addr = saddr(q_s), k_addr = saddr(k_s);
            for (int t = 0; t < ntiles; ++t) {
                const int s = t % kStages, a = t & 1;
                if (!mbar_wait(&full[s], (t / kStages) & 1, abort_flag)) break;
                if (!mbar_wait(&acc_empty[a], ((t >> 1) & 1) ^ 1, abort_flag)) break;
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + (uint32_t)(a * kKeys);
                const uint32_t kst = k_addr + (uint32_t)(s * kKeys * d * 2);
                for (int kk = 0; kk < (d >> 4); ++kk) {
                    const uint32_t off = (uint32_t)((kk >> 2) * kSubTileBytes + (kk & 3) * 32);
                    tc_mma_bf16(d_tmem, sw128_desc(q_addr + off), sw128_desc(kst + off), kIdesc,
                                kk > 0 ? 1u : 0u);
                }
                tc_commit(&empty[s]);
                tc_commit(&acc_full[a]);
            }
            tc_commit(mma_done);
            const long long t0 = clock64();
            while (!mbar_test(mma_done, 0) && clock64() - t0 < kSpinLimit) {
            }
        }
    } else {
        // ---------------- epilogue: one thread per query row ----------------
        const int sub = warp & 3;            // TMEM sub-partition this warp may read
        const int r = sub * 32 + lane;       // row slot = TMEM lane = query tile row
        const int row = rows_s[r];
        const int n_valid = row >= 0 ? valid_keys(row, nk, L.causal) : 0;
        uint64_t *H = heap_all + r;
        float *bv = bufv_all + r;
        int *bi = bufi_all + r;
        for (int e = 0; e < ksel; ++e) H[e * kRows] = 0ull;
        float thr = -INFINITY;
        bool ok = true;
        for (int t = 0; t < ntiles && ok; ++t) {
            const int a = t & 1;
            ok = mbar_wait(&acc_full[a], (t >> 1) & 1, abort_flag);
            ok = __all_sync(kFull, ok);   // the warp leaves together (tcgen05.ld is .sync.aligned)
            if (!ok) break;
            tc_fence_after();
            const uint32_t tbase = tmem_base + ((uint32_t)(sub * 32) << 16) + (uint32_t)(a * kKeys);
#pragma unroll 1
            for (int ch = 0; ch < kKeys / 32; ++ch) {
                float v[32];
                tc_ld32(tbase + (uint32_t)(ch * 32), v);
                const int col0 = t * kKeys + ch * 32;
                int cnt = 0;
                if (col0 + 32 <= n_valid) {
#pragma unroll
                    for (int jj = 0; jj < 32; ++jj) {
                        if (v[jj] >= thr) {
                            bv[cnt * kRows] = v[jj];
                            bi[cnt * kRows] = col0 + jj;
                            ++cnt;
                        }
                    }
                } else {
#pragma unroll
                    for (int jj = 0; jj < 32; ++jj) {
                        if (col0 + jj < n_valid && v[jj] >= thr) {
                            bv[cnt * kRows] = v[jj];
                            bi[cnt * kRows] = col0 + jj;
                            ++cnt;
                        }
                    }
                }
                // fold this chunk's survivors into the heap
                for (int e = 0; e < cnt; ++e) {
                    const uint64_t key = make_key(bv[e * kRows], bi[e * kRows]);
                    if (key > H[0]) heap_sift(H, ksel, key);
                }
                const uint64_t root = H[0];
                thr = root == 0ull ? -INFINITY : key_score(root);
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&acc_empty[a]);
        }
        if (!ok) {
            if (lane == 0) atomicOr(&L.counters[2], 2ULL);
        } else if (row >= 0) {
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
            const size_t grow = (size_t)h * nq + row;
            int32_t *out = L.ids + grow * L.c;
            for (int e = 0; e < L.k; ++e) out[e] = e < nr ? key_chunk(H[e * kRows]) : -1;
            for (int e = 0; e < L.m; ++e) out[L.k + e] = e < nm ? key_chunk(H[(nr + e) * kRows]) : -1;
            // random sentinels (RouteRelay §3.1 item 2, §3.4); accepted ids in bi[]
            int acc = 0;
            if (L.r > 0) {
                const int np = n_valid - nsel;
                if (np > L.r) {
                    uint32_t w4[4] = {0u, 0u, 0u, 0u};
                    int t = 0;
                    for (; acc < L.r && t < L.max_draws; ++t) {
                        if ((t & 3) == 0) {
                            const PhiloxOut o = philox4x32_10((uint32_t)(L.bh_offset + h), (uint32_t)row,
                                                              (uint32_t)layer, (uint32_t)(t >> 2),
                                                              L.seed_lo, L.seed_hi);
                            w4[0] = o.w[0]; w4[1] = o.w[1]; w4[2] = o.w[2]; w4[3] = o.w[3];
                        }
                        const int sel = t & 3;
                        const uint32_t w = sel == 0 ? w4[0] : sel == 1 ? w4[1] : sel == 2 ? w4[2] : w4[3];
                        const int j = (int)__umulhi(w, (uint32_t)n_valid);
                        if (in_keys(H, nsel, j) || in_ints(bi, acc, j)) continue;
                        bi[acc * kRows] = j;
                        ++acc;
                    }
                    if (acc < L.r) atomicAdd(&L.counters[7], 1ULL);
                }
                for (int j = 0; acc < L.r && j < n_valid; ++j) {
                    if (in_keys(H, nsel, j) || in_ints(bi, acc, j)) continue;
                    bi[acc * kRows] = j;
                    ++acc;
                }
            }
            for (int e = 0; e < L.r; ++e) out[L.k + L.m + e] = e < acc ? bi[e * kRows] : -1;
            L.alpha[grow] = key_score(H[(nr - 1) * kRows]);
            L.anchor_layer[grow] = layer;
            L.flags[grow] = 1;
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
    if (tid == 0 && *abort_flag) atomicOr(&L.counters[2], 2ULL);
}

// ---- host side -----------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
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

}  // namespace tc

bool route_rows_tc_supported(const LedgerDev &L, int dtype) {
    return dtype == kBF16 && (L.d == 64 || L.d == 128) && L.ksel <= 64 && L.r <= tc::kBuf;
}

size_t route_rows_tc_smem_bytes(const LedgerDev &L) { return tc::layout_of(L.d, L.ksel).total; }

cudaError_t route_rows_tc_prepare(size_t smem_bytes) {
    return cudaFuncSetAttribute(tc::route_rows_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)smem_bytes);
}

cudaError_t launch_route_rows_tc(const LedgerDev &L, const void *q, const void *k, int layer,
                                 bool use_list, cudaStream_t s) {
    tc::EncodeTiledFn enc = tc::encode_fn();
    if (!enc) return cudaErrorNotSupported;
    CUtensorMap map;
    const cuuint64_t dims[3] = {(cuuint64_t)L.d, (cuuint64_t)L.nk, (cuuint64_t)L.bh};
    const cuuint64_t strides[2] = {(cuuint64_t)L.d * 2, (cuuint64_t)L.nk * L.d * 2};
    const cuuint32_t box[3] = {64u, (cuuint32_t)tc::kKeys, 1u};
    const cuuint32_t estr[3] = {1u, 1u, 1u};
    const CUresult cr = enc(&map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(k), dims,
                            strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (cr != CUDA_SUCCESS) return cudaErrorInvalidValue;
    const size_t smem = tc::layout_of(L.d, L.ksel).total;
    dim3 grid((L.nq + tc::kRows - 1) / tc::kRows, L.bh);
    tc::route_rows_tc_kernel<<<grid, tc::kThreads, smem, s>>>(
        L, static_cast<const __nv_bfloat16 *>(q), map, layer, use_list ? 1 : 0);
    return cudaGetLastError();
}

}  // namespace rr
