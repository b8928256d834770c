// rr_tc.cuh -- Blackwell tensor-core machinery shared by the score-tile kernels.
//
// Method: "RouteRelay: Event-Triggered Cross-Layer Route Reuse for Efficient
// Dynamic Sparse Attention" (arXiv 2609.07306), cited as RouteRelay §x.
//
// Every kernel built on this header scores 128 query rows of one head
// against that head's key chunks (S = Qc Kc^T, §2.1 Eq. 1) in 128 x 128
// tiles on the tensor cores:
//   warp 0     TMA producer: 128-key x d tiles of Kc (bf16, 128-byte
//              swizzle) into a ring of shared-memory stages;
//   warp 1     allocates 512 TMEM columns (four 128x128 fp32 accumulators);
//              one elected lane issues tcgen05.mma (M=128, N=128, K=16 per
//              op) for every key tile and commits twice: to the stage's "empty"
//              barrier (the producer may refill it) and to the
//              accumulator's "full" barrier (the epilogue may read it);
//   warps 2-   epilogue, reading score tiles with tcgen05.ld; a warp may
//              only read the 32 TMEM lanes (= query rows) of its
//              sub-partition (warp index mod 4).
// The query tile is gathered by row index into the layout a 128-byte
// swizzled TMA load would produce, so rows may come from a list.
//
// Every wait is bounded; a timeout raises the CTA's abort flag, every role
// stops issuing, the producer drains the copies it issued, the MMA lane
// waits for its last commit, and teardown frees TMEM and sets bit 1 of the
// ledger's error word.
#pragma once

#include <cuda.h>
#include <float.h>
#include <limits.h>

#include "rr_device.cuh"
#include "rr_internal.h"

namespace rr {
namespace tc {

constexpr int kRows = 128;
constexpr int kKeys = 128;
constexpr int kMaxStages = 8;
constexpr int kAcc = 4;                    // TMEM accumulators (128 columns each)
constexpr int kTmemCols = kAcc * 128;
constexpr int kSubTileBytes = 128 * 128;   // 128 rows x 64 bf16 (one 128-byte swizzle span)
constexpr long long kSpinLimit = 1ll << 31;
constexpr int kNumBars = 2 * kMaxStages + 2 * kAcc + 2;

__host__ __device__ inline uint32_t up(uint32_t x, uint32_t a) { return (x + a - 1) / a * a; }

// ---- PTX wrappers (forms from the PTX ISA for sm_100a) -----------------------
__device__ __forceinline__ uint32_t saddr(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
// The dynamic shared-memory base rounded up to 1024 bytes (128-byte swizzled
// operands need it).  The offset is added to the shared array itself, so the
// compiler keeps the shared address space of every pointer derived from it.
__device__ __forceinline__ unsigned char *align_smem_1024(unsigned char *base) {
    return base + ((1024u - (saddr(base) & 1023u)) & 1023u);
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
// The same test, letting the thread sleep up to ~8 us until the phase
// completes (a waiting warp then takes no issue slots from the warps that
// share its scheduler).
__device__ __forceinline__ bool mbar_test_sleep(uint64_t *b, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(saddr(b)), "r"(parity), "r"(8192u)
        : "memory");
    return ok != 0;
}
// Non-blocking test of the phase (try_wait above may hold the thread for a
// while before it answers; test_wait answers at once).
__device__ __forceinline__ bool mbar_poll(uint64_t *b, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(saddr(b)), "r"(parity)
        : "memory");
    return ok != 0;
}
// Bounded wait for the phase of the given parity.  Returns false on timeout
// (and raises the CTA's abort flag) or when another role already aborted.
// A limit below the default polls with test_wait, so that the limit and not
// the hardware's own wait inside try_wait decides when the wait ends.
__device__ __forceinline__ bool mbar_wait(uint64_t *b, uint32_t parity, volatile int *abort_flag,
                                          long long limit = kSpinLimit) {
    if (limit < kSpinLimit) {
        const long long t0 = clock64();
        while (!mbar_poll(b, parity)) {
            if (*abort_flag) return false;
            if (clock64() - t0 > limit) {
                *abort_flag = 1;
                return false;
            }
        }
        return true;
    }
    if (mbar_test(b, parity)) return true;
    const long long t0 = clock64();
    while (!mbar_test_sleep(b, parity)) {
        if (*abort_flag) return false;
        if (clock64() - t0 > limit) {
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

// ---- warp-uniform issue: the whole warp runs the loop, one elected lane
// issues the instruction (operands stay in uniform registers; a loop run
// by a single lane pays a register move per operand and issues tcgen05.mma
// at about half the rate) -----------------------------------------------------
__device__ __forceinline__ void mbar_expect_tx_elect(uint64_t *b, uint32_t bytes) {
    asm volatile(
        "{\n\t.reg .pred e;\n\t"
        "elect.sync _|e, 0xffffffff;\n\t"
        "@e mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\n\t}" ::"r"(saddr(b)), "r"(bytes)
        : "memory");
}
__device__ __forceinline__ void tma_load_3d_elect(void *dst, const CUtensorMap *map, uint64_t *bar, int c0,
                                                  int c1, int c2) {
    asm volatile(
        "{\n\t.reg .pred e;\n\t"
        "elect.sync _|e, 0xffffffff;\n\t"
        "@e cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4, %5}], [%2];\n\t}" ::"r"(saddr(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(saddr(bar)), "r"(c0), "r"(c1), "r"(c2)
        : "memory");
}
__device__ __forceinline__ void tc_commit_elect(uint64_t *bar) {
    asm volatile(
        "{\n\t.reg .pred e;\n\t"
        "elect.sync _|e, 0xffffffff;\n\t"
        "@e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n\t}" ::"r"(
            saddr(bar))
        : "memory");
}
__device__ __forceinline__ void tc_mma_bf16_elect(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                                  uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p, e;\n\t"
        "elect.sync _|e, 0xffffffff;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}
__device__ __forceinline__ void tc_mma_bf16_ts_elect(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc,
                                                     uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p, e;\n\t"
        "elect.sync _|e, 0xffffffff;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}
// A bounded wait whose outcome the whole warp shares.
__device__ __forceinline__ bool mbar_wait_warp(uint64_t *b, uint32_t parity, volatile int *abort_flag) {
    return __all_sync(kFull, mbar_wait(b, parity, abort_flag));
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
// The same MMA with the A operand (M x K, row m in TMEM lane m, K elements
// packed two per 32-bit column) read from tensor memory.
__device__ __forceinline__ void tc_mma_bf16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc,
                                               uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
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

// ---- order-preserving keys of fp32 scores ---------------------------------------
__device__ __forceinline__ uint32_t ord32(float f) {
    const uint32_t u = __float_as_uint(f);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float unord32(uint32_t o) {
    return __uint_as_float((o & 0x80000000u) ? (o & 0x7FFFFFFFu) : ~o);
}

// ---- the CTA machinery ------------------------------------------------------------
// Byte offsets of the regions every score-tile kernel has in shared memory.
struct CtaLayout {
    uint32_t q, k, rows, bars, misc;
    int stages;
};

struct Cta {
    unsigned char *q_s, *k_s;
    int *rows_s;
    uint64_t *full, *empty, *acc_full, *acc_empty, *mma_done, *q_ready;
    uint32_t *tmem_slot;
    volatile int *abort_flag;
    int stages, n_rows, ntiles;
    uint32_t tmem_base;
};

// Rows, barriers, TMEM and the query tile.  Returns false when the CTA has
// no rows (all threads return together).
__device__ __forceinline__ bool cta_setup(Cta &c, unsigned char *smem, const CtaLayout &lay,
                                          const LedgerDev &L, const __nv_bfloat16 *Q,
                                          const int *list, const int *head_count, int use_list,
                                          bool q_to_smem = true) {
    const int tid = threadIdx.x, warp = tid >> 5;
    const int h = blockIdx.y;
    const int nq = L.nq, d = L.d;
    const int count = use_list ? head_count[h] : nq;
    const int row0 = blockIdx.x * kRows;
    if (row0 >= count) return false;
    c.q_s = smem + lay.q;
    c.k_s = smem + lay.k;
    c.rows_s = reinterpret_cast<int *>(smem + lay.rows);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + lay.bars);
    c.stages = lay.stages;
    c.full = bars;
    c.empty = bars + kMaxStages;
    c.acc_full = bars + 2 * kMaxStages;
    c.acc_empty = bars + 2 * kMaxStages + kAcc;
    c.mma_done = bars + 2 * kMaxStages + 2 * kAcc;
    c.q_ready = bars + 2 * kMaxStages + 2 * kAcc + 1;
    c.tmem_slot = reinterpret_cast<uint32_t *>(smem + lay.misc);
    c.abort_flag = reinterpret_cast<volatile int *>(smem + lay.misc + 4);
    c.n_rows = min(kRows, count - row0);

    if (tid < kRows) {
        int row = -1;
        if (tid < c.n_rows) row = use_list ? list[(size_t)h * nq + row0 + tid] : row0 + tid;
        c.rows_s[tid] = row;
    }
    if (tid == 0) {
        for (int s = 0; s < c.stages; ++s) {
            mbar_init(&c.full[s], 1);
            mbar_init(&c.empty[s], 1);
        }
        for (int a = 0; a < kAcc; ++a) {
            mbar_init(&c.acc_full[a], 1);
            mbar_init(&c.acc_empty[a], (blockDim.x >> 5) - 2);
        }
        mbar_init(c.mma_done, 1);
        mbar_init(c.q_ready, (blockDim.x >> 5) - 2);   // kernels that load the query tile into TMEM
        *c.abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         saddr(c.tmem_slot)),
                     "r"(kTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    __syncthreads();

    // query tile: gather rows by index into the 128-byte-swizzled K-major
    // layout (row r, 16-byte chunk c of its 64-element half kb lands at
    // kb*16KB + r*128 + ((c ^ (r & 7)) * 16)).  Kernels that keep the query
    // tile in TMEM load it themselves.
    const int c16 = q_to_smem ? (d >> 3) : 0;
    for (int e = tid; e < kRows * c16; e += blockDim.x) {
        const int r = e / c16, ch = e - r * c16;
        const int row = c.rows_s[r];
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        if (row >= 0) v = *reinterpret_cast<const uint4 *>(Q + ((size_t)h * nq + row) * d + ch * 8);
        const int kb = ch >> 3, cc = ch & 7;
        *reinterpret_cast<uint4 *>(c.q_s + kb * kSubTileBytes + r * 128 + ((cc ^ (r & 7)) << 4)) = v;
    }
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    // the block's last row bounds its key tiles under the causal mask; rows
    // from a list may come in any order
    int max_row = row0 + c.n_rows - 1;
    if (use_list) {
        max_row = -1;
        for (int e = 0; e < c.n_rows; ++e) max_row = max(max_row, c.rows_s[e]);
    }
    const int kend = L.causal ? min(L.nk, max_row + 1) : L.nk;
    c.ntiles = (kend + kKeys - 1) / kKeys;
    __syncthreads();
    tc_fence_after();
    c.tmem_base = *c.tmem_slot;
    return true;
}

// Tile schedule: pass p covers key tiles 0..nt-1, the second pass backwards
// (its first tiles are the ones most recently loaded).
__device__ __forceinline__ int tile_of(int g, int ntiles) { return g < ntiles ? g : 2 * ntiles - 1 - g; }

// TMA producer (the whole warp; one elected lane issues): `passes` sweeps
// over the key tiles into the ring.  Stage s is refilled once the MMAs that
// read it have completed (its empty barrier, committed by the MMA warp).
__device__ __forceinline__ void producer(Cta &c, const CUtensorMap *tmap_k, int d, int h, int passes) {
    if ((threadIdx.x & 31) == 0)
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(tmap_k)) : "memory");
    const int total = passes * c.ntiles;
    const uint32_t stage_bytes = (uint32_t)(kKeys * d * 2);
    int issued = 0;
    for (int g = 0; g < total; ++g) {
        const int s = g % c.stages;
        if (g >= c.stages && !mbar_wait_warp(&c.empty[s], ((g / c.stages) & 1) ^ 1, c.abort_flag)) break;
        mbar_expect_tx_elect(&c.full[s], stage_bytes);
        const int t = tile_of(g, c.ntiles);
        for (int kb = 0; kb < (d >> 6); ++kb)
            tma_load_3d_elect(c.k_s + s * stage_bytes + kb * kSubTileBytes, tmap_k, &c.full[s], kb * 64,
                              t * kKeys, h);
        ++issued;
    }
    // drain: every issued stage must have landed before the CTA exits
    for (int g = max(0, issued - c.stages); g < issued; ++g) {
        const int s = g % c.stages;
        const long long t0 = clock64();
        while (!mbar_test(&c.full[s], (g / c.stages) & 1) && clock64() - t0 < kSpinLimit) {
        }
    }
}

// MMA issuer (one lane): score tile g into accumulator g % kAcc.
// The descriptor of a K-major operand at byte offset `off` from another's
// start is that descriptor plus off / 16 (the start address field, bits
// 0..13, holds address / 16 and shared memory stays below 256 KB).
template <int kSteps>
__device__ __forceinline__ void mma_tile(uint32_t d_tmem, uint64_t qdesc, uint64_t kdesc) {
#pragma unroll
    for (int kk = 0; kk < kSteps; ++kk) {
        const uint64_t off16 = (uint64_t)((kk >> 2) * (kSubTileBytes >> 4) + (kk & 3) * 2);
        tc_mma_bf16_elect(d_tmem, qdesc + off16, kdesc + off16, kIdesc, kk > 0 ? 1u : 0u);
    }
}

// MMA issuer (the whole warp; one elected lane issues).
__device__ __forceinline__ void mma_issuer(Cta &c, int d, int passes) {
    const int total = passes * c.ntiles;
    const uint64_t qdesc = sw128_desc(saddr(c.q_s));
    const uint32_t k_addr = saddr(c.k_s);
    const uint32_t stage_bytes = (uint32_t)(kKeys * d * 2);
    const uint32_t tmem = __shfl_sync(kFull, c.tmem_base, 0);
    for (int g = 0; g < total; ++g) {
        const int s = g % c.stages, a = g % kAcc;
        if (!mbar_wait_warp(&c.full[s], (g / c.stages) & 1, c.abort_flag)) break;
        if (!mbar_wait_warp(&c.acc_empty[a], ((g / kAcc) & 1) ^ 1, c.abort_flag)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem + (uint32_t)(a * kKeys);
        const uint64_t kdesc = sw128_desc(k_addr + (uint32_t)s * stage_bytes);
        if (d == 128) mma_tile<8>(d_tmem, qdesc, kdesc);
        else mma_tile<4>(d_tmem, qdesc, kdesc);
        tc_commit_elect(&c.empty[s]);      // the producer may refill stage s
        tc_commit_elect(&c.acc_full[a]);   // the epilogue may read accumulator a
    }
    tc_commit_elect(c.mma_done);
    const long long t0 = clock64();
    while (!mbar_test(c.mma_done, 0) && clock64() - t0 < kSpinLimit) {
    }
}

__device__ __forceinline__ void cta_teardown(Cta &c, const LedgerDev &L) {
    tc_fence_before();
    __syncthreads();
    if ((threadIdx.x >> 5) == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(c.tmem_base),
                     "r"(kTmemCols)
                     : "memory");
    }
    if (threadIdx.x == 0 && *c.abort_flag) atomicOr(&L.counters[2], 2ULL);
}

// Epilogue helpers: wait for accumulator g (warp-uniform outcome) / hand it
// back.  ACC: accumulators in the ring (tile g uses accumulator g % ACC).
template <int ACC = kAcc>
__device__ __forceinline__ bool acc_wait(Cta &c, int g, long long limit = kSpinLimit) {
    bool ok = mbar_wait(&c.acc_full[g % ACC], (g / ACC) & 1, c.abort_flag, limit);
    ok = __all_sync(kFull, ok);   // the warp leaves together (tcgen05.ld is .sync.aligned)
    if (ok) tc_fence_after();
    return ok;
}
template <int ACC = kAcc>
__device__ __forceinline__ void acc_release(Cta &c, int g) {
    tc_fence_before();
    __syncwarp();
    if ((threadIdx.x & 31) == 0) mbar_arrive(&c.acc_empty[g % ACC]);
}

}  // namespace tc
}  // namespace rr
