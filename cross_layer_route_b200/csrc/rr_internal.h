// rr_internal.h -- internal types shared by the host library and the kernels.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace rr {

// Device-side view of one ledger, passed to kernels by value.
struct LedgerDev {
    // ledger proper (RouteRelay §3.1 Eq. 4, §4.1)
    int32_t *ids;           // [bh*nq, c]  route | near-miss | random
    float *alpha;           // [bh*nq]     weakest selected score at the row's last layer
    int32_t *anchor_layer;  // [bh*nq]     layer the row was last fully routed at
    uint8_t *flags;         // [bh*nq]     1 = fully routed at the last layer
    unsigned long long *counters;  // [16] RR_CNT_* slots (int64 in the C ABI)
    // per-layer scratch
    int32_t *list;          // [bh*nq]     per-head segments of flagged row ids, ascending
    int32_t *head_count;    // [bh]        flagged rows per head
    int32_t *retry_list;    // [bh*nq]     per-head rows whose tensor-core selection is redone
    int32_t *retry_count;   // [bh]        rows listed per head
    // buffers of the tensor-core selection path (null: the allocation-free
    // entry point, whose route kernel finishes its rows itself).  Row slot
    // s = (head * blocks_per_head + block) * 128 + position in the block.
    uint64_t *cand_keys = nullptr;   // [slots, kRowCap] kept (score, chunk) sort keys
    uint32_t *cand_masks = nullptr;  // [blocks, mt, 4, 128] kept columns per (tile, quarter, row),
                                     // only for heads of more than 32 key tiles
    uint2 *cand_meta = nullptr;      // [slots] {kept keys (all ones: redo the row), threshold}
    int32_t *und_list = nullptr;     // [bh*nq] relay rows whose test needs exact rescoring
    int32_t *und_count = nullptr;    // [1]
    // fp32 problems on the tensor cores: Kc split into three bf16 parts per
    // element (hi, mid, lo: x = hi + mid + lo exactly), rows [hi | mid | lo]
    uint16_t *ksplit = nullptr;      // [bh, nk, 3 d] bf16 bits
    int split = 0;                   // 1: the selection kernel takes fp32 Qc/Kc split in three
    int mt = 0;                      // key tiles per head: ceil(nk / 128)
    int bh, nq, nk, d;
    int k, m, r, c, ksel;   // ksel = k + m; c = k + m + r + g_sink + g_recent
    int g_sink = 0, g_recent = 0;   // mandatory global sentinels (sink, recent chunks)
    int causal;
    int bh_offset;
    int max_draws;          // cap on random draws per row (64 * c)
    float gamma;
    // per-row guard margins gamma_i of Eq. 8 ([bh*nq], caller-owned device
    // memory), or null for `gamma` on every row; per-row lifetime bound: a
    // row max_age or more layers past its anchor layer refreshes (0: off)
    const float *gamma_rows = nullptr;
    int max_age = 0;
    // hysteresis: a row built at layer a is reused without the test at
    // layers a+1 .. a+min_reuse (0: off); a row rebuilt at a relay layer is
    // marked (flags bit 1) and tests with max(gamma_i, gamma_h) until it
    // first passes (gamma_h 0: off)
    int min_reuse = 0;
    float gamma_h = 0.0f;
    // flags byte a rebuilt row receives (set by the host per launch): 1 at
    // an anchor layer, 1 | 2 at a relay layer when gamma_h > 0
    uint8_t rebuild_flag = 1;
    // budget, in SM clock cycles, of the selection kernel's accumulator waits
    // in its epilogue (0: the default, about a second); a test shortens it to
    // make a wait run out
    long long wait_budget = 0;
    uint32_t seed_lo, seed_hi;
};

enum Dtype { kF32 = 0, kBF16 = 1 };

// Selection buffer capacity of one row: a power of two >= 2 * ksel, >= 64.
inline int select_capacity(int ksel) {
    int cap = 64;
    while (cap < 2 * ksel) cap <<= 1;
    return cap;
}

// Launchers (return cudaSuccess or the launch error).
// Full routing of a set of rows.  bf16 problems with d in {64, 128}, k + m <=
// 64 and r <= 32 run on the tensor cores (rr_route_tc.cu); the others on the
// CUDA cores (rr_route_simt.cu).  prepare() sets the chosen kernel's shared
// memory attribute on the current device.
cudaError_t route_rows_prepare(const LedgerDev &L, int dtype);
// The same for every kernel at its largest layout (any config), once per device.
cudaError_t route_rows_prepare_all();
bool route_rows_tc_supported(const LedgerDev &L, int dtype);
cudaError_t route_rows_tc_prepare();
cudaError_t launch_route_rows_tc(const LedgerDev &L, const void *q, const void *k, int layer,
                                 bool use_list, cudaStream_t s);

// Tensor-core selection path (rr_select_tc.cu): the selection kernel writes
// every row's kept scores to the candidate buffers, the finishing kernel
// orders them and writes the ledger row.
struct CandSizes { size_t keys, masks, meta, und, ksplit; };
// Bytes of the buffers (all 0 when the problem does not run on the tensor cores).
CandSizes route_select_candidate_sizes(const LedgerDev &L, int dtype);
// fp32 problems the selection kernel takes with three-way bf16 splitting
// (d = 64, the same selection limits as the bf16 path).
bool route_select_split_supported(const LedgerDev &L, int dtype);
// Full routing of fp32 rows on the tensor cores (L.split): split Kc, select,
// finish; rows whose kept scores overflow are rebuilt on the CUDA cores.
cudaError_t launch_route_rows_split(const LedgerDev &L, const void *q, const void *k, int layer,
                                    bool use_list, cudaStream_t s);
// The CUDA-core route kernel alone (rr_route_simt.cu), whatever the problem.
// max_tiles > 0 caps the grid's tiles of 32 rows per head; each CTA then
// strides over the head's remaining tiles (the retry lists, usually empty).
cudaError_t launch_route_rows_simt(const LedgerDev &L, int dtype, const void *q, const void *k,
                                   int layer, bool use_list, cudaStream_t s, int max_tiles = 0);
size_t route_select_smem_bytes(const LedgerDev &L);
cudaError_t route_select_prepare();
// kAnchor: every row (or every listed row) is rebuilt.  kRelay: every row
// is routed and the relay test (Eq. 8) decides, row by row, whether the new
// route or the old one is kept.
enum class SelectMode { kAnchor = 0, kRelay = 1 };
cudaError_t launch_route_select(const LedgerDev &L, const void *q, const CUtensorMap &map, int layer,
                                bool use_list, SelectMode mode, cudaStream_t s);
// Exact routing on the CUDA cores of the rows in the per-head retry lists
// (rows whose kept scores overflowed on the selection path; rr_select_tc.cu).
cudaError_t launch_retry_rows_simt(const LedgerDev &L, const void *q, const void *k, int layer,
                                   cudaStream_t s);
// Exact heap selection of the rows in the per-head retry lists of the fused
// kernel route_rows_tc_kernel (rr_route_tc.cu).
cudaError_t launch_route_retry(const LedgerDev &L, const void *q, const CUtensorMap &map, int layer,
                               cudaStream_t s);
// One relay layer on the tensor-core selection path: route every row, take
// the relay decision from the kept scores, rescore exactly the rows that
// decision leaves open, rebuild the refreshed rows among them, roll up the
// counters.
cudaError_t launch_relay_oneshot(const LedgerDev &L, const void *q, const void *k, int layer,
                                 cudaStream_t s);
namespace tc {
// Tensor map of Kc [bh, nk, d] bf16: boxes of 128 keys x 64 dims, 128-byte swizzle.
cudaError_t key_tensor_map(const LedgerDev &L, const void *k, CUtensorMap *map);
// The same over bf16 key rows of row_elems elements (row_elems a multiple of 64).
cudaError_t key_rows_tensor_map(const void *k, int row_elems, int nk, int bh, CUtensorMap *map);
}
cudaError_t launch_route_rows(const LedgerDev &L, int dtype, const void *q, const void *k,
                              int layer, bool use_list, cudaStream_t s);
cudaError_t launch_relay_rescore(const LedgerDev &L, int dtype, const void *q, const void *k,
                                 int layer, cudaStream_t s);
// Relay rescoring from dense tensor-core score tiles (rr_route_tc.cu); used
// for the problems route_rows_tc_supported accepts.
cudaError_t launch_relay_rescore_tc(const LedgerDev &L, const void *q, const void *k, int layer,
                                    cudaStream_t s);
cudaError_t launch_compact(const LedgerDev &L, cudaStream_t s);
cudaError_t launch_finalize(const LedgerDev &L, int layer, long long add_rows,
                            long long add_pairs, long long add_full_pairs, cudaStream_t s);

}  // namespace rr
