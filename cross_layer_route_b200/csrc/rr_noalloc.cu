// rr_noalloc.cu -- a routing-layer entry point that allocates nothing.
//
// Some callers cannot call cudaMalloc at all: code that runs inside a host
// framework which owns every device allocation (a fixed memory pool handed
// out once at start-up), or code that must not reach the allocator on its
// latency path.  Such a caller can still hand over the inputs (Qc, Kc) and
// the outputs (the ledger arrays), but not a scratch workspace.  This file
// gives it one entry point, rr_route_layer_static, whose only scratch -- the
// per-head lists of refreshed rows and their lengths, written by the
// compaction kernel and read by the refresh kernel, and the per-head lists
// of rows whose tensor-core selection is redone -- lives in a fixed-size
// array in the library's own device memory.
//
// The array below is a file-scope __device__ variable: every GPU that loads
// this library holds it (about 8 MiB) until the process exits.  In host code
// its name is only a host-side stand-in, not a device address, so the host
// looks its address up once per device with cudaGetSymbolAddress and passes
// that address to the kernels.
#include <mutex>
#include <stdint.h>

#include "../../include/rr.h"
#include "rr_internal.h"

namespace {

constexpr int kStaticMaxRows = 1 << 20;   // bh * nq of one call, at most
constexpr int kStaticMaxHeads = 4096;     // bh of one call, at most
constexpr int kMaxDevices = 64;

// [0, R): refresh lists (per-head segments of nq entries); [R, R + H): rows
// listed per head; [R + H, 2R + H): lists of rows whose tensor-core
// selection is redone; [2R + H, 2R + 2H): their counts per head
// (R = kStaticMaxRows, H = kStaticMaxHeads).
static __device__ __align__(256) int32_t g_rr_static_scratch[2 * (kStaticMaxRows + kStaticMaxHeads)];

std::mutex g_setup_mutex;
int32_t *g_scratch_addr[kMaxDevices] = {nullptr};

// Per-device set-up, done once per device with that device current: the
// device address of the static scratch, and the kernels' shared-memory
// attributes at their largest layouts (so later calls make no host API call
// for them).  Returns nullptr on failure.
int32_t *static_scratch_on_current_device() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    if (!g_scratch_addr[dev]) {
        void *ptr = nullptr;
        if (cudaGetSymbolAddress(&ptr, g_rr_static_scratch) != cudaSuccess || !ptr) return nullptr;
        if (rr::route_rows_prepare_all() != cudaSuccess) return nullptr;
        g_scratch_addr[dev] = static_cast<int32_t *>(ptr);
    }
    return g_scratch_addr[dev];
}

long long full_pairs_of(const rr_config *c) {
    long long per_head = 0;
    if (!c->causal) {
        per_head = (long long)c->nq * c->nk;
    } else {
        for (int i = 0; i < c->nq; ++i) per_head += (i + 1 < c->nk) ? (i + 1) : c->nk;
    }
    return per_head * c->bh;
}

bool aligned(const void *p, uintptr_t a) { return ((uintptr_t)p & (a - 1)) == 0; }

}  // namespace

extern "C" rr_status rr_route_layer_static(const rr_config *cfg, const void *d_qc,
                                           const void *d_kc, int32_t layer, int32_t *d_ids,
                                           float *d_alpha, int32_t *d_anchor_layer,
                                           uint8_t *d_flags, int64_t *d_counters, void *stream) {
    if (!cfg || rr_ledger_workspace_bytes(cfg) == 0) return RR_EINVAL;
    if (!d_qc || !d_kc || !d_ids || !d_alpha || !d_anchor_layer || !d_flags || !d_counters)
        return RR_EINVAL;
    if (layer < 0 || !aligned(d_qc, 16) || !aligned(d_kc, 16) || !aligned(d_ids, 4) ||
        !aligned(d_alpha, 4) || !aligned(d_anchor_layer, 4) || !aligned(d_counters, 8))
        return RR_EINVAL;
    if ((long long)cfg->bh * cfg->nq > kStaticMaxRows || cfg->bh > kStaticMaxHeads)
        return RR_ECAPACITY;
    int32_t *scratch = static_scratch_on_current_device();
    if (!scratch) return RR_ECUDA;

    rr::LedgerDev D;
    D.ids = d_ids;
    D.alpha = d_alpha;
    D.anchor_layer = d_anchor_layer;
    D.flags = d_flags;
    D.counters = reinterpret_cast<unsigned long long *>(d_counters);
    D.list = scratch;
    D.head_count = scratch + kStaticMaxRows;
    D.retry_list = scratch + kStaticMaxRows + kStaticMaxHeads;
    D.retry_count = scratch + 2 * kStaticMaxRows + kStaticMaxHeads;
    D.bh = cfg->bh; D.nq = cfg->nq; D.nk = cfg->nk; D.d = cfg->d;
    D.k = cfg->k; D.m = cfg->m_near; D.r = cfg->r_rand;
    D.g_sink = cfg->g_sink; D.g_recent = cfg->g_recent;
    D.c = cfg->k + cfg->m_near + cfg->r_rand + cfg->g_sink + cfg->g_recent;
    D.ksel = cfg->k + cfg->m_near;
    D.causal = cfg->causal ? 1 : 0;
    D.bh_offset = cfg->bh_offset;
    D.max_draws = 64 * D.c;
    D.gamma = cfg->gamma;
    D.seed_lo = (uint32_t)(cfg->seed & 0xffffffffu);
    D.seed_hi = (uint32_t)(cfg->seed >> 32);

    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int H = cfg->anchor_interval;
    const bool anchor = layer == 0 || (H > 0 && layer % H == 0);
    cudaError_t e = cudaMemsetAsync(d_counters + RR_CNT_ROWS, 0, 2 * sizeof(int64_t), s);
    if (e == cudaSuccess) e = cudaMemsetAsync(d_counters + RR_CNT_FULL_PAIRS, 0, sizeof(int64_t), s);
    if (anchor) {
        const long long fp = full_pairs_of(cfg);
        if (e == cudaSuccess) e = rr::launch_route_rows(D, cfg->dtype, d_qc, d_kc, layer, false, s);
        if (e == cudaSuccess)
            e = rr::launch_finalize(D, layer, (long long)cfg->bh * cfg->nq, fp, fp, s);
    } else {
        if (e == cudaSuccess) e = rr::launch_relay_rescore(D, cfg->dtype, d_qc, d_kc, layer, s);
        if (e == cudaSuccess) e = rr::launch_compact(D, s);
        if (e == cudaSuccess) e = rr::launch_route_rows(D, cfg->dtype, d_qc, d_kc, layer, true, s);
        if (e == cudaSuccess) e = rr::launch_finalize(D, layer, 0, 0, 0, s);
    }
    return e == cudaSuccess ? RR_OK : RR_ECUDA;
}
