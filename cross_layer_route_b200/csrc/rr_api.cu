// rr_api.cu -- C ABI of the B200 RouteRelay router (declared in include/rr.h).
//
// Method: "RouteRelay: Event-Triggered Cross-Layer Route Reuse for Efficient
// Dynamic Sparse Attention" (arXiv 2609.07306), cited as RouteRelay §x.
//
// Host side only: argument validation, the workspace layout, the per-layer
// schedule (forced anchors every H layers, §3.2; relay = rescore -> compact
// -> refresh, §4.1-4.2) and the launches.  Every step of the routing path runs
// in the kernels; nothing here touches routing data.
#include <math.h>
#include <new>
#include <stdint.h>
#include <string.h>

#include "../../include/rr.h"
#include "rr_internal.h"

struct rr_ledger {
    rr_config cfg;
    rr::LedgerDev dev;
    char *ws;
    size_t ws_bytes;
    int device;         // device current at the first enqueue
    bool prepared;      // kernel attributes set on that device
    bool anchored;      // a full route started the current layer sequence
    int32_t last_layer; // last layer completed
    int stage;          // relay stages done at pending_layer (0 = none, 1 = rescore, 2 = compact)
    int32_t pending_layer;
};

namespace {

constexpr size_t kAlign = 256;

size_t align_up(size_t x) { return (x + kAlign - 1) & ~(kAlign - 1); }

struct Layout {
    size_t ids, alpha, anchor_layer, flags, counters, list, head_count, retry_list, retry_count;
    // tensor-core selection path only (size 0 otherwise)
    size_t cand_keys, cand_masks, cand_meta, und_list, und_count, ksplit;
    bool cand, split;
    size_t total;
};

bool config_ok(const rr_config *c) {
    if (!c) return false;
    if (c->bh < 1 || c->nq < 1 || c->nk < 1) return false;
    if (c->d < 8 || c->d > 256 || (c->d % 8) != 0) return false;
    if (c->dtype != RR_F32 && c->dtype != RR_BF16) return false;
    if (c->k < 1 || c->k > c->nk) return false;
    if (c->m_near < 0 || c->r_rand < 0) return false;
    if (c->k + c->m_near > 128 || c->r_rand > 128) return false;
    if (c->g_sink < 0 || c->g_recent < 0 || c->g_sink + c->g_recent > 32) return false;
    if (c->anchor_interval < 0 || c->bh_offset < 0) return false;
    if (!(c->gamma >= 0.0f) || !isfinite(c->gamma)) return false;
    if ((long long)c->bh * (long long)c->nq > (long long)INT32_MAX) return false;
    return true;
}

Layout layout_of(const rr_config *c) {
    const size_t rows = (size_t)c->bh * (size_t)c->nq;
    const size_t cc = (size_t)(c->k + c->m_near + c->r_rand + c->g_sink + c->g_recent);
    Layout L;
    size_t o = 0;
    L.ids = o;          o = align_up(o + rows * cc * sizeof(int32_t));
    L.alpha = o;        o = align_up(o + rows * sizeof(float));
    L.anchor_layer = o; o = align_up(o + rows * sizeof(int32_t));
    L.flags = o;        o = align_up(o + rows * sizeof(uint8_t));
    L.counters = o;     o = align_up(o + RR_NUM_COUNTERS * sizeof(int64_t));
    L.list = o;         o = align_up(o + rows * sizeof(int32_t));
    L.head_count = o;   o = align_up(o + (size_t)c->bh * sizeof(int32_t));
    L.retry_list = o;   o = align_up(o + rows * sizeof(int32_t));
    L.retry_count = o;  o = align_up(o + (size_t)c->bh * sizeof(int32_t));
    rr::LedgerDev t;
    t.bh = c->bh; t.nq = c->nq; t.nk = c->nk; t.d = c->d;
    t.k = c->k; t.m = c->m_near; t.r = c->r_rand; t.ksel = c->k + c->m_near;
    t.g_sink = c->g_sink; t.g_recent = c->g_recent; t.c = (int)cc;
    t.mt = (c->nk + 127) / 128;
    const rr::CandSizes cs = rr::route_select_candidate_sizes(t, c->dtype);
    L.cand = cs.keys > 0;
    L.cand_keys = o;    o = align_up(o + cs.keys);
    L.cand_masks = o;   o = align_up(o + cs.masks);
    L.cand_meta = o;    o = align_up(o + cs.meta);
    L.und_list = o;     o = align_up(o + cs.und);
    L.und_count = o;    o = align_up(o + (L.cand ? sizeof(int32_t) : 0));
    L.ksplit = o;       o = align_up(o + cs.ksplit);
    L.split = cs.ksplit > 0;
    L.total = o;
    return L;
}

// Score pairs of one full routing of every row (the counting rule of the
// evaluated-pairs metric, RouteRelay §5.2): each row costs its valid keys.
long long full_pairs(const rr_config *c) {
    long long per_head = 0;
    if (!c->causal) {
        per_head = (long long)c->nq * c->nk;
    } else {
        for (int i = 0; i < c->nq; ++i) per_head += (i + 1 < c->nk) ? (i + 1) : c->nk;
    }
    return per_head * c->bh;
}

bool aligned16(const void *p) { return ((uintptr_t)p & 15u) == 0; }

rr_status to_status(cudaError_t e) { return e == cudaSuccess ? RR_OK : RR_ECUDA; }

bool is_forced_anchor(const rr_ledger *L, int32_t layer) {
    const int H = L->cfg.anchor_interval;
    return H > 0 && layer % H == 0;
}

// Per-ledger device set-up, done at the first call that enqueues work: sets
// the kernels' shared-memory attribute on the current device and enqueues
// the zeroing of every counter slot.  Allocates nothing.
rr_status prepare(rr_ledger *L, cudaStream_t s) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return RR_ECUDA;
    if (L->prepared) return dev == L->device ? RR_OK : RR_EINVAL;
    if (rr::route_rows_prepare(L->dev, L->cfg.dtype) != cudaSuccess) return RR_ECUDA;
    if (cudaMemsetAsync(L->dev.counters, 0, RR_NUM_COUNTERS * sizeof(int64_t), s) != cudaSuccess)
        return RR_ECUDA;
    L->device = dev;
    L->prepared = true;
    return RR_OK;
}

// Zeroes the per-layer counter slots (rows, pairs, full pairs).
cudaError_t reset_layer_counters(rr_ledger *L, cudaStream_t s) {
    cudaError_t e = cudaMemsetAsync(L->dev.counters + RR_CNT_ROWS, 0, 2 * sizeof(int64_t), s);
    if (e == cudaSuccess)
        e = cudaMemsetAsync(L->dev.counters + RR_CNT_FULL_PAIRS, 0, sizeof(int64_t), s);
    return e;
}

rr_status check_inputs(const rr_ledger *L, const void *q, const void *k, int32_t layer) {
    if (!L || !q || !k || layer < 0) return RR_EINVAL;
    if (!aligned16(q) || !aligned16(k)) return RR_EINVAL;
    return RR_OK;
}

rr_status stage_rescore(rr_ledger *L, const void *q, const void *k, int32_t layer, cudaStream_t s) {
    if (!L->anchored || layer <= L->last_layer) return RR_ESTATE;
    const rr_status st = prepare(L, s);
    if (st != RR_OK) return st;
    cudaError_t e = reset_layer_counters(L, s);
    if (e == cudaSuccess) e = rr::launch_relay_rescore(L->dev, L->cfg.dtype, q, k, layer, s);
    if (e != cudaSuccess) return RR_ECUDA;
    L->stage = 1;
    L->pending_layer = layer;
    return RR_OK;
}

rr_status stage_compact(rr_ledger *L, int32_t layer, cudaStream_t s) {
    if (L->stage != 1 || layer != L->pending_layer) return RR_ESTATE;
    if (rr::launch_compact(L->dev, s) != cudaSuccess) return RR_ECUDA;
    L->stage = 2;
    return RR_OK;
}

// Flags byte of a row rebuilt at a relay layer: refreshed, and marked for
// the hysteresis margin when one is set.
uint8_t relay_rebuild_flag(const rr_ledger *L) { return (uint8_t)(1u | (L->dev.gamma_h > 0.0f ? 2u : 0u)); }

rr_status stage_refresh(rr_ledger *L, const void *q, const void *k, int32_t layer, cudaStream_t s) {
    if (L->stage != 2 || layer != L->pending_layer) return RR_ESTATE;
    L->dev.rebuild_flag = relay_rebuild_flag(L);
    cudaError_t e = rr::launch_route_rows(L->dev, L->cfg.dtype, q, k, layer, /*use_list=*/true, s);
    if (e == cudaSuccess) e = rr::launch_finalize(L->dev, layer, 0, 0, 0, s);
    if (e != cudaSuccess) return RR_ECUDA;
    L->stage = 0;
    L->last_layer = layer;
    return RR_OK;
}

rr_status do_full_route(rr_ledger *L, const void *q, const void *k, int32_t layer,
                        cudaStream_t s) {
    const rr_status st = prepare(L, s);
    if (st != RR_OK) return st;
    cudaError_t e = reset_layer_counters(L, s);
    if (e != cudaSuccess) return RR_ECUDA;
    L->dev.rebuild_flag = 1;
    e = rr::launch_route_rows(L->dev, L->cfg.dtype, q, k, layer, /*use_list=*/false, s);
    if (e != cudaSuccess) return RR_ECUDA;
    const long long fp = full_pairs(&L->cfg);
    e = rr::launch_finalize(L->dev, layer, (long long)L->cfg.bh * L->cfg.nq, fp, fp, s);
    if (e != cudaSuccess) return RR_ECUDA;
    L->anchored = true;
    L->last_layer = layer;
    L->stage = 0;
    return RR_OK;
}

// A relay layer on the tensor-core selection path (rr_select_tc.cu): every
// row is routed, the relay test is taken from the kept scores, and the
// ledger, flags and counters come out as the three stages would leave them.
rr_status do_relay_oneshot(rr_ledger *L, const void *q, const void *k, int32_t layer, cudaStream_t s) {
    const rr_status st = prepare(L, s);
    if (st != RR_OK) return st;
    cudaError_t e = reset_layer_counters(L, s);
    L->dev.rebuild_flag = relay_rebuild_flag(L);
    if (e == cudaSuccess) e = rr::launch_relay_oneshot(L->dev, q, k, layer, s);
    if (e == cudaSuccess) e = rr::launch_finalize(L->dev, layer, 0, 0, 0, s);
    if (e != cudaSuccess) return RR_ECUDA;
    L->stage = 0;
    L->last_layer = layer;
    return RR_OK;
}

}  // namespace

extern "C" {

size_t rr_ledger_workspace_bytes(const rr_config *cfg) {
    if (!config_ok(cfg)) return 0;
    return layout_of(cfg).total;
}

rr_status rr_ledger_create(const rr_config *cfg, void *d_workspace, size_t bytes,
                           rr_ledger **out) {
    if (!out) return RR_EINVAL;
    *out = nullptr;
    if (!config_ok(cfg) || !d_workspace) return RR_EINVAL;
    if (((uintptr_t)d_workspace & (kAlign - 1)) != 0) return RR_EINVAL;
    const Layout lay = layout_of(cfg);
    if (bytes < lay.total) return RR_ENOMEM;
    rr_ledger *L = new (std::nothrow) rr_ledger();
    if (!L) return RR_ENOMEM;
    L->cfg = *cfg;
    L->ws = static_cast<char *>(d_workspace);
    L->ws_bytes = bytes;
    L->device = -1;
    L->prepared = false;
    L->anchored = false;
    L->last_layer = -1;
    L->stage = 0;
    L->pending_layer = -1;
    rr::LedgerDev &D = L->dev;
    D.ids = reinterpret_cast<int32_t *>(L->ws + lay.ids);
    D.alpha = reinterpret_cast<float *>(L->ws + lay.alpha);
    D.anchor_layer = reinterpret_cast<int32_t *>(L->ws + lay.anchor_layer);
    D.flags = reinterpret_cast<uint8_t *>(L->ws + lay.flags);
    D.counters = reinterpret_cast<unsigned long long *>(L->ws + lay.counters);
    D.list = reinterpret_cast<int32_t *>(L->ws + lay.list);
    D.head_count = reinterpret_cast<int32_t *>(L->ws + lay.head_count);
    D.retry_list = reinterpret_cast<int32_t *>(L->ws + lay.retry_list);
    D.retry_count = reinterpret_cast<int32_t *>(L->ws + lay.retry_count);
    if (lay.cand) {
        D.cand_keys = reinterpret_cast<uint64_t *>(L->ws + lay.cand_keys);
        D.cand_masks = reinterpret_cast<uint32_t *>(L->ws + lay.cand_masks);
        D.cand_meta = reinterpret_cast<uint2 *>(L->ws + lay.cand_meta);
        D.und_list = reinterpret_cast<int32_t *>(L->ws + lay.und_list);
        D.und_count = reinterpret_cast<int32_t *>(L->ws + lay.und_count);
    }
    if (lay.split) {
        D.ksplit = reinterpret_cast<uint16_t *>(L->ws + lay.ksplit);
        D.split = 1;
    }
    D.mt = (cfg->nk + 127) / 128;
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
    *out = L;
    return RR_OK;
}

rr_status rr_ledger_destroy(rr_ledger *ledger) {
    delete ledger;
    return RR_OK;
}

rr_status rr_full_route(rr_ledger *ledger, const void *d_qc, const void *d_kc, int32_t layer,
                        void *stream) {
    const rr_status st = check_inputs(ledger, d_qc, d_kc, layer);
    if (st != RR_OK) return st;
    return do_full_route(ledger, d_qc, d_kc, layer, static_cast<cudaStream_t>(stream));
}

rr_status rr_relay_layer(rr_ledger *ledger, const void *d_qc, const void *d_kc, int32_t layer,
                         void *stream) {
    rr_status st = check_inputs(ledger, d_qc, d_kc, layer);
    if (st != RR_OK) return st;
    if (!ledger->anchored || layer <= ledger->last_layer) return RR_ESTATE;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (is_forced_anchor(ledger, layer)) return do_full_route(ledger, d_qc, d_kc, layer, s);
    if (ledger->dev.cand_keys) return do_relay_oneshot(ledger, d_qc, d_kc, layer, s);
    st = stage_rescore(ledger, d_qc, d_kc, layer, s);
    if (st == RR_OK) st = stage_compact(ledger, layer, s);
    if (st == RR_OK) st = stage_refresh(ledger, d_qc, d_kc, layer, s);
    return st;
}

rr_status rr_relay_rescore(rr_ledger *ledger, const void *d_qc, const void *d_kc, int32_t layer,
                           void *stream) {
    const rr_status st = check_inputs(ledger, d_qc, d_kc, layer);
    if (st != RR_OK) return st;
    return stage_rescore(ledger, d_qc, d_kc, layer, static_cast<cudaStream_t>(stream));
}

rr_status rr_relay_compact(rr_ledger *ledger, int32_t layer, void *stream) {
    if (!ledger || layer < 0) return RR_EINVAL;
    return stage_compact(ledger, layer, static_cast<cudaStream_t>(stream));
}

rr_status rr_relay_refresh(rr_ledger *ledger, const void *d_qc, const void *d_kc, int32_t layer,
                           void *stream) {
    const rr_status st = check_inputs(ledger, d_qc, d_kc, layer);
    if (st != RR_OK) return st;
    return stage_refresh(ledger, d_qc, d_kc, layer, static_cast<cudaStream_t>(stream));
}

rr_status rr_ledger_read(const rr_ledger *ledger, const rr_ledger_view *dst, void *stream) {
    if (!ledger || !dst) return RR_EINVAL;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const rr::LedgerDev &D = ledger->dev;
    const size_t rows = (size_t)D.bh * D.nq;
    cudaError_t e = cudaSuccess;
    if (dst->ids && e == cudaSuccess)
        e = cudaMemcpyAsync(dst->ids, D.ids, rows * D.c * sizeof(int32_t), cudaMemcpyDefault, s);
    if (dst->alpha && e == cudaSuccess)
        e = cudaMemcpyAsync(dst->alpha, D.alpha, rows * sizeof(float), cudaMemcpyDefault, s);
    if (dst->anchor_layer && e == cudaSuccess)
        e = cudaMemcpyAsync(dst->anchor_layer, D.anchor_layer, rows * sizeof(int32_t),
                            cudaMemcpyDefault, s);
    if (dst->flags && e == cudaSuccess)
        e = cudaMemcpyAsync(dst->flags, D.flags, rows * sizeof(uint8_t), cudaMemcpyDefault, s);
    if (dst->counters && e == cudaSuccess)
        e = cudaMemcpyAsync(dst->counters, D.counters, RR_NUM_COUNTERS * sizeof(int64_t),
                            cudaMemcpyDefault, s);
    return to_status(e);
}

rr_status rr_ledger_device_view(const rr_ledger *ledger, rr_ledger_view *view) {
    if (!ledger || !view) return RR_EINVAL;
    view->ids = ledger->dev.ids;
    view->alpha = ledger->dev.alpha;
    view->anchor_layer = ledger->dev.anchor_layer;
    view->flags = ledger->dev.flags;
    view->counters = reinterpret_cast<int64_t *>(ledger->dev.counters);
    return RR_OK;
}

rr_status rr_ledger_set_guard(rr_ledger *ledger, const float *d_gamma_rows, int32_t max_age) {
    if (!ledger || max_age < 0) return RR_EINVAL;
    ledger->dev.gamma_rows = d_gamma_rows;
    ledger->dev.max_age = max_age;
    return RR_OK;
}

rr_status rr_ledger_set_hysteresis(rr_ledger *ledger, int32_t min_reuse) {
    if (!ledger || min_reuse < 0) return RR_EINVAL;
    ledger->dev.min_reuse = min_reuse;
    return RR_OK;
}

rr_status rr_ledger_set_wait_budget(rr_ledger *ledger, int64_t cycles) {
    if (!ledger || cycles < 0) return RR_EINVAL;
    ledger->dev.wait_budget = (long long)cycles;
    return RR_OK;
}

rr_status rr_ledger_set_hysteresis_margin(rr_ledger *ledger, float gamma_h) {
    if (!ledger || !(gamma_h >= 0.0f) || !isfinite(gamma_h)) return RR_EINVAL;
    ledger->dev.gamma_h = gamma_h;
    return RR_OK;
}

const char *rr_status_string(rr_status status) {
    switch (status) {
        case RR_OK: return "RR_OK";
        case RR_EINVAL: return "RR_EINVAL: invalid argument";
        case RR_ESTATE: return "RR_ESTATE: call out of order";
        case RR_ENOMEM: return "RR_ENOMEM: workspace too small or out of host memory";
        case RR_ECUDA: return "RR_ECUDA: CUDA runtime error";
        case RR_EDEVICE: return "RR_EDEVICE: error recorded on the device";
        case RR_ECAPACITY: return "RR_ECAPACITY: problem exceeds the fixed capacity of the call";
    }
    return "RR_UNKNOWN";
}

}  // extern "C"
