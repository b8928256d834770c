/*
 * rr.h -- C ABI of the B200 RouteRelay router (librr.so).
 *
 * Method: "RouteRelay: Event-Triggered Cross-Layer Route Reuse for Efficient
 * Dynamic Sparse Attention" (arXiv 2609.07306), cited as RouteRelay §x.
 *
 * Per layer l and per head, a chunk-based dynamic sparse router scores
 * query-chunk representations Qc [nq, d] against key-chunk representations
 * Kc [nk, d] (S = Qc Kc^T, §2.1 Eq. 1) and routes every query row to its
 * top-k key chunks (§2.1 Eq. 2).  RouteRelay keeps, per query row, a ledger
 * (§3.1 Eq. 4, §4.1): the route (k ids), the sentinels (m near-miss ids =
 * the chunks ranked k+1..k+m, and r random ids drawn from the rest), and the
 * layer the row was last fully routed at.  Anchor layers fully route every
 * row.  Intermediate ("relay") layers rescore only the ledger's candidates
 * (§3.2 Eq. 5), compute alpha = min score over the route (Eq. 6) and
 * beta = max score over the sentinels (Eq. 7), keep the route when
 * alpha > beta + gamma (Eq. 8), and fully re-route only the rows that fail
 * (§4.1-4.2: compaction of the failing rows, then a refresh of only those).
 *
 * Conventions shared by every entry point:
 *  - Device memory is owned by the caller.  The library never allocates or
 *    frees device memory: the ledger lives in a caller-allocated workspace.
 *  - Qc and Kc are device pointers to contiguous row-major [bh, nq, d] and
 *    [bh, nk, d] arrays of the ledger's dtype (fp32 or bf16), 16-byte
 *    aligned, valid until the stream reaches the call.
 *  - Every call enqueues work on `stream` (a cudaStream_t; NULL is the
 *    legacy default stream) and returns without synchronising.  Argument
 *    and state errors are returned synchronously and enqueue nothing.
 *    Errors found on the device (an out-of-range ledger id, a bounded wait
 *    that timed out) are recorded in the ledger's error word (counters[2],
 *    see RR_CNT_ERROR), read back by rr_ledger_read.
 *  - The device that was current at rr_ledger_create must be current at
 *    every later call on that ledger.
 *  - Inputs must be finite.  Ties between equal scores are broken by the
 *    smaller chunk index; ids are stored best first.
 *  - Missing ids (a causal row with fewer valid chunks than slots) are -1.
 *  - No entry point throws; none keeps global state besides the ledger.
 */
#ifndef RR_H
#define RR_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    RR_OK = 0,
    RR_EINVAL = 1,   /* bad argument (null pointer, bad shape or size, misalignment) */
    RR_ESTATE = 2,   /* call out of order (relay before an anchor, layer not increasing) */
    RR_ENOMEM = 3,   /* workspace too small, or host memory for the handle */
    RR_ECUDA = 4,    /* a CUDA runtime call failed (launch, copy, attribute) */
    RR_EDEVICE = 5,  /* the device recorded an error (see the error word) */
    RR_ECAPACITY = 6 /* the problem exceeds a fixed capacity (rr_route_layer_static) */
} rr_status;

typedef enum { RR_F32 = 0, RR_BF16 = 1 } rr_dtype;

/* Problem statement of one ledger (RouteRelay §2.1, §3.1, §3.2, Table 1).
 * Limits: 1 <= k <= nk; k + m_near <= 128; r_rand <= 128; d a multiple of 8
 * with 8 <= d <= 256; gamma >= 0 and finite; anchor_interval >= 0;
 * g_sink, g_recent >= 0 with g_sink + g_recent <= 32. */
typedef struct {
    int32_t bh;              /* batch x heads held by this ledger */
    int32_t nq;              /* query chunks per head */
    int32_t nk;              /* key chunks per head */
    int32_t d;               /* chunk representation dim */
    int32_t dtype;           /* rr_dtype of Qc and Kc */
    int32_t k;               /* route width (top-k, Eq. 2) */
    int32_t m_near;          /* near-miss sentinels (§3.1 item 1) */
    int32_t r_rand;          /* random sentinels (§3.1 item 2) */
    int32_t anchor_interval; /* H: layers with layer % H == 0 are forced anchors (§3.2); 0 = none */
    int32_t causal;          /* nonzero: query chunk i routes only to key chunks j <= i */
    float gamma;             /* guard margin of Eq. 8 */
    int32_t bh_offset;       /* global index of this ledger's head 0 (keys the random draws) */
    uint64_t seed;           /* seed of the random sentinels */
    int32_t g_sink;          /* mandatory global sentinels (§3.1 item 3): sink chunks 0..g_sink-1 */
    int32_t g_recent;        /* ... and the row's recent chunks i-g_recent+1..i (0: none) */
} rr_config;

/* Opaque host-side handle.  It holds pointers into the caller's workspace
 * and the host-side layer state; it owns no device memory. */
typedef struct rr_ledger rr_ledger;

/* Counter slots of the ledger (int64 each). */
enum {
    RR_CNT_ROWS = 0,          /* rows fully routed at the last layer */
    RR_CNT_PAIRS = 1,         /* score pairs evaluated at the last layer */
    RR_CNT_ERROR = 2,         /* error word: bit 0 = a ledger id was out of range at relay;
                                 bit 1 = a bounded wait inside a tensor-core kernel timed out
                                 (that launch's rows were not scored: the layer's results are
                                 not valid, rerun it) */
    RR_CNT_ROWS_TOTAL = 3,    /* rows fully routed since rr_ledger_create */
    RR_CNT_PAIRS_TOTAL = 4,   /* score pairs since rr_ledger_create */
    RR_CNT_LAYERS = 5,        /* layers processed since rr_ledger_create */
    RR_CNT_LAST_LAYER = 6,    /* index of the last layer processed */
    RR_CNT_DRAW_CAP = 7,      /* rows whose random draws hit the draw cap and were filled in order */
    RR_CNT_FULL_PAIRS = 8,    /* score pairs of the rows fully routed at the last layer */
    RR_CNT_FULL_PAIRS_TOTAL = 9, /* the same, since rr_ledger_create */
    RR_CNT_RETRY_TOTAL = 10,  /* rows whose tensor-core selection was redone exactly (kept
                                 scores overflowed the record, or a wait ran out), since create */
    RR_NUM_COUNTERS = 16      /* slots 11..15 are reserved (0) */
};

/* Bytes of device workspace a ledger with this config needs (0 if the
 * config is invalid).  The workspace holds the ledger proper -- ids
 * [bh*nq, c] int32 with c = k + m_near + r_rand + g_sink + g_recent
 * (route | near-miss | random | global), alpha [bh*nq] f32, anchor layer [bh*nq] int32, refresh flags
 * [bh*nq] u8, counters [16] int64 -- plus the library's per-layer scratch
 * (refresh lists and counts; for problems routed on the tensor cores also
 * the kept scores each row hands from the selection kernel to the kernel
 * that orders them: 128 sort keys of 8 bytes and an 8-byte count and
 * threshold per row, rows rounded up to 128 per head, the list of relay rows
 * left for exact rescoring, and for fp32 problems the keys split into three
 * bf16 parts, 3 d bf16 per key row).  Pure host arithmetic. */
size_t rr_ledger_workspace_bytes(const rr_config *cfg);

/* Validates cfg, carves the ledger out of d_workspace (device memory of at
 * least rr_ledger_workspace_bytes(cfg) bytes, 256-byte aligned, owned by
 * the caller and kept alive until rr_ledger_destroy) and returns a handle
 * in *out.  Makes no CUDA call and does not touch device memory; the first
 * call that enqueues work records the current device, sets the kernels'
 * shared-memory attributes on it and zeroes the counters (on its stream).  The first layer of a sequence must be
 * an anchor (rr_full_route).  Errors: RR_EINVAL (bad config or pointer),
 * RR_ENOMEM (workspace too small / no host memory). */
rr_status rr_ledger_create(const rr_config *cfg, void *d_workspace, size_t bytes,
                           rr_ledger **out);

/* Frees the host handle (not the workspace).  NULL is allowed. */
rr_status rr_ledger_destroy(rr_ledger *ledger);

/* Anchor layer: full routing of every row (RouteRelay §2.1 Eq. 1-2; §4.1 "an
 * anchor layer constructs this state from a complete chunk-score matrix").
 * For every query row the library scores all valid key chunks, takes the
 * k + m_near best (score descending, index ascending): the first k become
 * the route, the next m_near the near-miss sentinels.  The mandatory
 * global sentinels (§3.1 item 3) are the sink chunks 0..g_sink-1 and then
 * the row's recent chunks i-g_recent+1..i, each kept if valid, outside the
 * route and near-miss and not already listed, in that order, -1 padded to
 * g_sink + g_recent slots at the end of the row.  r_rand random sentinels
 * are drawn without replacement from the remaining valid chunks (§3.1 item
 * 2, §3.4) with Philox4x32-10 (Salmon et al., SC'11), key (seed lo, seed
 * hi), counter (bh_offset + head, row, layer, t/4), word t%4, chunk = (word
 * * n_valid) >> 32, rejecting repeats; if the pool holds no more than
 * r_rand chunks it is taken whole in ascending order.  alpha
 * becomes the route's weakest score, the anchor layer becomes `layer`, every
 * refresh flag becomes 1.  Starts a new layer sequence at any `layer` >= 0.
 * The score matrix never reaches device memory.  Errors: RR_EINVAL,
 * RR_ECUDA. */
rr_status rr_full_route(rr_ledger *ledger, const void *d_qc, const void *d_kc, int32_t layer,
                        void *stream);

/* Intermediate layer (RouteRelay §3.2 Eq. 5-8, §4.1-4.2).  When
 * anchor_interval > 0 and layer % anchor_interval == 0 this is a forced
 * anchor and behaves as rr_full_route.  Otherwise, for every row: rescore
 * the ledger's candidates against this layer's Kc, alpha = min over the
 * route, beta = max over the sentinels (-inf if none), refresh flag =
 * !(alpha > beta + gamma).  Stable rows keep their ids and store this
 * layer's alpha.  Flagged rows are compacted into a per-head list and only
 * they are fully re-routed at this layer (route, near-miss and random
 * sentinels rebuilt as in rr_full_route; anchor layer <- layer).  No host
 * synchronisation: the refresh launch reads the device-side list.
 * Errors: RR_ESTATE if no anchor started the sequence or `layer` is not
 * greater than the previous layer; RR_EINVAL, RR_ECUDA. */
rr_status rr_relay_layer(rr_ledger *ledger, const void *d_qc, const void *d_kc, int32_t layer,
                         void *stream);

/* The three stages of rr_relay_layer, for callers that schedule or time
 * them one by one (RouteRelay §4.2).  They must be called in this order for
 * one layer; each does exactly its stage and none applies the forced-anchor
 * schedule (rr_relay_layer does).
 *  rr_relay_rescore: candidate rescoring and the challenge test of every row
 *    (Eq. 5-8): writes the refresh flags and, for stable rows, alpha.  Same
 *    preconditions as rr_relay_layer (RR_ESTATE otherwise).
 *  rr_relay_compact: the prefix sum over the flags that writes, per head,
 *    the ascending list of flagged rows and its length.  RR_ESTATE unless
 *    rr_relay_rescore of this `layer` came just before.
 *  rr_relay_refresh: full routing of the listed rows only (their route,
 *    near-miss and random sentinels rebuilt at `layer`, anchor layer <-
 *    `layer`) and the layer's counters.  The launch covers every possible
 *    row tile and tiles past a head's list length exit at once, so nothing
 *    waits on the host.  RR_ESTATE unless rr_relay_compact of this `layer`
 *    came just before. */
rr_status rr_relay_rescore(rr_ledger *ledger, const void *d_qc, const void *d_kc, int32_t layer,
                           void *stream);
rr_status rr_relay_compact(rr_ledger *ledger, int32_t layer, void *stream);
rr_status rr_relay_refresh(rr_ledger *ledger, const void *d_qc, const void *d_kc, int32_t layer,
                           void *stream);

/* Destination of rr_ledger_read.  Any pointer may be NULL (that part is not
 * copied).  Sizes: ids bh*nq*c int32 laid out [bh, nq, c] (route, then
 * near-miss, then random), alpha bh*nq f32, anchor_layer bh*nq int32, flags
 * bh*nq u8 (bit 0: the row was fully routed at the last layer; bit 1: the
 * row carries the hysteresis mark of rr_ledger_set_hysteresis_margin, never
 * set while that margin is 0), counters 16 int64 (the RR_CNT_* slots).  Host
 * (pinned or pageable) or device memory. */
typedef struct {
    int32_t *ids;
    float *alpha;
    int32_t *anchor_layer;
    uint8_t *flags;
    int64_t *counters;
} rr_ledger_view;

/* Enqueues copies of the ledger into dst (cudaMemcpyDefault, on `stream`).
 * The caller synchronises the stream before reading dst.  Errors: RR_EINVAL,
 * RR_ECUDA. */
rr_status rr_ledger_read(const rr_ledger *ledger, const rr_ledger_view *dst, void *stream);

/* Fills *view with the device addresses of the ledger's arrays inside the
 * workspace (no copy), for consumers on the same device. */
rr_status rr_ledger_device_view(const rr_ledger *ledger, rr_ledger_view *view);

/* Per-row relay trigger (RouteRelay §3.2).  d_gamma_rows: NULL (every row
 * uses cfg->gamma) or device memory of bh*nq floats holding each row's guard
 * margin gamma_i of Eq. 8 (row-major [bh, nq], values >= 0; a NaN margin
 * makes its row refresh); the caller owns it and keeps it valid and
 * unchanged until the relay calls that use it have run on the stream.
 * max_age: 0 (off) or the per-row lifetime bound -- the reading of the
 * page's forced anchors, which "bound the lifetime of stale random
 * sentinels", applied row by row: at a relay layer, a row whose ledger was
 * built max_age or more layers earlier (layer - anchor_layer >= max_age)
 * refreshes whatever Eq. 8 says; it is rescored first and counted like a
 * challenged row.  Takes effect from the next rr_relay_layer /
 * rr_relay_rescore call; no CUDA call.  Returns RR_EINVAL for a NULL ledger
 * or max_age < 0. */
rr_status rr_ledger_set_guard(rr_ledger *ledger, const float *d_gamma_rows, int32_t max_age);

/* Hysteresis (RouteRelay §3.2: "a refreshed row receives a minimum reuse
 * horizon of one layer"), the horizon made configurable.  min_reuse: 0 (off)
 * or h > 0 -- a row built at layer a (anchor or refresh) is reused without
 * the challenge test at layers a+1 .. a+h: its ids stay, its alpha is
 * stored, it counts as a stable row.  The lifetime bound of
 * rr_ledger_set_guard takes precedence where the two meet; a row kept inside
 * the horizon keeps its hysteresis mark (below).  Takes effect from the next
 * relay call; no CUDA call.  Returns RR_EINVAL for a NULL ledger or
 * min_reuse < 0. */
rr_status rr_ledger_set_hysteresis(rr_ledger *ledger, int32_t min_reuse);

/* Hysteresis, its second part (RouteRelay §3.2: a refreshed row "may use a
 * larger guard margin until its anchor margin recovers").  gamma_h: 0 (off)
 * or the larger margin, finite and >= 0.  Reading: a row rebuilt at a relay
 * layer is marked (flags bit 1; a row built at an anchor layer is not); a
 * marked row's test of Eq. 8 uses max(gamma_i, gamma_h), and the first time
 * it passes (alpha - beta above that margin: its margin has recovered) the
 * mark is cleared and later tests use gamma_i again.  The lifetime bound and
 * the reuse horizon of rr_ledger_set_guard / rr_ledger_set_hysteresis come
 * first, as in the test without the mark.  Takes effect from the next relay
 * call; no CUDA call.  Returns RR_EINVAL for a NULL ledger or a negative or
 * non-finite gamma_h. */
rr_status rr_ledger_set_hysteresis_margin(rr_ledger *ledger, float gamma_h);

/* One layer on caller-held ledger arrays, allocating nothing.  The paper
 * has no counterpart: this is a deployment variant for callers that cannot
 * call cudaMalloc -- code inside a host framework that owns every device
 * allocation, or code that must not reach an allocator while it runs.  They
 * pass the inputs (d_qc, d_kc as for rr_full_route) and the ledger arrays
 * (in/out, laid out as rr_ledger_read documents: ids [bh, nq, c] int32,
 * alpha [bh*nq] f32, anchor_layer [bh*nq] int32, flags [bh*nq] u8,
 * counters [16] int64, zeroed by the caller before the first layer); no
 * workspace.  Layer 0 and forced-anchor layers (layer % anchor_interval ==
 * 0) are full routing as in rr_full_route; other layers are one relay layer
 * as in rr_relay_layer (rescore, compact, refresh).  The only scratch, the
 * per-head refresh lists and their lengths (and the per-head lists of rows
 * whose tensor-core selection is redone), lives in a fixed array inside
 * the library: about 8 MiB of device memory that every GPU loading
 * librr.so holds until the process exits.  Limits: bh * nq <= 1048576 and
 * bh <= 4096; larger problems return RR_ECAPACITY and enqueue nothing.
 * The first call on a device looks up that array's device address and sets
 * the kernels' shared-memory attributes (set-up done once per device, with
 * the device current); make that first call before any stream capture.  Every call on a device shares the one array
 * and it keeps the last call's contents; nothing in it has to start at zero
 * (each call writes every list length it reads).  Calls that can overlap
 * on the GPU (different streams, or different ledgers run concurrently)
 * race on it: run them on one stream or serialise them.  The call keeps no
 * host state, so it cannot check the layer order: the caller must start a
 * sequence at layer 0 or an anchor layer and pass increasing layers.
 * Device-side errors land in d_counters[RR_CNT_ERROR] like the ledger's
 * (bit 0: an out-of-range ledger id; bit 1: a bounded wait timed out and the
 * layer's results are not valid); the caller reads that slot after the
 * stream reaches the call.  Errors: RR_EINVAL (bad config, null or
 * misaligned pointer, layer < 0), RR_ECAPACITY, RR_ECUDA.  Calls no
 * cudaMalloc, cudaFree or allocating library routine. */
rr_status rr_route_layer_static(const rr_config *cfg, const void *d_qc, const void *d_kc,
                                int32_t layer, int32_t *d_ids, float *d_alpha,
                                int32_t *d_anchor_layer, uint8_t *d_flags, int64_t *d_counters,
                                void *stream);

/* Test hook: the budget, in SM clock cycles, of the accumulator waits in the
 * epilogue of the tensor-core selection kernel (0, the default: about a
 * second, which only a stalled GPU exhausts).  Every wait in the tensor-core
 * kernels is bounded; when one runs out the CTA stops issuing, drains its
 * copies, waits for its last MMA, frees its TMEM and sets bit 1 of the error
 * word, and its rows are redone exactly on the retry path.  A short budget
 * makes that happen on purpose, so a test can check the path; production
 * callers leave it at 0.  No CUDA call; RR_EINVAL for a NULL ledger or a
 * negative budget. */
rr_status rr_ledger_set_wait_budget(rr_ledger *ledger, int64_t cycles);

/* Human-readable name of a status code (static string). */
const char *rr_status_string(rr_status status);

#ifdef __cplusplus
}
#endif

#endif /* RR_H */
