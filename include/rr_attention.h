/*
 * rr_attention.h -- C ABI of the sparse attention that consumes a route
 * (librr.so).
 *
 * Method: "RouteRelay: Event-Triggered Cross-Layer Route Reuse for Efficient
 * Dynamic Sparse Attention" (arXiv 2609.07306), cited as RouteRelay §x.
 * The router's output is a route per query chunk: the ids of the key chunks
 * it attends (§2.1 Eq. 2; the first k ids of a ledger row, rr.h).  The
 * selected chunks are expanded into token indices and attended with an
 * online softmax (§2.1); every layer attends with its own q, K, V over the
 * (possibly reused) route (§2.2 Eq. 3):
 *
 *     o_t = softmax(q_t K_T^T * scale) V_T,   T = tokens of the route's chunks
 *
 * Conventions (the page leaves them to the attention backend, §4.3):
 *  - Chunk j covers tokens j*chunk .. j*chunk + chunk - 1, for queries and
 *    keys alike; query token t belongs to query chunk t / chunk.
 *  - causal != 0: key token s is visible to query token t iff s <= t.
 *  - Route ids that are negative (-1 padding) or >= the number of key
 *    chunks are skipped; with causal, so are ids greater than the query
 *    chunk's own (they hold no visible token).  Every other entry
 *    contributes its chunk once per occurrence.
 *  - A query token with no visible key gets a zero output row.
 *  - Same stream, ownership and error conventions as rr.h: device memory is
 *    the caller's, the call enqueues on `stream` and returns without
 *    synchronising, argument errors return before any CUDA call.
 */
#ifndef RR_ATTENTION_H
#define RR_ATTENTION_H

#include <stddef.h>
#include <stdint.h>

#include "rr.h"

#ifdef __cplusplus
extern "C" {
#endif

/* Shape of one sparse-attention call.  Limits: bh, nq_tokens, nk_tokens >= 0
 * (bh == 0 or nq_tokens == 0: nothing to do); dh in {64, 128}; chunk in
 * {16, 32, 64, 128}; nq_tokens and nk_tokens multiples of chunk;
 * 0 <= width <= 1024; route_stride >= max(width, 1);
 * bh * (nq_tokens / chunk) <= 2^31 - 1; scale finite and >= 0. */
typedef struct {
    int32_t bh;           /* heads (batch x heads) */
    int32_t nq_tokens;    /* query tokens per head */
    int32_t nk_tokens;    /* key / value tokens per head */
    int32_t dh;           /* head dimension of q, k, v */
    int32_t chunk;        /* tokens per chunk */
    int32_t width;        /* route entries read per query chunk */
    int32_t route_stride; /* int32 elements from one query chunk's route to the next */
    int32_t causal;       /* nonzero: token-level causal mask (s <= t) */
    float scale;          /* softmax scale; 0 selects 1/sqrt(dh) (Eq. 3) */
} rr_attn_config;

/* Sparse attention over a route (RouteRelay §2.1, §2.2 Eq. 3).
 *   d_q     bf16 [bh, nq_tokens, dh], row-major, 16-byte aligned
 *   d_k     bf16 [bh, nk_tokens, dh], the same layout (may be NULL when nk_tokens == 0)
 *   d_v     bf16 [bh, nk_tokens, dh], the same layout
 *   d_route int32 [bh, nq_tokens / chunk, route_stride]; entries 0..width-1 of
 *           each query chunk's row are read.  A ledger's ids (rr_ledger_device_view)
 *           serve directly: route_stride = c, width = k.
 *   d_out   fp32 [bh, nq_tokens, dh], 16-byte aligned; written in full.
 * The scores and the softmax are fp32; P is rounded to bf16 before the
 * P.V product (both products run on the tensor cores with fp32
 * accumulation), so each output element is within about 2^-8 of the
 * softmax-weighted mean of |v| of the exact result.  Errors: RR_EINVAL
 * (bad shape, null or misaligned pointer), RR_ECUDA (launch). */
rr_status rr_sparse_attention(const rr_attn_config *cfg, const void *d_q, const void *d_k,
                              const void *d_v, const int32_t *d_route, float *d_out,
                              void *stream);

#ifdef __cplusplus
}
#endif

#endif /* RR_ATTENTION_H */
