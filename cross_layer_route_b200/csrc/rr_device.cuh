// rr_device.cuh -- device helpers of the B200 RouteRelay router.
//
// Method: "RouteRelay: Event-Triggered Cross-Layer Route Reuse for Efficient
// Dynamic Sparse Attention" (arXiv 2609.07306), cited as RouteRelay §x.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "rr_internal.h"

namespace rr {

constexpr unsigned kFull = 0xffffffffu;

__device__ __forceinline__ unsigned lane_id() { return threadIdx.x & 31u; }
__device__ __forceinline__ unsigned lanemask_lt() { return (1u << lane_id()) - 1u; }

// Strict ranking order of (score, chunk) pairs: higher score first, then the
// smaller chunk index (the tie reading of RouteRelay §2.1 Eq. 2).
__device__ __forceinline__ bool ranks_before(float s1, int j1, float s2, int j2) {
    return s1 > s2 || (s1 == s2 && j1 < j2);
}

// Number of key chunks query row `row` may route to (causal: 0..row).
__device__ __forceinline__ int valid_keys(int row, int nk, int causal) {
    return causal ? min(row + 1, nk) : nk;
}

// Mandatory global sentinels (RouteRelay §3.1 item 3, "sink and recent
// chunks"): candidate t < g_sink + g_recent of query row `row` is sink chunk
// t, then recent chunk row-g_recent+1+(t-g_sink).  A candidate is kept when
// it is valid, outside route U near-miss, and not a recent chunk that is
// also a sink chunk (listed once, as a sink).
__device__ __forceinline__ int global_cand(const LedgerDev &L, int row, int t) {
    return t < L.g_sink ? t : row - L.g_recent + 1 + (t - L.g_sink);
}
__device__ __forceinline__ bool global_cand_listable(const LedgerDev &L, int t, int j, int n_valid) {
    return j >= 0 && j < n_valid && !(t >= L.g_sink && j < L.g_sink);
}
// Whether valid chunk j is one of row's global candidates (such chunks are
// outside the random sentinels' pool).
__device__ __forceinline__ bool is_global_cand(const LedgerDev &L, int row, int n_valid, int j) {
    return j >= 0 && j < n_valid && (j < L.g_sink || (j <= row && j > row - L.g_recent));
}

// The relay decision of one row (RouteRelay §3.2), as the row's new flags
// byte: bit 0 = refresh, bit 1 = the row keeps (or, refreshed at this relay
// layer, receives) the hysteresis mark.  Refresh unless alpha > beta +
// gamma_i (Eq. 8; gamma_i from the per-row margins when the ledger has
// them).  A row whose ledger is max_age layers old refreshes in any case
// (the per-row lifetime bound; max_age 0 = off); otherwise a row built
// min_reuse or fewer layers ago is reused without the test (the hysteresis
// horizon; min_reuse 0 = off; the mark is left as it is).  A marked row
// tests with max(gamma_i, gamma_h) and loses the mark when it passes (the
// "larger guard margin until its anchor margin recovers"; gamma_h 0 = off).
// A NaN margin makes the row refresh.
__device__ __forceinline__ uint8_t relay_decide(const LedgerDev &L, size_t grow, int layer, float alpha,
                                                float beta) {
    const uint8_t refreshed = (uint8_t)(1u | (L.gamma_h > 0.0f ? 2u : 0u));
    const bool marked = L.gamma_h > 0.0f && (L.flags[grow] & 2u) != 0u;
    if (L.max_age > 0 || L.min_reuse > 0) {   // the row's age is read only when needed
        const int age = layer - L.anchor_layer[grow];
        if (L.max_age > 0 && age >= L.max_age) return refreshed;
        if (L.min_reuse > 0 && age <= L.min_reuse) return marked ? 2u : 0u;
    }
    float g = L.gamma_rows ? L.gamma_rows[grow] : L.gamma;
    if (marked && L.gamma_h > g) g = L.gamma_h;
    return (alpha > beta + g) ? (uint8_t)0u : refreshed;
}

// ---- Philox4x32-10 (Salmon, Moraes, Dror, Shaw, SC'11) --------------------
// Ten rounds; each multiplies counter words 0 and 2 by the two Philox
// multipliers, mixes the high halves with words 1 and 3 and the round key,
// and moves the low halves to words 1 and 3.  The key advances by the two
// Weyl increments between rounds.
struct PhiloxOut { uint32_t w[4]; };

__device__ __forceinline__ PhiloxOut philox4x32_10(uint32_t c0, uint32_t c1, uint32_t c2,
                                                   uint32_t c3, uint32_t k0, uint32_t k1) {
    const uint32_t kMulA = 0xD2511F53u, kMulB = 0xCD9E8D57u;
    const uint32_t kWeylA = 0x9E3779B9u, kWeylB = 0xBB67AE85u;
#pragma unroll
    for (int round = 0; round < 10; ++round) {
        const uint32_t hiA = __umulhi(kMulA, c0), loA = kMulA * c0;
        const uint32_t hiB = __umulhi(kMulB, c2), loB = kMulB * c2;
        const uint32_t n0 = hiB ^ c1 ^ k0;
        const uint32_t n2 = hiA ^ c3 ^ k1;
        c0 = n0; c1 = loB; c2 = n2; c3 = loA;
        k0 += kWeylA; k1 += kWeylB;
    }
    PhiloxOut o;
    o.w[0] = c0; o.w[1] = c1; o.w[2] = c2; o.w[3] = c3;
    return o;
}

// ---- element loads ----------------------------------------------------------
template <typename T> struct Elem;
template <> struct Elem<float> {
    static __device__ __forceinline__ float to_f32(float x) { return x; }
    // 16-byte vector of 4 elements
    static __device__ __forceinline__ void load4(const float *p, float *o) {
        float4 v = *reinterpret_cast<const float4 *>(p);
        o[0] = v.x; o[1] = v.y; o[2] = v.z; o[3] = v.w;
    }
};
template <> struct Elem<__nv_bfloat16> {
    static __device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }
    static __device__ __forceinline__ void load4(const __nv_bfloat16 *p, float *o) {
        uint2 v = *reinterpret_cast<const uint2 *>(p);
        __nv_bfloat162 a = *reinterpret_cast<__nv_bfloat162 *>(&v.x);
        __nv_bfloat162 b = *reinterpret_cast<__nv_bfloat162 *>(&v.y);
        float2 fa = __bfloat1622float2(a), fb = __bfloat1622float2(b);
        o[0] = fa.x; o[1] = fa.y; o[2] = fb.x; o[3] = fb.y;
    }
};

}  // namespace rr
