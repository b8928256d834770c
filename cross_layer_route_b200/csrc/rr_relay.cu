// rr_relay.cu -- relay-layer kernels of the B200 RouteRelay router.
//
// Method: "RouteRelay: Event-Triggered Cross-Layer Route Reuse for Efficient
// Dynamic Sparse Attention" (arXiv 2609.07306), cited as RouteRelay §x.
//
//  relay_rescore: candidate rescoring and the challenge test (§3.2 Eq. 5-8,
//      §4.2 "a GPU kernel computes alpha, beta, and one refresh flag per query
//      row").  Shapes the tensor-core full routing serves are rescored from
//      dense tensor-core tiles instead (relay_rescore_tc_kernel, in
//      rr_route_tc.cu); the kernels here take the others, one warp per
//      query row.  For d in {64, 128, 256} eight lanes
//      share a candidate (16-byte loads interleaved so that the eight read
//      one 128-byte line at a time; each keeps its eighth of q in registers);
//      other d use one lane per candidate.
//  compact_flags: the prefix sum that compacts unstable row ids (§4.2), one
//      CTA per head, writing an ascending per-head list and its length.
//  finalize_layer: per-layer counters (§4.1: the refreshed-row fraction is
//      "exposed to the runtime").
#include <float.h>

#include "rr_device.cuh"
#include "rr_internal.h"

namespace rr {
namespace {

constexpr int kRescoreThreads = 256;
constexpr int kRescoreWarps = kRescoreThreads / 32;
constexpr int kDMax = 256;

// Score of one candidate row k_j against the warp's query row (fp32 in
// shared memory), 16-byte key loads and 8 independent partial sums.
template <typename T> struct Vec16;
template <> struct Vec16<float> {
    static constexpr int kElems = 4;
    static __device__ __forceinline__ void fma16(const float *q, uint4 kv, float *acc, int slot) {
        const float4 qv = *reinterpret_cast<const float4 *>(q);
        acc[(slot * 4 + 0) & 7] = fmaf(qv.x, __uint_as_float(kv.x), acc[(slot * 4 + 0) & 7]);
        acc[(slot * 4 + 1) & 7] = fmaf(qv.y, __uint_as_float(kv.y), acc[(slot * 4 + 1) & 7]);
        acc[(slot * 4 + 2) & 7] = fmaf(qv.z, __uint_as_float(kv.z), acc[(slot * 4 + 2) & 7]);
        acc[(slot * 4 + 3) & 7] = fmaf(qv.w, __uint_as_float(kv.w), acc[(slot * 4 + 3) & 7]);
    }
};
template <> struct Vec16<__nv_bfloat16> {
    static constexpr int kElems = 8;
    static __device__ __forceinline__ void fma16(const float *q, uint4 kv, float *acc, int) {
        const float4 qa = *reinterpret_cast<const float4 *>(q);
        const float4 qb = *reinterpret_cast<const float4 *>(q + 4);
        // bf16 -> fp32 is exact: the bf16 bits become the high half
        acc[0] = fmaf(qa.x, __uint_as_float(kv.x << 16), acc[0]);
        acc[1] = fmaf(qa.y, __uint_as_float(kv.x & 0xffff0000u), acc[1]);
        acc[2] = fmaf(qa.z, __uint_as_float(kv.y << 16), acc[2]);
        acc[3] = fmaf(qa.w, __uint_as_float(kv.y & 0xffff0000u), acc[3]);
        acc[4] = fmaf(qb.x, __uint_as_float(kv.z << 16), acc[4]);
        acc[5] = fmaf(qb.y, __uint_as_float(kv.z & 0xffff0000u), acc[5]);
        acc[6] = fmaf(qb.z, __uint_as_float(kv.w << 16), acc[6]);
        acc[7] = fmaf(qb.w, __uint_as_float(kv.w & 0xffff0000u), acc[7]);
    }
};

template <typename T, int D>
__device__ __forceinline__ float dot_row(const float *qs, const T *kp, int d) {
    constexpr int E = Vec16<T>::kElems;
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    const uint4 *k4 = reinterpret_cast<const uint4 *>(kp);
    if constexpr (D > 0) {
        uint4 kv[D / E];
#pragma unroll
        for (int c = 0; c < D / E; ++c) kv[c] = __ldg(k4 + c);   // all loads in flight together
#pragma unroll
        for (int c = 0; c < D / E; ++c) Vec16<T>::fma16(qs + c * E, kv[c], acc, c);
    } else {
        const int nc = d / E;
        int c = 0;
        for (; c + 1 < nc; c += 2) {
            Vec16<T>::fma16(qs + c * E, __ldg(k4 + c), acc, 0);
            Vec16<T>::fma16(qs + (c + 1) * E, __ldg(k4 + c + 1), acc, 1);
        }
        if (c < nc) Vec16<T>::fma16(qs + c * E, __ldg(k4 + c), acc, 0);
    }
    return ((acc[0] + acc[1]) + (acc[2] + acc[3])) + ((acc[4] + acc[5]) + (acc[6] + acc[7]));
}

// One warp per query row, one lane per candidate (RouteRelay §3.2 Eq. 5-8).
template <typename T, int D>
__global__ void __launch_bounds__(kRescoreThreads)
relay_rescore_kernel(LedgerDev L, const T *__restrict__ Q, const T *__restrict__ K, int layer) {
    __shared__ __align__(16) float qs_all[kRescoreWarps][kDMax];
    __shared__ unsigned long long pair_sum[kRescoreWarps];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long long rows = (long long)L.bh * L.nq;
    const long long grow = (long long)blockIdx.x * kRescoreWarps + warp;
    const int d = D > 0 ? D : L.d;
    unsigned long long pairs = 0;
    if (grow < rows) {
        const int h = (int)(grow / L.nq);
        const int i = (int)(grow - (long long)h * L.nq);
        const int n_valid = valid_keys(i, L.nk, L.causal);
        float *qs = qs_all[warp];
        for (int t = lane * 4; t < d; t += 128) {
            float v[4];
            Elem<T>::load4(Q + grow * d + t, v);
            *reinterpret_cast<float4 *>(qs + t) = make_float4(v[0], v[1], v[2], v[3]);
        }
        __syncwarp();
        const int32_t *idr = L.ids + grow * L.c;
        const T *Kh = K + (size_t)h * L.nk * d;
        float amin = INFINITY, bmax = -INFINITY;
        bool bad = false;
        int ncand = 0;
        for (int e0 = 0; e0 < L.c; e0 += 32) {
            const int e = e0 + lane;
            const int j = e < L.c ? idr[e] : -1;
            const bool valid = j >= 0 && j < n_valid;
            bad |= j >= n_valid || j < -1;
            if (valid) {
                const float sc = dot_row<T, D>(qs, Kh + (size_t)j * d, d);
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
        if (lane == 0) {
            const uint8_t fl = relay_decide(L, (size_t)grow, layer, amin, bmax);  // Eq. 8
            const bool refresh = (fl & 1u) != 0u;
            L.flags[grow] = fl;
            if (!refresh) L.alpha[grow] = amin;
            if (any_bad) atomicOr(&L.counters[2], 1ULL);
        }
        pairs = (unsigned long long)ncand;
    }
    if (lane == 0) pair_sum[warp] = pairs;
    __syncthreads();
    if (threadIdx.x == 0) {
        unsigned long long s = 0;
        for (int w = 0; w < kRescoreWarps; ++w) s += pair_sum[w];
        if (s) atomicAdd(&L.counters[1], s);
    }
}

constexpr int kCompactThreads = 1024;

__global__ void __launch_bounds__(kCompactThreads) compact_flags_kernel(LedgerDev L) {
    __shared__ int warp_tot[kCompactThreads / 32];
    __shared__ unsigned long long warp_pairs[kCompactThreads / 32];
    const int h = blockIdx.x;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint8_t *fl = L.flags + (size_t)h * L.nq;
    int32_t *lst = L.list + (size_t)h * L.nq;
    int base = 0;
    unsigned long long pairs = 0;
    for (int i0 = 0; i0 < L.nq; i0 += kCompactThreads) {
        const int i = i0 + tid;
        const bool f = i < L.nq && (fl[i] & 1u) != 0;   // bit 0: refresh (bit 1: hysteresis mark)
        const unsigned wm = __ballot_sync(kFull, f);
        if (lane == 0) warp_tot[warp] = __popc(wm);
        __syncthreads();
        int before = 0, total = 0;
        for (int w = 0; w < kCompactThreads / 32; ++w) {
            const int t = warp_tot[w];
            before += w < warp ? t : 0;
            total += t;
        }
        if (f) {
            lst[base + before + __popc(wm & lanemask_lt())] = i;
            pairs += (unsigned long long)valid_keys(i, L.nk, L.causal);
        }
        base += total;
        __syncthreads();
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) pairs += __shfl_xor_sync(kFull, pairs, o);
    if (lane == 0) warp_pairs[warp] = pairs;
    __syncthreads();
    if (tid == 0) {
        unsigned long long s = 0;
        for (int w = 0; w < kCompactThreads / 32; ++w) s += warp_pairs[w];
        L.head_count[h] = base;
        if (base) atomicAdd(&L.counters[0], (unsigned long long)base);
        if (s) {
            atomicAdd(&L.counters[1], s);
            atomicAdd(&L.counters[8], s);
        }
    }
}

__global__ void finalize_layer_kernel(LedgerDev L, int layer, long long add_rows,
                                      long long add_pairs, long long add_full_pairs) {
    unsigned long long *c = L.counters;
    c[0] += (unsigned long long)add_rows;
    c[1] += (unsigned long long)add_pairs;
    c[8] += (unsigned long long)add_full_pairs;
    c[3] += c[0];
    c[4] += c[1];
    c[9] += c[8];
    c[5] += 1ULL;
    c[6] = (unsigned long long)(long long)layer;
}

}  // namespace

// Eight lanes per candidate: lane octet g of the warp scores candidate
// it*4 + g, each lane an eighth of the key row (R/8 bytes, R = d * elem
// size, a multiple of 128), with its eighth of the query row in registers.
// Per load instruction an octet reads one whole 128-byte line, so the warp
// touches 4 lines, each in full.
template <typename T, int D>
__global__ void __launch_bounds__(kRescoreThreads)
relay_rescore_oct_kernel(LedgerDev L, const T *__restrict__ Q, const T *__restrict__ K, int layer) {
    constexpr int E = Vec16<T>::kElems;         // elements per 16-byte load
    constexpr int kLanes = 8;                   // lanes per candidate
    constexpr int kChunks = D / E / kLanes;     // 16-byte loads per lane
    static_assert(kChunks >= 1, "one 16-byte load per lane at least");
    __shared__ unsigned long long pair_sum[kRescoreWarps];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int oct = lane >> 3, part = lane & 7;
    const long long rows = (long long)L.bh * L.nq;
    const long long grow = (long long)blockIdx.x * kRescoreWarps + warp;
    unsigned long long pairs = 0;
    if (grow < rows) {
        const int h = (int)(grow / L.nq);
        const int i = (int)(grow - (long long)h * L.nq);
        const int n_valid = valid_keys(i, L.nk, L.causal);
        // this lane's eighth of q, as fp32: the 16-byte chunks part, part + 8,
        // ... (eight lanes read one 128-byte line per load)
        float qv[kChunks * E];
        {
            const uint4 *q4 = reinterpret_cast<const uint4 *>(Q + grow * D) + part;
#pragma unroll
            for (int c = 0; c < kChunks; ++c) {
                const uint4 u = __ldg(q4 + kLanes * c);
                if constexpr (E == 8) {
                    qv[c * 8 + 0] = __uint_as_float(u.x << 16); qv[c * 8 + 1] = __uint_as_float(u.x & 0xffff0000u);
                    qv[c * 8 + 2] = __uint_as_float(u.y << 16); qv[c * 8 + 3] = __uint_as_float(u.y & 0xffff0000u);
                    qv[c * 8 + 4] = __uint_as_float(u.z << 16); qv[c * 8 + 5] = __uint_as_float(u.z & 0xffff0000u);
                    qv[c * 8 + 6] = __uint_as_float(u.w << 16); qv[c * 8 + 7] = __uint_as_float(u.w & 0xffff0000u);
                } else {
                    qv[c * 4 + 0] = __uint_as_float(u.x); qv[c * 4 + 1] = __uint_as_float(u.y);
                    qv[c * 4 + 2] = __uint_as_float(u.z); qv[c * 4 + 3] = __uint_as_float(u.w);
                }
            }
        }
        const int32_t *idr = L.ids + grow * L.c;
        const T *Kh = K + (size_t)h * L.nk * D;
        float amin = INFINITY, bmax = -INFINITY;
        bool bad = false;
        int ncand = 0;
#pragma unroll 2
        for (int e0 = 0; e0 < L.c; e0 += 32 / kLanes) {
            const int e = e0 + oct;
            const int j = e < L.c ? idr[e] : -1;
            const bool valid = j >= 0 && j < n_valid;
            bad |= j >= n_valid || j < -1;
            float acc[4] = {0.f, 0.f, 0.f, 0.f};
            if (valid) {
                const uint4 *k4 = reinterpret_cast<const uint4 *>(Kh + (size_t)j * D) + part;
                uint4 kv[kChunks];
#pragma unroll
                for (int c = 0; c < kChunks; ++c) kv[c] = __ldg(k4 + kLanes * c);
#pragma unroll
                for (int c = 0; c < kChunks; ++c) {
                    const uint4 u = kv[c];
                    if constexpr (E == 8) {
                        acc[0] = fmaf(qv[c * 8 + 0], __uint_as_float(u.x << 16), acc[0]);
                        acc[1] = fmaf(qv[c * 8 + 1], __uint_as_float(u.x & 0xffff0000u), acc[1]);
                        acc[2] = fmaf(qv[c * 8 + 2], __uint_as_float(u.y << 16), acc[2]);
                        acc[3] = fmaf(qv[c * 8 + 3], __uint_as_float(u.y & 0xffff0000u), acc[3]);
                        acc[0] = fmaf(qv[c * 8 + 4], __uint_as_float(u.z << 16), acc[0]);
                        acc[1] = fmaf(qv[c * 8 + 5], __uint_as_float(u.z & 0xffff0000u), acc[1]);
                        acc[2] = fmaf(qv[c * 8 + 6], __uint_as_float(u.w << 16), acc[2]);
                        acc[3] = fmaf(qv[c * 8 + 7], __uint_as_float(u.w & 0xffff0000u), acc[3]);
                    } else {
                        acc[0] = fmaf(qv[c * 4 + 0], __uint_as_float(u.x), acc[0]);
                        acc[1] = fmaf(qv[c * 4 + 1], __uint_as_float(u.y), acc[1]);
                        acc[2] = fmaf(qv[c * 4 + 2], __uint_as_float(u.z), acc[2]);
                        acc[3] = fmaf(qv[c * 4 + 3], __uint_as_float(u.w), acc[3]);
                    }
                }
            }
            float sc = (acc[0] + acc[1]) + (acc[2] + acc[3]);
            sc += __shfl_xor_sync(kFull, sc, 1);
            sc += __shfl_xor_sync(kFull, sc, 2);
            sc += __shfl_xor_sync(kFull, sc, 4);
            if (valid && part == 0) {
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
        if (lane == 0) {
            const uint8_t fl = relay_decide(L, (size_t)grow, layer, amin, bmax);  // Eq. 8
            const bool refresh = (fl & 1u) != 0u;
            L.flags[grow] = fl;
            if (!refresh) L.alpha[grow] = amin;
            if (any_bad) atomicOr(&L.counters[2], 1ULL);
        }
        pairs = (unsigned long long)ncand;
    }
    if (lane == 0) pair_sum[warp] = pairs;
    __syncthreads();
    if (threadIdx.x == 0) {
        unsigned long long s = 0;
        for (int w = 0; w < kRescoreWarps; ++w) s += pair_sum[w];
        if (s) atomicAdd(&L.counters[1], s);
    }
}

template <typename T>
static void rescore_dispatch(const LedgerDev &L, const void *q, const void *k, int layer,
                             unsigned grid, cudaStream_t s) {
    const T *Q = static_cast<const T *>(q);
    const T *K = static_cast<const T *>(k);
    switch (L.d) {
        case 64: relay_rescore_oct_kernel<T, 64><<<grid, kRescoreThreads, 0, s>>>(L, Q, K, layer); break;
        case 128: relay_rescore_oct_kernel<T, 128><<<grid, kRescoreThreads, 0, s>>>(L, Q, K, layer); break;
        case 256: relay_rescore_oct_kernel<T, 256><<<grid, kRescoreThreads, 0, s>>>(L, Q, K, layer); break;
        default: relay_rescore_kernel<T, 0><<<grid, kRescoreThreads, 0, s>>>(L, Q, K, layer); break;
    }
}

cudaError_t launch_relay_rescore(const LedgerDev &L, int dtype, const void *q, const void *k,
                                 int layer, cudaStream_t s) {
    if (route_rows_tc_supported(L, dtype)) return launch_relay_rescore_tc(L, q, k, layer, s);
    const long long rows = (long long)L.bh * L.nq;
    const unsigned grid = (unsigned)((rows + kRescoreWarps - 1) / kRescoreWarps);
    if (dtype == kBF16) rescore_dispatch<__nv_bfloat16>(L, q, k, layer, grid, s);
    else rescore_dispatch<float>(L, q, k, layer, grid, s);
    return cudaGetLastError();
}

cudaError_t launch_compact(const LedgerDev &L, cudaStream_t s) {
    compact_flags_kernel<<<L.bh, kCompactThreads, 0, s>>>(L);
    return cudaGetLastError();
}

cudaError_t launch_finalize(const LedgerDev &L, int layer, long long add_rows,
                            long long add_pairs, long long add_full_pairs, cudaStream_t s) {
    finalize_layer_kernel<<<1, 1, 0, s>>>(L, layer, add_rows, add_pairs, add_full_pairs);
    return cudaGetLastError();
}

}  // namespace rr
