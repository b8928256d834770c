// rr_route_simt.cu -- full routing of a set of query rows on the CUDA cores.
//
// Method: "RouteRelay: Event-Triggered Cross-Layer Route Reuse for Efficient
// Dynamic Sparse Attention" (arXiv 2609.07306), cited as RouteRelay §x.
//
// One kernel serves both the anchor layer (every row, §4.1 "an anchor layer
// constructs this state from a complete chunk-score matrix") and the refresh
// of the compacted unstable rows at a relay layer (§4.2, "a second kernel
// computes complete score rows only for the compacted IDs and updates their
// ledgers").  Per CTA: one head, 32 query rows (8 warps x 4 rows).  Key
// chunks of 64 are staged in shared memory (transposed, fp32), each warp
// scores its 4 rows against them (lane = key), and every score goes through
// a warp-wide threshold filter into a per-row candidate buffer in shared
// memory; a full buffer is sorted (bitonic, warp-cooperative) and cut back
// to the k + m best, whose weakest score becomes the new threshold.  The
// score matrix never leaves the SM.
#include <float.h>
#include <limits.h>

#include "rr_device.cuh"
#include "rr_internal.h"

namespace rr {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kRowsPerWarp = 4;
constexpr int kTileRows = kWarps * kRowsPerWarp;  // 32
constexpr int kKeyTile = 64;
constexpr int kKeyStride = kKeyTile + 1;          // padded row of the transposed key tile
constexpr int kRandMax = 128;

struct SmemLayout {
    size_t q_off, k_off, bs_off, bi_off, rows_off, rnd_off, total;
};

__host__ __device__ inline size_t align16(size_t x) { return (x + 15) & ~size_t(15); }

__host__ __device__ inline SmemLayout smem_layout(int d, int cap) {
    SmemLayout s;
    size_t o = 0;
    s.q_off = o;    o = align16(o + sizeof(float) * kTileRows * d);
    s.k_off = o;    o = align16(o + sizeof(float) * d * kKeyStride);
    s.bs_off = o;   o = align16(o + sizeof(float) * kTileRows * cap);
    s.bi_off = o;   o = align16(o + sizeof(int) * kTileRows * cap);
    s.rows_off = o; o = align16(o + sizeof(int) * kTileRows);
    s.rnd_off = o;  o = align16(o + sizeof(int) * kWarps * kRandMax);
    s.total = o;
    return s;
}

// Warp-cooperative bitonic sort of one row's candidate buffer, best first.
__device__ void warp_sort_best_first(float *bs, int *bi, int cnt, int cap) {
    const int lane = lane_id();
    for (int e = cnt + lane; e < cap; e += 32) { bs[e] = -INFINITY; bi[e] = INT_MAX; }
    __syncwarp();
    for (int size = 2; size <= cap; size <<= 1) {
        for (int stride = size >> 1; stride > 0; stride >>= 1) {
            for (int e = lane; e < (cap >> 1); e += 32) {
                const int lo = ((e & ~(stride - 1)) << 1) | (e & (stride - 1));
                const int hi = lo + stride;
                const bool best_first = (lo & size) == 0;
                const float a = bs[lo], b = bs[hi];
                const int ia = bi[lo], ib = bi[hi];
                const bool swap = best_first ? ranks_before(b, ib, a, ia) : ranks_before(a, ia, b, ib);
                if (swap) { bs[lo] = b; bs[hi] = a; bi[lo] = ib; bi[hi] = ia; }
            }
            __syncwarp();
        }
    }
}

__device__ __forceinline__ bool in_list(const int *lst, int n, int j) {
    for (int e = 0; e < n; ++e)
        if (lst[e] == j) return true;
    return false;
}

// Random sentinels of one row (RouteRelay §3.1 item 2, §3.4): r distinct
// chunks from the valid chunks outside route U near-miss, drawn with
// Philox4x32-10 (key = seed, counter = (global head, row, layer, t/4), word
// t%4, chunk = (word * n_valid) >> 32), repeats rejected; 32 draws per warp
// step, accepted in draw order.  A pool of at most r chunks is taken whole in
// ascending order; a row that exhausts max_draws is filled in ascending order.
__device__ void draw_random_sentinels(const LedgerDev &L, int ghead, int row, int layer,
                                      int n_valid, const int *excl, int n_excl, int n_glob,
                                      int *acc_buf, int32_t *out) {
    const int lane = lane_id();
    const int r = L.r;
    if (r == 0) return;
    const int np = n_valid - n_excl - n_glob;   // the global candidates are outside the pool
    int acc = 0;
    if (np > r) {
        for (int t0 = 0; acc < r && t0 < L.max_draws; t0 += 32) {
            const int t = t0 + lane;
            const PhiloxOut o = philox4x32_10((uint32_t)ghead, (uint32_t)row, (uint32_t)layer,
                                              (uint32_t)(t >> 2), L.seed_lo, L.seed_hi);
            const int sel = t & 3;
            const uint32_t w = sel == 0 ? o.w[0] : sel == 1 ? o.w[1] : sel == 2 ? o.w[2] : o.w[3];
            const int j = (int)__umulhi(w, (uint32_t)n_valid);
            const bool cand = t < L.max_draws && !in_list(excl, n_excl, j) &&
                              !is_global_cand(L, row, n_valid, j) && !in_list(acc_buf, acc, j);
            const unsigned cm = __ballot_sync(kFull, cand);
            const unsigned same = __match_any_sync(kFull, j) & cm;
            const bool first = cand && ((same & lanemask_lt()) == 0);
            const unsigned fm = __ballot_sync(kFull, first);
            const int pos = acc + __popc(fm & lanemask_lt());
            if (first && pos < r) acc_buf[pos] = j;
            acc = min(r, acc + __popc(fm));
            __syncwarp();
        }
        if (acc < r && lane == 0) atomicAdd(&L.counters[7], 1ULL);
    }
    for (int j0 = 0; acc < r && j0 < n_valid; j0 += 32) {
        const int j = j0 + lane;
        const bool cand = j < n_valid && !in_list(excl, n_excl, j) &&
                          !is_global_cand(L, row, n_valid, j) && !in_list(acc_buf, acc, j);
        const unsigned cm = __ballot_sync(kFull, cand);
        const int pos = acc + __popc(cm & lanemask_lt());
        if (cand && pos < r) acc_buf[pos] = j;
        acc = min(r, acc + __popc(cm));
        __syncwarp();
    }
    for (int e = lane; e < r; e += 32) out[e] = e < acc ? acc_buf[e] : -1;
}

template <typename T>
__global__ void __launch_bounds__(kThreads)
route_rows_kernel(LedgerDev L, const T *__restrict__ Q, const T *__restrict__ K, int layer,
                  int use_list, int cap) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    const SmemLayout lay = smem_layout(L.d, cap);
    float *Qs = reinterpret_cast<float *>(smem_raw + lay.q_off);
    float *Ks = reinterpret_cast<float *>(smem_raw + lay.k_off);
    float *bs_all = reinterpret_cast<float *>(smem_raw + lay.bs_off);
    int *bi_all = reinterpret_cast<int *>(smem_raw + lay.bi_off);
    int *rows_s = reinterpret_cast<int *>(smem_raw + lay.rows_off);
    int *rnd_all = reinterpret_cast<int *>(smem_raw + lay.rnd_off);

    const int h = blockIdx.y;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int d = L.d, nq = L.nq, nk = L.nk;
    const int count = use_list ? L.head_count[h] : nq;
    // tiles of 32 rows, grid-stride (a grid narrower than the rows, as the
    // retry lists use, takes several tiles per CTA)
    for (int row0 = blockIdx.x * kTileRows; row0 < count; row0 += gridDim.x * kTileRows) {
        __syncthreads();   // the previous tile's rows, queries and buffers are done with
        const int n_rows = min(kTileRows, count - row0);

        if (tid < kTileRows) {
            int row = -1;
            if (tid < n_rows) row = use_list ? L.list[(size_t)h * nq + row0 + tid] : row0 + tid;
            rows_s[tid] = row;
        }
        __syncthreads();
        // query tile -> shared (fp32), zero rows for empty slots
        const int d4 = d >> 2;
        for (int e = tid; e < kTileRows * d4; e += kThreads) {
            const int rr_ = e / d4, t = (e - rr_ * d4) * 4;
            const int row = rows_s[rr_];
            float v[4] = {0.f, 0.f, 0.f, 0.f};
            if (row >= 0) Elem<T>::load4(Q + ((size_t)h * nq + row) * d + t, v);
            *reinterpret_cast<float4 *>(Qs + rr_ * d + t) = make_float4(v[0], v[1], v[2], v[3]);
        }
        int max_row = -1;
        for (int e = 0; e < n_rows; ++e) max_row = max(max_row, rows_s[e]);
        const int kend = L.causal ? min(nk, max_row + 1) : nk;

        // per-row selection state (warp-uniform)
        int my_rows[kRowsPerWarp], my_kend[kRowsPerWarp], cnt[kRowsPerWarp];
        float thr[kRowsPerWarp];
    #pragma unroll
        for (int r = 0; r < kRowsPerWarp; ++r) {
            my_rows[r] = rows_s[warp * kRowsPerWarp + r];
            my_kend[r] = my_rows[r] >= 0 ? valid_keys(my_rows[r], nk, L.causal) : 0;
            cnt[r] = 0;
            thr[r] = -INFINITY;
        }

        for (int kc0 = 0; kc0 < kend; kc0 += kKeyTile) {
            __syncthreads();  // previous key tile fully consumed
            for (int e = tid; e < kKeyTile * d4; e += kThreads) {
                const int key = e / d4, t = (e - key * d4) * 4;
                const int j = kc0 + key;
                float v[4] = {0.f, 0.f, 0.f, 0.f};
                if (j < kend) Elem<T>::load4(K + ((size_t)h * nk + j) * d + t, v);
    #pragma unroll
                for (int u = 0; u < 4; ++u) Ks[(t + u) * kKeyStride + key] = v[u];
            }
            __syncthreads();

            float acc[kRowsPerWarp][2];
    #pragma unroll
            for (int r = 0; r < kRowsPerWarp; ++r) acc[r][0] = acc[r][1] = 0.f;
            const float4 *Q4 = reinterpret_cast<const float4 *>(Qs + warp * kRowsPerWarp * d);
            for (int t = 0; t < d; t += 4) {
                float4 qv[kRowsPerWarp];
    #pragma unroll
                for (int r = 0; r < kRowsPerWarp; ++r) qv[r] = Q4[r * d4 + (t >> 2)];
    #pragma unroll
                for (int tt = 0; tt < 4; ++tt) {
                    const float k0 = Ks[(t + tt) * kKeyStride + lane];
                    const float k1 = Ks[(t + tt) * kKeyStride + lane + 32];
    #pragma unroll
                    for (int r = 0; r < kRowsPerWarp; ++r) {
                        const float qq = tt == 0 ? qv[r].x : tt == 1 ? qv[r].y : tt == 2 ? qv[r].z : qv[r].w;
                        acc[r][0] = fmaf(qq, k0, acc[r][0]);
                        acc[r][1] = fmaf(qq, k1, acc[r][1]);
                    }
                }
            }

    #pragma unroll
            for (int r = 0; r < kRowsPerWarp; ++r) {
                float *bs = bs_all + (warp * kRowsPerWarp + r) * cap;
                int *bi = bi_all + (warp * kRowsPerWarp + r) * cap;
    #pragma unroll
                for (int u = 0; u < 2; ++u) {
                    const int j = kc0 + lane + 32 * u;
                    const float v = acc[r][u];
                    const bool p = j < my_kend[r] && v >= thr[r];
                    const unsigned msk = __ballot_sync(kFull, p);
                    if (msk) {
                        const int pos = cnt[r] + __popc(msk & lanemask_lt());
                        if (p) { bs[pos] = v; bi[pos] = j; }
                        cnt[r] += __popc(msk);
                        if (cnt[r] > cap - 32) {
                            __syncwarp();
                            warp_sort_best_first(bs, bi, cnt[r], cap);
                            cnt[r] = min(cnt[r], L.ksel);
                            thr[r] = cnt[r] == L.ksel ? bs[L.ksel - 1] : -INFINITY;
                        }
                    }
                }
            }
        }

        // finish every row of this warp: best-first order, ledger row write
    #pragma unroll 1
        for (int r = 0; r < kRowsPerWarp; ++r) {
            const int row = my_rows[r];
            if (row < 0) continue;
            float *bs = bs_all + (warp * kRowsPerWarp + r) * cap;
            int *bi = bi_all + (warp * kRowsPerWarp + r) * cap;
            __syncwarp();
            warp_sort_best_first(bs, bi, cnt[r], cap);
            const int n_valid = my_kend[r];
            const int nr = min(L.k, n_valid);
            const int nm = min(L.m, n_valid - nr);
            const size_t grow = (size_t)h * nq + row;
            int32_t *out = L.ids + grow * L.c;
            for (int e = lane; e < L.k + L.m; e += 32) {
                int id = -1;
                if (e < L.k) id = e < nr ? bi[e] : -1;
                else id = (e - L.k) < nm ? bi[nr + e - L.k] : -1;
                out[e] = id;
            }
            // mandatory global sentinels (g <= 32), after the random block
            const int g = L.g_sink + L.g_recent;
            int n_glob = 0;
            if (g > 0) {
                const int jg = lane < g ? global_cand(L, row, lane) : -1;
                const bool keep = lane < g && global_cand_listable(L, lane, jg, n_valid) &&
                                  !in_list(bi, nr + nm, jg);
                const unsigned km = __ballot_sync(kFull, keep);
                n_glob = __popc(km);
                int32_t *gout = out + L.k + L.m + L.r;
                if (keep) gout[__popc(km & lanemask_lt())] = jg;
                if (lane >= n_glob && lane < g) gout[lane] = -1;
            }
            draw_random_sentinels(L, L.bh_offset + h, row, layer, n_valid, bi, nr + nm, n_glob,
                                  rnd_all + warp * kRandMax, out + L.k + L.m);
            if (lane == 0) {
                L.alpha[grow] = bs[nr - 1];
                L.anchor_layer[grow] = layer;
                L.flags[grow] = L.rebuild_flag;
            }
        }
    }   // row tiles
}

}  // namespace

cudaError_t route_rows_prepare(const LedgerDev &L, int dtype) {
    // this kernel also rebuilds the retry lists of the tensor-core selection
    // path, so its attribute is set in every case
    const int smem = (int)smem_layout(L.d, select_capacity(L.ksel)).total;
    cudaError_t e;
    if (dtype == kBF16)
        e = cudaFuncSetAttribute(route_rows_kernel<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 smem);
    else
        e = cudaFuncSetAttribute(route_rows_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    // split fp32 problems: the selection kernel, with this kernel for the
    // rows whose kept scores overflow
    if (e == cudaSuccess && L.split) e = route_select_prepare();
    if (e == cudaSuccess && route_rows_tc_supported(L, dtype)) e = route_rows_tc_prepare();
    return e;
}

cudaError_t route_rows_prepare_all() {
    // the largest layout any config may launch: d = 256, k + m = 128
    const int smem = (int)smem_layout(256, select_capacity(128)).total;
    cudaError_t e = cudaFuncSetAttribute(route_rows_kernel<__nv_bfloat16>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(route_rows_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e == cudaSuccess) e = route_rows_tc_prepare();
    return e;
}

cudaError_t launch_route_rows(const LedgerDev &L, int dtype, const void *q, const void *k,
                              int layer, bool use_list, cudaStream_t s) {
    if (route_rows_tc_supported(L, dtype)) return launch_route_rows_tc(L, q, k, layer, use_list, s);
    if (dtype == kF32 && L.split && L.cand_keys && L.ksplit)
        return launch_route_rows_split(L, q, k, layer, use_list, s);
    return launch_route_rows_simt(L, dtype, q, k, layer, use_list, s);
}

cudaError_t launch_route_rows_simt(const LedgerDev &L, int dtype, const void *q, const void *k,
                                   int layer, bool use_list, cudaStream_t s, int max_tiles) {
    const int cap = select_capacity(L.ksel);
    const size_t smem = smem_layout(L.d, cap).total;
    int tiles = (L.nq + kTileRows - 1) / kTileRows;
    if (max_tiles > 0 && tiles > max_tiles) tiles = max_tiles;   // the CTAs stride over the rest
    dim3 grid(tiles, L.bh);
    if (dtype == kBF16)
        route_rows_kernel<__nv_bfloat16><<<grid, kThreads, smem, s>>>(
            L, static_cast<const __nv_bfloat16 *>(q), static_cast<const __nv_bfloat16 *>(k), layer,
            use_list ? 1 : 0, cap);
    else
        route_rows_kernel<float><<<grid, kThreads, smem, s>>>(
            L, static_cast<const float *>(q), static_cast<const float *>(k), layer,
            use_list ? 1 : 0, cap);
    return cudaGetLastError();
}

}  // namespace rr
