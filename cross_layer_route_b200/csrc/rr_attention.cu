// rr_attention.cu -- sparse attention over a route (declared in
// include/rr_attention.h).
//
// Method: "RouteRelay: Event-Triggered Cross-Layer Route Reuse for Efficient
// Dynamic Sparse Attention" (arXiv 2609.07306).  §2.1: the chunks a query
// row selects are expanded into token indices and attended with an online
// softmax; §2.2 Eq. 3: o_t = softmax(q_t K_T^T / sqrt(d)) V_T, T = the tokens
// of the route's chunks.
//
// One CTA = one query chunk of one head (CH tokens); warp w owns query rows
// 16w .. 16w+15 of the chunk.  The route's key chunks are visited one by one
// (the expansion: chunk j = tokens j*CH .. j*CH+CH-1, contiguous rows of K
// and V).  Each visit stages the chunk's K and V rows in shared memory with
// cp.async (two stages: the next chunk loads while this one is used), then
//   S = q K^T      bf16 mma.sync m16n8k16, q fragments held in registers,
//                  K fragments by ldmatrix from padded rows;
//   online softmax per query row in fp32 (running max m and sum l, the
//                  accumulators rescaled when m grows);
//   O += P V       P re-packed from the S accumulators into bf16 A fragments
//                  without leaving registers, V fragments by ldmatrix.trans.
// The last step divides O by l and writes fp32 rows.
//
// Shared-memory rows are padded by 8 elements (16 bytes): a row of DH bf16
// is 2*DH bytes, a multiple of 128, so unpadded rows would put all eight
// rows an ldmatrix reads in the same banks; with the pad, row r starts 4r
// banks further and each 8-row matrix read touches all 32 banks once.
#include <cuda_bf16.h>
#include <math.h>
#include <stdint.h>

#include "../../include/rr_attention.h"

namespace rr_attn {

constexpr int kMaxWidth = 1024;     // route entries read per query chunk
constexpr unsigned kFull = 0xffffffffu;

template <int DH, int CH>
struct Shape {
    static constexpr int kWarps = CH / 16;              // 16 query rows per warp
    static constexpr int kThreads = 32 * kWarps;
    // CTAs per SM the register budget is fitted to: three for chunks of up
    // to 64 tokens (at most 170 registers a thread, no spills); one for
    // chunks of 128 (eight warps, whose fragments would spill at three)
    static constexpr int kMinBlocks = kThreads >= 256 ? 1 : 3;
    static constexpr int kRow = DH + 8;                  // padded smem row (elements)
    static constexpr int kTile = CH * kRow;              // one staged K or V chunk (elements)
    static constexpr int kListBytes = kMaxWidth * 4 + 16;
    static constexpr int kSmem = kListBytes + 4 * kTile * 2;   // K and V, two stages each
    static constexpr int kSegs = CH * DH / 8;            // 16-byte pieces of one chunk
};

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(dst), "l"(src) : "memory");
}

__device__ __forceinline__ void cp_async_commit() {
    asm volatile("cp.async.commit_group;\n" ::: "memory");
}

// Waits until at most one committed group is still in flight.
__device__ __forceinline__ void cp_async_wait_one() {
    asm volatile("cp.async.wait_group 1;\n" ::: "memory");
}

__device__ __forceinline__ void ldmatrix_x4(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2,
                                            uint32_t &r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];\n"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}

__device__ __forceinline__ void ldmatrix_x4_trans(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2,
                                                  uint32_t &r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];\n"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}

// d += a (16x16 bf16, row) * b (16x8 bf16, col), fp32 accumulate.
__device__ __forceinline__ void mma_bf16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
        "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};\n"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Two floats as a bf16 pair, `lo` in the low half (round to nearest even).
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&v);
}

// Stages the CH rows of key chunk j (K and V) of head h into one stage.
template <int DH, int CH>
__device__ __forceinline__ void stage_chunk(const __nv_bfloat16 *__restrict__ kh,
                                            const __nv_bfloat16 *__restrict__ vh, int j,
                                            __nv_bfloat16 *sk, __nv_bfloat16 *sv) {
    using S = Shape<DH, CH>;
    const __nv_bfloat16 *kc = kh + (size_t)j * CH * DH;
    const __nv_bfloat16 *vc = vh + (size_t)j * CH * DH;
    for (int idx = threadIdx.x; idx < S::kSegs; idx += S::kThreads) {
        const int r = idx / (DH / 8);
        const int c = (idx % (DH / 8)) * 8;
        cp_async16(smem_u32(sk + r * S::kRow + c), kc + (size_t)r * DH + c);
        cp_async16(smem_u32(sv + r * S::kRow + c), vc + (size_t)r * DH + c);
    }
}

template <int DH, int CH>
__global__ void __launch_bounds__(Shape<DH, CH>::kThreads, Shape<DH, CH>::kMinBlocks)
sparse_attention_kernel(rr_attn_config cfg, const __nv_bfloat16 *__restrict__ q,
                        const __nv_bfloat16 *__restrict__ k, const __nv_bfloat16 *__restrict__ v,
                        const int32_t *__restrict__ route, float *__restrict__ out, float scale_log2) {
    using S = Shape<DH, CH>;
    extern __shared__ __align__(16) unsigned char smem[];
    int32_t *s_list = reinterpret_cast<int32_t *>(smem);
    int32_t *s_n = reinterpret_cast<int32_t *>(smem + kMaxWidth * 4);
    __nv_bfloat16 *s_k = reinterpret_cast<__nv_bfloat16 *>(smem + S::kListBytes);   // [2][CH][kRow]
    __nv_bfloat16 *s_v = s_k + 2 * S::kTile;                                          // [2][CH][kRow]

    const int nq_chunks = cfg.nq_tokens / CH;
    const int nk_chunks = cfg.nk_tokens / CH;
    const int h = blockIdx.x / nq_chunks;
    const int i = blockIdx.x % nq_chunks;
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int g = lane >> 2;    // fragment row (and B-fragment column)
    const int t = lane & 3;     // fragment column pair
    const bool causal = cfg.causal != 0;

    // The route's usable entries, in route order (warp 0, ordered ballot compaction).
    if (warp == 0) {
        const int32_t *rrow = route + ((size_t)h * nq_chunks + i) * (size_t)cfg.route_stride;
        int n = 0;
        for (int e0 = 0; e0 < cfg.width; e0 += 32) {
            const int e = e0 + lane;
            int j = -1;
            if (e < cfg.width) j = rrow[e];
            const bool ok = j >= 0 && j < nk_chunks && (!causal || j <= i);
            const unsigned b = __ballot_sync(kFull, ok);
            if (ok) s_list[n + __popc(b & ((1u << lane) - 1u))] = j;
            n += __popc(b);
        }
        if (lane == 0) *s_n = n;
    }
    __syncthreads();
    const int n_list = *s_n;

    const __nv_bfloat16 *kh = k + (size_t)h * cfg.nk_tokens * DH;
    const __nv_bfloat16 *vh = v + (size_t)h * cfg.nk_tokens * DH;
    if (n_list > 0) stage_chunk<DH, CH>(kh, vh, s_list[0], s_k, s_v);
    cp_async_commit();

    // q fragments of this warp's 16 rows (A operand, row-major 16 x DH).
    const int a0 = warp * 16 + g;          // query row within the chunk (and a0 + 8)
    const size_t qrow0 = (size_t)h * cfg.nq_tokens + (size_t)i * CH + a0;
    uint32_t qf[DH / 16][4];
    {
        const uint32_t *q0 = reinterpret_cast<const uint32_t *>(q + qrow0 * DH);
        const uint32_t *q1 = reinterpret_cast<const uint32_t *>(q + (qrow0 + 8) * DH);
#pragma unroll
        for (int kk = 0; kk < DH / 16; ++kk) {
            qf[kk][0] = q0[kk * 8 + t];
            qf[kk][1] = q1[kk * 8 + t];
            qf[kk][2] = q0[kk * 8 + 4 + t];
            qf[kk][3] = q1[kk * 8 + 4 + t];
        }
    }

    float o[DH / 8][4];
#pragma unroll
    for (int nd = 0; nd < DH / 8; ++nd) o[nd][0] = o[nd][1] = o[nd][2] = o[nd][3] = 0.f;
    float m0 = -INFINITY, m1 = -INFINITY;   // running max (log2 units) of rows a0, a0 + 8
    float l0 = 0.f, l1 = 0.f;               // this lane's part of the running sums

    // ldmatrix lane roles: lane supplies row (lane & 7) of matrix (lane >> 3).
    const int lm_row = lane & 7;
    const int lm_mat = lane >> 3;

    for (int e = 0; e < n_list; ++e) {
        const int st = e & 1;
        if (e + 1 < n_list)
            stage_chunk<DH, CH>(kh, vh, s_list[e + 1], s_k + (st ^ 1) * S::kTile, s_v + (st ^ 1) * S::kTile);
        cp_async_commit();
        cp_async_wait_one();
        __syncthreads();

        const __nv_bfloat16 *sk = s_k + st * S::kTile;
        const __nv_bfloat16 *sv = s_v + st * S::kTile;
        const bool diag = causal && s_list[e] == i;

        // S = q K^T for this warp's 16 rows x CH keys.
        float s[CH / 8][4];
#pragma unroll
        for (int n = 0; n < CH / 8; ++n) s[n][0] = s[n][1] = s[n][2] = s[n][3] = 0.f;
#pragma unroll
        for (int kk = 0; kk < DH / 16; ++kk) {
#pragma unroll
            for (int np = 0; np < CH / 16; ++np) {
                // matrices: keys 16np + {0, 0, 8, 8} + row, dims 16kk + {0, 8, 0, 8}
                const int key = np * 16 + lm_row + ((lm_mat >> 1) << 3);
                const int dim = kk * 16 + ((lm_mat & 1) << 3);
                uint32_t b0, b1, b2, b3;
                ldmatrix_x4(smem_u32(sk + key * S::kRow + dim), b0, b1, b2, b3);
                mma_bf16(s[2 * np], qf[kk], b0, b1);
                mma_bf16(s[2 * np + 1], qf[kk], b2, b3);
            }
        }

        // Online softmax (log2 domain).  Column of s[n][c]: 8n + 2t + (c & 1);
        // row: a0 + 8 * (c >> 1).  On the causal diagonal chunk key b is
        // visible to query a iff b <= a (token s <= t with equal chunk bases).
        float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
        for (int n = 0; n < CH / 8; ++n) {
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                float x = s[n][c] * scale_log2;
                if (diag) {
                    const int kb = n * 8 + 2 * t + (c & 1);
                    const int qa = a0 + ((c >> 1) << 3);
                    if (kb > qa) x = -INFINITY;
                }
                s[n][c] = x;
            }
            mx0 = fmaxf(mx0, fmaxf(s[n][0], s[n][1]));
            mx1 = fmaxf(mx1, fmaxf(s[n][2], s[n][3]));
        }
        mx0 = fmaxf(mx0, __shfl_xor_sync(kFull, mx0, 1));
        mx0 = fmaxf(mx0, __shfl_xor_sync(kFull, mx0, 2));
        mx1 = fmaxf(mx1, __shfl_xor_sync(kFull, mx1, 1));
        mx1 = fmaxf(mx1, __shfl_xor_sync(kFull, mx1, 2));
        const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);
        // a row with no visible key so far keeps m = -inf; use 0 as its base
        const float base0 = mn0 == -INFINITY ? 0.f : mn0;
        const float base1 = mn1 == -INFINITY ? 0.f : mn1;
        const float corr0 = exp2f(m0 - base0), corr1 = exp2f(m1 - base1);
        m0 = mn0;
        m1 = mn1;
        float ls0 = 0.f, ls1 = 0.f;
#pragma unroll
        for (int n = 0; n < CH / 8; ++n) {
            s[n][0] = exp2f(s[n][0] - base0);
            s[n][1] = exp2f(s[n][1] - base0);
            s[n][2] = exp2f(s[n][2] - base1);
            s[n][3] = exp2f(s[n][3] - base1);
            ls0 += s[n][0] + s[n][1];
            ls1 += s[n][2] + s[n][3];
        }
        l0 = l0 * corr0 + ls0;
        l1 = l1 * corr1 + ls1;
#pragma unroll
        for (int nd = 0; nd < DH / 8; ++nd) {
            o[nd][0] *= corr0;
            o[nd][1] *= corr0;
            o[nd][2] *= corr1;
            o[nd][3] *= corr1;
        }

        // O += P V: key step kk covers S columns 16kk .. 16kk+15 (tiles 2kk, 2kk+1).
#pragma unroll
        for (int kk = 0; kk < CH / 16; ++kk) {
            const uint32_t pa[4] = {pack_bf16(s[2 * kk][0], s[2 * kk][1]), pack_bf16(s[2 * kk][2], s[2 * kk][3]),
                                    pack_bf16(s[2 * kk + 1][0], s[2 * kk + 1][1]),
                                    pack_bf16(s[2 * kk + 1][2], s[2 * kk + 1][3])};
#pragma unroll
            for (int dp = 0; dp < DH / 16; ++dp) {
                // matrices: keys 16kk + {0, 8, 0, 8} + row, dims 16dp + {0, 0, 8, 8}
                const int key = kk * 16 + lm_row + ((lm_mat & 1) << 3);
                const int dim = dp * 16 + ((lm_mat >> 1) << 3);
                uint32_t b0, b1, b2, b3;
                ldmatrix_x4_trans(smem_u32(sv + key * S::kRow + dim), b0, b1, b2, b3);
                mma_bf16(o[2 * dp], pa, b0, b1);
                mma_bf16(o[2 * dp + 1], pa, b2, b3);
            }
        }
        __syncthreads();   // every warp is done with this stage before it is refilled
    }

    // Normalise: the row sums are spread over the four lanes of a quad.
    l0 += __shfl_xor_sync(kFull, l0, 1);
    l0 += __shfl_xor_sync(kFull, l0, 2);
    l1 += __shfl_xor_sync(kFull, l1, 1);
    l1 += __shfl_xor_sync(kFull, l1, 2);
    const float inv0 = l0 > 0.f ? 1.f / l0 : 0.f;
    const float inv1 = l1 > 0.f ? 1.f / l1 : 0.f;
    float *o0 = out + qrow0 * DH;
    float *o1 = out + (qrow0 + 8) * DH;
#pragma unroll
    for (int nd = 0; nd < DH / 8; ++nd) {
        *reinterpret_cast<float2 *>(o0 + nd * 8 + 2 * t) = make_float2(o[nd][0] * inv0, o[nd][1] * inv0);
        *reinterpret_cast<float2 *>(o1 + nd * 8 + 2 * t) = make_float2(o[nd][2] * inv1, o[nd][3] * inv1);
    }
}

template <int DH, int CH>
cudaError_t launch(const rr_attn_config &cfg, const void *q, const void *k, const void *v,
                   const int32_t *route, float *out, float scale, cudaStream_t s) {
    using S = Shape<DH, CH>;
    auto kern = sparse_attention_kernel<DH, CH>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, S::kSmem);
    if (e != cudaSuccess) return e;
    const unsigned blocks = (unsigned)((long long)cfg.bh * (cfg.nq_tokens / CH));
    const float scale_log2 = scale * 1.4426950408889634f;   // softmax in base 2: e^x = 2^(x log2 e)
    kern<<<blocks, S::kThreads, S::kSmem, s>>>(cfg, static_cast<const __nv_bfloat16 *>(q),
                                               static_cast<const __nv_bfloat16 *>(k),
                                               static_cast<const __nv_bfloat16 *>(v), route, out, scale_log2);
    return cudaGetLastError();
}

template <int DH>
cudaError_t launch_dh(const rr_attn_config &c, const void *q, const void *k, const void *v,
                      const int32_t *route, float *out, float scale, cudaStream_t s) {
    switch (c.chunk) {
        case 16: return launch<DH, 16>(c, q, k, v, route, out, scale, s);
        case 32: return launch<DH, 32>(c, q, k, v, route, out, scale, s);
        case 64: return launch<DH, 64>(c, q, k, v, route, out, scale, s);
        case 128: return launch<DH, 128>(c, q, k, v, route, out, scale, s);
    }
    return cudaErrorInvalidValue;
}

bool aligned(const void *p, uintptr_t a) { return ((uintptr_t)p & (a - 1)) == 0; }

bool config_ok(const rr_attn_config *c) {
    if (!c) return false;
    if (c->bh < 0 || c->nq_tokens < 0 || c->nk_tokens < 0) return false;
    if (c->dh != 64 && c->dh != 128) return false;
    if (c->chunk != 16 && c->chunk != 32 && c->chunk != 64 && c->chunk != 128) return false;
    if (c->nq_tokens % c->chunk != 0 || c->nk_tokens % c->chunk != 0) return false;
    if (c->width < 0 || c->width > kMaxWidth) return false;
    if (c->route_stride < (c->width > 1 ? c->width : 1)) return false;
    if (!(c->scale >= 0.f) || !isfinite(c->scale)) return false;
    if ((long long)c->bh * (c->nq_tokens / c->chunk) > 0x7fffffffLL) return false;
    return true;
}

}  // namespace rr_attn

extern "C" rr_status rr_sparse_attention(const rr_attn_config *cfg, const void *d_q, const void *d_k,
                                         const void *d_v, const int32_t *d_route, float *d_out,
                                         void *stream) {
    using namespace rr_attn;
    if (!config_ok(cfg)) return RR_EINVAL;
    if (cfg->bh == 0 || cfg->nq_tokens == 0) return RR_OK;
    if (!d_q || !d_out || !aligned(d_q, 16) || !aligned(d_out, 16)) return RR_EINVAL;
    if (cfg->width > 0 && (!d_route || !aligned(d_route, 4))) return RR_EINVAL;
    if (cfg->nk_tokens > 0 && (!d_k || !d_v || !aligned(d_k, 16) || !aligned(d_v, 16))) return RR_EINVAL;
    const float scale = cfg->scale > 0.f ? cfg->scale : 1.0f / sqrtf((float)cfg->dh);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const cudaError_t e = cfg->dh == 64 ? launch_dh<64>(*cfg, d_q, d_k, d_v, d_route, d_out, scale, s)
                                        : launch_dh<128>(*cfg, d_q, d_k, d_v, d_route, d_out, scale, s);
    return e == cudaSuccess ? RR_OK : RR_ECUDA;
}
