// simt_kernels.cu -- CUDA-core kernels of the DSA path:
//   * fold of W_index into the indexer query (+ e4m3 requantisation)
//   * fp32 indexer scores (tiny fp32 configuration)
//   * FP8 indexer scan for short query sets (decode), HBM-bound
//   * exact per-row radix top-k over scores held in memory
//   * exact fp32 sparse attention (tiny fp32 configuration)
//
// Method: "DeepSeek-V3.2与稀疏注意力技术革新", §2.2 (indexer), §2.3 (top-k
// selection, attention on the selected subset), §3.1 (MQA: heads share KV).
#include <cuda_fp8.h>

#include "dsa_device.cuh"
#include "dsa_kernels.h"

namespace dsa {

// ---------------------------------------------------------------------------
// a1: fold.  u_j = sum_i q_i W[i][j], an fp32 FMA chain in i = 0..127 for
// every output.  A CTA of FOLD_WARPS warps loads W once (fp32, 64 KB of
// shared memory) and folds groups of FOLD_WARPS * RPW rows: warp w takes RPW
// consecutive rows, lane l the columns 4l..4l+3 of each, so every step i is
// one 16-byte read of W[i][4l..4l+3], RPW/4 broadcast 16-byte reads of the
// rows' q_i (stored transposed) and 4 * RPW FMAs.  With many rows the grid is
// two CTAs per SM, each looping over row groups.
// E4M3: s_u = amax/448 (IEEE division), codes = e4m3_rn_satfinite(u_j / s_u),
// s_row = s_q * s_u.  The row's amax is a warp reduction; its codes are one
// 128-byte store.  Short query sets (decode) use fold_cols_kernel instead:
// thread j keeps column j of W in registers, one CTA per few rows, so the
// CTAs cover the GPU without each loading all of W into shared memory.
// ---------------------------------------------------------------------------
constexpr int FOLD_WARPS = 8;
constexpr int FOLD_COL_ROWS = 32;  // fold_cols_kernel: rows per CTA at most

__device__ __forceinline__ float e4m3_to_f32(uint8_t c) {
    __half_raw h = __nv_cvt_fp8_to_halfraw((__nv_fp8_storage_t)c, __NV_E4M3);
    return __half2float(__half(h));
}

template <int RPW>
constexpr uint32_t fold_smem_bytes() {
    return 128 * 128 * 4 + FOLD_WARPS * 128 * (RPW < 4 ? 4 : RPW) * 4;  // W, then per warp q^T [128][max(RPW,4)]
}

template <int RPW>
__global__ void __launch_bounds__(FOLD_WARPS * 32) fold_kernel(FoldArgs a) {
    constexpr int QW = RPW < 4 ? 4 : RPW;  // row slots of the transposed q (16-byte reads)
    extern __shared__ __align__(16) float fold_sm[];
    float* ws = fold_sm;                                            // [128][128]
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    float* qt = fold_sm + 128 * 128 + warp * 128 * QW;              // this warp's [128][QW]
    if (a.w_dtype == DSA_F32) {
        for (int e = threadIdx.x; e < 128 * 32; e += FOLD_WARPS * 32)
            ((float4*)ws)[e] = __ldg((const float4*)a.W + e);
    } else {
        for (int e = threadIdx.x; e < 128 * 16; e += FOLD_WARPS * 32) {
            const uint4 v = __ldg((const uint4*)a.W + e);  // 8 bf16
            const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
            float4 lo, hi;
            lo.x = __uint_as_float(w4[0] << 16), lo.y = __uint_as_float(w4[0] & 0xFFFF0000u);
            lo.z = __uint_as_float(w4[1] << 16), lo.w = __uint_as_float(w4[1] & 0xFFFF0000u);
            hi.x = __uint_as_float(w4[2] << 16), hi.y = __uint_as_float(w4[2] & 0xFFFF0000u);
            hi.z = __uint_as_float(w4[3] << 16), hi.w = __uint_as_float(w4[3] & 0xFFFF0000u);
            ((float4*)ws)[2 * e] = lo;
            ((float4*)ws)[2 * e + 1] = hi;
        }
    }
    __syncthreads();
    const int64_t groups = (a.T + FOLD_WARPS * RPW - 1) / (FOLD_WARPS * RPW);
    for (int64_t gi = blockIdx.x; gi < groups; gi += gridDim.x) {
        const int64_t r0 = (gi * FOLD_WARPS + warp) * RPW;
        if (r0 >= a.T) continue;
        __syncwarp();
        // this warp's rows, transposed: qt[i][rr] = q[r0 + rr][i] (0 past T)
#pragma unroll
        for (int rr = 0; rr < QW; ++rr) {
            const int64_t r = r0 + rr;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const int i = c * 32 + lane;
                float v = 0.f;
                if (rr < RPW && r < a.T)
                    v = a.idx_dtype == DSA_F32 ? __ldg((const float*)a.q_idx + r * 128 + i)
                                               : e4m3_to_f32(((const uint8_t*)a.q_idx)[r * 128 + i]);
                qt[i * QW + rr] = v;
            }
        }
        __syncwarp();
        float acc[RPW][4];
#pragma unroll
        for (int rr = 0; rr < RPW; ++rr)
#pragma unroll
            for (int c = 0; c < 4; ++c) acc[rr][c] = 0.f;
#pragma unroll 4
        for (int i = 0; i < 128; ++i) {
            const float4 w4 = *(const float4*)(ws + i * 128 + 4 * lane);
            float qv[QW];
#pragma unroll
            for (int rr = 0; rr < QW; rr += 4) {
                const float4 q4 = *(const float4*)(qt + i * QW + rr);
                qv[rr] = q4.x, qv[rr + 1] = q4.y, qv[rr + 2] = q4.z, qv[rr + 3] = q4.w;
            }
#pragma unroll
            for (int rr = 0; rr < RPW; ++rr) {
                acc[rr][0] = fmaf(qv[rr], w4.x, acc[rr][0]);
                acc[rr][1] = fmaf(qv[rr], w4.y, acc[rr][1]);
                acc[rr][2] = fmaf(qv[rr], w4.z, acc[rr][2]);
                acc[rr][3] = fmaf(qv[rr], w4.w, acc[rr][3]);
            }
        }
#pragma unroll
        for (int rr = 0; rr < RPW; ++rr) {
            const int64_t r = r0 + rr;
            if (r >= a.T) break;
            if (a.idx_dtype == DSA_F32) {
                ((float4*)a.u_out)[r * 32 + lane] = make_float4(acc[rr][0], acc[rr][1], acc[rr][2], acc[rr][3]);
                if (lane == 0) a.s_row_out[r] = 1.0f;
                continue;
            }
            float m = fmaxf(fmaxf(fabsf(acc[rr][0]), fabsf(acc[rr][1])), fmaxf(fabsf(acc[rr][2]), fabsf(acc[rr][3])));
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
            const float s_u = m == 0.f ? 1.0f : __fdiv_rn(m, 448.0f);
            uint32_t codes = 0;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const float y = m == 0.f ? 0.f : __fdiv_rn(acc[rr][c], s_u);
                codes |= (uint32_t)(uint8_t)__nv_cvt_float_to_fp8(y, __NV_SATFINITE, __NV_E4M3) << (8 * c);
            }
            ((uint32_t*)a.u_out)[r * 32 + lane] = codes;
            if (lane == 0) a.s_row_out[r] = __fmul_rn(__ldg(a.q_scale + r), s_u);
        }
    }
}

__global__ void __launch_bounds__(128) fold_cols_kernel(int64_t T, int idx_dtype, const void* __restrict__ q_idx,
                                                   const float* __restrict__ q_scale, int w_dtype,
                                                   const void* __restrict__ W, void* __restrict__ u_out,
                                                   float* __restrict__ s_row_out, int rows_per_cta) {
    __shared__ float qs[128];
    __shared__ float red[4];
    const int j = threadIdx.x;
    float w[128];
#pragma unroll
    for (int i = 0; i < 128; ++i) {
        if (w_dtype == DSA_F32)
            w[i] = __ldg((const float*)W + i * 128 + j);
        else
            w[i] = __bfloat162float(((const __nv_bfloat16*)W)[i * 128 + j]);
    }
    const int64_t r0 = (int64_t)blockIdx.x * rows_per_cta;
    for (int rr = 0; rr < rows_per_cta; ++rr) {
        const int64_t r = r0 + rr;
        if (r >= T) break;
        __syncthreads();
        if (idx_dtype == DSA_F32)
            qs[j] = __ldg((const float*)q_idx + r * 128 + j);
        else
            qs[j] = e4m3_to_f32(((const uint8_t*)q_idx)[r * 128 + j]);
        __syncthreads();
        float acc = 0.f;
#pragma unroll
        for (int i = 0; i < 128; ++i) acc = fmaf(qs[i], w[i], acc);
        if (idx_dtype == DSA_F32) {
            ((float*)u_out)[r * 128 + j] = acc;
            if (j == 0) s_row_out[r] = 1.0f;
            continue;
        }
        float a = fabsf(acc);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
        if ((j & 31) == 0) red[j >> 5] = a;
        __syncthreads();
        const float amax = fmaxf(fmaxf(red[0], red[1]), fmaxf(red[2], red[3]));
        const float s_u = amax == 0.f ? 1.0f : __fdiv_rn(amax, 448.0f);
        const float y = amax == 0.f ? 0.f : __fdiv_rn(acc, s_u);
        ((uint8_t*)u_out)[r * 128 + j] = (uint8_t)__nv_cvt_float_to_fp8(y, __NV_SATFINITE, __NV_E4M3);
        if (j == 0) s_row_out[r] = __fmul_rn(__ldg(q_scale + r), s_u);
    }
}

template <int RPW>
static void launch_fold_t(const FoldArgs& a, int64_t max_ctas, cudaStream_t s) {
    constexpr uint32_t smem = fold_smem_bytes<RPW>();
    cudaFuncSetAttribute(fold_kernel<RPW>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    int64_t grid = (a.T + FOLD_WARPS * RPW - 1) / (FOLD_WARPS * RPW);
    if (grid > max_ctas) grid = max_ctas;
    fold_kernel<RPW><<<(unsigned)grid, FOLD_WARPS * 32, smem, s>>>(a);
}

void launch_fold(const FoldArgs& a, cudaStream_t s) {
    if (a.T <= 0) return;
    // many rows: 8 (or 2) per warp, at most two persistent CTAs per SM of a
    // B200 (W is loaded once per CTA)
    if (a.T >= 148 * FOLD_WARPS * 8) {
        launch_fold_t<8>(a, 2 * 148, s);
        return;
    }
    if (a.T >= 1024) {
        launch_fold_t<2>(a, 2 * 148, s);
        return;
    }
    // few rows (decode): about four CTAs per SM before a CTA takes more than one row
    int64_t rows = (a.T + 148 * 4 - 1) / (148 * 4);
    if (rows > FOLD_COL_ROWS) rows = FOLD_COL_ROWS;
    const int64_t grid = (a.T + rows - 1) / rows;
    fold_cols_kernel<<<(unsigned)grid, 128, 0, s>>>(a.T, a.idx_dtype, a.q_idx, a.q_scale, a.w_dtype, a.W, a.u_out,
                                                    a.s_row_out, (int)rows);
}

// ---------------------------------------------------------------------------
// Fill a [rows, ld] float array with -inf.
// ---------------------------------------------------------------------------
__global__ void fill_neg_inf_kernel(float* p, int64_t rows, int64_t ld) {
    const int64_t n = rows * ld;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x)
        p[i] = -INFINITY;
}

void launch_fill_neg_inf(float* p, int64_t rows, int64_t ld, cudaStream_t s) {
    const int64_t n = rows * ld;
    if (n <= 0) return;
    int64_t blocks = (n + 255) / 256;
    if (blocks > 148 * 16) blocks = 148 * 16;
    fill_neg_inf_kernel<<<(unsigned)blocks, 256, 0, s>>>(p, rows, ld);
}

// ReLU applied on the bit pattern: every x <= 0 (and -0.0) becomes +0.0;
// +inf/NaN are clamped to +inf so that the key stays a finite-order value.
__device__ __forceinline__ float relu_key(float x) {
    int b = __float_as_int(x);
    b = max(b, 0);
    b = min(b, 0x7F800000);
    return __int_as_float(b);
}

// ---------------------------------------------------------------------------
// a2, fp32: scores[r, s] = ReLU(u_t . k_s) for s <= pos; grid (key chunks,
// rows), one thread per key.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(128) scores_f32_kernel(SeqView sv, const float* __restrict__ u,
                                                         const float* __restrict__ k_idx, int64_t row_begin,
                                                         float* __restrict__ scores, int64_t ld, StatusHdr* st) {
    __shared__ float us[128];
    const int64_t r = blockIdx.y;
    const int64_t t = row_begin + r;
    const RowInfo ri = row_info(sv, t);
    if (!ri.ok) {
        if (threadIdx.x == 0) report(st, DSA_ERR_INDEX, t);
        return;
    }
    us[threadIdx.x] = u[t * 128 + threadIdx.x];
    __syncthreads();
    const int64_t s = (int64_t)blockIdx.x * 128 + threadIdx.x;
    if (s > ri.pos) return;
    const float* kr = k_idx + (ri.key_base + s) * 128;
    float acc = 0.f;
#pragma unroll 8
    for (int i = 0; i < 128; ++i) acc = fmaf(us[i], __ldg(kr + i), acc);
    scores[r * ld + s] = relu_key(acc);
}

// ---------------------------------------------------------------------------
// a2, FP8 scan for short query sets: 8 lanes per key (16 codes each), fp32
// FMA of the exact e4m3 products, xor-shuffle reduction; score =
// ReLU((dot * s_k) * s_row).  HBM-bound: 132 bytes read per key.
// ---------------------------------------------------------------------------
#ifndef DSA_SCAN_KEYS
#define DSA_SCAN_KEYS 1024
#endif
constexpr int SCAN_KEYS = DSA_SCAN_KEYS;

// 16 e4m3 codes (one 16-byte slice of a key) dotted with 16 fp32 query
// values: the codes are decoded in pairs by the hardware conversion to f16
// (exact for every e4m3 value), then widened to fp32.
__device__ __forceinline__ float dot16_e4m3(const float (&uq)[16], uint4 v) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    float acc = 0.f;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
#pragma unroll
        for (int p = 0; p < 2; ++p) {
            const __half2_raw h2 = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(w[q] >> (16 * p)), __NV_E4M3);
            const float2 f = __half22float2(__half2(h2));
            acc = fmaf(uq[4 * q + 2 * p], f.x, acc);
            acc = fmaf(uq[4 * q + 2 * p + 1], f.y, acc);
        }
    }
    return acc;
}

#ifndef DSA_SCAN_UNROLL
#define DSA_SCAN_UNROLL 4
#endif
constexpr int SCAN_UNROLL = DSA_SCAN_UNROLL;  // keys per lane group in flight

__global__ void __launch_bounds__(256) scan_fp8_kernel(SeqView sv, const uint8_t* __restrict__ u8,
                                                       const float* __restrict__ s_row, const uint8_t* __restrict__ k8,
                                                       const float* __restrict__ k_scale, int64_t row_begin,
                                                       float* __restrict__ scores, int64_t ld, StatusHdr* st) {
    const int64_t r = blockIdx.y;
    const int64_t t = row_begin + r;
    const RowInfo ri = row_info(sv, t);
    if (!ri.ok) {
        if (threadIdx.x == 0) report(st, DSA_ERR_INDEX, t);
        return;
    }
    const int sub = threadIdx.x & 7;  // which 16-byte slice of the key
    float uq[16];
    {
        const uint4 v = *(const uint4*)(u8 + t * 128 + sub * 16);
        const uint8_t* b = (const uint8_t*)&v;
#pragma unroll
        for (int i = 0; i < 16; ++i) uq[i] = e4m3_to_f32(b[i]);
    }
    const float srow = s_row[t];
    const int64_t s_begin = (int64_t)blockIdx.x * SCAN_KEYS;
    const int64_t s_end = min(s_begin + SCAN_KEYS, ri.pos + 1);
    for (int64_t s0 = s_begin; s0 < s_end; s0 += 32 * SCAN_UNROLL) {
        uint4 kv[SCAN_UNROLL];
        float ks[SCAN_UNROLL];
#pragma unroll
        for (int u = 0; u < SCAN_UNROLL; ++u) {  // every load of the group first
            const int64_t s = s0 + u * 32 + (threadIdx.x >> 3);
            kv[u] = make_uint4(0u, 0u, 0u, 0u);
            ks[u] = 0.f;
            if (s < s_end) {
                kv[u] = __ldg((const uint4*)(k8 + (ri.key_base + s) * 128 + sub * 16));
                if (sub == 0) ks[u] = __ldg(k_scale + ri.key_base + s);
            }
        }
#pragma unroll
        for (int u = 0; u < SCAN_UNROLL; ++u) {
            const int64_t s = s0 + u * 32 + (threadIdx.x >> 3);
            float acc = dot16_e4m3(uq, kv[u]);
            acc += __shfl_xor_sync(0xffffffffu, acc, 1);
            acc += __shfl_xor_sync(0xffffffffu, acc, 2);
            acc += __shfl_xor_sync(0xffffffffu, acc, 4);
            if (sub == 0 && s < s_end) scores[r * ld + s] = relu_key(__fmul_rn(__fmul_rn(acc, ks[u]), srow));
        }
    }
}

void launch_scores_simt(const ScoresSimtArgs& a, cudaStream_t s) {
    if (a.row_count <= 0) return;
    if (a.fill) launch_fill_neg_inf(a.scores, a.row_count, a.ld, s);
    if (a.idx_dtype == DSA_F32) {
        dim3 grid((unsigned)((a.max_seqlen_k + 127) / 128), (unsigned)a.row_count);
        scores_f32_kernel<<<grid, 128, 0, s>>>(a.sv, (const float*)a.u, (const float*)a.k_idx, a.row_begin, a.scores,
                                                a.ld, a.st);
    } else {
        dim3 grid((unsigned)((a.max_seqlen_k + SCAN_KEYS - 1) / SCAN_KEYS), (unsigned)a.row_count);
        scan_fp8_kernel<<<grid, 256, 0, s>>>(a.sv, (const uint8_t*)a.u, a.s_row, (const uint8_t*)a.k_idx, a.k_scale,
                                             a.row_begin, a.scores, a.ld, a.st);
    }
}

// ---------------------------------------------------------------------------
// a3: exact top-k of one row per CTA by most-significant-digit radix select
// (4 digits of 8 bits over an order-preserving 32-bit key), then an emission
// pass in ascending index order.  Ties at the threshold go to the lowest
// indices.  Key order: NaN < -inf < ... < -0.0 == +0.0 < ... < +inf.  The
// emission gives each warp a contiguous index range: the warps count their
// keys above and in the bucket, one scan over the 32 warps gives each its
// output offset, and each warp places its keys with ballots.
// ---------------------------------------------------------------------------
constexpr int TOPK_NT = 1024;
constexpr int TOPK_WARPS = TOPK_NT / 32;

__device__ __forceinline__ uint32_t order_key(float x) {
    uint32_t u = __float_as_uint(x);
    if ((u & 0x7FFFFFFFu) > 0x7F800000u) return 0u;  // NaN: below everything
    if (u == 0x80000000u) u = 0u;                     // -0.0 == +0.0
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

constexpr int TOPK_BATCH = 8;  // 32-key rows of a warp's range loaded before any is used

// Index range of each warp in the emission: contiguous, a multiple of 32.
__device__ __forceinline__ int64_t topk_span(int64_t n) {
    return (((n + TOPK_WARPS - 1) / TOPK_WARPS) + 31) & ~(int64_t)31;
}

// The emission's placement: with wcnt[w] = (keys above the bucket, keys in
// the bucket) of warp w's index range [w*span, (w+1)*span), write the keys
// above the bucket and the first `need` keys of the bucket in ascending index
// order, then -1 up to `width`.  The bucket is the keys whose order key under
// `mask` equals `prefix`.  Called by all TOPK_NT threads.
__device__ void place_keys(const float* __restrict__ row, int64_t n, int64_t span, uint32_t prefix, uint32_t mask,
                           uint32_t need, int k, int width, uint32_t (*wcnt)[2], int32_t* __restrict__ out,
                           StatusHdr* st, int64_t t) {
    __shared__ uint32_t above_all;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int64_t w0 = (int64_t)warp * span, w1 = min(n, w0 + span);
    if (warp == 0) {  // exclusive prefixes over the warps, in index order
        const uint32_t a = wcnt[lane][0], e = wcnt[lane][1];
        uint32_t ia = a, ie = e;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t va = __shfl_up_sync(0xffffffffu, ia, o), ve = __shfl_up_sync(0xffffffffu, ie, o);
            if (lane >= o) ia += va, ie += ve;
        }
        wcnt[lane][0] = ia - a;
        wcnt[lane][1] = ie - e;
        if (lane == 31) above_all = ia;  // keys above the bucket in all
    }
    __syncthreads();
    uint32_t eq_before = wcnt[warp][1];
    uint32_t pos = wcnt[warp][0] + min(eq_before, need);
    const uint32_t lt = (1u << lane) - 1u;
    for (int64_t s0 = w0; s0 < w1; s0 += 32 * TOPK_BATCH) {
        uint32_t mk[TOPK_BATCH];  // the batch's loads first
#pragma unroll
        for (int j = 0; j < TOPK_BATCH; ++j) {
            const int64_t s = s0 + 32 * j + lane;
            mk[j] = s < w1 ? (order_key(row[s]) & mask) : 0u;
        }
#pragma unroll
        for (int j = 0; j < TOPK_BATCH; ++j) {
            const int64_t s = s0 + 32 * j + lane;
            const bool ab = s < w1 && mk[j] > prefix, eq = s < w1 && mk[j] == prefix;
            const uint32_t eqm = __ballot_sync(0xffffffffu, eq);
            const bool take = ab || (eq && eq_before + (uint32_t)__popc(eqm & lt) < need);
            const uint32_t tk = __ballot_sync(0xffffffffu, take);
            if (take && pos + (uint32_t)__popc(tk & lt) < (uint32_t)k) out[pos + __popc(tk & lt)] = (int32_t)s;
            pos += (uint32_t)__popc(tk);
            eq_before += (uint32_t)__popc(eqm);
        }
    }
    const uint32_t total = above_all + need;
    for (int64_t s = total + threadIdx.x; s < width; s += TOPK_NT) out[s] = -1;
    if (threadIdx.x == 0 && total != (uint32_t)k) report(st, DSA_ERR_INDEX, -1000000 - t);
}

__global__ void __launch_bounds__(TOPK_NT) topk_rows_kernel(SeqView sv, const float* __restrict__ scores, int64_t ld,
                                                            int64_t row_begin, int width, const int32_t* __restrict__ k_rows,
                                                            int32_t* __restrict__ idx, int64_t ld_idx, StatusHdr* st) {
    __shared__ uint32_t hist[256];
    __shared__ uint32_t wcnt[TOPK_WARPS][2];  // per warp: keys above, keys equal (then their prefixes)
    __shared__ uint32_t sel_bin, sel_above;
    const int64_t r = blockIdx.x;
    const int64_t t = row_begin + r;
    const RowInfo ri = row_info(sv, t);
    int32_t* out = idx + r * ld_idx;
    if (!ri.ok) {
        if (threadIdx.x == 0) report(st, DSA_ERR_INDEX, t);
        return;
    }
    const int64_t n = ri.pos + 1;
    const float* row = scores + r * ld;
    // this row's k (dynamic k: clamped to [0, width]); the row is `width` wide
    const int k = k_rows ? min(max(__ldg(k_rows + t), 0), width) : width;
    if (n <= k || k == 0) {
        for (int64_t s = threadIdx.x; s < width; s += TOPK_NT) out[s] = (s < n && s < k) ? (int32_t)s : -1;
        return;
    }
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    uint32_t prefix = 0, mask = 0;
    uint32_t need = (uint32_t)k;
    for (int pass = 0; pass < 4; ++pass) {
        const int shift = 24 - 8 * pass;
        for (int i = threadIdx.x; i < 256; i += TOPK_NT) hist[i] = 0;
        __syncthreads();
        for (int64_t s0 = 0; s0 < n; s0 += (int64_t)TOPK_NT * 4) {
            uint32_t kk[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int64_t s = s0 + j * TOPK_NT + threadIdx.x;
                kk[j] = s < n ? order_key(row[s]) : 0u;
            }
#pragma unroll
            for (int j = 0; j < 4; ++j)
                if (s0 + j * TOPK_NT + threadIdx.x < n && (kk[j] & mask) == prefix)
                    atomicAdd(&hist[(kk[j] >> shift) & 255u], 1u);
        }
        __syncthreads();
        if (threadIdx.x < 32) {
            // lane l owns bins [8l, 8l+8); count above from the top
            const int lane = threadIdx.x;
            uint32_t c[8], sum = 0;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                c[i] = hist[lane * 8 + i];
                sum += c[i];
            }
            uint32_t above = 0;  // count in lanes > lane
            uint32_t inc = sum;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const uint32_t v = __shfl_down_sync(0xffffffffu, inc, o);
                if (lane + o < 32) inc += v;
            }
            above = inc - sum;
            // the lane where the running count (from the top) first reaches need
            const bool mine = above < need && above + sum >= need;
            if (mine) {
                uint32_t acc = above;
                for (int i = 7; i >= 0; --i) {
                    if (acc + c[i] >= need) {
                        sel_bin = (uint32_t)(lane * 8 + i);
                        sel_above = acc;
                        break;
                    }
                    acc += c[i];
                }
            }
        }
        __syncthreads();
        const uint32_t bin = sel_bin;
        prefix |= bin << shift;
        mask |= 0xFFu << shift;
        need -= sel_above;
        const uint32_t in_bin = hist[bin];
        __syncthreads();
        if (in_bin == need) break;
    }
    // ---- emission: warp w owns indices [w*span, (w+1)*span) ----
    const int64_t span = topk_span(n);
    const int64_t w0 = (int64_t)warp * span, w1 = min(n, w0 + span);
    uint32_t n_above = 0, n_eq = 0;
    for (int64_t s0 = w0; s0 < w1; s0 += 32 * TOPK_BATCH) {
        uint32_t mk[TOPK_BATCH];
#pragma unroll
        for (int j = 0; j < TOPK_BATCH; ++j) {
            const int64_t s = s0 + 32 * j + lane;
            mk[j] = s < w1 ? (order_key(row[s]) & mask) : 0u;
        }
#pragma unroll
        for (int j = 0; j < TOPK_BATCH; ++j) {
            const bool in = s0 + 32 * j + lane < w1;
            n_above += in && mk[j] > prefix;
            n_eq += in && mk[j] == prefix;
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        n_above += __shfl_xor_sync(0xffffffffu, n_above, o);
        n_eq += __shfl_xor_sync(0xffffffffu, n_eq, o);
    }
    if (lane == 0) {
        wcnt[warp][0] = n_above;
        wcnt[warp][1] = n_eq;
    }
    __syncthreads();
    place_keys(row, n, span, prefix, mask, need, k, width, wcnt, out, st, t);
}

// ---------------------------------------------------------------------------
// a3 for non-negative scores (the selection's own ReLU scores, +inf for NaN):
// exact top-k of one row, same result as topk_rows_kernel.  A row is split
// over a cluster of CPR CTAs (contiguous index ranges, 32 warps each), which
// merge their counts through distributed shared memory:
//   1. Each CTA histograms its range over 4096 bins of 1/16 binade (fp32
//      bits >> 19); zero scores, typically half of a ReLU row, go to 32
//      per-lane bins summed afterwards, so they cause no atomic conflicts.
//      Every CTA sums the cluster's histograms and finds the same bucket:
//      the bin of the k-th largest score.
//   2. While the bucket holds more than TOPK_CAND keys, radix passes over the
//      row refine it by the next digit (bits 18..11, 10..3, 2..0).
//   3. One pass counts each warp's keys above and in the bucket and lists the
//      bucket's keys in the CTA's shared memory.
//   4. Every CTA refines the bucket by the remaining digits over all the
//      cluster's lists, until it is one score value or is taken whole.
//   5. The CTAs exchange their counts and place their keys: those above the
//      bucket and the first `need` of the bucket, in ascending index order.
// Three passes over the row (L2-resident after the scan) in the usual case.
// ---------------------------------------------------------------------------
constexpr int TOPK_CAND = 2048;
constexpr int TH_BINS = 4096, TH_SHIFT = 19;

DSA_DEV uint32_t ld_cluster_u32(uint32_t addr) {
    uint32_t v;
    asm volatile("ld.shared::cluster.u32 %0, [%1];" : "=r"(v) : "r"(addr) : "memory");
    return v;
}
DSA_DEV uint4 ld_cluster_v4(uint32_t addr) {
    uint4 v;
    asm volatile("ld.shared::cluster.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "r"(addr)
                 : "memory");
    return v;
}
DSA_DEV void st_cluster_u32(uint32_t addr, uint32_t v) {
    asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}

// Radix digit `pass` below the 1/16-binade bin: bits 18..11, 10..3, 2..0.
__device__ __forceinline__ void th_digit(int pass, int& shift, uint32_t& dm) {
    shift = pass == 0 ? 11 : (pass == 1 ? 3 : 0);
    dm = pass < 2 ? 0xFFu : 0x7u;
}

// Warp 0: the bin of a 256-bin digit histogram holding the need-th largest
// key, the keys above it and its count.
__device__ __forceinline__ void th_pick(const uint32_t* h, uint32_t need, uint32_t& b_sel, uint32_t& b_above,
                                        uint32_t& b_count) {
    const int lane = threadIdx.x & 31;
    uint32_t cc[8], sm = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        cc[i] = h[lane * 8 + i];
        sm += cc[i];
    }
    uint32_t in2 = sm;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t v = __shfl_down_sync(0xffffffffu, in2, o);
        if (lane + o < 32) in2 += v;
    }
    const uint32_t ab = in2 - sm;
    if (ab < need && ab + sm >= need) {
        uint32_t acc = ab;
        bool found = false;
#pragma unroll
        for (int i = 7; i >= 0; --i) {
            if (!found && acc + cc[i] >= need) {
                b_sel = (uint32_t)(lane * 8 + i);
                b_above = acc;
                b_count = cc[i];
                found = true;
            }
            acc += cc[i];
        }
    }
}

template <int CPR>
__global__ void __cluster_dims__(CPR, 1, 1) __launch_bounds__(TOPK_NT, 2)
    topk_hist_kernel(SeqView sv, const float* __restrict__ scores, int64_t ld, int64_t row_begin, int width,
                     const int32_t* __restrict__ k_rows, int32_t* __restrict__ idx, int64_t ld_idx, StatusHdr* st) {
    __shared__ __align__(16) uint32_t hb[TH_BINS + 32];
    __shared__ uint32_t ckey[TOPK_CAND];
    __shared__ int32_t cidx[TOPK_CAND];
    __shared__ uint32_t hs[256], hsum[256];
    __shared__ uint32_t wtot[TOPK_WARPS];
    __shared__ uint32_t wcnt[TOPK_WARPS][2];
    __shared__ uint32_t ctot[CPR][2];
    __shared__ uint32_t b_sel, b_above, b_count, n_cand;
    const uint32_t crank = CPR > 1 ? cluster_ctarank() : 0u;
    const int64_t r = blockIdx.x / CPR;
    const int64_t t = row_begin + r;
    const RowInfo ri = row_info(sv, t);
    int32_t* out = idx + r * ld_idx;
    // every decision below is the same in all CTAs of the cluster (same row,
    // same merged counts), so the cluster leaves or syncs together
    if (!ri.ok) {
        if (threadIdx.x == 0 && crank == 0) report(st, DSA_ERR_INDEX, t);
        return;
    }
    const int n = (int)(ri.pos + 1);  // index rows are int32: a row has fewer than 2^31 keys
    const float* row = scores + r * ld;
    const int k = k_rows ? min(max(__ldg(k_rows + t), 0), width) : width;
    if (n <= k || k == 0) {
        if (crank == 0)
            for (int s = threadIdx.x; s < width; s += TOPK_NT) out[s] = (s < n && s < k) ? s : -1;
        return;
    }
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    constexpr int TB = CPR > 1 ? TOPK_BATCH : 4;  // keys per lane loaded ahead (registers: two CTAs per SM)
    uint32_t need = (uint32_t)k;
    // warp g = crank * 32 + warp of the cluster owns [g * span, (g + 1) * span)
    const int span = (((n + CPR * TOPK_WARPS - 1) / (CPR * TOPK_WARPS)) + 31) & ~31;
    const int c0 = min(n, (int)crank * TOPK_WARPS * span), c1 = min(n, c0 + TOPK_WARPS * span);
    auto leave = [&](int code) {  // reported once; no indices; the cluster leaves together
        if (threadIdx.x == 0 && crank == 0) report(st, DSA_ERR_INDEX, code - t);
        if (crank == 0)
            for (int s = threadIdx.x; s < width; s += TOPK_NT) out[s] = -1;
        if constexpr (CPR > 1) cluster_sync();
    };

    // ---- 1. histogram of this CTA's range; the cluster's bucket ----
    for (int i = threadIdx.x; i < TH_BINS + 32; i += TOPK_NT) hb[i] = 0;
    if (threadIdx.x == 0) b_sel = 0xFFFFFFFFu;
    __syncthreads();
    for (int s0 = c0; s0 < c1; s0 += TOPK_NT * 4) {
        uint32_t kk[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int s = s0 + j * TOPK_NT + (int)threadIdx.x;
            kk[j] = s < c1 ? min(__float_as_uint(row[s]) >> TH_SHIFT, (uint32_t)TH_BINS - 1) : 0u;
        }
#pragma unroll
        for (int j = 0; j < 4; ++j)
            if (s0 + j * TOPK_NT + (int)threadIdx.x < c1) atomicAdd(&hb[kk[j] ? kk[j] : TH_BINS + lane], 1u);
    }
    __syncthreads();
    if (warp == 0) {  // bin 0 = the per-lane zero bins
        uint32_t z = hb[TH_BINS + lane];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
        if (lane == 0) hb[0] = z;
    }
    __syncthreads();
    static_assert(TH_BINS == 4 * TOPK_NT, "four bins per thread");
    uint32_t c[4];
    if constexpr (CPR > 1) {
        cluster_sync();  // every CTA's histogram is complete
        c[0] = c[1] = c[2] = c[3] = 0;
        const uint32_t my = smem_u32(hb + 4 * threadIdx.x);
#pragma unroll
        for (int q = 0; q < CPR; ++q) {
            const uint4 v = ld_cluster_v4(mapa(my, (uint32_t)q));
            c[0] += v.x, c[1] += v.y, c[2] += v.z, c[3] += v.w;
        }
    } else {
        const uint4 v = *(const uint4*)(hb + 4 * threadIdx.x);
        c[0] = v.x, c[1] = v.y, c[2] = v.z, c[3] = v.w;
    }
    const uint32_t sum = c[0] + c[1] + c[2] + c[3];
    uint32_t inc = sum;  // bins of this lane and the lanes above it, in this warp
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t v = __shfl_down_sync(0xffffffffu, inc, o);
        if (lane + o < 32) inc += v;
    }
    if (lane == 0) wtot[warp] = inc;
    __syncthreads();
    uint32_t above = inc - sum;
    for (int w = warp + 1; w < TOPK_WARPS; ++w) above += wtot[w];
    if (above < need && above + sum >= need) {
        uint32_t acc = above;
        bool found = false;
#pragma unroll
        for (int i = 3; i >= 0; --i) {
            if (!found && acc + c[i] >= need) {
                b_sel = 4 * threadIdx.x + i;
                b_above = acc;
                b_count = c[i];
                found = true;
            }
            acc += c[i];
        }
    }
    __syncthreads();
    if (b_sel == 0xFFFFFFFFu) {  // cannot happen with n > k keys counted
        leave(-4000000);
        return;
    }
    // the bucket in order-key space (non-negative scores: key = bits | 2^31)
    uint32_t prefix = 0x80000000u | (b_sel << TH_SHIFT);
    uint32_t mask = 0xFFFFFFFFu << TH_SHIFT;
    need -= b_above;
    uint32_t cnt = b_count;

    // ---- 2. refine an oversized bucket by radix passes over the row ----
    int lvl = 0;
    for (; lvl < 3 && cnt > (uint32_t)TOPK_CAND && cnt != need; ++lvl) {
        int shift;
        uint32_t dm;
        th_digit(lvl, shift, dm);
        for (int i = threadIdx.x; i < 256; i += TOPK_NT) hs[i] = 0;
        __syncthreads();
        for (int s0 = c0; s0 < c1; s0 += TOPK_NT * 4) {
            uint32_t kk[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int s = s0 + j * TOPK_NT + (int)threadIdx.x;
                kk[j] = s < c1 ? order_key(row[s]) : 0u;
            }
#pragma unroll
            for (int j = 0; j < 4; ++j)
                if (s0 + j * TOPK_NT + (int)threadIdx.x < c1 && (kk[j] & mask) == prefix)
                    atomicAdd(&hs[(kk[j] >> shift) & dm], 1u);
        }
        __syncthreads();
        if constexpr (CPR > 1) {
            cluster_sync();
            if (threadIdx.x < 256) {
                uint32_t v = 0;
                const uint32_t my = smem_u32(hs + threadIdx.x);
#pragma unroll
                for (int q = 0; q < CPR; ++q) v += ld_cluster_u32(mapa(my, (uint32_t)q));
                hsum[threadIdx.x] = v;
            }
            __syncthreads();
            if (warp == 0) th_pick(hsum, need, b_sel, b_above, b_count);
        } else {
            if (warp == 0) th_pick(hs, need, b_sel, b_above, b_count);
        }
        __syncthreads();
        prefix |= b_sel << shift;
        mask |= dm << shift;
        need -= b_above;
        cnt = b_count;
        if constexpr (CPR > 1) cluster_sync();  // the cluster's reads of hs are done
        else __syncthreads();
    }
    const bool listed = cnt <= (uint32_t)TOPK_CAND && cnt != need;  // else the bucket is taken whole or is one value

    // ---- 3. per warp: keys above the bucket, keys in it; list the bucket ----
    const int w0 = min(c1, c0 + warp * span), w1 = min(c1, w0 + span);
    if (threadIdx.x == 0) n_cand = 0;
    __syncthreads();
    uint32_t n_ab = 0, n_eq = 0;
    const uint32_t lt = (1u << lane) - 1u;
    for (int s00 = w0; s00 < w1; s00 += 32 * TB) {
        uint32_t kb[TB];
#pragma unroll
        for (int j = 0; j < TB; ++j) {
            const int s = s00 + 32 * j + lane;
            kb[j] = s < w1 ? order_key(row[s]) : 0u;
        }
#pragma unroll
        for (int j = 0; j < TB; ++j) {
            const int s = s00 + 32 * j + lane;
            const uint32_t key = kb[j];
            const bool ab = s < w1 && (key & mask) > prefix, eq = s < w1 && (key & mask) == prefix;
            n_ab += ab;
            const uint32_t eqm = __ballot_sync(0xffffffffu, eq);
            n_eq += (uint32_t)__popc(eqm) * (lane == 0);
            if (listed && eqm) {
                uint32_t base = 0;
                if (lane == 0) base = atomicAdd(&n_cand, (uint32_t)__popc(eqm));
                base = __shfl_sync(0xffffffffu, base, 0);
                const uint32_t slot = base + (uint32_t)__popc(eqm & lt);
                if (eq && slot < (uint32_t)TOPK_CAND) {
                    ckey[slot] = key;
                    cidx[slot] = s;
                }
            }
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        n_ab += __shfl_xor_sync(0xffffffffu, n_ab, o);
        n_eq += __shfl_xor_sync(0xffffffffu, n_eq, o);
    }
    if (lane == 0) {
        wcnt[warp][0] = n_ab;
        wcnt[warp][1] = n_eq;
    }
    __syncthreads();
    if constexpr (CPR > 1) cluster_sync();  // every CTA's list is complete

    // ---- 4. refine the listed bucket over the cluster's lists ----
    if (listed) {
        uint32_t nq[CPR], nc = 0;
#pragma unroll
        for (int q = 0; q < CPR; ++q) {
            nq[q] = CPR > 1 ? ld_cluster_u32(mapa(smem_u32(&n_cand), (uint32_t)q)) : n_cand;
            nc += nq[q];
        }
        if (nc != cnt) {  // the row changed under the passes
            leave(-5000000);
            return;
        }
        for (; lvl < 3 && cnt != need; ++lvl) {
            int shift;
            uint32_t dm;
            th_digit(lvl, shift, dm);
            for (int i = threadIdx.x; i < 256; i += TOPK_NT) hs[i] = 0;
            __syncthreads();
#pragma unroll
            for (int q = 0; q < CPR; ++q) {
                const uint32_t base = smem_u32(ckey);
                const uint32_t rb = CPR > 1 ? mapa(base, (uint32_t)q) : base;
                for (uint32_t i = threadIdx.x; i < nq[q]; i += TOPK_NT) {
                    const uint32_t key = CPR > 1 ? ld_cluster_u32(rb + 4 * i) : ckey[i];
                    if ((key & mask) == prefix) atomicAdd(&hs[(key >> shift) & dm], 1u);
                }
            }
            __syncthreads();
            if (warp == 0) th_pick(hs, need, b_sel, b_above, b_count);
            __syncthreads();
            prefix |= b_sel << shift;
            mask |= dm << shift;
            need -= b_above;
            cnt = b_count;
            __syncthreads();
        }
        // per warp: this CTA's listed keys above the refined bucket, and in it
        if (threadIdx.x < TOPK_WARPS) wcnt[threadIdx.x][1] = 0;
        __syncthreads();
        for (uint32_t i = threadIdx.x; i < n_cand; i += TOPK_NT) {
            const uint32_t km = ckey[i] & mask;
            const int w = (cidx[i] - c0) / span;
            if (km > prefix) atomicAdd(&wcnt[w][0], 1u);
            else if (km == prefix) atomicAdd(&wcnt[w][1], 1u);
        }
        __syncthreads();
    }

    // ---- 5. offsets over the warps and the cluster's CTAs; placement ----
    if (warp == 0) {  // exclusive prefixes over this CTA's warps, in index order
        const uint32_t a = wcnt[lane][0], e = wcnt[lane][1];
        uint32_t ia = a, ie = e;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t va = __shfl_up_sync(0xffffffffu, ia, o), ve = __shfl_up_sync(0xffffffffu, ie, o);
            if (lane >= o) ia += va, ie += ve;
        }
        wcnt[lane][0] = ia - a;
        wcnt[lane][1] = ie - e;
        if (lane == 31) {  // this CTA's totals, to every CTA of the cluster
            if constexpr (CPR > 1) {
#pragma unroll
                for (int q = 0; q < CPR; ++q) {
                    st_cluster_u32(mapa(smem_u32(&ctot[crank][0]), (uint32_t)q), ia);
                    st_cluster_u32(mapa(smem_u32(&ctot[crank][1]), (uint32_t)q), ie);
                }
            } else {
                ctot[0][0] = ia;
                ctot[0][1] = ie;
            }
        }
    }
    if constexpr (CPR > 1) cluster_sync();  // the last access to another CTA's shared memory
    else __syncthreads();
    uint32_t base_ab = 0, base_eq = 0, all_ab = 0;
#pragma unroll
    for (int q = 0; q < CPR; ++q) {
        if (q < (int)crank) base_ab += ctot[q][0], base_eq += ctot[q][1];
        all_ab += ctot[q][0];
    }
    uint32_t eq_before = base_eq + wcnt[warp][1];
    uint32_t pos = base_ab + wcnt[warp][0] + min(eq_before, need);
    for (int s0 = w0; s0 < w1; s0 += 32 * TB) {
        uint32_t mk[TB];  // the batch's loads first
#pragma unroll
        for (int j = 0; j < TB; ++j) {
            const int s = s0 + 32 * j + lane;
            mk[j] = s < w1 ? (order_key(row[s]) & mask) : 0u;
        }
#pragma unroll
        for (int j = 0; j < TB; ++j) {
            const int s = s0 + 32 * j + lane;
            const bool ab = s < w1 && mk[j] > prefix, eq = s < w1 && mk[j] == prefix;
            const uint32_t eqm = __ballot_sync(0xffffffffu, eq);
            const bool take = ab || (eq && eq_before + (uint32_t)__popc(eqm & lt) < need);
            const uint32_t tk = __ballot_sync(0xffffffffu, take);
            if (take && pos + (uint32_t)__popc(tk & lt) < (uint32_t)k) out[pos + __popc(tk & lt)] = s;
            pos += (uint32_t)__popc(tk);
            eq_before += (uint32_t)__popc(eqm);
        }
    }
    const uint32_t total = all_ab + need;
    if (crank == 0) {
        for (int s = (int)total + (int)threadIdx.x; s < width; s += TOPK_NT) out[s] = -1;
        if (threadIdx.x == 0 && total != (uint32_t)k) report(st, DSA_ERR_INDEX, -1000000 - t);
    }
}

void launch_topk_hist(const TopkArgs& a, cudaStream_t s) {
    if (a.row_count <= 0) return;
    // few rows (decode): four CTAs per row, so that every SM of a B200 works
    if (a.row_count < 2 * 148)
        topk_hist_kernel<4><<<(unsigned)(4 * a.row_count), TOPK_NT, 0, s>>>(a.sv, a.scores, a.ld, a.row_begin, a.k,
                                                                            a.k_rows, a.idx, a.ld_idx, a.st);
    else
        topk_hist_kernel<1><<<(unsigned)a.row_count, TOPK_NT, 0, s>>>(a.sv, a.scores, a.ld, a.row_begin, a.k, a.k_rows,
                                                                     a.idx, a.ld_idx, a.st);
}

void launch_topk_rows(const TopkArgs& a, cudaStream_t s) {
    if (a.row_count <= 0) return;
    topk_rows_kernel<<<(unsigned)a.row_count, TOPK_NT, 0, s>>>(a.sv, a.scores, a.ld, a.row_begin, a.k, a.k_rows, a.idx,
                                                              a.ld_idx, a.st);
}

// ---------------------------------------------------------------------------
// a4, fp32: one warp per (query, head); online softmax over the selected
// rows with expf; dk, dv <= 128 (multiples of 32).
// ---------------------------------------------------------------------------
template <int DK, int DV>
__global__ void attn_f32_kernel(SeqView sv, AttnF32Args a, const int32_t* __restrict__ idx, int64_t ld_idx, int k_sel,
                                StatusHdr* st) {
    const int64_t t = blockIdx.x;
    const int h = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (h >= a.heads) return;
    const RowInfo ri = row_info(sv, t);
    if (!ri.ok) {
        if (threadIdx.x == 0) report(st, DSA_ERR_INDEX, t);
        return;
    }
    constexpr int NQ = DK / 32, NV = DV / 32;
    const float* qp = a.q + t * a.q_stride_tok + h * a.q_stride_head;
    float q[NQ], o[NV];
#pragma unroll
    for (int i = 0; i < NQ; ++i) q[i] = qp[lane + 32 * i];
#pragma unroll
    for (int i = 0; i < NV; ++i) o[i] = 0.f;
    float m = -INFINITY, l = 0.f;
    const int32_t* ir = idx + t * ld_idx;
    for (int j = 0; j < k_sel; ++j) {
        const int32_t v = ir[j];
        if (v < 0) continue;
        if (v >= ri.seqlen_k) {
            if (lane == 0 && h == 0) report(st, DSA_ERR_INDEX, t);
            continue;
        }
        const int64_t row = ri.key_base + v;
        const float* kr = a.k + row * a.k_stride;
        float d = 0.f;
#pragma unroll
        for (int i = 0; i < NQ; ++i) d = fmaf(q[i], kr[lane + 32 * i], d);
#pragma unroll
        for (int o2 = 16; o2 > 0; o2 >>= 1) d += __shfl_xor_sync(0xffffffffu, d, o2);
        const float z = d * a.scale;
        if (z > m) {
            const float c = expf(m - z);
            l *= c;
#pragma unroll
            for (int i = 0; i < NV; ++i) o[i] *= c;
            m = z;
        }
        const float p = expf(z - m);
        l += p;
        const float* vr = a.v + row * a.v_stride;
#pragma unroll
        for (int i = 0; i < NV; ++i) o[i] = fmaf(p, vr[lane + 32 * i], o[i]);
    }
    float* op = a.out + t * a.out_stride_tok + h * a.out_stride_head;
    const float inv = l > 0.f ? 1.0f / l : 0.f;
#pragma unroll
    for (int i = 0; i < NV; ++i) op[lane + 32 * i] = o[i] * inv;
    if (a.lse && lane == 0) a.lse[t * a.heads + h] = l > 0.f ? m + logf(l) : -INFINITY;
}

template <int DK>
static bool launch_attn_f32_dk(int dv, const AttnF32Launch& L, cudaStream_t s) {
    dim3 grid((unsigned)L.total_q), block((unsigned)(L.a.heads * 32));
    switch (dv) {
        case 32: attn_f32_kernel<DK, 32><<<grid, block, 0, s>>>(L.sv, L.a, L.idx, L.ld_idx, L.k_sel, L.st); return true;
        case 64: attn_f32_kernel<DK, 64><<<grid, block, 0, s>>>(L.sv, L.a, L.idx, L.ld_idx, L.k_sel, L.st); return true;
        case 96: attn_f32_kernel<DK, 96><<<grid, block, 0, s>>>(L.sv, L.a, L.idx, L.ld_idx, L.k_sel, L.st); return true;
        case 128: attn_f32_kernel<DK, 128><<<grid, block, 0, s>>>(L.sv, L.a, L.idx, L.ld_idx, L.k_sel, L.st); return true;
    }
    return false;
}

bool launch_attn_f32(const AttnF32Launch& L, cudaStream_t s) {
    if (L.total_q <= 0) return true;
    switch (L.dk) {
        case 32: return launch_attn_f32_dk<32>(L.dv, L, s);
        case 64: return launch_attn_f32_dk<64>(L.dv, L, s);
        case 96: return launch_attn_f32_dk<96>(L.dv, L, s);
        case 128: return launch_attn_f32_dk<128>(L.dv, L, s);
    }
    return false;
}

// ---------------------------------------------------------------------------
// Failure-detection self test: one thread waits on an mbarrier that nothing
// arrives on, with a short budget, and records DSA_ERR_TIMEOUT.
// ---------------------------------------------------------------------------
__global__ void selftest_wait_kernel(StatusHdr* st, long long budget) {
    __shared__ __align__(8) uint64_t bar;
    const uint32_t b = smem_u32(&bar);
    if (threadIdx.x == 0) mbar_init(b, 1);
    __syncthreads();
    if (threadIdx.x == 0) mbar_wait(b, 0, nullptr, st, 0x5e1f, budget);
}

void launch_selftest_wait(StatusHdr* st, long long budget, cudaStream_t s) {
    selftest_wait_kernel<<<1, 32, 0, s>>>(st, budget);
}

}  // namespace dsa
