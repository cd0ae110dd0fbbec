// indexer_kl.cu -- the lightning indexer's KL distillation in the sparse
// training stage, on CUDA cores with fp32 arithmetic.
//
// Method: "DeepSeek-V3.2与稀疏注意力技术革新".  §4.1: the indexer learns by a
// KL-divergence loss to imitate the main attention's distribution, in the
// dense warm-up and then in the sparse stage.  §2.2: I[t,s] = ReLU(q_t ·
// W_index · k_s).  The pages give no formula for the loss.  Reading: the
// target p_t is the main attention's probabilities of query t averaged over
// the heads, over the candidates (here the selected set), and the indexer's
// distribution is r_t = softmax over the same set of I[t, .].  The loss is
// sum_t KL(p_t || r_t).  Training arithmetic is real-valued.
//
// attn_pmean_kernel: p[t, slot] = (1/H) sum_h exp(scale q[t,h].K[row] -
//   lse[t,h]) for every valid slot, 0 for empty ones.  One CTA per query and
//   16 heads, the same work layout as the attention backward; the groups
//   add their partial means with atomics, so p must start at zero.
// indexer_kl_kernel: one CTA of 128 threads per query.
//   u = q W;  x_s = u . k_s;  I_s = max(x_s, 0);  r = softmax_s(I);
//   loss_t = sum_s p_s (log p_s - log r_s)            (terms with p_s = 0 drop)
//   G_s = (r_s - p_s) [x_s > 0];  v = sum_s G_s k_s
//   d_q[t] = W v;  d_W += q_t^T v;  d_k[s] += G_s u   (atomics)
#include "dsa_kernels.h"

namespace dsa {

constexpr int PM_HG = 16;
constexpr int PM_THREADS = 256;

template <typename T>
__device__ __forceinline__ float kl_ld(const T* p);
template <>
__device__ __forceinline__ float kl_ld<float>(const float* p) {
    return __ldg(p);
}
template <>
__device__ __forceinline__ float kl_ld<__nv_bfloat16>(const __nv_bfloat16* p) {
    return __bfloat162float(*p);
}

__device__ __forceinline__ float pm_sum16(float x) {
    x += __shfl_xor_sync(0xffffffffu, x, 8);
    x += __shfl_xor_sync(0xffffffffu, x, 4);
    x += __shfl_xor_sync(0xffffffffu, x, 2);
    x += __shfl_xor_sync(0xffffffffu, x, 1);
    return x;
}

template <typename T>
__global__ void __launch_bounds__(PM_THREADS) attn_pmean_kernel(const __grid_constant__ AttnPmeanArgs a) {
    extern __shared__ float pm_smem[];
    const int dk = a.dk;
    float* sq = pm_smem;            // [16][dk]
    float* sk = sq + PM_HG * dk;    // [dk]
    float* sp = sk + dk;            // [16]
    const int64_t t = blockIdx.x;
    const int h0 = (int)blockIdx.y * PM_HG;
    const int tid = (int)threadIdx.x, hl = tid >> 4, part = tid & 15;
    const int h = h0 + hl;
    const bool hv = h < a.heads;
    const RowInfo ri = row_info(a.sv, t);
    if (!ri.ok) {
        if (tid == 0) report(a.st, DSA_ERR_INDEX, t);
        return;
    }
    const T* q = (const T*)a.q;
    const T* kp = (const T*)a.k;
    for (int i = tid; i < PM_HG * dk; i += PM_THREADS) {
        const int hh = i / dk, c = i - hh * dk;
        sq[i] = (h0 + hh < a.heads) ? kl_ld(q + t * a.q_stride_tok + (int64_t)(h0 + hh) * a.q_stride_head + c) : 0.f;
    }
    const float lse = hv ? __ldg(a.lse + t * a.heads + h) : 0.f;
    const float inv_h = 1.0f / (float)a.heads;
    const int32_t* ir = a.idx + t * a.ld_idx;
    for (int s = 0; s < a.k_sel; ++s) {
        const int32_t j = __ldg(ir + s);  // the same value in every thread
        if (j < 0) continue;
        if (j >= ri.seqlen_k) {
            if (tid == 0) report(a.st, DSA_ERR_INDEX, t);
            continue;
        }
        const int64_t row = ri.key_base + j;
        __syncthreads();  // sq staged; the previous row's sk / sp are read
        for (int c = tid; c < dk; c += PM_THREADS) sk[c] = kl_ld(kp + row * a.k_stride + c);
        __syncthreads();
        float z = 0.f;
        for (int c = part; c < dk; c += 16) z = fmaf(sq[hl * dk + c], sk[c], z);
        z = pm_sum16(z);
        if (part == 0) sp[hl] = hv ? expf(fmaf(z, a.scale, -lse)) : 0.f;
        __syncthreads();
        if (tid == 0) {
            float m = 0.f;
#pragma unroll
            for (int hh = 0; hh < PM_HG; ++hh) m += sp[hh];
            atomicAdd(a.p + t * a.ld_p + s, m * inv_h);
        }
    }
}

// one CTA (128 threads) per query; the slot arrays live in shared memory
constexpr int KL_THREADS = 128;

__device__ __forceinline__ float kl_block_sum(float v, float* red) {
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    const int w = (int)threadIdx.x >> 5, l = (int)threadIdx.x & 31;
    __syncthreads();
    if (l == 0) red[w] = v;
    __syncthreads();
    float s = 0.f;
#pragma unroll
    for (int i = 0; i < KL_THREADS / 32; ++i) s += red[i];
    return s;
}

__device__ __forceinline__ float kl_block_max(float v, float* red) {
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    const int w = (int)threadIdx.x >> 5, l = (int)threadIdx.x & 31;
    __syncthreads();
    if (l == 0) red[w] = v;
    __syncthreads();
    float s = -INFINITY;
#pragma unroll
    for (int i = 0; i < KL_THREADS / 32; ++i) s = fmaxf(s, red[i]);
    return s;
}

__global__ void __launch_bounds__(KL_THREADS) indexer_kl_kernel(const __grid_constant__ IndexerKlArgs a) {
    extern __shared__ float kl_smem[];
    float* su = kl_smem;          // [128] u = q W
    float* sq = su + 128;         // [128] q
    float* sv = sq + 128;         // [128] v = sum_s G_s k_s
    float* red = sv + 128;        // [4]
    float* sx = red + 4;          // [k_sel] x_s (NaN for empty slots)
    float* sg = sx + a.k_sel;     // [k_sel] G_s
    const int64_t t = blockIdx.x;
    const int i = (int)threadIdx.x;
    const RowInfo ri = row_info(a.sv, t);
    if (!ri.ok) {
        if (i == 0) report(a.st, DSA_ERR_INDEX, t);
        return;
    }
    sq[i] = __ldg(a.q + t * a.q_stride + i);
    __syncthreads();
    {
        float u = 0.f;
        for (int c = 0; c < 128; ++c) u = fmaf(sq[c], __ldg(a.W + c * 128 + i), u);
        su[i] = u;
    }
    __syncthreads();
    const int32_t* ir = a.idx + t * a.ld_idx;
    // x_s for every slot, one thread per slot
    float mx = -INFINITY;
    for (int s = i; s < a.k_sel; s += KL_THREADS) {
        const int32_t j = __ldg(ir + s);
        float x = __int_as_float(0x7fc00000);  // NaN marks an empty slot
        if (j >= 0 && j < ri.seqlen_k) {
            const float* kr = a.k + (ri.key_base + j) * a.k_stride;
            float d = 0.f;
            for (int c = 0; c < 128; ++c) d = fmaf(su[c], __ldg(kr + c), d);
            x = d;
            mx = fmaxf(mx, fmaxf(d, 0.f));
        } else if (j >= ri.seqlen_k) {
            report(a.st, DSA_ERR_INDEX, t);
        }
        sx[s] = x;
    }
    mx = kl_block_max(mx, red);
    float se = 0.f;
    for (int s = i; s < a.k_sel; s += KL_THREADS)
        if (!isnan(sx[s])) se += expf(fmaxf(sx[s], 0.f) - mx);
    se = kl_block_sum(se, red);
    const float lse = mx + logf(se);  // log sum_s exp(I_s); -inf + ... never used when the row is empty
    float loss = 0.f;
    for (int s = i; s < a.k_sel; s += KL_THREADS) {
        float g = 0.f;
        if (!isnan(sx[s])) {
            const float lr = fmaxf(sx[s], 0.f) - lse;  // log r_s
            const float p = __ldg(a.p + t * a.ld_p + s);
            if (p > 0.f) loss += p * (logf(p) - lr);
            g = sx[s] > 0.f ? expf(lr) - p : 0.f;
        }
        sg[s] = g;
    }
    loss = kl_block_sum(loss, red);
    if (i == 0 && a.loss) a.loss[t] = loss;
    // v = sum_s G_s k_s (thread i: column i) and d_k[s] += G_s u
    float v = 0.f;
    for (int s = 0; s < a.k_sel; ++s) {
        const float g = sg[s];
        if (g == 0.f) continue;  // the same branch in every thread
        const int64_t row = ri.key_base + __ldg(ir + s);
        v = fmaf(g, __ldg(a.k + row * a.k_stride + i), v);
        atomicAdd(a.d_k + row * a.d_k_stride + i, g * su[i]);
    }
    sv[i] = v;
    __syncthreads();
    // d_q = W v (row i of W against v), d_W[c][i] += q_c v_i
    float dq = 0.f;
    for (int c = 0; c < 128; ++c) dq = fmaf(__ldg(a.W + i * 128 + c), sv[c], dq);
    a.d_q[t * a.d_q_stride + i] = dq;
    for (int c = 0; c < 128; ++c) atomicAdd(a.d_W + c * 128 + i, sq[c] * sv[i]);
}

size_t attn_pmean_smem_bytes(int dk) { return (size_t)(PM_HG * dk + dk + PM_HG) * sizeof(float); }

bool launch_attn_pmean(const AttnPmeanArgs& a, int dtype_bf16, cudaStream_t s) {
    if (a.total_q <= 0) return true;
    if (a.dk < 1 || a.dk > kBwdMaxDk || a.heads < 1) return false;
    const size_t smem = attn_pmean_smem_bytes(a.dk);
    const dim3 grid((unsigned)a.total_q, (unsigned)((a.heads + PM_HG - 1) / PM_HG), 1);
    if (dtype_bf16) {
        if (cudaFuncSetAttribute(attn_pmean_kernel<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)smem) != cudaSuccess)
            return false;
        attn_pmean_kernel<__nv_bfloat16><<<grid, PM_THREADS, smem, s>>>(a);
    } else {
        if (cudaFuncSetAttribute(attn_pmean_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
            cudaSuccess)
            return false;
        attn_pmean_kernel<float><<<grid, PM_THREADS, smem, s>>>(a);
    }
    return cudaGetLastError() == cudaSuccess;
}

bool launch_indexer_kl(const IndexerKlArgs& a, cudaStream_t s) {
    if (a.total_q <= 0) return true;
    const size_t smem = (size_t)(3 * 128 + 4 + 2 * a.k_sel) * sizeof(float);
    if (smem > 200 * 1024) return false;
    if (cudaFuncSetAttribute(indexer_kl_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
        return false;
    indexer_kl_kernel<<<(unsigned)a.total_q, KL_THREADS, smem, s>>>(a);
    return cudaGetLastError() == cudaSuccess;
}

}  // namespace dsa
