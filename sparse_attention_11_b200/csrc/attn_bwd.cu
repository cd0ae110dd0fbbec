// attn_bwd.cu -- backward of the sparse MQA attention over the selected KV
// rows, on CUDA cores with fp32 arithmetic.
//
// Method: "DeepSeek-V3.2与稀疏注意力技术革新".  §2.3: the attention is
// standard attention over the k selected keys.  §3.1: the 128 query heads
// share one KV row.  §4.1: training runs the sparse attention in its sparse
// stage, so the selection needs gradients.  For query t, head h and selected
// row j:
//   P_j  = exp(scale * q.K_j - lse)      (lse from the forward)
//   dP_j = dO . V_j,   D = dO . O         (O the forward's stored output)
//   dS_j = P_j (dP_j - D)
//   dq   = scale * sum_j dS_j K_j
//   dK_j += scale * sum_h dS_j q_h,   dV_j += sum_h P_j dO_h
//
// This is the first, plainly correct version of this step.  One CTA takes one
// query and 16 of its heads.  The heads' q and dO rows are staged in shared
// memory as fp32.  For each selected row, 16 lanes per head form the two dot
// products, each thread accumulates 36 columns of its head's dq in
// registers, and the CTA reduces the 16 heads' contributions to the row's
// dK and dV before adding them to global memory with fp32 atomics.  dK and dV
// may be one buffer: with V the first dv columns of the KV row (MLA), passing
// dV = dK yields the tied gradient directly.
#include "dsa_kernels.h"

namespace dsa {

constexpr int BW_HG = 16;         // heads per CTA
constexpr int BW_THREADS = 256;   // 16 lanes per head
constexpr int BW_NQ = kBwdMaxDk / 16;  // dq columns per thread

template <typename T>
__device__ __forceinline__ float ldf(const T* p);
template <>
__device__ __forceinline__ float ldf<float>(const float* p) {
    return __ldg(p);
}
template <>
__device__ __forceinline__ float ldf<__nv_bfloat16>(const __nv_bfloat16* p) {
    return __bfloat162float(*p);
}

// sum over the 16 lanes of a half-warp (every lane of the warp takes part)
__device__ __forceinline__ float sum16(float x) {
    x += __shfl_xor_sync(0xffffffffu, x, 8);
    x += __shfl_xor_sync(0xffffffffu, x, 4);
    x += __shfl_xor_sync(0xffffffffu, x, 2);
    x += __shfl_xor_sync(0xffffffffu, x, 1);
    return x;
}

template <typename T>
__global__ void __launch_bounds__(BW_THREADS) attn_bwd_kernel(const __grid_constant__ AttnBwdArgs a) {
    extern __shared__ float bw_smem[];
    const int dk = a.dk, dv = a.dv;
    float* sq = bw_smem;              // [16][dk]
    float* sdo = sq + BW_HG * dk;     // [16][dv]
    float* sk = sdo + BW_HG * dv;     // [dk]  the selected K row
    float* svr = sk + dk;             // [dv]  the selected V row
    float* sp = svr + dv;             // [16]  P of each head
    float* sds = sp + BW_HG;          // [16]  dS of each head

    const int64_t t = blockIdx.x;
    const int h0 = (int)blockIdx.y * BW_HG;
    const int tid = (int)threadIdx.x, hl = tid >> 4, part = tid & 15;
    const int h = h0 + hl;
    const bool hv = h < a.heads;
    const RowInfo ri = row_info(a.sv, t);
    if (!ri.ok) {  // uniform over the CTA
        if (tid == 0) report(a.st, DSA_ERR_INDEX, t);
        return;
    }
    const T* q = (const T*)a.q;
    const T* kp = (const T*)a.k;
    const T* vp = (const T*)a.v;
    const T* op = (const T*)a.out;
    const T* dop = (const T*)a.dout;

    for (int i = tid; i < BW_HG * dk; i += BW_THREADS) {
        const int hh = i / dk, c = i - hh * dk;
        sq[i] = (h0 + hh < a.heads) ? ldf(q + t * a.q_stride_tok + (int64_t)(h0 + hh) * a.q_stride_head + c) : 0.f;
    }
    for (int i = tid; i < BW_HG * dv; i += BW_THREADS) {
        const int hh = i / dv, c = i - hh * dv;
        sdo[i] = (h0 + hh < a.heads) ? ldf(dop + t * a.dout_stride_tok + (int64_t)(h0 + hh) * a.dout_stride_head + c)
                                     : 0.f;
    }
    __syncthreads();

    // D = dO . O of this thread's head, and its lse
    float D = 0.f;
    if (hv) {
        const T* orow = op + t * a.out_stride_tok + (int64_t)h * a.out_stride_head;
        for (int c = part; c < dv; c += 16) D = fmaf(sdo[hl * dv + c], ldf(orow + c), D);
    }
    D = sum16(D);
    const float lse = hv ? __ldg(a.lse + t * a.heads + h) : 0.f;

    float acc[BW_NQ];
#pragma unroll
    for (int i = 0; i < BW_NQ; ++i) acc[i] = 0.f;

    const int32_t* ir = a.idx + t * a.ld_idx;
    for (int s = 0; s < a.k_sel; ++s) {
        const int32_t j = __ldg(ir + s);  // the same value in every thread
        if (j < 0) continue;
        if (j >= ri.seqlen_k) {
            if (tid == 0) report(a.st, DSA_ERR_INDEX, t);
            continue;
        }
        const int64_t row = ri.key_base + j;
        __syncthreads();  // the previous row's sk / svr / sp / sds are read
        for (int c = tid; c < dk; c += BW_THREADS) sk[c] = ldf(kp + row * a.k_stride + c);
        for (int c = tid; c < dv; c += BW_THREADS) svr[c] = ldf(vp + row * a.v_stride + c);
        __syncthreads();
        float z = 0.f, dp = 0.f;
        for (int c = part; c < dk; c += 16) z = fmaf(sq[hl * dk + c], sk[c], z);
        for (int c = part; c < dv; c += 16) dp = fmaf(sdo[hl * dv + c], svr[c], dp);
        z = sum16(z);
        dp = sum16(dp);
        const float P = hv ? expf(fmaf(z, a.scale, -lse)) : 0.f;
        const float ds = P * (dp - D);
#pragma unroll
        for (int i = 0; i < BW_NQ; ++i) {
            const int c = part + 16 * i;
            if (c < dk) acc[i] = fmaf(ds, sk[c], acc[i]);
        }
        if (part == 0) {
            sp[hl] = P;
            sds[hl] = ds;
        }
        __syncthreads();
        for (int c = tid; c < dk; c += BW_THREADS) {
            float g = 0.f;
#pragma unroll
            for (int hh = 0; hh < BW_HG; ++hh) g = fmaf(sds[hh], sq[hh * dk + c], g);
            atomicAdd(a.d_k + row * a.d_k_stride + c, g * a.scale);
        }
        for (int c = tid; c < dv; c += BW_THREADS) {
            float g = 0.f;
#pragma unroll
            for (int hh = 0; hh < BW_HG; ++hh) g = fmaf(sp[hh], sdo[hh * dv + c], g);
            atomicAdd(a.d_v + row * a.d_v_stride + c, g);
        }
    }
    if (hv) {
        float* dq = a.d_q + t * a.d_q_stride_tok + (int64_t)h * a.d_q_stride_head;
#pragma unroll
        for (int i = 0; i < BW_NQ; ++i) {
            const int c = part + 16 * i;
            if (c < dk) dq[c] = acc[i] * a.scale;
        }
    }
}

size_t attn_bwd_smem_bytes(int dk, int dv) {
    return (size_t)(BW_HG * dk + BW_HG * dv + dk + dv + 2 * BW_HG) * sizeof(float);
}

bool launch_attn_bwd(const AttnBwdArgs& a, int dtype_bf16, cudaStream_t s) {
    if (a.total_q <= 0) return true;
    if (a.dk < 1 || a.dk > kBwdMaxDk || a.dv < 1 || a.dv > kBwdMaxDv || a.heads < 1) return false;
    const size_t smem = attn_bwd_smem_bytes(a.dk, a.dv);
    const dim3 grid((unsigned)a.total_q, (unsigned)((a.heads + BW_HG - 1) / BW_HG), 1);
    if (dtype_bf16) {
        if (cudaFuncSetAttribute(attn_bwd_kernel<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)smem) != cudaSuccess)
            return false;
        attn_bwd_kernel<__nv_bfloat16><<<grid, BW_THREADS, smem, s>>>(a);
    } else {
        if (cudaFuncSetAttribute(attn_bwd_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
            cudaSuccess)
            return false;
        attn_bwd_kernel<float><<<grid, BW_THREADS, smem, s>>>(a);
    }
    return cudaGetLastError() == cudaSuccess;
}

}  // namespace dsa
