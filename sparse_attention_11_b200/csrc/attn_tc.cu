// attn_tc.cu -- sparse MQA attention over the selected KV rows on the
// 5th-generation tensor cores (BF16 in, fp32 accumulate).
//
// Method: "DeepSeek-V3.2与稀疏注意力技术革新", §2.3 (standard attention on the
// selected subset of k keys) and §3.1 (MLA in MQA mode: the 128 query heads
// share one KV row of 576 = 512 latent + 64 rope columns; V is 512 wide).
//
// For one query the work is two dense contractions over the gathered rows:
// S = Q K^T (128 x 576 by 576 x k) and O = P V (128 x k by k x 512).  O alone
// (128 x 512 fp32) fills a whole SM's tensor memory, so each query runs on a
// CTA pair (a cluster of two):
//   rank 0: contraction columns [0,256)   output columns [0,256)
//   rank 1: contraction columns [256,576) output columns [256,512)
// When V is the latent part of K (V = K[:, :512]) each CTA's V columns are
// the first 256 of its own K columns, so every gathered byte is used once.
//
// Softmax split: per 64-key tile each CTA holds a partial S for all 128 heads
// and all 64 keys.  Rank r finishes the scores of keys [32r, 32r+32) for all
// heads: it sends the other 32 partial columns to its peer and receives the
// peer's partials of its own 32 keys (st.async into the peer's shared memory,
// counted on the peer's mbarrier).  Both CTAs use the same running maximum:
// the sum of the two partial maxima of the tile, an upper bound of the true
// maximum that both can form from the exchanged data, with lazy rescaling
// (moved only when it grows by more than 2^8).  Each CTA then computes bf16
// probabilities for its 32 keys, sends them to the peer, and accumulates its
// half of O over all 64 keys.  The row sums are combined once at the end.
//
// Tensor memory per CTA (512 columns): O [0,256)  S [256,320)  P [320,352)
// Q [352, 352 + 32 * blocks).  Q and P are the A operands, read from TMEM
// (tcgen05.mma ... [a_tmem]); K/V tiles are B operands in shared memory,
// gathered by TMA tile::gather4 (4 rows x 64 columns per instruction, 128-byte
// swizzle) straight from the KV rows named by the index list.
//
// Warps: 0 gather producer, 1 MMA issuer (+TMEM owner), 2..5 softmax /
// exchange / epilogue (thread <-> head, the TMEM lane).
#include "dsa_kernels.h"

namespace dsa {

constexpr int AT_N = 64;                            // keys per tile
constexpr uint32_t AT_BLK = AT_N * 128;             // one 64-column block of a tile
constexpr uint32_t AT_KST = 5 * AT_BLK;             // K part of a stage (max 5 blocks)
constexpr uint32_t AT_VST = 4 * AT_BLK;             // V part (separate V only)
constexpr uint32_t AT_SX_PITCH = 144;               // 32 fp32 partials + partial max + pad
constexpr uint32_t AT_PX_PITCH = 80;                // 32 bf16 probabilities + pad
constexpr uint32_t AT_SX_BYTES = 128 * 9 * 16;      // bytes counted per tile
constexpr uint32_t AT_PX_BYTES = 128 * 4 * 16;
constexpr uint32_t TM_O = 0, TM_S = 256, TM_P = 320, TM_Q = 352;

template <int NST, bool VSEP>
struct AtLayout {
    static constexpr uint32_t STAGE = AT_KST + (VSEP ? AT_VST : 0);
    static constexpr uint32_t OFF_SX = NST * STAGE;                   // [2][128][144]
    static constexpr uint32_t OFF_PX = OFF_SX + 2 * 128 * AT_SX_PITCH;  // [2][128][80]
    static constexpr uint32_t OFF_LX = OFF_PX + 2 * 128 * AT_PX_PITCH;  // [128] fp32
    static constexpr uint32_t OFF_BAR = OFF_LX + 512;
    static constexpr uint32_t SMEM = OFF_BAR + 512 + 1024;
};

struct AtBars {
    uint64_t full[4];
    uint64_t empty[4];
    uint64_t s_full, s_empty, p_full, p_free, q_full, o_full;
    uint64_t sx_full[2], px_full[2], lx_full;  // filled by the peer (st.async, byte-counted)
    uint64_t sx_free[2], px_free[2];           // the peer consumed what this CTA sent
    uint64_t drain;
    uint32_t tmem_base;
    int abort;
    int max_slot;
};

template <int NST, bool VSEP>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(192, 1) attn_tc_kernel(const __grid_constant__ AttnTcArgs a) {
    using Lay = AtLayout<NST, VSEP>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    AtBars* bars = (AtBars*)(smem + Lay::OFF_BAR);
    const uint32_t warp = warp_id(), lane = lane_id();
    const uint32_t rank = cluster_ctarank(), peer = rank ^ 1u;
    StatusHdr* st = a.st;
    volatile int* abort = &bars->abort;

    const int64_t t = blockIdx.x >> 1;
    const RowInfo ri = row_info(a.sv, t);
    if (!ri.ok) {  // both CTAs of the pair take this exit together
        if (threadIdx.x == 0 && rank == 0) report(st, DSA_ERR_INDEX, t);
        return;
    }
    const int nb = rank ? 5 : 4;           // 64-column blocks of K held here
    const int col0 = rank ? 256 : 0;       // first K column
    const int dv0 = rank ? 256 : 0;        // first output column
    const int32_t* irow = a.idx + t * a.ld_idx;

    if (threadIdx.x == 0) {
        for (int i = 0; i < NST; ++i) {
            mbar_init(smem_u32(&bars->full[i]), 1);
            mbar_init(smem_u32(&bars->empty[i]), 1);
        }
        mbar_init(smem_u32(&bars->s_full), 1);
        mbar_init(smem_u32(&bars->s_empty), 4);
        mbar_init(smem_u32(&bars->p_full), 4);
        mbar_init(smem_u32(&bars->p_free), 1);
        mbar_init(smem_u32(&bars->q_full), 4);
        mbar_init(smem_u32(&bars->o_full), 1);
        for (int i = 0; i < 2; ++i) {
            mbar_init(smem_u32(&bars->sx_full[i]), 1);
            mbar_init(smem_u32(&bars->px_full[i]), 1);
            mbar_init(smem_u32(&bars->sx_free[i]), 4);
            mbar_init(smem_u32(&bars->px_free[i]), 4);
        }
        mbar_init(smem_u32(&bars->lx_full), 1);
        mbar_init(smem_u32(&bars->drain), 1);
        // arm the byte-counted barriers for their first phase
        for (int i = 0; i < 2; ++i) {
            mbar_arrive_expect_tx(smem_u32(&bars->sx_full[i]), AT_SX_BYTES);
            mbar_arrive_expect_tx(smem_u32(&bars->px_full[i]), AT_PX_BYTES);
        }
        mbar_arrive_expect_tx(smem_u32(&bars->lx_full), 128 * 4);
        bars->abort = 0;
        bars->max_slot = -1;
        fence_mbar_init();
    }
    if (warp == 1) tmem_alloc(smem_u32(&bars->tmem_base), 512);
    __syncthreads();
    // number of 64-slot tiles: up to the last valid slot of the index row
    {
        int m = -1;
        for (int j = threadIdx.x; j < a.k_sel; j += blockDim.x)
            if (__ldg(irow + j) >= 0) m = j;
        for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, o));
        if (lane == 0 && m >= 0) atomicMax(&bars->max_slot, m);
    }
    tc_fence_before();
    cluster_sync();  // barriers of both CTAs initialised and armed; max_slot final
    tc_fence_after();
    const uint32_t tmem = bars->tmem_base;
    const int n_tiles = (bars->max_slot + AT_N) / AT_N;

    const uint32_t s_stage0 = smem_u32(smem);
    if (warp == 0) {
        // ================= gather producer =================
        if (lane == 0) {
            tma_prefetch_desc(&a.tm_k);
            if (VSEP) tma_prefetch_desc(&a.tm_v);
        }
        uint32_t last_issued[NST];
        for (int i = 0; i < NST; ++i) last_issued[i] = 0xFFFFFFFFu;
        int32_t nxt[4];
        auto load_rows = [&](int j, int32_t (&rw)[4]) {
            if (lane < 16) {
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int slot = j * AT_N + lane * 4 + i;
                    rw[i] = slot < a.k_sel ? __ldg(irow + slot) : -1;
                }
            }
        };
        if (n_tiles > 0) load_rows(0, nxt);
        for (int j = 0; j < n_tiles; ++j) {
            const uint32_t s = j % NST;
            int32_t rows[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) rows[i] = nxt[i];
            if (j + 1 < n_tiles) load_rows(j + 1, nxt);
            if (lane < 16) {
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int32_t v = rows[i];
                    if (v >= ri.seqlen_k) report(st, DSA_ERR_INDEX, t);
                    rows[i] = (int32_t)(ri.key_base + ((v >= 0 && v < ri.seqlen_k) ? v : 0));
                }
            }
            if (!wait_warp(smem_u32(&bars->empty[s]), ((j / NST) & 1) ^ 1, abort, st, 0x2101)) break;
            if (lane == 0)
                mbar_arrive_expect_tx(smem_u32(&bars->full[s]), nb * AT_BLK + (VSEP ? AT_VST : 0));
            __syncwarp();
            if (lane < 16) {
                const uint32_t kst = s_stage0 + s * Lay::STAGE;
                for (int kb = 0; kb < nb; ++kb)
                    tma_gather4(kst + kb * AT_BLK + lane * 512, &a.tm_k, col0 + kb * 64, rows[0], rows[1], rows[2], rows[3],
                                smem_u32(&bars->full[s]));
                if (VSEP)
                    for (int vb = 0; vb < 4; ++vb)
                        tma_gather4(kst + AT_KST + vb * AT_BLK + lane * 512, &a.tm_v, dv0 + vb * 64, rows[0], rows[1], rows[2],
                                    rows[3], smem_u32(&bars->full[s]));
            }
            last_issued[s] = j;
            __syncwarp();
        }
        if (*abort && lane == 0)
            for (int s = 0; s < NST; ++s)
                if (last_issued[s] != 0xFFFFFFFFu)
                    mbar_wait(smem_u32(&bars->full[s]), (last_issued[s] / NST) & 1, nullptr, st, 0x2102, 1ll << 28);
    } else if (warp == 1) {
        // ================= MMA issuer =================
        constexpr uint32_t idesc_s = idesc_make(1, 1, false, 128, AT_N);
        constexpr uint32_t idesc_pv = idesc_make(1, 1, true, 128, 256);
        bool ok = n_tiles > 0 && wait_warp(smem_u32(&bars->q_full), 0, abort, st, 0x2201);
        auto issue_pv = [&](int jj) -> bool {
            if (!wait_warp(smem_u32(&bars->p_full), jj & 1, abort, st, 0x2202)) return false;
            tc_fence_after();
            if (lane == 0) {
                const uint32_t vbase = s_stage0 + (jj % NST) * Lay::STAGE + (VSEP ? AT_KST : 0);
#pragma unroll
                for (int ks = 0; ks < AT_N / 16; ++ks)
                    mma_bf16_ts(tmem + TM_O, tmem + TM_P + ks * 8, sdesc_sw128(vbase + ks * 2048, AT_BLK, 1024), idesc_pv,
                                (jj > 0 || ks > 0) ? 1u : 0u);
                mma_commit(smem_u32(&bars->empty[jj % NST]));
                mma_commit(smem_u32(&bars->p_free));
            }
            __syncwarp();
            return true;
        };
        for (int j = 0; ok && j < n_tiles; ++j) {
            const uint32_t s = j % NST;
            if (!wait_warp(smem_u32(&bars->full[s]), (j / NST) & 1, abort, st, 0x2203)) { ok = false; break; }
            if (!wait_warp(smem_u32(&bars->s_empty), (j & 1) ^ 1, abort, st, 0x2204)) { ok = false; break; }
            tc_fence_after();
            if (lane == 0) {
                const uint32_t kst = s_stage0 + s * Lay::STAGE;
                for (int kb = 0; kb < nb; ++kb)
#pragma unroll
                    for (int ks = 0; ks < 4; ++ks)
                        mma_bf16_ts(tmem + TM_S, tmem + TM_Q + kb * 32 + ks * 8,
                                    sdesc_sw128(kst + kb * AT_BLK + ks * 32, 16, 1024), idesc_s, (kb | ks) ? 1u : 0u);
                mma_commit(smem_u32(&bars->s_full));
            }
            __syncwarp();
            if (j >= 1 && !issue_pv(j - 1)) { ok = false; break; }
        }
        if (ok && n_tiles > 0 && issue_pv(n_tiles - 1)) {
            if (lane == 0) mma_commit(smem_u32(&bars->o_full));
        }
        if (*abort && lane == 0) {
            mma_commit(smem_u32(&bars->drain));
            mbar_wait(smem_u32(&bars->drain), 0, nullptr, st, 0x2205, 1ll << 28);
        }
    } else {
        // ================= softmax / exchange / epilogue =================
        const uint32_t quad = warp & 3;
        const int h = (int)(quad * 32 + lane);
        const uint32_t lane_off = (quad * 32) << 16;
        const int kh = (int)rank;             // this CTA's key half of every tile
        uint8_t* sx = smem + Lay::OFF_SX;
        uint8_t* px = smem + Lay::OFF_PX;
        float* lx = (float*)(smem + Lay::OFF_LX);
        const uint32_t peer_sx = mapa(smem_u32(sx), peer);
        const uint32_t peer_px = mapa(smem_u32(px), peer);
        const uint32_t peer_lx = mapa(smem_u32(lx), peer);
        // peer barrier addresses of buffer b are base + 8 b (same layout in both CTAs)
        const uint32_t peer_sx_full0 = mapa(smem_u32(&bars->sx_full[0]), peer);
        const uint32_t peer_px_full0 = mapa(smem_u32(&bars->px_full[0]), peer);
        const uint32_t peer_sx_free0 = mapa(smem_u32(&bars->sx_free[0]), peer);
        const uint32_t peer_px_free0 = mapa(smem_u32(&bars->px_free[0]), peer);
        const uint32_t my_sx_full0 = smem_u32(&bars->sx_full[0]), my_px_full0 = smem_u32(&bars->px_full[0]);
        const uint32_t my_sx_free0 = smem_u32(&bars->sx_free[0]), my_px_free0 = smem_u32(&bars->px_free[0]);
        const uint32_t peer_lx_full = mapa(smem_u32(&bars->lx_full), peer);
        const bool arm_thread = threadIdx.x == 64;
        float m_used = -INFINITY, l = 0.f;
        bool ok = true;
        if (n_tiles > 0) {
            // ---- Q half -> TMEM (A operand of S = Q K^T) ----
            const __nv_bfloat16* qrow = a.q + t * a.q_stride_tok + (int64_t)h * a.q_stride_head + col0;
            for (int kb = 0; kb < nb; ++kb) {
                uint32_t r[32];
                const uint4* src = (const uint4*)(qrow + kb * 64);
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const uint4 v = __ldg(src + i);
                    r[4 * i] = v.x; r[4 * i + 1] = v.y; r[4 * i + 2] = v.z; r[4 * i + 3] = v.w;
                }
                tmem_st32(tmem + lane_off + TM_Q + kb * 32, r);
            }
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(&bars->q_full));
        }
        int32_t nv0 = -1, nv1 = -1;
        if (n_tiles > 0) {
            nv0 = lane < a.k_sel ? __ldg(irow + lane) : -1;
            nv1 = lane + 32 < a.k_sel ? __ldg(irow + lane + 32) : -1;
        }
        for (int j = 0; ok && j < n_tiles; ++j) {
            const uint32_t b = j & 1, ph = (j >> 1) & 1;
            const int32_t v0 = nv0, v1 = nv1;
            if (j + 1 < n_tiles) {  // prefetch the next tile's slots
                const int sl0 = (j + 1) * AT_N + lane, sl1 = sl0 + 32;
                nv0 = sl0 < a.k_sel ? __ldg(irow + sl0) : -1;
                nv1 = sl1 < a.k_sel ? __ldg(irow + sl1) : -1;
            }
            const uint32_t mlo = __ballot_sync(0xffffffffu, v0 >= 0 && v0 < ri.seqlen_k);
            const uint32_t mhi = __ballot_sync(0xffffffffu, v1 >= 0 && v1 < ri.seqlen_k);
            const uint32_t mine = kh ? mhi : mlo;      // validity of this CTA's 32 keys
            if (!wait_warp(smem_u32(&bars->s_full), j & 1, abort, st, 0x2301)) { ok = false; break; }
            tc_fence_after();
            float sa[64];
            {
                uint32_t r0[32], r1[32];
                tmem_ld32(tmem + lane_off + TM_S, r0);
                tmem_ld32(tmem + lane_off + TM_S + 32, r1);
                tmem_wait_ld();
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    sa[i] = __uint_as_float(r0[i]);
                    sa[32 + i] = __uint_as_float(r1[i]);
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(&bars->s_empty));
            // partial maximum over the tile's valid keys
            float pm = -INFINITY;
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                if ((mlo >> i) & 1u) pm = fmaxf(pm, sa[i]);
                if ((mhi >> i) & 1u) pm = fmaxf(pm, sa[32 + i]);
            }
            // send the peer's 32 partial columns and the partial max
            if (!wait_warp_cluster(my_sx_free0 + 8 * b, ph ^ 1, abort, st, 0x2302)) { ok = false; break; }
            {
                const uint32_t dst = peer_sx + b * (128 * AT_SX_PITCH) + h * AT_SX_PITCH;
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    // the peer's keys: [32, 64) for rank 0, [0, 32) for rank 1
                    uint32_t w[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) w[e] = __float_as_uint(kh ? sa[4 * c + e] : sa[32 + 4 * c + e]);
                    st_async_v4(dst + c * 16, w[0], w[1], w[2], w[3], peer_sx_full0 + 8 * b);
                }
                st_async_v4(dst + 128, __float_as_uint(pm), 0u, 0u, 0u, peer_sx_full0 + 8 * b);
            }
            // receive the peer's partials of this CTA's 32 keys
            if (!wait_warp_cluster(my_sx_full0 + 8 * b, ph, abort, st, 0x2303)) { ok = false; break; }
            if (arm_thread && j + 2 < n_tiles) mbar_arrive_expect_tx(my_sx_full0 + 8 * b, AT_SX_BYTES);
            float s32[32];
            float pm_peer;
            {
                const float4* src = (const float4*)(sx + b * (128 * AT_SX_PITCH) + h * AT_SX_PITCH);
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    const float4 v = src[c];
                    const float pv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) s32[4 * c + e] = (kh ? sa[32 + 4 * c + e] : sa[4 * c + e]) + pv[e];
                }
                pm_peer = src[8].x;
            }
            __syncwarp();
            if (lane == 0) mbar_arrive_remote(peer_sx_free0 + 8 * b);
            // shared running maximum (identical in both CTAs), lazy rescale
            const float mb = (pm == -INFINITY || pm_peer == -INFINITY) ? -INFINITY : (pm + pm_peer) * a.scale_log2;
            float alpha = 1.f;
            if (mb > m_used + 8.0f) {
                alpha = m_used == -INFINITY ? 0.f : ex2(m_used - mb);
                l *= alpha;
                m_used = mb;
            }
            uint32_t pw[16];
            {
                float rs = 0.f;
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const float p0 = ((mine >> (2 * i)) & 1u) ? ex2(fmaf(s32[2 * i], a.scale_log2, -m_used)) : 0.f;
                    const float p1 = ((mine >> (2 * i + 1)) & 1u) ? ex2(fmaf(s32[2 * i + 1], a.scale_log2, -m_used)) : 0.f;
                    rs += p0 + p1;
                    pw[i] = pack_bf16(p0, p1);
                }
                l += rs;
            }
            // send this CTA's probabilities to the peer
            if (!wait_warp_cluster(my_px_free0 + 8 * b, ph ^ 1, abort, st, 0x2304)) { ok = false; break; }
            {
                const uint32_t dst = peer_px + b * (128 * AT_PX_PITCH) + h * AT_PX_PITCH;
#pragma unroll
                for (int c = 0; c < 4; ++c)
                    st_async_v4(dst + c * 16, pw[4 * c], pw[4 * c + 1], pw[4 * c + 2], pw[4 * c + 3], peer_px_full0 + 8 * b);
            }
            // O rescale and this CTA's P half -> TMEM once the previous P.V is done
            if (!wait_warp(smem_u32(&bars->p_free), (j & 1) ^ 1, abort, st, 0x2305)) { ok = false; break; }
            tc_fence_after();
            if (j > 0 && __any_sync(0xffffffffu, alpha != 1.f)) {
                for (int c = 0; c < 8; ++c) {
                    uint32_t r[32];
                    tmem_ld32(tmem + lane_off + TM_O + c * 32, r);
                    tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * alpha);
                    tmem_st32(tmem + lane_off + TM_O + c * 32, r);
                }
            }
            tmem_st16(tmem + lane_off + TM_P + 16 * kh, pw);
            // the peer's P half
            if (!wait_warp_cluster(my_px_full0 + 8 * b, ph, abort, st, 0x2306)) { ok = false; break; }
            if (arm_thread && j + 2 < n_tiles) mbar_arrive_expect_tx(my_px_full0 + 8 * b, AT_PX_BYTES);
            {
                uint32_t r[16];
                const uint4* src = (const uint4*)(px + b * (128 * AT_PX_PITCH) + h * AT_PX_PITCH);
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const uint4 v = src[c];
                    r[4 * c] = v.x; r[4 * c + 1] = v.y; r[4 * c + 2] = v.z; r[4 * c + 3] = v.w;
                }
                tmem_st16(tmem + lane_off + TM_P + 16 * (1 - kh), r);
            }
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(smem_u32(&bars->p_full));
                mbar_arrive_remote(peer_px_free0 + 8 * b);
            }
        }
        // ---- row sums of both halves ----
        float l_tot = 0.f;
        if (ok && n_tiles > 0) {
            st_async_b32(peer_lx + h * 4, __float_as_uint(l), peer_lx_full);
            if (wait_warp_cluster(smem_u32(&bars->lx_full), 0, abort, st, 0x2307)) l_tot = l + lx[h];
            else ok = false;
        }
        // ---- epilogue: O / l -> bf16 ----
        __nv_bfloat16* orow = a.out + t * a.out_stride_tok + (int64_t)h * a.out_stride_head + dv0;
        const bool have_o = ok && n_tiles > 0 && wait_warp(smem_u32(&bars->o_full), 0, abort, st, 0x2308);
        if (have_o) tc_fence_after();
        const float inv = l_tot > 0.f ? 1.0f / l_tot : 0.f;
        for (int c = 0; c < 8; ++c) {
            uint32_t r[32];
            if (have_o) {
                tmem_ld32(tmem + lane_off + TM_O + c * 32, r);
                tmem_wait_ld();
            }
            uint4* dst = (uint4*)(orow + c * 32);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                uint4 w;
                if (have_o) {
                    w.x = pack_bf16(__uint_as_float(r[8 * i + 0]) * inv, __uint_as_float(r[8 * i + 1]) * inv);
                    w.y = pack_bf16(__uint_as_float(r[8 * i + 2]) * inv, __uint_as_float(r[8 * i + 3]) * inv);
                    w.z = pack_bf16(__uint_as_float(r[8 * i + 4]) * inv, __uint_as_float(r[8 * i + 5]) * inv);
                    w.w = pack_bf16(__uint_as_float(r[8 * i + 6]) * inv, __uint_as_float(r[8 * i + 7]) * inv);
                } else {
                    w = make_uint4(0u, 0u, 0u, 0u);
                }
                dst[i] = w;
            }
        }
        if (rank == 0 && a.lse)
            a.lse[t * 128 + h] = (have_o && l_tot > 0.f) ? (m_used + __log2f(l_tot)) * 0.69314718055994531f : -INFINITY;
    }
    tc_fence_before();
    __syncwarp();
    cluster_sync();  // no DSMEM traffic may target a CTA that has exited
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, 512);
}

template <int NST, bool VSEP>
static bool launch_attn_tc_t(const AttnTcArgs& a, cudaStream_t s) {
    using Lay = AtLayout<NST, VSEP>;
    if (cudaFuncSetAttribute(attn_tc_kernel<NST, VSEP>, cudaFuncAttributeMaxDynamicSharedMemorySize, Lay::SMEM) !=
        cudaSuccess)
        return false;
    attn_tc_kernel<NST, VSEP><<<(unsigned)(2 * a.total_q), 192, Lay::SMEM, s>>>(a);
    return cudaGetLastError() == cudaSuccess;
}

bool launch_attn_tc(const AttnTcArgs& a, cudaStream_t s) {
    if (a.total_q <= 0) return true;
    return a.v_separate ? launch_attn_tc_t<2, true>(a, s) : launch_attn_tc_t<4, false>(a, s);
}

}  // namespace dsa
