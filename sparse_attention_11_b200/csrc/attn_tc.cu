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
// Softmax split.  Per 64-key tile each CTA holds a partial S for all 128
// heads and all 64 keys.  Rank r finishes keys [32r, 32r+32): it sends the
// other 32 partial columns to its peer and receives the peer's partials of
// its own keys (st.async into the peer's shared memory, byte-counted on the
// peer's mbarrier).  Both CTAs use the same running maximum: the sum of the
// two partial maxima of the tile, an upper bound of the true maximum that
// both form from the exchanged data, with lazy rescaling (moved only when it
// grows by more than 2^8).  Each CTA writes the bf16 probabilities of its
// keys into its own P tile (st.shared) and into the peer's (st.async), so
// both hold the full 128 x 64 P (the A operand of O += P V, in shared memory).
// Row sums are combined once at the end.
//
// Pipelining.  Stage A (read S, send the partial) and stage B (combine,
// probabilities, write P) run in separate warps, so consecutive tiles overlap;
// the MMA warp issues greedily: PV(u) as soon as P(u) is complete, else S(t)
// as soon as its K/V stage is full and the S buffer is free.
// P tiles are double-buffered and released by a tcgen05.commit that arrives
// on the p_free barrier of both CTAs (PV(t) done in both), so stage B waits
// for PV(t-2), and for PV(t-1) only when the running maximum moves.
//
// Gathers: seven producer warps copy the selected rows with 16-byte
// cp.async, 4 rows x 128 bytes per warp instruction, into the
// 128-byte-swizzled tile layout the MMA reads (row r's 16-byte chunk c at
// chunk c ^ (r & 7)).  Gather throughput grows with the number of issuing
// warps, so the producers are many and small (setmaxnreg moves their
// registers to the softmax warps).
//
// Tensor memory per CTA: O [0,256)  S [256,384) (two buffers)  Q [384,512)
// (four 64-column blocks; rank 1's fifth block, the rope part, is read from
// shared memory by SS MMAs).
// Warps: 0-6 producers, 7 MMA issuer (+TMEM owner), 8-15 softmax / exchange /
// epilogue: an A and a B warp per TMEM lane quadrant (thread <-> head).
#include "dsa_kernels.h"

namespace dsa {

// Exchange layout of the partial scores and of P: 16-byte chunk c (4 fp32
// partials, or 8 bf16 probabilities) of head row h at c*2048 + h*16.  A warp's
// stores of one chunk then cover 512 contiguous bytes, which the cluster's
// shared-memory path moves several times faster than 32 scattered 16-byte
// pieces; for P it is also the no-swizzle K-major operand layout of the MMA
// (8-row x 16-byte core matrices, 128 B apart along M and 2048 B along K).
__device__ __forceinline__ uint32_t chunk_off(int h, int c) { return (uint32_t)(c * 2048 + h * 16); }
constexpr int AT_N = 64;                           // keys per tile
constexpr uint32_t AT_BLK = AT_N * 128;            // one 64-column block of a tile
constexpr uint32_t AT_KST = 5 * AT_BLK;            // K part of a stage (max 5 blocks)
constexpr uint32_t AT_VST = 4 * AT_BLK;            // V part (separate V only)
constexpr uint32_t AT_TILE128 = 128 * 128;         // a 128-row x 128-byte swizzled tile
constexpr uint32_t AT_SX_BYTES = 128 * 128 + 128 * 4;  // partial scores + partial maxima
constexpr uint32_t AT_PX_BYTES = 128 * 64;         // the peer's half of P
constexpr uint32_t TM_O = 0, TM_S = 256, TM_Q = 384;  // S: two 64-column buffers
constexpr int AT_THREADS = 512;  // 7 producer + 1 MMA + 8 softmax warps
constexpr int AT_PRODUCERS = 7;
constexpr int AT_MMA_WARP = 7;
constexpr int AT_SOFT0 = 8;     // first softmax warp (a warpgroup boundary)

template <int NST, bool VSEP, int NPB = 2, int NSX = 2>
struct AtLayout {
    static constexpr uint32_t STAGE = AT_KST + (VSEP ? AT_VST : 0);
    static constexpr uint32_t OFF_QR = NST * STAGE;           // rank 1's 5th Q block (rope), A of SS MMAs
    static constexpr uint32_t OFF_P = OFF_QR + AT_TILE128;    // [NPB] P tiles
    static constexpr uint32_t OFF_SX = OFF_P + NPB * AT_TILE128;  // [NSX] partial-score tiles
    static constexpr uint32_t OFF_PM = OFF_SX + NSX * AT_TILE128; // [NSX][128] partial maxima
    static constexpr uint32_t OFF_LX = OFF_PM + NSX * 512;        // [128] row sums for the A warps' epilogue
    static constexpr uint32_t OFF_VM = OFF_LX + 1024;            // [64] validity bits of 2048 slots
    static constexpr uint32_t OFF_BAR = OFF_VM + 256;
    static constexpr uint32_t SMEM = OFF_BAR + 256;
};

struct AtBars {
    uint64_t full[4];
    uint64_t empty[4];
    uint64_t s_full[2], s_empty[2], q_full, o_full;
    uint64_t p_full[2];   // 4 local B warps + the peer's half of P (bytes)
    uint64_t p_free[2];   // PV done in both CTAs (multicast commit)
    uint64_t sx_full[2];  // the peer's partial scores (bytes)
    uint64_t sx_free[2];  // the peer consumed the partials this CTA sent
    uint64_t lx_full, lx_loc, drain;
    uint32_t tmem_base;
    int abort;
    int max_slot;
};
static_assert(sizeof(AtBars) <= 256, "barrier block");

__device__ __forceinline__ uint32_t swz(int row, int chunk) { return (uint32_t)(row * 128 + ((chunk ^ (row & 7)) << 4)); }

template <int NST, bool VSEP, int NPB, int NSX>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(AT_THREADS, 1)
    attn_tc_kernel(const __grid_constant__ AttnTcArgs a) {
    static_assert(AT_SOFT0 % 4 == 0 && AT_PRODUCERS < AT_SOFT0, "warp roles");
    using Lay = AtLayout<NST, VSEP, NPB, NSX>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    AtBars* bars = (AtBars*)(smem + Lay::OFF_BAR);
    uint32_t* vmask = (uint32_t*)(smem + Lay::OFF_VM);
    if ((uintptr_t)smem != (uintptr_t)smem_raw) {  // the layout needs a 1024-byte aligned base
        if (threadIdx.x == 0) report(a.st, DSA_ERR_UNSUPPORTED, -3);
        return;
    }
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
    const int nb = rank ? 5 : 4;      // 64-column blocks of K held here
    const int col0 = rank ? 256 : 0;  // first K column
    const int dv0 = rank ? 256 : 0;   // first output column
    const int32_t* irow = a.idx + t * a.ld_idx;

    if (threadIdx.x == 0) {
        for (int i = 0; i < NST; ++i) {
            mbar_init(smem_u32(&bars->full[i]), AT_PRODUCERS * 32);
            mbar_init(smem_u32(&bars->empty[i]), 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(smem_u32(&bars->s_full[i]), 1);
            mbar_init(smem_u32(&bars->s_empty[i]), 8);  // 4 A + 4 B warps read every S tile
        }
        mbar_init(smem_u32(&bars->q_full), 8);
        mbar_init(smem_u32(&bars->o_full), 1);
        for (int i = 0; i < 2; ++i) {
            mbar_init(smem_u32(&bars->p_full[i]), 4);  // (only NPB of them are used)
            mbar_init(smem_u32(&bars->p_free[i]), 2);
            mbar_init(smem_u32(&bars->sx_full[i]), 1);
            mbar_init(smem_u32(&bars->sx_free[i]), 4);
        }
        mbar_init(smem_u32(&bars->lx_full), 1);
        mbar_init(smem_u32(&bars->lx_loc), 4);
        mbar_init(smem_u32(&bars->drain), 1);
        // byte counts of the first phase of every peer-filled barrier
        for (int i = 0; i < NPB; ++i) mbar_expect_tx(smem_u32(&bars->p_full[i]), AT_PX_BYTES);
        for (int i = 0; i < NSX; ++i) {
            mbar_arrive_expect_tx(smem_u32(&bars->sx_full[i]), AT_SX_BYTES);
        }
        mbar_arrive_expect_tx(smem_u32(&bars->lx_full), 128 * 4);
        bars->abort = 0;
        bars->max_slot = -1;
        fence_mbar_init();
    }
    for (int i = threadIdx.x; i < 64; i += blockDim.x) vmask[i] = 0u;
    if (warp == AT_MMA_WARP) tmem_alloc(smem_u32(&bars->tmem_base), 512);
    // the softmax warps start their Q loads now; they land during the scan
    uint4 qreg[8] = {};
    const bool q_loader = warp >= AT_SOFT0;
    const __nv_bfloat16* qrow = a.q + t * a.q_stride_tok + (int64_t)((warp & 3) * 32 + lane) * a.q_stride_head + col0;
    if (q_loader) {  // block (warp - 3) >> 2 of this head's Q half
        const uint4* src = (const uint4*)(qrow + 64 * (((int)warp - AT_SOFT0) >> 2));
#pragma unroll
        for (int i = 0; i < 8; ++i) qreg[i] = __ldg(src + i);
    }
    __syncthreads();
    // validity bits of the index row and the number of 64-slot tiles (up to
    // the last valid slot)
    {
        int m = -1;
        for (int j0 = (int)(warp * 32); j0 < a.k_sel; j0 += (int)blockDim.x) {
            const int j = j0 + (int)lane;
            const int32_t v = j < a.k_sel ? __ldg(irow + j) : -1;
            const uint32_t bits = __ballot_sync(0xffffffffu, v >= 0 && v < ri.seqlen_k);
            if (v >= 0) m = j;
            if (lane == 0 && j0 < 2048) vmask[j0 >> 5] = bits;
        }
        for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, o));
        if (lane == 0 && m >= 0) atomicMax(&bars->max_slot, m);
    }
    tc_fence_before();
    cluster_sync();  // barriers of both CTAs initialised and armed; max_slot final
    tc_fence_after();
    const uint32_t tmem = bars->tmem_base;
    const int n_tiles = (bars->max_slot + AT_N) / AT_N;

    const uint32_t s_stage0 = smem_u32(smem);
    const uint32_t s_p0 = smem_u32(smem + Lay::OFF_P);
    const uint32_t s_qr = smem_u32(smem + Lay::OFF_QR);
    if (warp < AT_PRODUCERS) {
        // ================= gather producers (7 warps) =================
        asm volatile("setmaxnreg.dec.sync.aligned.u32 40;");
        // 16 groups of 4 keys per tile; warp w takes groups w, w+7, w+14
        const int sub = (int)(lane >> 3), chunk = (int)(lane & 7);
        const int ngrp = (16 - (int)warp + AT_PRODUCERS - 1) / AT_PRODUCERS;
        int32_t nxt[3] = {-1, -1, -1};
        auto load_idx = [&](int j) {
#pragma unroll
            for (int gi = 0; gi < 3; ++gi) {
                const int slot = j * AT_N + 4 * ((int)warp + AT_PRODUCERS * gi) + sub;
                nxt[gi] = (gi < ngrp && slot < a.k_sel) ? __ldg(irow + slot) : -1;
            }
        };
        if (n_tiles > 0) load_idx(0);
        for (int j = 0; j < n_tiles; ++j) {
            const uint32_t s = j % NST;
            int32_t cur[3];
#pragma unroll
            for (int gi = 0; gi < 3; ++gi) cur[gi] = nxt[gi];
            if (j + 1 < n_tiles) load_idx(j + 1);
            if (!wait_warp(smem_u32(&bars->empty[s]), ((j / NST) & 1) ^ 1, abort, st, 0x2101)) break;
            const uint32_t kst = s_stage0 + s * Lay::STAGE;
#pragma unroll
            for (int gi = 0; gi < 3; ++gi) {
                if (gi >= ngrp) break;
                const int32_t v = cur[gi];
                if (v >= ri.seqlen_k) report(st, DSA_ERR_INDEX, t);
                const int64_t r = ri.key_base + ((v >= 0 && v < ri.seqlen_k) ? v : 0);
                const int key = 4 * ((int)warp + AT_PRODUCERS * gi) + sub;  // key of the tile
                const __nv_bfloat16* src = a.k + r * a.k_stride + col0 + chunk * 8;
                const uint32_t dst = kst + swz(key, chunk);
                for (int kb = 0; kb < nb; ++kb) cp_async16(dst + kb * AT_BLK, src + kb * 64);
                if (VSEP) {
                    const __nv_bfloat16* vs = a.v + r * a.v_stride + dv0 + chunk * 8;
#pragma unroll
                    for (int vb = 0; vb < 4; ++vb) cp_async16(dst + AT_KST + vb * AT_BLK, vs + vb * 64);
                }
            }
            cp_async_arrive(smem_u32(&bars->full[s]));
        }
        asm volatile("cp.async.wait_all;" ::: "memory");
    } else if (warp == AT_MMA_WARP) {
        // ================= MMA issuer =================
        asm volatile("setmaxnreg.dec.sync.aligned.u32 40;");
        constexpr uint32_t idesc_s = idesc_make(1, 1, false, 128, AT_N);
        constexpr uint32_t idesc_pv = idesc_make(1, 1, true, 128, 256);
        bool ok = n_tiles > 0 && wait_warp(smem_u32(&bars->q_full), 0, abort, st, 0x2201);
        // Greedy issue: PV(ju) as soon as its P tile is complete (ju < js), else
        // S(js) as soon as its K/V stage is full and the S buffer is free.
        int js = 0, ju = 0;
        long long idle0 = clock64();
        while (ok && ju < n_tiles) {
            bool done = false;
            if (ju < js) {
                const uint32_t b = ju % NPB;
                if (__all_sync(0xffffffffu, mbar_probe(smem_u32(&bars->p_full[b]), (ju / NPB) & 1))) {
                    tc_fence_after();
                    if (lane == 0) {
                        if (ju + NPB < n_tiles) mbar_expect_tx(smem_u32(&bars->p_full[b]), AT_PX_BYTES);
                        const uint32_t vb = s_stage0 + (ju % NST) * Lay::STAGE + (VSEP ? AT_KST : 0);
                        const uint32_t pb = s_p0 + b * AT_TILE128;
#pragma unroll
                        for (int ks = 0; ks < AT_N / 16; ++ks)
                            mma_bf16_ss(tmem + TM_O, sdesc_noswz(pb + ks * 4096, 2048, 128),
                                        sdesc_sw128(vb + ks * 2048, AT_BLK, 1024), idesc_pv, (ju > 0 || ks > 0) ? 1u : 0u);
                        mma_commit(smem_u32(&bars->empty[ju % NST]));
                        mma_commit_mc(smem_u32(&bars->p_free[b]), (uint16_t)3);
                    }
                    __syncwarp();
                    ++ju;
                    done = true;
                }
            }
            if (!done && js < n_tiles) {
                const uint32_t s = js % NST, sb = js & 1;
                const bool rdy = mbar_probe(smem_u32(&bars->full[s]), (js / NST) & 1) &&
                                 mbar_probe(smem_u32(&bars->s_empty[sb]), ((js >> 1) & 1) ^ 1);
                if (__all_sync(0xffffffffu, rdy)) {
                    fence_proxy_async();
                    tc_fence_after();
                    if (lane == 0) {
                        const uint32_t kst = s_stage0 + s * Lay::STAGE;
                        const uint32_t d = tmem + TM_S + 64 * sb;
                        for (int kb = 0; kb < 4; ++kb)
#pragma unroll
                            for (int ks = 0; ks < 4; ++ks)
                                mma_bf16_ts(d, tmem + TM_Q + kb * 32 + ks * 8, sdesc_sw128(kst + kb * AT_BLK + ks * 32, 16, 1024),
                                            idesc_s, (kb | ks) ? 1u : 0u);
                        if (nb == 5)  // the rope block: Q from shared memory
#pragma unroll
                            for (int ks = 0; ks < 4; ++ks)
                                mma_bf16_ss(d, sdesc_sw128(s_qr + ks * 32, 16, 1024),
                                            sdesc_sw128(kst + 4 * AT_BLK + ks * 32, 16, 1024), idesc_s, 1u);
                        mma_commit(smem_u32(&bars->s_full[sb]));
                    }
                    __syncwarp();
                    ++js;
                    done = true;
                }
            }
            if (done) {
                idle0 = clock64();
            } else {
                const long long el = clock64() - idle0;
                bool give_up = *abort != 0;
                if (!give_up && el > (1ll << 20) && *(volatile int*)&st->code == DSA_ERR_TIMEOUT) give_up = true;
                if (!give_up && el > kWaitBudget) {
                    report(st, DSA_ERR_TIMEOUT, 0x2203);
                    give_up = true;
                }
                if (__any_sync(0xffffffffu, give_up)) {
                    *abort = 1;
                    ok = false;
                }
            }
        }
        if (ok && n_tiles > 0 && lane == 0) mma_commit(smem_u32(&bars->o_full));
        if (*abort && lane == 0) {
            mma_commit(smem_u32(&bars->drain));
            mbar_wait(smem_u32(&bars->drain), 0, nullptr, st, 0x2205, 1ll << 28);
        }
    } else {
        // ================= softmax / exchange / epilogue (8 warps) =================
        // Stage-specialised: warps 8..11 ("A", one per TMEM lane quadrant) read
        // each S tile, form the row's partial maximum and send the peer's 32
        // partial columns; warps 12..15 ("B") read their own 32 columns of the
        // same tile, combine them with the peer's partials, form the
        // probabilities and write P.  Both groups run every tile concurrently.
        asm volatile("setmaxnreg.inc.sync.aligned.u32 208;");
        const uint32_t quad = warp & 3;
        const bool is_b = warp >= AT_SOFT0 + 4;
        const int h = (int)(quad * 32 + lane);
        const uint32_t lane_off = (quad * 32) << 16;
        const int kh = (int)rank;  // this CTA's key half of every tile
        uint8_t* sx = smem + Lay::OFF_SX;
        const float* pmx = (const float*)(smem + Lay::OFF_PM);
        float* lx = (float*)(smem + Lay::OFF_LX);
        const uint32_t peer_sx = mapa(smem_u32(sx), peer);
        const uint32_t peer_pm = mapa(smem_u32(smem + Lay::OFF_PM), peer);
        const uint32_t peer_p = mapa(s_p0, peer);
        const uint32_t peer_sx_full0 = mapa(smem_u32(&bars->sx_full[0]), peer);
        const uint32_t peer_sx_free0 = mapa(smem_u32(&bars->sx_free[0]), peer);
        const uint32_t peer_p_full0 = mapa(smem_u32(&bars->p_full[0]), peer);
        const uint32_t peer_lx_full = mapa(smem_u32(&bars->lx_full), peer);
        const uint32_t my_sx_full0 = smem_u32(&bars->sx_full[0]), my_sx_free0 = smem_u32(&bars->sx_free[0]);
        const uint32_t my_p_full0 = smem_u32(&bars->p_full[0]), my_p_free0 = smem_u32(&bars->p_free[0]);
        const bool arm_thread = threadIdx.x == (AT_SOFT0 + 4) * 32;
        float m_used = -INFINITY, l = 0.f;
        bool ok = true;
        if (n_tiles > 0) {
            // ---- Q half -> TMEM (A operand of S = Q K^T); the A and B warps of a
            // quadrant take alternate 64-column blocks, block (is_b) was loaded early ----
            for (int kb = is_b ? 1 : 0; kb < nb; kb += 2) {
                uint32_t r[32];
                if (kb > 1) {
                    const uint4* src = (const uint4*)(qrow + kb * 64);
#pragma unroll
                    for (int i = 0; i < 8; ++i) qreg[i] = __ldg(src + i);
                }
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    r[4 * i] = qreg[i].x; r[4 * i + 1] = qreg[i].y; r[4 * i + 2] = qreg[i].z; r[4 * i + 3] = qreg[i].w;
                }
                if (kb < 4) {
                    tmem_st32(tmem + lane_off + TM_Q + kb * 32, r);
                } else {
                    uint8_t* qr = smem + Lay::OFF_QR;
#pragma unroll
                    for (int c = 0; c < 8; ++c)
                        *(uint4*)(qr + swz(h, c)) = make_uint4(r[4 * c], r[4 * c + 1], r[4 * c + 2], r[4 * c + 3]);
                }
            }
            tmem_wait_st();
            fence_proxy_async();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(&bars->q_full));
        }
        for (int u = 0; ok && u < n_tiles; ++u) {
            const uint32_t b = u & 1, ph = (u >> 1) & 1;  // S buffer and its phase
            const uint32_t xb = u % NSX, xph = (u / NSX) & 1;  // partial-score buffer and its phase
            const uint32_t mlo = u < 32 ? vmask[2 * u] : 0u, mhi = u < 32 ? vmask[2 * u + 1] : 0u;
            if (!wait_warp(smem_u32(&bars->s_full[b]), ph, abort, st, 0x2301)) { ok = false; break; }
            tc_fence_after();
            uint32_t r0[32], r1[32];
            tmem_ld32(tmem + lane_off + TM_S + 64 * b, r0);
            tmem_ld32(tmem + lane_off + TM_S + 64 * b + 32, r1);
            tmem_wait_ld();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(&bars->s_empty[b]));
            float pm = -INFINITY;  // partial maximum of this CTA's row over the tile's valid keys
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                if ((mlo >> i) & 1u) pm = fmaxf(pm, __uint_as_float(r0[i]));
                if ((mhi >> i) & 1u) pm = fmaxf(pm, __uint_as_float(r1[i]));
            }
            if (!is_b) {
                // ---- stage A: send the peer's 32 partial columns and the partial max ----
                if (!wait_warp(my_sx_free0 + 8 * xb, xph ^ 1, abort, st, 0x2302)) { ok = false; break; }
                const uint32_t dst = peer_sx + xb * AT_TILE128;
                const uint32_t bar = peer_sx_full0 + 8 * xb;
#pragma unroll
                for (int c = 0; c < 8; ++c) {  // the peer's keys: [32,64) for rank 0, [0,32) for rank 1
                    uint32_t w[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) w[e] = kh ? r0[4 * c + e] : r1[4 * c + e];
                    st_async_v4(dst + chunk_off(h, c), w[0], w[1], w[2], w[3], bar);
                }
                st_async_b32(peer_pm + xb * 512 + h * 4, __float_as_uint(pm), bar);
                continue;
            }
            // ---- stage B: combine, probabilities, both copies of P ----
            const uint32_t msk = kh ? mhi : mlo;
            if (!wait_warp(my_sx_full0 + 8 * xb, xph, abort, st, 0x2303)) { ok = false; break; }
            if (arm_thread && u + NSX < n_tiles) mbar_arrive_expect_tx(my_sx_full0 + 8 * xb, AT_SX_BYTES);
            float s32[32];
            {
                const uint8_t* rowp = sx + xb * AT_TILE128;
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    const float4 v = *(const float4*)(rowp + chunk_off(h, c));
                    const float pv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        s32[4 * c + e] = __uint_as_float(kh ? r1[4 * c + e] : r0[4 * c + e]) + pv[e];
                }
            }
            const float pm_peer = pmx[xb * 128 + h];
            __syncwarp();
            if (lane == 0) mbar_arrive_remote(peer_sx_free0 + 8 * xb);
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
                float rs0 = 0.f, rs1 = 0.f;
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const float p0 = ((msk >> (2 * i)) & 1u) ? ex2(fmaf(s32[2 * i], a.scale_log2, -m_used)) : 0.f;
                    const float p1 = ((msk >> (2 * i + 1)) & 1u) ? ex2(fmaf(s32[2 * i + 1], a.scale_log2, -m_used)) : 0.f;
                    rs0 += p0;
                    rs1 += p1;
                    pw[i] = pack_bf16(p0, p1);
                }
                l += rs0 + rs1;
            }
            // P tile pb is free once PV(u - NPB) is done in both CTAs
            const uint32_t pb = u % NPB;
            if (!wait_warp(my_p_free0 + 8 * pb, ((u / NPB) & 1) ^ 1, abort, st, 0x2304)) { ok = false; break; }
            {
                uint8_t* prow = smem + Lay::OFF_P + pb * AT_TILE128;
                const uint32_t pdst = peer_p + pb * AT_TILE128;
                const uint32_t bar = peer_p_full0 + 8 * pb;
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const int c = 4 * kh + q;
                    *(uint4*)(prow + chunk_off(h, c)) = make_uint4(pw[4 * q], pw[4 * q + 1], pw[4 * q + 2], pw[4 * q + 3]);
                    st_async_v4(pdst + chunk_off(h, c), pw[4 * q], pw[4 * q + 1], pw[4 * q + 2], pw[4 * q + 3], bar);
                }
            }
            if (u > 0 && __any_sync(0xffffffffu, alpha != 1.f)) {
                // O may be rescaled only between PV(u-1) and PV(u)
                const int w = u - 1;
                if (!wait_warp(my_p_free0 + 8 * (w % NPB), (w / NPB) & 1, abort, st, 0x2305)) { ok = false; break; }
                tc_fence_after();
                for (int c = 0; c < 8; ++c) {
                    uint32_t r[32];
                    const uint32_t ta = tmem + lane_off + TM_O + c * 32;
                    tmem_ld32(ta, r);
                    tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * alpha);
                    tmem_st32(ta, r);
                }
                tmem_wait_st();
            }
            fence_proxy_async();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(my_p_full0 + 8 * pb);
        }
        // ---- row sums: the B warps combine this CTA's sum with the peer's ----
        float l_tot = 0.f;
        if (is_b && ok && n_tiles > 0) {
            // the peer's sum lands in partial-max buffer n_tiles % NSX, free once the
            // peer has consumed this CTA's partials of tile n_tiles - NSX
            const uint32_t bf = n_tiles % NSX;
            ok = wait_warp(my_sx_free0 + 8 * bf, ((n_tiles / NSX) & 1) ^ 1, abort, st, 0x2307);
            if (ok) st_async_b32(peer_pm + bf * 512 + h * 4, __float_as_uint(l), peer_lx_full);
            if (ok && wait_warp(smem_u32(&bars->lx_full), 0, abort, st, 0x2308)) l_tot = l + pmx[bf * 128 + h];
            else ok = false;
            lx[h] = ok ? l_tot : 0.f;
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(&bars->lx_loc));
        }
        if (!is_b && n_tiles > 0) {
            // the A warps take the other half of the epilogue columns
            if (wait_warp(smem_u32(&bars->lx_loc), 0, abort, st, 0x2306)) l_tot = lx[h];
            else ok = false;
        }
        // ---- epilogue: O / l -> bf16 (this warp's 128 output columns) ----
        const int ocol = is_b ? 0 : 128;
        __nv_bfloat16* orow = a.out + t * a.out_stride_tok + (int64_t)h * a.out_stride_head + dv0 + ocol;
        const bool have_o = ok && n_tiles > 0 && l_tot > 0.f && wait_warp(smem_u32(&bars->o_full), 0, abort, st, 0x2309);
        if (have_o) tc_fence_after();
        const float inv = have_o ? 1.0f / l_tot : 0.f;
        for (int c = 0; c < 4; ++c) {
            uint32_t r[32];
            if (__any_sync(0xffffffffu, have_o)) {
                tmem_ld32(tmem + lane_off + TM_O + ocol + c * 32, r);
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
        if (rank == 0 && is_b && a.lse)
            a.lse[t * 128 + h] = have_o ? (m_used + __log2f(l_tot)) * 0.69314718055994531f : -INFINITY;
    }
    tc_fence_before();
    __syncwarp();
    cluster_sync();  // no DSMEM traffic may target a CTA that has exited
    tc_fence_after();
    if (warp == AT_MMA_WARP) tmem_dealloc(tmem, 512);
}

template <int NST, bool VSEP, int NPB, int NSX>
static bool launch_attn_tc_t(const AttnTcArgs& a, cudaStream_t s) {
    using Lay = AtLayout<NST, VSEP, NPB, NSX>;
    static_assert(Lay::SMEM <= 232448, "shared memory budget");
    if (cudaFuncSetAttribute(attn_tc_kernel<NST, VSEP, NPB, NSX>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             Lay::SMEM) != cudaSuccess)
        return false;
    attn_tc_kernel<NST, VSEP, NPB, NSX><<<(unsigned)(2 * a.total_q), AT_THREADS, Lay::SMEM, s>>>(a);
    return cudaGetLastError() == cudaSuccess;
}

#ifndef DSA_ATTN_NST
#define DSA_ATTN_NST 3
#define DSA_ATTN_NPB 2
#define DSA_ATTN_NSX 1
#endif

bool launch_attn_tc(const AttnTcArgs& a, cudaStream_t s) {
    if (a.total_q <= 0) return true;
    return a.v_separate ? launch_attn_tc_t<2, true, 2, 2>(a, s)
                        : launch_attn_tc_t<DSA_ATTN_NST, false, DSA_ATTN_NPB, DSA_ATTN_NSX>(a, s);
}

}  // namespace dsa
