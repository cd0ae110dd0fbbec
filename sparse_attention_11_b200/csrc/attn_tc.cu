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
// Persistence.  The grid holds as many CTA pairs as can be resident at once;
// pair p takes the queries p, p + P, p + 2P, ...  The K/V stages, S buffers,
// P tiles and exchange buffers run as rings over the pair's whole sequence of
// 64-key tiles, across query boundaries, so the gathers and MMAs of one query
// overlap the start and the end of its neighbours.  Per query the producers
// publish the index row's validity bits and tile count (a two-slot ring), the
// softmax warps load the next Q once the last S of the previous query has
// completed, and the first PV of a query waits until the previous query's
// epilogue has read O out of tensor memory.
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
// Row sums are combined once per query.
//
// Pipelining.  Stage A (read S, send the partial) and stage B (combine,
// probabilities, write P) run in separate warps, so consecutive tiles overlap;
// the MMA warp issues greedily from two cursors: PV(u) as soon as P(u) is
// complete, else S(t) as soon as its K/V stage is full and the S accumulators
// are free.  A tcgen05.mma takes about 50 cycles to issue from one thread,
// which makes the 16-20 N=64 MMAs of an S tile issue-bound; so two warps issue
// an S tile, each half of the contraction blocks into its own accumulator, and
// the softmax warps add the two.  P tiles are triple-buffered and released by a tcgen05.commit that
// arrives on the p_free barrier of both CTAs (PV(t) done in both), so stage B
// waits for PV(t-3), and for PV(t-1) only when the running maximum moves.
// The P exchange also keeps the two CTAs' PVs within three tiles of each
// other (a CTA's half of P(t+3) waits for PV(t) in both), which the
// two-arrival p_free barrier relies on.
//
// Gathers: six producer warps copy the selected rows with 16-byte
// cp.async, 4 rows x 128 bytes per warp instruction, into the
// 128-byte-swizzled tile layout the MMA reads (row r's 16-byte chunk c at
// chunk c ^ (r & 7)).  Gather throughput grows with the number of issuing
// warps, so the producers are many and small (setmaxnreg moves their
// registers to the softmax warps).
//
// Tensor memory per CTA: O [0,256)  S [256,384) (two partial accumulators)
// Q [384,512) (four 64-column blocks; rank 1's fifth block, the rope part, is
// read from shared memory by SS MMAs).
// Warps: 0-5 producers, 6 second S issuer, 7 MMA issuer (+TMEM owner), 8-15
// softmax / exchange / epilogue: an A and a B warp per TMEM lane quadrant
// (thread <-> head).
#include "dsa_kernels.h"

namespace dsa {

// Exchange layout of the partial scores and of P: 16-byte chunk c (4 fp32
// partials, or 8 bf16 probabilities) of head row h at c*2048 + h*16.  A warp's
// stores of one chunk then cover 512 contiguous bytes, which the cluster's
// shared-memory path moves several times faster than 32 scattered 16-byte
// pieces; for P it is also the no-swizzle K-major operand layout of the MMA
// (8-row x 16-byte core matrices, 128 B apart along M and 2048 B along K).
__device__ __forceinline__ uint32_t chunk_off(int h, int c) { return (uint32_t)(c * 2048 + h * 16); }
#ifndef DSA_ATTN_EPI_STAGE
#define DSA_ATTN_EPI_STAGE 1
#endif
constexpr int AT_N = 64;                           // keys per tile
constexpr uint32_t AT_BLK = AT_N * 128;            // one 64-column block of a tile
constexpr uint32_t AT_KST = 5 * AT_BLK;            // K part of a stage (max 5 blocks)
constexpr uint32_t AT_VST = 4 * AT_BLK;            // V part (separate V only)
constexpr uint32_t AT_TILE128 = 128 * 128;         // a 128-row x 128-byte tile
constexpr uint32_t AT_SX_BYTES = 128 * 128 + 128 * 4;  // partial scores + partial maxima
constexpr uint32_t AT_PX_BYTES = 128 * 64;         // the peer's half of P
constexpr uint32_t AT_LX_BYTES = 128 * 4;          // the peer's row sums
constexpr uint32_t TM_O = 0, TM_S = 256, TM_Q = 384;  // S: two 64-column partial accumulators
constexpr int AT_THREADS = 512;  // 6 producer + 2 MMA + 8 softmax warps
constexpr int AT_PRODUCERS = 6;
constexpr int AT_MMA2_WARP = 6;  // issues the second half of every S tile
constexpr int AT_MMA_WARP = 7;
constexpr int AT_SOFT0 = 8;      // first softmax warp (a warpgroup boundary)
// Register split (setmaxnreg): warpgroup 0 (producers 0-3) and warpgroup 1
// (producers 4-5 and the two MMA warps) give registers to the softmax
// warpgroups.  setmaxnreg.inc draws only on the registers the block was
// launched with, so the split must fit the launch total (threads x registers
// per thread at launch), or the softmax warps wait forever; the launcher
// checks the compiled count before every launch.
constexpr int AT_REGS_WG0 = 40;
constexpr int AT_REGS_WG1 = 56;
constexpr int AT_REGS_SOFT = 208;
constexpr int AT_REGS_SPLIT = 128 * AT_REGS_WG0 + 128 * AT_REGS_WG1 + (AT_THREADS - 256) * AT_REGS_SOFT;
static_assert(AT_SOFT0 == 8, "the register split assumes two producer/MMA warpgroups");
static_assert(AT_REGS_SPLIT <= ((65536 / AT_THREADS) & ~7) * AT_THREADS, "register split above the launch total");
constexpr int AT_SCAN_ROUNDS = (2048 / 32 + AT_PRODUCERS - 1) / AT_PRODUCERS;  // index-row words per producer warp
constexpr int AT_NTAB = 8;       // tile counts of the queries between the PV and the S cursor

template <int NST, bool VSEP, int NPB = 2, int NSX = 1>
struct AtLayout {
    static constexpr uint32_t STAGE = AT_KST + (VSEP ? AT_VST : 0);
    static constexpr uint32_t OFF_QR = NST * STAGE;               // rank 1's 5th Q block (rope), A of SS MMAs
    static constexpr uint32_t OFF_P = OFF_QR + AT_TILE128;        // [NPB] P tiles
    static constexpr uint32_t OFF_SX = OFF_P + NPB * AT_TILE128;  // [NSX] partial-score tiles
    static constexpr uint32_t OFF_PM = OFF_SX + NSX * AT_TILE128; // [NSX][128] partial maxima
    static constexpr uint32_t OFF_LX = OFF_PM + NSX * 512;        // [128] combined row sums (B -> A warps)
    static constexpr uint32_t OFF_LXR = OFF_LX + 512;             // [128] the peer's row sums
    static constexpr uint32_t OFF_VM = OFF_LXR + 512;             // [2][64] validity bits of 2048 slots
    static constexpr uint32_t OFF_INFO = OFF_VM + 512;            // [2][8] last used slot per producer warp, [8] tile counts
    static constexpr uint32_t OFF_BAR = OFF_INFO + 128;
    // epilogue staging: per softmax warp 32 rows x 64 output columns (bf16),
    // so that the output stores cover whole 128-byte lines; with three P
    // tiles, 32 rows x 32 columns (64-byte segments) to make room
    static constexpr bool EPI_STAGE = !VSEP && DSA_ATTN_EPI_STAGE;
    static constexpr int EPI_COLS = NPB >= 3 ? 32 : 64;
    static constexpr uint32_t EPI_WARP_BYTES = 32 * EPI_COLS * 2;
    static constexpr uint32_t OFF_EPI = OFF_BAR + 512;
    static constexpr uint32_t SMEM = OFF_EPI + (EPI_STAGE ? 8 * EPI_WARP_BYTES : 0);
};

struct AtBars {
    uint64_t full[4];
    uint64_t empty[4];
    uint64_t s_full, s_empty;  // the S tile (both issuers committed) / read by the 8 softmax warps
    uint64_t s_go;             // the second issuer may issue its half of the next S tile
    uint64_t q_full;         // Q of the next query with tiles is in place (4 A warps)
    uint64_t o_full;         // all PVs of a query done
    uint64_t o_free;         // its epilogue has read O (8 softmax warps)
    uint64_t p_full[3];      // 4 local B warps + the peer's half of P (bytes)
    uint64_t p_free[3];      // PV done in both CTAs (multicast commit)
    uint64_t sx_full[2];     // the peer's partial scores (bytes)
    uint64_t sx_free[2];     // the peer consumed the partials this CTA sent
    uint64_t lx_full;        // the peer's row sums (bytes)
    uint64_t lx_loc;         // the B warps combined the row sums (for the A warps)
    uint64_t drain;
    uint64_t info_full[2];   // query info published (7 producer warps)
    uint64_t info_empty[2];  // query info consumed (MMA warp + 8 softmax warps)
    uint64_t drain2;
    int go[2];  // stage of the S tile announced on s_go, -1: no more tiles
    uint32_t tmem_base;
    int abort;
};
static_assert(sizeof(AtBars) <= 512, "barrier block");

__device__ __forceinline__ uint32_t swz(int row, int chunk) { return (uint32_t)(row * 128 + ((chunk ^ (row & 7)) << 4)); }

template <int NST, bool VSEP, int NPB, int NSX>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(AT_THREADS, 1)
    attn_tc_kernel(const __grid_constant__ AttnTcArgs a) {
    static_assert(AT_SOFT0 % 4 == 0 && AT_PRODUCERS < AT_SOFT0, "warp roles");
    static_assert(NST >= 1 && NST <= 4 && NPB >= 1 && NPB <= 3 && NSX >= 1 && NSX <= 2, "barrier arrays");
    using Lay = AtLayout<NST, VSEP, NPB, NSX>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    AtBars* bars = (AtBars*)(smem + Lay::OFF_BAR);
    uint32_t* vmask = (uint32_t*)(smem + Lay::OFF_VM);
    int* pmax = (int*)(smem + Lay::OFF_INFO);  // [2][8]
    int* ntab = pmax + 16;                      // [AT_NTAB]
    if ((uintptr_t)smem != (uintptr_t)smem_raw) {  // the layout needs a 1024-byte aligned base
        if (threadIdx.x == 0) report(a.st, DSA_ERR_UNSUPPORTED, -3);
        return;
    }
    const uint32_t warp = warp_id(), lane = lane_id();
    const uint32_t rank = cluster_ctarank(), peer = rank ^ 1u;
    StatusHdr* st = a.st;
    volatile int* abort = &bars->abort;

    // queries of this pair: t = row_begin + pair + i * npairs
    const int64_t pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
    const int64_t nq = pair < a.row_count ? (a.row_count - pair + npairs - 1) / npairs : 0;
    const int nb = rank ? 5 : 4;      // 64-column blocks of K held here
    const int col0 = rank ? 256 : 0;  // first K column
    const int dv0 = rank ? 256 : 0;   // first output column

    if (threadIdx.x == 0) {
        for (int i = 0; i < NST; ++i) {
            mbar_init(smem_u32(&bars->full[i]), AT_PRODUCERS * 32);
            mbar_init(smem_u32(&bars->empty[i]), 1);
        }
        mbar_init(smem_u32(&bars->s_full), 2);   // one commit per issuer
        mbar_init(smem_u32(&bars->s_empty), 8);  // 4 A + 4 B warps read every S tile
        mbar_init(smem_u32(&bars->s_go), 1);
        mbar_init(smem_u32(&bars->drain2), 1);
        for (int i = 0; i < 3; ++i) {
            mbar_init(smem_u32(&bars->p_full[i]), 4);   // (only NPB of them are used)
            mbar_init(smem_u32(&bars->p_free[i]), 2);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(smem_u32(&bars->sx_full[i]), 1);
            mbar_init(smem_u32(&bars->sx_free[i]), 4);
            mbar_init(smem_u32(&bars->info_full[i]), AT_PRODUCERS);
            mbar_init(smem_u32(&bars->info_empty[i]), 9);
        }
        mbar_init(smem_u32(&bars->q_full), 4);
        mbar_init(smem_u32(&bars->o_full), 1);
        mbar_init(smem_u32(&bars->o_free), 8);
        mbar_init(smem_u32(&bars->lx_full), 1);
        mbar_init(smem_u32(&bars->lx_loc), 4);
        mbar_init(smem_u32(&bars->drain), 1);
        // byte counts of the first phase of every peer-filled barrier; each
        // later phase is armed once the one before it has completed
        for (int i = 0; i < NPB; ++i) mbar_expect_tx(smem_u32(&bars->p_full[i]), AT_PX_BYTES);
        for (int i = 0; i < NSX; ++i) mbar_arrive_expect_tx(smem_u32(&bars->sx_full[i]), AT_SX_BYTES);
        mbar_arrive_expect_tx(smem_u32(&bars->lx_full), AT_LX_BYTES);
        bars->abort = 0;
        fence_mbar_init();
    }
    if (warp == AT_MMA_WARP) tmem_alloc(smem_u32(&bars->tmem_base), 512);
    tc_fence_before();
    cluster_sync();  // barriers of both CTAs initialised and armed
    tc_fence_after();
    const uint32_t tmem = bars->tmem_base;

    const uint32_t s_stage0 = smem_u32(smem);
    const uint32_t s_p0 = smem_u32(smem + Lay::OFF_P);
    const uint32_t s_qr = smem_u32(smem + Lay::OFF_QR);
    // Half hf of the S tile of stage s: K-blocks 2hf, 2hf+1 (Q from TMEM) and, on
    // rank 1, K-steps 2hf, 2hf+1 of the rope block (Q from shared memory), into
    // accumulator hf.  Issued by one thread.
    auto s_half = [&](int hf, uint32_t s) {
        constexpr uint32_t idesc_s = idesc_make(1, 1, false, 128, AT_N);
        const uint32_t kst = s_stage0 + s * Lay::STAGE;
        const uint32_t d = tmem + TM_S + 64 * hf;
#pragma unroll
        for (int k2 = 0; k2 < 2; ++k2) {
            const int kb = 2 * hf + k2;
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
                mma_bf16_ts(d, tmem + TM_Q + kb * 32 + ks * 8, sdesc_sw128(kst + kb * AT_BLK + ks * 32, 16, 1024), idesc_s,
                            (k2 | ks) ? 1u : 0u);
        }
        if (nb == 5)
#pragma unroll
            for (int k2 = 0; k2 < 2; ++k2) {
                const int ks = 2 * hf + k2;
                mma_bf16_ss(d, sdesc_sw128(s_qr + ks * 32, 16, 1024), sdesc_sw128(kst + 4 * AT_BLK + ks * 32, 16, 1024),
                            idesc_s, 1u);
            }
    };
    if (warp < AT_PRODUCERS) {
        // ================= gather producers (6 warps) =================
        if (warp < 4) asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(AT_REGS_WG0));
        else asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(AT_REGS_WG1));
        // 16 groups of 4 keys per tile; warp w takes groups w, w+7, w+14
        const int sub = (int)(lane >> 3), chunk = (int)(lane & 7);
        const int ngrp = (16 - (int)warp + AT_PRODUCERS - 1) / AT_PRODUCERS;
        uint32_t g = 0;  // tile of the pair's whole sequence
        bool ok = true;
        for (int64_t qi = 0; ok && qi < nq; ++qi) {
            const int64_t t = a.row_begin + pair + qi * npairs;
            const RowInfo ri = row_info(a.sv, t);
            const int32_t* irow = a.idx + t * a.ld_idx;
            const uint32_t slot = (uint32_t)(qi & 1);
            // ---- query info: validity bits of the index row, last used slot ----
            if (!wait_warp(smem_u32(&bars->info_empty[slot]), (uint32_t)((qi >> 1) & 1) ^ 1u, abort, st, 0x2102)) {
                ok = false;
                break;
            }
            int m = -1;
            {
                int32_t v[AT_SCAN_ROUNDS];
#pragma unroll
                for (int r = 0; r < AT_SCAN_ROUNDS; ++r) {
                    const int j = ((int)warp + AT_PRODUCERS * r) * 32 + (int)lane;
                    v[r] = (ri.ok && j < a.k_sel) ? __ldg(irow + j) : -1;
                }
#pragma unroll
                for (int r = 0; r < AT_SCAN_ROUNDS; ++r) {
                    const int w = (int)warp + AT_PRODUCERS * r;  // 32-slot word of the row
                    const uint32_t bits = __ballot_sync(0xffffffffu, v[r] >= 0 && v[r] < ri.seqlen_k);
                    if (v[r] >= 0) m = w * 32 + (int)lane;
                    if (lane == 0 && w < 64) vmask[slot * 64 + w] = bits;
                }
                for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, o));
            }
            if (!ri.ok && warp == 0 && lane == 0 && rank == 0) report(st, DSA_ERR_INDEX, t);
            if (lane == 0) {
                pmax[slot * 8 + warp] = m;
                mbar_arrive(smem_u32(&bars->info_full[slot]));
            }
            if (!wait_warp(smem_u32(&bars->info_full[slot]), (uint32_t)((qi >> 1) & 1), abort, st, 0x2103)) {
                ok = false;
                break;
            }
            int mx = -1;
#pragma unroll
            for (int w = 0; w < AT_PRODUCERS; ++w) mx = max(mx, pmax[slot * 8 + w]);
            const int n_tiles = (mx + AT_N) / AT_N;
            // ---- pull the next query's index row and Q rows into L2 while this
            // query's tiles run (its scan and Q load then hit L2) ----
            if (qi + 1 < nq) {
                const int64_t tn = t + npairs;
                if (warp == 0) {
                    const char* ir = (const char*)(a.idx + tn * a.ld_idx);
                    for (int off = (int)lane * 128; off < a.k_sel * 4; off += 32 * 128) prefetch_l2(ir + off);
                } else if (warp <= 4) {
                    const int hh = (int)(warp - 1) * 32 + (int)lane;
                    const char* qr =
                        (const char*)(a.q + (tn - a.row_begin) * a.q_stride_tok + (int64_t)hh * a.q_stride_head + col0);
                    for (int kb = 0; kb < nb; ++kb) prefetch_l2(qr + kb * 128);
                }
            }
            // ---- the query's tiles ----
            int32_t nxt[3] = {-1, -1, -1};
            auto load_idx = [&](int j) {
#pragma unroll
                for (int gi = 0; gi < 3; ++gi) {
                    const int sj = j * AT_N + 4 * ((int)warp + AT_PRODUCERS * gi) + sub;
                    nxt[gi] = (gi < ngrp && sj < a.k_sel) ? __ldg(irow + sj) : -1;
                }
            };
            if (n_tiles > 0) load_idx(0);
            for (int j = 0; j < n_tiles; ++j, ++g) {
                const uint32_t s = g % NST;
                int32_t cur[3];
#pragma unroll
                for (int gi = 0; gi < 3; ++gi) cur[gi] = nxt[gi];
                if (j + 1 < n_tiles) load_idx(j + 1);
                if (!wait_warp(smem_u32(&bars->empty[s]), ((g / NST) & 1) ^ 1, abort, st, 0x2101)) {
                    ok = false;
                    break;
                }
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
        }
        asm volatile("cp.async.wait_all;" ::: "memory");
    } else if (warp == AT_MMA_WARP) {
        // ================= MMA issuer =================
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(AT_REGS_WG1));
        constexpr uint32_t idesc_pv = idesc_make(1, 1, true, 128, 256);
        // Two cursors over the pair's tile sequence.  S cursor: query qs (ns
        // tiles once its info is read, else -1), tile js, sequence tile gs,
        // nqs queries with tiles begun.  PV cursor: query-with-tiles nqu, tile
        // ju, sequence tile gu; tile counts of begun queries are kept in ntab.
        int64_t qs = 0;
        int js = 0, ns = -1, ju = 0;
        uint32_t gs = 0, nqs = 0, gu = 0, nqu = 0;
        bool ok = true;
        long long idle0 = clock64();
        while (ok && (qs < nq || nqu < nqs)) {
            bool done = false;
            // ---- PV cursor (S(gu) issued, so its query has begun) ----
            if (gu < gs) {
                const int nu = ntab[nqu % AT_NTAB];
                const uint32_t b = gu % NPB;
                bool rdy = mbar_probe(smem_u32(&bars->p_full[b]), (gu / NPB) & 1);
                if (ju == 0 && nqu > 0) rdy = rdy && mbar_probe(smem_u32(&bars->o_free), (nqu - 1) & 1);
                if (__all_sync(0xffffffffu, rdy)) {
                    tc_fence_after();
                    if (lane == 0) {
                        mbar_expect_tx(smem_u32(&bars->p_full[b]), AT_PX_BYTES);  // its next phase
                        const uint32_t vb = s_stage0 + (gu % NST) * Lay::STAGE + (VSEP ? AT_KST : 0);
                        const uint32_t pb = s_p0 + b * AT_TILE128;
#pragma unroll
                        for (int ks = 0; ks < AT_N / 16; ++ks)
                            mma_bf16_ss(tmem + TM_O, sdesc_noswz(pb + ks * 4096, 2048, 128),
                                        sdesc_sw128(vb + ks * 2048, AT_BLK, 1024), idesc_pv, (ju > 0 || ks > 0) ? 1u : 0u);
                        mma_commit(smem_u32(&bars->empty[gu % NST]));
                        mma_commit_mc(smem_u32(&bars->p_free[b]), (uint16_t)3);
                        if (ju + 1 == nu) mma_commit(smem_u32(&bars->o_full));
                    }
                    __syncwarp();
                    ++gu;
                    if (++ju == nu) {
                        ju = 0;
                        ++nqu;
                    }
                    done = true;
                }
            }
            // ---- S cursor ----
            if (!done && qs < nq) {
                if (ns < 0) {
                    const uint32_t slot = (uint32_t)(qs & 1);
                    if (__all_sync(0xffffffffu, mbar_probe(smem_u32(&bars->info_full[slot]), (uint32_t)((qs >> 1) & 1)))) {
                        int mx = -1;
#pragma unroll
                        for (int w = 0; w < AT_PRODUCERS; ++w) mx = max(mx, pmax[slot * 8 + w]);
                        ns = (mx + AT_N) / AT_N;
                        if (lane == 0) {
                            if (ns > 0) ntab[nqs % AT_NTAB] = ns;
                            mbar_arrive(smem_u32(&bars->info_empty[slot]));
                        }
                        __syncwarp();
                        if (ns == 0) {
                            ns = -1;
                            ++qs;
                        }
                        done = true;
                    }
                } else {
                    const uint32_t s = gs % NST;
                    bool rdy = mbar_probe(smem_u32(&bars->full[s]), (gs / NST) & 1) &&
                               mbar_probe(smem_u32(&bars->s_empty), (gs & 1) ^ 1);
                    if (js == 0) rdy = rdy && mbar_probe(smem_u32(&bars->q_full), nqs & 1);
                    if (__all_sync(0xffffffffu, rdy)) {
                        fence_proxy_async();
                        tc_fence_after();
                        if (lane == 0) {
                            // first half of S: blocks 0, 1 (+ rope K-steps 0, 1); the
                            // second issuer adds blocks 2, 3 (+ rope 2, 3) into its own
                            // accumulator
                            bars->go[gs & 1] = (int)s;
                            mbar_arrive(smem_u32(&bars->s_go));
                            s_half(0, s);
                            mma_commit(smem_u32(&bars->s_full));
                        }
                        __syncwarp();
                        ++gs;
                        if (++js == ns) {
                            js = 0;
                            ns = -1;
                            ++qs;
                            ++nqs;
                        }
                        done = true;
                    }
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
        if (ok && lane == 0) {  // no more S tiles
            bars->go[gs & 1] = -1;
            mbar_arrive(smem_u32(&bars->s_go));
        }
        if (*abort && lane == 0) {
            mma_commit(smem_u32(&bars->drain));
            mbar_wait(smem_u32(&bars->drain), 0, nullptr, st, 0x2205, 1ll << 28);
        }
    } else if (warp == AT_MMA2_WARP) {
        // ================= second S issuer =================
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(AT_REGS_WG1));
        for (uint32_t g = 0;; ++g) {
            if (!wait_warp(smem_u32(&bars->s_go), g & 1, abort, st, 0x2401)) break;
            const int s = *(volatile int*)&bars->go[g & 1];
            if (s < 0) break;
            fence_proxy_async();
            tc_fence_after();
            if (lane == 0) {
                s_half(1, (uint32_t)s);
                mma_commit(smem_u32(&bars->s_full));
            }
            __syncwarp();
        }
        if (*abort && lane == 0) {
            mma_commit(smem_u32(&bars->drain2));
            mbar_wait(smem_u32(&bars->drain2), 0, nullptr, st, 0x2405, 1ll << 28);
        }
    } else {
        // ================= softmax / exchange / epilogue (8 warps) =================
        // Stage-specialised: warps 8..11 ("A", one per TMEM lane quadrant) read
        // each S tile, form the row's partial maximum and send the peer's 32
        // partial columns; warps 12..15 ("B") read their own 32 columns of the
        // same tile, combine them with the peer's partials, form the
        // probabilities and write P.  Both groups run every tile concurrently.
        // Per query: load Q (after the previous query's last S), finish the
        // previous query (row sums, O / l), then the tiles.
        asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(AT_REGS_SOFT));
        const uint32_t quad = warp & 3;
        const bool is_b = warp >= AT_SOFT0 + 4;
        const int h = (int)(quad * 32 + lane);
        const uint32_t lane_off = (quad * 32) << 16;
        const int kh = (int)rank;  // this CTA's key half of every tile
        uint8_t* sx = smem + Lay::OFF_SX;
        const float* pmx = (const float*)(smem + Lay::OFF_PM);
        float* lx = (float*)(smem + Lay::OFF_LX);
        const float* lxr = (const float*)(smem + Lay::OFF_LXR);
        const uint32_t peer_sx = mapa(smem_u32(sx), peer);
        const uint32_t peer_pm = mapa(smem_u32(smem + Lay::OFF_PM), peer);
        const uint32_t peer_lxr = mapa(smem_u32(smem + Lay::OFF_LXR), peer);
        const uint32_t peer_p = mapa(s_p0, peer);
        const uint32_t peer_sx_full0 = mapa(smem_u32(&bars->sx_full[0]), peer);
        const uint32_t peer_sx_free0 = mapa(smem_u32(&bars->sx_free[0]), peer);
        const uint32_t peer_p_full0 = mapa(smem_u32(&bars->p_full[0]), peer);
        const uint32_t peer_lx_full = mapa(smem_u32(&bars->lx_full), peer);
        const uint32_t my_sx_full0 = smem_u32(&bars->sx_full[0]), my_sx_free0 = smem_u32(&bars->sx_free[0]);
        const uint32_t my_p_full0 = smem_u32(&bars->p_full[0]), my_p_free0 = smem_u32(&bars->p_free[0]);
        const bool arm_thread = threadIdx.x == (AT_SOFT0 + 4) * 32;
        const int ocol = is_b ? 0 : 128;  // this warp's 128 of the CTA's 256 output columns

        // Row sums, O / l -> bf16 and lse of query t, the e-th query with tiles.
        auto epilogue = [&](int64_t t, uint32_t e, float m_used, float l) -> bool {
            float l_tot = 0.f;
            if (is_b) {
                // the peer's buffer is free: it read its previous sums before its
                // A warps sent the partials of this query's tiles
                st_async_b32(peer_lxr + h * 4, __float_as_uint(l), peer_lx_full);
                if (!wait_warp(smem_u32(&bars->lx_full), e & 1, abort, st, 0x2308)) return false;
                l_tot = l + lxr[h];
                if (arm_thread) mbar_arrive_expect_tx(smem_u32(&bars->lx_full), AT_LX_BYTES);  // its next phase
                lx[h] = l_tot;
                __syncwarp();
                if (lane == 0) mbar_arrive(smem_u32(&bars->lx_loc));
            } else {
                if (!wait_warp(smem_u32(&bars->lx_loc), e & 1, abort, st, 0x2306)) return false;
                l_tot = lx[h];
            }
            if (!wait_warp(smem_u32(&bars->o_full), e & 1, abort, st, 0x2309)) return false;
            tc_fence_after();
            const bool have_o = l_tot > 0.f;
            const float inv = have_o ? 1.0f / l_tot : 0.f;
            uint32_t r[4][32];
#pragma unroll
            for (int c = 0; c < 4; ++c) tmem_ld32(tmem + lane_off + TM_O + ocol + c * 32, r[c]);
            tmem_wait_ld();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(&bars->o_free));  // O may be overwritten now
            uint4 w[16];  // this row's 128 output columns, bf16
#pragma unroll
            for (int c = 0; c < 4; ++c)
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    w[4 * c + i].x = pack_bf16(__uint_as_float(r[c][8 * i + 0]) * inv, __uint_as_float(r[c][8 * i + 1]) * inv);
                    w[4 * c + i].y = pack_bf16(__uint_as_float(r[c][8 * i + 2]) * inv, __uint_as_float(r[c][8 * i + 3]) * inv);
                    w[4 * c + i].z = pack_bf16(__uint_as_float(r[c][8 * i + 4]) * inv, __uint_as_float(r[c][8 * i + 5]) * inv);
                    w[4 * c + i].w = pack_bf16(__uint_as_float(r[c][8 * i + 6]) * inv, __uint_as_float(r[c][8 * i + 7]) * inv);
                }
            if constexpr (Lay::EPI_STAGE && Lay::EPI_COLS == 32) {
                // through this warp's staging tile, 32 columns at a time: row =
                // lane, 16-byte chunk k of the quarter at ((k ^ ((row >> 1) & 3)) << 4);
                // read back as 8 rows x 64 bytes per instruction
                uint8_t* stg = smem + Lay::OFF_EPI + (warp - AT_SOFT0) * Lay::EPI_WARP_BYTES;
                __nv_bfloat16* obase =
                    a.out + (t - a.row_begin) * a.out_stride_tok + (int64_t)(quad * 32) * a.out_stride_head + dv0 + ocol;
#pragma unroll
                for (int qc = 0; qc < 4; ++qc) {
#pragma unroll
                    for (int k = 0; k < 4; ++k)
                        *(uint4*)(stg + lane * 64 + ((k ^ ((lane >> 1) & 3)) << 4)) = w[4 * qc + k];
                    __syncwarp();
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const int row = 8 * i + (int)(lane >> 2), k = (int)(lane & 3);
                        const uint4 v = *(const uint4*)(stg + row * 64 + ((k ^ ((row >> 1) & 3)) << 4));
                        *(uint4*)(obase + (int64_t)row * a.out_stride_head + qc * 32 + k * 8) = v;
                    }
                    __syncwarp();
                }
            } else if constexpr (Lay::EPI_STAGE) {
                // through this warp's staging tile: row = lane, 16-byte chunk k of a
                // 64-column half at ((k ^ (row & 7)) << 4); read back as 4 rows x
                // 128 bytes per instruction
                uint8_t* stg = smem + Lay::OFF_EPI + (warp - AT_SOFT0) * Lay::EPI_WARP_BYTES;
                __nv_bfloat16* obase =
                    a.out + (t - a.row_begin) * a.out_stride_tok + (int64_t)(quad * 32) * a.out_stride_head + dv0 + ocol;
#pragma unroll
                for (int half = 0; half < 2; ++half) {
#pragma unroll
                    for (int k = 0; k < 8; ++k) *(uint4*)(stg + lane * 128 + ((k ^ (lane & 7)) << 4)) = w[8 * half + k];
                    __syncwarp();
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        const int row = 4 * i + (int)(lane >> 3), k = (int)(lane & 7);
                        const uint4 v = *(const uint4*)(stg + row * 128 + ((k ^ (row & 7)) << 4));
                        *(uint4*)(obase + (int64_t)row * a.out_stride_head + half * 64 + k * 8) = v;
                    }
                    __syncwarp();
                }
            } else {
                uint4* dst = (uint4*)(a.out + (t - a.row_begin) * a.out_stride_tok + (int64_t)h * a.out_stride_head + dv0 + ocol);
#pragma unroll
                for (int i = 0; i < 16; ++i) dst[i] = w[i];
            }
            if (rank == 0 && is_b && a.lse)
                a.lse[t * 128 + h] = have_o ? (m_used + __log2f(l_tot)) * 0.69314718055994531f : -INFINITY;
            return true;
        };

        uint32_t g = 0;    // tile of the pair's whole sequence
        uint32_t nqt = 0;  // queries with tiles begun
        bool ok = true;
        bool pend = false;  // a query's epilogue is still to be done
        int64_t t_pend = 0;
        float m_pend = -INFINITY, l_pend = 0.f;
        for (int64_t qi = 0; ok && qi < nq; ++qi) {
            const int64_t t = a.row_begin + pair + qi * npairs;
            const uint32_t slot = (uint32_t)(qi & 1);
            if (!wait_warp(smem_u32(&bars->info_full[slot]), (uint32_t)((qi >> 1) & 1), abort, st, 0x2310)) {
                ok = false;
                break;
            }
            int mx = -1;
#pragma unroll
            for (int w = 0; w < AT_PRODUCERS; ++w) mx = max(mx, pmax[slot * 8 + w]);
            const int n_tiles = (mx + AT_N) / AT_N;
            if (n_tiles == 0) {  // nothing selected: zero rows, lse -inf
                __syncwarp();
                if (lane == 0) mbar_arrive(smem_u32(&bars->info_empty[slot]));
                uint4* dst = (uint4*)(a.out + (t - a.row_begin) * a.out_stride_tok + (int64_t)h * a.out_stride_head + dv0 + ocol);
#pragma unroll
                for (int i = 0; i < 16; ++i) dst[i] = make_uint4(0u, 0u, 0u, 0u);
                if (rank == 0 && is_b && a.lse) a.lse[t * 128 + h] = -INFINITY;
                continue;
            }
            // ---- Q of this query -> TMEM (A operand of S = Q K^T), by the A warps,
            // which finish a query's tiles first; every S of the earlier queries
            // has completed (this warp saw its s_full) ----
            if (!is_b) {
                const __nv_bfloat16* qrow = a.q + (t - a.row_begin) * a.q_stride_tok + (int64_t)h * a.q_stride_head + col0;
                uint4 qreg[5][8];
#pragma unroll
                for (int kb = 0; kb < 5; ++kb) {
                    if (kb < nb) {
                        const uint4* src = (const uint4*)(qrow + kb * 64);
#pragma unroll
                        for (int j = 0; j < 8; ++j) qreg[kb][j] = __ldg(src + j);
                    }
                }
#pragma unroll
                for (int kb = 0; kb < 5; ++kb) {
                    if (kb >= nb) continue;
                    uint32_t r[32];
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        r[4 * j] = qreg[kb][j].x;
                        r[4 * j + 1] = qreg[kb][j].y;
                        r[4 * j + 2] = qreg[kb][j].z;
                        r[4 * j + 3] = qreg[kb][j].w;
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
            // ---- the previous query's epilogue (this query's first S overlap it) ----
            if (pend) {
                if (!epilogue(t_pend, nqt - 1, m_pend, l_pend)) {
                    ok = false;
                    break;
                }
                pend = false;
            }
            float m_used = -INFINITY, l = 0.f;
            for (int u = 0; ok && u < n_tiles; ++u, ++g) {
                const uint32_t xb = g % NSX, xph = (g / NSX) & 1;      // partial-score buffer and its phase
                const uint32_t mlo = vmask[slot * 64 + 2 * u], mhi = vmask[slot * 64 + 2 * u + 1];
                if (!wait_warp(smem_u32(&bars->s_full), g & 1, abort, st, 0x2301)) { ok = false; break; }
                tc_fence_after();
                // this CTA's partial S = accumulator 0 + accumulator 1, both key
                // halves read in one TMEM round trip; stage A sends the peer's
                // half on before it forms the partial maximum
                const uint32_t ta = tmem + lane_off + TM_S;
                const int ph_ = kh ^ 1, oh = kh;  // key halves: the peer's, this CTA's
                uint32_t rp[32], ro[32], xo[32];
                {
                    uint32_t x[32];
                    tmem_ld32(ta + 32 * ph_, rp);
                    tmem_ld32(ta + 64 + 32 * ph_, x);
                    tmem_ld32(ta + 32 * oh, ro);
                    tmem_ld32(ta + 64 + 32 * oh, xo);
                    tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 32; ++i) rp[i] = __float_as_uint(__uint_as_float(rp[i]) + __uint_as_float(x[i]));
                }
                if (!is_b) {
                    // ---- stage A: send the peer's 32 partial columns, then the partial max ----
                    if (!wait_warp(my_sx_free0 + 8 * xb, xph ^ 1, abort, st, 0x2302)) { ok = false; break; }
                    const uint32_t dst = peer_sx + xb * AT_TILE128;
                    const uint32_t bar = peer_sx_full0 + 8 * xb;
#pragma unroll
                    for (int c = 0; c < 8; ++c)
                        st_async_v4(dst + chunk_off(h, c), rp[4 * c], rp[4 * c + 1], rp[4 * c + 2], rp[4 * c + 3], bar);
                }
#pragma unroll
                for (int i = 0; i < 32; ++i) ro[i] = __float_as_uint(__uint_as_float(ro[i]) + __uint_as_float(xo[i]));
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(smem_u32(&bars->s_empty));
                const uint32_t mo = kh ? mhi : mlo, mp = kh ? mlo : mhi;  // valid slots of the own / peer half
                float pm = -INFINITY;  // partial maximum of this CTA's row over the tile's valid keys
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    if ((mo >> i) & 1u) pm = fmaxf(pm, __uint_as_float(ro[i]));
                    if ((mp >> i) & 1u) pm = fmaxf(pm, __uint_as_float(rp[i]));
                }
                if (!is_b) {
                    st_async_b32(peer_pm + xb * 512 + h * 4, __float_as_uint(pm), peer_sx_full0 + 8 * xb);
                    continue;
                }
                // ---- stage B: combine, probabilities, both copies of P ----
                const uint32_t msk = mo;
                if (!wait_warp(my_sx_full0 + 8 * xb, xph, abort, st, 0x2303)) { ok = false; break; }
                if (arm_thread) mbar_arrive_expect_tx(my_sx_full0 + 8 * xb, AT_SX_BYTES);  // its next phase
                float s32[32];
                {
                    const uint8_t* rowp = sx + xb * AT_TILE128;
#pragma unroll
                    for (int c = 0; c < 8; ++c) {
                        const float4 v = *(const float4*)(rowp + chunk_off(h, c));
                        const float pv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                        for (int e = 0; e < 4; ++e)
                            s32[4 * c + e] = __uint_as_float(ro[4 * c + e]) + pv[e];
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
                // P tile pb is free once PV(g - NPB) is done in both CTAs
                const uint32_t pb = g % NPB;
                if (!wait_warp(my_p_free0 + 8 * pb, ((g / NPB) & 1) ^ 1, abort, st, 0x2304)) { ok = false; break; }
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
                    // O may be rescaled only between PV(g-1) and PV(g)
                    const uint32_t w = g - 1;
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
            if (!ok) break;
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(&bars->info_empty[slot]));
            pend = true;
            t_pend = t;
            m_pend = m_used;
            l_pend = l;
            ++nqt;
        }
        if (ok && pend) ok = epilogue(t_pend, nqt - 1, m_pend, l_pend);
    }
    tc_fence_before();
    __syncwarp();
    cluster_sync();  // no DSMEM traffic may target a CTA that has exited
    tc_fence_after();
    if (warp == AT_MMA_WARP) tmem_dealloc(tmem, 512);
}

// CTA pairs of this shape that can be resident at once (the persistent grid).
template <int NST, bool VSEP, int NPB, int NSX>
static int attn_pairs_resident() {
    static int cached = 0;
    if (cached > 0) return cached;
    using Lay = AtLayout<NST, VSEP, NPB, NSX>;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * 1024, 1, 1);
    cfg.blockDim = dim3(AT_THREADS, 1, 1);
    cfg.dynamicSmemBytes = Lay::SMEM;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, (const void*)attn_tc_kernel<NST, VSEP, NPB, NSX>, &cfg) != cudaSuccess) {
        (void)cudaGetLastError();
        n = 0;
    }
    if (n > 0) cached = n;
    return n;
}

template <int NST, bool VSEP, int NPB, int NSX>
static bool launch_attn_tc_t(const AttnTcArgs& a, cudaStream_t s) {
    using Lay = AtLayout<NST, VSEP, NPB, NSX>;
    static_assert(Lay::SMEM <= 232448, "shared memory budget");
    if (cudaFuncSetAttribute(attn_tc_kernel<NST, VSEP, NPB, NSX>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             Lay::SMEM) != cudaSuccess)
        return false;
    // the setmaxnreg split must fit the registers the block is launched with
    cudaFuncAttributes fa;
    if (cudaFuncGetAttributes(&fa, (const void*)attn_tc_kernel<NST, VSEP, NPB, NSX>) != cudaSuccess ||
        (int64_t)fa.numRegs * AT_THREADS < (int64_t)AT_REGS_SPLIT)
        return false;
    const int pairs = attn_pairs_resident<NST, VSEP, NPB, NSX>();
    if (pairs <= 0) return false;
    const int64_t grid_pairs = a.row_count < pairs ? a.row_count : pairs;
    attn_tc_kernel<NST, VSEP, NPB, NSX><<<(unsigned)(2 * grid_pairs), AT_THREADS, Lay::SMEM, s>>>(a);
    return cudaGetLastError() == cudaSuccess;
}

#ifndef DSA_ATTN_NST
#define DSA_ATTN_NST 3
#define DSA_ATTN_NPB 3
#define DSA_ATTN_NSX 1
#endif

bool launch_attn_tc(const AttnTcArgs& a, cudaStream_t s) {
    if (a.row_count <= 0) return true;
    return a.v_separate ? launch_attn_tc_t<2, true, 2, 1>(a, s)
                        : launch_attn_tc_t<DSA_ATTN_NST, false, DSA_ATTN_NPB, DSA_ATTN_NSX>(a, s);
}

}  // namespace dsa
