// indexer_tc.cu -- lightning indexer on the 5th-generation tensor cores with
// the exact per-query top-k fused onto the score tiles.
//
// Method: "DeepSeek-V3.2与稀疏注意力技术革新", §2.2 (I[t,s] = ReLU(q_t W k_s)
// with 128-dim FP8 keys; W is folded into the query beforehand) and §2.3
// (each query keeps its k best keys; the page maintains the candidates with
// a "dynamic priority queue" -- here the exact selection is reached by a
// most-significant-digit radix descent over repeated score sweeps, so the
// L x L score matrix never leaves the SM).
//
// Work unit: a block of 128 consecutive queries of one sequence.  One CTA
// per block, 10 warps:
//   warp 0      TMA producer: the block's folded queries (128 x 128 e4m3,
//               once) and key tiles of 256 x 128 e4m3 (+ their fp32 scales)
//   warp 1      TMEM allocator and MMA issuer: tcgen05.mma kind::f8f6f4,
//               M=128 N=256 K=32, fp32 accumulators in two TMEM buffers
//   warps 2..9  epilogue: two threads per query row (its TMEM lane), one per
//               128-column half of each tile; each reads its 128 fp32 dots
//               per tile, forms the score ReLU((dot * s_k) * s_row) and
//               applies the sweep's action.  The two halves share the row's
//               histogram (shared-memory atomics) and, when emitting, trade
//               their per-tile counts so the indices stay in ascending order.
//
// Sweeps over the block's causal key tiles (a block stops as soon as every
// row's selection is determined):
//   HIST level 1..4  per-row histogram of the next radix digit of the score
//                    bits, over the keys of the row's current bucket
//   EMIT             writes each row's selected indices in ascending order
// Score keys are the fp32 bit patterns (non-negative after ReLU).  Digit
// 1 is ceil(bits / 2^23) (0 only for +0.0), then bits 22..15, 14..7, 6..0 of
// (bits - 1).  After each histogram the row knows how many keys lie above
// the bucket holding its K-th best; it stops refining once that bucket is
// taken whole or holds a single value (ties: lowest indices first, which
// the ascending emission order gives for free).
#include "dsa_kernels.h"

namespace dsa {

constexpr int IX_BM = 128;
constexpr int IX_BN = 256;
constexpr int IX_NST = 2;
const int kIndexerRowsPerBlock = IX_BM;

constexpr uint32_t IX_A_BYTES = IX_BM * 128;
constexpr uint32_t IX_B_BYTES = IX_BN * 128;
constexpr uint32_t IX_OFF_A = 0;
constexpr uint32_t IX_OFF_B = IX_OFF_A + IX_A_BYTES;
constexpr uint32_t IX_OFF_SC = IX_OFF_B + IX_NST * IX_B_BYTES;
constexpr uint32_t IX_OFF_HIST = IX_OFF_SC + IX_NST * IX_BN * 4;
constexpr uint32_t IX_OFF_ECNT = IX_OFF_HIST + 256 * IX_BM * 4;    // [2 tiles][2 halves][128 rows] uint2
constexpr uint32_t IX_OFF_BAR = IX_OFF_ECNT + 2 * 2 * IX_BM * 8;
constexpr int IX_EPI_WARPS = 8;
constexpr int IX_THREADS = 64 + 32 * IX_EPI_WARPS;
constexpr uint32_t IX_SMEM = IX_OFF_BAR + 256 + 1024;  // + alignment slack

enum : int { SW_STOP = 0, SW_HIST = 1, SW_EMIT = 2, SW_SCORES = 3 };

struct IxBars {
    uint64_t full[IX_NST];
    uint64_t empty[IX_NST];
    uint64_t acc_full[2];
    uint64_t acc_empty[2];
    uint64_t a_full;
    uint64_t dec;
    uint64_t drain;
    uint32_t tmem_base;
    int next_kind;
    int next_level;
    int any_unresolved;
    int abort;
};

// Scores of 32 consecutive columns as non-negative fp32 bit patterns,
// computed in place: ReLU((dot * s_k) * s_row), +inf/NaN clamped to +inf.
// The 32 lanes of work are independent so the chain latencies overlap.
__device__ __forceinline__ void chunk_keys(uint32_t (&v)[32], const float* scs, float srow) {
    const float4* s4 = (const float4*)scs;
#pragma unroll
    for (int q = 0; q < 8; ++q) {
        const float4 sk = s4[q];
        const float skv[4] = {sk.x, sk.y, sk.z, sk.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float x = __fmul_rn(__fmul_rn(__uint_as_float(v[4 * q + e]), skv[e]), srow);
            v[4 * q + e] = (uint32_t)min(max(__float_as_int(x), 0), 0x7F800000);
        }
    }
}

// Per-row radix state of the epilogue thread.
struct RowSel {
    int sh, P;          // current bucket: keys with ((bits - 1) >> sh) == P
    uint32_t need;      // keys still to take from the bucket
    uint32_t taken;     // bucket keys taken so far in the emission sweep
    int cnt;            // indices written
    bool take_all;      // pos + 1 <= k: the whole causal prefix
};

// One 32-column chunk, columns c with c <= lim are causal.
template <int MODE>  // SW_HIST level 1 (1), deeper level (4), SW_EMIT (2), SW_SCORES (3)
__device__ __forceinline__ void ep_chunk(uint32_t (&v)[32], const float* scs, float srow, int lim, int32_t sbase,
                                         RowSel& rs, uint32_t* myhist, int dshift, uint32_t dmask, int32_t* out, int kcap,
                                         float* srow_out) {
    chunk_keys(v, scs, srow);
#define KB(i) ((int)v[i])
    const uint32_t limmask = lim >= 31 ? 0xFFFFFFFFu : ((1u << (lim + 1)) - 1u);
    if (MODE == 1) {
#pragma unroll
        for (int i = 0; i < 32; ++i)
            if ((limmask >> i) & 1u) atomicAdd(&myhist[((uint32_t)KB(i) + 0x7FFFFFu) >> 23 << 7], 1u);
    } else if (MODE == 4) {
        uint32_t mem = 0;
#pragma unroll
        for (int i = 0; i < 32; ++i) mem |= (uint32_t)(((KB(i) - 1) >> rs.sh) == rs.P) << i;
        mem &= limmask;
        while (mem) {
            const int i = __ffs(mem) - 1;
            mem &= mem - 1;
            int ki = 0;
#pragma unroll
            for (int e = 0; e < 32; ++e) ki = (e == i) ? KB(e) : ki;
            atomicAdd(&myhist[(((uint32_t)(ki - 1) >> dshift) & dmask) << 7], 1u);
        }
    } else if (MODE == 2) {
        uint32_t above = 0, eq = 0;
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            const int hi = (KB(i) - 1) >> rs.sh;
            above |= (uint32_t)(hi > rs.P) << i;
            eq |= (uint32_t)(hi == rs.P) << i;
        }
        if (rs.take_all) above = 0xFFFFFFFFu, eq = 0;
        above &= limmask;
        eq &= limmask;
        uint32_t any = above | eq;
        while (any) {
            const int i = __ffs(any) - 1;
            any &= any - 1;
            bool e = (above >> i) & 1u;
            if (!e && rs.taken < rs.need) {
                e = true;
                ++rs.taken;
            }
            if (e) {
                if (rs.cnt < kcap) out[rs.cnt] = sbase + i;
                ++rs.cnt;
            }
        }
    } else if (MODE == 3) {
        if (srow_out) {
            float* dst = srow_out + sbase;
            if (limmask == 0xFFFFFFFFu && (((uintptr_t)dst) & 15) == 0) {
                // a whole, aligned chunk: eight 16-byte stores instead of 32
                // scalar ones, so the next TMEM load into v[] waits less
#pragma unroll
                for (int q = 0; q < 8; ++q)
                    ((float4*)dst)[q] = make_float4(__int_as_float(KB(4 * q)), __int_as_float(KB(4 * q + 1)),
                                                    __int_as_float(KB(4 * q + 2)), __int_as_float(KB(4 * q + 3)));
            } else {
#pragma unroll
                for (int i = 0; i < 32; ++i)
                    if ((limmask >> i) & 1u) dst[i] = __int_as_float(KB(i));
            }
        }
    }
}
#undef KB

// One 128-column half of a tile for one row (taddr, scs and s_tile already
// point at the half), one 32-column TMEM load at a time.
template <int MODE>
__device__ __forceinline__ void ep_tile(uint32_t taddr, bool ok, bool active, const float* scs, float srow, int64_t pos,
                                        int64_t s_tile, RowSel& rs, uint32_t* myhist, int dshift, uint32_t dmask,
                                        int32_t* out, int kcap, float* srow_out) {
#pragma unroll 1
    for (int ch = 0; ch < 4; ++ch) {
        uint32_t v[32];
        if (ok) {
            tmem_ld32(taddr + ch * 32, v);
            tmem_wait_ld();
        }
        if (!active) continue;
        const int64_t sb = s_tile + ch * 32;
        if (sb <= pos)
            ep_chunk<MODE>(v, scs + ch * 32, srow, (int)min((int64_t)31, pos - sb), (int32_t)sb, rs, myhist, dshift, dmask,
                           out, kcap, srow_out);
    }
}

// EMIT for one 128-column half of a tile.  Both halves of the row form their
// masks, trade (above, equal) counts through shared memory (slot ec, this
// half's counts at ec[half], the partner's at ec[half ^ 1]) with a two-warp
// barrier, then write their keys at their places in the ascending order: the
// first half's keys precede the second half's, the bucket's equal keys are
// taken in index order until the row has what it needs.
__device__ __forceinline__ void ep_emit_half(uint32_t taddr, bool ok, bool active, const float* scs, float srow, int64_t pos,
                                             int64_t s_half, int half, RowSel& rs, int32_t* out, int kcap, uint2* ec,
                                             int bar_id) {
    // ec[h * IX_BM]: the counts of half h of this row
    uint32_t abv[4], eqm[4];
    uint32_t n_above = 0, n_eq = 0;
#pragma unroll
    for (int ch = 0; ch < 4; ++ch) {
        uint32_t v[32];
        if (ok) {
            tmem_ld32(taddr + ch * 32, v);
            tmem_wait_ld();
        }
        abv[ch] = 0;
        eqm[ch] = 0;
        const int64_t sb = s_half + ch * 32;
        if (!active || sb > pos) continue;
        chunk_keys(v, scs + ch * 32, srow);
        const int lim = (int)min((int64_t)31, pos - sb);
        const uint32_t limmask = lim >= 31 ? 0xFFFFFFFFu : ((1u << (lim + 1)) - 1u);
        uint32_t above = 0, eq = 0;
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            const int hi = ((int)v[i] - 1) >> rs.sh;
            above |= (uint32_t)(hi > rs.P) << i;
            eq |= (uint32_t)(hi == rs.P) << i;
        }
        if (rs.take_all) above = 0xFFFFFFFFu, eq = 0;
        abv[ch] = above & limmask;
        eqm[ch] = eq & limmask;
        n_above += __popc(abv[ch]);
        n_eq += __popc(eqm[ch]);
    }
    ec[half * IX_BM] = make_uint2(n_above, n_eq);
    asm volatile("bar.sync %0, 64;" ::"r"(bar_id) : "memory");
    const uint2 c0 = half ? ec[0] : make_uint2(n_above, n_eq);
    const uint2 c1 = half ? make_uint2(n_above, n_eq) : ec[IX_BM];
    const uint32_t left = rs.need > rs.taken ? rs.need - rs.taken : 0u;
    const uint32_t t0 = min(c0.y, left), t1 = min(c1.y, left - t0);
    int pos_out = rs.cnt + (half ? (int)(c0.x + t0) : 0);
    uint32_t take = half ? t1 : t0;
#pragma unroll
    for (int ch = 0; ch < 4; ++ch) {
        uint32_t any = abv[ch] | eqm[ch];
        const int32_t sb = (int32_t)(s_half + ch * 32);
        while (any) {
            const int i = __ffs(any) - 1;
            any &= any - 1;
            bool e = (abv[ch] >> i) & 1u;
            if (!e && take > 0) {
                e = true;
                --take;
            }
            if (e) {
                if (pos_out < kcap) out[pos_out] = sb + i;
                ++pos_out;
            }
        }
    }
    rs.cnt += (int)(c0.x + t0 + c1.x + t1);
    rs.taken += t0 + t1;
}

// KMODE 0: the fused selection (index rows out); KMODE 1: the score sweep
// (scores out, optionally split over key tiles).  Each mode is its own
// instantiation, so neither carries the other's epilogue code.
template <int KMODE>
__global__ void __launch_bounds__(IX_THREADS, 1) indexer_tc_kernel(const __grid_constant__ IndexerTcArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    IxBars* bars = (IxBars*)(smem + IX_OFF_BAR);
    float* sc_s = (float*)(smem + IX_OFF_SC);
    uint32_t* hist = (uint32_t*)(smem + IX_OFF_HIST);
    const uint32_t warp = warp_id(), lane = lane_id();
    StatusHdr* st = a.st;
    volatile int* abort = &bars->abort;

    // ---- block -> (sequence, row range, key-tile split); heaviest blocks
    // launch first.  Score sweeps (mode 1) may split a row block's key tiles
    // over tile_splits CTAs, each taking a contiguous range of tiles ----
    const int nsplit = a.tile_splits > 1 ? a.tile_splits : 1;
    if (nsplit > 1 && KMODE != 1) {
        if (threadIdx.x == 0) report(a.st, DSA_ERR_UNSUPPORTED, -5);
        return;
    }
    const int split = (int)(blockIdx.x % nsplit);
    const int64_t bid = (int64_t)(blockIdx.x / nsplit);
    const int64_t nblk = (a.max_seqlen_q + IX_BM - 1) / IX_BM;
    const int b = (int)(bid % a.sv.batch);
    const int64_t jb = nblk - 1 - bid / a.sv.batch;
    const int64_t q0 = __ldg(a.sv.cu_q + b), sq = __ldg(a.sv.cu_q + b + 1) - q0;
    const int64_t key_base = __ldg(a.sv.cu_k + b), sk = __ldg(a.sv.cu_k + b + 1) - key_base;
    const int64_t i0 = jb * IX_BM;
    if (i0 >= sq) return;
    const int64_t nrows = min((int64_t)IX_BM, sq - i0);
    const int64_t pos_first = sk - sq + i0;
    const int64_t pos_last = pos_first + nrows - 1;
    if (pos_first < 0) {
        if (threadIdx.x == 0) report(st, DSA_ERR_INDEX, q0 + i0);
        return;
    }
    const int64_t t_first = q0 + i0;
    if (KMODE == 1 && (t_first + nrows <= a.row_begin || t_first >= a.row_begin + a.row_count)) return;
    const int n_tiles = (int)((pos_last + IX_BN) / IX_BN);
    const int per_split = (n_tiles + nsplit - 1) / nsplit;
    const int t_lo = split * per_split, t_hi = min(n_tiles, t_lo + per_split);  // this CTA's key tiles
    if (t_lo >= t_hi) return;
    int first_kind;
    if (KMODE == 1)
        first_kind = SW_SCORES;
    else
        first_kind = (pos_last + 1 > a.k || a.k_rows) ? SW_HIST : SW_STOP;

    const uint32_t sA = smem_u32(smem + IX_OFF_A);
    const uint32_t sB = smem_u32(smem + IX_OFF_B);

    if (threadIdx.x == 0) {
        for (int i = 0; i < IX_NST; ++i) {
            mbar_init(smem_u32(&bars->full[i]), 1);
            mbar_init(smem_u32(&bars->empty[i]), 1 + IX_EPI_WARPS);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(smem_u32(&bars->acc_full[i]), 1);
            mbar_init(smem_u32(&bars->acc_empty[i]), IX_EPI_WARPS);
        }
        mbar_init(smem_u32(&bars->a_full), 1);
        mbar_init(smem_u32(&bars->dec), 1);
        mbar_init(smem_u32(&bars->drain), 1);
        bars->abort = 0;
        fence_mbar_init();
    }
    if (warp == 1) tmem_alloc(smem_u32(&bars->tmem_base), 512);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bars->tmem_base;

    if (warp == 0) {
        // ================= TMA producer =================
        if (lane == 0) {
            tma_prefetch_desc(&a.tm_u);
            tma_prefetch_desc(&a.tm_k);
        }
        if (first_kind != SW_STOP) {
            if (lane == 0) {
                mbar_arrive_expect_tx(smem_u32(&bars->a_full), IX_A_BYTES);
                tma_load_2d(sA, &a.tm_u, 0, (int32_t)t_first, smem_u32(&bars->a_full));
            }
            uint32_t g = 0;
            uint32_t last_issued[IX_NST];
            for (int i = 0; i < IX_NST; ++i) last_issued[i] = 0xFFFFFFFFu;
            int kind = first_kind;
            for (int sw = 0; kind != SW_STOP; ++sw) {
                for (int tile = t_lo; tile < t_hi; ++tile, ++g) {
                    const uint32_t s = g % IX_NST;
                    if (!wait_warp(smem_u32(&bars->empty[s]), ((g / IX_NST) & 1) ^ 1, abort, st, 0x1101)) break;
                    const int64_t kr0 = key_base + (int64_t)tile * IX_BN;
                    float* scs = sc_s + s * IX_BN;
                    // full tiles with 16-byte aligned scales: one bulk copy; else plain loads
                    const bool bulk = (tile + 1) * IX_BN <= pos_last + 1 && ((uintptr_t)(a.k_scale + kr0) & 15) == 0;
                    if (!bulk) {
                        for (int i = lane; i < IX_BN; i += 32) {
                            const int64_t kr = kr0 + i;
                            scs[i] = (tile * IX_BN + i <= pos_last) ? __ldg(a.k_scale + kr) : 0.f;
                        }
                    }
                    __syncwarp();
                    if (lane == 0) {
                        mbar_arrive_expect_tx(smem_u32(&bars->full[s]), IX_B_BYTES + (bulk ? IX_BN * 4 : 0));
                        tma_load_2d(sB + s * IX_B_BYTES, &a.tm_k, 0, (int32_t)kr0, smem_u32(&bars->full[s]));
                        if (bulk) bulk_load(smem_u32(scs), a.k_scale + kr0, IX_BN * 4, smem_u32(&bars->full[s]));
                    }
                    last_issued[s] = g;
                    __syncwarp();
                }
                if (*abort) break;
                if (!wait_warp(smem_u32(&bars->dec), sw & 1, abort, st, 0x1102)) break;
                kind = *(volatile int*)&bars->next_kind;
            }
            // drain: every issued load must land before the CTA exits
            if (*abort && lane == 0) {
                for (int s = 0; s < IX_NST; ++s)
                    if (last_issued[s] != 0xFFFFFFFFu)
                        mbar_wait(smem_u32(&bars->full[s]), (last_issued[s] / IX_NST) & 1, nullptr, st, 0x1103, 1ll << 28);
            }
        }
    } else if (warp == 1) {
        // ================= MMA issuer =================
        constexpr uint32_t idesc = idesc_make(0, 0, false, IX_BM, IX_BN);
        if (first_kind != SW_STOP) {
            bool ok = wait_warp(smem_u32(&bars->a_full), 0, abort, st, 0x1201);
            uint32_t g = 0;
            int kind = first_kind;
            for (int sw = 0; ok && kind != SW_STOP; ++sw) {
                for (int tile = t_lo; tile < t_hi; ++tile, ++g) {
                    const uint32_t s = g % IX_NST, ab = g & 1;
                    if (!wait_warp(smem_u32(&bars->full[s]), (g / IX_NST) & 1, abort, st, 0x1202)) { ok = false; break; }
                    if (!wait_warp(smem_u32(&bars->acc_empty[ab]), ((g >> 1) & 1) ^ 1, abort, st, 0x1203)) { ok = false; break; }
                    tc_fence_after();
                    if (lane == 0) {
#pragma unroll
                        for (int ks = 0; ks < 4; ++ks) {
                            const uint64_t ad = sdesc_sw128(sA + ks * 32, 16, 1024);
                            const uint64_t bd = sdesc_sw128(sB + s * IX_B_BYTES + ks * 32, 16, 1024);
                            mma_fp8_ss(tmem + ab * IX_BN, ad, bd, idesc, ks > 0 ? 1u : 0u);
                        }
                        mma_commit(smem_u32(&bars->empty[s]));
                        mma_commit(smem_u32(&bars->acc_full[ab]));
                    }
                    __syncwarp();
                }
                if (!ok) break;
                if (!wait_warp(smem_u32(&bars->dec), sw & 1, abort, st, 0x1204)) break;
                kind = *(volatile int*)&bars->next_kind;
            }
            if (*abort && lane == 0) {
                mma_commit(smem_u32(&bars->drain));
                mbar_wait(smem_u32(&bars->drain), 0, nullptr, st, 0x1205, 1ll << 28);
            }
        }
    } else {
        // ================= epilogue: two threads per query row =================
        const uint32_t quad = warp & 3;
        const int half = (int)(warp - 2) >> 2;  // 128-column half of every tile
        const int row = (int)(quad * 32 + lane);
        const bool has_row = row < nrows;
        const int64_t t = t_first + row;
        const int64_t pos = pos_first + row;
        const float srow = has_row ? __ldg(a.s_row + t) : 0.f;
        const bool in_range = KMODE != 1 || (t >= a.row_begin && t < a.row_begin + a.row_count);
        // this row's k (dynamic k: clamped to [0, k]); the index row is k wide
        const int k_row = (KMODE == 0 && a.k_rows && has_row) ? min(max(__ldg(a.k_rows + t), 0), a.k) : a.k;
        const bool take_all = pos + 1 <= k_row && k_row > 0;
        // radix state
        int level = 0;
        RowSel rs;
        rs.sh = 31;
        rs.P = 0;
        rs.need = (uint32_t)k_row;
        rs.taken = 0;
        rs.cnt = 0;
        rs.take_all = take_all;
        bool resolved = !has_row || take_all || k_row == 0;
        if (k_row == 0) {  // nothing kept: a bucket no key falls into
            rs.P = 0x7FFFFFFF;
            rs.sh = 31;
        }
        uint32_t* myhist = hist + row;  // bin b at myhist[b * IX_BM]
        int32_t* out = (KMODE == 0 && has_row) ? a.idx + t * a.ld_idx : nullptr;
        float* srow_out = (KMODE == 1 && has_row && in_range) ? a.scores + (t - a.row_begin) * a.ld_scores : nullptr;
        for (int i = 128 * half; i < 128 * half + 128; ++i) myhist[i * IX_BM] = 0;
        asm volatile("bar.sync 1, 256;" ::: "memory");  // both halves cleared the row's bins

        uint32_t g = 0;
        int kind = first_kind;
        for (int sw = 0; kind != SW_STOP; ++sw) {
            const int lvl = level + 1;  // histogram level of this sweep (HIST)
            for (int tile = t_lo; tile < t_hi; ++tile, ++g) {
                const uint32_t s = g % IX_NST, ab = g & 1;
                bool ok = wait_warp(smem_u32(&bars->acc_full[ab]), (g >> 1) & 1, abort, st, 0x1301);
                ok = ok && wait_warp(smem_u32(&bars->full[s]), (g / IX_NST) & 1, abort, st, 0x1302);
                tc_fence_after();
                const float* scs = sc_s + s * IX_BN + 128 * half;
                const int64_t s_tile = (int64_t)tile * IX_BN + 128 * half;
                const bool active = ok && has_row && !(kind == SW_HIST && resolved);
                const uint32_t taddr = tmem + ((quad * 32) << 16) + ab * IX_BN + 128 * half;
                if constexpr (KMODE == 1) {
                    ep_tile<3>(taddr, ok, active, scs, srow, pos, s_tile, rs, myhist, 0, 0, out, a.k, srow_out);
                } else {
                    if (kind == SW_HIST && lvl == 1)
                        ep_tile<1>(taddr, ok, active, scs, srow, pos, s_tile, rs, myhist, 0, 0, out, a.k, srow_out);
                    else if (kind == SW_HIST)
                        ep_tile<4>(taddr, ok, active, scs, srow, pos, s_tile, rs, myhist, lvl == 2 ? 15 : lvl == 3 ? 7 : 0,
                                   lvl == 4 ? 127u : 255u, out, a.k, srow_out);
                    else if (kind == SW_EMIT)
                        ep_emit_half(taddr, ok, active, scs, srow, pos, s_tile, half, rs, out, a.k,
                                     (uint2*)(smem + IX_OFF_ECNT) + (tile & 1) * 2 * IX_BM + row, 2 + (int)quad);
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) {
                    mbar_arrive(smem_u32(&bars->acc_empty[ab]));
                    mbar_arrive(smem_u32(&bars->empty[s]));
                }
            }
            // ---- end of sweep: refine each row's bucket (both halves of the row
            // reach the same decision from the shared histogram); one thread
            // decides the next sweep ----
            if (kind == SW_HIST) {
                asm volatile("bar.sync 1, 256;" ::: "memory");  // every count of the sweep is in
                if (has_row && !resolved) {
                    uint32_t cum = 0;
                    int bsel = 0;
                    const int top = lvl == 4 ? 127 : 255;
                    for (int bb = top; bb >= 0; --bb) {
                        const uint32_t c = myhist[bb * IX_BM];
                        if (cum + c >= rs.need) { bsel = bb; break; }
                        cum += c;
                    }
                    const uint32_t in_bin = myhist[bsel * IX_BM];
                    rs.need -= cum;
                    if (lvl == 1) { rs.P = bsel - 1; rs.sh = 23; }
                    else if (lvl == 2) { rs.P = (rs.P << 8) | bsel; rs.sh = 15; }
                    else if (lvl == 3) { rs.P = (rs.P << 8) | bsel; rs.sh = 7; }
                    else { rs.P = (rs.P << 7) | bsel; rs.sh = 0; }
                    resolved = in_bin == rs.need || rs.P == -1 || lvl == 4;
                }
                level = lvl;
                if (threadIdx.x == 64) bars->any_unresolved = 0;
                asm volatile("bar.sync 1, 256;" ::: "memory");  // every histogram read is done
                for (int i = 128 * half; i < 128 * half + 128; ++i) myhist[i * IX_BM] = 0;
                if (has_row && !resolved) bars->any_unresolved = 1;
            }
            asm volatile("bar.sync 1, 256;" ::: "memory");
            if (threadIdx.x == 64) {
                int nk = kind == SW_HIST ? (bars->any_unresolved ? SW_HIST : SW_EMIT) : SW_STOP;
                if (*abort) nk = SW_STOP;
                bars->next_kind = nk;
                mbar_arrive(smem_u32(&bars->dec));
            }
            asm volatile("bar.sync 1, 256;" ::: "memory");
            kind = *(volatile int*)&bars->next_kind;
        }
        // ---- finish the index rows ----
        if (KMODE == 0 && has_row && half == 0) {
            if (first_kind == SW_STOP) {  // every row of the block keeps its whole prefix
                for (int64_t s = 0; s <= pos; ++s) out[s] = (int32_t)s;
                rs.cnt = (int)(pos + 1);
            }
            const int expect = (int)min((int64_t)k_row, pos + 1);
            if (rs.cnt != expect && !*abort) report(st, DSA_ERR_INDEX, -2000000 - t);
            for (int s = min(rs.cnt, a.k); s < a.k; ++s) out[s] = -1;
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, 512);
}

bool launch_indexer_tc(const IndexerTcArgs& a, cudaStream_t s) {
    if (a.mode != 0 && a.mode != 1) return false;
    const void* fn = a.mode == 1 ? (const void*)indexer_tc_kernel<1> : (const void*)indexer_tc_kernel<0>;
    if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, IX_SMEM) != cudaSuccess) return false;
    const int64_t nblk = (a.max_seqlen_q + IX_BM - 1) / IX_BM;
    const int64_t grid = nblk * a.sv.batch * (a.tile_splits > 1 ? a.tile_splits : 1);
    if (grid <= 0) return true;
    if (grid >= ((int64_t)1 << 31)) return false;
    if (a.mode == 1)
        indexer_tc_kernel<1><<<(unsigned)grid, IX_THREADS, IX_SMEM, s>>>(a);
    else
        indexer_tc_kernel<0><<<(unsigned)grid, IX_THREADS, IX_SMEM, s>>>(a);
    return cudaGetLastError() == cudaSuccess;
}

}  // namespace dsa
