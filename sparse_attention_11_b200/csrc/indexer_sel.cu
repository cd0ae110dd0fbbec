// indexer_sel.cu -- the lightning indexer fused with the exact per-query
// top-k on the 5th-generation tensor cores, for prefill shapes.
//
// Method: "DeepSeek-V3.2与稀疏注意力技术革新", §2.2 (I[t,s] = ReLU(q_t W k_s)
// over 128-dim FP8 keys; W is folded into the query beforehand) and §2.3 (each
// query keeps its k best keys; the page keeps its candidates in a "dynamic
// priority queue").  Here the candidates are kept as a per-row score window
// and a bitmask, and the selection is exact: identical to sorting the row's
// scores (ties to the lower key index).  The L x L scores never leave the SM.
//
// Work unit: a block of 128 consecutive queries of one sequence.  The grid is
// persistent (one CTA per SM); CTA i takes blocks i, 2G-1-i, 2G+i, ... of the
// heaviest-first order.  10 warps:
//   warp 0      TMA producer: the block's folded queries (128 x 128 e4m3),
//               key tiles of 256 x 128 e4m3 and their fp32 scales
//   warp 1      TMEM owner and MMA issuer: tcgen05.mma kind::f8f6f4,
//               M=128 N=256, fp32 accumulators in two TMEM buffers
//   warps 2..9  epilogue: two threads per query row, one per 128-column half
//               of each tile; the score is ReLU((dot * s_k) * s_row)
//
// Sweeps of one block (the MMAs are recomputed in each):
//   S1, S2  over a sample of the common causal prefix (every 16th key): a
//           per-row histogram of the sample's scores, by binade (S1) and then
//           at 1/64 binade around the binade holding the sample's rank
//           K_t * n_sample / n_keys (S2).  This estimates each row's K-th score.
//   H       over all causal keys: a per-row histogram at 1/128 binade over
//           two binades around the estimate (rows whose estimate is zero
//           histogram the zero score and the denormals exactly).  The bin
//           holding the K-th score is the row's bucket [lo, hi).
//   REF     (rare) when a bucket is too large to resolve, a further histogram
//           of the keys inside it at 256 finer bins.
//   E       over all causal keys: a bitmask per row of the keys at or above
//           lo (keys at or above hi are always kept), written to a per-CTA
//           scratch.  A bucket of a single score value takes its first `need`
//           keys in index order (the two threads of a row trade their per-tile
//           counts); a bucket of several values (at most kListCap keys) is
//           listed on chip with the scores, and its losers are cleared after.
// Finish: one warp per row turns the bitmask into the ascending index row.
#include "dsa_kernels.h"

namespace dsa {
namespace sel {

constexpr int BM = 128;
constexpr int BN = 256;
constexpr int NST = 2;
constexpr int EPI_WARPS = 8;
constexpr int THREADS = 64 + 32 * EPI_WARPS;
constexpr int kSampleStride = 16;
constexpr int kListCap = 96;
constexpr uint32_t kInfKey = 0x7F800000u;  // score key of +inf (and of NaN)

constexpr uint32_t A_BYTES = BM * 128;
constexpr uint32_t B_BYTES = BN * 128;
constexpr uint32_t OFF_A = 0;
constexpr uint32_t OFF_B = OFF_A + A_BYTES;
constexpr uint32_t OFF_SC = OFF_B + NST * B_BYTES;
constexpr uint32_t OFF_R = OFF_SC + NST * BN * 4;
constexpr uint32_t R_BYTES = 256 * BM * 4;                  // histogram [256 bins][128 rows]
constexpr uint32_t OFF_LIST = OFF_R;                        // E: bucket lists [kListCap][128 rows] of (index, key)
constexpr uint32_t OFF_STAGE = OFF_R + kListCap * BM * 8;   // E: 128 bytes per epilogue thread
constexpr uint32_t OFF_XCH = OFF_R + R_BYTES;               // E: per-tile member counts [2][2 halves][128 rows]
constexpr uint32_t OFF_LCNT = OFF_XCH + 2 * 2 * BM * 4;     // bucket list lengths [128]
constexpr uint32_t OFF_RINFO = OFF_LCNT + BM * 4;           // per-row finish record [128]
constexpr uint32_t OFF_BAR = OFF_RINFO + BM * 32;
constexpr uint32_t SMEM = OFF_BAR + 256 + 1024;             // + alignment slack
constexpr int kStageInts = (int)(NST * B_BYTES / 4 / EPI_WARPS);  // finish: index staging per warp (2048)
static_assert(OFF_STAGE + 32 * EPI_WARPS * 128 <= OFF_R + R_BYTES, "bucket lists and staging exceed the region");
static_assert(SMEM <= 232448, "shared memory");

enum : int { SK_STOP = 0, SK_S1 = 1, SK_S2 = 2, SK_H = 3, SK_REF = 4, SK_E = 5 };
// per-row resolution of its bucket
enum : int { RES_NONE = 0, RES_WHOLE = 1, RES_SINGLE = 2, RES_LIST = 3 };
// per-row kind (finish record)
enum : int { ROW_NONE = 0, ROW_EMPTY = 1, ROW_PREFIX = 2, ROW_SEL = 3 };

struct Bars {
    uint64_t full[NST];
    uint64_t empty[NST];
    uint64_t acc_full[2];
    uint64_t acc_empty[2];
    uint64_t a_full;
    uint64_t dec;
    uint64_t drain;
    uint32_t tmem_base;
    int next_kind;
    int any_flag;
    int abort;
};

struct RowRec {  // what the finish warp needs of a row
    int kind;
    int res;
    int pos;
    int kt;
    uint32_t need;  // RES_LIST: keys to take from the listed bucket
    uint32_t pad[3];
};

// ---------------------------------------------------------------------------
// packed fp32 pairs (sm_100a f32x2 arithmetic; each lane rounds like the
// scalar instruction)
// ---------------------------------------------------------------------------
DSA_DEV uint64_t pk(uint32_t lo, uint32_t hi) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "r"(lo), "r"(hi));
    return r;
}
DSA_DEV void upk(uint64_t v, uint32_t& lo, uint32_t& hi) { asm("mov.b64 {%0, %1}, %2;" : "=r"(lo), "=r"(hi) : "l"(v)); }
DSA_DEV uint64_t fmul2(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
DSA_DEV uint64_t fsub2(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}

// Raw scores (dot * s_k) * s_row of 32 columns, in place, as fp32 bits.  The
// ReLU is applied by the consumers: a negative raw score is the score +0.
DSA_DEV void raw_scores(uint32_t* v, const float* scs, uint64_t srow2) {
    const float4* s4 = (const float4*)scs;
#pragma unroll
    for (int q = 0; q < 8; ++q) {
        const float4 sk = s4[q];
        uint64_t a = pk(v[4 * q], v[4 * q + 1]), b = pk(v[4 * q + 2], v[4 * q + 3]);
        a = fmul2(fmul2(a, pk(__float_as_uint(sk.x), __float_as_uint(sk.y))), srow2);
        b = fmul2(fmul2(b, pk(__float_as_uint(sk.z), __float_as_uint(sk.w))), srow2);
        upk(a, v[4 * q], v[4 * q + 1]);
        upk(b, v[4 * q + 2], v[4 * q + 3]);
    }
}

// The score key of a raw score: its fp32 bits after ReLU, NaN counted as +inf.
// Keys order like the scores.
DSA_DEV uint32_t score_key(uint32_t raw) { return (uint32_t)__vimin_s32_relu((int)raw, (int)kInfKey); }

// Add 1 to the shared-memory counter at `addr` when `bin` is not 0 (a
// predicated reduction, so the 32 updates of a chunk need no branches).
DSA_DEV void red_if(uint32_t addr, int bin) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.s32 p, %1, 0;\n\t@p red.shared.add.u32 [%0], 1;\n\t}" ::"r"(addr), "r"(bin)
        : "memory");
}

// Histogram of 32 raw scores, bin = clamp((bits >> sh) + nc0, 0, 255) on the
// raw bits (nc0 = -c0).  With c0 >= 0 every non-positive raw score lands in
// bin 0 with the score +0, and with (kInfKey >> sh) - c0 >= 255 NaN lands in
// bin 255 with +inf, so the bins are those of the score keys.  Bin 0 is not
// counted (no decision needs it).  Columns past `lim` are skipped.  hbase is
// the shared address of the row's bin 0; bin b is b * 512 bytes further.
DSA_DEV void hist_chunk(const uint32_t* v, int sh, int nc0, int lim, uint32_t hbase) {
    if (lim >= 31) {
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            const int bin = __viaddmin_s32_relu((int)v[i] >> sh, nc0, 255);
            red_if(hbase + (bin << 9), bin);
        }
    } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            const int bin = __viaddmin_s32_relu((int)v[i] >> sh, nc0, 255);
            red_if(hbase + (bin << 9), i <= lim ? bin : 0);
        }
    }
}

// Histogram of the keys inside a bucket [lo, lo + w): bin 1 + ((key - lo) >> sh).
DSA_DEV void ref_chunk(const uint32_t* v, uint32_t lo, uint32_t w, int sh, int lim, uint32_t hbase) {
#pragma unroll
    for (int i = 0; i < 32; ++i) {
        const uint32_t d = score_key(v[i]) - lo;
        const int bin = 1 + (int)(d >> sh);
        red_if(hbase + (bin << 9), (d < w && i <= lim) ? bin : 0);
    }
}

// Bits of the columns whose raw score is below the threshold t (fp32 compare
// by the sign of the exact difference; x - t is +0 when x == t).  A NaN raw
// score gives a NaN difference with the sign clear: not below, like +inf.
// Four independent chains of eight keys each, so the funnel shifts overlap.
DSA_DEV uint32_t below_mask(const uint32_t* v, uint32_t t_bits) {
    const uint64_t t2 = pk(t_bits, t_bits);
    uint32_t m[4] = {0u, 0u, 0u, 0u};
#pragma unroll
    for (int q = 3; q >= 0; --q) {
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            uint32_t d0, d1;
            upk(fsub2(pk(v[8 * c + 2 * q], v[8 * c + 2 * q + 1]), t2), d0, d1);
            m[c] = __funnelshift_l(d1, m[c], 1);
            m[c] = __funnelshift_l(d0, m[c], 1);
        }
    }
    return m[0] | (m[1] << 8) | (m[2] << 16) | (m[3] << 24);
}

DSA_DEV uint32_t lim_mask(int lim) { return lim >= 31 ? 0xFFFFFFFFu : (lim < 0 ? 0u : ((2u << lim) - 1u)); }

// Keep the lowest n set bits of m.
DSA_DEV uint32_t keep_low(uint32_t m, uint32_t n) {
    if (n == 0) return 0u;
    if ((uint32_t)__popc(m) <= n) return m;
    const uint32_t p = __fns(m, 0, (int)n + 1);  // position of the (n+1)-th set bit
    return m & ((1u << p) - 1u);
}

// Per-row selection state, held identically by the row's two threads.
struct Row {
    int pos;        // local position of the query
    int kt;         // K_t = min(k_t, pos + 1)
    int kind;       // ROW_*
    bool active;    // still refining its bucket
    int sh, nc0;    // histogram parameters of the next H-type sweep
    uint32_t lo, hi;  // bucket of keys [lo, hi); hi == kInfKey + 1: includes +inf
    uint32_t need;    // keys still to take from the bucket
    int res;          // RES_*
    int r;            // rank of the K-th score in the sample
    bool s2;          // takes part in S2
};

DSA_DEV void clear_hist(uint32_t* hrow, int half) {
    for (int i = 128 * half; i < 128 * half + 128; ++i) hrow[i << 7] = 0u;
}

// Largest bin b in [bmin, 255] with (count of bins >= b) >= need; returns -1
// and the count above when no bin qualifies.
DSA_DEV int find_bin(const uint32_t* hrow, int bmin, uint32_t need, uint32_t& cum) {
    cum = 0;
    for (int b = 255; b >= bmin; --b) {
        const uint32_t c = hrow[b << 7];
        if (cum + c >= need) return b;
        cum += c;
    }
    return -1;
}

// After H or REF: the bucket holding the row's K-th score, and how it is
// resolved.  Sets row.active when a REF sweep is needed.
DSA_DEV void decide_bucket(Row& rw, const uint32_t* hrow, bool ref) {
    uint32_t cum;
    const int b = find_bin(hrow, 1, rw.need, cum);
    uint32_t lo, hi, c;
    bool known = true;
    if (ref) {
        // bins 1..254 of the previous bucket [rw.lo, rw.hi) at 2^sh keys each
        if (b < 1) {  // cannot happen (the bucket holds at least `need` keys); the count check reports it
            rw.res = RES_WHOLE;
            rw.active = false;
            return;
        }
        lo = rw.lo + ((uint32_t)(b - 1) << rw.sh);
        const uint64_t h64 = (uint64_t)lo + ((uint64_t)1 << rw.sh);
        hi = h64 < (uint64_t)rw.hi ? (uint32_t)h64 : rw.hi;
        c = hrow[b << 7];
    } else {
        const int c0 = -rw.nc0;
        if (b < 1) {  // the K-th score lies in bin 0: below the window
            lo = 0;
            hi = (uint32_t)(1 + c0) << rw.sh;
            known = false;
            c = 0;
        } else if (b == 255) {
            lo = (uint32_t)(255 + c0) << rw.sh;
            hi = kInfKey + 1;
            c = hrow[255 << 7];
        } else {
            lo = (uint32_t)(b + c0) << rw.sh;
            hi = (uint32_t)(b + c0 + 1) << rw.sh;
            c = hrow[b << 7];
        }
    }
    const uint32_t rem = rw.need - cum;
    rw.lo = lo;
    rw.hi = hi;
    rw.need = rem;
    if (hi - lo == 1u) {
        rw.res = RES_SINGLE;
    } else if (known && rem == c) {
        rw.res = RES_WHOLE;
    } else if (known && c <= (uint32_t)kListCap) {
        rw.res = RES_LIST;
    } else {
        rw.res = RES_NONE;
    }
    rw.active = rw.res == RES_NONE;
    if (rw.active) {  // next: 254 bins over [lo, hi)
        const uint32_t w1 = hi - lo - 1u;
        int s = 0;
        while ((w1 >> s) > 253u) ++s;
        rw.sh = s;
    }
}

// ---------------------------------------------------------------------------
// The kernel
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(THREADS, 1) indexer_sel_kernel(const __grid_constant__ IndexerTcArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    Bars* bars = (Bars*)(smem + OFF_BAR);
    float* sc_s = (float*)(smem + OFF_SC);
    uint32_t* hist = (uint32_t*)(smem + OFF_R);
    uint2* list = (uint2*)(smem + OFF_LIST);
    uint32_t* xch = (uint32_t*)(smem + OFF_XCH);
    uint32_t* lcnt = (uint32_t*)(smem + OFF_LCNT);
    RowRec* rrec = (RowRec*)(smem + OFF_RINFO);
    const uint32_t warp = warp_id(), lane = lane_id();
    StatusHdr* st = a.st;
    volatile int* abort = &bars->abort;

    if (threadIdx.x == 0) {
        for (int i = 0; i < NST; ++i) {
            mbar_init(smem_u32(&bars->full[i]), 1);
            mbar_init(smem_u32(&bars->empty[i]), 1 + EPI_WARPS);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(smem_u32(&bars->acc_full[i]), 1);
            mbar_init(smem_u32(&bars->acc_empty[i]), EPI_WARPS);
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

    const uint32_t sA = smem_u32(smem + OFF_A);
    const uint32_t sB = smem_u32(smem + OFF_B);
    const int64_t nblk = (a.max_seqlen_q + BM - 1) / BM;
    const int64_t nblk_all = nblk * a.sv.batch;
    const int G = (int)gridDim.x;
    uint32_t* scratch = a.sel_bits + (size_t)blockIdx.x * BM * (size_t)a.sel_words;

    // pipeline counters, continued across blocks and sweeps
    uint32_t g = 0;          // tiles
    uint32_t nsweep = 0;     // decisions (dec phases)
    uint32_t nblock = 0;     // blocks that loaded their queries (a_full phases)
    uint32_t last_issued[NST];  // producer: last tile issued into each stage (abort drain)
    for (int i = 0; i < NST; ++i) last_issued[i] = 0xFFFFFFFFu;

    for (int it = 0;; ++it) {
        // every role is done with the previous block's buffers; all threads agree on stopping
        tc_fence_before();
        const int stop = __syncthreads_or(*abort != 0);
        tc_fence_after();
        const int64_t base = (int64_t)it * G;
        if (base >= nblk_all || stop) break;
        const int64_t w = base + ((it & 1) ? (G - 1 - (int)blockIdx.x) : (int)blockIdx.x);
        if (w >= nblk_all) continue;
        // ---- the block: sequence b, rows [i0, i0 + nrows) of it ----
        const int b = (int)(w % a.sv.batch);
        const int64_t jb = nblk - 1 - w / a.sv.batch;
        const int64_t q0 = __ldg(a.sv.cu_q + b), sq = __ldg(a.sv.cu_q + b + 1) - q0;
        const int64_t key_base = __ldg(a.sv.cu_k + b), skeys = __ldg(a.sv.cu_k + b + 1) - key_base;
        const int64_t i0 = jb * BM;
        if (i0 >= sq) continue;
        const int nrows = (int)min((int64_t)BM, sq - i0);
        const int64_t pos_first = skeys - sq + i0;
        const int64_t pos_last = pos_first + nrows - 1;
        const int64_t t_first = q0 + i0;
        if (pos_first < 0) {
            if (threadIdx.x == 0) report(st, DSA_ERR_INDEX, t_first);
            continue;
        }
        const int n_tiles = (int)((pos_last + BN) / BN);
        // sample: packed key rows R = g/16 with 16 | g, key_base <= g <= key_base + pos_first
        const int64_t R0 = (key_base + kSampleStride - 1) / kSampleStride;
        const int64_t R1 = (key_base + pos_first) / kSampleStride;  // inclusive
        const int ns = (int)max((int64_t)0, R1 - R0 + 1);
        const int n_stiles = (ns + BN - 1) / BN;
        const bool need_sel = pos_last + 1 > a.k || a.k_rows != nullptr;
        const int first_kind = !need_sel ? SK_STOP : (ns > 0 ? SK_S1 : SK_H);

        if (warp == 0) {
            // ================= TMA producer =================
            if (first_kind != SK_STOP) {
                if (lane == 0) {
                    mbar_arrive_expect_tx(smem_u32(&bars->a_full), A_BYTES);
                    tma_load_2d(sA, &a.tm_u, 0, (int32_t)t_first, smem_u32(&bars->a_full));
                }
                ++nblock;
                int kind = first_kind;
                while (kind != SK_STOP) {
                    const bool samp = kind == SK_S1 || kind == SK_S2;
                    const int nt = samp ? n_stiles : n_tiles;
                    for (int tile = 0; tile < nt; ++tile, ++g) {
                        const uint32_t s = g % NST;
                        if (!wait_warp(smem_u32(&bars->empty[s]), ((g / NST) & 1) ^ 1, abort, st, 0x2101)) break;
                        float* scs = sc_s + s * BN;
                        if (samp) {
                            const int64_t r0 = R0 + (int64_t)tile * BN;
                            for (int i = lane; i < BN; i += 32)
                                scs[i] = (tile * BN + i < ns) ? __ldg(a.k_scale + (r0 + i) * kSampleStride) : 0.f;
                            __syncwarp();
                            if (lane == 0) {
                                mbar_arrive_expect_tx(smem_u32(&bars->full[s]), B_BYTES);
                                tma_load_2d(sB + s * B_BYTES, &a.tm_ks, 0, (int32_t)r0, smem_u32(&bars->full[s]));
                            }
                        } else {
                            const int64_t kr0 = key_base + (int64_t)tile * BN;
                            const bool bulk = (tile + 1) * BN <= pos_last + 1 && ((uintptr_t)(a.k_scale + kr0) & 15) == 0;
                            if (!bulk) {
                                for (int i = lane; i < BN; i += 32)
                                    scs[i] = (tile * BN + i <= pos_last) ? __ldg(a.k_scale + kr0 + i) : 0.f;
                            }
                            __syncwarp();
                            if (lane == 0) {
                                mbar_arrive_expect_tx(smem_u32(&bars->full[s]), B_BYTES + (bulk ? BN * 4 : 0));
                                tma_load_2d(sB + s * B_BYTES, &a.tm_k, 0, (int32_t)kr0, smem_u32(&bars->full[s]));
                                if (bulk) bulk_load(smem_u32(scs), a.k_scale + kr0, BN * 4, smem_u32(&bars->full[s]));
                            }
                        }
                        last_issued[s] = g;
                        __syncwarp();
                    }
                    if (__any_sync(0xffffffffu, *abort != 0)) break;
                    if (!wait_warp(smem_u32(&bars->dec), nsweep & 1, abort, st, 0x2102)) break;
                    ++nsweep;
                    kind = *(volatile int*)&bars->next_kind;
                }
            }
        } else if (warp == 1) {
            // ================= MMA issuer =================
            constexpr uint32_t idesc = idesc_make(0, 0, false, BM, BN);
            if (first_kind != SK_STOP) {
                bool ok = wait_warp(smem_u32(&bars->a_full), nblock & 1, abort, st, 0x2201);
                ++nblock;
                int kind = first_kind;
                while (ok && kind != SK_STOP) {
                    const int nt = (kind == SK_S1 || kind == SK_S2) ? n_stiles : n_tiles;
                    for (int tile = 0; tile < nt; ++tile, ++g) {
                        const uint32_t s = g % NST, ab = g & 1;
                        if (!wait_warp(smem_u32(&bars->full[s]), (g / NST) & 1, abort, st, 0x2202)) { ok = false; break; }
                        if (!wait_warp(smem_u32(&bars->acc_empty[ab]), ((g >> 1) & 1) ^ 1, abort, st, 0x2203)) { ok = false; break; }
                        tc_fence_after();
                        if (lane == 0) {
#pragma unroll
                            for (int ks = 0; ks < 4; ++ks) {
                                const uint64_t ad = sdesc_sw128(sA + ks * 32, 16, 1024);
                                const uint64_t bd = sdesc_sw128(sB + s * B_BYTES + ks * 32, 16, 1024);
                                mma_fp8_ss(tmem + ab * BN, ad, bd, idesc, ks > 0 ? 1u : 0u);
                            }
                            mma_commit(smem_u32(&bars->empty[s]));
                            mma_commit(smem_u32(&bars->acc_full[ab]));
                        }
                        __syncwarp();
                    }
                    if (!ok) break;
                    if (!wait_warp(smem_u32(&bars->dec), nsweep & 1, abort, st, 0x2204)) break;
                    ++nsweep;
                    kind = *(volatile int*)&bars->next_kind;
                }
            }
        } else {
            // ================= epilogue: two threads per query row =================
            const uint32_t quad = warp & 3;
            const int half = (int)(warp - 2) >> 2;
            const int row = (int)(quad * 32 + lane);
            const bool has_row = row < nrows;
            const int64_t t = t_first + row;
            uint32_t* hrow = hist + row;
            const uint32_t hbase = smem_u32(hrow);
            Row rw;
            rw.pos = (int)(pos_first + row);
            const int k_row = (a.k_rows && has_row) ? min(max(__ldg(a.k_rows + t), 0), a.k) : a.k;
            rw.kt = (int)min((int64_t)k_row, (int64_t)rw.pos + 1);
            rw.kind = !has_row ? ROW_NONE : (k_row == 0 ? ROW_EMPTY : (rw.pos + 1 <= k_row ? ROW_PREFIX : ROW_SEL));
            rw.active = rw.kind == ROW_SEL;
            rw.res = RES_NONE;
            rw.need = (uint32_t)rw.kt;
            rw.lo = 0;
            rw.hi = kInfKey + 1;
            rw.s2 = false;
            // rank of the K-th score in the sample of the common prefix
            rw.r = ns > 0 ? max(1, (int)(((double)rw.kt * ns) / (double)(pos_first + 1) + 0.5)) : 0;
            // without a sample: binade bins (bin 0 holds [0, 2^23))
            rw.sh = 23;
            rw.nc0 = 0;
            const float srow = has_row ? __ldg(a.s_row + t) : 0.f;
            const uint64_t srow2 = pk(__float_as_uint(srow), __float_as_uint(srow));
            uint32_t* sel_row = scratch + (size_t)row * a.sel_words;
            uint32_t taken = 0;  // single-valued bucket: members taken so far (both halves agree)

            if (first_kind != SK_STOP) {
                clear_hist(hrow, half);
                asm volatile("bar.sync 1, 256;" ::: "memory");
            }
            int kind = first_kind;
            int nsw_block = 0;
            while (kind != SK_STOP) {
                const bool samp = kind == SK_S1 || kind == SK_S2;
                const int nt = samp ? n_stiles : n_tiles;
                int sh = rw.sh, nc0 = rw.nc0;
                if (kind == SK_S1) { sh = 23; nc0 = 1; }  // bins: 0 negative, 1 [0, 2^23), e+1 binade e
                bool act = has_row && !*abort &&
                           (kind == SK_E ? rw.kind == ROW_SEL
                                         : (kind == SK_S2 ? rw.s2 : (kind == SK_REF ? rw.active : rw.kind == ROW_SEL)));
                if (kind == SK_S1 || kind == SK_H) act = act && rw.kind == ROW_SEL;
                // E: thresholds of the row's bucket
                const uint32_t lo_t = rw.lo == 0 ? 0xFF800000u : rw.lo;  // -inf: every raw score is at or above
                const bool no_above = rw.hi > kInfKey;
                const uint32_t hi_t = no_above ? kInfKey : rw.hi;
                const uint32_t ref_w = rw.hi - rw.lo;
                bool single_any = false;
                if (kind == SK_E) {
                    if (threadIdx.x == 64) bars->any_flag = 0;
                    if (half == 0) lcnt[row] = 0;
                    asm volatile("bar.sync 1, 256;" ::: "memory");
                    if (act && rw.res == RES_SINGLE) bars->any_flag = 1;
                    asm volatile("bar.sync 1, 256;" ::: "memory");
                    single_any = bars->any_flag != 0;
                }
                uint32_t* stage = (uint32_t*)(smem + OFF_STAGE) + (threadIdx.x - 64) * 32;
                for (int tile = 0; tile < nt; ++tile, ++g) {
                    const uint32_t s = g % NST, ab = g & 1;
                    bool ok = wait_warp(smem_u32(&bars->acc_full[ab]), (g >> 1) & 1, abort, st, 0x2301);
                    ok = ok && wait_warp(smem_u32(&bars->full[s]), (g / NST) & 1, abort, st, 0x2302);
                    tc_fence_after();
                    const float* scs = sc_s + s * BN + 128 * half;
                    const int s_half = tile * BN + 128 * half;  // first key (local or sample index) of this half
                    const uint32_t taddr = tmem + ((quad * 32) << 16) + ab * BN + 128 * half;
                    // keys of this half that count: causal for the row, or inside the sample
                    const int last = samp ? ns - 1 : rw.pos;
                    const bool live = ok && act && s_half <= last;
                    // E: the half's four bitmask words (selected, bucket members), shifted in chunk by chunk
                    uint32_t sel0 = 0, sel1 = 0, sel2 = 0, sel3 = 0, mem0 = 0, mem1 = 0, mem2 = 0, mem3 = 0;
#pragma unroll 1
                    for (int pr = 0; pr < 2; ++pr) {
                        uint32_t v[64];
                        if (ok) {
                            tmem_ld64(taddr + pr * 64, v);
                            tmem_wait_ld();
                        }
#pragma unroll
                        for (int hc = 0; hc < 2; ++hc) {
                            uint32_t* vc = v + 32 * hc;
                            const int ch = 2 * pr + hc;
                            const int sb = s_half + ch * 32;
                            uint32_t sw = 0, mw = 0;
                            if (live && sb <= last) {
                                raw_scores(vc, scs + ch * 32, srow2);
                                const int lim = min(31, last - sb);
                                if (kind == SK_REF) {
                                    ref_chunk(vc, rw.lo, ref_w, rw.sh, lim, hbase);
                                } else if (kind != SK_E) {
                                    hist_chunk(vc, sh, nc0, lim, hbase);
                                } else {
                                    const uint32_t lm = lim_mask(lim);
                                    const uint32_t ge = ~below_mask(vc, lo_t) & lm;
                                    const uint32_t ab_m = no_above ? 0u : (~below_mask(vc, hi_t) & lm);
                                    if (rw.res == RES_WHOLE) {
                                        sw = ge;
                                    } else {
                                        sw = rw.res == RES_LIST ? ge : ab_m;
                                        mw = ge & ~ab_m;
                                        if (rw.res == RES_LIST && mw) {
                                            // stage the raw scores, then list the bucket's keys with their score keys
                                            uint4* st4 = (uint4*)stage;
#pragma unroll
                                            for (int q = 0; q < 8; ++q)
                                                st4[q ^ (lane & 7)] =
                                                    make_uint4(vc[4 * q], vc[4 * q + 1], vc[4 * q + 2], vc[4 * q + 3]);
                                            uint32_t m = mw;
                                            while (m) {
                                                const int i = __ffs(m) - 1;
                                                m &= m - 1;
                                                const uint32_t raw = stage[(((i >> 2) ^ (lane & 7)) << 2) | (i & 3)];
                                                const uint32_t slot = atomicAdd(lcnt + row, 1u);
                                                if (slot < (uint32_t)kListCap)
                                                    list[slot * BM + row] = make_uint2((uint32_t)(sb + i), score_key(raw));
                                            }
                                        }
                                    }
                                }
                            }
                            sel0 = sel1, sel1 = sel2, sel2 = sel3, sel3 = sw;
                            mem0 = mem1, mem1 = mem2, mem2 = mem3, mem3 = mw;
                        }
                    }
                    if (kind == SK_E) {
                        if (single_any) {
                            // a single-valued bucket takes its first `need` keys in index order: the
                            // first half's keys of a tile precede the second half's
                            uint32_t cnt = 0;
                            if (live && rw.res == RES_SINGLE)
                                cnt = __popc(mem0) + __popc(mem1) + __popc(mem2) + __popc(mem3);
                            uint32_t* xc = xch + (tile & 1) * 2 * BM;
                            xc[half * BM + row] = cnt;
                            asm volatile("bar.sync %0, 64;" ::"r"(2 + (int)quad) : "memory");
                            const uint32_t c_first = xc[row], c_second = xc[BM + row];
                            if (live && rw.res == RES_SINGLE) {
                                const uint32_t before = taken + (half ? c_first : 0u);
                                uint32_t left = rw.need > before ? rw.need - before : 0u;
                                uint32_t kp = keep_low(mem0, left);
                                sel0 |= kp;
                                left -= __popc(kp);
                                kp = keep_low(mem1, left);
                                sel1 |= kp;
                                left -= __popc(kp);
                                kp = keep_low(mem2, left);
                                sel2 |= kp;
                                left -= __popc(kp);
                                sel3 |= keep_low(mem3, left);
                            }
                            taken += c_first + c_second;
                        }
                        if (live) *(uint4*)(sel_row + 8 * tile + 4 * half) = make_uint4(sel0, sel1, sel2, sel3);
                    }
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) {
                        mbar_arrive(smem_u32(&bars->acc_empty[ab]));
                        mbar_arrive(smem_u32(&bars->empty[s]));
                    }
                }
                // ---- end of sweep: each row reads the histogram (both halves reach the same
                // decision); one thread publishes the next sweep ----
                int next = SK_STOP;
                if (kind != SK_E) {
                    asm volatile("bar.sync 1, 256;" ::: "memory");  // every count of the sweep is in
                    bool flag = false;
                    if (kind == SK_S1) {
                        if (has_row && rw.kind == ROW_SEL) {
                            uint32_t cum;
                            const int b1 = find_bin(hrow, 2, (uint32_t)rw.r, cum);
                            if (b1 < 0) {
                                rw.sh = 0;  // the estimate is zero: exact bins at the bottom, {0} alone in bin 0
                                rw.nc0 = 0;
                            } else {
                                const int e = b1 - 1;  // binade (biased exponent) of the sample's rank-r score
                                int c0 = ((e - 1) << 6) - 1;
                                c0 = min(max(c0, 0), (int)(kInfKey >> 17) - 255);
                                rw.sh = 17;
                                rw.nc0 = -c0;
                                rw.s2 = true;
                                flag = true;
                            }
                        }
                        next = SK_H;
                    } else if (kind == SK_S2) {
                        if (has_row && rw.s2) {
                            uint32_t cum;
                            const int b2 = find_bin(hrow, 1, (uint32_t)rw.r, cum);
                            if (b2 >= 1 && b2 <= 254) {
                                const int64_t tau = (int64_t)(b2 - rw.nc0) << 17;  // lower edge of the estimate's bin
                                int64_t L = tau - ((int64_t)1 << 23);
                                if (L < ((int64_t)1 << 16)) L = (int64_t)1 << 16;
                                int c0 = (int)(L >> 16) - 1;
                                c0 = min(c0, (int)(kInfKey >> 16) - 255);
                                rw.sh = 16;
                                rw.nc0 = -c0;
                            }  // else keep the S2 window (four binades at 1/64) for H
                            rw.s2 = false;
                        }
                        next = SK_H;
                    } else {  // SK_H / SK_REF
                        if (has_row && rw.active) {
                            decide_bucket(rw, hrow, kind == SK_REF);
                            flag = rw.active;
                        }
                    }
                    if (threadIdx.x == 64) bars->any_flag = 0;
                    asm volatile("bar.sync 1, 256;" ::: "memory");  // every histogram read is done
                    clear_hist(hrow, half);
                    if (flag) bars->any_flag = 1;
                    asm volatile("bar.sync 1, 256;" ::: "memory");
                    const bool any = bars->any_flag != 0;
                    if (kind == SK_S1) next = any ? SK_S2 : SK_H;
                    else if (kind == SK_H || kind == SK_REF) next = any ? SK_REF : SK_E;
                }
                if (++nsw_block > 12 && next != SK_STOP) {  // S1 S2 H REF x5 E is the longest chain
                    if (threadIdx.x == 64) report(st, DSA_ERR_INDEX, -4000000 - t_first);
                    next = SK_STOP;
                }
                if (threadIdx.x == 64) {
                    bars->next_kind = *abort ? SK_STOP : next;
                    mbar_arrive(smem_u32(&bars->dec));
                }
                asm volatile("bar.sync 1, 256;" ::: "memory");
                kind = *(volatile int*)&bars->next_kind;
            }
            // ---- finish records ----
            if (half == 0) {
                RowRec rr;
                rr.kind = rw.kind;
                rr.res = rw.res;
                rr.pos = rw.pos;
                rr.kt = rw.kt;
                rr.need = rw.need;
                rrec[row] = rr;
            }
            __threadfence_block();
            asm volatile("bar.sync 1, 256;" ::: "memory");  // every bitmask word and list entry is in
            // ---- finish: one warp per row; bucket losers cleared, bitmask -> ascending indices ----
            const int ew = (int)warp - 2;
            int* stg = (int*)(smem + OFF_B) + ew * kStageInts;
            for (int rr_i = ew * (BM / EPI_WARPS); rr_i < (ew + 1) * (BM / EPI_WARPS); ++rr_i) {
                if (rr_i >= nrows || __any_sync(0xffffffffu, *abort != 0)) break;
                const RowRec rr = rrec[rr_i];
                const int64_t tr = t_first + rr_i;
                int32_t* out = a.idx + tr * a.ld_idx;
                if (rr.kind != ROW_SEL) {
                    const int n = rr.kind == ROW_PREFIX ? rr.pos + 1 : 0;
                    for (int j = lane; j < a.k; j += 32) out[j] = j < n ? j : -1;
                    continue;
                }
                uint32_t* srow_bits = scratch + (size_t)rr_i * a.sel_words;
                if (rr.res == RES_LIST) {
                    // bucket members ranked by (score key desc, index asc); ranks >= need lose
                    const uint32_t C = min(lcnt[rr_i], (uint32_t)kListCap);
                    for (uint32_t j = lane; j < C; j += 32) {
                        const uint2 e = list[j * BM + rr_i];
                        uint32_t rank = 0;
                        for (uint32_t i = 0; i < C; ++i) {
                            const uint2 f = list[i * BM + rr_i];
                            rank += (f.y > e.y || (f.y == e.y && f.x < e.x)) ? 1u : 0u;
                        }
                        if (rank >= rr.need) atomicAnd(srow_bits + (e.x >> 5), ~(1u << (e.x & 31)));
                    }
                    __syncwarp();  // orders the lanes' updates before the reads below
                }
                // bitmask -> indices, staged in shared memory, then written out coalesced;
                // eight words per lane in flight
                const int nw = (rr.pos >> 5) + 1;
                int written = 0;
                for (int gb = 0; gb < nw; gb += 256) {
                    uint32_t wv[8];
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        const int wi = gb + 32 * j + (int)lane;
                        wv[j] = wi < nw ? __ldcg(srow_bits + wi) : 0u;
                    }
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        if (gb + 32 * j >= nw) break;
                        const int wi = gb + 32 * j + (int)lane;
                        uint32_t sbits = wv[j];
                        const int c = __popc(sbits);
                        int incl = c;
#pragma unroll
                        for (int o = 1; o < 32; o <<= 1) {
                            const int y = __shfl_up_sync(0xffffffffu, incl, o);
                            if ((int)lane >= o) incl += y;
                        }
                        const int total = __shfl_sync(0xffffffffu, incl, 31);
                        int off = written + incl - c;
                        while (sbits) {
                            const int i = __ffs(sbits) - 1;
                            sbits &= sbits - 1;
                            if (off < kStageInts) stg[off] = wi * 32 + i;
                            else if (off < a.k) out[off] = wi * 32 + i;
                            ++off;
                        }
                        written += total;
                    }
                }
                __syncwarp();
                const int nstg = min(written, min(kStageInts, a.k));
                for (int j = lane; j < nstg; j += 32) out[j] = stg[j];
                for (int j = written + (int)lane; j < a.k; j += 32) out[j] = -1;
                if (written != rr.kt && !*abort && lane == 0) report(st, DSA_ERR_INDEX, -3000000 - tr);
                __syncwarp();
            }
        }
    }
    // drain on abort: loads and MMAs in flight must land before TMEM and the CTA go away
    if (*abort) {
        if (warp == 0 && lane == 0) {
            for (int s = 0; s < NST; ++s)
                if (last_issued[s] != 0xFFFFFFFFu)
                    mbar_wait(smem_u32(&bars->full[s]), (last_issued[s] / NST) & 1, nullptr, st, 0x2103, 1ll << 28);
        }
        if (warp == 1 && lane == 0) {
            mma_commit(smem_u32(&bars->drain));
            mbar_wait(smem_u32(&bars->drain), 0, nullptr, st, 0x2205, 1ll << 28);
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, 512);
}

}  // namespace sel

int indexer_sel_ctas(int64_t blocks, int sms) {
    const int64_t g = blocks < sms ? blocks : sms;
    return g < 1 ? 1 : (int)g;
}

bool launch_indexer_sel(const IndexerTcArgs& a, int ctas, cudaStream_t s) {
    if (cudaFuncSetAttribute(sel::indexer_sel_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, sel::SMEM) !=
        cudaSuccess)
        return false;
    if (ctas <= 0) return true;
    sel::indexer_sel_kernel<<<ctas, sel::THREADS, sel::SMEM, s>>>(a);
    return cudaGetLastError() == cudaSuccess;
}

}  // namespace dsa
