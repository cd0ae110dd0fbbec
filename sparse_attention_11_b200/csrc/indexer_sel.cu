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
// persistent (one CTA per SM); CTAs take blocks in heaviest-first order from
// an atomic counter in the workspace.  18 warps:
//   warp 0      TMA producer: the block's folded queries (128 x 128 e4m3),
//               key tiles of 256 x 128 e4m3 and their fp32 scales (own ring)
//   warp 1      TMEM owner and MMA issuer: tcgen05.mma kind::f8f6f4,
//               M=128 N=256, fp32 accumulators in two TMEM buffers
//   warps 2..17 epilogue: four threads per query row (its TMEM lane), one per
//               64-column quarter of each tile; the score is
//               ReLU((dot * s_k) * s_row), formed on packed f32x2 pairs
//
// Sweeps of one block (the MMAs are recomputed in each):
//   S1, S2  over a sample of the common causal prefix (every 16th key): a
//           per-row histogram of the sample's scores, by binade (S1) and then
//           at 1/64 binade (S2).  The ranks r -/+ (4 sqrt(r) + 1) around the
//           row's sample rank r = K_t * n_sample / n_keys bound its K-th score.
//   H       over all causal keys: a per-row histogram of 256 bins spanning
//           that band, 1/128 binade or coarser (rows whose band reaches zero
//           keep the score 0 in a bin of its own).  The bin holding the K-th
//           score is the row's bucket [lo, hi).
//   REF     (rare) when a bucket is too large to resolve, a further histogram
//           of the keys inside it at 256 finer bins.
//   E       over all causal keys: a bitmask per row of the keys at or above
//           lo (keys at or above hi are always kept), written to a per-CTA
//           scratch.  A bucket of a single score value takes its first `need`
//           keys in index order (the four threads of a row trade their
//           per-tile counts); a bucket of several values (at most kListCap
//           keys) is listed on chip with the scores, and its losers are
//           cleared after.
// Histogram updates are unpredicated shared-memory reductions: keys that no
// row counts go to bin 0, which no decision reads.
// Finish: one warp per row turns the bitmask into the ascending index row.
#include "dsa_kernels.h"

namespace dsa {
namespace sel {

constexpr int BM = 128;
constexpr int BN = 256;
constexpr int NST = 2;                         // key-code stages (released by the MMAs)
constexpr int NSC = 4;                         // key-scale slots (released by the epilogue)
constexpr int EPI_WARPS = 16;                  // four per TMEM lane quarter: one per 64-column quarter of a tile
constexpr int EPI_THREADS = 32 * EPI_WARPS;
constexpr int THREADS = 64 + EPI_THREADS;
constexpr int kSampleStride = 16;
constexpr int kListCap = 96;
constexpr uint32_t kInfKey = 0x7F800000u;  // score key of +inf (and of NaN)

constexpr uint32_t A_BYTES = BM * 128;
constexpr uint32_t B_BYTES = BN * 128;
constexpr uint32_t OFF_A = 0;
constexpr uint32_t OFF_B = OFF_A + A_BYTES;
constexpr uint32_t OFF_SC = OFF_B + NST * B_BYTES;
constexpr uint32_t OFF_R = OFF_SC + NSC * BN * 4;
constexpr uint32_t R_BYTES = 256 * BM * 4;                  // histogram [256 bins][128 rows]
constexpr uint32_t OFF_LIST = OFF_R;                        // E: bucket lists [kListCap][128 rows] of (index, key)
constexpr uint32_t OFF_STAGE = OFF_R + kListCap * BM * 8;   // E: 64 bytes per epilogue thread
constexpr uint32_t OFF_XCH = OFF_R + R_BYTES;               // E: per-tile member counts [2][4 quarters][128 rows]
constexpr uint32_t OFF_LCNT = OFF_XCH + 2 * 4 * BM * 4;     // bucket list lengths [128]
constexpr uint32_t OFF_RSTATE = OFF_LCNT + BM * 4;          // per-row selection state [128]
constexpr uint32_t OFF_BAR = OFF_RSTATE + BM * 64;
constexpr uint32_t SMEM = OFF_BAR + 256 + 1024;             // + alignment slack
constexpr int kStageInts = (int)(R_BYTES / 4 / EPI_WARPS);  // finish: index staging per warp in the region (2048)
static_assert(OFF_STAGE + EPI_THREADS * 64 <= OFF_R + R_BYTES, "bucket lists and staging exceed the region");
static_assert(SMEM <= 232448, "shared memory");

enum : int { SK_STOP = 0, SK_S1 = 1, SK_S2 = 2, SK_H = 3, SK_REF = 4, SK_E = 5 };
// per-row resolution of its bucket
enum : int { RES_NONE = 0, RES_WHOLE = 1, RES_SINGLE = 2, RES_LIST = 3 };
// per-row kind (finish record)
enum : int { ROW_NONE = 0, ROW_EMPTY = 1, ROW_PREFIX = 2, ROW_SEL = 3 };

struct Bars {
    uint64_t full[NST];
    uint64_t empty[NST];
    uint64_t sc_full[NSC];
    uint64_t sc_empty[NSC];
    uint64_t acc_full[2];
    uint64_t acc_empty[2];
    uint64_t a_full;
    uint64_t dec;
    uint64_t drain;
    uint32_t tmem_base;
    int next_block[2];
    int next_kind;
    int any_flag;
    int zmode;        // the block's H sweep keeps the score 0 in a bin of its own
    int any_h;        // some row needs the H sweep
    int abort;
};

// Per-row selection state, one record per row of the block in shared memory:
// written by the row's first thread (its decisions), read by all four.
struct RowState {
    int pos;          // local position of the query
    int kt;           // K_t = min(k_t, pos + 1)
    int kind;         // ROW_*
    int res;          // RES_*
    int sh, nc0;      // histogram parameters of the next H-type sweep (bin = (bits >> sh) + nc0)
    uint32_t lo, hi;  // bucket of score keys [lo, hi); hi == kInfKey + 1: includes +inf
    uint32_t need;    // keys still to take from the bucket
    int r;            // rank of the K-th score in the sample
    int r_lo, r_hi;   // sample ranks bounding the K-th score (about 4 sigma either side)
    int s2;           // takes part in S2
    int active;       // takes part in the next H / REF sweep
    int pad[2];
};
static_assert(sizeof(RowState) == 64, "RowState layout");
static_assert(sizeof(Bars) <= 256, "barrier block");

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

// Add 1 to the shared-memory counter at `addr`.  Every key of a chunk is
// counted (no predicate, no branch); keys that no decision needs (below the
// window, past the causal limit, outside the bucket) go to bin 0, which no
// decision reads.
DSA_DEV void red_add(uint32_t addr) { asm volatile("red.shared.add.u32 [%0], 1;" ::"r"(addr) : "memory"); }

// Histogram of 32 raw scores, bin = clamp((bits >> sh) + nc0, 0, 255) on the
// raw bits (nc0 = -c0).  With c0 >= 0 every non-positive raw score lands in
// bin 0 with the score +0, and with (kInfKey >> sh) - c0 >= 255 NaN lands in
// bin 255 with +inf, so the bins are those of the score keys.  Columns past
// `lim` go to bin 0.  hbase is the shared address of the row's bin 0; bin b is
// b * 512 bytes further.
DSA_DEV void hist_chunk(const uint32_t* v, int sh, int nc0, int lim, uint32_t hbase) {
    if (lim >= 31) {
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            const int bin = __viaddmin_s32_relu((int)v[i] >> sh, nc0, 255);
            red_add(hbase + (bin << 9));
        }
    } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            const int bin = __viaddmin_s32_relu((int)v[i] >> sh, nc0, 255);
            red_add(hbase + ((i <= lim ? bin : 0) << 9));
        }
    }
}

// The same with the zero score in a bin of its own: bin 0 holds exactly the
// score 0 (every non-positive raw score), bin 1 the positive scores below the
// window, bins 2..254 the window, bin 255 the rest.  For blocks with rows
// whose K-th score may be 0 or close to it.  Bin 0 is not read either (a K-th
// score of 0 is a single-valued bucket, taken in index order), so the columns
// past `lim` go there too.
DSA_DEV void hist_chunk_z(const uint32_t* v, int sh, int nc0, int lim, uint32_t hbase) {
#pragma unroll
    for (int i = 0; i < 32; ++i) {
        const int t = ((int)v[i] >> sh) + nc0;
        const int bin = __vimin_s32_relu(max(t, min((int)v[i], 1)), 255);
        red_add(hbase + ((i <= lim ? bin : 0) << 9));
    }
}

// Histogram of the keys inside a bucket [lo, lo + w): bin 1 + ((key - lo) >> sh);
// the other keys go to bin 0.
DSA_DEV void ref_chunk(const uint32_t* v, uint32_t lo, uint32_t w, int sh, int lim, uint32_t hbase) {
#pragma unroll
    for (int i = 0; i < 32; ++i) {
        const uint32_t d = score_key(v[i]) - lo;
        const int bin = (d < w && i <= lim) ? 1 + (int)(d >> sh) : 0;
        red_add(hbase + (bin << 9));
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

DSA_DEV void clear_hist(uint32_t* hrow, int quarter) {
#pragma unroll 8
    for (int i = 64 * quarter; i < 64 * quarter + 64; ++i) hrow[i << 7] = 0u;
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
__device__ __noinline__ void decide_bucket(RowState& rw, const uint32_t* hrow, bool ref, bool zmode) {
    uint32_t cum;
    const int b = find_bin(hrow, 1, rw.need, cum);
    uint32_t lo, hi, c;
    bool known = true;
    if (ref) {
        // bins 1..254 of the previous bucket [rw.lo, rw.hi) at 2^sh keys each
        if (b < 1) {  // cannot happen (the bucket holds at least `need` keys); the count check reports it
            rw.res = RES_WHOLE;
            rw.active = 0;
            return;
        }
        lo = rw.lo + ((uint32_t)(b - 1) << rw.sh);
        const uint64_t h64 = (uint64_t)lo + ((uint64_t)1 << rw.sh);
        hi = h64 < (uint64_t)rw.hi ? (uint32_t)h64 : rw.hi;
        c = hrow[b << 7];
    } else {
        const int c0 = -rw.nc0;
        if (b < 1) {  // the K-th score lies in bin 0: below the window (zmode: the score 0 itself)
            lo = 0;
            hi = zmode ? 1u : (uint32_t)(1 + c0) << rw.sh;
            known = false;
            c = 0;
        } else if (b == 1 && zmode) {  // the positive scores below the window
            lo = 1;
            hi = (uint32_t)(2 + c0) << rw.sh;
            c = hrow[1 << 7];
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
// Stage 16 raw scores of this thread (one 64-byte row of four 16-byte chunks,
// the chunk order rotated by lane so that eight lanes cover every bank).
DSA_DEV void stage16(uint4* row, const uint32_t* v, uint32_t lane) {
    const uint32_t r = (lane >> 1) & 3;
#pragma unroll
    for (int q = 0; q < 4; ++q) row[q ^ r] = make_uint4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
}
DSA_DEV uint32_t staged(const uint32_t* row, int i, uint32_t lane) {
    return row[((((uint32_t)i >> 2) ^ ((lane >> 1) & 3)) << 2) | ((uint32_t)i & 3)];
}

// After the emission sweep: a listed bucket (at most kListCap keys with their
// score keys, in shared memory) keeps its `need` best (score key desc, index
// asc); the others are cleared from the row's bitmask.  One warp per row.
__device__ __noinline__ void resolve_lists(const int64_t sel_words, uint32_t* scratch, const RowState* rstate,
                                           const uint2* list, const uint32_t* lcnt, int ew, uint32_t lane, int nrows) {
    constexpr int kRowsPerWarp = BM / EPI_WARPS;
    for (int j = 0; j < kRowsPerWarp; ++j) {
        const int rr_i = ew * kRowsPerWarp + j;
        if (rr_i >= nrows) break;
        const RowState& rr = rstate[rr_i];
        if (rr.kind != ROW_SEL || rr.res != RES_LIST) continue;
        const uint32_t need = rr.need;
        // entries name keys of this row (0..pos): checked before the bitmask is touched
        const uint32_t nk = (uint32_t)rr.pos + 1;
        uint32_t* srow_bits = scratch + (size_t)rr_i * sel_words;
        const uint32_t C = min(lcnt[rr_i], (uint32_t)kListCap);
        const uint2 e0 = lane < C ? list[lane * BM + rr_i] : make_uint2(0u, 0u);
        const uint2 e1 = lane + 32 < C ? list[(lane + 32) * BM + rr_i] : make_uint2(0u, 0u);
        const uint2 e2 = lane + 64 < C ? list[(lane + 64) * BM + rr_i] : make_uint2(0u, 0u);
        uint32_t r0 = 0, r1 = 0, r2 = 0;
#pragma unroll 4
        for (uint32_t i = 0; i < C; ++i) {
            const uint2 f = list[i * BM + rr_i];
            r0 += (f.y > e0.y || (f.y == e0.y && f.x < e0.x)) ? 1u : 0u;
            r1 += (f.y > e1.y || (f.y == e1.y && f.x < e1.x)) ? 1u : 0u;
            r2 += (f.y > e2.y || (f.y == e2.y && f.x < e2.x)) ? 1u : 0u;
        }
        if (lane < C && r0 >= need && e0.x < nk) atomicAnd(srow_bits + (e0.x >> 5), ~(1u << (e0.x & 31)));
        if (lane + 32 < C && r1 >= need && e1.x < nk) atomicAnd(srow_bits + (e1.x >> 5), ~(1u << (e1.x & 31)));
        if (lane + 64 < C && r2 >= need && e2.x < nk) atomicAnd(srow_bits + (e2.x >> 5), ~(1u << (e2.x & 31)));
    }
}

// After S1 (binade histogram of the sample): where the row's H window goes.
// Returns bit 0: S2 refines it; bit 1: the block needs the zero-separating
// histogram; bit 2: the row needs H without S2.
__device__ __noinline__ int decide_s1(RowState& rw, const uint32_t* hrow) {
    // binades (bin = biased exponent + 1) of the sample's scores at the ranks bounding the K-th;
    // -1 when the rank reaches the zero / denormal bins
    uint32_t cum;
    const int b_top = find_bin(hrow, 2, (uint32_t)rw.r_lo, cum);
    const int b_bot = find_bin(hrow, 2, (uint32_t)rw.r_hi, cum);
    if (b_top < 0) {
        // the K-th score is 0 or tiny: zero in bin 0, then binades
        rw.sh = 23;
        rw.nc0 = 0;
        return 2 | 4;
    }
    if (b_bot < 0) {
        // the band reaches 0: zero in bin 0, then 1/32-binade bins up to two binades above the band
        // (eight binades; lower scores in bin 1)
        const int e_top = b_top - 1;
        const int c0 = min(max(((e_top + 2) << 5) - 255, 0), (int)(kInfKey >> 18) - 255);
        rw.sh = 18;
        rw.nc0 = -c0;
        return 2 | 4;
    }
    if (b_top - b_bot <= 1) {
        // a narrow band: S2 refines it at 1/64 binade over four binades
        const int e_bot = b_bot - 1;
        int c0 = ((e_bot - 1) << 6) - 1;
        c0 = min(max(c0, 0), (int)(kInfKey >> 17) - 255);
        rw.sh = 17;
        rw.nc0 = -c0;
        rw.s2 = 1;
        return 1;
    }
    // a wide band: H covers it from one binade below to two above
    const int e_bot = b_bot - 1, e_top = b_top - 1;
    const int64_t L = (int64_t)max(e_bot - 1, 1) << 23;
    const int64_t span = ((int64_t)(e_top + 2) << 23) - L;
    int sh2 = 16;
    while (((int64_t)254 << sh2) < span && sh2 < 23) ++sh2;
    int c0 = (int)(L >> sh2) - 1;
    c0 = min(max(c0, 0), (int)(kInfKey >> sh2) - 255);
    rw.sh = sh2;
    rw.nc0 = -c0;
    return 4;
}

// After S2 (1/64-binade histogram of the sample over four binades): the H
// window, 254 bins from 1/8 binade below the band (the rank r_hi bin) to 1/8
// binade above it (the rank r_lo bin), as fine as fit (1/256 binade or coarser).
__device__ __noinline__ void decide_s2(RowState& rw, const uint32_t* hrow) {
    uint32_t cum;
    const int b2_top = find_bin(hrow, 1, (uint32_t)rw.r_lo, cum);
    const int b2_bot = find_bin(hrow, 1, (uint32_t)rw.r_hi, cum);
    const int c0s = -rw.nc0;
    if (b2_top >= 1 && b2_top <= 254 && b2_bot >= 1 && b2_bot <= b2_top) {
        const int64_t lo_e = ((int64_t)(b2_bot + c0s) << 17) - ((int64_t)1 << 20);
        const int64_t hi_e = ((int64_t)(b2_top + c0s + 1) << 17) + ((int64_t)1 << 20);
        int sh2 = 15;
        while (((int64_t)254 << sh2) < hi_e - max(lo_e, (int64_t)1 << sh2) && sh2 < 23) ++sh2;
        const int64_t L = lo_e < ((int64_t)1 << sh2) ? ((int64_t)1 << sh2) : lo_e;
        int c0 = (int)(L >> sh2) - 1;
        c0 = min(max(c0, 0), (int)(kInfKey >> sh2) - 255);
        rw.sh = sh2;
        rw.nc0 = -c0;
    }  // else H over the S2 window (four binades at 1/64)
    rw.s2 = 0;
}

// The finish: one warp per row turns the row's bitmask into its ascending
// index row (lanes take eight consecutive words each, indices are staged in
// shared memory and written out coalesced), -1 after the K_t-th.
__device__ __noinline__ void finish_rows(int32_t* idx, int64_t ld_idx, const int k_out, const int64_t sel_words,
                                         StatusHdr* st, const uint32_t* scratch, const RowState* rstate, int* stg,
                                         int64_t t_first, int nrows, int ew, uint32_t lane, volatile int* abort) {
    constexpr int kRowsPerWarp = BM / EPI_WARPS;
    const int kcap = min(kStageInts, k_out);  // indices past it go straight to memory
    for (int j = 0; j < kRowsPerWarp; ++j) {
        const int rr_i = ew * kRowsPerWarp + j;
        if (rr_i >= nrows || __any_sync(0xffffffffu, *abort != 0)) break;
        const int kind = rstate[rr_i].kind, pos = rstate[rr_i].pos, kt = rstate[rr_i].kt;
        const int64_t tr = t_first + rr_i;
        int32_t* out = idx + tr * ld_idx;
        if (kind != ROW_SEL) {
            const int n = kind == ROW_PREFIX ? pos + 1 : 0;
            for (int jj = lane; jj < k_out; jj += 32) out[jj] = jj < n ? jj : -1;
            continue;
        }
        const uint32_t* srow_bits = scratch + (size_t)rr_i * sel_words;
        const int nw = (pos >> 5) + 1;
        int written = 0;
        for (int gb = 0; gb < nw; gb += 256) {
            const int w0 = gb + 8 * (int)lane;
            uint4 wa = make_uint4(0u, 0u, 0u, 0u), wb = make_uint4(0u, 0u, 0u, 0u);
            if (w0 < nw) {
                wa = __ldcg((const uint4*)(srow_bits + w0));
                wb = __ldcg((const uint4*)(srow_bits + w0 + 4));
            }
            uint32_t wv[8] = {wa.x, wa.y, wa.z, wa.w, wb.x, wb.y, wb.z, wb.w};
#pragma unroll
            for (int q = 0; q < 8; ++q)
                if (w0 + q >= nw) wv[q] = 0u;  // words past the row's last key are not written
            int c = 0;
#pragma unroll
            for (int q = 0; q < 8; ++q) c += __popc(wv[q]);
            int incl = c;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, incl, o);
                if ((int)lane >= o) incl += y;
            }
            const int total = __shfl_sync(0xffffffffu, incl, 31);
            int off = written + incl - c;
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                uint32_t sbits = wv[q];
                const int kb = (w0 + q) * 32;
                while (sbits) {
                    const int i = __ffs(sbits) - 1;
                    sbits &= sbits - 1;
                    if (off < kcap) stg[off] = kb + i;
                    else if (off < k_out) out[off] = kb + i;
                    ++off;
                }
            }
            written += total;
        }
        __syncwarp();
        const int nstg = min(written, kcap);
        if ((((uintptr_t)out) & 15) == 0) {
            const int n4 = nstg >> 2;
            for (int jj = lane; jj < n4; jj += 32) ((int4*)out)[jj] = ((const int4*)stg)[jj];
            for (int jj = 4 * n4 + (int)lane; jj < nstg; jj += 32) out[jj] = stg[jj];
        } else {
            for (int jj = lane; jj < nstg; jj += 32) out[jj] = stg[jj];
        }
        for (int jj = written + (int)lane; jj < k_out; jj += 32) out[jj] = -1;
        if (written != kt && !*abort && lane == 0) report(st, DSA_ERR_INDEX, -3000000 - tr);
        __syncwarp();
    }
}

__global__ void __maxnreg__(96) indexer_sel_kernel(const __grid_constant__ IndexerTcArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    Bars* bars = (Bars*)(smem + OFF_BAR);
    float* sc_s = (float*)(smem + OFF_SC);
    uint32_t* hist = (uint32_t*)(smem + OFF_R);
    uint2* list = (uint2*)(smem + OFF_LIST);
    uint32_t* xch = (uint32_t*)(smem + OFF_XCH);
    uint32_t* lcnt = (uint32_t*)(smem + OFF_LCNT);
    RowState* rstate = (RowState*)(smem + OFF_RSTATE);
    const uint32_t warp = warp_id(), lane = lane_id();
    StatusHdr* st = a.st;
    volatile int* abort = &bars->abort;

    if (threadIdx.x == 0) {
        for (int i = 0; i < NST; ++i) {
            mbar_init(smem_u32(&bars->full[i]), 1);
            mbar_init(smem_u32(&bars->empty[i]), 1);
        }
        for (int i = 0; i < NSC; ++i) {
            mbar_init(smem_u32(&bars->sc_full[i]), 1);
            mbar_init(smem_u32(&bars->sc_empty[i]), EPI_WARPS);
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
    uint32_t* scratch = a.sel_bits + (size_t)blockIdx.x * BM * (size_t)a.sel_words;

    // pipeline counters, continued across blocks and sweeps
    uint32_t g = 0;          // tiles
    uint32_t nsweep = 0;     // decisions (dec phases)
    uint32_t nblock = 0;     // blocks that loaded their queries (a_full phases)
    uint32_t last_issued[NST];  // producer: last tile issued into each stage (abort drain)
    uint32_t last_sc[NSC];      // producer: last tile whose scales went into each slot
    for (int i = 0; i < NST; ++i) last_issued[i] = 0xFFFFFFFFu;
    for (int i = 0; i < NSC; ++i) last_sc[i] = 0xFFFFFFFFu;

    for (int it = 0;; ++it) {
        // blocks are handed out heaviest first through a counter in the workspace header
        if (threadIdx.x == 0) bars->next_block[it & 1] = (int)atomicAdd(a.work_counter, 1u);
        // every role is done with the previous block's buffers; all threads agree on stopping
        tc_fence_before();
        const int stop = __syncthreads_or(*abort != 0);
        tc_fence_after();
        const int64_t w = bars->next_block[it & 1];
        if (w >= nblk_all || stop) break;
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
                        const uint32_t s = g % NST, c = g % NSC;
                        // key codes: the stage is free once the MMAs of tile g - NST completed
                        if (!wait_warp(smem_u32(&bars->empty[s]), ((g / NST) & 1) ^ 1, abort, st, 0x2101)) break;
                        if (lane == 0) {
                            mbar_arrive_expect_tx(smem_u32(&bars->full[s]), B_BYTES);
                            if (samp)
                                tma_load_2d(sB + s * B_BYTES, &a.tm_ks, 0, (int32_t)(R0 + (int64_t)tile * BN),
                                            smem_u32(&bars->full[s]));
                            else
                                tma_load_2d(sB + s * B_BYTES, &a.tm_k, 0, (int32_t)(key_base + (int64_t)tile * BN),
                                            smem_u32(&bars->full[s]));
                        }
                        last_issued[s] = g;
                        // key scales: the slot is free once the epilogue read tile g - NSC
                        if (!wait_warp(smem_u32(&bars->sc_empty[c]), ((g / NSC) & 1) ^ 1, abort, st, 0x2104)) break;
                        float* scs = sc_s + c * BN;
                        last_sc[c] = g;
                        if (samp) {
                            const int64_t r0 = R0 + (int64_t)tile * BN;
                            for (int i = lane; i < BN; i += 32)
                                scs[i] = (tile * BN + i < ns) ? __ldg(a.k_scale + (r0 + i) * kSampleStride) : 0.f;
                            __syncwarp();
                            if (lane == 0) mbar_arrive(smem_u32(&bars->sc_full[c]));
                        } else {
                            const int64_t kr0 = key_base + (int64_t)tile * BN;
                            const bool bulk = (tile + 1) * BN <= pos_last + 1 && ((uintptr_t)(a.k_scale + kr0) & 15) == 0;
                            if (bulk) {
                                if (lane == 0) {
                                    mbar_arrive_expect_tx(smem_u32(&bars->sc_full[c]), BN * 4);
                                    bulk_load(smem_u32(scs), a.k_scale + kr0, BN * 4, smem_u32(&bars->sc_full[c]));
                                }
                            } else {
                                for (int i = lane; i < BN; i += 32)
                                    scs[i] = (tile * BN + i <= pos_last) ? __ldg(a.k_scale + kr0 + i) : 0.f;
                                __syncwarp();
                                if (lane == 0) mbar_arrive(smem_u32(&bars->sc_full[c]));
                            }
                        }
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
            // ================= epilogue: four threads per query row =================
            const int ew = (int)warp - 2;          // epilogue warp 0..15
            const uint32_t quad = warp & 3;        // TMEM lane quarter (rows 32 quad ..)
            const int quarter = ew >> 2;           // 64-column quarter of every tile
            const int row = (int)(quad * 32 + lane);
            const bool has_row = row < nrows;
            const int64_t t = t_first + row;
            uint32_t* hrow = hist + row;
            const uint32_t hbase = smem_u32(hrow);
            RowState* rsp = rstate + row;
            if (quarter == 0) {
                RowState rw;
                rw.pos = (int)(pos_first + row);
                const int k_row = (a.k_rows && has_row) ? min(max(__ldg(a.k_rows + t), 0), a.k) : a.k;
                rw.kt = (int)min((int64_t)k_row, (int64_t)rw.pos + 1);
                rw.kind = !has_row ? ROW_NONE : (k_row == 0 ? ROW_EMPTY : (rw.pos + 1 <= k_row ? ROW_PREFIX : ROW_SEL));
                rw.res = RES_NONE;
                rw.sh = 23;  // without a sample: binade bins (bin 0 holds [0, 2^23))
                rw.nc0 = 0;
                rw.lo = 0;
                rw.hi = kInfKey + 1;
                rw.need = (uint32_t)rw.kt;
                // rank of the K-th score in the sample of the common prefix, and the ranks about
                // 4 sigma either side
                rw.r = ns > 0 ? max(1, (int)(((double)rw.kt * ns) / (double)(pos_first + 1) + 0.5)) : 0;
                const int dr = (int)ceilf(4.0f * sqrtf((float)rw.r)) + 1;
                rw.r_lo = max(1, rw.r - dr);
                rw.r_hi = rw.r + dr;
                rw.s2 = 0;
                rw.active = rw.kind == ROW_SEL;
                rw.pad[0] = rw.pad[1] = 0;
                *rsp = rw;
            }
            const float srow = has_row ? __ldg(a.s_row + t) : 0.f;
            const uint64_t srow2 = pk(__float_as_uint(srow), __float_as_uint(srow));
            uint32_t* sel_row = scratch + (size_t)row * a.sel_words;
            uint4* stage = (uint4*)(smem + OFF_STAGE) + (threadIdx.x - 64) * 4;
            uint32_t taken = 0;  // single-valued bucket: members taken so far (the row's four threads agree)

            if (first_kind != SK_STOP) clear_hist(hrow, quarter);
            if (threadIdx.x == 64) {
                bars->zmode = 0;
                bars->any_h = 0;
            }
            asm volatile("bar.sync 1, %0;" ::"n"(EPI_THREADS) : "memory");  // row states in, bins cleared
            int kind = first_kind;
            int nsw_block = 0;
            while (kind != SK_STOP) {
                const bool samp = kind == SK_S1 || kind == SK_S2;
                const int nt = samp ? n_stiles : n_tiles;
                const bool zmode = bars->zmode != 0;
                const int row_kind = rsp->kind;
                const bool act = has_row && !*abort &&
                                 (kind == SK_S2 ? rsp->s2 != 0
                                                : (kind == SK_REF || kind == SK_H ? rsp->active != 0 : row_kind == ROW_SEL));
                const int last = samp ? ns - 1 : rsp->pos;  // keys that count: causal, or inside the sample
                int next = SK_STOP;
                if (kind == SK_E) {
                    // ---------------- emission sweep ----------------
                    const int res = rsp->res;
                    const uint32_t lo = rsp->lo, hi = rsp->hi, need = rsp->need;
                    const uint32_t lo_t = lo == 0 ? 0xFF800000u : lo;  // -inf: every raw score is at or above
                    const uint32_t above_en = hi > kInfKey ? 0u : 0xFFFFFFFFu;
                    const uint32_t hi_t = hi > kInfKey ? kInfKey : hi;
                    const bool sel_ge = res == RES_WHOLE || res == RES_LIST;
                    const uint32_t mem_en = res == RES_WHOLE ? 0u : 0xFFFFFFFFu;
                    const bool capture = res == RES_LIST;
                    const bool single = res == RES_SINGLE;
                    if (threadIdx.x == 64) bars->any_flag = 0;
                    if (quarter == 0) lcnt[row] = 0;
                    asm volatile("bar.sync 1, %0;" ::"n"(EPI_THREADS) : "memory");
                    if (act && single) bars->any_flag = 1;
                    asm volatile("bar.sync 1, %0;" ::"n"(EPI_THREADS) : "memory");
                    const bool single_any = bars->any_flag != 0;
                    for (int tile = 0; tile < nt; ++tile, ++g) {
                        const uint32_t c = g % NSC, ab = g & 1;
                        bool ok = wait_warp(smem_u32(&bars->acc_full[ab]), (g >> 1) & 1, abort, st, 0x2301);
                        ok = ok && wait_warp(smem_u32(&bars->sc_full[c]), (g / NSC) & 1, abort, st, 0x2302);
                        tc_fence_after();
                        const float* scs = sc_s + c * BN + 64 * quarter;
                        const int s_q = tile * BN + 64 * quarter;
                        const bool live = ok && act && s_q <= last;
                        uint32_t sel0 = 0, sel1 = 0, mem0 = 0, mem1 = 0;
#pragma unroll 1
                        for (int hc = 0; hc < 2; ++hc) {
                            uint32_t vc[32];
                            if (ok) {
                                tmem_ld32(tmem + ((quad * 32) << 16) + ab * BN + 64 * quarter + 32 * hc, vc);
                                tmem_wait_ld();
                            }
                            const int sb = s_q + 32 * hc;
                            uint32_t sw = 0, mw = 0;
                            if (live && sb <= last) {
                                raw_scores(vc, scs + 32 * hc, srow2);
                                const uint32_t lm = lim_mask(min(31, last - sb));
                                const uint32_t ge = ~below_mask(vc, lo_t) & lm;
                                const uint32_t ab_m = ~below_mask(vc, hi_t) & lm & above_en;
                                sw = sel_ge ? ge : ab_m;
                                mw = ge & ~ab_m & mem_en;
                                if (capture && mw) {
                                    // a listed bucket's keys with their score keys, 16 staged at a time
#pragma unroll
                                    for (int h16 = 0; h16 < 2; ++h16) {
                                        uint32_t m = (mw >> (16 * h16)) & 0xFFFFu;
                                        if (m) {
                                            stage16(stage, vc + 16 * h16, lane);
                                            while (m) {
                                                const int i = __ffs(m) - 1;
                                                m &= m - 1;
                                                const uint32_t slot = atomicAdd(lcnt + row, 1u);
                                                if (slot < (uint32_t)kListCap)
                                                    list[slot * BM + row] =
                                                        make_uint2((uint32_t)(sb + 16 * h16 + i),
                                                                   score_key(staged((const uint32_t*)stage, i, lane)));
                                            }
                                        }
                                    }
                                }
                            }
                            sel0 = sel1, sel1 = sw;
                            mem0 = mem1, mem1 = mw;
                        }
                        if (single_any) {
                            // a single-valued bucket takes its first `need` keys in index order: the
                            // quarters of a tile in order
                            uint32_t cnt = 0;
                            if (live && single) cnt = __popc(mem0) + __popc(mem1);
                            uint32_t* xc = xch + (tile & 1) * 4 * BM;
                            xc[quarter * BM + row] = cnt;
                            asm volatile("bar.sync %0, 128;" ::"r"(2 + (int)quad) : "memory");
                            const uint32_t c0 = xc[row], c1 = xc[BM + row], c2 = xc[2 * BM + row], c3 = xc[3 * BM + row];
                            if (live && single) {
                                const uint32_t before = taken + (quarter > 0 ? c0 : 0u) + (quarter > 1 ? c1 : 0u) +
                                                        (quarter > 2 ? c2 : 0u);
                                uint32_t left = need > before ? need - before : 0u;
                                const uint32_t kp = keep_low(mem0, left);
                                sel0 |= kp;
                                left -= __popc(kp);
                                sel1 |= keep_low(mem1, left);
                            }
                            taken += c0 + c1 + c2 + c3;
                        }
                        if (live) *(uint2*)(sel_row + 8 * tile + 2 * quarter) = make_uint2(sel0, sel1);
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) {
                            mbar_arrive(smem_u32(&bars->acc_empty[ab]));
                            mbar_arrive(smem_u32(&bars->sc_empty[c]));
                        }
                    }
                    // ---- listed buckets keep their `need` best ----
                    asm volatile("bar.sync 1, %0;" ::"n"(EPI_THREADS) : "memory");  // every list entry is in
                    resolve_lists(a.sel_words, scratch, rstate, (const uint2*)(smem + OFF_LIST), lcnt, ew, lane, nrows);
                    __threadfence_block();
                    next = SK_STOP;
                } else {
                    // ---------------- histogram sweeps: S1, S2, H, REF ----------------
                    int sh = rsp->sh, nc0 = rsp->nc0;
                    if (kind == SK_S1) { sh = 23; nc0 = 1; }  // bins: 0 negative, 1 [0, 2^23), e+1 binade e
                    const int hmode = kind == SK_REF ? 2 : (kind == SK_H && zmode ? 1 : 0);
                    const uint32_t ref_lo = rsp->lo, ref_w = rsp->hi - rsp->lo;
                    for (int tile = 0; tile < nt; ++tile, ++g) {
                        const uint32_t c = g % NSC, ab = g & 1;
                        bool ok = wait_warp(smem_u32(&bars->acc_full[ab]), (g >> 1) & 1, abort, st, 0x2303);
                        ok = ok && wait_warp(smem_u32(&bars->sc_full[c]), (g / NSC) & 1, abort, st, 0x2304);
                        tc_fence_after();
                        const float* scs = sc_s + c * BN + 64 * quarter;
                        const int s_q = tile * BN + 64 * quarter;
                        const bool live = ok && act && s_q <= last;
#pragma unroll 1
                        for (int hc = 0; hc < 2; ++hc) {
                            uint32_t vc[32];
                            if (ok) {
                                tmem_ld32(tmem + ((quad * 32) << 16) + ab * BN + 64 * quarter + 32 * hc, vc);
                                tmem_wait_ld();
                            }
                            const int sb = s_q + 32 * hc;
                            if (live && sb <= last) {
                                raw_scores(vc, scs + 32 * hc, srow2);
                                const int lim = min(31, last - sb);
                                if (hmode == 0) hist_chunk(vc, sh, nc0, lim, hbase);
                                else if (hmode == 1) hist_chunk_z(vc, sh, nc0, lim, hbase);
                                else ref_chunk(vc, ref_lo, ref_w, sh, lim, hbase);
                            }
                        }
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) {
                            mbar_arrive(smem_u32(&bars->acc_empty[ab]));
                            mbar_arrive(smem_u32(&bars->sc_empty[c]));
                        }
                    }
                    // ---- end of sweep: the row's first thread reads the histogram and decides ----
                    asm volatile("bar.sync 1, %0;" ::"n"(EPI_THREADS) : "memory");  // every count of the sweep is in
                    bool flag = false, zflag = false, hflag = false;
                    if (quarter == 0 && has_row && row_kind == ROW_SEL) {
                        if (kind == SK_S1) {
                            const int f = decide_s1(*rsp, hrow);
                            flag = f & 1;
                            zflag = (f & 2) != 0;
                            hflag = (f & 4) != 0;
                        } else if (kind == SK_S2) {
                            if (rsp->s2) {
                                decide_s2(*rsp, hrow);
                                hflag = true;
                            }
                        } else if (rsp->active) {  // SK_H / SK_REF
                            decide_bucket(*rsp, hrow, kind == SK_REF, zmode);
                            flag = rsp->active != 0;
                        }
                    }
                    if (threadIdx.x == 64) bars->any_flag = 0;  // any_h accumulates over the block's sweeps
                    asm volatile("bar.sync 1, %0;" ::"n"(EPI_THREADS) : "memory");  // every histogram read is done
                    clear_hist(hrow, quarter);
                    if (flag) bars->any_flag = 1;
                    if (zflag) bars->zmode = 1;
                    if (hflag) bars->any_h = 1;
                    asm volatile("bar.sync 1, %0;" ::"n"(EPI_THREADS) : "memory");
                    const bool any = bars->any_flag != 0, any_h = bars->any_h != 0;
                    if (kind == SK_S1) next = any ? SK_S2 : (any_h ? SK_H : SK_E);
                    else if (kind == SK_S2) next = any_h ? SK_H : SK_E;
                    else next = any ? SK_REF : SK_E;
                }
                if (++nsw_block > 12 && next != SK_STOP) {  // the longest chain is S1 S2 H REF x5 E
                    if (threadIdx.x == 64) report(st, DSA_ERR_INDEX, -4000000 - t_first);
                    next = SK_STOP;
                }
                if (threadIdx.x == 64) {
                    bars->next_kind = *abort ? SK_STOP : next;
                    mbar_arrive(smem_u32(&bars->dec));
                }
                asm volatile("bar.sync 1, %0;" ::"n"(EPI_THREADS) : "memory");
                kind = *(volatile int*)&bars->next_kind;
            }
            __threadfence_block();
            asm volatile("bar.sync 1, %0;" ::"n"(EPI_THREADS) : "memory");  // every bitmask word is final
            // ---- finish: bitmask -> ascending indices, staged in the region ----
            finish_rows(a.idx, a.ld_idx, a.k, a.sel_words, st, scratch, rstate, (int*)(smem + OFF_R) + ew * kStageInts,
                        t_first, nrows, ew, lane, abort);
        }
    }
    // drain on abort: loads and MMAs in flight must land before TMEM and the CTA go away
    if (*abort) {
        if (warp == 0 && lane == 0) {
            for (int s = 0; s < NST; ++s)
                if (last_issued[s] != 0xFFFFFFFFu)
                    mbar_wait(smem_u32(&bars->full[s]), (last_issued[s] / NST) & 1, nullptr, st, 0x2103, 1ll << 28);
            for (int c = 0; c < NSC; ++c)
                if (last_sc[c] != 0xFFFFFFFFu)
                    mbar_wait(smem_u32(&bars->sc_full[c]), (last_sc[c] / NSC) & 1, nullptr, st, 0x2105, 1ll << 28);
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
    // the register file is split over the SM's four partitions: 18 warps fit only at <= 96 registers
    cudaFuncAttributes fa;
    if (cudaFuncGetAttributes(&fa, sel::indexer_sel_kernel) != cudaSuccess || fa.maxThreadsPerBlock < sel::THREADS)
        return false;
    if (ctas <= 0) return true;
    sel::indexer_sel_kernel<<<ctas, sel::THREADS, sel::SMEM, s>>>(a);
    return cudaGetLastError() == cudaSuccess;
}

}  // namespace dsa
