/*
 * dsa_oracle.c -- plain, slow, obviously-correct CPU oracle for the
 * DeepSeek Sparse Attention (DSA) forward hot path.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or
 * call this file; only the tests, the package's smoke check and the
 * benchmark's CPU-baseline leg do.  It shares no code, header, table or
 * helper with the CUDA library.
 *
 * Source pages (cited by title and section):
 *   [V32] "DeepSeek-V3.2与稀疏注意力技术革新" (intelliparadigm.com)
 *         §2.2 lightning indexer: I[t,s] = ReLU(q_t . W_index . k_s), 128-dim
 *              FP8 indexer keys;
 *         §2.3 fine-grained token selection: each query keeps its k = 2048
 *              highest-scoring keys; attention then runs on that subset;
 *         §3.1 MLA integration in MQA mode: all query heads share one KV.
 *
 * Arithmetic: every sum/product below is carried in IEEE double.  Values that
 * the method itself stores in a narrower type (the folded query, scale
 * factors, e4m3 codes, fp32 scores) are rounded to that type exactly where the
 * method stores them, and nowhere else.  No blocking, fusion or reordering.
 *
 * Readings of the pages that this file takes (the pages are silent on them):
 *   - "q_t . W_index . k_s" is read with q_t a row vector, so the folded query
 *     is u = q W (u_j = sum_i q_i W[i][j]) and the score is u . k.
 *   - FP8 means OCP E4M3 (bias 7, no infinities, max 448).  Per-token scales
 *     are fp32 absmax/448.  The folded query is requantised the same way:
 *     s_u = fp32(amax|u| / 448), u8_j = e4m3_rne_satfinite(fp32(u_j / s_u)),
 *     and the row scale is s_row = fp32(s_q * s_u).  amax = 0 gives s_u = 1.
 *   - ReLU maps every x <= 0 (and -0.0) to +0.0; zero scores stay candidates.
 *   - Causal and inclusive: a query at position pos sees keys 0..pos of its
 *     own sequence; it keeps K = min(k, pos + 1) of them.
 *   - Ties in the score go to the lower key index; -0.0 equals +0.0; a NaN
 *     score ranks below every number.
 *   - Attention: z_j = scale * (q_h . K_j) over the selected rows j, softmax
 *     over j, output sum_j p_j V_j, lse = log(sum_j exp(z_j)) (natural log).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_F32 0
#define ORC_BF16 1
#define ORC_E4M3 2
#define ORC_DI 128 /* indexer dimension, [V32] §2.2 */

/* ------------------------------------------------------------------------- */
/* Number formats                                                             */
/* ------------------------------------------------------------------------- */

/* OCP 8-bit floating point, E4M3: sign, 4 exponent bits (bias 7), 3 mantissa
 * bits.  Exponent field 0 is subnormal: m * 2^-9.  S.1111.111 is NaN. */
double orc_e4m3_decode(uint8_t c) {
    int s = c >> 7, e = (c >> 3) & 15, m = c & 7;
    double v;
    if (e == 15 && m == 7) return NAN;
    if (e == 0)
        v = ldexp((double)m, -9);
    else
        v = ldexp((double)(8 + m), e - 10); /* (1 + m/8) * 2^(e-7) */
    return s ? -v : v;
}

/* Round-to-nearest-even onto the E4M3 grid with saturation to +-448.  Done by
 * brute force: scan every non-negative finite code for the nearest value; on
 * an exact tie keep the code whose mantissa LSB is 0 (the even one). */
uint8_t orc_e4m3_encode(float xf) {
    double x = (double)xf, a;
    uint8_t sign, best = 0;
    double best_err = INFINITY;
    int c;
    if (isnan(x)) return 0x7F;
    sign = (uint8_t)(signbit(x) ? 0x80 : 0x00);
    a = fabs(x);
    if (a >= 448.0) return (uint8_t)(sign | 0x7E);
    for (c = 0; c <= 0x7E; ++c) {
        double err = fabs(orc_e4m3_decode((uint8_t)c) - a);
        if (err < best_err || (err == best_err && (c & 1) == 0)) {
            best_err = err;
            best = (uint8_t)c;
        }
    }
    return (uint8_t)(sign | best);
}

/* bfloat16 is the top half of an IEEE binary32. */
double orc_bf16_decode(uint16_t b) {
    uint32_t u = ((uint32_t)b) << 16;
    float f;
    memcpy(&f, &u, 4);
    return (double)f;
}

static double load_elem(const void* base, int dtype, int64_t i) {
    switch (dtype) {
        case ORC_F32: return (double)((const float*)base)[i];
        case ORC_BF16: return orc_bf16_decode(((const uint16_t*)base)[i]);
        case ORC_E4M3: return orc_e4m3_decode(((const uint8_t*)base)[i]);
    }
    return NAN;
}

/* ------------------------------------------------------------------------- */
/* Step a1: fold W_index into the query ([V32] §2.2)                          */
/* ------------------------------------------------------------------------- */

/* q_idx: [n, 128] of idx_dtype (F32 or E4M3); q_scale: [n] (E4M3 only).
 * W: [128, 128] of w_dtype (F32 or BF16), row-major, W[i][j] at i*128+j.
 * F32: u_out is float [n,128] holding fp32(q W); s_row_out[r] = 1.
 * E4M3: u_out is uint8 [n,128] e4m3 codes of the requantised folded query,
 *       s_row_out[r] = fp32(s_q * s_u). */
void orc_fold(int64_t n, int idx_dtype, const void* q_idx, const float* q_scale,
              int w_dtype, const void* W, void* u_out, float* s_row_out) {
    int64_t r;
#pragma omp parallel for schedule(static)
    for (r = 0; r < n; ++r) {
        double q[ORC_DI];
        float uf[ORC_DI];
        int i, j;
        for (i = 0; i < ORC_DI; ++i) q[i] = load_elem(q_idx, idx_dtype, r * ORC_DI + i);
        for (j = 0; j < ORC_DI; ++j) {
            double acc = 0.0;
            for (i = 0; i < ORC_DI; ++i) acc += q[i] * load_elem(W, w_dtype, (int64_t)i * ORC_DI + j);
            uf[j] = (float)acc;
        }
        if (idx_dtype == ORC_F32) {
            memcpy((float*)u_out + r * ORC_DI, uf, sizeof(uf));
            s_row_out[r] = 1.0f;
        } else {
            float amax = 0.0f, s_u;
            uint8_t* dst = (uint8_t*)u_out + r * ORC_DI;
            for (j = 0; j < ORC_DI; ++j)
                if (fabsf(uf[j]) > amax) amax = fabsf(uf[j]);
            if (amax == 0.0f) {
                s_u = 1.0f;
                for (j = 0; j < ORC_DI; ++j) dst[j] = 0;
            } else {
                s_u = (float)((double)amax / 448.0);
                for (j = 0; j < ORC_DI; ++j) dst[j] = orc_e4m3_encode((float)((double)uf[j] / (double)s_u));
            }
            s_row_out[r] = (float)((double)q_scale[r] * (double)s_u);
        }
    }
}

/* ------------------------------------------------------------------------- */
/* Step a2: indexer scores ([V32] §2.2)                                       */
/* ------------------------------------------------------------------------- */

/* One query row against keys key_base .. key_base+ncand-1 (its causal
 * prefix).  u: the folded query row (F32 floats or E4M3 codes), s_row its
 * scale.  k_idx: [total_k, 128] of the same dtype, k_scale: [total_k] (E4M3).
 * out[s] = fp32 ReLU score for s < ncand, -inf for ncand <= s < ncols. */
static void scores_row(int idx_dtype, const void* u, int64_t urow, float s_row,
                       const void* k_idx, const float* k_scale, int64_t key_base,
                       int64_t ncand, int64_t ncols, float* out) {
    double uu[ORC_DI];
    int64_t s;
    int i;
    for (i = 0; i < ORC_DI; ++i) uu[i] = load_elem(u, idx_dtype, urow * ORC_DI + i);
    for (s = 0; s < ncand; ++s) {
        int64_t kr = key_base + s;
        double dot = 0.0, x;
        for (i = 0; i < ORC_DI; ++i) dot += uu[i] * load_elem(k_idx, idx_dtype, kr * ORC_DI + i);
        if (idx_dtype == ORC_F32)
            x = dot;
        else
            x = (double)s_row * (double)k_scale[kr] * dot;
        out[s] = x > 0.0 ? (float)x : 0.0f;
    }
    for (; s < ncols; ++s) out[s] = -INFINITY;
}

void orc_scores(int64_t n, int idx_dtype, const void* u, const float* s_row,
                const void* k_idx, const float* k_scale, const int64_t* key_base,
                const int64_t* ncand, int64_t ld, float* out) {
    int64_t r;
#pragma omp parallel for schedule(dynamic, 1)
    for (r = 0; r < n; ++r)
        scores_row(idx_dtype, u, r, s_row[r], k_idx, k_scale, key_base[r], ncand[r], ld, out + r * ld);
}

/* ------------------------------------------------------------------------- */
/* Step a3: top-k selection ([V32] §2.3)                                      */
/* ------------------------------------------------------------------------- */

typedef struct {
    float score;
    int32_t idx;
} orc_cand;

/* a ranks before b?  Higher score first; NaN below every number; equal
 * scores (-0.0 == +0.0, NaN == NaN) go to the lower index. */
static int cand_cmp(const void* pa, const void* pb) {
    const orc_cand* a = (const orc_cand*)pa;
    const orc_cand* b = (const orc_cand*)pb;
    int na = isnan(a->score), nb = isnan(b->score);
    if (!na && !nb && a->score != b->score) return a->score > b->score ? -1 : 1;
    if (na != nb) return na ? 1 : -1;
    return a->idx < b->idx ? -1 : (a->idx > b->idx ? 1 : 0);
}

/* scores: [n, ld]; row r has candidates 0..ncand[r]-1.  Writes the
 * K = min(k, ncand) selected key indices in rank order into idx[r*ld_idx ..],
 * then -1 up to k. */
static void topk_row(const float* sc, int64_t ncand, int32_t k, orc_cand* buf, int32_t* idx) {
    int64_t s, K = ncand < k ? ncand : k;
    for (s = 0; s < ncand; ++s) {
        buf[s].score = sc[s];
        buf[s].idx = (int32_t)s;
    }
    qsort(buf, (size_t)ncand, sizeof(orc_cand), cand_cmp);
    for (s = 0; s < K; ++s) idx[s] = buf[s].idx;
    for (; s < k; ++s) idx[s] = -1;
}

void orc_topk(int64_t n, const float* scores, int64_t ld, const int64_t* ncand, int32_t k,
              int32_t* idx, int64_t ld_idx) {
    int64_t r;
#pragma omp parallel
    {
        orc_cand* buf = (orc_cand*)malloc(sizeof(orc_cand) * (size_t)(ld > 0 ? ld : 1));
#pragma omp for schedule(dynamic, 1)
        for (r = 0; r < n; ++r) topk_row(scores + r * ld, ncand[r], k, buf, idx + r * ld_idx);
        free(buf);
    }
}

/* Dynamic k ([V32] §6 names a per-query k as a future direction): row r
 * keeps K_r = min(clamp(k_rows[r], 0, k), ncand[r]) keys by the same order,
 * written in its row of width k (ld_idx >= k) with -1 after them. */
void orc_topk_dyn(int64_t n, const float* scores, int64_t ld, const int64_t* ncand, const int32_t* k_rows,
                  int32_t k, int32_t* idx, int64_t ld_idx) {
    int64_t r;
#pragma omp parallel
    {
        orc_cand* buf = (orc_cand*)malloc(sizeof(orc_cand) * (size_t)(ld > 0 ? ld : 1));
#pragma omp for schedule(dynamic, 1)
        for (r = 0; r < n; ++r) {
            int32_t kr = k_rows[r] < 0 ? 0 : (k_rows[r] > k ? k : k_rows[r]);
            int32_t* row = idx + r * ld_idx;
            int32_t s;
            topk_row(scores + r * ld, ncand[r], kr, buf, row);
            for (s = kr; s < k; ++s) row[s] = -1;
        }
        free(buf);
    }
}

/* ------------------------------------------------------------------------- */
/* Step a4: sparse MQA attention over the selected rows ([V32] §2.3, §3.1)     */
/* ------------------------------------------------------------------------- */

/* q: [n, H, dk] (dtype), K rows at Kc + row*k_stride (dk elems), V rows at
 * Vc + row*v_stride (dv elems); selected rows are key_base[r] + idx[r, j] for
 * j < nsel with idx >= 0 (negative entries are skipped).
 * out: double [n, H, dv]; lse: double [n, H] (natural log), -inf if empty. */
static void attn_row(int dtype, int H, int dk, int dv, const void* q, int64_t r,
                     const void* Kc, int64_t k_stride, const void* Vc, int64_t v_stride,
                     int64_t key_base, const int32_t* idx, int32_t nsel, double scale,
                     double* z, double* out, double* lse) {
    int h, d;
    int32_t j;
    for (h = 0; h < H; ++h) {
        const int64_t qoff = (r * H + h) * (int64_t)dk;
        double m = -INFINITY, den = 0.0;
        double* o = out + (r * H + h) * (int64_t)dv;
        for (d = 0; d < dv; ++d) o[d] = 0.0;
        for (j = 0; j < nsel; ++j) {
            double dot = 0.0;
            int64_t row;
            if (idx[j] < 0) continue;
            row = key_base + idx[j];
            for (d = 0; d < dk; ++d) dot += load_elem(q, dtype, qoff + d) * load_elem(Kc, dtype, row * k_stride + d);
            z[j] = scale * dot;
            if (z[j] > m) m = z[j];
        }
        if (m == -INFINITY) {
            lse[r * H + h] = -INFINITY;
            continue;
        }
        for (j = 0; j < nsel; ++j) {
            double w;
            int64_t row;
            if (idx[j] < 0) continue;
            row = key_base + idx[j];
            w = exp(z[j] - m);
            den += w;
            for (d = 0; d < dv; ++d) o[d] += w * load_elem(Vc, dtype, row * v_stride + d);
        }
        for (d = 0; d < dv; ++d) o[d] /= den;
        lse[r * H + h] = m + log(den);
    }
}

void orc_attention(int64_t n, int dtype, int H, int dk, int dv, const void* q,
                   const void* Kc, int64_t k_stride, const void* Vc, int64_t v_stride,
                   const int64_t* key_base, const int32_t* idx, int64_t ld_idx, int32_t nsel,
                   double scale, double* out, double* lse) {
    int64_t r;
#pragma omp parallel
    {
        double* z = (double*)malloc(sizeof(double) * (size_t)(nsel > 0 ? nsel : 1));
#pragma omp for schedule(dynamic, 1)
        for (r = 0; r < n; ++r)
            attn_row(dtype, H, dk, dv, q, r, Kc, k_stride, Vc, v_stride, key_base[r],
                     idx + r * ld_idx, nsel, scale, z, out, lse);
        free(z);
    }
}

/* ------------------------------------------------------------------------- */
/* Whole path for a list of query rows: fold -> scores -> top-k -> attention   */
/* ------------------------------------------------------------------------- */

/* Row-gathered query inputs: q_idx [n,128] (+ q_scale [n]), q [n,H,dk].
 * Key-side inputs are the full packed arrays.  key_base[r] is the packed row
 * of the sequence's first key, pos[r] the query's position in it.
 * Outputs: idx [n,k] (rank order, -1 padded), out [n,H,dv], lse [n,H].
 * max_ncand bounds pos[r]+1 (scratch size). */
void orc_forward_rows(int64_t n, int idx_dtype, const void* q_idx, const float* q_scale,
                      int w_dtype, const void* W, const void* k_idx, const float* k_scale,
                      const int64_t* key_base, const int64_t* pos, int64_t max_ncand, int32_t k,
                      int attn_dtype, int H, int dk, int dv, const void* q,
                      const void* Kc, int64_t k_stride, const void* Vc, int64_t v_stride,
                      double scale, int32_t* idx, double* out, double* lse) {
    size_t ub = idx_dtype == ORC_F32 ? sizeof(float) : 1;
    void* u = malloc((size_t)n * ORC_DI * ub);
    float* s_row = (float*)malloc(sizeof(float) * (size_t)(n > 0 ? n : 1));
    int64_t r;
    orc_fold(n, idx_dtype, q_idx, q_scale, w_dtype, W, u, s_row);
#pragma omp parallel
    {
        float* sc = (float*)malloc(sizeof(float) * (size_t)(max_ncand > 0 ? max_ncand : 1));
        orc_cand* buf = (orc_cand*)malloc(sizeof(orc_cand) * (size_t)(max_ncand > 0 ? max_ncand : 1));
        double* z = (double*)malloc(sizeof(double) * (size_t)(k > 0 ? k : 1));
#pragma omp for schedule(dynamic, 1)
        for (r = 0; r < n; ++r) {
            int64_t nc = pos[r] + 1;
            scores_row(idx_dtype, u, r, s_row[r], k_idx, k_scale, key_base[r], nc, nc, sc);
            topk_row(sc, nc, k, buf, idx + r * (int64_t)k);
            attn_row(attn_dtype, H, dk, dv, q, r, Kc, k_stride, Vc, v_stride, key_base[r],
                     idx + r * (int64_t)k, k, scale, z, out, lse);
        }
        free(sc);
        free(buf);
        free(z);
    }
    free(u);
    free(s_row);
}

int orc_num_threads(void) {
#ifdef _OPENMP
    extern int omp_get_max_threads(void);
    return omp_get_max_threads();
#else
    return 1;
#endif
}
