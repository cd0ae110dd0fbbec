// dsa_kernels.h -- internal launch interface between the C-ABI layer
// (api.cu) and the kernel translation units.  Not part of the public ABI.
#pragma once
#include "dsa_device.cuh"

namespace dsa {

struct FoldArgs {
    int64_t T;
    int idx_dtype;
    const void* q_idx;
    const float* q_scale;
    int w_dtype;
    const void* W;
    void* u_out;
    float* s_row_out;
};
void launch_fold(const FoldArgs& a, cudaStream_t s);

void launch_fill_neg_inf(float* p, int64_t rows, int64_t ld, cudaStream_t s);

// Scores into memory with CUDA cores: fp32 indexer, or FP8 scan for short
// query sets.  Entries s > pos are -inf.
struct ScoresSimtArgs {
    SeqView sv;
    int idx_dtype;
    const void* u;  // folded query [total_q,128] (f32 or e4m3 codes)
    const float* s_row;
    const void* k_idx;
    const float* k_scale;
    int64_t row_begin, row_count, max_seqlen_k;
    float* scores;
    int64_t ld;
    StatusHdr* st;
    bool fill;  // write -inf to every entry past a row's position (dsa_index_scores)
};
void launch_scores_simt(const ScoresSimtArgs& a, cudaStream_t s);

struct TopkArgs {
    SeqView sv;
    const float* scores;
    int64_t ld, row_begin, row_count;
    int k;                   // row width, and the k of rows without k_rows
    const int32_t* k_rows;   // nullable: per-row k (clamped to [0, k]), indexed by the absolute row
    int32_t* idx;
    int64_t ld_idx;
    StatusHdr* st;
};
void launch_topk_rows(const TopkArgs& a, cudaStream_t s);
// The same selection for non-negative scores (ReLU scores, +inf for NaN),
// by a histogram of 1/16 binade bins, then the boundary bin's keys on chip.
void launch_topk_hist(const TopkArgs& a, cudaStream_t s);

struct AttnF32Args {
    int heads;
    const float* q;
    int64_t q_stride_tok, q_stride_head;
    const float* k;
    int64_t k_stride;
    const float* v;
    int64_t v_stride;
    float scale;
    float* out;
    int64_t out_stride_tok, out_stride_head;
    float* lse;
};
struct AttnF32Launch {
    SeqView sv;
    AttnF32Args a;
    int dk, dv;
    int64_t total_q;
    const int32_t* idx;
    int64_t ld_idx;
    int k_sel;
    StatusHdr* st;
};
bool launch_attn_f32(const AttnF32Launch& L, cudaStream_t s);

void launch_selftest_wait(StatusHdr* st, long long budget, cudaStream_t s);

// ---------------------------------------------------------------------------
// tcgen05 FP8 lightning indexer with the fused exact top-k (prefill shapes).
// mode 0: fused selection -> idx; mode 1: write scores (rows in range).
// ---------------------------------------------------------------------------
struct IndexerTcArgs {
    SeqView sv;
    int mode;
    int64_t total_q, max_seqlen_q;
    const float* s_row;     // [total_q]
    const float* k_scale;   // [total_k]
    int k;                  // top-k size and index row width (mode 0)
    const int32_t* k_rows;  // nullable: per-row k (clamped to [0, k])
    int32_t* idx;           // mode 0: [total_q, ld_idx]
    int64_t ld_idx;
    float* scores;          // mode 1: [row_count, ld]
    int64_t ld_scores, row_begin, row_count;
    int tile_splits;        // mode 1: CTAs per row block, each over a contiguous range of key tiles
    StatusHdr* st;
    CUtensorMap tm_u;       // folded query codes [total_q,128], box 128x128
    CUtensorMap tm_k;       // key codes [total_k,128], box 128x256
    // the sampled-threshold selection (launch_indexer_sel) only:
    uint32_t* sel_bits;     // per-CTA bitmask scratch, [ctas][128 rows][sel_words]
    int64_t sel_words;      // 8 * ceil(max_seqlen_k / 256)
    CUtensorMap tm_ks;      // every 16th key row [ceil(total_k/16),128], box 128x256
    uint32_t* work_counter; // row blocks handed out so far (zero at launch)
};
bool launch_indexer_tc(const IndexerTcArgs& a, cudaStream_t s);
extern const int kIndexerRowsPerBlock;

// The fused indexer / exact top-k with a sampled score window (prefill
// shapes): a persistent grid of `ctas` CTAs, each with its own bitmask scratch.
int indexer_sel_ctas(int64_t blocks, int sms);
bool launch_indexer_sel(const IndexerTcArgs& a, int ctas, cudaStream_t s);

// ---------------------------------------------------------------------------
// tcgen05 BF16 sparse MQA attention, 128 heads, dk 576, dv 512, CTA pairs.
// ---------------------------------------------------------------------------
struct AttnTcArgs {
    SeqView sv;
    int64_t total_q;
    const __nv_bfloat16* q;
    int64_t q_stride_tok, q_stride_head;
    float scale_log2;       // softmax scale * log2(e)
    __nv_bfloat16* out;
    int64_t out_stride_tok, out_stride_head;
    float* lse;
    const int32_t* idx;
    int64_t ld_idx;
    int k_sel;
    int v_separate;         // 0: V = K[:, :512] (same rows); 1: own tensor
    StatusHdr* st;
    const __nv_bfloat16* k; // K rows [total_k, >= 576], row stride k_stride
    int64_t k_stride;
    const __nv_bfloat16* v; // V rows [total_k, >= 512] (v_separate)
    int64_t v_stride;
    // query rows [row_begin, row_begin + row_count) are processed; q and out
    // point at row row_begin (row t at (t - row_begin) * stride_tok); idx and
    // lse are indexed by the absolute row t
    int64_t row_begin, row_count;
};
bool launch_attn_tc(const AttnTcArgs& a, cudaStream_t s);

// ---------------------------------------------------------------------------
// Backward of the sparse attention (CUDA cores, fp32 arithmetic).
// ---------------------------------------------------------------------------
constexpr int kBwdMaxDk = 576, kBwdMaxDv = 512;
struct AttnBwdArgs {
    SeqView sv;
    int64_t total_q;
    int heads, dk, dv;
    float scale;
    const void* q;          // [total_q, heads, >= dk] (bf16 or f32)
    int64_t q_stride_tok, q_stride_head;
    const void* k;          // K rows, row stride k_stride
    int64_t k_stride;
    const void* v;          // V rows, row stride v_stride (may alias k)
    int64_t v_stride;
    const void* out;        // the forward's output
    int64_t out_stride_tok, out_stride_head;
    const float* lse;       // the forward's lse, [total_q, heads]
    const void* dout;       // gradient of the output
    int64_t dout_stride_tok, dout_stride_head;
    const int32_t* idx;
    int64_t ld_idx;
    int k_sel;
    float* d_q;             // written
    int64_t d_q_stride_tok, d_q_stride_head;
    float* d_k;             // accumulated
    int64_t d_k_stride;
    float* d_v;             // accumulated (may alias d_k)
    int64_t d_v_stride;
    StatusHdr* st;
};
bool launch_attn_bwd(const AttnBwdArgs& a, int dtype_bf16, cudaStream_t s);

// ---------------------------------------------------------------------------
// Indexer KL distillation (sparse stage): the attention target over the
// selected rows, then the KL loss and its gradients (CUDA cores, fp32).
// ---------------------------------------------------------------------------
struct AttnPmeanArgs {
    SeqView sv;
    int64_t total_q;
    int heads, dk;
    float scale;
    const void* q;          // [total_q, heads, >= dk]
    int64_t q_stride_tok, q_stride_head;
    const void* k;          // K rows, row stride k_stride
    int64_t k_stride;
    const float* lse;       // the forward's lse, [total_q, heads]
    const int32_t* idx;
    int64_t ld_idx;
    int k_sel;
    float* p;               // [total_q, ld_p], accumulated over head groups (zeroed by the caller)
    int64_t ld_p;
    StatusHdr* st;
};
bool launch_attn_pmean(const AttnPmeanArgs& a, int dtype_bf16, cudaStream_t s);

struct IndexerKlArgs {
    SeqView sv;
    int64_t total_q;
    const float* q;         // [total_q, 128] real-valued indexer query
    int64_t q_stride;
    const float* W;         // [128, 128], u = q W
    const float* k;         // [total_k, 128] real-valued indexer keys
    int64_t k_stride;
    const int32_t* idx;
    int64_t ld_idx;
    int k_sel;
    const float* p;         // target per slot [total_q, ld_p]
    int64_t ld_p;
    float* loss;            // [total_q] per query (nullable)
    float* d_q;             // [total_q, d_q_stride], written
    int64_t d_q_stride;
    float* d_W;             // [128, 128], accumulated
    float* d_k;             // [total_k, d_k_stride], accumulated
    int64_t d_k_stride;
    StatusHdr* st;
};
bool launch_indexer_kl(const IndexerKlArgs& a, cudaStream_t s);

}  // namespace dsa
