// api.cu -- the C ABI of libdsa (declared in include/dsa.h): argument
// validation, workspace layout, TMA descriptor encoding and kernel dispatch.
// Every numeric step runs in the kernels; this file only checks and routes.
#include <string.h>

#ifndef DSA_NO_NVTX
#include <nvtx3/nvToolsExt.h>
#endif

#include "dsa_kernels.h"

using namespace dsa;

namespace {

// An NVTX range over one entry point (host side: its validation and
// enqueueing), named after it, for timeline tools; a no-op when no tool is
// attached, and compiled out with DSA_NO_NVTX.
struct Range {
#ifndef DSA_NO_NVTX
    explicit Range(const char* name) { nvtxRangePushA(name); }
    ~Range() { nvtxRangePop(); }
#else
    explicit Range(const char*) {}
#endif
};

constexpr size_t kHdr = 256;
constexpr int64_t kTcIndexerMinRows = 64;  // prefill-shaped query sets use the tensor-core indexer
constexpr int32_t kTcAttnMaxSel = 2048;    // slots per query of the tensor-core attention

size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

bool aligned(const void* p, size_t a) { return ((uintptr_t)p % a) == 0; }

int check_seqs(const dsa_seqs* s) {
    if (!s || s->batch < 1 || !s->cu_seqlens_q || !s->cu_seqlens_k) return DSA_ERR_INVALID_ARG;
    if (s->total_q < 0 || s->total_k < 0 || s->max_seqlen_q < 0 || s->max_seqlen_k < 0) return DSA_ERR_INVALID_ARG;
    if (s->total_k >= (int64_t)1 << 31 || s->total_q >= (int64_t)1 << 31) return DSA_ERR_UNSUPPORTED;
    if (s->max_seqlen_q > s->total_q || s->max_seqlen_k > s->total_k) return DSA_ERR_INVALID_ARG;
    return DSA_OK;
}

int check_indexer(const dsa_seqs* s, const dsa_indexer_args* ia) {
    if (!ia) return DSA_ERR_INVALID_ARG;
    if (ia->dtype == DSA_F32) {
        if (ia->w_dtype != DSA_F32 || ia->q_idx_scale || ia->k_idx_scale) return DSA_ERR_UNSUPPORTED;
    } else if (ia->dtype == DSA_E4M3) {
        if (ia->w_dtype != DSA_BF16) return DSA_ERR_UNSUPPORTED;
        if ((s->total_q && !ia->q_idx_scale) || (s->total_k && !ia->k_idx_scale)) return DSA_ERR_INVALID_ARG;
    } else {
        return DSA_ERR_UNSUPPORTED;
    }
    if (!ia->w_index || (s->total_q && !ia->q_idx) || (s->total_k && !ia->k_idx)) return DSA_ERR_INVALID_ARG;
    if (!aligned(ia->q_idx, 16) || !aligned(ia->k_idx, 16) || !aligned(ia->w_index, 16)) return DSA_ERR_INVALID_ARG;
    return DSA_OK;
}

bool attn_is_tc(const dsa_attn_args* aa) { return aa->dtype == DSA_BF16; }
bool attn_v_separate(const dsa_attn_args* aa) { return !(aa->v == aa->k && aa->v_stride == aa->k_stride); }

int check_attn(const dsa_seqs* s, const dsa_attn_args* aa) {
    if (!aa) return DSA_ERR_INVALID_ARG;
    if (s->total_q && (!aa->q || !aa->out)) return DSA_ERR_INVALID_ARG;
    if (s->total_k && (!aa->k || !aa->v)) return DSA_ERR_INVALID_ARG;
    if (aa->dtype == DSA_BF16) {
        if (aa->heads != 128 || aa->dk != 576 || aa->dv != 512) return DSA_ERR_UNSUPPORTED;
        if (!aligned(aa->q, 16) || !aligned(aa->k, 16) || !aligned(aa->v, 16) || !aligned(aa->out, 16))
            return DSA_ERR_INVALID_ARG;
        if (aa->k_stride < 576 || aa->v_stride < 512 || aa->k_stride % 8 || aa->v_stride % 8) return DSA_ERR_INVALID_ARG;
        if (aa->q_stride_tok % 8 || aa->q_stride_head % 8 || aa->out_stride_tok % 8 || aa->out_stride_head % 8)
            return DSA_ERR_INVALID_ARG;
    } else if (aa->dtype == DSA_F32) {
        if (aa->heads < 1 || aa->heads > 32) return DSA_ERR_UNSUPPORTED;
        const bool okd = (aa->dk % 32 == 0 && aa->dk >= 32 && aa->dk <= 128);
        const bool okv = (aa->dv % 32 == 0 && aa->dv >= 32 && aa->dv <= 128);
        if (!okd || !okv) return DSA_ERR_UNSUPPORTED;
        if (aa->k_stride < aa->dk || aa->v_stride < aa->dv) return DSA_ERR_INVALID_ARG;
    } else {
        return DSA_ERR_UNSUPPORTED;
    }
    if (aa->q_stride_head < aa->dk || aa->q_stride_tok < (int64_t)aa->heads * aa->q_stride_head) return DSA_ERR_INVALID_ARG;
    if (aa->out_stride_head < aa->dv || aa->out_stride_tok < (int64_t)aa->heads * aa->out_stride_head)
        return DSA_ERR_INVALID_ARG;
    return DSA_OK;
}

bool use_tc_indexer(const dsa_seqs* s, const dsa_indexer_args* ia) {
    return ia->dtype == DSA_E4M3 && s->max_seqlen_q >= kTcIndexerMinRows;
}

// The fused indexer/top-k runs one CTA per 128-row block, which covers the
// sweeps over the block's whole key range.  With few blocks (a short
// prefill, or a query chunk over a long prefix: context-parallel ranks,
// chunked prefill), most SMs idle and the longest block sets the time.
// There the selection runs as two launches instead: a tensor-core score
// sweep with each block's key tiles split over several CTAs, then the exact
// top-k per row from the scores in memory.  Both rank the same scores
// exactly, so the indices are identical.  Measured on a B200: two launches
// win up to 64 blocks (8K prefill 0.40 against 0.45 ms; 2048 rows over 32K
// keys 0.48 against 0.90), break even at 32 blocks over 32K keys, and lose
// from 96 blocks on (12K prefill 0.79 against 0.49 ms), where the score
// buffer's traffic grows with rows x keys.  The choice depends only on the
// shapes, so the workspace size agrees with the call.
#ifndef DSA_SPLIT_MAX_BLOCKS
#define DSA_SPLIT_MAX_BLOCKS 80
#endif
constexpr int64_t kSplitMaxBlocks = DSA_SPLIT_MAX_BLOCKS;  // two launches below this many row blocks
constexpr int64_t kSplitMinKeys = 2049;        // key ranges longer than 2048 (shorter ones need few sweeps)
constexpr size_t kSplitMaxScoreBytes = (size_t)8 << 30;

int64_t indexer_blocks(const dsa_seqs* s) { return ((s->max_seqlen_q + 127) / 128) * (int64_t)s->batch; }

bool use_split_select(const dsa_seqs* s, const dsa_indexer_args* ia) {
    return use_tc_indexer(s, ia) && indexer_blocks(s) < kSplitMaxBlocks && s->max_seqlen_k >= kSplitMinKeys &&
           (size_t)s->total_q * (size_t)s->max_seqlen_k * 4 <= kSplitMaxScoreBytes;
}

// the selection needs a score buffer in the workspace
bool needs_scores(const dsa_seqs* s, const dsa_indexer_args* ia) {
    return !use_tc_indexer(s, ia) || use_split_select(s, ia);
}

int sm_count() {
    int sms = 148, dev = 0;
    if (cudaGetDevice(&dev) == cudaSuccess) {
        int v = 0;
        if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess && v > 0) sms = v;
    }
    return sms;
}

// the fused selection (sampled score window, bitmask per row) runs
bool use_fused_select(const dsa_seqs* s, const dsa_indexer_args* ia) {
    return use_tc_indexer(s, ia) && !use_split_select(s, ia);
}
int64_t sel_words(const dsa_seqs* s) { return 8 * ((s->max_seqlen_k + 255) / 256); }
int sel_ctas(const dsa_seqs* s) { return indexer_sel_ctas(indexer_blocks(s), sm_count()); }

// CTAs per row block for a score sweep: about two per SM in all, each over
// at least four 256-key tiles.
int score_tile_splits(const dsa_seqs* s) {
    const int sms = sm_count();
    const int64_t blocks = indexer_blocks(s) > 0 ? indexer_blocks(s) : 1;
    const int64_t max_tiles = (s->max_seqlen_k + 255) / 256;
    int64_t n = (2 * sms + blocks - 1) / blocks;
    const int64_t cap = max_tiles / 4 > 1 ? max_tiles / 4 : 1;
    if (n > cap) n = cap;
    if (n > 64) n = 64;
    return n < 1 ? 1 : (int)n;
}

struct WsLayout {
    size_t u, s_row, idx, scores, sel, total;
};

WsLayout ws_layout(const dsa_seqs* s, const dsa_indexer_args* ia, int32_t k, bool with_idx, bool with_scores) {
    WsLayout L;
    size_t off = kHdr;
    const size_t ub = (ia && ia->dtype == DSA_F32) ? 4 : 1;
    L.u = off;
    off = align256(off + (size_t)s->total_q * 128 * ub);
    L.s_row = off;
    off = align256(off + (size_t)s->total_q * 4);
    L.idx = off;
    if (with_idx) off = align256(off + (size_t)s->total_q * (size_t)k * 4);
    L.scores = off;
    if (with_scores) off = align256(off + (size_t)s->total_q * (size_t)s->max_seqlen_k * 4);
    // the fused selection's bitmask scratch: 128 rows of sel_words per CTA
    L.sel = off;
    if (with_idx && ia && use_fused_select(s, ia))
        off = align256(off + (size_t)sel_ctas(s) * 128 * (size_t)sel_words(s) * 4);
    L.total = off;
    return L;
}

// dsa_forward_host: the forward's workspace, then two device staging buffers
// each for query and output chunks of DSA_HOST_CHUNK_ROWS rows.
struct HostLayout {
    WsLayout fwd;
    size_t q[2], o[2], q_chunk_bytes, o_chunk_bytes, total;
    int64_t chunk;
};

HostLayout host_layout(const dsa_seqs* s, const dsa_indexer_args* ia, const dsa_attn_args* aa, int32_t k) {
    HostLayout H;
    H.fwd = ws_layout(s, ia, k, true, needs_scores(s, ia));
    H.chunk = s->total_q < DSA_HOST_CHUNK_ROWS ? s->total_q : DSA_HOST_CHUNK_ROWS;
    H.q_chunk_bytes = (size_t)H.chunk * (size_t)aa->heads * (size_t)aa->dk * 2;
    H.o_chunk_bytes = (size_t)H.chunk * (size_t)aa->heads * (size_t)aa->dv * 2;
    size_t off = H.fwd.total;
    for (int i = 0; i < 2; ++i) {
        H.q[i] = off;
        off = align256(off + H.q_chunk_bytes);
    }
    for (int i = 0; i < 2; ++i) {
        H.o[i] = off;
        off = align256(off + H.o_chunk_bytes);
    }
    H.total = off;
    return H;
}

bool packed_q_out(const dsa_attn_args* aa) {
    return aa->q_stride_head == aa->dk && aa->q_stride_tok == (int64_t)aa->heads * aa->dk &&
           aa->out_stride_head == aa->dv && aa->out_stride_tok == (int64_t)aa->heads * aa->dv;
}

SeqView seq_view(const dsa_seqs* s) {
    SeqView v;
    v.batch = s->batch;
    v.cu_q = s->cu_seqlens_q;
    v.cu_k = s->cu_seqlens_k;
    return v;
}

StatusHdr* hdr(void* ws) { return (StatusHdr*)ws; }

int check_ws(void* ws, size_t have, size_t need) {
    if (!ws || !aligned(ws, 256)) return DSA_ERR_INVALID_ARG;
    if (have < need) return DSA_ERR_WORKSPACE;
    return DSA_OK;
}

int cuda_status() { return cudaGetLastError() == cudaSuccess ? DSA_OK : DSA_ERR_CUDA; }

// ---- TMA descriptors through the driver entry point (no link-time libcuda) ----
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return (EncodeTiledFn) nullptr;
        return (EncodeTiledFn)p;
    }();
    return fn;
}

// 2-D row-major map: `cols` x `rows` elements, row pitch in bytes, box
// box_cols x box_rows, 128-byte swizzle.
bool make_map_2d(CUtensorMap* m, CUtensorMapDataType dt, const void* base, uint64_t cols, uint64_t rows,
                 uint64_t pitch_bytes, uint32_t box_cols, uint32_t box_rows) {
    EncodeTiledFn f = encode_fn();
    if (!f) return false;
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {pitch_bytes};
    cuuint32_t box[2] = {box_cols, box_rows};
    cuuint32_t estr[2] = {1, 1};
    return f(m, dt, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
             CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int run_fold(const dsa_seqs* s, const dsa_indexer_args* ia, void* u, float* s_row, cudaStream_t st) {
    FoldArgs f;
    f.T = s->total_q;
    f.idx_dtype = ia->dtype;
    f.q_idx = ia->q_idx;
    f.q_scale = ia->q_idx_scale;
    f.w_dtype = ia->w_dtype;
    f.W = ia->w_index;
    f.u_out = u;
    f.s_row_out = s_row;
    launch_fold(f, st);
    return cuda_status();
}

// fill: write -inf past each row's position (the dsa_index_scores contract;
// the selection reads only positions 0..pos and skips it)
int run_scores_simt(const dsa_seqs* s, const dsa_indexer_args* ia, const void* u, const float* s_row, int64_t row_begin,
                    int64_t row_count, float* scores, int64_t ld, StatusHdr* h, cudaStream_t st, bool fill) {
    ScoresSimtArgs a;
    a.sv = seq_view(s);
    a.idx_dtype = ia->dtype;
    a.u = u;
    a.s_row = s_row;
    a.k_idx = ia->k_idx;
    a.k_scale = ia->k_idx_scale;
    a.row_begin = row_begin;
    a.row_count = row_count;
    a.max_seqlen_k = s->max_seqlen_k;
    a.scores = scores;
    a.ld = ld;
    a.st = h;
    a.fill = fill;
    launch_scores_simt(a, st);
    return cuda_status();
}

int run_indexer_tc(const dsa_seqs* s, const dsa_indexer_args* ia, const void* u, const float* s_row, int mode, int32_t k,
                   int32_t* idx, int64_t ld_idx, float* scores, int64_t ld_scores, int64_t row_begin, int64_t row_count,
                   StatusHdr* h, cudaStream_t st) {
    IndexerTcArgs a;
    memset(&a, 0, sizeof(a));
    a.sv = seq_view(s);
    a.mode = mode;
    a.total_q = s->total_q;
    a.max_seqlen_q = s->max_seqlen_q;
    a.s_row = s_row;
    a.k_scale = ia->k_idx_scale;
    a.k = k;
    a.k_rows = mode == 0 ? ia->k_per_row : nullptr;
    a.idx = idx;
    a.ld_idx = ld_idx;
    a.scores = scores;
    a.ld_scores = ld_scores;
    a.row_begin = row_begin;
    a.row_count = row_count;
    a.tile_splits = mode == 1 ? score_tile_splits(s) : 1;
    a.st = h;
    if (!make_map_2d(&a.tm_u, CU_TENSOR_MAP_DATA_TYPE_UINT8, u, 128, (uint64_t)s->total_q, 128, 128, 128))
        return DSA_ERR_CUDA;
    if (!make_map_2d(&a.tm_k, CU_TENSOR_MAP_DATA_TYPE_UINT8, ia->k_idx, 128, (uint64_t)s->total_k, 128, 128, 256))
        return DSA_ERR_CUDA;
    if (!launch_indexer_tc(a, st)) return DSA_ERR_CUDA;
    return cuda_status();
}

// The fused selection: persistent CTAs, each with its slice of the bitmask
// scratch at w + L.sel.
constexpr size_t kWorkCounterOffset = 64;  // inside the 256-byte status header

int run_indexer_sel(const dsa_seqs* s, const dsa_indexer_args* ia, const void* u, const float* s_row, int32_t k,
                    int32_t* idx, int64_t ld_idx, uint32_t* sel_bits, StatusHdr* h, cudaStream_t st) {
    IndexerTcArgs a;
    memset(&a, 0, sizeof(a));
    a.sv = seq_view(s);
    a.mode = 0;
    a.total_q = s->total_q;
    a.max_seqlen_q = s->max_seqlen_q;
    a.s_row = s_row;
    a.k_scale = ia->k_idx_scale;
    a.k = k;
    a.k_rows = ia->k_per_row;
    a.idx = idx;
    a.ld_idx = ld_idx;
    a.tile_splits = 1;
    a.st = h;
    a.sel_bits = sel_bits;
    a.sel_words = sel_words(s);
    if (!make_map_2d(&a.tm_u, CU_TENSOR_MAP_DATA_TYPE_UINT8, u, 128, (uint64_t)s->total_q, 128, 128, 128))
        return DSA_ERR_CUDA;
    if (!make_map_2d(&a.tm_k, CU_TENSOR_MAP_DATA_TYPE_UINT8, ia->k_idx, 128, (uint64_t)s->total_k, 128, 128, 256))
        return DSA_ERR_CUDA;
    // every 16th key row: rows of 128 codes, 16 * 128 bytes apart
    if (!make_map_2d(&a.tm_ks, CU_TENSOR_MAP_DATA_TYPE_UINT8, ia->k_idx, 128, (uint64_t)((s->total_k + 15) / 16),
                     16 * 128, 128, 256))
        return DSA_ERR_CUDA;
    // the persistent CTAs take row blocks from a counter in the status header
    a.work_counter = (uint32_t*)((uint8_t*)h + kWorkCounterOffset);
    if (cudaMemsetAsync(a.work_counter, 0, sizeof(uint32_t), st) != cudaSuccess) return DSA_ERR_CUDA;
    if (!launch_indexer_sel(a, sel_ctas(s), st)) return DSA_ERR_CUDA;
    return cuda_status();
}

int run_topk(const dsa_seqs* s, const float* scores, int64_t ld, int64_t row_begin, int64_t row_count, int32_t k,
             int32_t* idx, int64_t ld_idx, StatusHdr* h, cudaStream_t st, const int32_t* k_rows = nullptr,
             bool nonneg = false) {
    TopkArgs a;
    a.k_rows = k_rows;
    a.sv = seq_view(s);
    a.scores = scores;
    a.ld = ld;
    a.row_begin = row_begin;
    a.row_count = row_count;
    a.k = k;
    a.idx = idx;
    a.ld_idx = ld_idx;
    a.st = h;
    if (nonneg) launch_topk_hist(a, st);  // the selection's own ReLU scores
    else launch_topk_rows(a, st);
    return cuda_status();
}

// Tensor-core attention over query rows [row_begin, row_begin + row_count);
// q and out point at row row_begin.
int run_attn_tc_rows(const dsa_seqs* s, const dsa_attn_args* aa, const int32_t* idx, int64_t ld_idx, int32_t k_sel,
                     int64_t row_begin, int64_t row_count, const void* q, void* out, StatusHdr* h, cudaStream_t st) {
    AttnTcArgs a;
    memset(&a, 0, sizeof(a));
    a.sv = seq_view(s);
    a.total_q = s->total_q;
    a.q = (const __nv_bfloat16*)q;
    a.q_stride_tok = aa->q_stride_tok;
    a.q_stride_head = aa->q_stride_head;
    a.scale_log2 = aa->scale * 1.4426950408889634f;
    a.out = (__nv_bfloat16*)out;
    a.out_stride_tok = aa->out_stride_tok;
    a.out_stride_head = aa->out_stride_head;
    a.lse = aa->lse;
    a.idx = idx;
    a.ld_idx = ld_idx;
    a.k_sel = k_sel;
    a.v_separate = attn_v_separate(aa) ? 1 : 0;
    a.st = h;
    a.k = (const __nv_bfloat16*)aa->k;
    a.k_stride = aa->k_stride;
    a.v = (const __nv_bfloat16*)aa->v;
    a.v_stride = aa->v_stride;
    a.row_begin = row_begin;
    a.row_count = row_count;
    if (!launch_attn_tc(a, st)) return DSA_ERR_CUDA;
    return cuda_status();
}

int run_attn(const dsa_seqs* s, const dsa_attn_args* aa, const int32_t* idx, int64_t ld_idx, int32_t k_sel, StatusHdr* h,
             cudaStream_t st) {
    if (s->total_q == 0) return DSA_OK;
    if (attn_is_tc(aa)) return run_attn_tc_rows(s, aa, idx, ld_idx, k_sel, 0, s->total_q, aa->q, aa->out, h, st);
    AttnF32Launch L;
    L.sv = seq_view(s);
    L.a.heads = aa->heads;
    L.a.q = (const float*)aa->q;
    L.a.q_stride_tok = aa->q_stride_tok;
    L.a.q_stride_head = aa->q_stride_head;
    L.a.k = (const float*)aa->k;
    L.a.k_stride = aa->k_stride;
    L.a.v = (const float*)aa->v;
    L.a.v_stride = aa->v_stride;
    L.a.scale = aa->scale;
    L.a.out = (float*)aa->out;
    L.a.out_stride_tok = aa->out_stride_tok;
    L.a.out_stride_head = aa->out_stride_head;
    L.a.lse = aa->lse;
    L.dk = aa->dk;
    L.dv = aa->dv;
    L.total_q = s->total_q;
    L.idx = idx;
    L.ld_idx = ld_idx;
    L.k_sel = k_sel;
    L.st = h;
    if (!launch_attn_f32(L, st)) return DSA_ERR_UNSUPPORTED;
    return cuda_status();
}

}  // namespace

extern "C" {

const char* dsa_status_string(int status) {
    switch (status) {
        case DSA_OK: return "ok";
        case DSA_ERR_INVALID_ARG: return "invalid argument";
        case DSA_ERR_UNSUPPORTED: return "unsupported dtype/shape combination";
        case DSA_ERR_WORKSPACE: return "workspace too small";
        case DSA_ERR_CUDA: return "CUDA error";
        case DSA_ERR_TIMEOUT: return "device wait timed out";
        case DSA_ERR_INDEX: return "index or sequence bounds out of range";
    }
    return "unknown status";
}

int dsa_version(void) { return 1003; }

int dsa_workspace_size(int op, const dsa_seqs* seqs, int32_t k, const dsa_indexer_args* ia, const dsa_attn_args* aa,
                       size_t* bytes) {
    if (!bytes) return DSA_ERR_INVALID_ARG;
    int r = check_seqs(seqs);
    if (r) return r;
    switch (op) {
        case DSA_OP_FOLD:
        case DSA_OP_TOPK:
        case DSA_OP_SPARSE_ATTN: *bytes = kHdr; return DSA_OK;
        case DSA_OP_INDEX_SCORES:
            if (!ia) return DSA_ERR_INVALID_ARG;
            *bytes = ws_layout(seqs, ia, 0, false, false).total;
            return DSA_OK;
        case DSA_OP_FORWARD:
            if (!ia || k < 1) return DSA_ERR_INVALID_ARG;
            *bytes = ws_layout(seqs, ia, k, true, needs_scores(seqs, ia)).total;
            return DSA_OK;
        case DSA_OP_FORWARD_HOST:
            if (!ia || !aa || k < 1 || aa->heads < 1 || aa->dk < 1 || aa->dv < 1) return DSA_ERR_INVALID_ARG;
            *bytes = host_layout(seqs, ia, aa, k).total;
            return DSA_OK;
    }
    return DSA_ERR_INVALID_ARG;
}

int dsa_fold(const dsa_seqs* seqs, const dsa_indexer_args* ia, void* u_out, float* s_row_out, void* ws, size_t ws_bytes,
             dsa_stream_t stream) {
    const Range range("dsa_fold");
    int r = check_seqs(seqs);
    if (!r) r = check_indexer(seqs, ia);
    if (!r && seqs->total_q && (!u_out || !s_row_out || !aligned(u_out, 16))) r = DSA_ERR_INVALID_ARG;
    if (!r) r = check_ws(ws, ws_bytes, kHdr);
    if (r) return r;
    return run_fold(seqs, ia, u_out, s_row_out, (cudaStream_t)stream);
}

int dsa_index_scores(const dsa_seqs* seqs, const dsa_indexer_args* ia, int64_t row_begin, int64_t row_count,
                     float* scores, int64_t ld_scores, void* ws, size_t ws_bytes, dsa_stream_t stream) {
    const Range range("dsa_index_scores");
    int r = check_seqs(seqs);
    if (!r) r = check_indexer(seqs, ia);
    if (r) return r;
    if (row_begin < 0 || row_count < 0 || row_begin + row_count > seqs->total_q) return DSA_ERR_INVALID_ARG;
    if (row_count && (!scores || ld_scores < seqs->max_seqlen_k)) return DSA_ERR_INVALID_ARG;
    const WsLayout L = ws_layout(seqs, ia, 0, false, false);
    r = check_ws(ws, ws_bytes, L.total);
    if (r) return r;
    if (row_count == 0) return DSA_OK;
    cudaStream_t st = (cudaStream_t)stream;
    uint8_t* w = (uint8_t*)ws;
    r = run_fold(seqs, ia, w + L.u, (float*)(w + L.s_row), st);
    if (r) return r;
    if (use_tc_indexer(seqs, ia)) {
        launch_fill_neg_inf(scores, row_count, ld_scores, st);
        return run_indexer_tc(seqs, ia, w + L.u, (const float*)(w + L.s_row), 1, 0, nullptr, 0, scores, ld_scores,
                              row_begin, row_count, hdr(ws), st);
    }
    return run_scores_simt(seqs, ia, w + L.u, (const float*)(w + L.s_row), row_begin, row_count, scores, ld_scores,
                           hdr(ws), st, true);
}

int dsa_topk(const dsa_seqs* seqs, const float* scores, int64_t ld_scores, int64_t row_begin, int64_t row_count,
             int32_t k, int32_t* idx, int64_t ld_idx, void* ws, size_t ws_bytes, dsa_stream_t stream) {
    const Range range("dsa_topk");
    int r = check_seqs(seqs);
    if (r) return r;
    if (k < 1 || row_begin < 0 || row_count < 0 || row_begin + row_count > seqs->total_q) return DSA_ERR_INVALID_ARG;
    if (row_count && (!scores || !idx || ld_scores < seqs->max_seqlen_k || ld_idx < k)) return DSA_ERR_INVALID_ARG;
    r = check_ws(ws, ws_bytes, kHdr);
    if (r) return r;
    return run_topk(seqs, scores, ld_scores, row_begin, row_count, k, idx, ld_idx, hdr(ws), (cudaStream_t)stream);
}

int dsa_sparse_attn_bwd(const dsa_seqs* seqs, const dsa_attn_args* aa, const int32_t* idx, int64_t ld_idx,
                        int32_t k_sel, const void* d_out, int64_t d_out_stride_tok, int64_t d_out_stride_head,
                        float* d_q, int64_t d_q_stride_tok, int64_t d_q_stride_head, float* d_k, int64_t d_k_stride,
                        float* d_v, int64_t d_v_stride, void* ws, size_t ws_bytes, dsa_stream_t stream) {
    const Range range("dsa_sparse_attn_bwd");
    int r = check_seqs(seqs);
    if (r) return r;
    if (!aa) return DSA_ERR_INVALID_ARG;
    if (aa->dtype != DSA_BF16 && aa->dtype != DSA_F32) return DSA_ERR_UNSUPPORTED;
    if (aa->heads < 1 || aa->dk < 1 || aa->dv < 1) return DSA_ERR_INVALID_ARG;
    if (aa->dk > kBwdMaxDk || aa->dv > kBwdMaxDv || aa->heads > 65535 * 16) return DSA_ERR_UNSUPPORTED;
    if (k_sel < 0 || ld_idx < k_sel) return DSA_ERR_INVALID_ARG;
    if (seqs->total_q && (!aa->q || !aa->out || !aa->lse || !d_out || !d_q || (k_sel && !idx)))
        return DSA_ERR_INVALID_ARG;
    if (seqs->total_k && (!aa->k || !aa->v || !d_k || !d_v)) return DSA_ERR_INVALID_ARG;
    if (aa->q_stride_head < aa->dk || aa->q_stride_tok < (int64_t)aa->heads * aa->q_stride_head) return DSA_ERR_INVALID_ARG;
    if (aa->out_stride_head < aa->dv || aa->out_stride_tok < (int64_t)aa->heads * aa->out_stride_head)
        return DSA_ERR_INVALID_ARG;
    if (d_out_stride_head < aa->dv || d_out_stride_tok < (int64_t)aa->heads * d_out_stride_head)
        return DSA_ERR_INVALID_ARG;
    if (d_q_stride_head < aa->dk || d_q_stride_tok < (int64_t)aa->heads * d_q_stride_head) return DSA_ERR_INVALID_ARG;
    if (aa->k_stride < aa->dk || aa->v_stride < aa->dv || d_k_stride < aa->dk || d_v_stride < aa->dv)
        return DSA_ERR_INVALID_ARG;
    r = check_ws(ws, ws_bytes, kHdr);
    if (r) return r;
    if (seqs->total_q == 0) return DSA_OK;
    AttnBwdArgs a;
    memset(&a, 0, sizeof(a));
    a.sv = seq_view(seqs);
    a.total_q = seqs->total_q;
    a.heads = aa->heads;
    a.dk = aa->dk;
    a.dv = aa->dv;
    a.scale = aa->scale;
    a.q = aa->q;
    a.q_stride_tok = aa->q_stride_tok;
    a.q_stride_head = aa->q_stride_head;
    a.k = aa->k;
    a.k_stride = aa->k_stride;
    a.v = aa->v;
    a.v_stride = aa->v_stride;
    a.out = aa->out;
    a.out_stride_tok = aa->out_stride_tok;
    a.out_stride_head = aa->out_stride_head;
    a.lse = aa->lse;
    a.dout = d_out;
    a.dout_stride_tok = d_out_stride_tok;
    a.dout_stride_head = d_out_stride_head;
    a.idx = idx;
    a.ld_idx = ld_idx;
    a.k_sel = k_sel;
    a.d_q = d_q;
    a.d_q_stride_tok = d_q_stride_tok;
    a.d_q_stride_head = d_q_stride_head;
    a.d_k = d_k;
    a.d_k_stride = d_k_stride;
    a.d_v = d_v;
    a.d_v_stride = d_v_stride;
    a.st = hdr(ws);
    if (!launch_attn_bwd(a, aa->dtype == DSA_BF16, (cudaStream_t)stream)) return DSA_ERR_CUDA;
    return cuda_status();
}

int dsa_attn_target(const dsa_seqs* seqs, const dsa_attn_args* aa, const int32_t* idx, int64_t ld_idx, int32_t k_sel,
                    float* p, int64_t ld_p, void* ws, size_t ws_bytes, dsa_stream_t stream) {
    const Range range("dsa_attn_target");
    int r = check_seqs(seqs);
    if (r) return r;
    if (!aa) return DSA_ERR_INVALID_ARG;
    if (aa->dtype != DSA_BF16 && aa->dtype != DSA_F32) return DSA_ERR_UNSUPPORTED;
    if (aa->heads < 1 || aa->dk < 1) return DSA_ERR_INVALID_ARG;
    if (aa->dk > kBwdMaxDk || aa->heads > 65535 * 16) return DSA_ERR_UNSUPPORTED;
    if (k_sel < 0 || ld_idx < k_sel || ld_p < k_sel) return DSA_ERR_INVALID_ARG;
    if (seqs->total_q && (!aa->q || !aa->lse || !p || (k_sel && !idx))) return DSA_ERR_INVALID_ARG;
    if (seqs->total_k && !aa->k) return DSA_ERR_INVALID_ARG;
    if (aa->q_stride_head < aa->dk || aa->q_stride_tok < (int64_t)aa->heads * aa->q_stride_head) return DSA_ERR_INVALID_ARG;
    if (aa->k_stride < aa->dk) return DSA_ERR_INVALID_ARG;
    r = check_ws(ws, ws_bytes, kHdr);
    if (r) return r;
    if (seqs->total_q == 0) return DSA_OK;
    cudaStream_t st = (cudaStream_t)stream;
    if (cudaMemsetAsync(p, 0, (size_t)seqs->total_q * (size_t)ld_p * sizeof(float), st) != cudaSuccess)
        return DSA_ERR_CUDA;
    AttnPmeanArgs a;
    memset(&a, 0, sizeof(a));
    a.sv = seq_view(seqs);
    a.total_q = seqs->total_q;
    a.heads = aa->heads;
    a.dk = aa->dk;
    a.scale = aa->scale;
    a.q = aa->q;
    a.q_stride_tok = aa->q_stride_tok;
    a.q_stride_head = aa->q_stride_head;
    a.k = aa->k;
    a.k_stride = aa->k_stride;
    a.lse = aa->lse;
    a.idx = idx;
    a.ld_idx = ld_idx;
    a.k_sel = k_sel;
    a.p = p;
    a.ld_p = ld_p;
    a.st = hdr(ws);
    if (!launch_attn_pmean(a, aa->dtype == DSA_BF16, st)) return DSA_ERR_CUDA;
    return cuda_status();
}

int dsa_indexer_kl(const dsa_seqs* seqs, const float* q_idx, int64_t q_stride, const float* W, const float* k_idx,
                   int64_t k_stride, const int32_t* idx, int64_t ld_idx, int32_t k_sel, const float* p, int64_t ld_p,
                   float* loss, float* d_q, int64_t d_q_stride, float* d_W, float* d_k, int64_t d_k_stride, void* ws,
                   size_t ws_bytes, dsa_stream_t stream) {
    const Range range("dsa_indexer_kl");
    int r = check_seqs(seqs);
    if (r) return r;
    if (k_sel < 0 || k_sel > 16384 || ld_idx < k_sel || ld_p < k_sel) return DSA_ERR_INVALID_ARG;
    if (!W || !d_W) return DSA_ERR_INVALID_ARG;
    if (seqs->total_q && (!q_idx || !p || !d_q || (k_sel && !idx))) return DSA_ERR_INVALID_ARG;
    if (seqs->total_k && (!k_idx || !d_k)) return DSA_ERR_INVALID_ARG;
    if (q_stride < 128 || k_stride < 128 || d_q_stride < 128 || d_k_stride < 128) return DSA_ERR_INVALID_ARG;
    r = check_ws(ws, ws_bytes, kHdr);
    if (r) return r;
    if (seqs->total_q == 0) return DSA_OK;
    IndexerKlArgs a;
    memset(&a, 0, sizeof(a));
    a.sv = seq_view(seqs);
    a.total_q = seqs->total_q;
    a.q = q_idx;
    a.q_stride = q_stride;
    a.W = W;
    a.k = k_idx;
    a.k_stride = k_stride;
    a.idx = idx;
    a.ld_idx = ld_idx;
    a.k_sel = k_sel;
    a.p = p;
    a.ld_p = ld_p;
    a.loss = loss;
    a.d_q = d_q;
    a.d_q_stride = d_q_stride;
    a.d_W = d_W;
    a.d_k = d_k;
    a.d_k_stride = d_k_stride;
    a.st = hdr(ws);
    if (!launch_indexer_kl(a, (cudaStream_t)stream)) return DSA_ERR_CUDA;
    return cuda_status();
}

int dsa_sparse_attn(const dsa_seqs* seqs, const dsa_attn_args* aa, const int32_t* idx, int64_t ld_idx, int32_t k_sel,
                    void* ws, size_t ws_bytes, dsa_stream_t stream) {
    const Range range("dsa_sparse_attn");
    int r = check_seqs(seqs);
    if (!r) r = check_attn(seqs, aa);
    if (r) return r;
    if (k_sel < 0 || ld_idx < k_sel || (seqs->total_q && k_sel && !idx)) return DSA_ERR_INVALID_ARG;
    if (attn_is_tc(aa) && k_sel > kTcAttnMaxSel) return DSA_ERR_UNSUPPORTED;
    r = check_ws(ws, ws_bytes, kHdr);
    if (r) return r;
    return run_attn(seqs, aa, idx, ld_idx, k_sel, hdr(ws), (cudaStream_t)stream);
}

namespace {
int select_into(const dsa_seqs* seqs, const dsa_indexer_args* ia, int32_t k, int32_t* idx, int64_t ldi,
                const WsLayout& L, void* ws, cudaStream_t st) {
    uint8_t* w = (uint8_t*)ws;
    int r = run_fold(seqs, ia, w + L.u, (float*)(w + L.s_row), st);
    if (r) return r;
    float* sc = (float*)(w + L.scores);
    const int64_t ld = seqs->max_seqlen_k;
    if (use_split_select(seqs, ia)) {
        // scores past each row's position are left unwritten: the top-k reads 0..pos
        r = run_indexer_tc(seqs, ia, w + L.u, (const float*)(w + L.s_row), 1, 0, nullptr, 0, sc, ld, 0, seqs->total_q,
                           hdr(ws), st);
        if (!r) r = run_topk(seqs, sc, ld, 0, seqs->total_q, k, idx, ldi, hdr(ws), st, ia->k_per_row, true);
        return r;
    }
    if (use_tc_indexer(seqs, ia))
        return run_indexer_sel(seqs, ia, w + L.u, (const float*)(w + L.s_row), k, idx, ldi, (uint32_t*)(w + L.sel),
                               hdr(ws), st);
    r = run_scores_simt(seqs, ia, w + L.u, (const float*)(w + L.s_row), 0, seqs->total_q, sc, ld, hdr(ws), st, false);
    if (!r) r = run_topk(seqs, sc, ld, 0, seqs->total_q, k, idx, ldi, hdr(ws), st, ia->k_per_row, true);
    return r;
}
}  // namespace

int dsa_select(const dsa_seqs* seqs, const dsa_indexer_args* ia, int32_t k, int32_t* idx, int64_t ld_idx, void* ws,
               size_t ws_bytes, dsa_stream_t stream) {
    const Range range("dsa_select");
    int r = check_seqs(seqs);
    if (!r) r = check_indexer(seqs, ia);
    if (r) return r;
    if (k < 1 || (seqs->total_q && (!idx || ld_idx < k))) return DSA_ERR_INVALID_ARG;
    const WsLayout L = ws_layout(seqs, ia, k, true, needs_scores(seqs, ia));
    r = check_ws(ws, ws_bytes, L.total);
    if (r) return r;
    if (seqs->total_q == 0) return DSA_OK;
    return select_into(seqs, ia, k, idx, ld_idx, L, ws, (cudaStream_t)stream);
}

int dsa_forward(const dsa_seqs* seqs, const dsa_indexer_args* ia, const dsa_attn_args* aa, int32_t k, int32_t* idx_out,
                int64_t ld_idx, void* ws, size_t ws_bytes, dsa_stream_t stream) {
    const Range range("dsa_forward");
    int r = check_seqs(seqs);
    if (!r) r = check_indexer(seqs, ia);
    if (!r) r = check_attn(seqs, aa);
    if (r) return r;
    if (k < 1) return DSA_ERR_INVALID_ARG;
    if (attn_is_tc(aa) && k > kTcAttnMaxSel) return DSA_ERR_UNSUPPORTED;
    if (idx_out && ld_idx < k) return DSA_ERR_INVALID_ARG;
    const WsLayout L = ws_layout(seqs, ia, k, true, needs_scores(seqs, ia));
    r = check_ws(ws, ws_bytes, L.total);
    if (r) return r;
    if (seqs->total_q == 0) return DSA_OK;
    cudaStream_t st = (cudaStream_t)stream;
    int32_t* idx = idx_out ? idx_out : (int32_t*)((uint8_t*)ws + L.idx);
    const int64_t ldi = idx_out ? ld_idx : k;
    r = select_into(seqs, ia, k, idx, ldi, L, ws, st);
    if (r) return r;
    return run_attn(seqs, aa, idx, ldi, k, hdr(ws), st);
}

int dsa_forward_host(const dsa_seqs* seqs, const dsa_indexer_args* ia, const dsa_attn_args* aa, int32_t k,
                     int32_t* idx_out, int64_t ld_idx, void* ws, size_t ws_bytes, dsa_stream_t stream,
                     dsa_stream_t h2d_stream, dsa_stream_t d2h_stream) {
    const Range range("dsa_forward_host");
    int r = check_seqs(seqs);
    if (!r) r = check_indexer(seqs, ia);
    if (!r) r = check_attn(seqs, aa);
    if (r) return r;
    if (!attn_is_tc(aa)) return DSA_ERR_UNSUPPORTED;
    if (k < 1 || !packed_q_out(aa) || (idx_out && ld_idx < k)) return DSA_ERR_INVALID_ARG;
    if (k > kTcAttnMaxSel) return DSA_ERR_UNSUPPORTED;
    const HostLayout H = host_layout(seqs, ia, aa, k);
    r = check_ws(ws, ws_bytes, H.total);
    if (r) return r;
    if (seqs->total_q == 0) return DSA_OK;
    cudaStream_t st = (cudaStream_t)stream, sh = (cudaStream_t)h2d_stream, sd = (cudaStream_t)d2h_stream;
    uint8_t* w = (uint8_t*)ws;
    int32_t* idx = idx_out ? idx_out : (int32_t*)(w + H.fwd.idx);
    const int64_t ldi = idx_out ? ld_idx : k;
    const size_t q_row = (size_t)aa->heads * aa->dk * 2, o_row = (size_t)aa->heads * aa->dv * 2;

    // events: start, Q chunk in [2], attention done [2], output chunk out [2]
    cudaEvent_t ev[7] = {};
    auto done = [&](int status) {
        for (cudaEvent_t e : ev)
            if (e) cudaEventDestroy(e);  // released once pending work completes
        return status;
    };
    for (cudaEvent_t& e : ev)
        if (cudaEventCreateWithFlags(&e, cudaEventDisableTiming) != cudaSuccess) return done(DSA_ERR_CUDA);
    cudaEvent_t ev_start = ev[0], *ev_q = ev + 1, *ev_a = ev + 3, *ev_o = ev + 5;
    // the copy streams follow the work already queued on `stream`
    if (cudaEventRecord(ev_start, st) != cudaSuccess || cudaStreamWaitEvent(sh, ev_start, 0) != cudaSuccess ||
        cudaStreamWaitEvent(sd, ev_start, 0) != cudaSuccess)
        return done(DSA_ERR_CUDA);
    // the selection runs while the first query chunk is copied in
    r = select_into(seqs, ia, k, idx, ldi, H.fwd, ws, st);
    if (r) return done(r);
    const int64_t nchunks = (seqs->total_q + H.chunk - 1) / H.chunk;
    for (int64_t c = 0; c < nchunks; ++c) {
        const int b = (int)(c & 1);
        const int64_t r0 = c * H.chunk, n = (seqs->total_q - r0) < H.chunk ? (seqs->total_q - r0) : H.chunk;
        void* qd = w + H.q[b];
        void* od = w + H.o[b];
        // Q in: the attention of chunk c-2 has finished reading this buffer
        if (c >= 2 && cudaStreamWaitEvent(sh, ev_a[b], 0) != cudaSuccess) return done(DSA_ERR_CUDA);
        if (cudaMemcpyAsync(qd, (const uint8_t*)aa->q + (size_t)r0 * q_row, (size_t)n * q_row, cudaMemcpyHostToDevice,
                            sh) != cudaSuccess ||
            cudaEventRecord(ev_q[b], sh) != cudaSuccess)
            return done(DSA_ERR_CUDA);
        // attention: Q is in, and the output copy of chunk c-2 has left this buffer
        if (cudaStreamWaitEvent(st, ev_q[b], 0) != cudaSuccess) return done(DSA_ERR_CUDA);
        if (c >= 2 && cudaStreamWaitEvent(st, ev_o[b], 0) != cudaSuccess) return done(DSA_ERR_CUDA);
        r = run_attn_tc_rows(seqs, aa, idx, ldi, k, r0, n, qd, od, hdr(ws), st);
        if (r) return done(r);
        if (cudaEventRecord(ev_a[b], st) != cudaSuccess) return done(DSA_ERR_CUDA);
        // output out
        if (cudaStreamWaitEvent(sd, ev_a[b], 0) != cudaSuccess ||
            cudaMemcpyAsync((uint8_t*)aa->out + (size_t)r0 * o_row, od, (size_t)n * o_row, cudaMemcpyDeviceToHost, sd) !=
                cudaSuccess ||
            cudaEventRecord(ev_o[b], sd) != cudaSuccess)
            return done(DSA_ERR_CUDA);
    }
    // `stream` is ordered after the last output copies
    for (int b = 0; b < 2 && b < nchunks; ++b)
        if (cudaStreamWaitEvent(st, ev_o[b], 0) != cudaSuccess) return done(DSA_ERR_CUDA);
    return done(DSA_OK);
}

int dsa_sync_status(void* ws, dsa_stream_t stream, int64_t* detail) {
    if (!ws) return DSA_ERR_INVALID_ARG;
    cudaStream_t st = (cudaStream_t)stream;
    StatusHdr h;
    if (cudaStreamSynchronize(st) != cudaSuccess) return DSA_ERR_CUDA;
    if (cudaMemcpyAsync(&h, ws, sizeof(h), cudaMemcpyDeviceToHost, st) != cudaSuccess) return DSA_ERR_CUDA;
    if (cudaMemsetAsync(ws, 0, sizeof(h), st) != cudaSuccess) return DSA_ERR_CUDA;
    if (cudaStreamSynchronize(st) != cudaSuccess) return DSA_ERR_CUDA;
    if (detail) *detail = h.detail;
    return h.code;
}

int dsa_selftest_wait_timeout(void* ws, size_t ws_bytes, int64_t budget_cycles, dsa_stream_t stream) {
    int r = check_ws(ws, ws_bytes, kHdr);
    if (r) return r;
    if (budget_cycles < 1 || budget_cycles > ((int64_t)1 << 34)) return DSA_ERR_INVALID_ARG;
    launch_selftest_wait(hdr(ws), (long long)budget_cycles, (cudaStream_t)stream);
    return cuda_status();
}

}  // extern "C"

// ---------------------------------------------------------------------------
// dsa_select_noalloc: dsa_select for callers that cannot allocate device
// memory.  Its scratch (status header, folded query codes and their scales)
// is the static device array below; see include/dsa.h for the contract.
// ---------------------------------------------------------------------------
#include <mutex>

namespace {
constexpr int64_t kNoAllocMaxRows = 32768;
constexpr size_t kNoAllocU = kHdr;                                        // e4m3 [rows,128]
constexpr size_t kNoAllocS = kNoAllocU + (size_t)kNoAllocMaxRows * 128;  // fp32 [rows]
constexpr size_t kNoAllocBytes = kNoAllocS + (size_t)kNoAllocMaxRows * 4;
constexpr int kNoAllocMaxDevices = 64;

// Every GPU that loads the library holds this array until the process exits.
static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocBytes];

std::mutex g_noalloc_mu;
void* g_noalloc_ptr[kNoAllocMaxDevices];  // device address of the array, per device

// Device address of the scratch array on the current device, looked up once
// per device with that device current (a host-side reference to the array
// is only a stand-in and must never be passed to a kernel).
int noalloc_scratch(uint8_t** out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kNoAllocMaxDevices) return DSA_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    if (!g_noalloc_ptr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return DSA_ERR_CUDA;
        g_noalloc_ptr[dev] = p;
    }
    *out = (uint8_t*)g_noalloc_ptr[dev];
    return DSA_OK;
}
}  // namespace

extern "C" int dsa_select_noalloc(const dsa_seqs* seqs, const dsa_indexer_args* ia, int32_t k, int32_t* idx,
                                  int64_t ld_idx, dsa_stream_t stream) {
    const Range range("dsa_select_noalloc");
    int r = check_seqs(seqs);
    if (!r) r = check_indexer(seqs, ia);
    if (r) return r;
    if (k < 1 || (seqs->total_q && (!idx || ld_idx < k))) return DSA_ERR_INVALID_ARG;
    if (!use_tc_indexer(seqs, ia)) return DSA_ERR_UNSUPPORTED;  // needs the fused (no score buffer) path
    if (seqs->total_q > kNoAllocMaxRows) return DSA_ERR_WORKSPACE;
    if (seqs->total_q == 0) return DSA_OK;
    uint8_t* w = nullptr;
    r = noalloc_scratch(&w);
    if (r) return r;
    cudaStream_t st = (cudaStream_t)stream;
    // the status header must start at zero; the code rows are rewritten in full
    if (cudaMemsetAsync(w, 0, kHdr, st) != cudaSuccess) return DSA_ERR_CUDA;
    r = run_fold(seqs, ia, w + kNoAllocU, (float*)(w + kNoAllocS), st);
    if (!r)
        r = run_indexer_tc(seqs, ia, w + kNoAllocU, (const float*)(w + kNoAllocS), 0, k, idx, ld_idx, nullptr, 0, 0, 0,
                           hdr(w), st);
    if (r) return r;
    StatusHdr h;
    if (cudaMemcpyAsync(&h, w, sizeof(h), cudaMemcpyDeviceToHost, st) != cudaSuccess) return DSA_ERR_CUDA;
    if (cudaStreamSynchronize(st) != cudaSuccess) return DSA_ERR_CUDA;
    return h.code;
}
