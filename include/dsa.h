/*
 * dsa.h -- C ABI of libdsa, the B200 (sm_100a) DeepSeek Sparse Attention
 * forward path: lightning indexer -> per-query causal top-k -> sparse MQA
 * attention over the selected KV rows.
 *
 * Source of the method: "DeepSeek-V3.2与稀疏注意力技术革新" (intelliparadigm.com)
 *   §2.2  lightning indexer, I[t,s] = ReLU(q_t . W_index . k_s), 128-dim FP8 keys
 *   §2.3  fine-grained token selection, top-k with k = 2048 per query
 *   §3.1  MLA integration, MQA mode: every query head shares one KV row
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * - All tensor pointers are DEVICE pointers owned by the caller, row-major,
 *   with the row strides given in ELEMENTS.  The library allocates no device
 *   memory: every call takes a caller-owned device workspace `ws` of at least
 *   dsa_workspace_size() bytes (256-byte aligned).  The first 256 bytes of a
 *   workspace are its status header; zero them once before first use
 *   (e.g. cudaMemset).
 * - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy default
 *   stream).  Their return value only reports argument validation and launch
 *   errors; nothing is launched when it is not DSA_OK.  Errors found on the
 *   device (a wait that ran out, an index outside its sequence) are recorded
 *   in the workspace status header and returned by dsa_sync_status().
 * - No C++ exception crosses this interface.  Calls keep no global mutable
 *   state and may be made from several host threads on distinct workspaces.
 * - Sequences: `batch` sequences are packed along the token axis.
 *   cu_seqlens_q / cu_seqlens_k are DEVICE int64 arrays of batch+1 prefix
 *   offsets.  The queries of sequence b are its LAST seqlen_q(b) positions:
 *   query i of sequence b sits at position
 *       pos = seqlen_k(b) - seqlen_q(b) + i
 *   and may attend to keys 0..pos of its own sequence (causal, inclusive).
 *   Prefill is seqlen_q == seqlen_k; decode is seqlen_q == 1.
 * - Key indices produced and consumed by this library are LOCAL positions
 *   within the sequence (0..seqlen_k-1); -1 marks an unused slot.
 */
#ifndef DSA_H
#define DSA_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define DSA_API __attribute__((visibility("default")))
#else
#define DSA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* dsa_stream_t; /* cudaStream_t */

enum dsa_status_code {
    DSA_OK = 0,
    DSA_ERR_INVALID_ARG = 1, /* null/misaligned pointer, bad size or stride */
    DSA_ERR_UNSUPPORTED = 2, /* dtype / head / dim combination not built */
    DSA_ERR_WORKSPACE = 3,   /* ws_bytes smaller than dsa_workspace_size() */
    DSA_ERR_CUDA = 4,        /* a CUDA runtime/driver call failed */
    DSA_ERR_TIMEOUT = 5,     /* device: a bounded wait ran out (no hang) */
    DSA_ERR_INDEX = 6        /* device: index or cu_seqlens out of range */
};

enum dsa_dtype {
    DSA_F32 = 0,  /* IEEE binary32 */
    DSA_BF16 = 1, /* bfloat16 */
    DSA_E4M3 = 2  /* OCP FP8 E4M3 (stored as one byte per element) */
};

/* Operation selector for dsa_workspace_size. */
enum dsa_op {
    DSA_OP_FOLD = 0,
    DSA_OP_INDEX_SCORES = 1,
    DSA_OP_TOPK = 2,
    DSA_OP_SPARSE_ATTN = 3,
    DSA_OP_FORWARD = 4,
    DSA_OP_FORWARD_HOST = 5
};

/* Query rows per chunk of dsa_forward_host (the pipeline's fill and drain
 * are one chunk's copy each, so smaller chunks shorten them). */
#define DSA_HOST_CHUNK_ROWS 1024

/* Packed variable-length batch (see "Sequences" above). */
typedef struct dsa_seqs {
    int32_t batch;               /* B >= 1 */
    int64_t total_q;             /* = cu_seqlens_q[B] */
    int64_t total_k;             /* = cu_seqlens_k[B] */
    int64_t max_seqlen_q;        /* >= every seqlen_q(b) */
    int64_t max_seqlen_k;        /* >= every seqlen_k(b) */
    const int64_t* cu_seqlens_q; /* device, [B+1] */
    const int64_t* cu_seqlens_k; /* device, [B+1] */
} dsa_seqs;

/* Lightning indexer operands (§2.2).  The indexer dimension is fixed at 128.
 * dtype DSA_F32:  q_idx, k_idx are float [*,128]; scales must be NULL;
 *                 w_index is DSA_F32.
 * dtype DSA_E4M3: q_idx, k_idx are e4m3 codes [*,128] with one fp32 scale
 *                 per token (value = code * scale); w_index is DSA_BF16.
 * k_per_row (nullable, device int32 [total_q]): dynamic k, the per-query
 * budget the page names as a future direction (§6).  Query t keeps
 * K_t = min(clamp(k_per_row[t], 0, k), pos_t + 1) keys instead of
 * min(k, pos_t + 1); the index row keeps its width k (-1 after the K_t kept
 * keys).  NULL: every query uses k.                                        */
typedef struct dsa_indexer_args {
    int32_t dtype;            /* DSA_F32 | DSA_E4M3 */
    const void* q_idx;        /* [total_q, 128], rows contiguous */
    const float* q_idx_scale; /* [total_q] (E4M3) */
    int32_t w_dtype;          /* DSA_F32 | DSA_BF16 */
    const void* w_index;      /* [128, 128], W[i][j] at i*128 + j */
    const void* k_idx;        /* [total_k, 128], rows contiguous */
    const float* k_idx_scale; /* [total_k] (E4M3) */
    const int32_t* k_per_row; /* nullable: per-query k (see above) */
} dsa_indexer_args;

/* Sparse MQA attention operands (§2.3, §3.1).
 * Supported: DSA_BF16 with heads=128, dk=576, dv=512 (MLA latent 512 + rope
 * 64; tcgen05 tensor-core kernel); DSA_F32 with heads<=32, dk,dv in
 * {32,64,96,128} (exact fp32 SIMT kernel).  v may alias k (V = first dv
 * columns of each K row, as in MLA) by passing v = k and v_stride = k_stride.
 * BF16 requires 16-byte aligned q/k/v/out, k_stride and v_stride multiples of
 * 8, q row strides multiples of 8, and at most 2048 index slots per query
 * (k_sel / k <= 2048); larger values return DSA_ERR_UNSUPPORTED. */
typedef struct dsa_attn_args {
    int32_t dtype;          /* DSA_BF16 | DSA_F32 (q, k, v and out) */
    int32_t heads, dk, dv;
    const void* q;          /* [total_q, heads, dk] */
    int64_t q_stride_tok, q_stride_head;
    const void* k;          /* [total_k, >=dk], row stride k_stride */
    int64_t k_stride;
    const void* v;          /* [total_k, >=dv], row stride v_stride */
    int64_t v_stride;
    float scale;            /* softmax scale applied to q.k */
    void* out;              /* [total_q, heads, dv] */
    int64_t out_stride_tok, out_stride_head;
    float* lse;             /* nullable: [total_q, heads] natural-log LSE */
} dsa_attn_args;

/* Human-readable name of a status code (static string). */
DSA_API const char* dsa_status_string(int status);

/* Library ABI version (major*1000 + minor).  1001: dsa_indexer_args gained
 * k_per_row.  1002: dsa_sparse_attn_bwd.  1003: dsa_attn_target,
 * dsa_indexer_kl. */
DSA_API int dsa_version(void);

/* Workspace bytes needed by `op` for this problem (k = top-k size, used by
 * DSA_OP_FORWARD/DSA_OP_TOPK; ia/aa may be NULL where the op does not use
 * them).  Returns DSA_OK and writes *bytes, or an error status. */
DSA_API int dsa_workspace_size(int op, const dsa_seqs* seqs, int32_t k, const dsa_indexer_args* ia,
                       const dsa_attn_args* aa, size_t* bytes);

/* Step a1 -- fold W_index into the indexer query (§2.2: q_t . W_index is a
 * row vector u_t = q_t W_index, so I[t,s] = ReLU(u_t . k_s)).
 * F32:  u_out float [total_q,128] = fp32(q W); s_row_out[t] = 1.
 * E4M3: u' = q8 W (q8 the decoded codes), s_u = fp32(amax|u'|/448) (1 when
 *       amax = 0), u_out = e4m3 codes of fp32(u'/s_u) (round to nearest even,
 *       saturating), s_row_out[t] = fp32(q_idx_scale[t] * s_u).
 * u_out must be 16-byte aligned (DSA_ERR_INVALID_ARG otherwise).          */
DSA_API int dsa_fold(const dsa_seqs* seqs, const dsa_indexer_args* ia, void* u_out, float* s_row_out,
             void* ws, size_t ws_bytes, dsa_stream_t stream);

/* Step a2 -- lightning indexer scores for query rows
 * [row_begin, row_begin+row_count) (§2.2).  scores is float
 * [row_count, ld_scores], ld_scores >= max_seqlen_k.  Entry s of a row is
 * ReLU(s_row * s_k[s] * (u . k_s)) for s <= pos (exactly the values the
 * fused forward path ranks), and -inf for pos < s < ld_scores.
 * This entry point exists for tests and inspection; dsa_forward never writes
 * the L x L scores to memory. */
DSA_API int dsa_index_scores(const dsa_seqs* seqs, const dsa_indexer_args* ia, int64_t row_begin,
                     int64_t row_count, float* scores, int64_t ld_scores, void* ws,
                     size_t ws_bytes, dsa_stream_t stream);

/* Step a3 -- exact per-query top-k over given scores (§2.3).  For each row
 * t in [row_begin, row_begin+row_count): candidates are s = 0..pos_t with
 * score scores[(t-row_begin)*ld_scores + s]; K_t = min(k, pos_t+1) of them
 * are kept: highest score first, ties to the lower index, -0.0 == +0.0, NaN
 * below every number.  idx is int32 [row_count, ld_idx], ld_idx >= k: the K_t
 * kept indices in ascending index order, then -1 up to k. */
DSA_API int dsa_topk(const dsa_seqs* seqs, const float* scores, int64_t ld_scores, int64_t row_begin,
             int64_t row_count, int32_t k, int32_t* idx, int64_t ld_idx, void* ws,
             size_t ws_bytes, dsa_stream_t stream);

/* Step a4 -- sparse MQA attention (§2.3, §3.1).  For every query t and head
 * h: z_j = scale * (q[t,h,:dk] . K[row_j,:dk]) over the slots j < k_sel of
 * idx row t holding a valid local index (>= 0); out[t,h,:dv] =
 * sum_j softmax(z)_j V[row_j,:dv]; lse[t,h] = log sum_j exp(z_j).  row_j is
 * cu_seqlens_k[b] + idx[t,j].  A row with no valid slot gives out = 0 and
 * lse = -inf.  An index >= seqlen_k(b) is skipped and recorded as
 * DSA_ERR_INDEX. */
DSA_API int dsa_sparse_attn(const dsa_seqs* seqs, const dsa_attn_args* aa, const int32_t* idx,
                    int64_t ld_idx, int32_t k_sel, void* ws, size_t ws_bytes, dsa_stream_t stream);

/* Backward of dsa_sparse_attn (the training step's attention, §4.1 sparse
 * stage; the attention itself §2.3, §3.1), over the same selection.
 * aa describes the forward call: q, k, v, scale, dtype, heads, dk, dv and
 * strides as for dsa_sparse_attn.  aa->out and aa->lse (required here) hold
 * the forward's output and lse.  For every query t, head h and valid slot j
 * of idx row t (row_j = cu_seqlens_k[b] + idx[t,j]):
 *     P_j  = exp(scale * q[t,h].K[row_j] - lse[t,h])
 *     dP_j = d_out[t,h] . V[row_j],   D = d_out[t,h] . out[t,h]
 *     dS_j = P_j (dP_j - D)
 *     d_q[t,h,:dk]      = scale * sum_j dS_j K[row_j,:dk]      (written)
 *     d_k[row_j,:dk]   += scale * dS_j q[t,h,:dk]              (accumulated)
 *     d_v[row_j,:dv]   += P_j d_out[t,h,:dv]                   (accumulated)
 * d_out: same dtype as q, [total_q, heads, >= dv] with the given strides.
 * d_q, d_k, d_v: float32.  d_k and d_v accumulate, so zero them first.
 * d_v may be d_k itself (same pointer and stride): with V the first dv
 * columns of K (MLA), d_k then receives the tied gradient.  Rows whose
 * position is invalid are reported (DSA_ERR_INDEX) and their d_q is not
 * written.  Supported: bf16 or f32, dk <= 576, dv <= 512, any head count.
 * This first version runs on CUDA cores.  Workspace: a status header
 * (256 bytes). */
DSA_API int dsa_sparse_attn_bwd(const dsa_seqs* seqs, const dsa_attn_args* aa, const int32_t* idx, int64_t ld_idx,
                                int32_t k_sel, const void* d_out, int64_t d_out_stride_tok,
                                int64_t d_out_stride_head, float* d_q, int64_t d_q_stride_tok,
                                int64_t d_q_stride_head, float* d_k, int64_t d_k_stride, float* d_v,
                                int64_t d_v_stride, void* ws, size_t ws_bytes, dsa_stream_t stream);

/* Training target of the indexer's KL distillation in the sparse stage
 * (§4.1): the main attention's probabilities of every selected key, averaged
 * over the heads,
 *     p[t, j] = (1/heads) sum_h exp(scale * q[t,h].K[row_j] - lse[t,h])
 * for every valid slot j of idx row t, and 0 for empty slots.  aa describes
 * the forward call (q, k, scale, dtype, heads, dk; aa->lse, required, holds
 * the forward's lse; v and out are not read).  p: float [total_q, ld_p],
 * ld_p >= k_sel.  The call zeroes the whole array, then writes it.  Over a
 * row's valid slots, p sums to 1.  Supported: bf16 or f32, dk <= 576.
 * Workspace: a status header (256 bytes). */
DSA_API int dsa_attn_target(const dsa_seqs* seqs, const dsa_attn_args* aa, const int32_t* idx, int64_t ld_idx,
                            int32_t k_sel, float* p, int64_t ld_p, void* ws, size_t ws_bytes, dsa_stream_t stream);

/* The indexer's KL distillation loss over the selection and its gradients
 * (§4.1, sparse stage; I from §2.2).  Real-valued fp32 inputs: the indexer
 * query q_idx [total_q, q_stride >= 128], W [128,128] row-major
 * (u = q W), and the indexer keys k_idx [total_k, k_stride >= 128].  For
 * every query t over the valid slots j of its idx row:
 *     x_j = (q_t W) . k_j,  I_j = max(x_j, 0),  r = softmax_j(I)
 *     loss[t] = sum_j p_j (log p_j - log r_j)    (terms with p_j = 0 drop)
 *     G_j = (r_j - p_j) [x_j > 0]
 *     d_q[t] = W sum_j G_j k_j                          (written)
 *     d_W   += q_t^T sum_j G_j k_j                      (accumulated)
 *     d_k[row_j] += G_j (q_t W)                         (accumulated)
 * p is the target per slot (e.g. from dsa_attn_target), summing to 1 over
 * each row's valid slots.  loss (float [total_q]) may be NULL.  Zero d_W and
 * d_k first.  k_sel <= 16384.  Workspace: a status header (256 bytes). */
DSA_API int dsa_indexer_kl(const dsa_seqs* seqs, const float* q_idx, int64_t q_stride, const float* W,
                           const float* k_idx, int64_t k_stride, const int32_t* idx, int64_t ld_idx, int32_t k_sel,
                           const float* p, int64_t ld_p, float* loss, float* d_q, int64_t d_q_stride, float* d_W,
                           float* d_k, int64_t d_k_stride, void* ws, size_t ws_bytes, dsa_stream_t stream);

/* Steps a1-a3 -- fold, then the indexer and the top-k: idx (int32
 * [total_q, ld_idx], ld_idx >= k) receives, for every query, its
 * K_t = min(k, pos+1) selected keys in ascending index order followed by -1
 * (the selection dsa_topk makes on the scores of dsa_index_scores).
 * Workspace: DSA_OP_FORWARD.
 *
 * The path depends on the shapes only:
 * - Prefill-shaped E4M3 problems run one fused tensor-core indexer / top-k
 *   kernel, one CTA per 128 query rows of a sequence, and the scores never
 *   reach memory.
 * - When such a problem has fewer than 80 row blocks (ceil(max_seqlen_q /
 *   128) x batch) over max_seqlen_k > 2048 keys, and the score buffer
 *   (total_q x max_seqlen_k floats) fits in 8 GiB, the selection runs in two
 *   launches instead: a short prefill (up to about 10K tokens) or a query
 *   chunk over a long prefix.
 *   The first launch is a score sweep that splits each block's key range over
 *   several CTAs; the second selects per row from the scores (as below for
 *   decode).  The scores pass through the workspace, and the result is the
 *   same.
 * - Decode-shaped (max_seqlen_q < 64) or F32 problems scan the keys with
 *   CUDA cores into a workspace score buffer, then select per row: a
 *   histogram of the row's scores in 4096 bins of 1/16 binade, the bin of
 *   the k-th score refined on chip, one placement pass.
 * All paths give the same indices. */
DSA_API int dsa_select(const dsa_seqs* seqs, const dsa_indexer_args* ia, int32_t k, int32_t* idx,
                       int64_t ld_idx, void* ws, size_t ws_bytes, dsa_stream_t stream);

/* dsa_select without a workspace, for callers that cannot allocate device
 * memory: code running inside a host framework that owns every byte of the
 * GPU through its own pool and allows no further cudaMalloc (an inference
 * engine's plugin, for example), or a latency-critical path that must not
 * pay for an allocation.  This entry point has no counterpart in the paper;
 * it is a deployment convenience of this library.
 *
 * Same result as dsa_select.  Only prefill-shaped E4M3 inputs
 * (max_seqlen_q >= 64) are served, always by the fused tensor-core indexer
 * with the scratch-free radix selection (no bitmask scratch; slower than
 * dsa_select's selection at long sequences, the same indices), with at
 * most 32768 query rows in total; more rows return DSA_ERR_WORKSPACE, other
 * shapes DSA_ERR_UNSUPPORTED, and nothing is launched.
 *
 * The scratch it needs (a status header, the folded query codes and their
 * scales: about 4.3 MB) is a static array inside the library that every GPU
 * loading the library keeps until the process exits.  The first call on a
 * device looks up that array's device address (once per device); make that
 * first call before any stream capture begins.  The address is kept for the
 * life of the process: do not call this entry point after a reset of the
 * device's primary context (cudaDeviceReset) in the same process.  All calls share the one
 * array, so calls whose work overlaps on the GPU (other streams, other host
 * threads) race; serialise them.  The status header is cleared at the start
 * of every call.  The call allocates nothing, waits for `stream` to finish
 * the work, and returns the device-side status (DSA_OK, DSA_ERR_TIMEOUT,
 * DSA_ERR_INDEX) or a validation / CUDA error. */
DSA_API int dsa_select_noalloc(const dsa_seqs* seqs, const dsa_indexer_args* ia, int32_t k, int32_t* idx,
                               int64_t ld_idx, dsa_stream_t stream);

/* The whole hot path: a1 fold -> a2+a3 indexer/top-k (as dsa_select) -> a4
 * sparse attention.  idx_out (nullable; int32
 * [total_q, ld_idx]) receives the selected indices as dsa_topk would
 * return them for the scores of dsa_index_scores; when NULL they live in
 * the workspace. */
DSA_API int dsa_forward(const dsa_seqs* seqs, const dsa_indexer_args* ia, const dsa_attn_args* aa,
                int32_t k, int32_t* idx_out, int64_t ld_idx, void* ws, size_t ws_bytes,
                dsa_stream_t stream);

/* dsa_forward with the attention query and output in HOST memory, for a
 * caller whose activations live on the host.  aa->q and aa->out are host
 * pointers (page-locked, e.g. cudaHostAlloc, so the copies run
 * asynchronously); every other operand is a device pointer as in
 * dsa_forward.  BF16 tensor-core attention only (heads 128, dk 576, dv 512),
 * with packed q [total_q, 128, 576] and out [total_q, 128, 512]
 * (q_stride_head = dk, q_stride_tok = heads*dk, likewise for out); other
 * strides return DSA_ERR_INVALID_ARG.
 *
 * The selection (a1-a3) runs first on `stream` for all queries.  The
 * attention then runs in chunks of DSA_HOST_CHUNK_ROWS query rows: chunk c's
 * Q is copied in on `h2d_stream` while chunk c-1's attention runs on `stream`
 * and chunk c-2's output is copied out on `d2h_stream`, so the two PCIe
 * directions and the compute overlap.  Two device staging buffers each for Q
 * and output chunks live in the workspace (DSA_OP_FORWARD_HOST).  The three
 * streams may be the same stream (no overlap then).  The call returns once
 * the work is enqueued; `stream` is ordered after the last output copy, so
 * synchronising `stream` makes the host output visible.  Results are
 * identical to dsa_forward's.  The paper has no counterpart: this is the
 * host-memory front end of this library. */
DSA_API int dsa_forward_host(const dsa_seqs* seqs, const dsa_indexer_args* ia, const dsa_attn_args* aa, int32_t k,
                             int32_t* idx_out, int64_t ld_idx, void* ws, size_t ws_bytes, dsa_stream_t stream,
                             dsa_stream_t h2d_stream, dsa_stream_t d2h_stream);

/* Synchronise `stream`, return the first device-side error recorded in the
 * workspace status header since the last call (DSA_OK if none), write its
 * detail word to *detail (nullable), and clear the header. */
DSA_API int dsa_sync_status(void* ws, dsa_stream_t stream, int64_t* detail);

/* Failure-detection self test: launches one kernel that waits, with a budget
 * of `budget_cycles` SM clock cycles, on an mbarrier that nothing arrives
 * on.  The wait gives up, the kernel records DSA_ERR_TIMEOUT in the
 * workspace status header and returns; nothing hangs or faults.  Read the
 * result with dsa_sync_status. */
DSA_API int dsa_selftest_wait_timeout(void* ws, size_t ws_bytes, int64_t budget_cycles, dsa_stream_t stream);

#ifdef __cplusplus
}
#endif
#endif /* DSA_H */
