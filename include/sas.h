/*
 * sas.h -- C ABI of libsas, SAS gated block-sparse attention on B200 (sm_100a).
 *
 * The method ("SAS: Simple Attention Sparsification via End-to-End Optimization of
 * Context Ranking"): a selector scores the b-token history blocks of each query
 * block; g = softmax(s) over those history blocks; the hard Top-K of s plus the
 * current block B_0 (gate 1, causal) is attended with the log-gate added to the
 * logits, o = softmax(q K_S^T + log g_S) V_S.  Training carries the gradient back
 * to s through log g = s - LSE(s); inference drops the gate and attends the Top-K
 * blocks only.
 *
 * Conventions shared by every entry point
 *   - Pointers are DEVICE pointers owned by the caller; the library never
 *     allocates or frees memory.  Scratch ("workspace") is caller-owned, sized by
 *     the matching *_workspace_size query and must be 256-byte aligned.
 *   - Every call is asynchronous on the caller's stream; no implicit
 *     synchronisation.  Calls are thread-safe and re-entrant.
 *   - Arguments are checked on the host before anything is launched; a failed
 *     check returns an error code and has no side effect.  Launch failures
 *     return SAS_ERR_CUDA.  Nothing aborts, traps or throws across the ABI.
 *   - Device-side failures are reported through a status word the caller owns:
 *     one int32 of device memory, passed as `status` to every call whose kernels
 *     wait on one another inside the GPU (the attention forward and backward,
 *     and the decode calls).  Every such wait gives up after a bounded time; the
 *     kernel then writes SAS_ERR_DEVICE_TIMEOUT into the word it was given, stops
 *     its work (its outputs are then undefined) and returns, leaving the context
 *     usable.  The word must hold 0 before its first use; sas_get_device_status
 *     reads and clears it.  A call writes only the word it is given, so callers
 *     that want their own report (a stream each, a thread each) pass their own
 *     word; the library keeps no mutable state of its own.
 *   - Layouts are row-major with the last index contiguous:
 *       training  q, o, dO, dq : [B, n, Hq, d]     k, v, dk, dv : [B, n, Hkv, d]
 *                 s, ds        : [B, Hkv, Cq, Cq]  (Cq = n / b; row c scores the
 *                                                   history blocks m < c)
 *                 idx          : [B, Hkv, Cq, K]   int32, ascending, -1 padded
 *                 lse_s        : [B, Hkv, Cq]      fp32, LSE of row c over m < c
 *                 lse          : [B, Hq, n]        fp32, natural log, incl. gate
 *       decode    q, o         : [B, Hq, d]        caches : [B, Hkv, Tmax, d]
 *                 s            : [B, Hkv, s_cols]  idx    : [B, Hkv, K]
 *   - Query head hq reads KV head hq / (Hq / Hkv) (grouped-query attention); the
 *     heads of one group share one score row and one selection.
 *   - The softmax scale is softmax_scale if > 0, else 1/sqrt(d).
 *   - Preconditions the library cannot check cheaply (undefined results, never a
 *     memory fault): scores are finite; idx rows were produced by
 *     sas_topk_select (ascending, in range, -1 padded).
 */
#ifndef SAS_H_
#define SAS_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t; NULL is the legacy default stream. */
typedef struct CUstream_st* sas_stream_t;

typedef enum {
    SAS_OK = 0,
    SAS_ERR_INVALID_VALUE = 1,       /* null pointer, bad shape, inconsistent sizes */
    SAS_ERR_UNSUPPORTED = 2,         /* valid but not implemented (e.g. head_dim) */
    SAS_ERR_WORKSPACE_TOO_SMALL = 3, /* ws_bytes below the *_workspace_size query */
    SAS_ERR_CUDA = 4,                /* a CUDA runtime/driver call failed */
    SAS_ERR_DEVICE_TIMEOUT = 5,      /* a bounded device-side wait gave up */
    SAS_ERR_DEVICE_BOUNDS = 6        /* debug-bounds build only: a kernel's index check failed (the
                                        access was skipped); the status word holds the source line
                                        in its bits 8 and up */
} sas_status;

typedef enum { SAS_F32 = 0, SAS_BF16 = 1 } sas_dtype;
typedef enum { SAS_SCOPE_SPARSE = 0, SAS_SCOPE_FULL = 1 } sas_scope;
/* Gate.  SOFTMAX is the method: log g = s - LSE(s) added to the logits inside the
 * attention softmax.  The others are the ablations of SAS's design choices
 * (jaehun.me review, "Why the Four Design Choices Matter"; shibing624 review,
 * Fig. 2):
 *   SIGMOID  log g = log sigmoid(s), inside the softmax   (gate activation)
 *   RAW      log g = s, inside the softmax                (gate activation)
 *   OUTER    g = softmax(s) weights each selected block's values outside a
 *            gate-free softmax: o = sum_j g_m(j) p_j v_j  (gate placement, Eq. 5)
 *   STE      hard gate: the forward is plain Top-K attention; the backward passes
 *            dL/dh straight through to g = softmax(s), for every history block,
 *            a dropped block's keys weighted exp(z - lse) with the forward's lse
 *            (ranking preservation, Eq. 7). */
typedef enum {
    SAS_GATE_SOFTMAX = 0,
    SAS_GATE_SIGMOID = 1,
    SAS_GATE_RAW = 2,
    SAS_GATE_OUTER = 3,
    SAS_GATE_STE = 4
} sas_gate;

/* Training-shape problem.  Sparse scope attends the Top-K history blocks of each
 * query block plus the current block; full scope attends every history block,
 * all gated (the "training scope" design choice of SAS, shibing624 review
 * Fig. 2(d); jaehun.me review, "Why the Four Design Choices Matter"). */
typedef struct {
    int32_t batch, n_q_heads, n_kv_heads, head_dim;
    int32_t seq_len;    /* n, a multiple of block_size */
    int32_t block_size; /* b */
    int32_t top_k;      /* K (ignored in full scope) */
    int32_t scope;      /* sas_scope */
    int32_t dtype;      /* sas_dtype of q, k, v, o, dO, dq, dk, dv */
    float softmax_scale;
    int32_t gate;       /* sas_gate; lse_s is read by SOFTMAX, OUTER and STE */
} sas_attn_desc;

/* Decode-shape problem: one new token per sequence; ctx_len[b] counts the cached
 * tokens including the new one, so the query sits at t = ctx_len[b] - 1, its
 * current (partial) block is [C_b * b, t] and C_b = floor(t / b) full history
 * blocks precede it. */
typedef struct {
    int32_t batch, n_q_heads, n_kv_heads, head_dim;
    int32_t block_size;
    int32_t top_k;
    int32_t max_ctx; /* Tmax, the cache's token capacity per (sequence, kv head) */
    int32_t dtype;   /* sas_dtype of q, caches and o */
    float softmax_scale;
} sas_decode_desc;

/*
 * sas_topk_select -- the gate normaliser and the hard Top-K of the scores.
 *   Pages: log g_m = s_m - LSE(s) (jaehun.me review, section 4.2.2, "Gate
 *   activation"); S = Top-K(s, K) over the history blocks (jaehun.me review,
 *   Background Eq. 3; walkthrough Step 3), with the threshold selection of the
 *   training kernel (shibing624 review, method section, last paragraph).
 *   Ties go to the lower block index; -0.0 and +0.0 are equal.
 * s        [batch, n_kv_heads, n_rows, row_len] fp32.
 * ctx_len  NULL: training rows, row r has min(r, row_len) candidates (blocks
 *          0..r-1).  Non-NULL (device int32 [batch]): decode rows, n_rows must
 *          be 1 and row (b, h) has min(floor((ctx_len[b]-1)/block_size), row_len)
 *          candidates.
 * idx      [batch, n_kv_heads, n_rows, top_k] int32 out: the min(K, candidates)
 *          chosen blocks ascending, then -1.  May be NULL (only lse_s wanted, as
 *          in full scope); top_k must then still be >= 0.
 * lse_s    [batch, n_kv_heads, n_rows] fp32 out, LSE over the candidates (-inf
 *          for a row without candidates).  May be NULL.
 * Errors: SAS_ERR_INVALID_VALUE for non-positive sizes, top_k < 0, s == NULL,
 *         both outputs NULL, n_rows != 1 with ctx_len, block_size <= 0 with
 *         ctx_len.
 */
sas_status sas_topk_select(const float* s, int32_t batch, int32_t n_kv_heads, int32_t n_rows, int32_t row_len,
                           const int32_t* ctx_len, int32_t block_size, int32_t top_k, int32_t* idx, float* lse_s,
                           sas_stream_t stream);

/*
 * sas_gated_attn_fwd -- o = softmax(sigma q K_S^T + log g_S) V_S for every query
 *   row (shibing624 review, SAS equation; jaehun.me review, Eq. 9 and the
 *   Kernel implementation paragraph).  Selected history block m of query block c
 *   adds log g_m to the logits of its b tokens, per desc->gate:
 *   s[b,h,c,m] - lse_s[b,h,c] (SOFTMAX), log sigmoid(s[b,h,c,m]) (SIGMOID) or
 *   s[b,h,c,m] (RAW); the current block adds 0 and is causally masked;
 *   unselected blocks are skipped.
 * q, k, v  bf16 or fp32 per desc->dtype; s [B,Hkv,Cq,Cq] fp32; lse_s [B,Hkv,Cq]
 *          fp32 (from sas_topk_select), may be NULL for the SIGMOID and RAW gates;
 *          idx [B,Hkv,Cq,K] (sparse scope; NULL in full scope).
 * o        out, same dtype and layout as q.   lse out [B,Hq,n] fp32.
 * status   the caller's device status word (see the conventions above).
 * Errors: SAS_ERR_INVALID_VALUE (null pointers, seq_len % block_size != 0,
 *         n_q_heads % n_kv_heads != 0, sizes <= 0, top_k < 0, idx NULL in
 *         sparse scope with top_k > 0); SAS_ERR_UNSUPPORTED (head_dim not 64 or
 *         128, block_size not in {16, 32, 64}).
 */
sas_status sas_gated_attn_fwd(const sas_attn_desc* desc, const void* q, const void* k, const void* v,
                              const float* s, const float* lse_s, const int32_t* idx, void* o, float* lse,
                              int32_t* status, sas_stream_t stream);

/* Kernel family a training call runs. */
typedef enum { SAS_PATH_SIMT = 0, SAS_PATH_TENSOR_CORE = 1 } sas_path;

/*
 * sas_attn_path -- which kernels sas_gated_attn_fwd and sas_gated_attn_bwd run for
 *   this problem, given 16-byte aligned tensors (a misaligned q, k, v, o, dO, dq,
 *   dk or dv sends a call to the SIMT kernels as well).
 *   SAS_PATH_TENSOR_CORE: the tcgen05 / TMEM / TMA kernels (bf16, head_dim 128,
 *   block_size 64, 2, 4 or 8 query heads per kv head, shared memory permitting).
 *   SAS_PATH_SIMT: the CUDA-core kernels (fp32, and every other shape), tens of
 *   times slower on the training workloads.
 * fwd_path, bwd_path  host int32 out (either may be NULL).
 * Errors: SAS_ERR_INVALID_VALUE (bad desc); SAS_ERR_UNSUPPORTED (a shape neither
 *   path takes: head_dim not 64 or 128, block_size not 16, 32 or 64).
 */
sas_status sas_attn_path(const sas_attn_desc* desc, int32_t* fwd_path, int32_t* bwd_path);

/* Bytes of workspace sas_gated_attn_bwd needs for this problem (0 on bad desc). */
size_t sas_gated_attn_bwd_workspace_size(const sas_attn_desc* desc);

/*
 * sas_gated_attn_bwd -- gradients of a loss L through the forward above, given
 *   dO = dL/do: dq, dk, dv and the selector-score gradient ds.  The log-gate
 *   gradient of a selected block is the sum of the logit gradients of its tokens
 *   over the query rows and heads sharing the score row (jaehun.me review,
 *   Kernel implementation paragraph; inner-gate gradient, section 4.2.2 Eq. 5),
 *   carried to s through the gate's log g (0 for m >= c):
 *     SOFTMAX  ds[b,h,c,m] = dlogg_m - g_m * sum_{m'<c} dlogg_{m'}  (m < c),
 *              so unselected blocks receive gradient only through the
 *              normaliser (jaehun.me review, "Training scope"; shibing624
 *              review, Fig. 4);
 *     SIGMOID  ds = dlogg_m * (1 - g_m);   RAW  ds = dlogg_m
 *              (dlogg of an unselected block is 0, so so is its ds);
 *     OUTER    as SOFTMAX with dlogg_m = g_m sum_{i, j in m} p_ij dO_i.v_j;
 *     STE      as SOFTMAX with dlogg_m = g_m sum_{i, j in m} exp(z_ij - lse_i)
 *              (dO_i.v_j - D_i) over every history block m < c.
 * o, lse   the forward's outputs.   dq, dk, dv out (dtype of q), ds out fp32.
 * workspace, ws_bytes  caller scratch of at least the queried size.
 * status   the caller's device status word.
 * Errors: as sas_gated_attn_fwd, plus SAS_ERR_WORKSPACE_TOO_SMALL.
 */
sas_status sas_gated_attn_bwd(const sas_attn_desc* desc, const void* q, const void* k, const void* v,
                              const void* o, const float* lse, const void* dO, const float* s, const float* lse_s,
                              const int32_t* idx, void* dq, void* dk, void* dv, float* ds, void* workspace,
                              size_t ws_bytes, int32_t* status, sas_stream_t stream);

/*
 * sas_gated_attn_bwd_timed -- sas_gated_attn_bwd with CUDA events recorded on
 *   `stream` around its two kernels, so that each can be timed live: events[0]
 *   before the first (dq and ds, query-major), events[1] between it and the
 *   second (dk and dv, key-major), events[2] after the second.  events holds
 *   three cudaEvent_t (as void*) the caller created; nothing else differs.
 * Errors: as sas_gated_attn_bwd; SAS_ERR_INVALID_VALUE for NULL events.
 */
sas_status sas_gated_attn_bwd_timed(const sas_attn_desc* desc, const void* q, const void* k, const void* v,
                                    const void* o, const float* lse, const void* dO, const float* s,
                                    const float* lse_s, const int32_t* idx, void* dq, void* dk, void* dv, float* ds,
                                    void* workspace, size_t ws_bytes, void* const* events, int32_t* status,
                                    sas_stream_t stream);

/*
 * Parameter-free pooled-key scorer (jaehun.me review, walkthrough Step 1: scores
 * from the query and per-block key summaries; Limitations: pooling-based block
 * summaries).  SAS's trained selector is not given; this is its weight-free
 * form, mean pooling on both sides, producing the score array s the selection
 * and the gate read.
 *
 * sas_pooled_scores -- training shape:
 *   s[b,h,c,m] = sigma qbar[b,h,c] . kbar[b,h,m] for m < c, 0 for m >= c, with
 *   qbar the mean of q over query block c's tokens and the G query heads of kv
 *   head h, kbar the mean of k over block m's tokens, sigma = desc->softmax_scale
 *   (1/sqrt(d) when 0).  Only batch, heads, head_dim, seq_len, block_size, dtype
 *   and softmax_scale of desc are read.
 * q [B,n,Hq,d], k [B,n,Hkv,d] (16-byte aligned); s out [B,Hkv,Cq,Cq] fp32.
 * workspace of sas_pooled_scores_workspace_size bytes (256-byte aligned).
 * Errors: SAS_ERR_INVALID_VALUE (bad desc or pointers, misalignment);
 *   SAS_ERR_UNSUPPORTED (d * elem not a multiple of 16, d > 256, or
 *   G * d * elem > 2 KB); SAS_ERR_WORKSPACE_TOO_SMALL.
 */
size_t sas_pooled_scores_workspace_size(const sas_attn_desc* desc);
sas_status sas_pooled_scores(const sas_attn_desc* desc, const void* q, const void* k, float* s, void* workspace,
                             size_t ws_bytes, sas_stream_t stream);

/*
 * sas_pool_key_blocks -- decode shape: block summaries of a contiguous cache,
 *   ksum[b,h,m] = mean of k_cache[b,h,m*b:(m+1)*b] for m in [block_begin,
 *   block_end), stored in desc->dtype (bf16 rounded to nearest); other entries
 *   are left as they are, so a caller extends the summaries as blocks fill.
 * k_cache [B,Hkv,max_ctx,d] (16-byte aligned); ksum [B,Hkv,nsum,d], caller-owned.
 * Errors: SAS_ERR_INVALID_VALUE (bad desc, pointers, range outside [0, nsum] or
 *   past max_ctx); SAS_ERR_UNSUPPORTED (d * elem not a multiple of 16, d > 256).
 *
 * sas_decode_scores -- s[b,h,m] = sigma qbar[b,h] . ksum[b,h,m] for the
 *   floor((ctx_len[b]-1)/b) full history blocks, 0 for the rest of the row;
 *   qbar = mean of the new token's q over the G heads of kv head h.
 * q [B,Hq,d]; ksum [B,Hkv,nsum,d] in desc->dtype (16-byte aligned); ctx_len
 *   device int32 [B]; s out [B,Hkv,s_cols] fp32, ready for sas_topk_select or
 *   sas_sparse_decode_select.
 * Errors: SAS_ERR_INVALID_VALUE (bad desc or pointers, nsum or s_cols <= 0);
 *   SAS_ERR_UNSUPPORTED (head_dim not 64 or 128).
 */
sas_status sas_pool_key_blocks(const sas_decode_desc* desc, const void* k_cache, int32_t block_begin,
                               int32_t block_end, void* ksum, int32_t nsum, sas_stream_t stream);

/*
 * sas_pool_key_blocks_paged -- the same summaries from a paged cache (the layout
 *   of sas_sparse_decode_paged: pages of one block, [num_pages, block_size, Hkv,
 *   d], page_table [B, pages_per_seq] device int32).  A page id outside [0,
 *   num_pages) gives a zero summary.
 * Errors: SAS_ERR_INVALID_VALUE (bad desc or pointers, pages_per_seq or
 *   num_pages <= 0, range outside [0, min(nsum, pages_per_seq)], k_pages not
 *   16-byte aligned); SAS_ERR_UNSUPPORTED as sas_pool_key_blocks.
 */
sas_status sas_pool_key_blocks_paged(const sas_decode_desc* desc, const void* k_pages, const int32_t* page_table,
                                     int32_t pages_per_seq, int32_t num_pages, int32_t block_begin, int32_t block_end,
                                     void* ksum, int32_t nsum, sas_stream_t stream);
sas_status sas_decode_scores(const sas_decode_desc* desc, const void* q, const void* ksum, int32_t nsum,
                             const int32_t* ctx_len, float* s, int32_t s_cols, sas_stream_t stream);

/* Bytes of workspace sas_sparse_decode needs for this problem (0 on bad desc). */
size_t sas_sparse_decode_workspace_size(const sas_decode_desc* desc);

/*
 * sas_sparse_decode -- inference attention of one new token per sequence over
 *   its Top-K history blocks plus its current partial block, with no gate
 *   (jaehun.me review, walkthrough Step 6; shibing624 review, method section:
 *   at inference the gate is dropped and plain hard Top-K remains).
 *   o = softmax(sigma q K_S^T) V_S.
 * q        [B,Hq,d]; k_cache, v_cache [B,Hkv,max_ctx,d]; ctx_len device int32 [B]
 *          (1 <= ctx_len[b] <= max_ctx); idx [B,Hkv,top_k] from sas_topk_select in
 *          decode mode, or NULL for dense attention over all ctx_len[b] tokens
 *          (the full-attention comparator).
 * o        out [B,Hq,d], dtype of q.
 * status   the caller's device status word.
 * Errors: SAS_ERR_INVALID_VALUE (null pointers, sizes <= 0, heads not divisible,
 *         top_k < 0); SAS_ERR_UNSUPPORTED (head_dim not 64 or 128, block_size
 *         not a multiple of 16 up to 256, more than 16 query heads per kv
 *         head); SAS_ERR_WORKSPACE_TOO_SMALL.
 */
sas_status sas_sparse_decode(const sas_decode_desc* desc, const void* q, const void* k_cache, const void* v_cache,
                             const int32_t* ctx_len, const int32_t* idx, void* o, void* workspace, size_t ws_bytes,
                             int32_t* status, sas_stream_t stream);

/*
 * sas_sparse_decode_select -- the decode step with its selection fused: the
 *   Top-K of the block scores (as sas_topk_select in decode mode: ties to the
 *   lower index) and the gate-free attention of sas_sparse_decode, in one launch
 *   and without workspace (one thread-block cluster per (sequence, kv head)).
 *   The selection stage is the decode bottleneck the SAS reviews report at long
 *   context (shibing624 review, Fig. 7c; jaehun.me review, Decoding Efficiency).
 * s        [B, Hkv, s_cols] fp32 block scores; row (b, h) scores blocks
 *          0 .. floor((ctx_len[b]-1)/block_size) - 1, which must be <= s_cols.
 * idx_out  [B, Hkv, top_k] int32 out (nullable): the chosen blocks, ascending,
 *          -1 padded.
 * Other arguments as sas_sparse_decode.
 * Errors: as sas_sparse_decode; SAS_ERR_UNSUPPORTED unless dtype is bf16,
 *         head_dim 128, block_size 64, at most 16 query heads per kv head and
 *         every pointer 16-byte aligned.
 */
sas_status sas_sparse_decode_select(const sas_decode_desc* desc, const void* q, const void* k_cache,
                                    const void* v_cache, const int32_t* ctx_len, const float* s, int32_t s_cols,
                                    void* o, int32_t* idx_out, int32_t* status, sas_stream_t stream);

/*
 * sas_sparse_decode_paged -- the decode step over a paged KV cache, the form the
 *   pages' serving backend uses (jaehun.me review, "Our Perspective: Strengths",
 *   engineering completeness: paged KV cache, GQA, CUDA graphs; shibing624
 *   review, engineering paragraph).  A page holds one block (block_size tokens)
 *   of every kv head.  One launch, no workspace and no host synchronisation, so
 *   the call can be captured in a CUDA graph and replayed with new q, s,
 *   ctx_len and page_table contents.
 * k_pages, v_pages  [num_pages, block_size, Hkv, d] pools (token-major within a
 *          page, kv heads interleaved); 16-byte aligned.
 * page_table  device int32 [B, pages_per_seq]: entry (b, j) is the page holding
 *          block j (tokens j*block_size ..) of sequence b.  A page id outside
 *          [0, num_pages), or a block at or past pages_per_seq, reads as zeros.
 * ctx_len  device int32 [B], 1 <= ctx_len[b] <= desc->max_ctx, and
 *          desc->max_ctx <= pages_per_seq * block_size (ragged lengths allowed).
 * s, s_cols  when s != NULL the attended blocks are the Top-K of the scores, as
 *          sas_sparse_decode_select (idx_out nullable, as there);
 * idx      else when idx != NULL, the given blocks, as sas_sparse_decode;
 *          else every block (dense comparator).
 * q, o, status  as sas_sparse_decode.
 * Errors: SAS_ERR_INVALID_VALUE (null pointers, pages_per_seq or num_pages <= 0,
 *         max_ctx > pages_per_seq * block_size, s_cols <= 0 with s, unaligned
 *         pools); SAS_ERR_UNSUPPORTED unless dtype is bf16, head_dim 128,
 *         block_size 64 and at most 16 query heads per kv head.
 */
sas_status sas_sparse_decode_paged(const sas_decode_desc* desc, const void* q, const void* k_pages,
                                   const void* v_pages, const int32_t* page_table, int32_t pages_per_seq,
                                   int32_t num_pages, const int32_t* ctx_len, const int32_t* idx, const float* s,
                                   int32_t s_cols, void* o, int32_t* idx_out, int32_t* status, sas_stream_t stream);

/*
 * sas_sparse_decode_noalloc -- the decode of sas_sparse_decode (same arguments
 *   apart from the workspace, same kernels, same results) for callers that
 *   cannot allocate device memory: a plugin inside a host program that owns
 *   every byte of device memory, or a serving loop that may not call cudaMalloc
 *   (which synchronises the device) between decode steps.  It takes no
 *   workspace.  The paper has no counterpart to this entry point; it exists for
 *   those callers only.
 * Scratch: problems the tensor-core decode kernel takes (bf16, head_dim 128,
 *   block_size 64, at most 16 query heads per kv head, 16-byte aligned
 *   pointers) need none.  The others run the split-K kernels, whose partials
 *   live in a fixed 4 MiB array inside the library (every GPU that loads the
 *   library holds it until the process exits); a problem whose partials need
 *   more returns SAS_ERR_WORKSPACE_TOO_SMALL before any launch (long dense
 *   calls can; sparse calls of the Qwen3 decode shapes need about 1.4 MiB).
 * The first call on a device looks up the array's device address, once per
 *   device, with that device current; make that first call before any stream
 *   capture.  The address is kept for the life of the process, so a program
 *   that resets a device (cudaDeviceReset) must not call this entry point on
 *   that device afterwards.  Nothing is allocated (no cudaMalloc or cudaFree,
 *   no allocating library routine).
 * All calls share the one array: each call writes every partial it later reads,
 *   so nothing has to start at zero, but calls that overlap on the GPU (other
 *   streams, other host threads) race on it and must be serialised by the caller.
 * Errors: as sas_sparse_decode, with SAS_ERR_WORKSPACE_TOO_SMALL meaning the
 *   built-in array is too small for this problem.
 */
sas_status sas_sparse_decode_noalloc(const sas_decode_desc* desc, const void* q, const void* k_cache,
                                     const void* v_cache, const int32_t* ctx_len, const int32_t* idx, void* o,
                                     int32_t* status, sas_stream_t stream);

/* sas_get_device_status -- synchronises `stream`, then reads the caller's device
 * status word and clears it: SAS_OK (the word held 0) or the code a kernel wrote
 * there (SAS_ERR_DEVICE_TIMEOUT: a bounded wait gave up; SAS_ERR_DEVICE_BOUNDS: in
 * the debug-bounds build, an index check failed; either way the outputs of the
 * calls since the last read are undefined).  SAS_ERR_CUDA if the synchronisation
 * or the copy fails; SAS_ERR_INVALID_VALUE for a NULL word. */
sas_status sas_get_device_status(int32_t* status, sas_stream_t stream);

/* sas_selftest_bounded_wait -- self-test of the failure path of the tensor-core
 * kernels, without a fault.  One CTA allocates tensor memory, issues a
 * tensor-core MMA and, from its MMA-issuing thread, waits on an mbarrier that
 * nothing ever arrives at, through the same bounded-wait routine the kernels
 * use, limited to limit_ms (1..10000) instead of their fixed limit.  The wait
 * gives up and records SAS_ERR_DEVICE_TIMEOUT in *status; a second warp waiting
 * on another such barrier sees the abort flag and leaves; the issuing thread
 * drains its MMAs and the tensor memory is freed, exactly as in the kernels.
 * trace (nullable, device int32 [4]) receives 1s for the phases reached: the
 * wait gave up, the other warp left on the abort flag, the MMAs drained, the
 * tensor memory was freed.  The context stays usable; no fault, trap or hang is
 * involved.  Errors: SAS_ERR_INVALID_VALUE for a limit out of range or a NULL
 * status word. */
sas_status sas_selftest_bounded_wait(int32_t limit_ms, int32_t* status, int32_t* trace, sas_stream_t stream);

/* sas_sparse_decode_launch_floor -- launches, on `stream`, an empty kernel with the
 * grid, cluster, block size and dynamic shared memory that sas_sparse_decode_select
 * launches for the same arguments.  It reads and writes no buffer; timing it gives
 * the launch floor under the fused decode step.  Arguments and errors as for
 * sas_sparse_decode_select (no status word, no idx_out). */
sas_status sas_sparse_decode_launch_floor(const sas_decode_desc* desc, const void* q, const void* k_cache,
                                          const void* v_cache, const int32_t* ctx_len, const float* s,
                                          int32_t s_cols, void* o, sas_stream_t stream);

/* sas_phase_trace_read -- in a library built with SAS_PHASE_TRACE
 * (`python -m trainable_block_sparse_sas_b200.build --phase-trace`, giving
 * libsas_trace.so), the decode kernel records per CTA (row = blockIdx.y *
 * gridDim.x + blockIdx.x, the first 1024 CTAs) 32 uint64 slots: %clock64 at its
 * phase boundaries (0 entry, 1 ctx_len read, 2 cluster barrier passed, 3 staged
 * scores landed, 4 threshold known, 5 candidates placed, 6 selection done, 7 first
 * K/V block landed, 8 last block consumed, 9 partial merged in the CTA, 10 the
 * cluster's slices received, 11 exit), (%globaltimer, %clock64) pairs at entry
 * (12, 13) and exit (14, 15), the SM id (16), the candidate count (17), the blocks
 * this CTA streamed (18) and the grid's CTAs (31).  Slots a launch did not reach
 * keep older values.  Copies `rows` rows (1..1024) to host memory after a device
 * synchronisation.  SAS_ERR_UNSUPPORTED in builds without the trace;
 * SAS_ERR_INVALID_VALUE for a NULL destination or rows out of range. */
sas_status sas_phase_trace_read(uint64_t* host_dst, int32_t rows);

/* Number of kernels this library has launched in this process (all devices),
 * counted on the host at each successful launch. */
uint64_t sas_launch_count(void);

/* Static English text for a status code. */
const char* sas_status_string(sas_status status);

/* Library version, major * 10000 + minor * 100 + patch. */
int32_t sas_version(void);

#ifdef __cplusplus
}
#endif

#endif /* SAS_H_ */
