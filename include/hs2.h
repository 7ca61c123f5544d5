/*
 * hs2.h -- C ABI of the B200 (sm_100a) HySparse2 hybrid-block attention library.
 *
 * The hybrid block described by the pages: one causal full-attention layer over
 * a single shared MQA K/V cache that, having run, decides per query which
 * positions the next layers see (individual tokens: 1,024 chosen earlier
 * positions plus a compulsory window of the latest 128), then sparse-attention
 * layers that read that same cache at those same positions; the cross-decoder
 * caches come from a projection of self-decoder activations (KV Bridging).
 *
 * Sources, cited by page title and section:
 *   [NF] "Xiaomi's MiMo-V3 Architecture Reduces Prefill Compute by 80%" (news flash)
 *   [LB] "Xiaomi Unveils HySparse2 Architecture for MiMo-V3: Designed to Improve
 *        Long-Context Agent Inference" (Lynxflow blog), sections "Two-Level KV
 *        Sharing: Enabling Prefill Early Exit" and "Token-Level Sparse Selection:
 *        Precision and Efficiency Balance"
 *   [AX] "What HySparse2 is actually optimizing" (Agentik explainer), sections
 *        "2. Two levels of KV sharing" and "3. Token-level selection and unified
 *        KV cache"
 *   [AN] "Xiaomi unveils HySparse2, reducing million-token prefill compute to
 *        about one-fifth of the baseline" (AINews article), FP8 caches and MQA
 *
 * Conventions for every call
 *   - All pointers are DEVICE pointers unless stated otherwise; the caller owns
 *     every buffer (including the workspace) and keeps it alive until the work
 *     queued on `stream` has finished.  The library allocates and frees nothing
 *     and never synchronizes, except hs2_last_status.
 *   - Every compute call only validates its arguments on the host and enqueues
 *     kernels on `stream` (NULL = the legacy default stream); it returns before
 *     the work runs.
 *   - Layouts are row-major and contiguous:
 *       Q, O          [batch][n_q][heads][head_dim]
 *       K, V cache    [batch][kv_capacity][head_dim]   (one K/V head shared by all
 *                     query heads: MQA)
 *       k/v scales    [batch][kv_capacity] fp32        (E4M3 caches only)
 *       LSE           [batch][n_q][heads] fp32, natural-log sum of exp of the
 *                     scaled logits
 *       scores        [batch][n_q][score_stride] fp32
 *       idx           [batch][n_q][idx_stride] int32, ascending positions,
 *                     -1 after the first cnt entries
 *       cnt           [batch][n_q] int32
 *   - Positions: query row r of sequence b sits at p = q_pos0[b] + r and attends
 *     to cache rows 0..p (causal).  q_pos0 is a device int32 array [batch]; the
 *     caller guarantees 0 <= q_pos0[b], q_pos0[b] + n_q <= max_ctx <= kv_capacity.
 *   - Pointers must be 16-byte aligned; head_dim must be 64 or 128.
 *   - Synchronous errors (bad argument, unsupported shape or dtype, workspace
 *     too small) are returned before anything is enqueued.  Conditions found on
 *     the device (a bounded wait that ran out, an index outside the cache in a
 *     checked launch) are written to a status word at the start of the workspace
 *     and read back with hs2_last_status.  A failed launch returns HS2_ERR_CUDA.
 */
#ifndef HS2_H
#define HS2_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Exported symbols keep default visibility even when the library is built with
 * -fvisibility=hidden. */
#if defined(__GNUC__)
#define HS2_API __attribute__((visibility("default")))
#else
#define HS2_API
#endif

/* Same handle as cudaStream_t. */
typedef struct CUstream_st* hs2_stream_t;

typedef enum {
    HS2_OK = 0,
    HS2_ERR_INVALID_ARG = 1,   /* null pointer, bad size, misaligned pointer */
    HS2_ERR_UNSUPPORTED = 2,   /* shape/dtype combination without a kernel   */
    HS2_ERR_WORKSPACE = 3,     /* workspace smaller than hs2_workspace_size  */
    HS2_ERR_CUDA = 4,          /* a launch failed                            */
    HS2_ERR_TIMEOUT = 5,       /* a bounded device wait gave up              */
    HS2_ERR_INDEX = 6          /* an index outside [0, p] met by a kernel    */
} hs2_status;

typedef enum {
    HS2_F32 = 0,
    HS2_BF16 = 1,
    HS2_E4M3 = 2               /* e4m3 ("fn") codes with one fp32 scale per cache row */
} hs2_dtype;

/* Problem description; plain data, read by the callee and not retained. */
typedef struct {
    int32_t batch;          /* sequences B >= 1                                      */
    int32_t n_q;            /* query rows per sequence (1 = decode step)             */
    int32_t heads;          /* query heads H sharing the K/V head (16 on the tensor-
                               core paths; 1..16 on the f32 path)                    */
    int32_t head_dim;       /* D: 64 or 128 (128 on the tensor-core paths)           */
    int32_t window;         /* W, forced recent window (128 in the pages)            */
    int32_t budget;         /* K_sel, global positions per query (1,024)             */
    int32_t q_dtype;        /* hs2_dtype of Q and O: HS2_F32 or HS2_BF16             */
    int32_t kv_dtype;       /* hs2_dtype of the cache: F32 (with F32 Q), BF16, E4M3  */
    float   softmax_scale;  /* 0 selects 1/sqrt(head_dim)                            */
    int32_t idx_stride;     /* row capacity of idx (>= window + budget)              */
    int64_t kv_capacity;    /* cache rows per sequence                               */
    int64_t max_ctx;        /* upper bound of q_pos0[b] + n_q over the batch          */
} hs2_attn_desc;

/*
 * Workspace bytes the three attention calls need for `desc` (the largest of the
 * three).  Decode (n_q = 1) and f32 descriptions select from importance rows: if
 * `scores_in_workspace` is non-zero they are kept in the workspace
 * ([batch][n_q][max_ctx] fp32) when the caller passes no scores buffer.  Decode
 * descriptions with max_ctx > 393216 and budget <= 4096 also hold the selection's
 * per-sequence histograms and lists (about 45 KB + 4 * budget bytes per sequence).  Prefill
 * on the tensor-core path (n_q > 1, budget <= 4096) selects from candidate lists
 * that its second pass streams into the workspace (room for max_ctx + 128
 * (importance, position) pairs of 8 bytes per query row; in practice a few
 * thousand are written) and needs no importance rows.  Returns 0 for an invalid
 * description.
 */
HS2_API size_t hs2_workspace_size(const hs2_attn_desc* desc, int32_t scores_in_workspace);

/*
 * Clears the status block at the start of `workspace` (the device status word and
 * the merge counters, 4 KB; enqueued on `stream`).  Call once on a newly
 * allocated workspace before its first use.
 */
HS2_API hs2_status hs2_workspace_init(void* workspace, hs2_stream_t stream);

/*
 * Full-attention layer of a hybrid block plus its token-level selection.
 *
 * [LB] "Two-Level KV Sharing" (KV Reuse): the full layer, having run, chooses
 * the positions for the layers after it; [NF]: a budget of 1,024 chosen tokens,
 * and the latest 128 are kept by the later layers no matter what.
 * The pages give no scoring rule ([AX] "What is not documented"); this library
 * scores key j for query row i as sum over heads h of the softmax probability
 * P_h[i][j] = exp(scale * q_h.k_j - LSE_h[i]) computed in fp32, and breaks ties
 * toward the lower position.  Selection per row at position p:
 *   window  = [max(0, p - W + 1), p]
 *   global  = the min(K_sel, p - W + 1) best of [0, p - W]
 *   idx     = ascending union, cnt = min(p + 1, W + K_sel)
 *
 * q, k, v     inputs as in the conventions; k_scale/v_scale only for E4M3 caches
 * o           [batch][n_q][heads][head_dim] in q_dtype: softmax(QK^T) V
 * lse         optional (NULL) [batch][n_q][heads]
 * idx, cnt    selection output
 * scores      optional [batch][n_q][max_ctx] fp32 importance (entries beyond p
 *             are unspecified); NULL keeps them in the workspace where the
 *             selection needs them (see hs2_workspace_size).  The selection does
 *             not depend on whether they are requested.
 */
HS2_API hs2_status hs2_full_attn_select(const hs2_attn_desc* desc, const void* q, const void* k,
                                const void* v, const float* k_scale, const float* v_scale,
                                const int32_t* q_pos0, void* o, float* lse, int32_t* idx,
                                int32_t* cnt, float* scores, void* workspace, size_t ws_bytes,
                                hs2_stream_t stream);

/*
 * Number of kernels one hs2_full_attn_select call with `desc` enqueues on its
 * stream (the attention kernels plus the selection; the count depends on the
 * shapes and on the current device's SM count).  0 for an invalid description.
 * Host only: nothing is launched.
 */
HS2_API int32_t hs2_full_attn_launches(const hs2_attn_desc* desc);

/*
 * Selection alone, from a caller-given importance array.
 *
 * block_size 1: token level as above ([LB] "Token-Level Sparse Selection").
 * block_size > 1: the first-generation rule ([NF]: importance decided per group
 * of 64 tokens, a group with one important member kept in full): blocks of block_size
 * positions tile [0, p - W] from position 0, a block scores the max of its
 * tokens, the floor(K_sel / block_size) best blocks (ties to the lower block) are
 * kept, plus the window.  idx_stride must then be >= W + K_sel.
 * scores: [batch][n_q][score_row_stride] fp32, any finite values.
 */
HS2_API hs2_status hs2_topk_select(const hs2_attn_desc* desc, const float* scores,
                           int64_t score_row_stride, const int32_t* q_pos0, int32_t block_size,
                           int32_t* idx, int32_t* cnt, void* workspace, size_t ws_bytes,
                           hs2_stream_t stream);

/*
 * One sparse-attention layer with KV Reuse ([AX] section 2: a sparse layer keeps
 * no cache and no selector of its own, it reads the full layer's cache at the
 * full layer's chosen positions; [AX] section 3: window and global positions sit
 * in one cache, so a single softmax covers the whole chosen set).  q is this layer's own query; idx/cnt as produced by
 * hs2_full_attn_select (positions must lie in [0, kv_capacity)).
 * o: [batch][n_q][heads][head_dim] in q_dtype; lse optional.
 */
HS2_API hs2_status hs2_sparse_attn(const hs2_attn_desc* desc, const void* q, const void* k, const void* v,
                           const float* k_scale, const float* v_scale, const int32_t* idx,
                           const int32_t* cnt, void* o, float* lse, void* workspace,
                           size_t ws_bytes, hs2_stream_t stream);

/*
 * hs2_sparse_attn without a workspace argument, for callers that cannot
 * allocate device memory at the point where they call the library: for example
 * a plugin inside an inference engine that planned all of its memory up front,
 * or code whose only device memory is the inputs and outputs it was handed.
 * The pages have no counterpart; it exists for such callers only.
 *
 * Same arguments, kernel and results as hs2_sparse_attn with bf16 or e4m3
 * caches (an f32 description returns HS2_ERR_UNSUPPORTED).  Its scratch (split
 * partials, semaphore counters, status word) is a fixed 4 MiB array inside the
 * library, held on every GPU that loads the library until the process exits.
 *   - Every valid description is served.  When the partials of the split plan
 *     hs2_sparse_attn would use do not fit the array (on a 148-SM B200 with
 *     1,152-entry index rows: 252 to 295 rows), the rows run one CTA each,
 *     which needs no partials; the output then equals hs2_sparse_attn's within
 *     rounding, not bit for bit.  A problem whose scratch would still exceed
 *     4 MiB would be rejected with HS2_ERR_WORKSPACE before anything is
 *     enqueued; no supported shape reaches that limit.
 *   - The first call on each device looks up the array's device address with
 *     the device current; make that first call before any stream capture.
 *   - Every call first clears the array's status word and counters on
 *     `stream` (one memset node), so a call never depends on what an earlier
 *     one left there; the partials are fully written before they are read.
 *     All calls share the array: calls that overlap on the GPU (different
 *     streams, or different host threads on one device) race on it and must
 *     be ordered by the caller.
 *   - Conditions found on the device (an index outside the cache) are handled
 *     as in hs2_sparse_attn (the entry is skipped) but are not reported: there
 *     is no caller workspace to hold the status word.
 * It calls no allocating routine.
 */
HS2_API hs2_status hs2_sparse_attn_noalloc(const hs2_attn_desc* desc, const void* q, const void* k,
                                           const void* v, const float* k_scale, const float* v_scale,
                                           const int32_t* idx, const int32_t* cnt, void* o, float* lse,
                                           hs2_stream_t stream);

/*
 * KV Bridging projection ([LB] "Two-Level KV Sharing": the caches of the
 * cross-decoder's full layers are projections of self-decoder activations, a
 * separate K/V weight per target layer; [AN]: the second half of the model
 * obtains its caches this way from the first half, and the million-token caches
 * are FP8).
 *
 * hidden [batch][n][d_model] bf16, w_kv [d_model][2*head_dim] bf16 (columns
 * 0..D-1 give K, D..2D-1 give V; no bias).  Rows t = 0..n-1 of sequence b are
 * written to cache rows pos0[b] + t of k, v ([batch][kv_capacity][head_dim]),
 * from fp32 accumulators:
 *   kv_dtype HS2_BF16  rounded to nearest even bf16; k_scale, v_scale unused
 *                      (may be NULL)
 *   kv_dtype HS2_E4M3  quantized per token exactly as hs2_kv_quantize_fp8 does
 *                      it, separately for the K row and the V row: s = amax/448
 *                      of the row's fp32 accumulators (s = 1 for a zero row),
 *                      codes = e4m3(x / s) round to nearest even, saturating;
 *                      codes to k, v (uint8) and s to k_scale, v_scale
 *                      ([batch][kv_capacity] fp32, required)
 * pos0 is a device int32 array; pos0[b] + n <= kv_capacity (a row outside the
 * cache is not written).  d_model must be a multiple of 64, n >= 1, head_dim
 * 128.  No workspace: the call allocates nothing and reports only synchronous
 * errors.
 */
HS2_API hs2_status hs2_kv_bridge_proj(const void* hidden, const void* w_kv, int32_t batch, int32_t n,
                              int32_t d_model, int32_t head_dim, const int32_t* pos0,
                              int32_t kv_dtype, int64_t kv_capacity, void* k, void* v,
                              float* k_scale, float* v_scale, hs2_stream_t stream);

/*
 * FP8 cache quantizer ([AN]: the one-million-token analysis uses FP8 caches).
 * For each of `rows` rows of head_dim fp32 values: s = amax / 448 (IEEE fp32
 * division; s = 1 for an all-zero row), codes = e4m3 of x / s with round to
 * nearest even and saturation to +-448.  src [rows][head_dim] fp32, codes
 * [rows][head_dim] uint8, scales [rows] fp32.
 */
HS2_API hs2_status hs2_kv_quantize_fp8(const float* src, int64_t rows, int32_t head_dim, uint8_t* codes,
                               float* scales, hs2_stream_t stream);

/*
 * Waits for `stream`, reads and clears the device status word kept at the start
 * of `workspace`, and returns it (HS2_OK, HS2_ERR_TIMEOUT or HS2_ERR_INDEX), or
 * HS2_ERR_CUDA if the stream reported an error.
 */
HS2_API hs2_status hs2_last_status(void* workspace, hs2_stream_t stream);

/* Static text for a status code. */
HS2_API const char* hs2_status_string(hs2_status status);

#ifdef __cplusplus
}
#endif

#endif /* HS2_H */
