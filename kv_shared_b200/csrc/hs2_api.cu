// hs2_api.cu -- the extern "C" boundary of libhs2 (declared in include/hs2.h).
//
// Host code only: argument validation, workspace layout, kernel dispatch.  No
// allocation, no synchronization (except hs2_last_status), no global state but
// two caches filled once (SM counts, the driver's tensor-map encoder).
#include <cmath>
#include <cstring>
#include <mutex>

#include <cudaTypedefs.h>

#include "common.cuh"
#include "internal.h"

namespace hs2 {

int num_sms() {
    static int cache[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
    if (cache[dev] == 0) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
        cache[dev] = n;
    }
    return cache[dev];
}

static PFN_cuTensorMapEncodeTiled_v12000 tmap_encoder() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

bool make_tmap_2d(CUtensorMap* map, const void* base, CUtensorMapDataType dtype, int elem_bytes,
                  uint64_t cols, uint64_t rows, uint64_t row_bytes, uint32_t box_cols, uint32_t box_rows,
                  bool swizzle128) {
    auto enc = tmap_encoder();
    if (!enc) return false;
    (void)elem_bytes;
    const cuuint64_t dims[2] = {cols, rows};
    const cuuint64_t strides[1] = {row_bytes};
    const cuuint32_t box[2] = {box_cols, box_rows};
    const cuuint32_t estr[2] = {1, 1};
    const CUresult r = enc(map, dtype, 2, const_cast<void*>(base), dims, strides, box, estr,
                           CU_TENSOR_MAP_INTERLEAVE_NONE,
                           swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                           CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

}  // namespace hs2

using namespace hs2;

namespace {

size_t a256(size_t x) { return (x + 255) & ~size_t(255); }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

enum class Path { F32, TC };

// Validates the description; on success reports which kernel family serves it.
hs2_status check_desc(const hs2_attn_desc* d, Path* path) {
    if (!d) return HS2_ERR_INVALID_ARG;
    if (d->batch < 1 || d->n_q < 1 || d->heads < 1 || d->window < 1 || d->budget < 0)
        return HS2_ERR_INVALID_ARG;
    if (d->idx_stride < d->window + d->budget) return HS2_ERR_INVALID_ARG;
    if (d->kv_capacity < 1 || d->max_ctx < d->n_q || d->max_ctx > d->kv_capacity) return HS2_ERR_INVALID_ARG;
    if (!(d->softmax_scale >= 0.f) || std::isinf(d->softmax_scale)) return HS2_ERR_INVALID_ARG;
    if (static_cast<int64_t>(d->batch) * d->kv_capacity >= (int64_t(1) << 31)) return HS2_ERR_UNSUPPORTED;
    if (static_cast<int64_t>(d->batch) * d->n_q >= (int64_t(1) << 31)) return HS2_ERR_UNSUPPORTED;
    if (d->head_dim != 64 && d->head_dim != 128) return HS2_ERR_UNSUPPORTED;
    if (d->q_dtype == HS2_F32 && d->kv_dtype == HS2_F32) {
        if (d->heads > 16) return HS2_ERR_UNSUPPORTED;
        *path = Path::F32;
        return HS2_OK;
    }
    if (d->q_dtype == HS2_BF16 && (d->kv_dtype == HS2_BF16 || d->kv_dtype == HS2_E4M3)) {
        if (d->heads != 16 || d->head_dim != 128) return HS2_ERR_UNSUPPORTED;
        *path = Path::TC;
        return HS2_OK;
    }
    return HS2_ERR_UNSUPPORTED;
}

float eff_scale(const hs2_attn_desc* d) {
    return d->softmax_scale > 0.f ? d->softmax_scale : 1.f / std::sqrt(static_cast<float>(d->head_dim));
}

int64_t score_pitch(const hs2_attn_desc* d) { return (d->max_ctx + 63) / 64 * 64; }

// prefill on tensor cores selects from candidates streamed out of its second pass, so it
// needs no importance rows (budgets up to kFusedSelectMaxBudget)
bool fused_prefill_select(const hs2_attn_desc* d, Path path) {
    return path == Path::TC && d->n_q > 1 && d->budget <= kFusedSelectMaxBudget;
}

// decode on tensor cores selects long rows from the histograms its attention kernels build
// while they write the importance rows (budgets up to kFusedSelectMaxBudget); shorter rows
// fit the cluster select's shared memory, which is faster for them
bool hist_decode_select(const hs2_attn_desc* d, Path path) {
    return path == Path::TC && d->n_q == 1 && d->budget <= kFusedSelectMaxBudget && d->max_ctx >= kHistSelectMinCtx;
}

// bytes after the status block needed by hs2_full_attn_select
size_t full_region(const hs2_attn_desc* d, Path path, bool scores_in_ws) {
    const size_t rows = static_cast<size_t>(d->batch) * d->n_q;
    const bool fused = fused_prefill_select(d, path);
    size_t n = 0;
    if (path == Path::TC && d->n_q == 1)
        n += a256(decode_ws_bytes(d->batch, d->max_ctx, d->kv_dtype == HS2_E4M3)) +
             (hist_decode_select(d, path) ? a256(dec_select_ws_bytes(d->batch, d->budget)) : 0);
    if (path == Path::TC && d->n_q > 1) n += a256(prefill_ws_bytes(d->batch, d->n_q, d->max_ctx, fused, d->kv_dtype == HS2_E4M3));
    if (scores_in_ws && !fused) n += a256(sizeof(float) * rows * static_cast<size_t>(score_pitch(d)));
    return n;
}

size_t sparse_region(const hs2_attn_desc* d, Path path) {
    if (path == Path::F32) return 0;
    return a256(sparse_ws_bytes(d->batch * d->n_q, d->idx_stride));
}

hs2_status from_cuda(cudaError_t e) { return e == cudaSuccess ? HS2_OK : HS2_ERR_CUDA; }

}  // namespace

extern "C" {

size_t hs2_workspace_size(const hs2_attn_desc* desc, int32_t scores_in_workspace) {
    Path path;
    if (check_desc(desc, &path) != HS2_OK) return 0;
    const size_t f = full_region(desc, path, scores_in_workspace != 0);
    const size_t s = sparse_region(desc, path);
    return kStatusBytes + (f > s ? f : s);
}

hs2_status hs2_workspace_init(void* workspace, hs2_stream_t stream) {
    if (!workspace || !aligned16(workspace)) return HS2_ERR_INVALID_ARG;
    return from_cuda(cudaMemsetAsync(workspace, 0, kStatusBytes, reinterpret_cast<cudaStream_t>(stream)));
}

hs2_status hs2_full_attn_select(const hs2_attn_desc* desc, const void* q, const void* k, const void* v,
                                const float* k_scale, const float* v_scale, const int32_t* q_pos0, void* o,
                                float* lse, int32_t* idx, int32_t* cnt, float* scores, void* workspace,
                                size_t ws_bytes, hs2_stream_t stream) {
    Path path;
    hs2_status s = check_desc(desc, &path);
    if (s != HS2_OK) return s;
    if (!q || !k || !v || !q_pos0 || !o || !idx || !cnt || !workspace) return HS2_ERR_INVALID_ARG;
    const bool kv8 = desc->kv_dtype == HS2_E4M3;
    if (kv8 && (!k_scale || !v_scale)) return HS2_ERR_INVALID_ARG;
    const void* ptrs[] = {q, k, v, o, idx, cnt, workspace};
    for (const void* p : ptrs)
        if (!aligned16(p)) return HS2_ERR_INVALID_ARG;
    if ((lse && !aligned16(lse)) || (scores && !aligned16(scores)) || !aligned16(q_pos0)) return HS2_ERR_INVALID_ARG;
    if (ws_bytes < hs2_workspace_size(desc, scores == nullptr)) return HS2_ERR_WORKSPACE;

    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    uint32_t* status = reinterpret_cast<uint32_t*>(ws);
    uint8_t* region = ws + kStatusBytes;
    const size_t rows = static_cast<size_t>(desc->batch) * desc->n_q;
    float* score_buf = scores;
    int64_t score_ld = desc->max_ctx;
    size_t used = 0;
    const bool fused = fused_prefill_select(desc, path);
    const bool hist_sel = hist_decode_select(desc, path);
    DecSelState sel{};                                   // decode: histograms, counters, lists
    if (path == Path::TC && desc->n_q == 1) {
        used = a256(decode_ws_bytes(desc->batch, desc->max_ctx, kv8));
        if (hist_sel) {
            sel = dec_select_state(region + used, desc->batch, desc->budget);
            used += a256(dec_select_ws_bytes(desc->batch, desc->budget));
        }
    } else if (path == Path::TC) {
        used = a256(prefill_ws_bytes(desc->batch, desc->n_q, desc->max_ctx, fused, kv8));
    }
    if (!score_buf && !fused) {
        score_buf = reinterpret_cast<float*>(region + used);
        score_ld = score_pitch(desc);
    }
    (void)rows;
    const float scale = eff_scale(desc);
    cudaError_t e;
    if (path == Path::F32) {
        F32Args a{};
        a.batch = desc->batch; a.n_q = desc->n_q; a.heads = desc->heads; a.head_dim = desc->head_dim;
        a.cap = desc->kv_capacity; a.max_ctx = desc->max_ctx; a.q_pos0 = q_pos0;
        a.q = static_cast<const float*>(q); a.k = static_cast<const float*>(k); a.v = static_cast<const float*>(v);
        a.scale = scale; a.o = static_cast<float*>(o); a.lse = lse;
        a.scores = score_buf; a.score_ld = score_ld; a.status = status;
        e = launch_f32_full(a, st);
    } else if (desc->n_q > 1) {
        PrefillArgs a{};
        a.batch = desc->batch; a.n_q = desc->n_q; a.cap = desc->kv_capacity; a.max_ctx = desc->max_ctx;
        a.q_pos0 = q_pos0; a.q = q; a.k = k; a.v = v; a.scale = scale; a.o = o; a.lse = lse;
        a.k_scale = k_scale; a.v_scale = v_scale; a.kv8 = kv8;
        a.scores = score_buf; a.score_ld = score_ld; a.ws = region; a.status = status;
        a.fused_select = fused; a.window = desc->window; a.budget = desc->budget;
        a.idx_stride = desc->idx_stride; a.idx = idx; a.cnt = cnt;
        e = launch_prefill_full(a, st);
        if (fused) return from_cuda(e);
    } else {
        DecodeArgs a{};
        a.batch = desc->batch; a.cap = desc->kv_capacity; a.max_ctx = desc->max_ctx; a.q_pos0 = q_pos0;
        a.q = q; a.k = k; a.v = v; a.k_scale = k_scale; a.v_scale = v_scale; a.kv8 = kv8;
        a.scale = scale; a.o = o; a.lse = lse; a.scores = score_buf; a.score_ld = score_ld;
        a.ws = region; a.status = status;
        a.window = desc->window; a.sel = sel;
        e = launch_decode_full(a, st);
    }
    if (e != cudaSuccess) return HS2_ERR_CUDA;
    SelectArgs sa{};
    sa.rows = desc->batch * desc->n_q; sa.n_q = desc->n_q; sa.q_pos0 = q_pos0; sa.max_ctx = desc->max_ctx;
    sa.scores = score_buf; sa.score_ld = score_ld; sa.window = desc->window; sa.budget = desc->budget;
    sa.block_size = 1; sa.idx_stride = desc->idx_stride; sa.idx = idx; sa.cnt = cnt; sa.status = status;
    if (hist_sel) {
        HistSelectArgs ha{};
        ha.rows = desc->batch; ha.q_pos0 = q_pos0; ha.max_ctx = desc->max_ctx;
        ha.window = desc->window; ha.budget = desc->budget; ha.idx_stride = desc->idx_stride;
        ha.scores = score_buf; ha.score_ld = score_ld;
        ha.hist = sel.hist; ha.ctl = sel.ctl; ha.above = sel.above; ha.tie = sel.tie;
        ha.idx = idx; ha.cnt = cnt; ha.status = status;
        return from_cuda(launch_hist_select(ha, st));
    }
    return from_cuda(launch_select(sa, st));
}

int32_t hs2_full_attn_launches(const hs2_attn_desc* desc) {
    Path path;
    if (check_desc(desc, &path) != HS2_OK) return 0;
    int32_t n = 1;                                      // the selection
    if (path == Path::F32) n += 1;
    else if (desc->n_q > 1) n += 2;                     // prefill: log-sum-exp pass, output pass
    else n += plan_decode(desc->batch, desc->max_ctx, desc->kv_dtype == HS2_E4M3).fused ? 1 : 3;  // or: 2 passes + merge
    return n;
}

hs2_status hs2_topk_select(const hs2_attn_desc* desc, const float* scores, int64_t score_row_stride,
                           const int32_t* q_pos0, int32_t block_size, int32_t* idx, int32_t* cnt,
                           void* workspace, size_t ws_bytes, hs2_stream_t stream) {
    if (!desc || !scores || !q_pos0 || !idx || !cnt || !workspace) return HS2_ERR_INVALID_ARG;
    if (desc->batch < 1 || desc->n_q < 1 || desc->window < 1 || desc->budget < 0 || block_size < 1 ||
        desc->idx_stride < desc->window + desc->budget || desc->max_ctx < desc->n_q ||
        score_row_stride < desc->max_ctx)
        return HS2_ERR_INVALID_ARG;
    if (static_cast<int64_t>(desc->batch) * desc->n_q >= (int64_t(1) << 31) || desc->max_ctx >= (int64_t(1) << 31))
        return HS2_ERR_UNSUPPORTED;
    const void* ptrs[] = {scores, q_pos0, idx, cnt, workspace};
    for (const void* p : ptrs)
        if (!aligned16(p)) return HS2_ERR_INVALID_ARG;
    if (ws_bytes < kStatusBytes) return HS2_ERR_WORKSPACE;
    SelectArgs sa{};
    sa.rows = desc->batch * desc->n_q; sa.n_q = desc->n_q; sa.q_pos0 = q_pos0; sa.max_ctx = desc->max_ctx;
    sa.scores = scores; sa.score_ld = score_row_stride; sa.window = desc->window; sa.budget = desc->budget;
    sa.block_size = block_size; sa.idx_stride = desc->idx_stride; sa.idx = idx; sa.cnt = cnt;
    sa.status = static_cast<uint32_t*>(workspace);
    return from_cuda(launch_select(sa, reinterpret_cast<cudaStream_t>(stream)));
}

hs2_status hs2_sparse_attn(const hs2_attn_desc* desc, const void* q, const void* k, const void* v,
                           const float* k_scale, const float* v_scale, const int32_t* idx, const int32_t* cnt,
                           void* o, float* lse, void* workspace, size_t ws_bytes, hs2_stream_t stream) {
    Path path;
    hs2_status s = check_desc(desc, &path);
    if (s != HS2_OK) return s;
    if (!q || !k || !v || !idx || !cnt || !o || !workspace) return HS2_ERR_INVALID_ARG;
    const bool kv8 = desc->kv_dtype == HS2_E4M3;
    if (kv8 && (!k_scale || !v_scale)) return HS2_ERR_INVALID_ARG;
    const void* ptrs[] = {q, k, v, idx, cnt, o, workspace};
    for (const void* p : ptrs)
        if (!aligned16(p)) return HS2_ERR_INVALID_ARG;
    if (lse && !aligned16(lse)) return HS2_ERR_INVALID_ARG;
    if (ws_bytes < kStatusBytes + sparse_region(desc, path)) return HS2_ERR_WORKSPACE;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    uint32_t* status = reinterpret_cast<uint32_t*>(ws);
    const float scale = eff_scale(desc);
    if (path == Path::F32) {
        F32Args a{};
        a.batch = desc->batch; a.n_q = desc->n_q; a.heads = desc->heads; a.head_dim = desc->head_dim;
        a.cap = desc->kv_capacity; a.max_ctx = desc->max_ctx;
        a.q = static_cast<const float*>(q); a.k = static_cast<const float*>(k); a.v = static_cast<const float*>(v);
        a.scale = scale; a.o = static_cast<float*>(o); a.lse = lse;
        a.idx = idx; a.cnt = cnt; a.idx_stride = desc->idx_stride; a.status = status;
        return from_cuda(launch_f32_sparse(a, st));
    }
    SparseArgs a{};
    a.rows = desc->batch * desc->n_q; a.n_q = desc->n_q; a.cap = desc->kv_capacity; a.idx_stride = desc->idx_stride;
    a.q = q; a.k = k; a.v = v; a.k_scale = k_scale; a.v_scale = v_scale; a.kv8 = kv8;
    a.idx = idx; a.cnt = cnt; a.scale = scale; a.o = o; a.lse = lse;
    a.ws = ws + kStatusBytes; a.status = status;
    return from_cuda(launch_sparse(a, st));
}

// Sparse attention without a caller workspace (see include/hs2.h): same checks
// and kernel as hs2_sparse_attn, scratch taken from the library's fixed array.
hs2_status hs2_sparse_attn_noalloc(const hs2_attn_desc* desc, const void* q, const void* k, const void* v,
                                   const float* k_scale, const float* v_scale, const int32_t* idx,
                                   const int32_t* cnt, void* o, float* lse, hs2_stream_t stream) {
    Path path;
    hs2_status s = check_desc(desc, &path);
    if (s != HS2_OK) return s;
    if (path != Path::TC) return HS2_ERR_UNSUPPORTED;
    if (!q || !k || !v || !idx || !cnt || !o) return HS2_ERR_INVALID_ARG;
    const bool kv8 = desc->kv_dtype == HS2_E4M3;
    if (kv8 && (!k_scale || !v_scale)) return HS2_ERR_INVALID_ARG;
    const void* ptrs[] = {q, k, v, idx, cnt, o};
    for (const void* p : ptrs)
        if (!aligned16(p)) return HS2_ERR_INVALID_ARG;
    if (lse && !aligned16(lse)) return HS2_ERR_INVALID_ARG;
    SparseArgs a{};
    a.rows = desc->batch * desc->n_q; a.n_q = desc->n_q; a.cap = desc->kv_capacity; a.idx_stride = desc->idx_stride;
    a.q = q; a.k = k; a.v = v; a.k_scale = k_scale; a.v_scale = v_scale; a.kv8 = kv8;
    a.idx = idx; a.cnt = cnt; a.scale = eff_scale(desc); a.o = o; a.lse = lse;
    bool too_large = false;
    const cudaError_t e = launch_sparse_noalloc(a, reinterpret_cast<cudaStream_t>(stream), &too_large);
    if (too_large) return HS2_ERR_WORKSPACE;
    return from_cuda(e);
}

hs2_status hs2_kv_bridge_proj(const void* hidden, const void* w_kv, int32_t batch, int32_t n, int32_t d_model,
                              int32_t head_dim, const int32_t* pos0, int32_t kv_dtype, int64_t kv_capacity, void* k,
                              void* v, float* k_scale, float* v_scale, hs2_stream_t stream) {
    if (!hidden || !w_kv || !pos0 || !k || !v || batch < 1 || n < 1 || d_model < 1 || kv_capacity < n)
        return HS2_ERR_INVALID_ARG;
    const bool kv8 = kv_dtype == HS2_E4M3;
    if (kv_dtype != HS2_BF16 && !kv8) return HS2_ERR_UNSUPPORTED;
    if (kv8 && (!k_scale || !v_scale)) return HS2_ERR_INVALID_ARG;
    const void* ptrs[] = {hidden, w_kv, pos0, k, v};
    for (const void* p : ptrs)
        if (!aligned16(p)) return HS2_ERR_INVALID_ARG;
    if (kv8 && ((reinterpret_cast<uintptr_t>(k_scale) & 3u) || (reinterpret_cast<uintptr_t>(v_scale) & 3u)))
        return HS2_ERR_INVALID_ARG;
    if (head_dim != 128 || d_model % 64 != 0) return HS2_ERR_UNSUPPORTED;
    if (static_cast<int64_t>(batch) * n >= (int64_t(1) << 31) || static_cast<int64_t>(batch) * kv_capacity >= (int64_t(1) << 31))
        return HS2_ERR_UNSUPPORTED;
    BridgeArgs a{};
    a.hidden = hidden; a.w_kv = w_kv; a.batch = batch; a.n = n; a.d_model = d_model;
    a.pos0 = pos0; a.cap = kv_capacity; a.k = k; a.v = v; a.status = nullptr;
    a.k_scale = k_scale; a.v_scale = v_scale; a.kv8 = kv8;
    return from_cuda(launch_bridge(a, reinterpret_cast<cudaStream_t>(stream)));
}

hs2_status hs2_kv_quantize_fp8(const float* src, int64_t rows, int32_t head_dim, uint8_t* codes, float* scales,
                               hs2_stream_t stream) {
    if (!src || !codes || !scales || rows < 0) return HS2_ERR_INVALID_ARG;
    if (head_dim != 64 && head_dim != 128) return HS2_ERR_UNSUPPORTED;
    if (!aligned16(src) || !aligned16(codes) || (reinterpret_cast<uintptr_t>(scales) & 3u)) return HS2_ERR_INVALID_ARG;
    if (rows >= (int64_t(1) << 34)) return HS2_ERR_UNSUPPORTED;
    return from_cuda(launch_fp8_quantize(src, rows, head_dim, codes, scales, reinterpret_cast<cudaStream_t>(stream)));
}

hs2_status hs2_last_status(void* workspace, hs2_stream_t stream) {
    if (!workspace) return HS2_ERR_INVALID_ARG;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (cudaStreamSynchronize(st) != cudaSuccess) return HS2_ERR_CUDA;
    uint32_t word = 0;
    if (cudaMemcpy(&word, workspace, sizeof(word), cudaMemcpyDeviceToHost) != cudaSuccess) return HS2_ERR_CUDA;
    if (word != 0 && cudaMemset(workspace, 0, sizeof(word)) != cudaSuccess) return HS2_ERR_CUDA;
    return static_cast<hs2_status>(word);
}

const char* hs2_status_string(hs2_status status) {
    switch (status) {
        case HS2_OK: return "ok";
        case HS2_ERR_INVALID_ARG: return "invalid argument";
        case HS2_ERR_UNSUPPORTED: return "unsupported shape or dtype";
        case HS2_ERR_WORKSPACE: return "workspace too small";
        case HS2_ERR_CUDA: return "CUDA launch or stream error";
        case HS2_ERR_TIMEOUT: return "a bounded device wait timed out";
        case HS2_ERR_INDEX: return "index outside the cache";
    }
    return "unknown status";
}

}  // extern "C"
