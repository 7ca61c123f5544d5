// internal.h -- launch interfaces between the C-ABI layer and the kernel files.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

namespace hs2 {

// Number of SMs of the current device (cached per device).
int num_sms();


// Builds a 2-D tiled tensor map (row-major [rows][cols] of `elem_bytes` elements,
// row pitch `row_bytes`), box [box_rows][box_cols], 128-byte swizzle when
// `swizzle128` is set.  Returns false if the driver rejects it.
bool make_tmap_2d(CUtensorMap* map, const void* base, CUtensorMapDataType dtype, int elem_bytes,
                  uint64_t cols, uint64_t rows, uint64_t row_bytes, uint32_t box_cols,
                  uint32_t box_rows, bool swizzle128);

// ---------------------------------------------------------------- decode (n_q == 1)
struct DecodePlan {
    bool fused;          // one cooperative launch, logits in tensor memory
    int wb;              // fused: sequences per wave (CTAs = wb * splits <= SMs)
    int splits;          // key splits per sequence
    int chunk;           // keys per split (multiple of 64)
    int s_ld;            // row pitch of the logit buffer (multiple of 64; 0 when fused)
};
DecodePlan plan_decode(int batch, int64_t max_ctx, bool kv8);
size_t decode_ws_bytes(int batch, int64_t max_ctx, bool kv8);   // logits + partials + counters

// Token-level selection of a decode call (budget <= kFusedSelectMaxBudget): the attention
// kernels count the candidate importances of each row into a histogram (bins dec_bin, built in
// shared memory and added per CTA), and launch_hist_select takes the row's K best from the
// bins above the cutoff bin and the best of that bin.  The histogram and the counters of a row
// are zeroed by the attention kernels before they add to them.
constexpr int kDecTieCap = 4096;          // cutoff-bin keys kept per row (more: passes over the row)
struct DecSelState {
    int* hist;                            // [B][kDecHistRow]: coarse bins, then the refinement's fine bins
    int* ctl;                             // [B][4]: keys above the cutoff class, keys of it, CTAs done,
                                          //         CTAs past the refinement count
    int* above;                           // [B][budget] positions above the cutoff bin
    unsigned long long* tie;              // [B][kDecTieCap] (importance bits, ~position)
};
size_t dec_select_ws_bytes(int batch, int budget);
DecSelState dec_select_state(void* ws, int batch, int budget);
// Rows at least this long take the histogram selection; shorter ones the cluster select of
// launch_select, which holds them in shared memory (faster there than the histogram's
// counting inside the attention kernel and its passes over the rows).
constexpr int64_t kHistSelectMinCtx = 16 * 24576 + 1;

struct HistSelectArgs {
    int rows;                             // = batch (one query row per sequence)
    const int32_t* q_pos0;
    int64_t max_ctx;
    int window, budget, idx_stride;
    const float* scores;                  // [rows][score_ld]
    int64_t score_ld;
    int* hist;
    int* ctl;
    int* above;
    unsigned long long* tie;
    int slice;                            // keys per CTA (set by launch_hist_select)
    bool vec4;                            // rows 16-byte aligned: float4 loads (set there too)
    int32_t* idx;
    int32_t* cnt;
    uint32_t* status;
};
cudaError_t launch_hist_select(const HistSelectArgs& a, cudaStream_t st);

struct DecodeArgs {
    int batch;
    int64_t cap;
    int64_t max_ctx;
    const int32_t* q_pos0;
    const void* q;            // [B][16][128] bf16
    const void* k;            // [B][cap][128] bf16 or e4m3
    const void* v;
    const float* k_scale;     // [B][cap] (e4m3)
    const float* v_scale;
    bool kv8;
    float scale;
    void* o;                  // [B][16][128] bf16
    float* lse;               // [B][16] or null
    float* scores;            // [B][score_ld]
    int64_t score_ld;
    void* ws;                 // decode scratch (decode_ws_bytes)
    uint32_t* status;
    int window;               // candidates of a row: keys [0, p - window]
    DecSelState sel;          // selection histogram and counters (hist null: none built)
};
cudaError_t launch_decode_full(const DecodeArgs& a, cudaStream_t st);

// ---------------------------------------------------------------- prefill (n_q > 1), tcgen05
// Token-level selection of a prefill call runs fused: pass 2 streams each row's
// candidates (keys whose importance reaches the row's running cutoff bound) into the
// workspace, and launch_cand_select picks the top K from them.  Budgets above
// kFusedSelectMaxBudget use the importance rows and launch_select instead.
constexpr int kFusedSelectMaxBudget = 4096;

struct CandSelectArgs {
    int rows, n_q;
    const int32_t* q_pos0;
    int64_t max_ctx;
    int window, budget, idx_stride;
    const uint32_t* hist;     // [rows][kImpBins] candidates per importance bin
    const int* cand_cnt;      // [rows][2] entries per segment
    const uint2* cand;        // [rows][2][cand_seg] (importance bits, position)
    int64_t cand_seg;
    int map_words;            // set by launch_cand_select: bitmap words per CTA (0: position lists)
    int32_t* idx;
    int32_t* cnt;
    uint32_t* status;
};
cudaError_t launch_cand_select(const CandSelectArgs& a, cudaStream_t st);

struct PrefillArgs {
    int batch, n_q;
    int64_t cap, max_ctx;
    const int32_t* q_pos0;
    const void* q;            // [B][n_q][16][128] bf16
    const void* k;            // [B][cap][128] bf16, or e4m3 codes when kv8
    const void* v;
    const float* k_scale;     // [B][cap] (kv8)
    const float* v_scale;
    bool kv8;
    float scale;
    void* o;                  // [B][n_q][16][128] bf16
    float* lse;               // [B][n_q][16] natural log, or null
    float* scores;            // [B][n_q][score_ld] importance rows, or null
    int64_t score_ld;
    void* ws;                 // prefill_ws_bytes
    uint32_t* status;
    bool fused_select;        // selection fused into pass 2 (then idx/cnt are written here)
    int window, budget, idx_stride;
    int32_t* idx;
    int32_t* cnt;
};
size_t prefill_ws_bytes(int batch, int n_q, int64_t max_ctx, bool fused_select, bool kv8);
cudaError_t launch_prefill_full(const PrefillArgs& a, cudaStream_t st);

// ---------------------------------------------------------------- selection
struct SelectArgs {
    int rows;                 // batch * n_q
    int n_q;
    const int32_t* q_pos0;
    const float* scores;
    int64_t score_ld;
    int window, budget, block_size, idx_stride;
    int32_t* idx;
    int32_t* cnt;
    int64_t max_ctx;          // positions are clamped below it (violations flag HS2_ERR_INDEX)
    uint32_t* status;
};
cudaError_t launch_select(const SelectArgs& a, cudaStream_t st);


// ---------------------------------------------------------------- sparse attention
struct SparsePlan {
    int splits;
    int chunk;               // selected entries per split (multiple of 64; of 16 in cluster mode)
    bool cluster;            // one cluster of CTAs per row, partials merged on chip
};
SparsePlan plan_sparse(int rows, int idx_stride);
size_t sparse_ws_bytes(int rows, int idx_stride);

struct SparseArgs {
    int rows, n_q;
    int64_t cap;
    int idx_stride;
    const void* q;            // [rows][16][128] bf16
    const void* k;
    const void* v;
    const float* k_scale;
    const float* v_scale;
    bool kv8;
    const int32_t* idx;
    const int32_t* cnt;
    float scale;
    void* o;                  // [rows][16][128] bf16
    float* lse;
    void* ws;
    uint32_t* status;
    bool one_split;           // one CTA per row whatever the row count (no split partials)
};
cudaError_t launch_sparse(const SparseArgs& a, cudaStream_t st);

// Same kernel with its scratch in a fixed device array (no caller workspace).  When
// the split plan's partials would not fit the array, the rows run one CTA each, which
// needs none; *too_large is set, and nothing launched, only if even that does not fit.
cudaError_t launch_sparse_noalloc(const SparseArgs& a, cudaStream_t st, bool* too_large);
size_t sparse_noalloc_capacity();

// ---------------------------------------------------------------- fp32 SIMT path
struct F32Args {
    int batch, n_q, heads, head_dim;
    int64_t cap;
    int64_t max_ctx;
    const int32_t* q_pos0;
    const float* q;
    const float* k;
    const float* v;
    float scale;
    float* o;
    float* lse;
    float* scores;           // [rows][score_ld]
    int64_t score_ld;
    // sparse
    const int32_t* idx;
    const int32_t* cnt;
    int idx_stride;
    uint32_t* status;
};
cudaError_t launch_f32_full(const F32Args& a, cudaStream_t st);
cudaError_t launch_f32_sparse(const F32Args& a, cudaStream_t st);

// ---------------------------------------------------------------- KV bridge GEMM
struct BridgeArgs {
    const void* hidden;      // [batch][n][d_model] bf16
    const void* w_kv;        // [d_model][256] bf16
    int batch, n, d_model;
    const int32_t* pos0;     // [batch] device
    int64_t cap;
    void* k;                 // [batch][cap][128] bf16, or e4m3 codes when kv8
    void* v;
    float* k_scale;          // [batch][cap] per-row scales (kv8 only)
    float* v_scale;
    bool kv8;
    uint32_t* status;        // may be null
};
cudaError_t launch_bridge(const BridgeArgs& a, cudaStream_t st);

// ---------------------------------------------------------------- fp8 quantizer
cudaError_t launch_fp8_quantize(const float* src, int64_t rows, int head_dim, uint8_t* codes,
                                float* scales, cudaStream_t st);

}  // namespace hs2
