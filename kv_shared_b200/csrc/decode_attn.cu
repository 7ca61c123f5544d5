// decode_attn.cu -- full-attention layer of a hybrid block for one new query
// token per sequence (decode), with the per-key importance the selection needs.
//
// Importance of key j = sum over the 16 query heads of the softmax probability
// P_h[j] = exp(s_h[j] - LSE_h) (the pages leave the rule open: "What HySparse2 is
// actually optimizing", "What is not documented"), so every probability must be
// normalized by the FINAL log-sum-exp.  Two streaming passes over each split of
// the cache:
//
//   pass A  S = scale * K q^T for all heads (mma.sync, M = 16 heads), the scaled
//           logits kept, and a running (max, sum) per head -> per-split partials.
//   pass B  the partials of all splits merged into LSE, the logits re-read, P
//           formed exactly normalized, importance = sum_h P written and O = P V
//           accumulated (no online rescaling: LSE is final); the split partials
//           of O are then summed per (sequence, head).
//
// Single-launch path (dec_fused_kernel, splits of up to 4096 keys): one
// cooperative launch, the logits kept in tensor memory between the passes, the
// splits of a sequence exchanging (max, sum) through counters.  Two-kernel path
// (contexts over 148 x 4096 keys): dec_qk_kernel, dec_pv_kernel and
// dec_merge_kernel, the logits through a [B][16][S_ld] fp32 buffer (64 B per key).
// K is read once (pass A) and V once (pass B).  Tiles of 64 keys stream through
// TMA rings with 128-byte swizzle; e4m3 tiles feed f16 MMAs straight from shared
// memory (e4m3 -> f16 is exact) and the per-token scales are folded into the
// logits and into P.
#include "common.cuh"
#include "e4m3_mma.cuh"
#include "internal.h"
#include "tcgen05.cuh"

namespace hs2 {
namespace {

constexpr int H = 16;
constexpr int D = 128;
constexpr int TILE = 64;
constexpr int STAGES = 4;
constexpr int NT = 128;            // 4 warps, each owns 16 keys of a tile

struct Params {
    int B;
    int64_t cap;
    int64_t max_ctx;
    int splits, chunk, s_ld;
    const int32_t* q_pos0;
    const __nv_bfloat16* q;
    const float* k_scale;
    const float* v_scale;
    float sc2;                      // softmax scale * log2(e)
    float* S;                       // [B][H][s_ld] logits, log2 units
    float2* part_ml;                // [B][splits][H]: (max, sum) in log2 units
    float* part_vmax;               // [B][splits]: largest V scale of the split (e4m3)
    float* part_o;                  // [B][splits][H][D]
    int* counter;                   // fused path: [3][B] in the status block
    __nv_bfloat16* o;               // [B][H][D]
    float* lse;                     // [B][H] natural log, or null
    float* scores;                  // [B][score_ld]
    int64_t score_ld;
    uint32_t* status;
    int window;                     // candidates of a row for the selection: keys [0, p - window]
    int* ghist;                     // [B][kDecHistRow] selection histogram (coarse, fine), or null
    int* gctl;                      // [B][4] selection counters (zeroed with the histogram)
};

// Zeroes row b's selection histogram and counters (n threads from thread t), before any CTA
// adds to them; each thread's stores are made visible before it goes on.
__device__ __forceinline__ void zero_select_state(const Params& a, int b, int t, int n) {
    for (int i = t; i < kDecHistRow; i += n) a.ghist[static_cast<size_t>(b) * kDecHistRow + i] = 0;
    if (t < 4) a.gctl[4 * b + t] = 0;
    __threadfence();
}

// Counts the candidate keys among a thread's four importance values into the shared-memory
// histogram hs (keys below c_end = p - window + 1; valid[e] marks keys that exist).
__device__ __forceinline__ void count_candidates(int* hs, const float (&sc)[4], const int (&key)[4],
                                                 const bool (&valid)[4], int c_end) {
#pragma unroll
    for (int e = 0; e < 4; ++e)
        if (valid[e] && key[e] < c_end) atomicAdd(&hs[dec_bin(__float_as_uint(sc[e]))], 1);
}

// Adds a CTA's shared-memory histogram to row b's and clears it (threads t, t + n, ...).
__device__ __forceinline__ void flush_hist(const Params& a, int* hs, int b, int t, int n) {
    for (int i = t; i < kDecHistBins; i += n) {
        const int c = hs[i];
        if (c) {
            atomicAdd(a.ghist + static_cast<size_t>(b) * kDecHistRow + i, c);
            hs[i] = 0;
        }
    }
}

template <bool KV8>
struct Layout {
    static constexpr int RAW = KV8 ? TILE * 128 : TILE * 256;   // one cache tile as loaded
    static constexpr int STILE = 16 * 32 * 4 * 2;               // logits tile: 2 boxes 16x32 fp32
};

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
    return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

// Q A-fragments of the m16n8k16 tile: 16 heads x 128 dims, 8 k-steps.
__device__ __forceinline__ void load_q_frags(const __nv_bfloat16* qb, int g, int t, uint32_t (&qa)[8][4]) {
    const uint32_t* q32 = reinterpret_cast<const uint32_t*>(qb);
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
        qa[ks][0] = __ldg(q32 + (g * D + 16 * ks + 2 * t) / 2);
        qa[ks][1] = __ldg(q32 + ((g + 8) * D + 16 * ks + 2 * t) / 2);
        qa[ks][2] = __ldg(q32 + (g * D + 16 * ks + 2 * t + 8) / 2);
        qa[ks][3] = __ldg(q32 + ((g + 8) * D + 16 * ks + 2 * t + 8) / 2);
    }
}

__device__ __forceinline__ void merge_ml(float& m, float& l, float m2, float l2) {
    const float mn = fmaxf(m, m2);
    if (mn == -INFINITY) return;
    l = l * ex2(m - mn) + l2 * ex2(m2 - mn);
    m = mn;
}

// ------------------------------------------------------------------ pass A
template <bool KV8>
__global__ void __launch_bounds__(NT) dec_qk_kernel(const __grid_constant__ CUtensorMap kmap, Params a) {
    using L = Layout<KV8>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = align1024(smem_raw);
    uint8_t* raw = smem;
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + STAGES * L::RAW);
    __shared__ float red_m[4][H], red_l[4][H], red_v[4];

    const int b = blockIdx.y, split = blockIdx.x;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, g = lane >> 2, t = lane & 3;
    const int p = checked_pos(a.q_pos0[b], a.max_ctx, a.status);
    const int k_begin = split * a.chunk;
    const int k_end = min(p + 1, k_begin + a.chunk);
    const int n_tiles = k_end > k_begin ? (k_end - k_begin + TILE - 1) / TILE : 0;

    if (tid == 0) {
        prefetch_tmap(&kmap);
        for (int s = 0; s < STAGES; ++s) mbar_init(&full[s], 1);
        fence_mbar_init();
    }
    if (a.ghist && split == 0) zero_select_state(a, b, tid, NT);   // dec_pv adds to it
    __syncthreads();

    auto issue = [&](int i, int s) {
        const int row = static_cast<int>(b * a.cap) + k_begin + i * TILE;
        mbar_arrive_expect_tx(&full[s], L::RAW);
        if (KV8) {
            tma_load_2d(raw + s * L::RAW, &kmap, &full[s], 0, row);
        } else {
            tma_load_2d(raw + s * L::RAW, &kmap, &full[s], 0, row);
            tma_load_2d(raw + s * L::RAW + TILE * 128, &kmap, &full[s], 64, row);
        }
    };
    if (tid == 0)
        for (int s = 0; s < STAGES && s < n_tiles; ++s) issue(s, s);

    // e4m3 keys: f16 MMAs straight from the raw tile (Q in f16, k order permuted, scaled
    // by 1 / qscale); the largest V scale of the split is kept for pass B's f16 P
    uint32_t qa[8][4];
    float qscale = 1.f, vmax = 0.f;
    if (KV8) qscale = load_q_frags_e4m3(a.q + static_cast<size_t>(b) * H * D, g, t, qa);
    else load_q_frags(a.q + static_cast<size_t>(b) * H * D, g, t, qa);

    float m2[2] = {-INFINITY, -INFINITY}, l2[2] = {0.f, 0.f};
    float* Sg = a.S + (static_cast<size_t>(b) * H + g) * a.s_ld;
    float* Sg8 = Sg + static_cast<size_t>(8) * a.s_ld;
    const float* ksc = KV8 ? a.k_scale + b * a.cap : nullptr;
    const float* vsc = KV8 ? a.v_scale + b * a.cap : nullptr;
    const float sc2 = a.sc2 * qscale;
    // e4m3: lane l of a warp holds the key scale (l < 16) or the V scale (l >= 16) of key
    // l % 16 of its 16 keys of a tile: one coalesced load per tile, issued four tiles ahead
    // so that the memory latency stays off the tile's path
    auto load_sc = [&](int i) -> float {
        const int key = k_begin + i * TILE + warp * 16 + (lane & 15);
        return (i < n_tiles && key < k_end) ? __ldg((lane < 16 ? ksc : vsc) + key) : 0.f;
    };
    float sc_p[4] = {0.f, 0.f, 0.f, 0.f};
    if (KV8)
#pragma unroll
        for (int j = 0; j < 4; ++j) sc_p[j] = load_sc(j);

    for (int i = 0; i < n_tiles; ++i) {
        const int s = i % STAGES;
        const float sc_cur = sc_p[0];
        if (KV8) {
            sc_p[0] = sc_p[1]; sc_p[1] = sc_p[2]; sc_p[2] = sc_p[3];
            sc_p[3] = load_sc(i + 4);
            if (lane >= 16) vmax = fmaxf(vmax, sc_cur);
        }
        bool ok = mbar_wait(&full[s], (i / STAGES) & 1, a.status);
        const int tile_key0 = k_begin + i * TILE;
        const uint8_t* tile = raw + s * L::RAW;
        const uint32_t tbase = smem_u32(tile);
        float acc[2][4];
        if (KV8) {
            qk_e4m3(tbase, warp * 16, qa, acc, lane);
        } else {
#pragma unroll
            for (int nt = 0; nt < 2; ++nt) {
#pragma unroll
                for (int e = 0; e < 4; ++e) acc[nt][e] = 0.f;
                const int r = warp * 16 + nt * 8 + (lane & 7);
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
                    uint32_t b0, b1, b2, b3;
                    ldsm_x4(tbase + swz_off<TILE>(r, 4 * kk + (lane >> 3)), b0, b1, b2, b3);
                    mma_bf16(acc[nt], qa[2 * kk], b0, b1);
                    mma_bf16(acc[nt], qa[2 * kk + 1], b2, b3);
                }
            }
        }
        // logits (log2 units), masked past the last key
        const int key0 = tile_key0 + warp * 16 + 2 * t;
        float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
            const int key = key0 + nt * 8;
            float f0 = sc2, f1 = sc2;
            if (KV8) {
                f0 *= __shfl_sync(0xffffffffu, sc_cur, nt * 8 + 2 * t);
                f1 *= __shfl_sync(0xffffffffu, sc_cur, nt * 8 + 2 * t + 1);
            }
            acc[nt][0] = (key < k_end) ? acc[nt][0] * f0 : -INFINITY;
            acc[nt][1] = (key + 1 < k_end) ? acc[nt][1] * f1 : -INFINITY;
            acc[nt][2] = (key < k_end) ? acc[nt][2] * f0 : -INFINITY;
            acc[nt][3] = (key + 1 < k_end) ? acc[nt][3] * f1 : -INFINITY;
            if (key < k_end) {
                *reinterpret_cast<float2*>(Sg + key) = make_float2(acc[nt][0], acc[nt][1]);
                *reinterpret_cast<float2*>(Sg8 + key) = make_float2(acc[nt][2], acc[nt][3]);
            }
            mx[0] = fmaxf(mx[0], fmaxf(acc[nt][0], acc[nt][1]));
            mx[1] = fmaxf(mx[1], fmaxf(acc[nt][2], acc[nt][3]));
        }
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
            const float mn = fmaxf(m2[hh], mx[hh]);
            if (mn != -INFINITY) {
                float sum = l2[hh] * ex2(m2[hh] - mn);
#pragma unroll
                for (int nt = 0; nt < 2; ++nt)
                    sum += ex2(acc[nt][2 * hh] - mn) + ex2(acc[nt][2 * hh + 1] - mn);
                l2[hh] = sum;
                m2[hh] = mn;
            }
        }
        if (__syncthreads_or(!ok)) break;
        if (tid == 0 && i + STAGES < n_tiles) issue(i + STAGES, s);
    }

    // reduce (max, sum) over the quad, then over warps
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
#pragma unroll
        for (int off = 1; off <= 2; off <<= 1) {
            const float om = __shfl_xor_sync(0xffffffffu, m2[hh], off);
            const float ol = __shfl_xor_sync(0xffffffffu, l2[hh], off);
            merge_ml(m2[hh], l2[hh], om, ol);
        }
    }
    if (t == 0) {
        red_m[warp][g] = m2[0]; red_l[warp][g] = l2[0];
        red_m[warp][g + 8] = m2[1]; red_l[warp][g + 8] = l2[1];
    }
    if (KV8) {
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) vmax = fmaxf(vmax, __shfl_xor_sync(0xffffffffu, vmax, off));
        if (lane == 0) red_v[warp] = vmax;
    }
    __syncthreads();
    if (tid < H) {
        float m = red_m[0][tid], l = red_l[0][tid];
        for (int w = 1; w < 4; ++w) merge_ml(m, l, red_m[w][tid], red_l[w][tid]);
        a.part_ml[(static_cast<size_t>(b) * a.splits + split) * H + tid] = make_float2(m, l);
    }
    if (KV8 && tid == 0)
        a.part_vmax[static_cast<size_t>(b) * a.splits + split] =
            fmaxf(fmaxf(red_v[0], red_v[1]), fmaxf(red_v[2], red_v[3]));
}

// ------------------------------------------------------------------ pass B
template <bool KV8>
__global__ void __launch_bounds__(NT) dec_pv_kernel(const __grid_constant__ CUtensorMap vmap,
                                                    const __grid_constant__ CUtensorMap smap, Params a) {
    using L = Layout<KV8>;
    constexpr int STAGE = L::RAW + L::STILE;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = align1024(smem_raw);
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + STAGES * STAGE);
    float4* red_o4 = reinterpret_cast<float4*>(smem);              // [4][16][32] after the tiles
    __shared__ int hs[kDecHistBins];                               // this CTA's selection counts

    const int b = blockIdx.y, split = blockIdx.x;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, g = lane >> 2, t = lane & 3;
    const int p = checked_pos(a.q_pos0[b], a.max_ctx, a.status);
    const int k_begin = split * a.chunk;
    const int k_end = min(p + 1, k_begin + a.chunk);
    const int n_tiles = k_end > k_begin ? (k_end - k_begin + TILE - 1) / TILE : 0;

    if (tid == 0) {
        prefetch_tmap(&vmap);
        prefetch_tmap(&smap);
        for (int s = 0; s < STAGES; ++s) mbar_init(&full[s], 1);
        fence_mbar_init();
    }
    for (int i = tid; i < kDecHistBins; i += NT) hs[i] = 0;
    const int c_end = p - a.window + 1;
    __syncthreads();

    auto issue = [&](int i, int s) {
        uint8_t* st = smem + s * STAGE;
        const int key = k_begin + i * TILE;
        const int row = static_cast<int>(b * a.cap) + key;
        mbar_arrive_expect_tx(&full[s], STAGE);
        tma_load_2d(st, &vmap, &full[s], 0, row);
        if (!KV8) tma_load_2d(st + TILE * 128, &vmap, &full[s], 64, row);
        tma_load_2d(st + L::RAW, &smap, &full[s], key, b * H);
        tma_load_2d(st + L::RAW + 2048, &smap, &full[s], key + 32, b * H);
    };
    if (tid == 0)
        for (int s = 0; s < STAGES && s < n_tiles; ++s) issue(s, s);

    // final log-sum-exp per head: all splits' partials are read in parallel (thread t
    // takes head t % 16 and every 8th split), then the 8 groups are combined
    __shared__ float2 lse_part[NT / H][H];
    __shared__ float lse_s[H];
    {
        const int h = tid & (H - 1), grp = tid >> 4;
        float m = -INFINITY, l = 0.f;
        const float2* pml = a.part_ml + static_cast<size_t>(b) * a.splits * H;
#pragma unroll 4
        for (int s = grp; s < a.splits; s += NT / H) {
            const float2 ml = pml[s * H + h];
            merge_ml(m, l, ml.x, ml.y);
        }
        lse_part[grp][h] = make_float2(m, l);
        __syncthreads();
        if (tid < H) {
            float mm = -INFINITY, ll = 0.f;
            for (int q = 0; q < NT / H; ++q) merge_ml(mm, ll, lse_part[q][tid].x, lse_part[q][tid].y);
            lse_s[tid] = mm + log2f(ll);
            if (split == 0 && a.lse) a.lse[static_cast<size_t>(b) * H + tid] = lse_s[tid] * kLn2;
        }
        __syncthreads();
    }
    float lse2[2] = {lse_s[g], lse_s[g + 8]};

    float o[16][4];
#pragma unroll
    for (int n = 0; n < 16; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;
    const float* vsc = KV8 ? a.v_scale + b * a.cap : nullptr;
    float* score_row = a.scores + b * a.score_ld;
    // e4m3 values: P V in f16 with P * v_scale * 2^pe, the largest product of the split
    // (at most its largest V scale, P <= 1) scaled to 2^14 or below; O is scaled back
    float pscale = 1.f, pinv = 1.f;
    if (KV8) {
        const float vm = a.part_vmax[static_cast<size_t>(b) * a.splits + split];
        int ex = 0;
        if (vm > 0.f) frexpf(vm, &ex);          // vm < 2^ex
        pscale = ldexpf(1.f, 14 - ex);
        pinv = ldexpf(1.f, ex - 14);
    }
    // e4m3: lane l holds the V scale of key l % 16 of the warp's 16 keys of a tile, loaded
    // four tiles ahead (one coalesced load per tile)
    auto load_vs = [&](int i) -> float {
        const int key = k_begin + i * TILE + warp * 16 + (lane & 15);
        return (i < n_tiles && key < k_end) ? __ldg(vsc + key) : 0.f;
    };
    float vs_p[4] = {0.f, 0.f, 0.f, 0.f};
    if (KV8)
#pragma unroll
        for (int j = 0; j < 4; ++j) vs_p[j] = load_vs(j);

    for (int i = 0; i < n_tiles; ++i) {
        const int s = i % STAGES;
        const float vs_cur = vs_p[0];
        if (KV8) {
            vs_p[0] = vs_p[1]; vs_p[1] = vs_p[2]; vs_p[2] = vs_p[3];
            vs_p[3] = load_vs(i + 4);
        }
        bool ok = mbar_wait(&full[s], (i / STAGES) & 1, a.status);
        uint8_t* st = smem + s * STAGE;
        const int tile_key0 = k_begin + i * TILE;
        uint8_t* vt = st;
        if (KV8) {
            if (tile_key0 + TILE > k_end) {
                // tail tile: zero the e4m3 rows past the last key (codes there may be NaN)
                for (int it = tid; it < TILE * 8; it += NT) {
                    const int r = it >> 3, c = it & 7;
                    if (tile_key0 + r >= k_end) *reinterpret_cast<uint4*>(vt + r * 128 + c * 16) = make_uint4(0, 0, 0, 0);
                }
                __syncthreads();
            }
        } else if (tile_key0 + TILE > k_end) {
            // tail tile: zero the V rows past the last key (cache rows there may hold
            // anything, and 0 * NaN would poison the accumulators)
            for (int it = tid; it < TILE * 16; it += NT) {
                const int r = it >> 4, c = it & 15;
                if (tile_key0 + r >= k_end)
                    *reinterpret_cast<uint4*>(vt + swz_off<TILE>(r, c)) = make_uint4(0, 0, 0, 0);
            }
            __syncthreads();
        }
        // logits of this warp's 16 keys from the swizzled [16 heads][2 x 32 keys] tile
        const uint8_t* stile = st + L::RAW;
        const int c0 = 16 * (warp & 1) + 2 * t;
        const uint8_t* half = stile + (warp >> 1) * 2048;
        auto sld = [&](int hr, int c) {
            return *reinterpret_cast<const float2*>(half + hr * 128 + (((c >> 2) ^ (hr & 7)) << 4) + (c & 3) * 4);
        };
        const float2 sgl = sld(g, c0), sg8l = sld(g + 8, c0), sgh = sld(g, c0 + 8), sg8h = sld(g + 8, c0 + 8);
        const int kl = tile_key0 + warp * 16 + 2 * t, kh = kl + 8;
        const bool v0 = kl < k_end, v1 = kl + 1 < k_end, v2 = kh < k_end, v3 = kh + 1 < k_end;
        const float p00 = v0 ? ex2(sgl.x - lse2[0]) : 0.f, p01 = v1 ? ex2(sgl.y - lse2[0]) : 0.f;
        const float p10 = v0 ? ex2(sg8l.x - lse2[1]) : 0.f, p11 = v1 ? ex2(sg8l.y - lse2[1]) : 0.f;
        const float p02 = v2 ? ex2(sgh.x - lse2[0]) : 0.f, p03 = v3 ? ex2(sgh.y - lse2[0]) : 0.f;
        const float p12 = v2 ? ex2(sg8h.x - lse2[1]) : 0.f, p13 = v3 ? ex2(sg8h.y - lse2[1]) : 0.f;
        // importance: sum over the 16 heads (pair here, then across the 8 row groups)
        float sc[4] = {p00 + p10, p01 + p11, p02 + p12, p03 + p13};
#pragma unroll
        for (int off = 4; off <= 16; off <<= 1)
#pragma unroll
            for (int e = 0; e < 4; ++e) sc[e] += __shfl_xor_sync(0xffffffffu, sc[e], off);
        if (g == 0) {
            if (v0) score_row[kl] = sc[0];
            if (v1) score_row[kl + 1] = sc[1];
            if (v2) score_row[kh] = sc[2];
            if (v3) score_row[kh + 1] = sc[3];
        }
        const uint32_t vbase = smem_u32(vt);
        if (KV8) {
            const float f0 = __shfl_sync(0xffffffffu, vs_cur, 2 * t) * pscale;
            const float f1 = __shfl_sync(0xffffffffu, vs_cur, 2 * t + 1) * pscale;
            const float f2 = __shfl_sync(0xffffffffu, vs_cur, 2 * t + 8) * pscale;
            const float f3 = __shfl_sync(0xffffffffu, vs_cur, 2 * t + 9) * pscale;
            uint32_t pa[4];
            pa[0] = pack_f16(p00 * f0, p01 * f1);
            pa[1] = pack_f16(p10 * f0, p11 * f1);
            pa[2] = pack_f16(p02 * f2, p03 * f3);
            pa[3] = pack_f16(p12 * f2, p13 * f3);
            pv_e4m3(vbase, warp * 16, pa, o, lane);
        } else {
            uint32_t pa[4];
            pa[0] = pack_bf16(p00, p01);
            pa[1] = pack_bf16(p10, p11);
            pa[2] = pack_bf16(p02, p03);
            pa[3] = pack_bf16(p12, p13);
            const int vr = warp * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                uint32_t b0, b1, b2, b3;
                ldsm_x4_t(vbase + swz_off<TILE>(vr, 2 * c + (lane >> 4)), b0, b1, b2, b3);
                mma_bf16(o[2 * c], pa, b0, b1);
                mma_bf16(o[2 * c + 1], pa, b2, b3);
            }
        }
        // selection counts, after the MMAs so that they stay off the tile's path
        if (a.ghist && g == 0) count_candidates(hs, sc, {kl, kl + 1, kh, kh + 1}, {v0, v1, v2, v3}, c_end);
        if (__syncthreads_or(!ok)) break;
        if (tid == 0 && i + STAGES < n_tiles) issue(i + STAGES, s);
    }

    // this split's O partial: the 4 warps' accumulators through shared memory (the stage
    // area, free once every tile is consumed) as [warp][n][lane] float4 (conflict-free),
    // each (n, lane) slot summed over the warps in a fixed order; the partials of all splits
    // are summed by dec_merge_kernel.  e4m3: accumulator n holds dims 32 (n / 4) + 16 ((n / 2)
    // % 2) + 4 t + n % 2 and that + 2 (see pv_e4m3), scaled by pscale.
    __syncthreads();
#pragma unroll
    for (int n = 0; n < 16; ++n)
        red_o4[(warp * 16 + n) * 32 + lane] = make_float4(o[n][0] * pinv, o[n][1] * pinv, o[n][2] * pinv, o[n][3] * pinv);
    __syncthreads();
    float* my = a.part_o + (static_cast<size_t>(b) * a.splits + split) * H * D;
#pragma unroll
    for (int k = 0; k < 512 / NT; ++k) {
        const int e = tid + k * NT, n = e >> 5, ln = e & 31;
        float4 sum = red_o4[e];
#pragma unroll
        for (int w4 = 1; w4 < 4; ++w4) {
            const float4 v = red_o4[w4 * 512 + e];
            sum.x += v.x; sum.y += v.y; sum.z += v.z; sum.w += v.w;
        }
        const int h = ln >> 2, tq = ln & 3;
        if (KV8) {
            const int d = 32 * (n >> 2) + 16 * ((n >> 1) & 1) + 4 * tq + (n & 1);
            my[h * D + d] = sum.x;
            my[h * D + d + 2] = sum.y;
            my[(h + 8) * D + d] = sum.z;
            my[(h + 8) * D + d + 2] = sum.w;
        } else {
            const int d = 8 * n + 2 * tq;
            *reinterpret_cast<float2*>(my + h * D + d) = make_float2(sum.x, sum.y);
            *reinterpret_cast<float2*>(my + (h + 8) * D + d) = make_float2(sum.z, sum.w);
        }
    }
    if (a.ghist) flush_hist(a, hs, b, tid, NT);      // every warp's counts are in (barriers above)
}

// O = sum of the split partials: CTA (row, group) = (blockIdx.x / 8, blockIdx.x % 8) takes
// dims 16 group .. + 15 of row (sequence, head): 4 float4 columns x 32 split lanes, the
// lanes combined in a fixed order.
constexpr int kMergeGroups = 8;
__global__ void __launch_bounds__(NT) dec_merge_kernel(Params a) {
    __shared__ float4 part[32][4];
    const int row = blockIdx.x / kMergeGroups, grp = blockIdx.x % kMergeGroups;
    const int b = row / H, h = row % H;
    const int c4 = threadIdx.x & 3, sl = threadIdx.x >> 2;
    const float4* src = reinterpret_cast<const float4*>(a.part_o + static_cast<size_t>(b) * a.splits * H * D + h * D) +
                        4 * grp + c4;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 4
    for (int sp = sl; sp < a.splits; sp += 32) {
        const float4 v = __ldg(src + static_cast<size_t>(sp) * (H * D / 4));
        acc.x += v.x; acc.y += v.y; acc.z += v.z; acc.w += v.w;
    }
    part[sl][c4] = acc;
    __syncthreads();
    if (threadIdx.x < 4) {
        float4 t = part[0][c4];
        for (int q = 1; q < 32; ++q) {
            const float4 v = part[q][c4];
            t.x += v.x; t.y += v.y; t.z += v.z; t.w += v.w;
        }
        uint2 packed;
        packed.x = pack_bf16(t.x, t.y);
        packed.y = pack_bf16(t.z, t.w);
        *reinterpret_cast<uint2*>(a.o + (static_cast<size_t>(b) * H + h) * D + 16 * grp + 4 * c4) = packed;
    }
}

// ------------------------------------------------------------------ fused passes (one launch)
// When a split's logits fit in tensor memory (64 tiles of 64 keys: 16 heads x 4096 keys of
// fp32 = 256 KB), both passes run in one cooperative launch and the logits never leave the
// SM: the 64-byte-per-key round trip through HBM disappears.  One CTA per SM; the sequences
// are taken in waves of `wb` (CTA = group * splits + split, sequence = wave * wb + group).
//
// Warp 8 streams the K tiles then the V tiles of every wave through a ring of TMA stages
// (full/empty mbarriers); warps 0-3 and 4-7 are two consumer groups taking the even and the
// odd tiles.  Per wave a CTA runs pass A over its keys with the logits stored to tensor
// memory (tile i, warp quarter q: lanes 32 q + 16 (i / 32), columns 16 (i % 32); the 16x256b
// store shape is the mma.sync accumulator layout of the warp's 16 keys), publishes its
// (max, sum) per head, waits -- bounded -- until every split of the sequence has (the first
// V tiles are in flight meanwhile), and runs pass B with the logits read back from tensor
// memory.  Each split leaves its O partial in the workspace and counts itself in (second
// counter); after its waves every CTA sums the partials of a few (sequence, head) rows, each
// once its sequence is complete, and the last row of a sequence (third counter) returns the
// sequence's three counters to zero.
constexpr int kFusedMaxTiles = 64;
constexpr int FNT = 288;                       // 2 x 4 consumer warps + 1 producer warp
constexpr int FCONS = 256;
constexpr size_t kFusedMinSmem = 120 * 1024;   // more than half an SM: one CTA per SM

template <bool KV8>
struct FusedLayout {
    static constexpr int FS = KV8 ? 16 : 8;    // stages of the K/V stream (128 KB)
    // The two consumer groups take alternate loads.  With an odd depth, load ld - FS of
    // stage ld % FS belongs to the other group, which may lag: a group waiting for load ld
    // before ld - FS has landed would see the phase of ld - 2 FS, whose parity equals ld's,
    // and read a stale tile.  An even depth keeps every stage within one group.
    static_assert(FS % 2 == 0, "the ring depth must be even (stage parity per consumer group)");
    static constexpr size_t VSC = KV8 ? kFusedMaxTiles * TILE * 4 : 0;   // V scales of the split
    static constexpr size_t BYTES = 1024 + FS * Layout<KV8>::RAW + 2 * FS * 8 + 8 * H * D * 4 + VSC + kDecHistBins * 4;
};

__device__ __forceinline__ void bar_sync(int id, int n) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}

__device__ __forceinline__ int ld_acquire(const int* p) {
    int v;
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// Bounded wait until *p >= target; false (status set) on timeout.
__device__ __forceinline__ bool wait_count(const int* p, int target, uint32_t* status) {
    const uint64_t t0 = global_ns();
#pragma unroll 1
    for (uint32_t i = 0; i < kWaitPolls; ++i) {
        if (ld_acquire(p) >= target) return true;
        if ((i & 15) == 15) {
            if (global_ns() - t0 > kWaitNs) break;
            __nanosleep(64);
        }
    }
    set_status(status, HS2_ERR_TIMEOUT);
    return false;
}

template <bool KV8>
__global__ void __launch_bounds__(FNT, 1) dec_fused_kernel(const __grid_constant__ CUtensorMap kmap,
                                                           const __grid_constant__ CUtensorMap vmap, Params a,
                                                           int wb) {
    using L = Layout<KV8>;
    constexpr int FS = FusedLayout<KV8>::FS;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = align1024(smem_raw);
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + FS * L::RAW);
    uint64_t* empty = full + FS;
    float4* red_o4 = reinterpret_cast<float4*>(empty + FS);          // [8][16][32] O partials
    float* vsm = reinterpret_cast<float*>(red_o4 + 8 * 16 * 32);      // [64 tiles][64] (e4m3)
    int* hs = reinterpret_cast<int*>(vsm + (KV8 ? kFusedMaxTiles * TILE : 0));   // selection counts
    __shared__ float red_m[8][H], red_l[8][H], red_v[8];
    __shared__ float2 lse_part[FCONS / H][H];
    __shared__ float lse_s[H];
    __shared__ uint32_t tmem_base;
    __shared__ volatile int s_abort;
    __shared__ int s_ok[4];

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, g = lane >> 2, t = lane & 3;
    const int group = blockIdx.x / a.splits, split = blockIdx.x % a.splits;
    const int nw = (a.B - group + wb - 1) / wb;                       // waves with a sequence for this group
    const int k_begin = split * a.chunk;
    int* cnt_ml = a.counter;                                          // [B]: splits done with pass A
    int* cnt_o = a.counter + a.B;                                     // [B]: splits done with pass B
    int* cnt_m = a.counter + 2 * a.B;                                 // [B]: rows of O merged

    if (warp == 0) umma::tmem_alloc(&tmem_base, 512);
    if (tid == 32) {
        prefetch_tmap(&kmap);
        prefetch_tmap(&vmap);
        for (int s = 0; s < FS; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 4);
        }
        fence_mbar_init();
        s_abort = 0;
    }
    for (int i = tid; i < kDecHistBins; i += FNT) hs[i] = 0;
    umma::fence_before();
    __syncthreads();
    umma::fence_after();
    const uint32_t tmem = tmem_base;

    auto tiles_of = [&](int w, int& k_end) {
        const int p = checked_pos(a.q_pos0[w * wb + group], a.max_ctx, a.status);
        k_end = min(p + 1, k_begin + a.chunk);
        return k_end > k_begin ? (k_end - k_begin + TILE - 1) / TILE : 0;
    };

    if (warp == 8) {
        // ---------------- producer: K tiles then V tiles of each wave, one TMA stream
        if (lane == 0) {
            uint32_t n_issued = 0;
            bool run = true;
            for (int w = 0; w < nw && run; ++w) {
                int k_end;
                const int n = tiles_of(w, k_end);
                const int row0 = static_cast<int>((w * wb + group) * a.cap) + k_begin;
                for (int j = 0; j < 2 * n; ++j) {
                    const uint32_t ld = n_issued;
                    const int s = ld % FS;
                    if (ld >= FS && !mbar_wait(&empty[s], ((ld / FS) & 1u) ^ 1u, a.status)) s_abort = 1;
                    if (s_abort) {
                        run = false;
                        break;
                    }
                    const bool is_v = j >= n;
                    const int row = row0 + (is_v ? j - n : j) * TILE;
                    const CUtensorMap* m = is_v ? &vmap : &kmap;
                    uint8_t* dst = smem + s * L::RAW;
                    mbar_arrive_expect_tx(&full[s], L::RAW);
                    tma_load_2d(dst, m, &full[s], 0, row);
                    if (!KV8) tma_load_2d(dst + TILE * 128, m, &full[s], 64, row);
                    ++n_issued;
                }
            }
            // after an abort, let the copies in flight land before the CTA exits (bounded)
            if (!run)
                for (uint32_t ld = n_issued > FS ? n_issued - FS : 0; ld < n_issued; ++ld)
                    mbar_wait(&full[ld % FS], (ld / FS) & 1u, nullptr, 100000000ull);
        }
        __syncwarp();
    } else {
        // ---------------- consumers: group c takes tiles c, c + 2, ...; q = warp quarter
        const int c = warp >> 2, q = warp & 3, gtid = tid & 127;
        auto take = [&](uint32_t ld) -> bool {    // warp-uniform; false once the CTA aborts
            if (__any_sync(0xffffffffu, s_abort != 0)) return false;
            const bool okw = __all_sync(0xffffffffu, mbar_wait(&full[ld % FS], (ld / FS) & 1u, a.status));
            if (!okw && lane == 0) s_abort = 1;
            return okw;
        };
        auto release = [&](uint32_t ld) {
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[ld % FS]);
        };
        // the selection state of this CTA's sequences is zeroed here, each split taking its share
        // of every one of them: a split adds to a sequence's histogram only after that
        // sequence's exchange, which every split reaches after this
        if (a.ghist) {
            for (int w = 0; w < nw; ++w) {
                const int b = w * wb + group;
                const int lo = split * kDecHistRow / a.splits, hi = (split + 1) * kDecHistRow / a.splits;
                for (int i = lo + tid; i < hi; i += FCONS) a.ghist[static_cast<size_t>(b) * kDecHistRow + i] = 0;
                if (split == 0 && tid < 4) a.gctl[4 * b + tid] = 0;
            }
            __threadfence();
        }
        uint32_t wbase = 0;                       // loads of the earlier waves
        for (int w = 0; w < nw; ++w) {
            const int b = w * wb + group;
            int k_end;
            const int n_tiles = tiles_of(w, k_end);
            const int c_end = checked_pos(a.q_pos0[b], a.max_ctx, nullptr) - a.window + 1;

            // ---- pass A: logits to tensor memory, running (max, sum) per head.  e4m3 keys:
            // f16 MMAs straight from the raw tile (Q in f16, k order permuted, scaled by
            // 1 / qscale); the largest V scale of the split is kept for pass B's f16 P
            uint32_t qa[8][4];
            float qscale = 1.f, vmax = 0.f;
            if (KV8) qscale = load_q_frags_e4m3(a.q + static_cast<size_t>(b) * H * D, g, t, qa);
            else load_q_frags(a.q + static_cast<size_t>(b) * H * D, g, t, qa);
            const float sc2 = a.sc2 * qscale;
            float m2[2] = {-INFINITY, -INFINITY}, l2[2] = {0.f, 0.f};
            const float* ksc = KV8 ? a.k_scale + b * a.cap : nullptr;
            const float* vsc = KV8 ? a.v_scale + b * a.cap : nullptr;
            // e4m3: lane l of a warp holds the key scale (l < 16) or the V scale (l >= 16) of
            // key l % 16 of its 16 keys of a tile, copied asynchronously into the warp's ring of
            // 8 slots (in the O-partial area, free during pass A) four of the group's tiles
            // ahead, so that the memory latency stays off the tile's path.  The V scales also
            // go to shared memory for pass B (the same warp reads them back).
            float* sc_ring = reinterpret_cast<float*>(red_o4) + warp * 8 * 32;
            auto issue_sc = [&](int i) {
                const int key = k_begin + i * TILE + q * 16 + (lane & 15);
                const bool valid = i < n_tiles && key < k_end;
                cp_async4_zfill(sc_ring + ((i >> 1) & 7) * 32 + lane, valid ? (lane < 16 ? ksc : vsc) + key : ksc,
                                valid);
                cp_async_commit();
            };
            if (KV8)
#pragma unroll
                for (int j = 0; j < 4; ++j) issue_sc(c + 2 * j);
            for (int i = c; i < n_tiles; i += 2) {
                const uint32_t ld = wbase + i;
                float sc_cur = 0.f;
                if (KV8) {
                    issue_sc(i + 8);
                    cp_async_wait<4>();
                    sc_cur = sc_ring[((i >> 1) & 7) * 32 + lane];
                    if (lane >= 16) {
                        vmax = fmaxf(vmax, sc_cur);
                        vsm[i * TILE + q * 16 + (lane & 15)] = sc_cur;
                    }
                }
                const bool okt = take(ld);
                const int tile_key0 = k_begin + i * TILE;
                const uint32_t tbase = smem_u32(smem + (ld % FS) * L::RAW);
                if (okt) {
                    float acc[2][4];
                    if (KV8) {
                        qk_e4m3(tbase, q * 16, qa, acc, lane);
                    } else {
#pragma unroll
                        for (int nt = 0; nt < 2; ++nt) {
#pragma unroll
                            for (int e = 0; e < 4; ++e) acc[nt][e] = 0.f;
                            const int r = q * 16 + nt * 8 + (lane & 7);
#pragma unroll
                            for (int kk = 0; kk < 4; ++kk) {
                                uint32_t b0, b1, b2, b3;
                                ldsm_x4(tbase + swz_off<TILE>(r, 4 * kk + (lane >> 3)), b0, b1, b2, b3);
                                mma_bf16(acc[nt], qa[2 * kk], b0, b1);
                                mma_bf16(acc[nt], qa[2 * kk + 1], b2, b3);
                            }
                        }
                    }
                    const int key0 = tile_key0 + q * 16 + 2 * t;
                    float mx[2] = {-INFINITY, -INFINITY};
                    uint32_t sv[8];
#pragma unroll
                    for (int nt = 0; nt < 2; ++nt) {
                        const int key = key0 + nt * 8;
                        float f0 = sc2, f1 = sc2;
                        if (KV8) {
                            f0 *= __shfl_sync(0xffffffffu, sc_cur, nt * 8 + 2 * t);
                            f1 *= __shfl_sync(0xffffffffu, sc_cur, nt * 8 + 2 * t + 1);
                        }
                        acc[nt][0] = (key < k_end) ? acc[nt][0] * f0 : -INFINITY;
                        acc[nt][1] = (key + 1 < k_end) ? acc[nt][1] * f1 : -INFINITY;
                        acc[nt][2] = (key < k_end) ? acc[nt][2] * f0 : -INFINITY;
                        acc[nt][3] = (key + 1 < k_end) ? acc[nt][3] * f1 : -INFINITY;
#pragma unroll
                        for (int e = 0; e < 4; ++e) sv[4 * nt + e] = __float_as_uint(acc[nt][e]);
                        mx[0] = fmaxf(mx[0], fmaxf(acc[nt][0], acc[nt][1]));
                        mx[1] = fmaxf(mx[1], fmaxf(acc[nt][2], acc[nt][3]));
                    }
                    umma::tmem_st16x256_x2(
                        tmem + (static_cast<uint32_t>(32 * q + 16 * (i >> 5)) << 16) + 16 * (i & 31), sv);
#pragma unroll
                    for (int hh = 0; hh < 2; ++hh) {
                        const float mn = fmaxf(m2[hh], mx[hh]);
                        if (mn != -INFINITY) {
                            float sum = l2[hh] * ex2(m2[hh] - mn);
#pragma unroll
                            for (int nt = 0; nt < 2; ++nt)
                                sum += ex2(acc[nt][2 * hh] - mn) + ex2(acc[nt][2 * hh + 1] - mn);
                            l2[hh] = sum;
                            m2[hh] = mn;
                        }
                    }
                }
                release(ld);
            }
            umma::tmem_st_wait();
            if (KV8) asm volatile("cp.async.wait_all;" ::: "memory");   // the ring is O-partial space again
            // ---- exchange: publish this split's (max, sum), wait for the other splits
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
#pragma unroll
                for (int off = 1; off <= 2; off <<= 1) {
                    const float om = __shfl_xor_sync(0xffffffffu, m2[hh], off);
                    const float ol = __shfl_xor_sync(0xffffffffu, l2[hh], off);
                    merge_ml(m2[hh], l2[hh], om, ol);
                }
            }
            if (t == 0) {
                red_m[warp][g] = m2[0]; red_l[warp][g] = l2[0];
                red_m[warp][g + 8] = m2[1]; red_l[warp][g + 8] = l2[1];
            }
            if (KV8) {
#pragma unroll
                for (int off = 1; off < 32; off <<= 1) vmax = fmaxf(vmax, __shfl_xor_sync(0xffffffffu, vmax, off));
                if (lane == 0) red_v[warp] = vmax;
            }
            bar_sync(3, FCONS);
            // e4m3 values: P V in f16 with P * v_scale * 2^pe, the largest product of the split
            // (at most its largest V scale, P <= 1) scaled to 2^14 or below; O is scaled back
            float pscale = 1.f, pinv = 1.f;
            if (KV8) {
                float vm = red_v[0];
#pragma unroll
                for (int k = 1; k < 8; ++k) vm = fmaxf(vm, red_v[k]);
                int ex = 0;
                if (vm > 0.f) frexpf(vm, &ex);      // vm < 2^ex
                pscale = ldexpf(1.f, 14 - ex);
                pinv = ldexpf(1.f, ex - 14);
            }
            if (tid < H) {
                float m = red_m[0][tid], l = red_l[0][tid];
                for (int k = 1; k < 8; ++k) merge_ml(m, l, red_m[k][tid], red_l[k][tid]);
                a.part_ml[(static_cast<size_t>(b) * a.splits + split) * H + tid] = make_float2(m, l);
                __threadfence();
            }
            bar_sync(3, FCONS);
            if (tid == 0) {
                bool arrived = false;
                if (!s_abort) {
                    atomicAdd(&cnt_ml[b], 1);
                    arrived = wait_count(&cnt_ml[b], a.splits, a.status);
                    __threadfence();
                }
                if (!arrived) s_abort = 1;
            }
            bar_sync(3, FCONS);
            {
                const int h = tid & (H - 1), grp = tid >> 4;
                float m = -INFINITY, l = 0.f;
                const float2* pml = a.part_ml + static_cast<size_t>(b) * a.splits * H;
                if (!s_abort)
                    for (int s = grp; s < a.splits; s += FCONS / H) {
                        const float2 ml = __ldcg(pml + s * H + h);
                        merge_ml(m, l, ml.x, ml.y);
                    }
                lse_part[grp][h] = make_float2(m, l);
                bar_sync(3, FCONS);
                if (tid < H) {
                    float mm = -INFINITY, ll = 0.f;
                    for (int k = 0; k < FCONS / H; ++k) merge_ml(mm, ll, lse_part[k][tid].x, lse_part[k][tid].y);
                    lse_s[tid] = mm + log2f(ll);
                    if (split == 0 && a.lse && !s_abort) a.lse[static_cast<size_t>(b) * H + tid] = lse_s[tid] * kLn2;
                }
                bar_sync(3, FCONS);
            }
            const float lse2[2] = {lse_s[g], lse_s[g + 8]};

            // ---- pass B: P from the logits in tensor memory, importance, O = P V
            float o[16][4];
#pragma unroll
            for (int n = 0; n < 16; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;
            float* score_row = a.scores + b * a.score_ld;
            for (int i = c; i < n_tiles; i += 2) {
                const uint32_t ld = wbase + n_tiles + i;
                uint32_t sr[8];
                umma::tmem_ld16x256_x2(tmem + (static_cast<uint32_t>(32 * q + 16 * (i >> 5)) << 16) + 16 * (i & 31),
                                       sr);
                const int tile_key0 = k_begin + i * TILE;
                const int kl = tile_key0 + q * 16 + 2 * t, kh = kl + 8;
                const bool v0 = kl < k_end, v1 = kl + 1 < k_end, v2 = kh < k_end, v3 = kh + 1 < k_end;
                float f0 = 1.f, f1 = 1.f, f2 = 1.f, f3 = 1.f;
                if (KV8) {                        // V scales kept by pass A (zero past the end)
                    const float* vs = vsm + (kl - k_begin);
                    f0 = vs[0] * pscale; f1 = vs[1] * pscale; f2 = vs[8] * pscale; f3 = vs[9] * pscale;
                }
                const bool okt = take(ld);
                uint8_t* vt = smem + (ld % FS) * L::RAW;
                if (tile_key0 + TILE > k_end) {
                    // tail tile: zero the V rows past the last key (cache rows there may hold
                    // anything, and 0 * NaN would poison O); the stage is refilled by TMA later,
                    // so order these writes before the async proxy
                    if (okt) {
                        if (KV8) {
                            for (int it = gtid; it < TILE * 8; it += 128) {
                                const int r = it >> 3, cc = it & 7;
                                if (tile_key0 + r >= k_end)
                                    *reinterpret_cast<uint4*>(vt + r * 128 + cc * 16) = make_uint4(0, 0, 0, 0);
                            }
                        } else {
                            for (int it = gtid; it < TILE * 16; it += 128) {
                                const int r = it >> 4, cc = it & 15;
                                if (tile_key0 + r >= k_end)
                                    *reinterpret_cast<uint4*>(vt + swz_off<TILE>(r, cc)) = make_uint4(0, 0, 0, 0);
                            }
                        }
                    }
                    umma::fence_proxy_async();
                    bar_sync(1 + c, 128);
                }
                umma::tmem_ld_wait();
                if (okt) {
                    const float2 sgl = make_float2(__uint_as_float(sr[0]), __uint_as_float(sr[1]));
                    const float2 sg8l = make_float2(__uint_as_float(sr[2]), __uint_as_float(sr[3]));
                    const float2 sgh = make_float2(__uint_as_float(sr[4]), __uint_as_float(sr[5]));
                    const float2 sg8h = make_float2(__uint_as_float(sr[6]), __uint_as_float(sr[7]));
                    const float p00 = v0 ? ex2(sgl.x - lse2[0]) : 0.f, p01 = v1 ? ex2(sgl.y - lse2[0]) : 0.f;
                    const float p10 = v0 ? ex2(sg8l.x - lse2[1]) : 0.f, p11 = v1 ? ex2(sg8l.y - lse2[1]) : 0.f;
                    const float p02 = v2 ? ex2(sgh.x - lse2[0]) : 0.f, p03 = v3 ? ex2(sgh.y - lse2[0]) : 0.f;
                    const float p12 = v2 ? ex2(sg8h.x - lse2[1]) : 0.f, p13 = v3 ? ex2(sg8h.y - lse2[1]) : 0.f;
                    float sc[4] = {p00 + p10, p01 + p11, p02 + p12, p03 + p13};
#pragma unroll
                    for (int off = 4; off <= 16; off <<= 1)
#pragma unroll
                        for (int e = 0; e < 4; ++e) sc[e] += __shfl_xor_sync(0xffffffffu, sc[e], off);
                    if (g == 0) {
                        if (v0) score_row[kl] = sc[0];
                        if (v1) score_row[kl + 1] = sc[1];
                        if (v2) score_row[kh] = sc[2];
                        if (v3) score_row[kh + 1] = sc[3];
                    }
                    const uint32_t vbase = smem_u32(vt);
                    uint32_t pa[4];
                    if (KV8) {
                        pa[0] = pack_f16(p00 * f0, p01 * f1);
                        pa[1] = pack_f16(p10 * f0, p11 * f1);
                        pa[2] = pack_f16(p02 * f2, p03 * f3);
                        pa[3] = pack_f16(p12 * f2, p13 * f3);
                        pv_e4m3(vbase, q * 16, pa, o, lane);
                    } else {
                        pa[0] = pack_bf16(p00, p01);
                        pa[1] = pack_bf16(p10, p11);
                        pa[2] = pack_bf16(p02, p03);
                        pa[3] = pack_bf16(p12, p13);
                        const int vr = q * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
#pragma unroll
                        for (int cv = 0; cv < 8; ++cv) {
                            uint32_t b0, b1, b2, b3;
                            ldsm_x4_t(vbase + swz_off<TILE>(vr, 2 * cv + (lane >> 4)), b0, b1, b2, b3);
                            mma_bf16(o[2 * cv], pa, b0, b1);
                            mma_bf16(o[2 * cv + 1], pa, b2, b3);
                        }
                    }
                    // selection counts, after the MMAs so that they stay off the tile's path
                    if (a.ghist && g == 0) count_candidates(hs, sc, {kl, kl + 1, kh, kh + 1}, {v0, v1, v2, v3}, c_end);
                }
                release(ld);
            }

            // ---- this split's O partial: the 8 warps' accumulators go to shared memory as
            // [warp][n][lane] float4 (conflict-free), then each (n, lane) slot is summed over the
            // warps in a fixed order; the partials are merged at the end.  e4m3: accumulator n
            // holds dims 32 (n / 4) + 16 ((n / 2) % 2) + 4 t + n % 2 and that + 2 (see pv_e4m3),
            // scaled by pscale
#pragma unroll
            for (int n = 0; n < 16; ++n)
                red_o4[(warp * 16 + n) * 32 + lane] =
                    make_float4(o[n][0] * pinv, o[n][1] * pinv, o[n][2] * pinv, o[n][3] * pinv);
            bar_sync(3, FCONS);
            float* my = a.part_o + (static_cast<size_t>(b) * a.splits + split) * H * D;
#pragma unroll
            for (int k = 0; k < 512 / FCONS; ++k) {
                const int e = tid + k * FCONS, n = e >> 5, ln = e & 31;
                float4 sum = red_o4[e];
#pragma unroll
                for (int w8 = 1; w8 < 8; ++w8) {
                    const float4 v = red_o4[w8 * 512 + e];
                    sum.x += v.x; sum.y += v.y; sum.z += v.z; sum.w += v.w;
                }
                const int h = ln >> 2, tq = ln & 3;
                if (KV8) {
                    const int d = 32 * (n >> 2) + 16 * ((n >> 1) & 1) + 4 * tq + (n & 1);
                    my[h * D + d] = sum.x;
                    my[h * D + d + 2] = sum.y;
                    my[(h + 8) * D + d] = sum.z;
                    my[(h + 8) * D + d + 2] = sum.w;
                } else {
                    const int d = 8 * n + 2 * tq;
                    *reinterpret_cast<float2*>(my + h * D + d) = make_float2(sum.x, sum.y);
                    *reinterpret_cast<float2*>(my + (h + 8) * D + d) = make_float2(sum.z, sum.w);
                }
            }
            bar_sync(3, FCONS);
            if (a.ghist) flush_hist(a, hs, b, tid, FCONS);   // the next wave's counts start after its exchange
            if (tid == 0 && !s_abort) {
                __threadfence();                  // the CTA's partial, ordered by the barrier
                atomicAdd(&cnt_o[b], 1);
            }
            wbase += 2 * n_tiles;
        }

        // ---- O = sum of the split partials, spread over all CTAs: rows (sequence, head) in
        // sequence order, four per pass (64 threads each: 32 float4 columns x 2 split lanes)
        const int k4 = tid >> 6, c4 = tid & 31, sl = (tid >> 5) & 1;
        for (int base = blockIdx.x; base < a.B * H; base += 4 * gridDim.x) {
            const int item = base + k4 * gridDim.x;
            const bool have = item < a.B * H;
            const int b = have ? item / H : 0, h = item % H;
            bar_sync(3, FCONS);               // s_ok and red_o4 of the previous pass are free
            if ((tid & 63) == 0) s_ok[k4] = (have && !s_abort) ? wait_count(&cnt_o[b], a.splits, a.status) : 0;
            bar_sync(3, FCONS);
            const bool go = have && s_ok[k4] != 0;
            if (have && !go) s_abort = 1;
            float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
            if (go) {
                const float4* src =
                    reinterpret_cast<const float4*>(a.part_o + static_cast<size_t>(b) * a.splits * H * D + h * D) + c4;
#pragma unroll 4
                for (int sp = sl; sp < a.splits; sp += 2) {
                    const float4 v = __ldcg(src + static_cast<size_t>(sp) * (H * D / 4));
                    acc.x += v.x; acc.y += v.y; acc.z += v.z; acc.w += v.w;
                }
            }
            if (sl == 1) red_o4[k4 * 32 + c4] = acc;
            bar_sync(3, FCONS);
            if (go && sl == 0) {
                const float4 v = red_o4[k4 * 32 + c4];
                uint2 packed;
                packed.x = pack_bf16(acc.x + v.x, acc.y + v.y);
                packed.y = pack_bf16(acc.z + v.z, acc.w + v.w);
                *reinterpret_cast<uint2*>(a.o + (static_cast<size_t>(b) * H + h) * D + 4 * c4) = packed;
                // the last of the 16 rows of b returns the sequence's counters to zero (every
                // row's CTA has passed its wait on cnt_o by then)
                if (c4 == 0 && atomicAdd(&cnt_m[b], 1) == H - 1) {
                    cnt_ml[b] = 0;
                    cnt_o[b] = 0;
                    cnt_m[b] = 0;
                }
            }
        }
    }
    umma::fence_before();
    __syncthreads();
    umma::fence_after();
    if (warp == 0) umma::tmem_dealloc(tmem, 512);
}

template <bool KV8>
size_t smem_a() { return 1024 + STAGES * Layout<KV8>::RAW + STAGES * 8; }
template <bool KV8>
size_t smem_b() {
    static_assert(STAGES * (Layout<KV8>::RAW + Layout<KV8>::STILE) >= 4 * H * D * 4, "O partials reuse the stages");
    return 1024 + STAGES * (Layout<KV8>::RAW + Layout<KV8>::STILE) + STAGES * 8;
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

template <bool KV8>
cudaError_t launch_impl(const DecodeArgs& da, cudaStream_t st) {
    const DecodePlan pl = plan_decode(da.batch, da.max_ctx, KV8);
    Params a{};
    a.B = da.batch; a.cap = da.cap; a.max_ctx = da.max_ctx; a.splits = pl.splits; a.chunk = pl.chunk; a.s_ld = pl.s_ld;
    a.q_pos0 = da.q_pos0;
    a.q = static_cast<const __nv_bfloat16*>(da.q);
    a.k_scale = da.k_scale; a.v_scale = da.v_scale;
    a.sc2 = da.scale * kLog2e;
    uint8_t* ws = static_cast<uint8_t*>(da.ws);
    a.S = pl.fused ? nullptr : reinterpret_cast<float*>(ws);
    ws += align256(sizeof(float) * da.batch * H * static_cast<size_t>(pl.s_ld));
    a.part_ml = reinterpret_cast<float2*>(ws);
    ws += align256(sizeof(float2) * da.batch * pl.splits * H);
    a.part_o = reinterpret_cast<float*>(ws);
    ws += align256(sizeof(float) * da.batch * pl.splits * H * D);
    a.part_vmax = reinterpret_cast<float*>(ws);                      // two-kernel path, e4m3
    // fused path: three [B] counters in the status block (zero when idle)
    a.counter = reinterpret_cast<int*>(da.status) + kCounterOffsetInts;
    a.o = static_cast<__nv_bfloat16*>(da.o);
    a.lse = da.lse;
    a.scores = da.scores; a.score_ld = da.score_ld;
    a.status = da.status;
    a.window = da.window;
    a.ghist = da.sel.hist;
    a.gctl = da.sel.ctl;

    CUtensorMap kmap, vmap, smap;
    const uint64_t rows = static_cast<uint64_t>(da.batch) * da.cap;
    const int eb = KV8 ? 1 : 2;
    const CUtensorMapDataType dt = KV8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    const uint32_t box_cols = KV8 ? 128 : 64;
    if (!make_tmap_2d(&kmap, da.k, dt, eb, D, rows, D * eb, box_cols, TILE, true)) return cudaErrorInvalidValue;
    if (!make_tmap_2d(&vmap, da.v, dt, eb, D, rows, D * eb, box_cols, TILE, true)) return cudaErrorInvalidValue;
    if (pl.fused) {
        size_t sm = FusedLayout<KV8>::BYTES;
        if (sm < kFusedMinSmem) sm = kFusedMinSmem;
        cudaError_t e = cudaFuncSetAttribute(dec_fused_kernel<KV8>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             static_cast<int>(sm));
        if (e != cudaSuccess) return e;
        cudaLaunchConfig_t cfg{};
        cfg.gridDim = dim3(pl.wb * pl.splits);
        cfg.blockDim = dim3(FNT);
        cfg.dynamicSmemBytes = sm;
        cfg.stream = st;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeCooperative;     // all CTAs resident: the splits wait on one another
        attr[0].val.cooperative = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        return cudaLaunchKernelEx(&cfg, dec_fused_kernel<KV8>, kmap, vmap, a, pl.wb);
    }
    if (!make_tmap_2d(&smap, a.S, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, pl.s_ld,
                      static_cast<uint64_t>(da.batch) * H, static_cast<uint64_t>(pl.s_ld) * 4, 32, 16, true))
        return cudaErrorInvalidValue;

    const dim3 grid(pl.splits, da.batch);
    const size_t sa = smem_a<KV8>(), sb = smem_b<KV8>();
    cudaError_t e = cudaFuncSetAttribute(dec_qk_kernel<KV8>, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(sa));
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(dec_pv_kernel<KV8>, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(sb));
    if (e != cudaSuccess) return e;
    dec_qk_kernel<KV8><<<grid, NT, sa, st>>>(kmap, a);
    dec_pv_kernel<KV8><<<grid, NT, sb, st>>>(vmap, smap, a);
    dec_merge_kernel<<<da.batch * H * kMergeGroups, NT, 0, st>>>(a);
    return cudaGetLastError();
}

}  // namespace

DecodePlan plan_decode(int batch, int64_t max_ctx, bool kv8) {
    DecodePlan pl;
    // fused: enough splits that each fits tensor memory, as many sequences per wave as
    // the SMs allow, waves balanced, then as many splits as the SMs allow
    const int sms = num_sms();
    const int64_t cap_keys = static_cast<int64_t>(kFusedMaxTiles) * TILE;
    const int64_t min_splits = (max_ctx + cap_keys - 1) / cap_keys;
    if (batch >= 1 && min_splits <= sms && 3 * batch <= kMaxCounters) {
        int wb = static_cast<int>(sms / min_splits);
        if (wb > batch) wb = batch;
        const int waves = (batch + wb - 1) / wb;
        {
            wb = (batch + waves - 1) / waves;
            int64_t chunk = (max_ctx + sms / wb - 1) / (sms / wb);
            chunk = (chunk + TILE - 1) / TILE * TILE;
            pl.fused = true;
            pl.wb = wb;
            pl.chunk = static_cast<int>(chunk);
            pl.splits = static_cast<int>((max_ctx + chunk - 1) / chunk);
            pl.s_ld = 0;
            return pl;
        }
    }
    pl.fused = false;
    pl.wb = 0;
    // two-kernel path: two CTAs per SM suffice to stream a bf16 cache; e4m3 tiles are
    // decoded in registers with per-key scales, which takes four
    int splits = ((kv8 ? 4 : 2) * num_sms()) / (batch > 0 ? batch : 1);
    if (splits < 1) splits = 1;
    int64_t chunk = (max_ctx + splits - 1) / splits;
    chunk = (chunk + TILE - 1) / TILE * TILE;
    if (chunk < TILE) chunk = TILE;
    pl.chunk = static_cast<int>(chunk);
    pl.splits = static_cast<int>((max_ctx + chunk - 1) / chunk);
    if (pl.splits < 1) pl.splits = 1;
    pl.s_ld = static_cast<int>((max_ctx + TILE - 1) / TILE * TILE);
    return pl;
}

size_t decode_ws_bytes(int batch, int64_t max_ctx, bool kv8) {
    const DecodePlan pl = plan_decode(batch, max_ctx, kv8);
    return align256(sizeof(float) * batch * H * static_cast<size_t>(pl.s_ld)) +
           align256(sizeof(float2) * batch * pl.splits * H) +
           align256(sizeof(float) * batch * pl.splits * H * D) + align256(sizeof(float) * batch * pl.splits);
}

cudaError_t launch_decode_full(const DecodeArgs& a, cudaStream_t st) {
    return a.kv8 ? launch_impl<true>(a, st) : launch_impl<false>(a, st);
}

}  // namespace hs2
