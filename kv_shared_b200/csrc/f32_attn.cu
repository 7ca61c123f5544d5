// f32_attn.cu -- fp32 CUDA-core path of the hybrid block (full attention with
// importance, and sparse attention), for fp32 caches.
//
// Used where the inputs are fp32: rounding Q or K to bf16/tf32 for the tensor
// cores would move each importance value by ~1e-4 relative, far more than the
// tie band the selection is checked with.  One warp per query row; all heads of
// the row are handled by that warp so the head sum of the importance is formed
// in registers.  Two passes over the keys: log-sum-exp per head, then exactly
// normalized probabilities, importance and O.  The same structure serves the
// sparse layer over the selected positions.
#include "common.cuh"
#include "internal.h"

namespace hs2 {
namespace {

constexpr int WARPS = 4;
constexpr int HMAX = 16;

template <int D>
struct RowSmem {
    float q[HMAX][D];
    float P[32][HMAX + 1];
};

// dot products of key row kr (D floats) with every head's (pre-scaled) query
template <int D>
__device__ __forceinline__ void dots(const float* __restrict__ kr, const float (*q)[D], int H, float* s) {
#pragma unroll
    for (int h = 0; h < HMAX; ++h) s[h] = 0.f;
#pragma unroll 4
    for (int i = 0; i < D / 4; ++i) {
        const float4 kv = __ldg(reinterpret_cast<const float4*>(kr) + i);
#pragma unroll
        for (int h = 0; h < HMAX; ++h) {
            if (h >= H) break;
            const float4 qq = *reinterpret_cast<const float4*>(&q[h][4 * i]);
            s[h] = fmaf(qq.x, kv.x, s[h]);
            s[h] = fmaf(qq.y, kv.y, s[h]);
            s[h] = fmaf(qq.z, kv.z, s[h]);
            s[h] = fmaf(qq.w, kv.w, s[h]);
        }
    }
}

// SPARSE=false: keys 0..p;  SPARSE=true: keys idx[0..cnt)
template <int D, bool SPARSE>
__global__ void __launch_bounds__(WARPS * 32) f32_kernel(F32Args a) {
    __shared__ RowSmem<D> sm[WARPS];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int row = blockIdx.x * WARPS + warp;
    const int rows = a.batch * a.n_q;
    if (row >= rows) return;
    const int b = row / a.n_q, r = row % a.n_q;
    const int H = a.heads;
    RowSmem<D>& S = sm[warp];
    const float* qrow = a.q + static_cast<size_t>(row) * H * D;
    for (int i = lane; i < H * D; i += 32) S.q[i / D][i % D] = qrow[i] * a.scale;
    __syncwarp();

    const float* kb = a.k + static_cast<size_t>(b) * a.cap * D;
    const float* vb = a.v + static_cast<size_t>(b) * a.cap * D;
    int n;
    const int32_t* ids = nullptr;
    if (SPARSE) {
        n = a.cnt[row];
        if (n < 0 || n > a.idx_stride) {
            if (lane == 0) set_status(a.status, HS2_ERR_INDEX);
            n = n < 0 ? 0 : a.idx_stride;
        }
        ids = a.idx + static_cast<size_t>(row) * a.idx_stride;
    } else {
        n = checked_pos(a.q_pos0[b] + r, a.max_ctx, a.status) + 1;
    }
    auto key_of = [&](int e) -> int {
        if (!SPARSE) return e;
        int j = ids[e];
        if (j < 0 || j >= a.cap) { set_status(a.status, HS2_ERR_INDEX); j = -1; }
        return j;
    };

    // pass 1: per-head max and sum of exp
    float m[HMAX], l[HMAX], s[HMAX];
#pragma unroll
    for (int h = 0; h < HMAX; ++h) { m[h] = -INFINITY; l[h] = 0.f; }
    for (int e = lane; e < n; e += 32) {
        const int j = key_of(e);
        if (j < 0) continue;
        dots<D>(kb + static_cast<size_t>(j) * D, S.q, H, s);
#pragma unroll
        for (int h = 0; h < HMAX; ++h) {
            if (h >= H) break;
            if (s[h] > m[h]) { l[h] = l[h] * expf(m[h] - s[h]) + 1.f; m[h] = s[h]; }
            else l[h] += expf(s[h] - m[h]);
        }
    }
    float lse[HMAX];
#pragma unroll
    for (int h = 0; h < HMAX; ++h) {
        if (h >= H) break;
        const float M = warp_max(m[h]);
        const float part = (m[h] == -INFINITY) ? 0.f : l[h] * expf(m[h] - M);
        const float Lh = warp_sum(part);
        lse[h] = M + logf(Lh);
    }

    // pass 2: P, importance, O
    constexpr int DV = D / 32;
    float o[HMAX][DV];
#pragma unroll
    for (int h = 0; h < HMAX; ++h)
#pragma unroll
        for (int i = 0; i < DV; ++i) o[h][i] = 0.f;
    float* srow = SPARSE ? nullptr : a.scores + static_cast<size_t>(row) * a.score_ld;
    for (int e0 = 0; e0 < n; e0 += 32) {
        const int e = e0 + lane;
        int j = -1;
        if (e < n) {
            j = key_of(e);
            if (j >= 0) {
                dots<D>(kb + static_cast<size_t>(j) * D, S.q, H, s);
                float tot = 0.f;
#pragma unroll
                for (int h = 0; h < HMAX; ++h) {
                    if (h >= H) break;
                    const float P = expf(s[h] - lse[h]);
                    S.P[lane][h] = P;
                    tot += P;
                }
                if (!SPARSE) srow[j] = tot;
            }
        }
        if (j < 0)
            for (int h = 0; h < H; ++h) S.P[lane][h] = 0.f;
        __syncwarp();
        const int m_e = min(32, n - e0);
        for (int u = 0; u < m_e; ++u) {
            const int jj = __shfl_sync(0xffffffffu, j, u);
            if (jj < 0) continue;
            const float* vr = vb + static_cast<size_t>(jj) * D;
            float vv[DV];
#pragma unroll
            for (int i = 0; i < DV; ++i) vv[i] = __ldg(vr + lane + 32 * i);
#pragma unroll
            for (int h = 0; h < HMAX; ++h) {
                if (h >= H) break;
                const float P = S.P[u][h];
#pragma unroll
                for (int i = 0; i < DV; ++i) o[h][i] = fmaf(P, vv[i], o[h][i]);
            }
        }
        __syncwarp();
    }
    float* orow = a.o + static_cast<size_t>(row) * H * D;
#pragma unroll
    for (int h = 0; h < HMAX; ++h) {
        if (h >= H) break;
#pragma unroll
        for (int i = 0; i < DV; ++i) orow[h * D + lane + 32 * i] = o[h][i];
    }
    if (a.lse && lane < H) {
        float v = lse[0];
#pragma unroll
        for (int h = 1; h < HMAX; ++h) if (h == lane) v = lse[h];
        a.lse[static_cast<size_t>(row) * H + lane] = v;
    }
}

template <bool SPARSE>
cudaError_t launch(const F32Args& a, cudaStream_t st) {
    const int rows = a.batch * a.n_q;
    if (rows <= 0) return cudaSuccess;
    const dim3 grid((rows + WARPS - 1) / WARPS);
    if (a.head_dim == 64) f32_kernel<64, SPARSE><<<grid, WARPS * 32, 0, st>>>(a);
    else f32_kernel<128, SPARSE><<<grid, WARPS * 32, 0, st>>>(a);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_f32_full(const F32Args& a, cudaStream_t st) { return launch<false>(a, st); }
cudaError_t launch_f32_sparse(const F32Args& a, cudaStream_t st) { return launch<true>(a, st); }

}  // namespace hs2
