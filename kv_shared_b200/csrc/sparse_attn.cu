// sparse_attn.cu -- sparse-attention layer of a hybrid block (KV Reuse).
//
// "What HySparse2 is actually optimizing", section 2: a sparse layer keeps no
// cache or selector of its own and reads the full layer's cache at the full
// layer's chosen positions; section 3: window and global positions sit in one
// cache, so a single softmax covers the whole chosen set.
//
// For each query row (16 heads) the selected cache rows are gathered by index
// with 16-byte cp.async copies into shared memory (swizzled so ldmatrix reads
// are conflict-free), all 16 heads are computed against each gathered row once
// (mma.sync m16n8k16, M = the 16 heads), and the softmax stays online in
// registers.  A row's selected set is split across CTAs when there are few rows
// (decode); split partials (max, sum, O) are merged by the last CTA of the row
// (semaphore counter, no spin).  e4m3 rows are converted to bf16 in shared
// memory (exact) and their per-token scales folded into the logits and into P.
#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace hs2 {
namespace {

constexpr int H = 16;
constexpr int D = 128;
constexpr int SUB = 64;            // gathered rows per pipeline stage
constexpr int NT = 128;            // 4 warps x 16 rows
constexpr int kMaxSplits = 32;     // bound of the split count (shared-memory merge tables)

struct Params {
    int rows, n_q, idx_stride, splits, chunk;
    int64_t cap;
    const __nv_bfloat16* q;
    const uint8_t* k;
    const uint8_t* v;
    const float* k_scale;
    const float* v_scale;
    const int32_t* idx;
    const int32_t* cnt;
    float sc2;
    float2* part_ml;               // [rows][splits][H]
    float* part_o;                 // [rows][splits][H][D]
    int* counter;                  // [rows]
    __nv_bfloat16* o;
    float* lse;
    uint32_t* status;
};

template <bool KV8>
struct Layout {
    static constexpr int ROWB = KV8 ? 128 : 256;      // bytes per gathered cache row
    static constexpr int STAGE = 2 * SUB * ROWB;       // K rows then V rows
    static constexpr int CVT = KV8 ? 2 * SUB * 256 : 0;
};

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
    return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

__device__ __forceinline__ void merge_ml(float& m, float& l, float m2, float l2) {
    const float mn = fmaxf(m, m2);
    if (mn == -INFINITY) return;
    l = l * ex2(m - mn) + l2 * ex2(m2 - mn);
    m = mn;
}

template <bool KV8>
__global__ void __launch_bounds__(NT) sparse_kernel(Params a) {
    using L = Layout<KV8>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = align1024(smem_raw);
    uint8_t* cvt = smem + 2 * L::STAGE;                    // e4m3 only: K bf16 then V bf16
    float* red_o = reinterpret_cast<float*>(cvt + L::CVT); // [H][D]
    int* sidx = reinterpret_cast<int*>(red_o + H * D);     // [chunk] cache row per entry (-1 invalid)
    float* sks = reinterpret_cast<float*>(sidx + a.chunk); // [chunk] k scales (e4m3)
    float* svs = sks + a.chunk;                            // [chunk] v scales (e4m3)
    __shared__ float wm[4][H], wl[4][H];
    __shared__ int s_last;

    const int row = blockIdx.y, split = blockIdx.x;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, g = lane >> 2, t = lane & 3;
    const int b = row / a.n_q;
    int c = a.cnt[row];
    if (c < 0 || c > a.idx_stride) {                       // a count the index row cannot hold
        if (tid == 0) set_status(a.status, HS2_ERR_INDEX);
        c = c < 0 ? 0 : a.idx_stride;
    }
    const int e_begin = split * a.chunk;
    const int e_end = min(c, e_begin + a.chunk);
    const int n_sub = e_end > e_begin ? (e_end - e_begin + SUB - 1) / SUB : 0;
    const int32_t* irow = a.idx + static_cast<size_t>(row) * a.idx_stride;
    const size_t seq_base = static_cast<size_t>(b) * a.cap;

    // every index (and scale) of this CTA's entries, loaded once up front
    for (int e = tid; e < a.chunk; e += NT) {
        int j = -1;
        if (e_begin + e < e_end) {
            j = irow[e_begin + e];
            if (j < 0 || j >= a.cap) { set_status(a.status, HS2_ERR_INDEX); j = -1; }
        }
        sidx[e] = j;
        if (KV8) {
            sks[e] = j >= 0 ? a.k_scale[seq_base + j] : 0.f;
            svs[e] = j >= 0 ? a.v_scale[seq_base + j] : 0.f;
        }
    }
    __syncthreads();

    // gather sub-tile i into stage s (cp.async, zero-filled past the end)
    auto gather = [&](int i, int s) {
        uint8_t* st = smem + s * L::STAGE;
        const int* si = sidx + i * SUB;
        constexpr int CH = L::ROWB / 16;                   // 16-byte chunks per row
        for (int it = tid; it < SUB * CH; it += NT) {
            const int r = it / CH, ch = it % CH;
            const int j = si[r];
            const size_t off = (seq_base + (j >= 0 ? j : 0)) * L::ROWB + ch * 16;
            uint32_t dk, dv;
            if (KV8) {
                dk = r * 128 + ((ch ^ (r & 7)) << 4);
                dv = SUB * 128 + dk;
            } else {
                dk = swz_off<SUB>(r, ch);
                dv = SUB * 256 + dk;
            }
            cp_async16_zfill(st + dk, a.k + off, j >= 0);
            cp_async16_zfill(st + dv, a.v + off, j >= 0);
        }
        cp_async_commit();
    };

    uint32_t qa[8][4];
    {
        const uint32_t* q32 = reinterpret_cast<const uint32_t*>(a.q + static_cast<size_t>(row) * H * D);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
            qa[ks][0] = __ldg(q32 + (g * D + 16 * ks + 2 * t) / 2);
            qa[ks][1] = __ldg(q32 + ((g + 8) * D + 16 * ks + 2 * t) / 2);
            qa[ks][2] = __ldg(q32 + (g * D + 16 * ks + 2 * t + 8) / 2);
            qa[ks][3] = __ldg(q32 + ((g + 8) * D + 16 * ks + 2 * t + 8) / 2);
        }
    }

    if (n_sub > 0) gather(0, 0);
    if (n_sub > 1) gather(1, 1);

    float m2[2] = {-INFINITY, -INFINITY}, l2[2] = {0.f, 0.f};
    float o[16][4];
#pragma unroll
    for (int n = 0; n < 16; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;

    for (int i = 0; i < n_sub; ++i) {
        const int s = i & 1;
        if (i + 1 < n_sub) cp_async_wait<1>(); else cp_async_wait<0>();
        __syncthreads();
        uint8_t* st = smem + s * L::STAGE;
        const uint8_t* kt = st;
        const uint8_t* vt = st + SUB * L::ROWB;
        if (KV8) {
            // e4m3 rows (128-byte swizzle) -> bf16 tiles (swz_off layout), exact
            for (int it = tid; it < 2 * SUB * 8; it += NT) {
                const int half = it / (SUB * 8), rr = (it / 8) % SUB, c8 = it & 7;
                const uint8_t* src = st + half * SUB * 128 + rr * 128 + ((c8 ^ (rr & 7)) << 4);
                uint8_t* dst = cvt + half * SUB * 256;
                const uint4 in = *reinterpret_cast<const uint4*>(src);
                const uint16_t* bb = reinterpret_cast<const uint16_t*>(&in);
                uint4 lo, hi;
                lo.x = e4m3x2_to_bf16x2(bb[0]); lo.y = e4m3x2_to_bf16x2(bb[1]);
                lo.z = e4m3x2_to_bf16x2(bb[2]); lo.w = e4m3x2_to_bf16x2(bb[3]);
                hi.x = e4m3x2_to_bf16x2(bb[4]); hi.y = e4m3x2_to_bf16x2(bb[5]);
                hi.z = e4m3x2_to_bf16x2(bb[6]); hi.w = e4m3x2_to_bf16x2(bb[7]);
                *reinterpret_cast<uint4*>(dst + swz_off<SUB>(rr, 2 * c8)) = lo;
                *reinterpret_cast<uint4*>(dst + swz_off<SUB>(rr, 2 * c8 + 1)) = hi;
            }
            __syncthreads();
            kt = cvt;
            vt = cvt + SUB * 256;
        }
        // S = Q K^T for this warp's 16 gathered rows
        float acc[2][4];
        const uint32_t kb = smem_u32(kt);
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
#pragma unroll
            for (int e = 0; e < 4; ++e) acc[nt][e] = 0.f;
            const int r = warp * 16 + nt * 8 + (lane & 7);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
                uint32_t b0, b1, b2, b3;
                ldsm_x4(kb + swz_off<SUB>(r, 4 * kk + (lane >> 3)), b0, b1, b2, b3);
                mma_bf16(acc[nt], qa[2 * kk], b0, b1);
                mma_bf16(acc[nt], qa[2 * kk + 1], b2, b3);
            }
        }
        const int* si = sidx + i * SUB;
        float vf[2][2];
        float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
            const int r0 = warp * 16 + nt * 8 + 2 * t;
            const bool ok0 = si[r0] >= 0, ok1 = si[r0 + 1] >= 0;
            float f0 = a.sc2, f1 = a.sc2;
            if (KV8) {
                f0 *= sks[i * SUB + r0]; f1 *= sks[i * SUB + r0 + 1];
                vf[nt][0] = svs[i * SUB + r0]; vf[nt][1] = svs[i * SUB + r0 + 1];
            } else {
                vf[nt][0] = vf[nt][1] = 1.f;
            }
            acc[nt][0] = ok0 ? acc[nt][0] * f0 : -INFINITY;
            acc[nt][1] = ok1 ? acc[nt][1] * f1 : -INFINITY;
            acc[nt][2] = ok0 ? acc[nt][2] * f0 : -INFINITY;
            acc[nt][3] = ok1 ? acc[nt][3] * f1 : -INFINITY;
            mx[0] = fmaxf(mx[0], fmaxf(acc[nt][0], acc[nt][1]));
            mx[1] = fmaxf(mx[1], fmaxf(acc[nt][2], acc[nt][3]));
        }
        float alpha[2];
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
            mx[hh] = fmaxf(mx[hh], __shfl_xor_sync(0xffffffffu, mx[hh], 1));
            mx[hh] = fmaxf(mx[hh], __shfl_xor_sync(0xffffffffu, mx[hh], 2));
            const float mn = fmaxf(m2[hh], mx[hh]);
            alpha[hh] = (mn == -INFINITY) ? 1.f : ex2(m2[hh] - mn);
            m2[hh] = mn;
        }
        float pr[2][4];
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int hh = e >> 1;
                pr[nt][e] = (m2[hh] == -INFINITY) ? 0.f : ex2(acc[nt][e] - m2[hh]);
            }
#pragma unroll
        for (int hh = 0; hh < 2; ++hh)
            l2[hh] = l2[hh] * alpha[hh] + pr[0][2 * hh] + pr[0][2 * hh + 1] + pr[1][2 * hh] + pr[1][2 * hh + 1];
#pragma unroll
        for (int n = 0; n < 16; ++n) {
            o[n][0] *= alpha[0]; o[n][1] *= alpha[0];
            o[n][2] *= alpha[1]; o[n][3] *= alpha[1];
        }
        uint32_t pa[4];
        pa[0] = pack_bf16(pr[0][0] * vf[0][0], pr[0][1] * vf[0][1]);
        pa[1] = pack_bf16(pr[0][2] * vf[0][0], pr[0][3] * vf[0][1]);
        pa[2] = pack_bf16(pr[1][0] * vf[1][0], pr[1][1] * vf[1][1]);
        pa[3] = pack_bf16(pr[1][2] * vf[1][0], pr[1][3] * vf[1][1]);
        const uint32_t vb = smem_u32(vt);
        const int vr = warp * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
#pragma unroll
        for (int cc = 0; cc < 8; ++cc) {
            uint32_t b0, b1, b2, b3;
            ldsm_x4_t(vb + swz_off<SUB>(vr, 2 * cc + (lane >> 4)), b0, b1, b2, b3);
            mma_bf16(o[2 * cc], pa, b0, b1);
            mma_bf16(o[2 * cc + 1], pa, b2, b3);
        }
        __syncthreads();
        if (i + 2 < n_sub) gather(i + 2, s);
    }

    // merge the 4 warps: quad-reduce l, then a common max per head
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
        l2[hh] += __shfl_xor_sync(0xffffffffu, l2[hh], 1);
        l2[hh] += __shfl_xor_sync(0xffffffffu, l2[hh], 2);
    }
    if (t == 0) {
        wm[warp][g] = m2[0]; wl[warp][g] = l2[0];
        wm[warp][g + 8] = m2[1]; wl[warp][g + 8] = l2[1];
    }
    __syncthreads();
    float M[2], f[2];
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
        const int h = g + 8 * hh;
        M[hh] = fmaxf(fmaxf(wm[0][h], wm[1][h]), fmaxf(wm[2][h], wm[3][h]));
        f[hh] = (M[hh] == -INFINITY) ? 0.f : ex2(m2[hh] - M[hh]);
    }
    // each warp's rescaled O goes to its own padded slab in the drained stage buffers,
    // then the four slabs are summed (no shared atomics)
    constexpr int RP = D + 4;                              // padded row (floats)
    float* slab = reinterpret_cast<float*>(smem) + warp * H * RP;
#pragma unroll
    for (int n = 0; n < 16; ++n) {
        const int d = 8 * n + 2 * t;
        *reinterpret_cast<float2*>(&slab[g * RP + d]) = make_float2(o[n][0] * f[0], o[n][1] * f[0]);
        *reinterpret_cast<float2*>(&slab[(g + 8) * RP + d]) = make_float2(o[n][2] * f[1], o[n][3] * f[1]);
    }
    __syncthreads();
    {
        const float* sb = reinterpret_cast<const float*>(smem);
        for (int i = tid; i < H * D; i += NT) {
            const int h = i / D, d = i % D;
            red_o[i] = sb[h * RP + d] + sb[H * RP + h * RP + d] + sb[2 * H * RP + h * RP + d] + sb[3 * H * RP + h * RP + d];
        }
    }
    __syncthreads();
    // per-head CTA (max, sum); threads 0..15 own head tid
    __shared__ float cm[H], cl[H];
    if (tid < H) {
        const float Mh = fmaxf(fmaxf(wm[0][tid], wm[1][tid]), fmaxf(wm[2][tid], wm[3][tid]));
        float Lh = 0.f;
        if (Mh != -INFINITY)
            for (int w = 0; w < 4; ++w) Lh += wl[w][tid] * ex2(wm[w][tid] - Mh);
        cm[tid] = Mh; cl[tid] = Lh;
    }
    __syncthreads();

    if (a.splits == 1) {
        for (int i = tid; i < H * D; i += NT) {
            const int h = i / D;
            const float val = cl[h] > 0.f ? red_o[i] / cl[h] : 0.f;
            a.o[static_cast<size_t>(row) * H * D + i] = __float2bfloat16_rn(val);
        }
        if (a.lse && tid < H)
            a.lse[static_cast<size_t>(row) * H + tid] = cl[tid] > 0.f ? (cm[tid] + log2f(cl[tid])) * kLn2 : -INFINITY;
        return;
    }
    float* my = a.part_o + (static_cast<size_t>(row) * a.splits + split) * H * D;
    for (int i = tid; i < H * D; i += NT) my[i] = red_o[i];
    if (tid < H) a.part_ml[(static_cast<size_t>(row) * a.splits + split) * H + tid] = make_float2(cm[tid], cl[tid]);
    __threadfence();
    __syncthreads();
    if (tid == 0) s_last = (atomicAdd(&a.counter[row], 1) == a.splits - 1);
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    if (tid == 0) a.counter[row] = 0;          // ready for the next launch
    // merge the splits: every split's (max, sum) is staged in shared memory by one
    // parallel round of loads, then the partial outputs are weighted and summed with
    // independent 16-byte loads (4 per thread per split)
    __shared__ float2 sml[kMaxSplits][H];
    __shared__ float sw[kMaxSplits][H];
    __shared__ float fm[H], finv[H];
    const float2* pml = a.part_ml + static_cast<size_t>(row) * a.splits * H;
    for (int i = tid; i < a.splits * H; i += NT) sml[i / H][i % H] = __ldcg(pml + i);
    __syncthreads();
    if (tid < H) {
        float m = -INFINITY, l = 0.f;
        for (int sp = 0; sp < a.splits; ++sp) merge_ml(m, l, sml[sp][tid].x, sml[sp][tid].y);
        fm[tid] = m;
        finv[tid] = l > 0.f ? 1.f / l : 0.f;
        if (a.lse) a.lse[static_cast<size_t>(row) * H + tid] = l > 0.f ? (m + log2f(l)) * kLn2 : -INFINITY;
    }
    __syncthreads();
    for (int i = tid; i < a.splits * H; i += NT) {
        const int sp = i / H, h = i % H;
        const float mm = sml[sp][h].x;
        sw[sp][h] = (mm == -INFINITY) ? 0.f : ex2(mm - fm[h]) * finv[h];
    }
    __syncthreads();
    const float4* base4 = reinterpret_cast<const float4*>(a.part_o + static_cast<size_t>(row) * a.splits * H * D);
    constexpr int F4 = H * D / 4;                  // float4 per split partial
    constexpr int PER = F4 / NT;                   // 4 per thread
    float4 acc[PER];
#pragma unroll
    for (int k = 0; k < PER; ++k) acc[k] = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 3
    for (int sp = 0; sp < a.splits; ++sp) {
        float4 v[PER];
#pragma unroll
        for (int k = 0; k < PER; ++k) v[k] = __ldcg(base4 + static_cast<size_t>(sp) * F4 + tid + k * NT);
#pragma unroll
        for (int k = 0; k < PER; ++k) {
            const float w = sw[sp][(tid + k * NT) / (D / 4)];
            acc[k].x += w * v[k].x; acc[k].y += w * v[k].y; acc[k].z += w * v[k].z; acc[k].w += w * v[k].w;
        }
    }
#pragma unroll
    for (int k = 0; k < PER; ++k) {
        const int f = tid + k * NT;
        uint2 packed;
        packed.x = pack_bf16(acc[k].x, acc[k].y);
        packed.y = pack_bf16(acc[k].z, acc[k].w);
        *reinterpret_cast<uint2*>(a.o + static_cast<size_t>(row) * H * D + 4 * f) = packed;
    }
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

template <bool KV8>
size_t smem_bytes(int chunk) {
    using L = Layout<KV8>;
    return 1024 + 2 * L::STAGE + L::CVT + H * D * 4 + static_cast<size_t>(chunk) * 4 * (KV8 ? 3 : 1);
}

template <bool KV8>
cudaError_t launch_impl(const SparseArgs& sa, cudaStream_t st) {
    const SparsePlan pl = plan_sparse(sa.rows, sa.idx_stride);
    Params a{};
    a.rows = sa.rows; a.n_q = sa.n_q; a.idx_stride = sa.idx_stride;
    a.splits = pl.splits; a.chunk = pl.chunk; a.cap = sa.cap;
    a.q = static_cast<const __nv_bfloat16*>(sa.q);
    a.k = static_cast<const uint8_t*>(sa.k);
    a.v = static_cast<const uint8_t*>(sa.v);
    a.k_scale = sa.k_scale; a.v_scale = sa.v_scale;
    a.idx = sa.idx; a.cnt = sa.cnt;
    a.sc2 = sa.scale * kLog2e;
    uint8_t* ws = static_cast<uint8_t*>(sa.ws);
    a.part_ml = reinterpret_cast<float2*>(ws);
    ws += align256(sizeof(float2) * sa.rows * pl.splits * H);
    a.part_o = reinterpret_cast<float*>(ws);
    ws += align256(sizeof(float) * static_cast<size_t>(sa.rows) * pl.splits * H * D);
    // semaphore counters live in the status block (zeroed by hs2_workspace_init; the
    // last CTA of a row resets its counter)
    a.counter = reinterpret_cast<int*>(sa.status) + kCounterOffsetInts;
    a.o = static_cast<__nv_bfloat16*>(sa.o);
    a.lse = sa.lse;
    a.status = sa.status;
    const size_t sm = smem_bytes<KV8>(pl.chunk);
    cudaError_t e;
    e = cudaFuncSetAttribute(sparse_kernel<KV8>, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(sm));
    if (e != cudaSuccess) return e;
    sparse_kernel<KV8><<<dim3(pl.splits, sa.rows), NT, sm, st>>>(a);
    return cudaGetLastError();
}

}  // namespace

SparsePlan plan_sparse(int rows, int idx_stride) {
    SparsePlan pl;
    // enough CTAs to cover the SMs twice; one CTA per row when rows alone do
    int splits = (2 * num_sms() + rows - 1) / (rows > 0 ? rows : 1);
    if (rows > kMaxCounters) splits = 1;           // semaphore counters exist for kMaxCounters rows
    int max_splits = (idx_stride + SUB - 1) / SUB;
    if (max_splits > kMaxSplits) max_splits = kMaxSplits;
    if (splits > max_splits) splits = max_splits;
    if (splits < 1) splits = 1;
    int chunk = (idx_stride + splits - 1) / splits;
    chunk = (chunk + SUB - 1) / SUB * SUB;
    pl.chunk = chunk;
    pl.splits = (idx_stride + chunk - 1) / chunk;
    return pl;
}

size_t sparse_ws_bytes(int rows, int idx_stride) {
    const SparsePlan pl = plan_sparse(rows, idx_stride);
    if (pl.splits == 1) return 0;
    return align256(sizeof(float2) * rows * pl.splits * H) +
           align256(sizeof(float) * static_cast<size_t>(rows) * pl.splits * H * D) +
           align256(sizeof(int) * rows);
}

cudaError_t launch_sparse(const SparseArgs& a, cudaStream_t st) {
    if (a.rows <= 0) return cudaSuccess;
    return a.kv8 ? launch_impl<true>(a, st) : launch_impl<false>(a, st);
}

}  // namespace hs2

// ---------------------------------------------------------------------------
// Variant without a caller workspace, for callers that cannot allocate device
// memory when they call us.  Its scratch (status word, split partials and the
// semaphore counters) lives in one fixed file-scope device array that every GPU
// loading this library keeps until the process exits.
namespace hs2 {
namespace {

constexpr size_t kNoAllocScratchBytes = size_t(4) << 20;     // 4 MiB per device

static __device__ __align__(256) uint8_t g_sparse_scratch[kNoAllocScratchBytes];

std::mutex g_scratch_mu;
void* g_scratch_addr[64] = {nullptr};

// Device address of g_sparse_scratch on the current device, looked up once per
// device (host code cannot use the symbol itself as a device pointer).
cudaError_t scratch_address(void** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (!g_scratch_addr[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_sparse_scratch);
        if (e != cudaSuccess) return e;
        // status word and semaphore counters start at zero (the counters return to
        // zero at the end of every call)
        e = cudaMemset(p, 0, kStatusBytes);
        if (e != cudaSuccess) return e;
        g_scratch_addr[dev] = p;
    }
    *out = g_scratch_addr[dev];
    return cudaSuccess;
}

}  // namespace

size_t sparse_noalloc_capacity() { return kNoAllocScratchBytes; }

cudaError_t launch_sparse_noalloc(const SparseArgs& in, cudaStream_t st, bool* too_large) {
    *too_large = false;
    if (in.rows <= 0) return cudaSuccess;
    if (kStatusBytes + sparse_ws_bytes(in.rows, in.idx_stride) > kNoAllocScratchBytes) {
        *too_large = true;
        return cudaSuccess;
    }
    void* base = nullptr;
    const cudaError_t e = scratch_address(&base);
    if (e != cudaSuccess) return e;
    SparseArgs a = in;
    a.status = static_cast<uint32_t*>(base);
    a.ws = static_cast<uint8_t*>(base) + kStatusBytes;
    return launch_sparse(a, st);
}

}  // namespace hs2
