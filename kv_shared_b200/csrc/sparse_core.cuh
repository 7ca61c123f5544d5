// sparse_core.cuh -- the per-CTA arithmetic of the many-rows sparse-attention
// kernel: each warp's 16 gathered rows of a 64-row sub-tile against the 16 query
// heads (mma.sync m16n8k16, M = the heads, online softmax in registers), and the
// reduction of the four warps' states to one (max, sum, O) per head.
#pragma once

#include "common.cuh"
#include "e4m3_mma.cuh"

namespace hs2 {
namespace sparse {

constexpr int H = 16;
constexpr int D = 128;
constexpr int SUB = 64;            // gathered rows per sub-tile
constexpr int NT = 128;            // 4 warps x 16 rows
constexpr int RP = D + 4;          // padded slab row (floats) of the warp merge
static_assert((RP * 4) % 16 == 0, "slab rows stay 16-byte aligned");
// Two buffers per warp (one gather in flight while the other is attended) and three CTAs
// per SM: a third buffer per warp, which leaves room for only two CTAs per SM, was slower,
// while the third CTA hides the latency of the per-warp MMA chains and softmax.
constexpr int STAGES = 2;
constexpr int MIN_CTAS = 3;        // resident CTAs per SM the register budget must allow

// One stage (the four warps' buffers for one sub-tile) holds SUB K rows and SUB V rows as
// copied, each row padded by 16 bytes so that the 8 rows an ldmatrix phase reads fall on
// distinct banks; see WarpSlot for the layout of a warp's share.
template <bool KV8>
struct Layout {
    static constexpr int ROWB = KV8 ? 128 : 256;      // bytes per gathered cache row
    static constexpr int ROWP = ROWB + 16;             // row pitch in a buffer
    static constexpr int STAGE = 2 * SUB * ROWP;       // K and V rows of one sub-tile
    static constexpr int CVT = KV8 ? 2 * SUB * 256 : 0;
    static constexpr int SLABS = 4 * H * RP * 4;       // warp-merge slabs (bytes)
};

__device__ __forceinline__ uint8_t* align128(uint8_t* p) {
    return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 127) & ~uintptr_t(127));
}

__device__ __forceinline__ void merge_ml(float& m, float& l, float m2, float l2) {
    const float mn = fmaxf(m, m2);
    if (mn == -INFINITY) return;
    l = l * ex2(m - mn) + l2 * ex2(m2 - mn);
    m = mn;
}

// Per-thread softmax state: rows g and g + 8 of the 16 heads (m2, l2 per head
// half), O fragments of 16 column blocks of 8.
struct State {
    float m2[2], l2[2];
    float o[16][4];
    __device__ __forceinline__ void init() {
        m2[0] = m2[1] = -INFINITY;
        l2[0] = l2[1] = 0.f;
#pragma unroll
        for (int n = 0; n < 16; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;
    }
};

// Q fragments (A operand, 16 heads x 128) of one query row, straight from global.
__device__ __forceinline__ void load_q(const __nv_bfloat16* qrow, uint32_t (&qa)[8][4], int g, int t) {
    const uint32_t* q32 = reinterpret_cast<const uint32_t*>(qrow);
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
        qa[ks][0] = __ldg(q32 + (g * D + 16 * ks + 2 * t) / 2);
        qa[ks][1] = __ldg(q32 + ((g + 8) * D + 16 * ks + 2 * t) / 2);
        qa[ks][2] = __ldg(q32 + (g * D + 16 * ks + 2 * t + 8) / 2);
        qa[ks][3] = __ldg(q32 + ((g + 8) * D + 16 * ks + 2 * t + 8) / 2);
    }
}

// Each warp gathers and attends its own 16 rows of every 64-row sub-tile, with its own
// buffers and cp.async groups, so that no warp waits for another's rows.  A warp's slot
// holds its 16 K rows, then its 16 V rows, each padded by 16 bytes so that the 8 rows an
// ldmatrix phase reads fall on distinct banks.
template <bool KV8>
struct WarpSlot {
    static constexpr int BYTES = 2 * 16 * Layout<KV8>::ROWP;
    static constexpr int CVT = KV8 ? 2 * 16 * 256 : 0;      // the warp's converted K, V (e4m3)
};

// Issues the 16-byte cp.async copies of this warp's 16 rows `si` (cache row per entry, -1 =
// none: zero-filled) into its slot `ws`; consecutive lanes copy consecutive chunks of a row.
// No commit.
template <bool KV8>
__device__ __forceinline__ void gather_warp_rows(uint8_t* ws, const int* si, const uint8_t* k, const uint8_t* v,
                                                 size_t seq_base, int lane) {
    using L = Layout<KV8>;
    constexpr int CH = L::ROWB / 16;                   // 16-byte chunks per row
    constexpr int RPI = 32 / CH;                       // rows per instruction
    const int ch = lane % CH;
#pragma unroll
    for (int u = 0; u < 16 / RPI; ++u) {
        const int r = u * RPI + lane / CH;
        const int j = si[r];
        const size_t off = (seq_base + (j >= 0 ? j : 0)) * L::ROWB + ch * 16;
        // bf16: padded rows; e4m3: 128-byte rows with the chunk index XOR-ed by row % 8, the
        // layout the f16 MMA helpers read
        const uint32_t d = KV8 ? r * 128 + ((ch ^ (r & 7)) << 4) : r * L::ROWP + ch * 16;
        cp_async16_zfill(ws + d, k + off, j >= 0);
        cp_async16_zfill(ws + 16 * L::ROWP + d, v + off, j >= 0);
    }
}

// This warp's landed 16 rows (slot `ws`) are scored against the 16 heads, the online
// softmax advanced and P V added.  bf16 rows: bf16 MMAs on the padded rows.  e4m3 rows: f16
// MMAs straight from the gathered codes (`qa` are Q's f16 fragments in the helpers' k order,
// `sc2` already divided by Q's power-of-two scale); P times the V scale enters the f16 MMA
// multiplied by `pscale` (a power of two that keeps the CTA's largest V scale at 2^14), and
// O accumulates in the helpers' dim order (see pv_e4m3), pscale included.  `si` / `sks` /
// `svs`: the rows' cache rows and (e4m3) per-token scales.
template <bool KV8>
__device__ __forceinline__ void attend_warp_rows(const uint8_t* ws, const int* si, const float* sks,
                                                 const float* svs, const uint32_t (&qa)[8][4], float sc2,
                                                 float pscale, State& s, int lane) {
    using L = Layout<KV8>;
    const int t = lane & 3;
    const uint8_t* kt = ws;
    const uint8_t* vt = ws + 16 * L::ROWP;
    auto off = [](int r, int ch) -> uint32_t { return static_cast<uint32_t>(r * L::ROWP + ch * 16); };
    // S = Q K^T for the warp's 16 rows
    float acc[2][4];
    const uint32_t kb = smem_u32(kt);
    if (KV8) {
        qk_e4m3(kb, 0, qa, acc, lane);
    } else {
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
#pragma unroll
            for (int e = 0; e < 4; ++e) acc[nt][e] = 0.f;
            const int r = nt * 8 + (lane & 7);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
                uint32_t b0, b1, b2, b3;
                ldsm_x4(kb + off(r, 4 * kk + (lane >> 3)), b0, b1, b2, b3);
                mma_bf16(acc[nt], qa[2 * kk], b0, b1);
                mma_bf16(acc[nt], qa[2 * kk + 1], b2, b3);
            }
        }
    }
    float vf[2][2];
    float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
        const int r0 = nt * 8 + 2 * t;
        const bool ok0 = si[r0] >= 0, ok1 = si[r0 + 1] >= 0;
        float f0 = sc2, f1 = sc2;
        if (KV8) {
            f0 *= sks[r0]; f1 *= sks[r0 + 1];
            vf[nt][0] = svs[r0] * pscale; vf[nt][1] = svs[r0 + 1] * pscale;
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
        const float mn = fmaxf(s.m2[hh], mx[hh]);
        alpha[hh] = (mn == -INFINITY) ? 1.f : ex2(s.m2[hh] - mn);
        s.m2[hh] = mn;
    }
    float pr[2][4];
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int hh = e >> 1;
            pr[nt][e] = (s.m2[hh] == -INFINITY) ? 0.f : ex2(acc[nt][e] - s.m2[hh]);
        }
#pragma unroll
    for (int hh = 0; hh < 2; ++hh)
        s.l2[hh] = s.l2[hh] * alpha[hh] + pr[0][2 * hh] + pr[0][2 * hh + 1] + pr[1][2 * hh] + pr[1][2 * hh + 1];
#pragma unroll
    for (int n = 0; n < 16; ++n) {
        s.o[n][0] *= alpha[0]; s.o[n][1] *= alpha[0];
        s.o[n][2] *= alpha[1]; s.o[n][3] *= alpha[1];
    }
    uint32_t pa[4];
    if (KV8) {
        pa[0] = pack_f16(pr[0][0] * vf[0][0], pr[0][1] * vf[0][1]);
        pa[1] = pack_f16(pr[0][2] * vf[0][0], pr[0][3] * vf[0][1]);
        pa[2] = pack_f16(pr[1][0] * vf[1][0], pr[1][1] * vf[1][1]);
        pa[3] = pack_f16(pr[1][2] * vf[1][0], pr[1][3] * vf[1][1]);
        pv_e4m3(smem_u32(vt), 0, pa, s.o, lane);
        return;
    }
    pa[0] = pack_bf16(pr[0][0] * vf[0][0], pr[0][1] * vf[0][1]);
    pa[1] = pack_bf16(pr[0][2] * vf[0][0], pr[0][3] * vf[0][1]);
    pa[2] = pack_bf16(pr[1][0] * vf[1][0], pr[1][1] * vf[1][1]);
    pa[3] = pack_bf16(pr[1][2] * vf[1][0], pr[1][3] * vf[1][1]);
    const uint32_t vb = smem_u32(vt);
    const int vr = (lane & 7) + ((lane >> 3) & 1) * 8;
#pragma unroll
    for (int cc = 0; cc < 8; ++cc) {
        uint32_t b0, b1, b2, b3;
        ldsm_x4_t(vb + off(vr, 2 * cc + (lane >> 4)), b0, b1, b2, b3);
        mma_bf16(s.o[2 * cc], pa, b0, b1);
        mma_bf16(s.o[2 * cc + 1], pa, b2, b3);
    }
}

// Reduces the four warps' states to this CTA's per-head (max, sum) in cm/cl and its
// unnormalized O (rescaled to that max) in red_o[H][D].  `slabs` (Layout::SLABS bytes)
// must be free shared memory (the drained stages); wm/wl are [4][H] scratch.  e4m3: O is in
// pv_e4m3's dim order and carries the factor 1 / `oscale`, both undone here.
template <bool KV8>
__device__ __forceinline__ void cta_reduce(const State& s, float* slabs, float* red_o, float (*wm)[H],
                                           float (*wl)[H], float* cm, float* cl, int tid, int warp, int lane,
                                           float oscale) {
    const int g = lane >> 2, t = lane & 3;
    float l2[2] = {s.l2[0], s.l2[1]};
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
        l2[hh] += __shfl_xor_sync(0xffffffffu, l2[hh], 1);
        l2[hh] += __shfl_xor_sync(0xffffffffu, l2[hh], 2);
    }
    if (t == 0) {
        wm[warp][g] = s.m2[0]; wl[warp][g] = l2[0];
        wm[warp][g + 8] = s.m2[1]; wl[warp][g + 8] = l2[1];
    }
    __syncthreads();
    float f[2];
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
        const int h = g + 8 * hh;
        const float M = fmaxf(fmaxf(wm[0][h], wm[1][h]), fmaxf(wm[2][h], wm[3][h]));
        f[hh] = (M == -INFINITY) ? 0.f : ex2(s.m2[hh] - M) * oscale;
    }
    // each warp's rescaled O goes to its own padded slab, then the four are summed
    float* slab = slabs + warp * H * RP;
#pragma unroll
    for (int n = 0; n < 16; ++n) {
        if (KV8) {                                       // pv_e4m3's dim order
            const int d = 32 * (n >> 2) + 16 * ((n >> 1) & 1) + 4 * t + (n & 1);
            slab[g * RP + d] = s.o[n][0] * f[0];
            slab[g * RP + d + 2] = s.o[n][1] * f[0];
            slab[(g + 8) * RP + d] = s.o[n][2] * f[1];
            slab[(g + 8) * RP + d + 2] = s.o[n][3] * f[1];
        } else {
            const int d = 8 * n + 2 * t;
            *reinterpret_cast<float2*>(&slab[g * RP + d]) = make_float2(s.o[n][0] * f[0], s.o[n][1] * f[0]);
            *reinterpret_cast<float2*>(&slab[(g + 8) * RP + d]) = make_float2(s.o[n][2] * f[1], s.o[n][3] * f[1]);
        }
    }
    __syncthreads();
    for (int i = tid; i < H * D / 4; i += NT) {            // 16-byte slab reads (RP * 4 B is a multiple of 16)
        const int h = (4 * i) / D, d = (4 * i) % D;
        float4 acc = *reinterpret_cast<const float4*>(&slabs[h * RP + d]);
#pragma unroll
        for (int w = 1; w < 4; ++w) {
            const float4 u = *reinterpret_cast<const float4*>(&slabs[w * H * RP + h * RP + d]);
            acc.x += u.x; acc.y += u.y; acc.z += u.z; acc.w += u.w;
        }
        *reinterpret_cast<float4*>(&red_o[4 * i]) = acc;
    }
    if (tid < H) {
        const float Mh = fmaxf(fmaxf(wm[0][tid], wm[1][tid]), fmaxf(wm[2][tid], wm[3][tid]));
        float Lh = 0.f;
        if (Mh != -INFINITY)
            for (int w = 0; w < 4; ++w) Lh += wl[w][tid] * ex2(wm[w][tid] - Mh);
        cm[tid] = Mh; cl[tid] = Lh;
    }
    __syncthreads();
}

}  // namespace sparse
}  // namespace hs2
