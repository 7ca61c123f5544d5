// sparse_attn.cu -- sparse-attention layer of a hybrid block (KV Reuse).
//
// "What HySparse2 is actually optimizing", section 2: a sparse layer keeps no
// cache or selector of its own and reads the full layer's cache at the full
// layer's chosen positions; section 3: window and global positions sit in one
// cache, so a single softmax covers the whole chosen set.
//
// For each query row (16 heads) the selected cache rows are gathered by index
// with 16-byte cp.async copies into shared memory (swizzled or padded so that
// ldmatrix reads are conflict-free), all 16 heads are computed against each
// gathered row once (mma.sync m16n8k16, M = the 16 heads), and the softmax stays
// online in registers.  Few rows (decode): one 4-CTA cluster per row, the CTAs'
// partials merged through distributed shared memory.  Many rows (prefill): one
// CTA per row, or a few split CTAs per row whose partials (max, sum, O) the last
// of them merges (semaphore counter, no spin).  e4m3 rows feed f16 MMAs straight
// from shared memory as gathered (exact conversion of each code pair in registers),
// their per-token scales folded into the logits and into P.
#include <mutex>

#include <cooperative_groups.h>

#include "common.cuh"
#include "e4m3_mma.cuh"
#include "internal.h"
#include "sparse_core.cuh"

namespace cg = cooperative_groups;

namespace hs2 {
namespace {

using sparse::D;
using sparse::H;
using sparse::Layout;
using sparse::NT;
using sparse::SUB;
constexpr int kMaxSplits = 32;     // bound of the split count (shared-memory merge tables)
constexpr int kWT = 16;            // selected entries per warp tile (cluster kernel)
constexpr int kClusterEntries = 1152;              // entries a cluster covers (72 warp tiles)

// Shape of the cluster kernel: NC CTAs per query row, each of 72 / NC warps.  Few rows take
// 8 CTAs of 9 warps (two per SM: a row spread over more SMs); enough rows to fill the GPU
// take 4 CTAs of 18 warps (one per SM: fewer CTAs for each row to wait on).
template <int NC>
struct CShape {
    static constexpr int kCluster = NC;
    static constexpr int kCW = kClusterEntries / kWT / NC;    // warps per CTA
    static constexpr int kCEntries = kWT * kCW;               // entries per CTA
    static constexpr int kCNT = 32 * kCW;                     // threads per CTA
    static constexpr int kHPC = H / NC;                       // heads each CTA finalizes
    static_assert(H % NC == 0 && kCW * NC * kWT == kClusterEntries, "the work splits evenly");
};
// rows up to which a launch takes the 8-CTA shape (8 x 18 CTAs fit one wave on 148 SMs)
constexpr int kWideClusterRows = 18;

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

// The selected count of `row`, clamped to what the index row can hold (flagged).
__device__ __forceinline__ int checked_count(const Params& a, int row) {
    int c = a.cnt[row];
    if (c < 0 || c > a.idx_stride) {
        if (threadIdx.x == 0) set_status(a.status, HS2_ERR_INDEX);
        c = c < 0 ? 0 : a.idx_stride;
    }
    return c;
}

// Entries [e_begin, e_begin + n) of the row's index list into sidx (and their e4m3
// scales into sks/svs); entries at or past `c`, and out-of-range rows (flagged),
// become -1.  The index loads do not wait for the count.
// Slots [n, n_alloc) (padding up to whole sub-tiles) become -1 as well.
template <bool KV8>
__device__ __forceinline__ void load_entries(const Params& a, int row, int e_begin, int n, int n_alloc, int c,
                                             int* sidx, float* sks, float* svs, size_t seq_base) {
    // eight entries per thread at a time: all their loads are in flight together (a row's
    // 1152 indices otherwise cost nine dependent round trips)
    constexpr int U = 8;
    const int32_t* irow = a.idx + static_cast<size_t>(row) * a.idx_stride;
    for (int e0 = threadIdx.x; e0 < n_alloc; e0 += U * NT) {
        int j[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int e = e0 + u * NT, ge = e_begin + e;
            j[u] = (e < n_alloc && e < n && ge < a.idx_stride) ? __ldg(irow + ge) : -1;
        }
        float ks[U], vs[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int e = e0 + u * NT, ge = e_begin + e;
            if (e >= n || ge >= c) j[u] = -1;
            else if (j[u] < 0 || j[u] >= a.cap) { set_status(a.status, HS2_ERR_INDEX); j[u] = -1; }
            if (KV8) {
                ks[u] = j[u] >= 0 ? __ldg(a.k_scale + seq_base + j[u]) : 0.f;
                vs[u] = j[u] >= 0 ? __ldg(a.v_scale + seq_base + j[u]) : 0.f;
            }
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int e = e0 + u * NT;
            if (e < n_alloc) {
                sidx[e] = j[u];
                if (KV8) { sks[e] = ks[u]; svs[e] = vs[u]; }
            }
        }
    }
}

template <bool KV8>
__global__ void __launch_bounds__(NT, sparse::MIN_CTAS) sparse_kernel(Params a) {
    using L = Layout<KV8>;
    using sparse::STAGES;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = sparse::align128(smem_raw);
    using WS = sparse::WarpSlot<KV8>;
    static_assert(4 * WS::BYTES == L::STAGE && 4 * WS::CVT == L::CVT, "four warps' slots make a sub-tile");
    uint8_t* cvt = smem + STAGES * L::STAGE;               // e4m3: room the warp merge below uses
    int* sidx = reinterpret_cast<int*>(cvt + L::CVT);      // [chunk] cache row per entry (-1 invalid)
    float* sks = reinterpret_cast<float*>(sidx + a.chunk); // [chunk] k scales (e4m3)
    float* svs = sks + a.chunk;                            // [chunk] v scales (e4m3)
    // after the sub-tiles the stages (and the e4m3 tiles after them) hold the warp slabs,
    // then these:
    float* red_o = reinterpret_cast<float*>(smem + L::SLABS);                  // [H][D]
    float2 (*sml)[H] = reinterpret_cast<float2 (*)[H]>(red_o + H * D);        // [kMaxSplits][H]
    float (*sw)[H] = reinterpret_cast<float (*)[H]>(sml + kMaxSplits);        // [kMaxSplits][H]
    static_assert(L::SLABS + H * D * 4 + kMaxSplits * H * 12 <= STAGES * L::STAGE + L::CVT,
                  "merge scratch fits the stage area");
    __shared__ float wm[4][H], wl[4][H], cm[H], cl[H];
    __shared__ int s_last;

    const int row = blockIdx.y, split = blockIdx.x;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int b = row / a.n_q;
    const int c = checked_count(a, row);
    const int e_begin = split * a.chunk;
    const int e_end = min(c, e_begin + a.chunk);
    const int n_sub = e_end > e_begin ? (e_end - e_begin + SUB - 1) / SUB : 0;
    const size_t seq_base = static_cast<size_t>(b) * a.cap;

    // the queries (needed at the first sub-tile) and every index (and scale) of this CTA's
    // entries, loaded once up front, their latencies overlapped
    // (e4m3: Q as f16 fragments in the e4m3 helpers' k order, divided by a power of two)
    uint32_t qa[8][4];
    float qscale = 1.f;
    if (KV8) qscale = load_q_frags_e4m3(a.q + static_cast<size_t>(row) * H * D, lane >> 2, lane & 3, qa);
    else sparse::load_q(a.q + static_cast<size_t>(row) * H * D, qa, lane >> 2, lane & 3);
    load_entries<KV8>(a, row, e_begin, a.chunk, a.chunk, c, sidx, sks, svs, seq_base);
    __syncthreads();
    // e4m3: P * v_scale enters the f16 MMAs times pscale, a power of two that brings the
    // largest V scale of this CTA's entries to 2^14 (f16 keeps 2^-14 .. 65504 normal)
    float pscale = 1.f;
    if (KV8) {
        float vmax = 0.f;
        for (int e = tid; e < a.chunk; e += NT) vmax = fmaxf(vmax, svs[e]);
        vmax = __uint_as_float(__reduce_max_sync(0xffffffffu, __float_as_uint(vmax)));   // >= 0: bits order
        if (lane == 0) wm[0][warp] = vmax;
        __syncthreads();
        vmax = fmaxf(fmaxf(wm[0][0], wm[0][1]), fmaxf(wm[0][2], wm[0][3]));
        __syncthreads();
        int ex = 0;
        if (vmax > 0.f) frexpf(vmax, &ex);               // vmax < 2^ex
        pscale = ldexpf(1.f, 14 - ex);
    }
    // this warp's rows 16 warp .. 16 warp + 15 of every sub-tile, through its own STAGES slots
    uint8_t* wslots = smem + warp * STAGES * WS::BYTES;
    auto gather = [&](int i) {
        sparse::gather_warp_rows<KV8>(wslots + (i % STAGES) * WS::BYTES, sidx + i * SUB + warp * 16, a.k, a.v,
                                      seq_base, lane);
        cp_async_commit();
    };
    static_assert(STAGES == 2, "one gather in flight per warp while the other slot is attended");
    if (n_sub > 0) gather(0);

    sparse::State stt;
    stt.init();
    for (int i = 0; i < n_sub; ++i) {
        // the slot of sub-tile i - 1 (read by this warp's last, completed, step) takes i + 1;
        // then sub-tile i must have landed, every lane's copies visible to the warp
        __syncwarp();
        if (i + 1 < n_sub) {
            gather(i + 1);
            cp_async_wait<1>();
        } else {
            cp_async_wait<0>();
        }
        __syncwarp();
        const int e = i * SUB + warp * 16;
        sparse::attend_warp_rows<KV8>(wslots + (i % STAGES) * WS::BYTES, sidx + e, sks + e, svs + e, qa,
                                      a.sc2 * qscale, pscale, stt, lane);
    }
    sparse::cta_reduce<KV8>(stt, reinterpret_cast<float*>(smem), red_o, wm, wl, cm, cl, tid, warp, lane, 1.f / pscale);

    if (a.splits == 1) {
        for (int i = tid; i < H * D / 4; i += NT) {
            const int h = (4 * i) / D;
            const float inv = cl[h] > 0.f ? 1.f / cl[h] : 0.f;
            const float4 v = *reinterpret_cast<const float4*>(&red_o[4 * i]);
            uint2 packed;
            packed.x = pack_bf16(v.x * inv, v.y * inv);
            packed.y = pack_bf16(v.z * inv, v.w * inv);
            *reinterpret_cast<uint2*>(a.o + static_cast<size_t>(row) * H * D + 4 * i) = packed;
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
    __shared__ float fm[H], finv[H];
    const float2* pml = a.part_ml + static_cast<size_t>(row) * a.splits * H;
    for (int i = tid; i < a.splits * H; i += NT) sml[i / H][i % H] = __ldcg(pml + i);
    __syncthreads();
    if (tid < H) {
        float m = -INFINITY, l = 0.f;
        for (int sp = 0; sp < a.splits; ++sp) sparse::merge_ml(m, l, sml[sp][tid].x, sml[sp][tid].y);
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

// ---------------------------------------------------------------- cluster kernel
// Few rows (decode): the kCluster CTAs of a cluster share one query row, CTA r taking
// entries [r kCEntries, (r + 1) kCEntries).  Every warp owns one 16-entry warp tile:
// it loads its indices, gathers its K/V rows (16-byte cp.async into its own swizzled
// slice of shared memory), scores them against the 16 heads and forms its partial
// (max, sum, O) with no CTA-wide barrier on the way.  The warps' partials are folded
// into one per CTA with shared-memory float atomics, each CTA pushes its partial of
// heads 4p .. 4p + 3 into CTA p's shared memory (distributed shared memory stores),
// and after one cluster barrier CTA p finalizes those heads from its own memory.  Four
// CTAs of 18 warps per row (one per SM) were faster than eight of 9 warps (two per SM):
// 7.6 against 7.9 us per warm layer at 32 rows.
template <bool KV8, int NC>
struct CLayout {
    static constexpr int kCluster = CShape<NC>::kCluster, kCW = CShape<NC>::kCW, kHPC = CShape<NC>::kHPC;
    static constexpr int ROWB = KV8 ? 128 : 256;          // bytes per gathered row
    static constexpr int RAW = 2 * kWT * ROWB;            // one warp's gathered K then V rows
    static constexpr int TILE = 2 * kWT * 256;            // one warp's bf16 K then V tiles (= RAW)
    static constexpr int RAW_OFF = 0;
    static constexpr int GATHER_END = kCW * (KV8 ? RAW : TILE);
    static constexpr int SLAB_BYTES = kCW * H * sparse::RP * 4;   // the warps' rescaled O, after the compute
    static constexpr int Q_OFF = GATHER_END > SLAB_BYTES ? GATHER_END : SLAB_BYTES;
    static constexpr int RECV_OFF = Q_OFF + H * D * 2;    // [kCluster][kHPC][D] f32 pushed partials
    static constexpr int BYTES = RECV_OFF + kCluster * kHPC * D * 4;
};

// This warp's 16 gathered rows against the 16 heads: state `s` receives the tile's
// own (max, sum, O) (no prior state).  `ok0/ok1`: validity of rows 2t, 2t + 1 of each
// 8-row half; fk/fv: per-row logit and value factors (e4m3 scales; 1 for bf16).
__device__ __forceinline__ void attend_warp_tile(const uint8_t* kt, const uint8_t* vt, const uint8_t* qs,
                                                 const bool (&ok)[2][2], const float (&fk)[2][2],
                                                 const float (&fv)[2][2], float sc2, sparse::State& s, int lane) {
    float acc[2][4];
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[nt][e] = 0.f;
    const uint32_t kb = smem_u32(kt), qb = smem_u32(qs);
    const int qr = (lane & 7) + ((lane >> 3) & 1) * 8;     // A fragments: matrices (rows 0-7 | 8-15) x (k lo | hi)
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
        uint32_t qa[2][4];
#pragma unroll
        for (int u = 0; u < 2; ++u)
            ldsm_x4(qb + swz_off<kWT>(qr, 2 * (2 * kk + u) + (lane >> 4)), qa[u][0], qa[u][1], qa[u][2], qa[u][3]);
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
            uint32_t b0, b1, b2, b3;
            ldsm_x4(kb + swz_off<kWT>(nt * 8 + (lane & 7), 4 * kk + (lane >> 3)), b0, b1, b2, b3);
            mma_bf16(acc[nt], qa[0], b0, b1);
            mma_bf16(acc[nt], qa[1], b2, b3);
        }
    }
    float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
        acc[nt][0] = ok[nt][0] ? acc[nt][0] * (sc2 * fk[nt][0]) : -INFINITY;
        acc[nt][1] = ok[nt][1] ? acc[nt][1] * (sc2 * fk[nt][1]) : -INFINITY;
        acc[nt][2] = ok[nt][0] ? acc[nt][2] * (sc2 * fk[nt][0]) : -INFINITY;
        acc[nt][3] = ok[nt][1] ? acc[nt][3] * (sc2 * fk[nt][1]) : -INFINITY;
        mx[0] = fmaxf(mx[0], fmaxf(acc[nt][0], acc[nt][1]));
        mx[1] = fmaxf(mx[1], fmaxf(acc[nt][2], acc[nt][3]));
    }
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
        mx[hh] = fmaxf(mx[hh], __shfl_xor_sync(0xffffffffu, mx[hh], 1));
        mx[hh] = fmaxf(mx[hh], __shfl_xor_sync(0xffffffffu, mx[hh], 2));
        s.m2[hh] = mx[hh];
    }
    float pr[2][4];
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int hh = e >> 1;
            pr[nt][e] = (mx[hh] == -INFINITY) ? 0.f : ex2(acc[nt][e] - mx[hh]);
        }
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
        float l = pr[0][2 * hh] + pr[0][2 * hh + 1] + pr[1][2 * hh] + pr[1][2 * hh + 1];
        l += __shfl_xor_sync(0xffffffffu, l, 1);
        l += __shfl_xor_sync(0xffffffffu, l, 2);
        s.l2[hh] = l;
    }
    uint32_t pa[4];
    pa[0] = pack_bf16(pr[0][0] * fv[0][0], pr[0][1] * fv[0][1]);
    pa[1] = pack_bf16(pr[0][2] * fv[0][0], pr[0][3] * fv[0][1]);
    pa[2] = pack_bf16(pr[1][0] * fv[1][0], pr[1][1] * fv[1][1]);
    pa[3] = pack_bf16(pr[1][2] * fv[1][0], pr[1][3] * fv[1][1]);
    const uint32_t vb = smem_u32(vt);
    const int vr = (lane & 7) + ((lane >> 3) & 1) * 8;
#pragma unroll
    for (int cc = 0; cc < 8; ++cc) {
        uint32_t b0, b1, b2, b3;
        ldsm_x4_t(vb + swz_off<kWT>(vr, 2 * cc + (lane >> 4)), b0, b1, b2, b3);
#pragma unroll
        for (int e = 0; e < 4; ++e) s.o[2 * cc][e] = 0.f, s.o[2 * cc + 1][e] = 0.f;
        mma_bf16(s.o[2 * cc], pa, b0, b1);
        mma_bf16(s.o[2 * cc + 1], pa, b2, b3);
    }
}

// The same for e4m3 rows: f16 MMAs straight from the gathered rows (128-byte swizzled, see
// e4m3_mma.cuh); `qa` are Q's f16 fragments in the permuted k order, scaled by 1 / qscale
// (folded into sc2q); P * v_scale is scaled by a power of two so that the warp's largest
// product stays at or below 2^14 in f16.  s.o ends in pv_e4m3's accumulator layout (dims
// permuted), scaled back to plain P V.
__device__ __forceinline__ void attend_warp_tile_e4m3(uint32_t kb, uint32_t vb, const uint32_t (&qa)[8][4],
                                                      const bool (&ok)[2][2], const float (&fk)[2][2],
                                                      const float (&fv)[2][2], float sc2q, float vmax,
                                                      sparse::State& s, int lane) {
    float acc[2][4];
    qk_e4m3(kb, 0, qa, acc, lane);
    float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
        acc[nt][0] = ok[nt][0] ? acc[nt][0] * (sc2q * fk[nt][0]) : -INFINITY;
        acc[nt][1] = ok[nt][1] ? acc[nt][1] * (sc2q * fk[nt][1]) : -INFINITY;
        acc[nt][2] = ok[nt][0] ? acc[nt][2] * (sc2q * fk[nt][0]) : -INFINITY;
        acc[nt][3] = ok[nt][1] ? acc[nt][3] * (sc2q * fk[nt][1]) : -INFINITY;
        mx[0] = fmaxf(mx[0], fmaxf(acc[nt][0], acc[nt][1]));
        mx[1] = fmaxf(mx[1], fmaxf(acc[nt][2], acc[nt][3]));
    }
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
        mx[hh] = fmaxf(mx[hh], __shfl_xor_sync(0xffffffffu, mx[hh], 1));
        mx[hh] = fmaxf(mx[hh], __shfl_xor_sync(0xffffffffu, mx[hh], 2));
        s.m2[hh] = mx[hh];
    }
    float pr[2][4];
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int hh = e >> 1;
            pr[nt][e] = (mx[hh] == -INFINITY) ? 0.f : ex2(acc[nt][e] - mx[hh]);
        }
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
        float l = pr[0][2 * hh] + pr[0][2 * hh + 1] + pr[1][2 * hh] + pr[1][2 * hh + 1];
        l += __shfl_xor_sync(0xffffffffu, l, 1);
        l += __shfl_xor_sync(0xffffffffu, l, 2);
        s.l2[hh] = l;
    }
    int ex = 0;
    if (vmax > 0.f) frexpf(vmax, &ex);                  // vmax < 2^ex
    const float pscale = ldexpf(1.f, 14 - ex), pinv = ldexpf(1.f, ex - 14);
    uint32_t pa[4];
    pa[0] = pack_f16(pr[0][0] * fv[0][0] * pscale, pr[0][1] * fv[0][1] * pscale);
    pa[1] = pack_f16(pr[0][2] * fv[0][0] * pscale, pr[0][3] * fv[0][1] * pscale);
    pa[2] = pack_f16(pr[1][0] * fv[1][0] * pscale, pr[1][1] * fv[1][1] * pscale);
    pa[3] = pack_f16(pr[1][2] * fv[1][0] * pscale, pr[1][3] * fv[1][1] * pscale);
#pragma unroll
    for (int n = 0; n < 16; ++n) s.o[n][0] = s.o[n][1] = s.o[n][2] = s.o[n][3] = 0.f;
    pv_e4m3(vb, 0, pa, s.o, lane);
#pragma unroll
    for (int n = 0; n < 16; ++n) {
        s.o[n][0] *= pinv; s.o[n][1] *= pinv; s.o[n][2] *= pinv; s.o[n][3] *= pinv;
    }
}

template <bool KV8, int NC>
__global__ void __launch_bounds__(CShape<NC>::kCNT, (CShape<NC>::kCNT <= 288 ? 2 : 1)) sparse_cluster_kernel(Params a) {
    using CL = CLayout<KV8, NC>;
    constexpr int kCluster = CShape<NC>::kCluster, kCW = CShape<NC>::kCW, kCEntries = CShape<NC>::kCEntries;
    constexpr int kCNT = CShape<NC>::kCNT, kHPC = CShape<NC>::kHPC;
    extern __shared__ uint8_t csm_raw[];
    uint8_t* csm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(csm_raw) + 127) & ~uintptr_t(127));
    uint8_t* qs = csm + CL::Q_OFF;                                    // [H][D] bf16, swz_off<16>
    float* recv_o = reinterpret_cast<float*>(csm + CL::RECV_OFF);    // [kCluster][kHPC][D]
    __shared__ float wm[kCW][H], wl[kCW][H], cmx[H], csum[H];
    __shared__ float2 recv_ml[kCluster][kHPC];

    cg::cluster_group cluster = cg::this_cluster();
    const int rank = static_cast<int>(cluster.block_rank());
    const int row = blockIdx.y;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, g = lane >> 2, t = lane & 3;
    const int b = row / a.n_q;
    const size_t seq_base = static_cast<size_t>(b) * a.cap;
    // a peer's shared memory may be written only once the peer runs: arrive now, wait
    // just before the pushes
    asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
    // the row's queries (16 heads x 128) into shared memory, one 16-byte chunk per thread
    // (bf16 rows; e4m3 rows take Q's fragments straight from global memory)
    if (!KV8 && tid < H * 16) {
        const int r = tid >> 4, ch = tid & 15;
        cp_async16(qs + swz_off<kWT>(r, ch), reinterpret_cast<const uint8_t*>(a.q + static_cast<size_t>(row) * H * D) +
                                                 r * 256 + ch * 16);
    }
    cp_async_commit();

    // ---- this warp's 16 entries: lane l < 16 holds entry e0 + l (the index load does not
    // wait for the count)
    const int e0 = rank * kCEntries + warp * kWT;
    int j = -1;
    if (lane < kWT && e0 + lane < a.idx_stride) j = a.idx[static_cast<size_t>(row) * a.idx_stride + e0 + lane];
    const int c = checked_count(a, row);
    float ksc = 0.f, vsc = 0.f;
    if (lane < kWT) {
        if (e0 + lane >= c) j = -1;
        else if (j < 0 || j >= a.cap) { set_status(a.status, HS2_ERR_INDEX); j = -1; }
        if (KV8 && j >= 0) { ksc = a.k_scale[seq_base + j]; vsc = a.v_scale[seq_base + j]; }
    } else {
        j = -1;
    }
    // ---- gather: a row's 16-byte chunks on consecutive lanes (whole rows per instruction)
    uint8_t* raw = csm + CL::RAW_OFF + warp * CL::RAW;
    {
        constexpr int CH = CL::ROWB / 16;                   // chunks per row: 16 (bf16) or 8 (e4m3)
        constexpr int RPI = 32 / CH;                        // rows per instruction
        const int ch = lane % CH;
#pragma unroll
        for (int u = 0; u < kWT / RPI; ++u) {
            const int r = u * RPI + lane / CH;
            const int jr = __shfl_sync(0xffffffffu, j, r);
            const size_t off = (seq_base + (jr >= 0 ? jr : 0)) * CL::ROWB + ch * 16;
            uint32_t dk;
            if (KV8) dk = r * 128 + ((ch ^ (r & 7)) << 4);
            else dk = swz_off<kWT>(r, ch);
            cp_async16_zfill(raw + dk, a.k + off, jr >= 0);
            cp_async16_zfill(raw + kWT * CL::ROWB + dk, a.v + off, jr >= 0);
        }
        cp_async_commit();
    }
    // per-lane row facts for the fragment layout: rows 8 nt + 2t and 8 nt + 2t + 1
    bool ok[2][2];
    float fk[2][2], fv[2][2];
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            const int r = nt * 8 + 2 * t + e;
            ok[nt][e] = __shfl_sync(0xffffffffu, j, r) >= 0;
            fk[nt][e] = KV8 ? __shfl_sync(0xffffffffu, ksc, r) : 1.f;
            fv[nt][e] = KV8 ? __shfl_sync(0xffffffffu, vsc, r) : 1.f;
        }
    // e4m3: Q's f16 fragments and the warp's largest V scale while the rows land
    uint32_t qa8[8][4];
    float qscale = 1.f, vmax = 0.f;
    if (KV8) {
        qscale = load_q_frags_e4m3(a.q + static_cast<size_t>(row) * H * D, g, t, qa8);
        vmax = vsc;                                      // 0 for lanes without a row
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) vmax = fmaxf(vmax, __shfl_xor_sync(0xffffffffu, vmax, off));
    }
    cp_async_wait<1>();                                  // the queries (committed first) have landed
    __syncthreads();
    cp_async_wait<0>();                                  // and this warp's rows
    __syncwarp();
    sparse::State st;
    if (KV8)
        attend_warp_tile_e4m3(smem_u32(raw), smem_u32(raw + kWT * CL::ROWB), qa8, ok, fk, fv, a.sc2 * qscale, vmax,
                              st, lane);
    else
        attend_warp_tile(raw, raw + kWT * CL::ROWB, qs, ok, fk, fv, a.sc2, st, lane);

    // ---- fold the warps into the push: each warp writes its own (max, sum) and its O
    // (relative to its own max) to a padded slab in the gather area (free once every
    // warp has computed: the barrier below); the push then weights and sums the slabs.
    if (t == 0) {
        wm[warp][g] = st.m2[0]; wl[warp][g] = st.l2[0];
        wm[warp][g + 8] = st.m2[1]; wl[warp][g + 8] = st.l2[1];
    }
    constexpr int RP = sparse::RP;
    float* slabs = reinterpret_cast<float*>(csm);
    __syncthreads();                                     // every warp is done with the gather area
    float* slab = slabs + warp * H * RP;
#pragma unroll
    for (int n = 0; n < 16; ++n) {
        if (KV8) {                                       // pv_e4m3's dim order
            const int d = 32 * (n >> 2) + 16 * ((n >> 1) & 1) + 4 * t + (n & 1);
            slab[g * RP + d] = st.o[n][0];
            slab[g * RP + d + 2] = st.o[n][1];
            slab[(g + 8) * RP + d] = st.o[n][2];
            slab[(g + 8) * RP + d + 2] = st.o[n][3];
        } else {
            const int d = 8 * n + 2 * t;
            *reinterpret_cast<float2*>(&slab[g * RP + d]) = make_float2(st.o[n][0], st.o[n][1]);
            *reinterpret_cast<float2*>(&slab[(g + 8) * RP + d]) = make_float2(st.o[n][2], st.o[n][3]);
        }
    }
    if (tid < H) {
        float M = -INFINITY;
        for (int w = 0; w < kCW; ++w) M = fmaxf(M, wm[w][tid]);
        float L = 0.f;
        if (M != -INFINITY)
            for (int w = 0; w < kCW; ++w) L += wl[w][tid] * ex2(wm[w][tid] - M);
        cmx[tid] = M; csum[tid] = L;
    }
    __syncthreads();
    asm volatile("barrier.cluster.wait.aligned;" ::: "memory");
    // ---- push heads kHPC p .. kHPC p + kHPC - 1 of this CTA's partial (weighted slab sum) to CTA p
    for (int i = tid; i < H * D / 4; i += kCNT) {
        const int h = (4 * i) / D, d = (4 * i) % D;
        const float M = cmx[h];
        float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
        if (M != -INFINITY) {
#pragma unroll
            for (int w = 0; w < kCW; ++w) {
                const float mw = wm[w][h];
                if (mw == -INFINITY) continue;
                const float wt = ex2(mw - M);
                const float4 u = *reinterpret_cast<const float4*>(slabs + w * H * RP + h * RP + d);
                v.x += wt * u.x; v.y += wt * u.y; v.z += wt * u.z; v.w += wt * u.w;
            }
        }
        float* dst = cluster.map_shared_rank(recv_o, h / kHPC) + (rank * kHPC + h % kHPC) * D + d;
        *reinterpret_cast<float4*>(dst) = v;
    }
    if (tid < H) *cluster.map_shared_rank(&recv_ml[rank][tid % kHPC], tid / kHPC) = make_float2(cmx[tid], csum[tid]);
    cluster.sync();                                      // pushes complete and visible; none after it
    // ---- finalize heads kHPC rank .. kHPC rank + kHPC - 1 from this CTA's own memory
    if (tid < kHPC * D) {
        const int hh = tid / D, d = tid % D, h = kHPC * rank + hh;
        float M = -INFINITY;
#pragma unroll
        for (int cc = 0; cc < kCluster; ++cc) M = fmaxf(M, recv_ml[cc][hh].x);
        float L = 0.f;
        if (M != -INFINITY)
#pragma unroll
            for (int cc = 0; cc < kCluster; ++cc) L += recv_ml[cc][hh].y * ex2(recv_ml[cc][hh].x - M);
        const float inv = L > 0.f ? 1.f / L : 0.f;
        float acc = 0.f;
#pragma unroll
        for (int cc = 0; cc < kCluster; ++cc) {
            const float mc = recv_ml[cc][hh].x;
            if (mc != -INFINITY) acc += ex2(mc - M) * inv * recv_o[(cc * kHPC + hh) * D + d];
        }
        a.o[(static_cast<size_t>(row) * H + h) * D + d] = __float2bfloat16_rn(acc);
        if (a.lse && d == 0)
            a.lse[static_cast<size_t>(row) * H + h] = L > 0.f ? (M + log2f(L)) * kLn2 : -INFINITY;
    }
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// One CTA per row over the whole index row: no split partials, no counters.
SparsePlan plan_sparse_single(int idx_stride) {
    SparsePlan pl;
    pl.cluster = false;
    pl.splits = 1;
    pl.chunk = (idx_stride + SUB - 1) / SUB * SUB;
    return pl;
}

template <bool KV8>
size_t smem_bytes(int chunk) {
    using L = Layout<KV8>;
    return 128 + sparse::STAGES * L::STAGE + L::CVT + static_cast<size_t>(chunk) * 4 * (KV8 ? 3 : 1);
}

template <bool KV8>
cudaError_t launch_impl(const SparseArgs& sa, cudaStream_t st) {
    const SparsePlan pl = sa.one_split ? plan_sparse_single(sa.idx_stride) : plan_sparse(sa.rows, sa.idx_stride);
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
    cudaError_t e;
    if (pl.cluster) {
        auto launch = [&](auto shape) -> cudaError_t {
            constexpr int NC = decltype(shape)::kCluster;
            auto kern = sparse_cluster_kernel<KV8, NC>;
            const size_t sm = CLayout<KV8, NC>::BYTES + 128;
            cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                   static_cast<int>(sm));
            if (err != cudaSuccess) return err;
            cudaLaunchConfig_t cfg{};
            cfg.gridDim = dim3(NC, sa.rows);
            cfg.blockDim = dim3(CShape<NC>::kCNT);
            cfg.dynamicSmemBytes = sm;
            cfg.stream = st;
            cudaLaunchAttribute attr[1];
            attr[0].id = cudaLaunchAttributeClusterDimension;
            attr[0].val.clusterDim.x = NC;
            attr[0].val.clusterDim.y = 1;
            attr[0].val.clusterDim.z = 1;
            cfg.attrs = attr;
            cfg.numAttrs = 1;
            return cudaLaunchKernelEx(&cfg, kern, a);
        };
        return sa.rows <= kWideClusterRows ? launch(CShape<8>{}) : launch(CShape<4>{});
    }
    const size_t sm = smem_bytes<KV8>(pl.chunk);
    e = cudaFuncSetAttribute(sparse_kernel<KV8>, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(sm));
    if (e != cudaSuccess) return e;
    sparse_kernel<KV8><<<dim3(pl.splits, sa.rows), NT, sm, st>>>(a);
    return cudaGetLastError();
}

}  // namespace

SparsePlan plan_sparse(int rows, int idx_stride) {
    SparsePlan pl;
    pl.cluster = false;
    // few rows: one cluster of kCluster CTAs per row, merged on chip
    if (rows <= num_sms() && idx_stride <= kClusterEntries) {
        pl.cluster = true;
        pl.splits = rows <= kWideClusterRows ? CShape<8>::kCluster : CShape<4>::kCluster;
        pl.chunk = kClusterEntries / pl.splits;
        return pl;
    }
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
    if (pl.splits == 1 || pl.cluster) return 0;
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
    SparseArgs a = in;
    // the split plan when its partials fit the array, else one CTA per row (no partials)
    a.one_split = kStatusBytes + sparse_ws_bytes(in.rows, in.idx_stride) > kNoAllocScratchBytes;
    if (a.one_split && kStatusBytes > kNoAllocScratchBytes) {
        *too_large = true;
        return cudaSuccess;
    }
    void* base = nullptr;
    cudaError_t e = scratch_address(&base);
    if (e != cudaSuccess) return e;
    // status word and split counters start every call at zero, in stream order (a call
    // that ended early, e.g. after a failed launch, may have left a counter set)
    e = cudaMemsetAsync(base, 0, kStatusBytes, st);
    if (e != cudaSuccess) return e;
    a.status = static_cast<uint32_t*>(base);
    a.ws = static_cast<uint8_t*>(base) + kStatusBytes;
    return launch_sparse(a, st);
}

}  // namespace hs2
