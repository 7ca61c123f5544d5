// prefill_attn.cu -- full-attention layer of a hybrid block for a chunk of new
// query rows (prefill), with the head-summed key importance, on tcgen05.
//
// Importance of key j for row i = sum over the 16 query heads of
// P_h[i][j] = exp(s_h[i][j] - LSE_h[i]) (the pages leave the rule open: "What
// HySparse2 is actually optimizing", "What is not documented").  The final
// log-sum-exp is needed before any probability is formed, hence two passes
// over the causal key range of each block of 8 query rows:
//
//   pass 1  S = Q K^T with M = 8 rows x 16 heads = 128 (all query heads share the
//           one K/V head, so stacking them in M reuses every K tile 128 times);
//           one thread per (row, head) keeps a running max and sum -> LSE.
//   pass 2  S' = K Q^T (M = 128 keys, N = 128 (row, head)): one thread per key
//           owns all 128 probabilities of its key, so the 16-head sum of the
//           importance is plain register adds.  P goes to shared memory as the
//           MN-major A operand of O += P V (V is MN-major straight from the
//           cache); O stays in tensor memory for the whole key loop.
//
// Roles (320 threads): warp 0 issues TMA loads, one thread of warp 1 issues the
// MMAs (and warp 1 owns the tensor memory), warps 2..9 do the softmax work: two
// warps per tensor-memory lane quarter, each owning 64 of the 128 columns.
// Every wait is bounded; a wait that gives up flags the status word and makes
// all roles leave their loops.
#include "common.cuh"
#include "internal.h"
#include "tcgen05.cuh"

namespace hs2 {
namespace {

constexpr int H = 16;
constexpr int D = 128;
constexpr int ROWS = 8;                         // query rows per CTA
constexpr int MT = ROWS * H;                    // 128 (row, head) pairs
constexpr int KT = 128;                         // keys per tile
constexpr int NT = 320;
constexpr int NSOFT = 256;                      // softmax threads (warps 2..9)
constexpr int TILE_BYTES = KT * D * 2;          // 32 KB: two 128-row x 64-col swizzled boxes
constexpr int BOX_BYTES = TILE_BYTES / 2;

struct Params {
    int B, n_q;
    int64_t cap, max_ctx;
    const int32_t* q_pos0;
    float sc2;                                  // scale * log2(e)
    float* lse2;                                // [B][n_q][H] log2 units (pass 1 out, pass 2 in)
    float* lse_user;                            // [B][n_q][H] natural log or null
    float* scores;                              // [B][n_q][score_ld]
    int64_t score_ld;
    __nv_bfloat16* o;                           // [B][n_q][H][D]
    uint32_t* status;
};

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
    return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

// K-major descriptor of the 16-wide K step kk of a [128 x 128] bf16 tile held as two
// 128 x 64 swizzled boxes
__device__ __forceinline__ uint64_t kmajor_desc(uint32_t base, int kk) {
    return umma::sdesc_sw128(base + (kk >> 2) * BOX_BYTES + (kk & 3) * 32, 16, 1024);
}

// MN-major descriptor of the 16-row K step kk of a [128 (K) x 128 (MN)] tile held as two
// [128 x 64] swizzled boxes (MN groups of 64 one box apart)
__device__ __forceinline__ uint64_t mnmajor_desc(uint32_t base, int kk) {
    return umma::sdesc_sw128(base + kk * 2048, BOX_BYTES, 1024);
}

__device__ __forceinline__ bool wait_or_abort(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                              uint32_t* status) {
    if (*abort_flag) return false;
    if (!mbar_wait(bar, parity, status)) { *abort_flag = 1; return false; }
    return true;
}

__device__ __forceinline__ void named_sync(int id, int n) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}

// Tensor-memory S buffers: three 128-column tiles in flight, so that the MMA can
// run ahead while the two softmax warpgroups each work on their own key tile.
constexpr int NSB = 3;

// ------------------------------------------------------------------ pass 1: LSE
constexpr int P1_STAGES = 4;

__global__ void __launch_bounds__(NT, 1) prefill_lse_kernel(const __grid_constant__ CUtensorMap qmap,
                                                           const __grid_constant__ CUtensorMap kmap, Params a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = align1024(smem_raw);
    uint8_t* qs = smem;
    uint8_t* ks = smem + TILE_BYTES;
    __shared__ uint64_t q_full, k_full[P1_STAGES], k_empty[P1_STAGES], s_full[NSB], s_empty[NSB];
    __shared__ uint32_t tmem_base;
    __shared__ volatile int abort_flag;
    __shared__ float2 part[2][MT];

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int blocks_per_seq = (a.n_q + ROWS - 1) / ROWS;
    const int b = blockIdx.x / blocks_per_seq;
    const int r0 = (blockIdx.x % blocks_per_seq) * ROWS;
    const int pos_base = a.q_pos0[b] + r0;
    const int last_row = min(r0 + ROWS, a.n_q) - 1;
    const int p_max = checked_pos(a.q_pos0[b] + last_row, a.max_ctx, a.status);
    const int n_kt = (p_max + KT) / KT;

    if (threadIdx.x == 0) {
        prefetch_tmap(&qmap);
        prefetch_tmap(&kmap);
        mbar_init(&q_full, 1);
        for (int s = 0; s < P1_STAGES; ++s) { mbar_init(&k_full[s], 1); mbar_init(&k_empty[s], 1); }
        for (int s = 0; s < NSB; ++s) { mbar_init(&s_full[s], 1); mbar_init(&s_empty[s], 128); }
        fence_mbar_init();
        abort_flag = 0;
    }
    if (warp == 1) umma::tmem_alloc(&tmem_base, 512);
    umma::fence_before();
    __syncthreads();
    umma::fence_after();
    const uint32_t tmem = tmem_base;

    if (warp == 0) {
        if (lane == 0) {
            const int qrow = (b * a.n_q + r0) * H;
            mbar_arrive_expect_tx(&q_full, TILE_BYTES);
            tma_load_2d(qs, &qmap, &q_full, 0, qrow);
            tma_load_2d(qs + BOX_BYTES, &qmap, &q_full, 64, qrow);
            for (int i = 0; i < n_kt; ++i) {
                const int s = i % P1_STAGES;
                if (i >= P1_STAGES && !wait_or_abort(&k_empty[s], ((i / P1_STAGES) - 1) & 1, &abort_flag, a.status)) break;
                uint8_t* dst = ks + s * TILE_BYTES;
                const int krow = static_cast<int>(b * a.cap) + i * KT;
                mbar_arrive_expect_tx(&k_full[s], TILE_BYTES);
                tma_load_2d(dst, &kmap, &k_full[s], 0, krow);
                tma_load_2d(dst + BOX_BYTES, &kmap, &k_full[s], 64, krow);
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            constexpr uint32_t idesc = umma::idesc_bf16(128, 128, false, false);
            const uint32_t qb = smem_u32(qs);
            if (wait_or_abort(&q_full, 0, &abort_flag, a.status)) {
                for (int i = 0; i < n_kt; ++i) {
                    const int s = i % P1_STAGES, sb = i % NSB;
                    if (!wait_or_abort(&k_full[s], (i / P1_STAGES) & 1, &abort_flag, a.status)) break;
                    if (i >= NSB && !wait_or_abort(&s_empty[sb], ((i / NSB) - 1) & 1, &abort_flag, a.status)) break;
                    umma::fence_after();
                    const uint32_t kb = smem_u32(ks + s * TILE_BYTES);
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk)
                        umma::mma_bf16_ss(tmem + sb * 128, kmajor_desc(qb, kk), kmajor_desc(kb, kk), idesc, kk > 0);
                    umma::commit(&k_empty[s]);
                    umma::commit(&s_full[sb]);
                }
            }
        }
    } else {
        // softmax warpgroup g takes key tiles i = g, g+2, ...; each thread owns TMEM lane
        // m = (row, head) and all 128 columns of a tile, read in 32-column chunks with the
        // next chunk's load in flight while the current one is reduced
        const int quarter = warp & 3, g = (warp - 2) >> 2;
        const int m = quarter * 32 + lane;
        const int row = r0 + (m >> 4);
        const int p = pos_base + (m >> 4);
        const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
        float run_m = -INFINITY, run_l = 0.f;
        auto reduce_chunk = [&](const uint32_t (&r)[32], int key0) {
            float v[32];
            float mx = -INFINITY;
            const bool need_mask = key0 + 31 > p;
#pragma unroll
            for (int c = 0; c < 32; ++c) {
                float x = __uint_as_float(r[c]) * a.sc2;
                if (need_mask && key0 + c > p) x = -INFINITY;
                v[c] = x;
                mx = fmaxf(mx, x);
            }
            const float mn = fmaxf(run_m, mx);
            if (mn != -INFINITY) {
                float s0 = 0.f, s1 = 0.f, s2 = 0.f, s3 = 0.f;
#pragma unroll
                for (int c = 0; c < 32; c += 4) {
                    s0 += ex2(v[c] - mn);
                    s1 += ex2(v[c + 1] - mn);
                    s2 += ex2(v[c + 2] - mn);
                    s3 += ex2(v[c + 3] - mn);
                }
                run_l = run_l * ex2(run_m - mn) + ((s0 + s1) + (s2 + s3));
                run_m = mn;
            }
        };
        for (int i = g; i < n_kt; i += 2) {
            const int sb = i % NSB;
            if (!wait_or_abort(&s_full[sb], (i / NSB) & 1, &abort_flag, a.status)) break;
            umma::fence_after();
            const uint32_t ta = tmem + lane_base + sb * 128;
            const int key0 = i * KT;
            uint32_t ra[32], rb[32];
            umma::tmem_ld32(ta, ra);
            umma::tmem_ld_wait();
            umma::tmem_ld32(ta + 32, rb);
            reduce_chunk(ra, key0);
            umma::tmem_ld_wait();
            umma::tmem_ld32(ta + 64, ra);
            reduce_chunk(rb, key0 + 32);
            umma::tmem_ld_wait();
            umma::tmem_ld32(ta + 96, rb);
            reduce_chunk(ra, key0 + 64);
            umma::tmem_ld_wait();
            umma::fence_before();
            mbar_arrive(&s_empty[sb]);
            reduce_chunk(rb, key0 + 96);
        }
        // combine the two warpgroups' key tiles
        part[g][m] = make_float2(run_m, run_l);
        named_sync(1, NSOFT);
        if (g == 0 && row < a.n_q && !abort_flag) {
            const float2 o = part[1][m];
            const float mn = fmaxf(run_m, o.x);
            const float l = (run_m == -INFINITY ? 0.f : run_l * ex2(run_m - mn)) +
                            (o.x == -INFINITY ? 0.f : o.y * ex2(o.x - mn));
            const float l2 = mn + log2f(l);
            const size_t oi = (static_cast<size_t>(b) * a.n_q + row) * H + (m & 15);
            a.lse2[oi] = l2;
            if (a.lse_user) a.lse_user[oi] = l2 * kLn2;
        }
    }
    umma::fence_before();
    __syncthreads();
    if (warp == 1) {
        umma::fence_after();
        umma::tmem_dealloc(tmem, 512);
    }
}

// One 32-column chunk of an S' row (pass 2): columns = rows 2C, 2C+1 x 16 heads.
// Probabilities P = 2^(S' sc2 - LSE2), the two rows' importance (written to the score
// rows), and bf16 pairs of P into pk[16 C .. 16 C + 15].
template <int C>
__device__ __forceinline__ void p2_chunk(const uint32_t (&r)[32], int key, int pos_base, int r0, int n_q,
                                         float sc2, const float* lse_s, float* srow0, int64_t score_ld,
                                         uint32_t (&pk)[64]) {
#pragma unroll
    for (int rr = 0; rr < 2; ++rr) {
        const int row = 2 * C + rr;
        const bool valid = key <= pos_base + row;
        float acc0 = 0.f, acc1 = 0.f;
#pragma unroll
        for (int h = 0; h < H; h += 2) {
            const int col = rr * H + h;
            const float2 l2 = *reinterpret_cast<const float2*>(&lse_s[C * 32 + col]);
            float p0 = ex2(__uint_as_float(r[col]) * sc2 - l2.x);
            float p1 = ex2(__uint_as_float(r[col + 1]) * sc2 - l2.y);
            if (!valid) { p0 = 0.f; p1 = 0.f; }
            acc0 += p0;
            acc1 += p1;
            pk[C * 16 + (col >> 1)] = pack_bf16(p0, p1);
        }
        if (valid && r0 + row < n_q) srow0[row * score_ld + key] = acc0 + acc1;
    }
}

// ------------------------------------------------------------------ pass 2: P, importance, O
constexpr int P2_STAGES = 2;                    // K and V tiles each double-buffered

__global__ void __launch_bounds__(NT, 1) prefill_out_kernel(const __grid_constant__ CUtensorMap qmap,
                                                           const __grid_constant__ CUtensorMap kmap,
                                                           const __grid_constant__ CUtensorMap vmap, Params a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = align1024(smem_raw);
    uint8_t* qs = smem;
    uint8_t* kst = smem + TILE_BYTES;                         // K stages
    uint8_t* vst = kst + P2_STAGES * TILE_BYTES;              // V stages
    uint8_t* ps = vst + P2_STAGES * TILE_BYTES;               // P tiles (one per warpgroup)
    __shared__ uint64_t q_full, k_full[P2_STAGES], k_empty[P2_STAGES], v_full[P2_STAGES], v_empty[P2_STAGES];
    __shared__ uint64_t s_full[NSB], s_empty[NSB], p_full[2], p_empty[2], o_full;
    __shared__ uint32_t tmem_base;
    __shared__ volatile int abort_flag;
    __shared__ __align__(16) float lse_s[MT];

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int blocks_per_seq = (a.n_q + ROWS - 1) / ROWS;
    const int b = blockIdx.x / blocks_per_seq;
    const int r0 = (blockIdx.x % blocks_per_seq) * ROWS;
    const int pos_base = a.q_pos0[b] + r0;
    const int last_row = min(r0 + ROWS, a.n_q) - 1;
    const int p_max = checked_pos(a.q_pos0[b] + last_row, a.max_ctx, a.status);
    const int n_kt = (p_max + KT) / KT;

    if (threadIdx.x == 0) {
        prefetch_tmap(&qmap);
        prefetch_tmap(&kmap);
        prefetch_tmap(&vmap);
        mbar_init(&q_full, 1);
        for (int s = 0; s < P2_STAGES; ++s) {
            mbar_init(&k_full[s], 1); mbar_init(&k_empty[s], 1);
            mbar_init(&v_full[s], 1); mbar_init(&v_empty[s], 1);
        }
        for (int s = 0; s < NSB; ++s) { mbar_init(&s_full[s], 1); mbar_init(&s_empty[s], 128); }
        for (int s = 0; s < 2; ++s) { mbar_init(&p_full[s], 128); mbar_init(&p_empty[s], 1); }
        mbar_init(&o_full, 1);
        fence_mbar_init();
        abort_flag = 0;
    }
    if (warp == 1) umma::tmem_alloc(&tmem_base, 512);
    umma::fence_before();
    __syncthreads();
    umma::fence_after();
    const uint32_t tmem = tmem_base;            // S' buffers at columns 0, 128, 256; O at 384
    constexpr uint32_t kOcol = NSB * 128;

    if (warp == 0) {
        if (lane == 0) {
            const int qrow = (b * a.n_q + r0) * H;
            mbar_arrive_expect_tx(&q_full, TILE_BYTES);
            tma_load_2d(qs, &qmap, &q_full, 0, qrow);
            tma_load_2d(qs + BOX_BYTES, &qmap, &q_full, 64, qrow);
            // K runs one tile ahead of V: K(t) is needed by S'(t), V(t) only by O after P(t)
            for (int t = 0; t <= n_kt; ++t) {
                if (t < n_kt) {
                    const int s = t % P2_STAGES;
                    if (t >= P2_STAGES && !wait_or_abort(&k_empty[s], ((t / P2_STAGES) - 1) & 1, &abort_flag, a.status)) break;
                    const int krow = static_cast<int>(b * a.cap) + t * KT;
                    mbar_arrive_expect_tx(&k_full[s], TILE_BYTES);
                    tma_load_2d(kst + s * TILE_BYTES, &kmap, &k_full[s], 0, krow);
                    tma_load_2d(kst + s * TILE_BYTES + BOX_BYTES, &kmap, &k_full[s], 64, krow);
                }
                if (t >= 1) {
                    const int j = t - 1, s = j % P2_STAGES;
                    if (j >= P2_STAGES && !wait_or_abort(&v_empty[s], ((j / P2_STAGES) - 1) & 1, &abort_flag, a.status)) break;
                    const int vrow = static_cast<int>(b * a.cap) + j * KT;
                    mbar_arrive_expect_tx(&v_full[s], TILE_BYTES);
                    tma_load_2d(vst + s * TILE_BYTES, &vmap, &v_full[s], 0, vrow);
                    tma_load_2d(vst + s * TILE_BYTES + BOX_BYTES, &vmap, &v_full[s], 64, vrow);
                }
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            constexpr uint32_t idesc_s = umma::idesc_bf16(128, 128, false, false);
            constexpr uint32_t idesc_o = umma::idesc_bf16(128, 128, true, true);
            const uint32_t qb = smem_u32(qs), pb = smem_u32(ps);
            bool ok = wait_or_abort(&q_full, 0, &abort_flag, a.status);
            // S'(i) runs two tiles ahead of O += P(i-2) V(i-2)
            for (int i = 0; ok && i < n_kt + 2; ++i) {
                if (i < n_kt) {                 // S'(i) = K(i) Q^T
                    const int s = i % P2_STAGES, sb = i % NSB;
                    if (!(ok = wait_or_abort(&k_full[s], (i / P2_STAGES) & 1, &abort_flag, a.status))) break;
                    if (i >= NSB && !(ok = wait_or_abort(&s_empty[sb], ((i / NSB) - 1) & 1, &abort_flag, a.status))) break;
                    umma::fence_after();
                    const uint32_t kb = smem_u32(kst + s * TILE_BYTES);
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk)
                        umma::mma_bf16_ss(tmem + sb * 128, kmajor_desc(kb, kk), kmajor_desc(qb, kk), idesc_s, kk > 0);
                    umma::commit(&k_empty[s]);
                    umma::commit(&s_full[sb]);
                }
                if (i >= 2) {                   // O += P(j) V(j), j = i - 2
                    const int j = i - 2, s = j % P2_STAGES, pg = j & 1;
                    if (!(ok = wait_or_abort(&p_full[pg], (j >> 1) & 1, &abort_flag, a.status))) break;
                    if (!(ok = wait_or_abort(&v_full[s], (j / P2_STAGES) & 1, &abort_flag, a.status))) break;
                    umma::fence_after();
                    const uint32_t vb = smem_u32(vst + s * TILE_BYTES);
                    const uint32_t pbj = pb + pg * TILE_BYTES;
#pragma unroll
                    for (int kk = 0; kk < KT / 16; ++kk)
                        umma::mma_bf16_ss(tmem + kOcol, mnmajor_desc(pbj, kk), mnmajor_desc(vb, kk), idesc_o,
                                          (j > 0 || kk > 0) ? 1u : 0u);
                    umma::commit(&p_empty[pg]);
                    umma::commit(&v_empty[s]);
                }
            }
            umma::commit(&o_full);
        }
    } else {
        const int quarter = warp & 3, g = (warp - 2) >> 2;
        const int st = threadIdx.x - 64;        // 0..255
        // log-sum-exp of the 128 (row, head) columns; rows past n_q get +inf (P = 0)
        if (st < MT) {
            const int row = r0 + (st >> 4);
            lse_s[st] = row < a.n_q ? a.lse2[(static_cast<size_t>(b) * a.n_q + row) * H + (st & 15)] : INFINITY;
        }
        named_sync(1, NSOFT);
        const int kl = quarter * 32 + lane;     // the key lane this thread owns in S'
        const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
        float* srow0 = a.scores + (static_cast<size_t>(b) * a.n_q + r0) * a.score_ld;
        uint8_t* pg_tile = ps + g * TILE_BYTES;
        // one 32-column chunk = rows 2c, 2c+1 x 16 heads: probabilities, the two rows'
        // importance, bf16 pairs for the P tile
        uint32_t pk[64];
        for (int i = g; i < n_kt; i += 2) {
            const int sb = i % NSB;
            if (!wait_or_abort(&s_full[sb], (i / NSB) & 1, &abort_flag, a.status)) break;
            umma::fence_after();
            const uint32_t ta = tmem + lane_base + sb * 128;
            const int key = i * KT + kl;
            uint32_t ra[32], rb[32];
            umma::tmem_ld32(ta, ra);
            umma::tmem_ld_wait();
            umma::tmem_ld32(ta + 32, rb);
            p2_chunk<0>(ra, key, pos_base, r0, a.n_q, a.sc2, lse_s, srow0, a.score_ld, pk);
            umma::tmem_ld_wait();
            umma::tmem_ld32(ta + 64, ra);
            p2_chunk<1>(rb, key, pos_base, r0, a.n_q, a.sc2, lse_s, srow0, a.score_ld, pk);
            umma::tmem_ld_wait();
            umma::tmem_ld32(ta + 96, rb);
            p2_chunk<2>(ra, key, pos_base, r0, a.n_q, a.sc2, lse_s, srow0, a.score_ld, pk);
            umma::tmem_ld_wait();
            umma::fence_before();
            mbar_arrive(&s_empty[sb]);
            p2_chunk<3>(rb, key, pos_base, r0, a.n_q, a.sc2, lse_s, srow0, a.score_ld, pk);
            // last tile: cache rows past the last query position may hold anything, and
            // 0 * NaN would poison O, so this key's V row is zeroed (the K row only feeds
            // probabilities that are forced to 0 above).  V(i) is resident: S'(i) was
            // computed, and V(i) is loaded before K(i + 1).
            if (i == n_kt - 1 && key > p_max) {
                if (!wait_or_abort(&v_full[i % P2_STAGES], (i / P2_STAGES) & 1, &abort_flag, a.status)) break;
                uint8_t* vrow = vst + (i % P2_STAGES) * TILE_BYTES + kl * 128;
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    *reinterpret_cast<uint4*>(vrow + c * 16) = make_uint4(0, 0, 0, 0);
                    *reinterpret_cast<uint4*>(vrow + BOX_BYTES + c * 16) = make_uint4(0, 0, 0, 0);
                }
            }
            // this warpgroup's P tile is free once O += P(i-2) V(i-2) has completed
            if (i >= 2 && !wait_or_abort(&p_empty[g], ((i >> 1) - 1) & 1, &abort_flag, a.status)) break;
            // row `kl` of the MN-major P tile: m = (row, head) 0..127 in two 64-wide groups
            uint8_t* prow = pg_tile + (kl >> 3) * 1024 + (kl & 7) * 128;
#pragma unroll
            for (int cc = 0; cc < 16; ++cc) {
                const uint4 w = make_uint4(pk[4 * cc], pk[4 * cc + 1], pk[4 * cc + 2], pk[4 * cc + 3]);
                *reinterpret_cast<uint4*>(prow + (cc >> 3) * BOX_BYTES + (((cc & 7) ^ (kl & 7)) << 4)) = w;
            }
            umma::fence_proxy_async();
            mbar_arrive(&p_full[g]);
        }
        // O epilogue: this thread owns TMEM lane m = (row, head) of the O accumulator and
        // columns 64 g .. 64 g + 63
        if (wait_or_abort(&o_full, 0, &abort_flag, a.status)) {
            umma::fence_after();
            const int m = quarter * 32 + lane;
            const int row = r0 + (m >> 4);
            __nv_bfloat16* orow = a.o + ((static_cast<size_t>(b) * a.n_q + row) * H + (m & 15)) * D + g * 64;
#pragma unroll 1
            for (int c = 0; c < 64; c += 32) {
                uint32_t r[32];
                umma::tmem_ld32(tmem + lane_base + kOcol + g * 64 + c, r);
                umma::tmem_ld_wait();
                if (row < a.n_q) {
#pragma unroll
                    for (int j = 0; j < 32; j += 8) {
                        uint4 w;
                        w.x = pack_bf16(__uint_as_float(r[j]), __uint_as_float(r[j + 1]));
                        w.y = pack_bf16(__uint_as_float(r[j + 2]), __uint_as_float(r[j + 3]));
                        w.z = pack_bf16(__uint_as_float(r[j + 4]), __uint_as_float(r[j + 5]));
                        w.w = pack_bf16(__uint_as_float(r[j + 6]), __uint_as_float(r[j + 7]));
                        *reinterpret_cast<uint4*>(orow + c + j) = w;
                    }
                }
            }
        }
    }
    umma::fence_before();
    __syncthreads();
    if (warp == 1) {
        umma::fence_after();
        umma::tmem_dealloc(tmem, 512);
    }
}

}  // namespace

size_t prefill_ws_bytes(int batch, int n_q) {
    return (sizeof(float) * static_cast<size_t>(batch) * n_q * H + 255) & ~size_t(255);
}

cudaError_t launch_prefill_full(const PrefillArgs& pa, cudaStream_t st) {
    const int rows = pa.batch * pa.n_q;
    if (rows <= 0) return cudaSuccess;
    CUtensorMap qmap, kmap, vmap;
    const uint64_t kv_rows = static_cast<uint64_t>(pa.batch) * pa.cap;
    if (!make_tmap_2d(&qmap, pa.q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, D, static_cast<uint64_t>(rows) * H, D * 2, 64, 128, true) ||
        !make_tmap_2d(&kmap, pa.k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, D, kv_rows, D * 2, 64, KT, true) ||
        !make_tmap_2d(&vmap, pa.v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, D, kv_rows, D * 2, 64, KT, true))
        return cudaErrorInvalidValue;
    Params a{};
    a.B = pa.batch; a.n_q = pa.n_q; a.cap = pa.cap; a.max_ctx = pa.max_ctx; a.q_pos0 = pa.q_pos0;
    a.sc2 = pa.scale * kLog2e;
    a.lse2 = static_cast<float*>(pa.ws);
    a.lse_user = pa.lse;
    a.scores = pa.scores; a.score_ld = pa.score_ld;
    a.o = static_cast<__nv_bfloat16*>(pa.o);
    a.status = pa.status;
    const int blocks = pa.batch * ((pa.n_q + ROWS - 1) / ROWS);
    const size_t s1 = 1024 + TILE_BYTES + P1_STAGES * TILE_BYTES;
    const size_t s2 = 1024 + TILE_BYTES + 2 * P2_STAGES * TILE_BYTES + 2 * TILE_BYTES;
    cudaError_t e = cudaFuncSetAttribute(prefill_lse_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(s1));
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(prefill_out_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(s2));
    if (e != cudaSuccess) return e;
    prefill_lse_kernel<<<blocks, NT, s1, st>>>(qmap, kmap, a);
    prefill_out_kernel<<<blocks, NT, s2, st>>>(qmap, kmap, vmap, a);
    return cudaGetLastError();
}

}  // namespace hs2
