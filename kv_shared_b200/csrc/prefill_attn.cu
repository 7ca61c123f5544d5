// prefill_attn.cu -- full-attention layer of a hybrid block for a chunk of new
// query rows (prefill), with the head-summed key importance, on tcgen05.
//
// Importance of key j for row i = sum over the 16 query heads of
// P_h[i][j] = exp(s_h[i][j] - LSE_h[i]) (the pages leave the rule open: "What
// HySparse2 is actually optimizing", "What is not documented").  The final
// log-sum-exp is needed before any probability is formed, hence two passes
// over the causal key range of each block of 16 query rows.
//
// All 16 query heads share the one K/V head, so a CTA stacks (row, head) pairs
// in the MMA's M dimension: 16 rows x 16 heads = 256 pairs, as two 128-lane
// halves that both consume every K (and V) tile the CTA loads.  Each tile is
// fetched from L2 once per 256 pairs; with fewer pairs per tile the kernels are
// bound by the L2-to-SM traffic rather than by the tensor or exponential units.
//
//   pass 1  S_h = Q_h K^T per half h; one thread per (row, head) keeps a
//           running max and sum -> LSE.
//   pass 2  S_h = Q_h K^T; P_h = exp2(S_h sc2 - LSE2) is written back into the
//           same tensor-memory columns as packed bf16 and used from there as
//           the A operand of O_h += P_h V, so P never touches shared memory.
//           The importance sums P over the 16 lanes (heads) of each row with a
//           warp-shuffle transpose-reduction.
//
// Roles (576 threads): warp 0 issues TMA loads, one thread of warp 1 issues the
// MMAs (warp 1 owns the tensor memory), warps 2..9 work on half 0 and warps
// 10..17 on half 1, two warps per tensor-memory lane quarter (a warp may only
// touch its quarter, warp % 4), so that four softmax warps per SM sub-partition
// hide the tensor-memory and exponential latencies.  Every wait is bounded; a
// wait that gives up flags the status word and makes all roles leave their loops.
#include "common.cuh"
#include "internal.h"
#include "tcgen05.cuh"

namespace hs2 {
namespace {

constexpr int H = 16;
constexpr int D = 128;
constexpr int ROWS = 16;                        // query rows per CTA
constexpr int HALF_ROWS = ROWS / 2;             // rows per 128-lane half
constexpr int KT = 128;                         // keys per tile
constexpr int NT = 576;
constexpr int NSOFT = 512;                      // softmax threads (warps 2..17)
constexpr int TILE_BYTES = KT * D * 2;          // 32 KB: two 128-row x 64-col swizzled boxes
constexpr int BOX_BYTES = TILE_BYTES / 2;

struct Params {
    int B, n_q;
    int64_t cap, max_ctx;
    const int32_t* q_pos0;
    const void* q;                              // [B][n_q][H][D] bf16 (pass 2 reads it directly)
    float sc2;                                  // scale * log2(e), > 0
    float* lse2;                                // [B][n_q][H] log2 units (pass 1 out, pass 2 in)
    float* lse_user;                            // [B][n_q][H] natural log or null
    float* scores;                              // [B][n_q][score_ld] or null (no importance rows)
    int64_t score_ld;
    __nv_bfloat16* o;                           // [B][n_q][H][D]
    uint32_t* status;
    // streaming selection (pass 2): keys of [0, p - window] whose importance reaches the
    // row's running cutoff bound are appended to the row's candidate list
    int window, budget;
    // e4m3 caches: the kernels read exact bf16 copies of the codes (cap = their padded row
    // count per sequence) and apply these per-token scales in fp32
    const float* ksc;                           // [B][cap] K row scales (0 past max_ctx)
    const float* vsc;                           // [B][cap] V row scales
    uint2* cand;                                // [B*n_q][2][cand_seg] (importance bits, position) or null:
    int64_t cand_seg;                           // one segment per key half of the tiles
    int* cand_cnt;                              // [B*n_q][2] entries appended per segment
    uint32_t* hist;                             // [B*n_q][kImpBins] candidates per importance bin
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

__device__ __forceinline__ void named_sync(int id, int n) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}

__device__ __forceinline__ bool wait_or_abort(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                              uint32_t* status) {
    if (*abort_flag) return false;
    if (!mbar_wait(bar, parity, status)) { *abort_flag = 1; return false; }
    return true;
}

// the MMA issuer's waits: it sits on the critical path of every handoff, so it polls
// without ever being suspended
__device__ __forceinline__ bool spin_or_abort(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                              uint32_t* status) {
    if (*abort_flag) return false;
    if (!mbar_wait_spin(bar, parity, status)) { *abort_flag = 1; return false; }
    return true;
}

// one arrival per warp, after every lane's tensor-memory accesses are ordered before it
__device__ __forceinline__ void warp_arrive(uint64_t* bar) {
    umma::fence_before();
    __syncwarp();
    if ((threadIdx.x & 31) == 0) mbar_arrive(bar);
}

// ---- packed fp32 pairs (one instruction for two lanes of arithmetic on sm_100)
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) {
    uint64_t d;
    asm("{\n\t.reg .b64 ra, rb, rc;\n\t"
        "mov.b64 ra, {%1, %2};\n\tmov.b64 rb, {%3, %4};\n\tmov.b64 rc, {%5, %6};\n\t"
        "fma.rn.f32x2 %0, ra, rb, rc;\n\t}"
        : "=l"(d) : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
    float2 r;
    asm("mov.b64 {%0, %1}, %2;" : "=f"(r.x), "=f"(r.y) : "l"(d));
    return r;
}
__device__ __forceinline__ float2 add2(float2 a, float2 b) {
    uint64_t d;
    asm("{\n\t.reg .b64 ra, rb;\n\t"
        "mov.b64 ra, {%1, %2};\n\tmov.b64 rb, {%3, %4};\n\t"
        "add.rn.f32x2 %0, ra, rb;\n\t}"
        : "=l"(d) : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    float2 r;
    asm("mov.b64 {%0, %1}, %2;" : "=f"(r.x), "=f"(r.y) : "l"(d));
    return r;
}
__device__ __forceinline__ float max3(float a, float b, float c) {
    float d;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}

// 2^x for a pair on the FMA pipe (the exponential unit is the bottleneck of pass 1, so a
// share of the exponentials moves here): x = j + r with j the nearest integer (added to
// and taken back from 1.5 * 2^23, whose ulp is 1) and r in [-1/2, 1/2]; 2^r by a degree-5
// polynomial, the minimax relative-error fit of 2^r on that interval by Lawson's algorithm
// (least squares reweighted by the error until it equioscillates; exp2_poly_fit.py beside
// this package prints the coefficients): max relative error 2.1e-7 in fp32 Horner form,
// like the exponential unit's; 2^j enters through the exponent bits.  x is clamped at -125 so
// that the result stays a normal number (it is then below 2^-124, nothing beside the
// row maximum's 1).
__device__ __forceinline__ float2 exp2_poly2(float2 x) {
    constexpr float kMagic = 12582912.f;                       // 1.5 * 2^23
    x.x = fmaxf(x.x, -125.f);
    x.y = fmaxf(x.y, -125.f);
    const float2 t = add2(x, make_float2(kMagic, kMagic));
    const float2 j = add2(t, make_float2(-kMagic, -kMagic));
    const float2 r = add2(x, make_float2(-j.x, -j.y));
    float2 p = make_float2(1.3276455e-3f, 1.3276455e-3f);
    p = fma2(p, r, make_float2(9.6755400e-3f, 9.6755400e-3f));
    p = fma2(p, r, make_float2(5.5507135e-2f, 5.5507135e-2f));
    p = fma2(p, r, make_float2(2.4022120e-1f, 2.4022120e-1f));
    p = fma2(p, r, make_float2(6.9314694e-1f, 6.9314694e-1f));
    p = fma2(p, r, make_float2(1.0000001f, 1.0000001f));
    return make_float2(__int_as_float(__float_as_int(p.x) + (__float_as_int(t.x) << 23)),
                       __int_as_float(__float_as_int(p.y) + (__float_as_int(t.y) << 23)));
}

// Which groups of 4 of a 32-value chunk take exp2_poly2 in pass 1 (bit g: group g).
constexpr uint32_t kPass1PolyGroups = 0x11;                    // groups 0, 4: 8 of 32 (measured best)

// e4m3 caches: the scales of a tile's 128 keys (K, then V in pass 2) travel through a
// ring of shared-memory slots, written by the producer warp when it issues the tile's
// loads and read by the softmax warps when they process its S.  The producer is at most
// (K stages + 2 S buffers) tiles ahead of the oldest tile still being read, so 8 slots
// never overwrite one in use.
constexpr int SC_SLOTS = 8;

// ------------------------------------------------------------------ pass 1: LSE
constexpr int P1_STAGES = 4;
static_assert(P1_STAGES + 2 < SC_SLOTS, "scale ring shorter than the pass-1 lookahead");

template <bool KV8>
__global__ void __launch_bounds__(NT, 1) prefill_lse_kernel(const __grid_constant__ CUtensorMap qmap,
                                                           const __grid_constant__ CUtensorMap kmap, Params a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = align1024(smem_raw);
    uint8_t* qs = smem;                                       // Q halves 0, 1
    uint8_t* ks = smem + 2 * TILE_BYTES;
    float* ring = reinterpret_cast<float*>(ks + P1_STAGES * TILE_BYTES);   // [SC_SLOTS][KT] (e4m3)
    __shared__ uint64_t q_full, k_full[P1_STAGES], k_empty[P1_STAGES], s_full[2][2], s_empty[2][2];
    __shared__ uint64_t sc_full[SC_SLOTS];
    __shared__ uint32_t tmem_base;
    __shared__ volatile int abort_flag;
    __shared__ float2 part[NSOFT];

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
        for (int s = 0; s < 2; ++s)
            for (int h = 0; h < 2; ++h) { mbar_init(&s_full[s][h], 1); mbar_init(&s_empty[s][h], 8); }
        for (int s = 0; s < SC_SLOTS; ++s) mbar_init(&sc_full[s], 32);
        fence_mbar_init();
        abort_flag = 0;
    }
    if (warp == 1) umma::tmem_alloc(&tmem_base, 512);
    umma::fence_before();
    __syncthreads();
    umma::fence_after();
    const uint32_t tmem = tmem_base;            // S of (buffer u, half h) at column (2u + h) * 128

    if (warp == 0) {
        if (KV8 || lane == 0) {
            if (lane == 0) {
                const int qrow = (b * a.n_q + r0) * H;
                mbar_arrive_expect_tx(&q_full, 2 * TILE_BYTES);
                for (int h = 0; h < 2; ++h) {
                    tma_load_2d(qs + h * TILE_BYTES, &qmap, &q_full, 0, qrow + h * 128);
                    tma_load_2d(qs + h * TILE_BYTES + BOX_BYTES, &qmap, &q_full, 64, qrow + h * 128);
                }
            }
            for (int i = 0; i < n_kt; ++i) {
                const int s = i % P1_STAGES;
                bool ok = true;
                if (lane == 0 && i >= P1_STAGES)
                    ok = wait_or_abort(&k_empty[s], ((i / P1_STAGES) - 1) & 1, &abort_flag, a.status);
                if (KV8) ok = __shfl_sync(0xffffffffu, ok, 0);
                if (!ok) break;
                const int krow = static_cast<int>(b * a.cap) + i * KT;
                if (lane == 0) {
                    uint8_t* dst = ks + s * TILE_BYTES;
                    mbar_arrive_expect_tx(&k_full[s], TILE_BYTES);
                    tma_load_2d(dst, &kmap, &k_full[s], 0, krow);
                    tma_load_2d(dst + BOX_BYTES, &kmap, &k_full[s], 64, krow);
                }
                if (KV8) {      // the tile's 128 key scales into ring slot i % SC_SLOTS, asynchronously:
                                // each lane's copy arrives on the slot's barrier when it lands
                    cp_async16(ring + (i % SC_SLOTS) * KT + 4 * lane, a.ksc + krow + 4 * lane);
                    cp_async_arrive_noinc(&sc_full[i % SC_SLOTS]);
                }
            }
            if (KV8) asm volatile("cp.async.wait_all;" ::: "memory");   // no copy in flight when the CTA leaves
        }
    } else if (warp == 1) {
        if (lane == 0) {
            constexpr uint32_t idesc = umma::idesc_bf16(128, 128, false, false);
            const uint32_t qb = smem_u32(qs);
            bool ok = spin_or_abort(&q_full, 0, &abort_flag, a.status);
            for (int i = 0; ok && i < n_kt; ++i) {
                const int s = i % P1_STAGES, u = i & 1;
                if (!(ok = spin_or_abort(&k_full[s], (i / P1_STAGES) & 1, &abort_flag, a.status))) break;
                const uint32_t kb = smem_u32(ks + s * TILE_BYTES);
                for (int h = 0; h < 2; ++h) {
                    if (i >= 2 && !(ok = spin_or_abort(&s_empty[u][h], ((i >> 1) - 1) & 1, &abort_flag, a.status))) break;
                    umma::fence_after();
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk)
                        umma::mma_bf16_ss(tmem + (2 * u + h) * 128, kmajor_desc(qb + h * TILE_BYTES, kk),
                                          kmajor_desc(kb, kk), idesc, kk > 0);
                    umma::commit(&s_full[u][h]);
                }
                umma::commit(&k_empty[s]);
            }
        }
    } else {
        // half h, key-column half c of every tile: each thread owns TMEM lane m =
        // (row, head) of its half and columns 64 c .. 64 c + 63 of each tile, read in two
        // 32-column chunks (the second in flight while the first is reduced); the two
        // column halves' running (max, sum) are merged at the end
        const int sw = warp - 2, quarter = warp & 3;
        const int h = sw >> 3, c = (sw >> 2) & 1;
        const int m = quarter * 32 + lane;
        const int lrow = h * HALF_ROWS + (m >> 4);
        const int row = r0 + lrow;
        const int p = pos_base + lrow;
        const float sc2 = a.sc2;
        const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
        float run_m = -INFINITY, run_l = 0.f;
        // scale > 0, so the row maximum of S sc2 is sc2 times the maximum of S
        auto reduce_chunk = [&](const uint32_t (&r)[32], int key0, const float* kscale) {
            float v[32];
#pragma unroll
            for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(r[j]);
            if (KV8) {          // logit = (q . code) * key scale, exact in the oracle's terms
                const float2 z = make_float2(0.f, 0.f);
#pragma unroll
                for (int j = 0; j < 32; j += 4) {
                    const float4 c = *reinterpret_cast<const float4*>(kscale + j);
                    const float2 p0 = fma2(make_float2(v[j], v[j + 1]), make_float2(c.x, c.y), z);
                    const float2 p1 = fma2(make_float2(v[j + 2], v[j + 3]), make_float2(c.z, c.w), z);
                    v[j] = p0.x; v[j + 1] = p0.y; v[j + 2] = p1.x; v[j + 3] = p1.y;
                }
            }
            if (key0 + 31 > p) {
#pragma unroll
                for (int j = 0; j < 32; ++j)
                    if (key0 + j > p) v[j] = -INFINITY;
            }
            float m0 = max3(v[0], v[1], v[2]), m1 = max3(v[3], v[4], v[5]);
#pragma unroll
            for (int j = 6; j < 30; j += 4) {
                m0 = max3(m0, v[j], v[j + 1]);
                m1 = max3(m1, v[j + 2], v[j + 3]);
            }
            const float mx = max3(m0, m1, fmaxf(v[30], v[31]));
            const float mn = fmaxf(run_m, mx * sc2);
            if (mn != -INFINITY) {
                const float2 s2 = make_float2(sc2, sc2), nm = make_float2(-mn, -mn);
                float2 acc0 = make_float2(0.f, 0.f), acc1 = acc0;
#pragma unroll
                for (int j = 0; j < 32; j += 4) {
                    const float2 x0 = fma2(make_float2(v[j], v[j + 1]), s2, nm);
                    const float2 x1 = fma2(make_float2(v[j + 2], v[j + 3]), s2, nm);
                    if ((kPass1PolyGroups >> (j / 4)) & 1u) {
                        acc0 = add2(acc0, exp2_poly2(x0));
                        acc1 = add2(acc1, exp2_poly2(x1));
                    } else {
                        acc0 = add2(acc0, make_float2(ex2(x0.x), ex2(x0.y)));
                        acc1 = add2(acc1, make_float2(ex2(x1.x), ex2(x1.y)));
                    }
                }
                const float2 acc = add2(acc0, acc1);
                run_l = run_l * ex2(run_m - mn) + (acc.x + acc.y);
                run_m = mn;
            }
        };
        for (int i = 0; i < n_kt; ++i) {
            const int u = i & 1;
            if (!wait_or_abort(&s_full[u][h], (i >> 1) & 1, &abort_flag, a.status)) break;
            if (KV8 && !__all_sync(0xffffffffu, wait_or_abort(&sc_full[i % SC_SLOTS], (i / SC_SLOTS) & 1, &abort_flag,
                                                              a.status)))
                break;
            umma::fence_after();
            const uint32_t ta = tmem + lane_base + (2 * u + h) * 128 + 64 * c;
            const int key0 = i * KT + 64 * c;
            const float* kscale = ring + (i % SC_SLOTS) * KT + 64 * c;
            uint32_t ra[32], rb[32];
            umma::tmem_ld32(ta, ra);
            umma::tmem_ld_wait();
            umma::tmem_ld32(ta + 32, rb);
            reduce_chunk(ra, key0, kscale);
            umma::tmem_ld_wait();
            warp_arrive(&s_empty[u][h]);
            reduce_chunk(rb, key0 + 32, kscale + 32);
        }
        part[sw * 32 + lane] = make_float2(run_m, run_l);
        named_sync(1, NSOFT);
        if (c == 0 && row < a.n_q && !abort_flag) {
            const float2 o = part[(sw + 4) * 32 + lane];          // the other column half, same lane
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

// ------------------------------------------------------------------ pass 2: P, importance, O

// Sum over the 8 lanes that share t % 4 (lane bits 2..4) of eight float2 values, one
// per 16x256b repetition j; afterwards lane t holds in v[0] the sum for repetition t / 4.
__device__ __forceinline__ float2 transpose_reduce8(float2 (&v)[8], int t) {
    const bool b4 = t & 16, b3 = t & 8, b2 = t & 4;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const float2 lo = v[j], hi = v[j + 4];
        const float2 send = b4 ? lo : hi, keep = b4 ? hi : lo;
        v[j] = add2(keep, make_float2(__shfl_xor_sync(0xffffffffu, send.x, 16),
                                      __shfl_xor_sync(0xffffffffu, send.y, 16)));
    }
#pragma unroll
    for (int j = 0; j < 2; ++j) {
        const float2 lo = v[j], hi = v[j + 2];
        const float2 send = b3 ? lo : hi, keep = b3 ? hi : lo;
        v[j] = add2(keep, make_float2(__shfl_xor_sync(0xffffffffu, send.x, 8),
                                      __shfl_xor_sync(0xffffffffu, send.y, 8)));
    }
    const float2 lo = v[0], hi = v[1];
    const float2 send = b2 ? lo : hi, keep = b2 ? hi : lo;
    return add2(keep, make_float2(__shfl_xor_sync(0xffffffffu, send.x, 4),
                                  __shfl_xor_sync(0xffffffffu, send.y, 4)));
}

// One 64-key chunk of one row (16 lanes = the row's 16 heads) of S_h, read with the
// 16x256b shape: thread t holds heads t/4 (A) and t/4 + 8 (B) at keys
// key_base + 8j + 2(t%4) + {0, 1}.  Forms P, writes it back as packed bf16 (16x128b
// shape, key pair -> one column) and leaves in imp[j] the pair's sum over its two heads;
// transpose_reduce8(imp) then gives lane t the row's importance of keys key_base + 2t,
// key_base + 2t + 1.
// e4m3 caches (KV8): S holds q . code; the key pair's scales come from `sc` (K scales of
// the tile at sc[0 .. 127], V scales at sc[128 .. 255], chunk-relative key index), the K
// scale multiplies the logit and the V scale multiplies P before its bf16 rounding for
// O += P V (the importance uses P itself).
template <bool KV8>
__device__ __forceinline__ void p2_chunk(const uint32_t (&r)[32], uint32_t p_taddr, int key_base, int p, float sc2,
                                         float lse_a, float lse_b, float2 (&imp)[8], int t, const float* sc) {
    const float2 s2 = make_float2(sc2, sc2);
    const float2 na = make_float2(-lse_a, -lse_a), nb = make_float2(-lse_b, -lse_b);
    const bool need_mask = key_base + 63 > p;
    uint32_t pk[16];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        float2 c2 = s2, vs = make_float2(1.f, 1.f);
        if (KV8) {
            const float2 k2 = *reinterpret_cast<const float2*>(sc + 8 * j + 2 * (t & 3));
            vs = *reinterpret_cast<const float2*>(sc + KT + 8 * j + 2 * (t & 3));
            c2 = fma2(s2, k2, make_float2(0.f, 0.f));
        }
        const float2 xa = fma2(make_float2(__uint_as_float(r[4 * j]), __uint_as_float(r[4 * j + 1])), c2, na);
        const float2 xb = fma2(make_float2(__uint_as_float(r[4 * j + 2]), __uint_as_float(r[4 * j + 3])), c2, nb);
        float2 pa = make_float2(ex2(xa.x), ex2(xa.y)), pb = make_float2(ex2(xb.x), ex2(xb.y));
        if (need_mask) {
            const int k0 = key_base + 8 * j + 2 * (t & 3);
            if (k0 > p) { pa.x = 0.f; pb.x = 0.f; }
            if (k0 + 1 > p) { pa.y = 0.f; pb.y = 0.f; }
        }
        if (KV8) {
            const float2 z = make_float2(0.f, 0.f);
            const float2 qa = fma2(pa, vs, z), qb = fma2(pb, vs, z);
            pk[2 * j] = pack_bf16(qa.x, qa.y);
            pk[2 * j + 1] = pack_bf16(qb.x, qb.y);
        } else {
            pk[2 * j] = pack_bf16(pa.x, pa.y);
            pk[2 * j + 1] = pack_bf16(pb.x, pb.y);
        }
        imp[j] = add2(pa, pb);
    }
    umma::tmem_st16x128_x8(p_taddr, pk);
}

// Streaming selection state of one query row, in shared memory.  Candidates are the keys
// of [0, p - W] whose importance is at least thr when they appear; thr only rises, and
// only to the floor of a bin at or above which K candidates have already been counted,
// so every key of the row's final top K is a candidate (a key below thr has K better
// ones before it, and the lower position wins ties).  The bins count candidates only:
// every key at or above the current thr is a candidate, so the counts from thr's bin
// up are those of all keys seen.
struct __align__(16) RowSel {
    uint32_t hist[kImpBins];
    float thr;
};

// Appends this warp's candidates among its two keys per lane (positions k, k + 1) to its
// own segment `seg` of the row's list, `count` entries long so far (the same in every lane).
__device__ __forceinline__ void p2_candidates(float2 v, int k, int last_cand, RowSel& rs, uint2* seg, int& count,
                                              int lane) {
    const float th = *reinterpret_cast<volatile float*>(&rs.thr);
    const bool a0 = k <= last_cand && v.x >= th;
    const bool a1 = k + 1 <= last_cand && v.y >= th;
    const uint32_t m0 = __ballot_sync(0xffffffffu, a0), m1 = __ballot_sync(0xffffffffu, a1);
    if ((m0 | m1) == 0u) return;
    const uint32_t lt = (1u << lane) - 1u;
    int off = count + __popc(m0 & lt) + __popc(m1 & lt);
    count += __popc(m0) + __popc(m1);
    if (a0) {
        atomicAdd(&rs.hist[imp_bin(v.x)], 1u);
        seg[off++] = make_uint2(__float_as_uint(v.x), static_cast<uint32_t>(k));
    }
    if (a1) {
        atomicAdd(&rs.hist[imp_bin(v.y)], 1u);
        seg[off] = make_uint2(__float_as_uint(v.y), static_cast<uint32_t>(k + 1));
    }
}

// Raises rs.thr to the floor of the highest bin b with at least K candidates in bins >= b
// (a warp reads the bins while others may still add to them: a stale count is smaller,
// which only lowers the bound).
__device__ __forceinline__ void p2_raise_threshold(RowSel& rs, int K, int lane) {
    uint32_t h[kImpPerLane], mine = 0u;
#pragma unroll
    for (int j = 0; j < kImpPerLane; ++j) {
        h[j] = *reinterpret_cast<volatile uint32_t*>(&rs.hist[kImpPerLane * lane + j]);
        mine += h[j];
    }
    uint32_t above = mine;                                     // suffix sum over lanes >= lane
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_down_sync(0xffffffffu, above, o);
        if (lane + o < 32) above += y;
    }
    uint32_t cum = above - mine;                               // counts of the lanes above
    int best = -1;
#pragma unroll
    for (int j = kImpPerLane - 1; j >= 0; --j) {
        cum += h[j];
        if (best < 0 && cum >= static_cast<uint32_t>(K)) best = kImpPerLane * lane + j;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) best = max(best, __shfl_xor_sync(0xffffffffu, best, o));
    if (lane == 0 && best > 0) {
        const float f = imp_bin_floor(best);
        if (f > rs.thr) *reinterpret_cast<volatile float*>(&rs.thr) = f;
    }
}

// Pass 2 runs 8 query rows (128 (row, head) pairs) per CTA, with the queries in tensor
// memory: both MMAs then read only K or V from shared memory (the tensor core and TMA
// together draw about 77 bytes per cycle from shared memory, which bounds these
// kernels), and tensor memory holds Q, O and two S buffers.  P(i) is written as packed
// bf16 into the S(i) buffer, each softmax warp into the 32 columns at the start of the
// 64 it read, and PV(i) takes it from there as its A operand.  S(i + 2), into the same
// buffer, is issued right after PV(i) by the same thread: the tensor pipe executes one
// thread's MMAs in issue order, so PV(i) has read P before S overwrites it, and the
// softmax writes P(i + 2) only after S(i + 2) has completed, hence after PV(i).
constexpr int ROWS2 = 8;
constexpr int KS2 = 3;                          // K stages of pass 2
constexpr int VS2 = 3;                          // V stages of pass 2
constexpr int NSB2 = 2;                         // S/P buffers at columns 0, 128
constexpr uint32_t kQcol = 256;                 // Q (packed bf16 pairs) at columns 256 .. 319
constexpr uint32_t kOcol = 384;                 // O at columns 384 .. 511
static_assert(KS2 + 2 < SC_SLOTS, "scale ring shorter than the pass-2 lookahead");

template <bool KV8>
__global__ void __launch_bounds__(NT, 1) prefill_out_kernel(const __grid_constant__ CUtensorMap qmap,
                                                           const __grid_constant__ CUtensorMap kmap,
                                                           const __grid_constant__ CUtensorMap vmap, Params a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = align1024(smem_raw);
    uint8_t* kst = smem;                                      // K stages
    uint8_t* vst = kst + KS2 * TILE_BYTES;                    // V stages
    float* ring = reinterpret_cast<float*>(vst + VS2 * TILE_BYTES);   // [SC_SLOTS][2][KT] (e4m3)
    __shared__ uint64_t k_full[KS2], k_empty[KS2], v_full[VS2], v_empty[VS2];
    __shared__ uint64_t sc_full[SC_SLOTS];
    __shared__ uint64_t s_full[NSB2], p_full[NSB2], q_tm, o_full;
    __shared__ uint32_t tmem_base;
    __shared__ volatile int abort_flag;
    __shared__ RowSel rsel[ROWS2];

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int blocks_per_seq = (a.n_q + ROWS2 - 1) / ROWS2;
    const int b = blockIdx.x / blocks_per_seq;
    const int r0 = (blockIdx.x % blocks_per_seq) * ROWS2;
    const int pos_base = a.q_pos0[b] + r0;
    const int last_row = min(r0 + ROWS2, a.n_q) - 1;
    const int p_max = checked_pos(a.q_pos0[b] + last_row, a.max_ctx, a.status);
    const int n_kt = (p_max + KT) / KT;

    if (threadIdx.x == 0) {
        prefetch_tmap(&kmap);
        prefetch_tmap(&vmap);
        for (int s = 0; s < KS2; ++s) { mbar_init(&k_full[s], 1); mbar_init(&k_empty[s], 1); }
        for (int s = 0; s < VS2; ++s) { mbar_init(&v_full[s], 1); mbar_init(&v_empty[s], 1); }
        for (int u = 0; u < NSB2; ++u) { mbar_init(&s_full[u], 1); mbar_init(&p_full[u], 16); }
        mbar_init(&q_tm, 16);
        mbar_init(&o_full, 1);
        for (int s = 0; s < SC_SLOTS; ++s) mbar_init(&sc_full[s], 32);
        fence_mbar_init();
        abort_flag = 0;
    }
    for (int i = threadIdx.x; i < ROWS2 * kImpBins; i += NT) rsel[i / kImpBins].hist[i % kImpBins] = 0u;
    if (threadIdx.x < ROWS2) rsel[threadIdx.x].thr = a.budget > 0 ? 0.f : INFINITY;
    if (warp == 1) umma::tmem_alloc(&tmem_base, 512);
    umma::fence_before();
    __syncthreads();
    umma::fence_after();
    const uint32_t tmem = tmem_base;            // S/P buffers at 0, 128; Q at 256; O at 384

    if (warp == 0) {
        if (KV8 || lane == 0) {
            // K runs one tile ahead of V: K(t) is needed by S(t), V(t) only after P(t)
            for (int t = 0; t <= n_kt; ++t) {
                if (t < n_kt) {
                    const int s = t % KS2;
                    bool ok = true;
                    if (lane == 0 && t >= KS2) ok = wait_or_abort(&k_empty[s], ((t / KS2) - 1) & 1, &abort_flag, a.status);
                    if (KV8) ok = __shfl_sync(0xffffffffu, ok, 0);
                    if (!ok) break;
                    const int krow = static_cast<int>(b * a.cap) + t * KT;
                    if (lane == 0) {
                        mbar_arrive_expect_tx(&k_full[s], TILE_BYTES);
                        tma_load_2d(kst + s * TILE_BYTES, &kmap, &k_full[s], 0, krow);
                        tma_load_2d(kst + s * TILE_BYTES + BOX_BYTES, &kmap, &k_full[s], 64, krow);
                    }
                    if (KV8) {  // the tile's 128 K and 128 V scales into ring slot t % SC_SLOTS,
                                // asynchronously (each lane's copies arrive on the slot's barrier)
                        float* slot = ring + (t % SC_SLOTS) * 2 * KT;
                        cp_async16(slot + 4 * lane, a.ksc + krow + 4 * lane);
                        cp_async16(slot + KT + 4 * lane, a.vsc + krow + 4 * lane);
                        cp_async_arrive_noinc(&sc_full[t % SC_SLOTS]);
                    }
                }
                if (t >= 1) {
                    const int j = t - 1, s = j % VS2;
                    bool ok = true;
                    if (lane == 0 && j >= VS2) ok = wait_or_abort(&v_empty[s], ((j / VS2) - 1) & 1, &abort_flag, a.status);
                    if (KV8) ok = __shfl_sync(0xffffffffu, ok, 0);
                    if (!ok) break;
                    if (lane == 0) {
                        const int vrow = static_cast<int>(b * a.cap) + j * KT;
                        mbar_arrive_expect_tx(&v_full[s], TILE_BYTES);
                        tma_load_2d(vst + s * TILE_BYTES, &vmap, &v_full[s], 0, vrow);
                        tma_load_2d(vst + s * TILE_BYTES + BOX_BYTES, &vmap, &v_full[s], 64, vrow);
                    }
                }
            }
            if (KV8) asm volatile("cp.async.wait_all;" ::: "memory");   // no copy in flight when the CTA leaves
        }
    } else if (warp == 1) {
        if (lane == 0) {
            constexpr uint32_t idesc_s = umma::idesc_bf16(128, 128, false, false);
            constexpr uint32_t idesc_o = umma::idesc_bf16(128, 128, false, true);
            auto issue_s = [&](int t) {                 // S(t) = Q K(t)^T into buffer t % NSB2, Q from tensor memory
                const int s = t % KS2;
                const uint32_t kb = smem_u32(kst + s * TILE_BYTES);
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk)
                    umma::mma_bf16_ts(tmem + (t % NSB2) * 128, tmem + kQcol + kk * 8, kmajor_desc(kb, kk), idesc_s,
                                      kk > 0);
                umma::commit(&s_full[t % NSB2]);
                umma::commit(&k_empty[s]);
            };
            bool ok = spin_or_abort(&q_tm, 0, &abort_flag, a.status);
            for (int t = 0; ok && t < NSB2 && t < n_kt; ++t) {
                if (!(ok = spin_or_abort(&k_full[t % KS2], (t / KS2) & 1, &abort_flag, a.status))) break;
                umma::fence_after();
                issue_s(t);
            }
            for (int i = 0; ok && i < n_kt; ++i) {
                // O += P(i) V(i); P(i) sits in the first 32 columns of each 64-column half of
                // buffer i % NSB2 (keys 0..63, then 64..127)
                const int vs = i % VS2, u = i % NSB2;
                if (!(ok = spin_or_abort(&p_full[u], (i / NSB2) & 1, &abort_flag, a.status))) break;
                if (!(ok = spin_or_abort(&v_full[vs], (i / VS2) & 1, &abort_flag, a.status))) break;
                umma::fence_after();
                const uint32_t vb = smem_u32(vst + vs * TILE_BYTES);
#pragma unroll
                for (int kk = 0; kk < KT / 16; ++kk)
                    umma::mma_bf16_ts(tmem + kOcol, tmem + u * 128 + (kk >> 2) * 64 + (kk & 3) * 8, mnmajor_desc(vb, kk),
                                      idesc_o, (i > 0 || kk > 0) ? 1u : 0u);
                umma::commit(&v_empty[vs]);
                // S(i + 2) into the same buffer, after PV(i) in issue order
                if (i + NSB2 < n_kt) {
                    if (!(ok = spin_or_abort(&k_full[(i + NSB2) % KS2], ((i + NSB2) / KS2) & 1, &abort_flag, a.status)))
                        break;
                    umma::fence_after();
                    issue_s(i + NSB2);
                }
            }
            umma::commit(&o_full);
        }
    } else {
        // 16 warps: warp (quarter, s, kh) owns row 2 quarter + s (TMEM lanes 32 quarter + 16 s,
        // the row's 16 heads) and keys 64 kh .. 64 kh + 63 of every tile
        const int sw = warp - 2, quarter = warp & 3;
        const int s = (sw >> 2) & 1, kh = (sw >> 3) & 1;
        const int lrow = 2 * quarter + s;
        const int row = r0 + lrow;
        const int p = pos_base + lrow;
        const bool row_ok = row < a.n_q;
        const size_t li = (static_cast<size_t>(b) * a.n_q + row) * H;
        const float lse_a = row_ok ? a.lse2[li + (lane >> 2)] : INFINITY;      // P = 0 for rows past n_q
        const float lse_b = row_ok ? a.lse2[li + (lane >> 2) + 8] : INFINITY;
        float* srow = (row_ok && a.scores) ? a.scores + (static_cast<size_t>(b) * a.n_q + row) * a.score_ld : nullptr;
        const bool vec2 = (a.score_ld & 1) == 0;
        const size_t grow = static_cast<size_t>(b) * a.n_q + row;
        uint2* crow = (row_ok && a.cand) ? a.cand + (2 * grow + kh) * a.cand_seg : nullptr;   // this warp's segment
        int ccount = 0;
        const int last_cand = p - a.window;                  // candidates: positions 0 .. p - W
        RowSel& rs = rsel[lrow];
        const float sc2 = a.sc2;
        const uint32_t lanes = static_cast<uint32_t>(32 * quarter + 16 * s) << 16;
        const int vt = sw * 32 + lane;                        // V row this thread clears in the last tile
        // the queries into tensor memory: this thread writes lane m = 32 quarter + lane (pair
        // (row m / 16, head m % 16)), columns kQcol + 16 cg .. + 15 (dims 32 cg .. 32 cg + 31)
        {
            const int m = 32 * quarter + lane, cg = sw >> 2;
            const int qr = r0 + (m >> 4);
            uint32_t qv[16];
            if (qr < a.n_q) {
                const uint4* src = reinterpret_cast<const uint4*>(
                    static_cast<const uint8_t*>(a.q) + ((static_cast<size_t>(b) * a.n_q + qr) * H + (m & 15)) * D * 2 +
                    cg * 64);
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const uint4 v = __ldg(src + j);
                    qv[4 * j] = v.x; qv[4 * j + 1] = v.y; qv[4 * j + 2] = v.z; qv[4 * j + 3] = v.w;
                }
            } else {
#pragma unroll
                for (int j = 0; j < 16; ++j) qv[j] = 0u;
            }
            umma::tmem_st32x16(tmem + (static_cast<uint32_t>(32 * quarter) << 16) + kQcol + 16 * cg, qv);
            umma::tmem_st_wait();
            warp_arrive(&q_tm);
        }
        for (int i = 0; i < n_kt; ++i) {
            const int u = i % NSB2;
            // warp-uniform decision: the tensor-memory accesses below are warp-collective
            if (!__all_sync(0xffffffffu, wait_or_abort(&s_full[u], (i / NSB2) & 1, &abort_flag, a.status))) break;
            umma::fence_after();
            // last tile: cache rows past the last query position may hold anything, and
            // 0 * NaN would poison O, so those V rows are zeroed before P(i) is released
            // (the K rows only feed probabilities that are forced to 0); no early exit, so
            // that every lane reaches the warp's arrival
            if (i == n_kt - 1 && vt < KT && i * KT + vt > p_max &&
                wait_or_abort(&v_full[i % VS2], (i / VS2) & 1, &abort_flag, a.status)) {
                uint8_t* vrow = vst + (i % VS2) * TILE_BYTES + vt * 128;
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    *reinterpret_cast<uint4*>(vrow + c * 16) = make_uint4(0, 0, 0, 0);
                    *reinterpret_cast<uint4*>(vrow + BOX_BYTES + c * 16) = make_uint4(0, 0, 0, 0);
                }
                umma::fence_proxy_async();
            }
            uint32_t r[32];
            float2 imp[8];
            const int key0 = i * KT + 64 * kh;
            const uint32_t ta = tmem + u * 128 + lanes + 64 * kh;     // this warp's 64 S columns
            const float* sc = ring + (i % SC_SLOTS) * 2 * KT + 64 * kh;
            if (KV8 && !__all_sync(0xffffffffu, wait_or_abort(&sc_full[i % SC_SLOTS], (i / SC_SLOTS) & 1, &abort_flag,
                                                              a.status)))
                break;
            umma::tmem_ld16x256_x8(ta, r);
            umma::tmem_ld_wait();
            p2_chunk<KV8>(r, ta, key0, p, sc2, lse_a, lse_b, imp, lane, sc);    // P into the first 32
            umma::tmem_st_wait();
            warp_arrive(&p_full[u]);
            // importance of the row's keys key0 + 2 lane, + 1: reduced and stored after P has
            // been handed to the MMA issuer, off the S -> P -> PV path
            const float2 sv = transpose_reduce8(imp, lane);
            const int k = key0 + 2 * lane;
            if (srow) {
                if (vec2 && k + 1 <= p) {
                    *reinterpret_cast<float2*>(srow + k) = sv;
                } else {
                    if (k <= p) srow[k] = sv.x;
                    if (k + 1 <= p) srow[k + 1] = sv.y;
                }
            }
            if (crow && key0 <= last_cand) {
                p2_candidates(sv, k, last_cand, rs, crow, ccount, lane);
                if (kh == 0 && (i & 3) == 3) p2_raise_threshold(rs, a.budget, lane);
            }
        }
        // the row's candidate count and bins, for the selection kernel
        named_sync(2, NSOFT);
        if (crow) {
            if (kh == 0) {
#pragma unroll
                for (int j = 0; j < kImpPerLane; j += 4)
                    reinterpret_cast<uint4*>(a.hist + grow * kImpBins)[lane * (kImpPerLane / 4) + j / 4] =
                        *reinterpret_cast<const uint4*>(&rs.hist[kImpPerLane * lane + j]);
            }
            if (lane == 0) a.cand_cnt[2 * grow + kh] = ccount;
        }
        // O epilogue: 4 warps per lane quarter; this thread owns TMEM lane m = (row, head)
        // and columns 32 cc .. 32 cc + 31
        if (__all_sync(0xffffffffu, wait_or_abort(&o_full, 0, &abort_flag, a.status))) {
            umma::fence_after();
            const int m = quarter * 32 + lane;
            const int cc = sw >> 2;
            const int orow_i = r0 + (m >> 4);
            uint32_t r[32];
            umma::tmem_ld32(tmem + (static_cast<uint32_t>(quarter * 32) << 16) + kOcol + 32 * cc, r);
            umma::tmem_ld_wait();
            if (orow_i < a.n_q) {
                __nv_bfloat16* orow = a.o + ((static_cast<size_t>(b) * a.n_q + orow_i) * H + (m & 15)) * D + 32 * cc;
#pragma unroll
                for (int j = 0; j < 32; j += 8) {
                    uint4 w;
                    w.x = pack_bf16(__uint_as_float(r[j]), __uint_as_float(r[j + 1]));
                    w.y = pack_bf16(__uint_as_float(r[j + 2]), __uint_as_float(r[j + 3]));
                    w.z = pack_bf16(__uint_as_float(r[j + 4]), __uint_as_float(r[j + 5]));
                    w.w = pack_bf16(__uint_as_float(r[j + 6]), __uint_as_float(r[j + 7]));
                    *reinterpret_cast<uint4*>(orow + j) = w;
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

// e4m3 cache rows 0 .. max_ctx - 1 of every sequence -> exact bf16 copies of their codes,
// [B][capw][128] with capw = max_ctx rounded up to the 128-key tile, zero rows after
// max_ctx; and the row scales copied to [B][capw] (0 after max_ctx), 16-byte aligned per
// tile.  Each thread converts 8 codes.
__global__ void __launch_bounds__(256) widen_e4m3_kernel(const uint8_t* __restrict__ k8, const uint8_t* __restrict__ v8,
                                                         const float* __restrict__ ks, const float* __restrict__ vs,
                                                         int B, int64_t cap, int64_t max_ctx, int64_t capw,
                                                         __nv_bfloat16* __restrict__ kw, __nv_bfloat16* __restrict__ vw,
                                                         float* __restrict__ ksw, float* __restrict__ vsw) {
    const int64_t n = static_cast<int64_t>(B) * capw * 16;
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int64_t row = i >> 4;
        const int c = static_cast<int>(i & 15);
        const int64_t b = row / capw, t = row % capw;
        uint4 ko = make_uint4(0, 0, 0, 0), vo = ko;
        float kscale = 0.f, vscale = 0.f;
        if (t < max_ctx) {
            const int64_t src = (b * cap + t) * D + c * 8;
            const uint2 kc = *reinterpret_cast<const uint2*>(k8 + src);
            const uint2 vc = *reinterpret_cast<const uint2*>(v8 + src);
            ko = make_uint4(e4m3x2_to_bf16x2(kc.x & 0xffff), e4m3x2_to_bf16x2(kc.x >> 16),
                            e4m3x2_to_bf16x2(kc.y & 0xffff), e4m3x2_to_bf16x2(kc.y >> 16));
            vo = make_uint4(e4m3x2_to_bf16x2(vc.x & 0xffff), e4m3x2_to_bf16x2(vc.x >> 16),
                            e4m3x2_to_bf16x2(vc.y & 0xffff), e4m3x2_to_bf16x2(vc.y >> 16));
            if (c == 0) { kscale = ks[b * cap + t]; vscale = vs[b * cap + t]; }
        }
        reinterpret_cast<uint4*>(kw + row * D)[c] = ko;
        reinterpret_cast<uint4*>(vw + row * D)[c] = vo;
        if (c == 0) { ksw[row] = kscale; vsw[row] = vscale; }
    }
}

}  // namespace

namespace {
size_t al256(size_t x) { return (x + 255) & ~size_t(255); }
int64_t widened_rows(int64_t max_ctx) { return (max_ctx + KT - 1) / KT * KT; }
// entries of one warp's candidate segment: the keys of its 64-key half of every tile
int64_t cand_segment(int64_t max_ctx) { return (max_ctx + 1) / 2 + KT / 2; }
}  // namespace

size_t prefill_ws_bytes(int batch, int n_q, int64_t max_ctx, bool fused_select, bool kv8) {
    const size_t rows = static_cast<size_t>(batch) * n_q;
    size_t n = al256(sizeof(float) * rows * H);                               // log-sum-exp (log2)
    if (fused_select)
        n += al256(sizeof(uint32_t) * rows * kImpBins) + al256(sizeof(int) * 2 * rows) +
             al256(sizeof(uint2) * rows * 2 * static_cast<size_t>(cand_segment(max_ctx)));   // bins, counts, lists
    if (kv8) {                                                                // widened K, V and scales
        const size_t wr = static_cast<size_t>(batch) * widened_rows(max_ctx);
        n += 2 * al256(wr * D * 2) + 2 * al256(wr * 4);
    }
    return n;
}

cudaError_t launch_prefill_full(const PrefillArgs& pa, cudaStream_t st) {
    const int rows = pa.batch * pa.n_q;
    if (rows <= 0) return cudaSuccess;
    uint8_t* ws = static_cast<uint8_t*>(pa.ws);
    // e4m3 cache: the tiles come from exact bf16 copies of the codes in the workspace (the
    // end of the prefill region), the scales are applied in the kernels
    const void* kb = pa.k;
    const void* vb = pa.v;
    int64_t cap = pa.cap;
    const float* ksw = nullptr;
    const float* vsw = nullptr;
    cudaError_t e = cudaSuccess;
    if (pa.kv8) {
        const int64_t capw = widened_rows(pa.max_ctx);
        const size_t wr = static_cast<size_t>(pa.batch) * capw;
        uint8_t* w = ws + prefill_ws_bytes(pa.batch, pa.n_q, pa.max_ctx, pa.fused_select, false);
        __nv_bfloat16* kw = reinterpret_cast<__nv_bfloat16*>(w);
        w += al256(wr * D * 2);
        __nv_bfloat16* vw = reinterpret_cast<__nv_bfloat16*>(w);
        w += al256(wr * D * 2);
        float* kscw = reinterpret_cast<float*>(w);
        w += al256(wr * 4);
        float* vscw = reinterpret_cast<float*>(w);
        const int64_t work = static_cast<int64_t>(wr) * 16;
        const int grid = static_cast<int>(work / 256 + 1 < 8 * 148 ? work / 256 + 1 : 8 * 148);
        widen_e4m3_kernel<<<grid, 256, 0, st>>>(static_cast<const uint8_t*>(pa.k), static_cast<const uint8_t*>(pa.v),
                                                pa.k_scale, pa.v_scale, pa.batch, pa.cap, pa.max_ctx, capw, kw, vw,
                                                kscw, vscw);
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
        kb = kw; vb = vw; cap = capw; ksw = kscw; vsw = vscw;
    }
    CUtensorMap qmap, kmap, vmap;
    const uint64_t kv_rows = static_cast<uint64_t>(pa.batch) * cap;
    if (!make_tmap_2d(&qmap, pa.q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, D, static_cast<uint64_t>(rows) * H, D * 2, 64, 128, true) ||
        !make_tmap_2d(&kmap, kb, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, D, kv_rows, D * 2, 64, KT, true) ||
        !make_tmap_2d(&vmap, vb, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, D, kv_rows, D * 2, 64, KT, true))
        return cudaErrorInvalidValue;
    Params a{};
    a.B = pa.batch; a.n_q = pa.n_q; a.cap = cap; a.max_ctx = pa.max_ctx; a.q_pos0 = pa.q_pos0; a.q = pa.q;
    a.ksc = ksw; a.vsc = vsw;
    a.sc2 = pa.scale * kLog2e;
    a.lse2 = reinterpret_cast<float*>(ws);
    ws += al256(sizeof(float) * static_cast<size_t>(rows) * H);
    a.lse_user = pa.lse;
    a.scores = pa.scores; a.score_ld = pa.score_ld;
    a.o = static_cast<__nv_bfloat16*>(pa.o);
    a.status = pa.status;
    a.window = pa.window; a.budget = pa.budget;
    CandSelectArgs cs{};
    if (pa.fused_select) {
        a.hist = reinterpret_cast<uint32_t*>(ws);
        ws += al256(sizeof(uint32_t) * static_cast<size_t>(rows) * kImpBins);
        a.cand_cnt = reinterpret_cast<int*>(ws);
        ws += al256(sizeof(int) * 2 * static_cast<size_t>(rows));
        a.cand = reinterpret_cast<uint2*>(ws);
        a.cand_seg = cand_segment(pa.max_ctx);
        cs.rows = rows; cs.n_q = pa.n_q; cs.q_pos0 = pa.q_pos0; cs.max_ctx = pa.max_ctx;
        cs.window = pa.window; cs.budget = pa.budget; cs.idx_stride = pa.idx_stride;
        cs.hist = a.hist; cs.cand_cnt = a.cand_cnt; cs.cand = a.cand; cs.cand_seg = a.cand_seg;
        cs.idx = pa.idx; cs.cnt = pa.cnt; cs.status = pa.status;
    }
    const int blocks = pa.batch * ((pa.n_q + ROWS - 1) / ROWS);
    const int blocks2 = pa.batch * ((pa.n_q + ROWS2 - 1) / ROWS2);
    const size_t s1 = 1024 + 2 * TILE_BYTES + P1_STAGES * TILE_BYTES + (pa.kv8 ? SC_SLOTS * KT * 4 : 0);
    const size_t s2 = 1024 + (KS2 + VS2) * TILE_BYTES + (pa.kv8 ? SC_SLOTS * 2 * KT * 4 : 0);
    auto k1 = pa.kv8 ? prefill_lse_kernel<true> : prefill_lse_kernel<false>;
    auto k2 = pa.kv8 ? prefill_out_kernel<true> : prefill_out_kernel<false>;
    e = cudaFuncSetAttribute(k1, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(s1));
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(k2, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(s2));
    if (e != cudaSuccess) return e;
    k1<<<blocks, NT, s1, st>>>(qmap, kmap, a);
    k2<<<blocks2, NT, s2, st>>>(qmap, kmap, vmap, a);
    e = cudaGetLastError();
    if (e != cudaSuccess || !pa.fused_select) return e;
    return launch_cand_select(cs, st);
}

}  // namespace hs2
