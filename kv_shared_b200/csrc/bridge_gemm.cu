// bridge_gemm.cu -- KV Bridging projection on the fifth-generation tensor cores.
//
// "Xiaomi Unveils HySparse2 Architecture for MiMo-V3", section "Two-Level KV
// Sharing: Enabling Prefill Early Exit": the KV cache of the cross-decoder's
// full-attention layers is generated directly from the self-decoder's hidden
// states, each target layer with its own K/V projection.  Here:
//   [K | V] = hidden [rows x d_model] * W_kv [d_model x 2D],  bf16 in, fp32
//   accumulation, rounded to bf16 and written to cache rows pos0[b] + t.
//
// One CTA computes up to 256 rows x 256 columns (all of K and V for its tokens) as two
// M = 128 halves that share every W_kv tile, so that W_kv (re-read from L2 by every CTA)
// costs half as much traffic per row; the rows are spread evenly over one CTA per SM
// (221 or 222 rows each for the 32768-row agent workload: one wave on every SM):
//   warp 0        TMA producer: two A tiles [128 x 64] (K-major, 128-byte swizzle) and
//                 the B tile [64 x 256] as four [64 x 64] boxes of W_kv, which is
//                 row-major (d_model x 2D) and therefore an MN-major B operand
//   warp 1        allocates 512 TMEM columns; one thread issues tcgen05.mma
//                 (M=128, N=256, K=16, one per half) and commits each stage back
//   warps 2..9    epilogue: tcgen05.ld of the fp32 accumulator rows (warp 2 + 4 h + j
//                 takes half h, TMEM lane quarter (2 + j) % 4), then either bf16
//                 rounding, or -- for an FP8 cache ("Xiaomi unveils HySparse2 ...",
//                 AINews article: the million-token caches are FP8) -- the per-token
//                 e4m3 quantizer of hs2_kv_quantize_fp8 applied to the fp32 row:
//                 amax over the row's 128 K (then V) accumulators, s = amax / 448,
//                 codes = e4m3(x / s) rounded to nearest even and saturated; stores
//                 into the cache rows (and the row scales)
// A 3-stage mbarrier pipeline (64 KB per stage) keeps TMA and MMA overlapped.
#include "common.cuh"
#include "internal.h"
#include "tcgen05.cuh"

namespace hs2 {
namespace {

constexpr int BM = 128;                      // rows of one MMA half
constexpr int MH = 2;                        // halves per CTA
constexpr int BMC = BM * MH;                 // rows per CTA
constexpr int BN = 256;
constexpr int BK = 64;                       // one 128-byte swizzle atom of bf16
constexpr int STAGES = 3;
constexpr int A_BYTES = BM * BK * 2;         // 16 KB per half
constexpr int B_BYTES = BK * BN * 2;         // 32 KB (four 64x64 boxes)
constexpr int STAGE_BYTES = MH * A_BYTES + B_BYTES;
constexpr int NT = 64 + 128 * MH;

struct Params {
    int rows;                                // batch * n
    int n;                                   // tokens per sequence
    int d_model;
    int64_t cap;
    const int32_t* pos0;
    uint8_t* k;                              // [B][cap][128] bf16 or e4m3 codes
    uint8_t* v;
    float* k_scale;                          // [B][cap] (e4m3 only)
    float* v_scale;
    bool kv8;
    uint32_t* status;                        // may be null
};

// 32 fp32 values -> 32 e4m3 codes (x / s, round to nearest even, saturating), as the
// cache quantizer computes them
__device__ __forceinline__ void quant32_e4m3(const uint32_t (&r)[32], float s, uint8_t* dst) {
    uint32_t w[8];
#pragma unroll
    for (int j = 0; j < 32; j += 4) {
        const float y0 = __fdiv_rn(__uint_as_float(r[j + 0]), s), y1 = __fdiv_rn(__uint_as_float(r[j + 1]), s);
        const float y2 = __fdiv_rn(__uint_as_float(r[j + 2]), s), y3 = __fdiv_rn(__uint_as_float(r[j + 3]), s);
        uint16_t lo, hi;
        // the second source operand lands in the low byte
        asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(lo) : "f"(y1), "f"(y0));
        asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(hi) : "f"(y3), "f"(y2));
        w[j / 4] = static_cast<uint32_t>(lo) | (static_cast<uint32_t>(hi) << 16);
    }
    reinterpret_cast<uint4*>(dst)[0] = make_uint4(w[0], w[1], w[2], w[3]);
    reinterpret_cast<uint4*>(dst)[1] = make_uint4(w[4], w[5], w[6], w[7]);
}

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
    return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

__global__ void __launch_bounds__(NT, 1) bridge_kernel(const __grid_constant__ CUtensorMap amap,
                                                      const __grid_constant__ CUtensorMap bmap, Params a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = align1024(smem_raw);
    __shared__ uint64_t full[STAGES], empty[STAGES], acc_ready;
    __shared__ uint32_t tmem_base;
    __shared__ int abort_flag;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // this CTA's rows [m0, m1): the rows spread evenly over the grid (between BM and BMC
    // rows per CTA); a half past m1 still loads and multiplies rows of the next CTA (or
    // zero-filled ones past the end) and stores nothing
    const int m0 = static_cast<int>(static_cast<int64_t>(blockIdx.x) * a.rows / gridDim.x);
    const int m1 = static_cast<int>(static_cast<int64_t>(blockIdx.x + 1) * a.rows / gridDim.x);
    const int nk = a.d_model / BK;
    const int mh = (m0 + BM < m1) ? MH : 1;         // halves holding rows of this CTA

    if (threadIdx.x == 0) {
        prefetch_tmap(&amap);
        prefetch_tmap(&bmap);
        for (int s = 0; s < STAGES; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); }
        mbar_init(&acc_ready, 1);
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
            for (int kb = 0; kb < nk; ++kb) {
                const int s = kb % STAGES;
                if (kb >= STAGES && !mbar_wait(&empty[s], ((kb / STAGES) - 1) & 1, a.status)) {
                    abort_flag = 1;
                    break;
                }
                uint8_t* st = smem + s * STAGE_BYTES;
                mbar_arrive_expect_tx(&full[s], mh * A_BYTES + B_BYTES);
                for (int h = 0; h < mh; ++h) tma_load_2d(st + h * A_BYTES, &amap, &full[s], kb * BK, m0 + h * BM);
#pragma unroll
                for (int nb = 0; nb < BN / 64; ++nb)
                    tma_load_2d(st + MH * A_BYTES + nb * (BK * 128), &bmap, &full[s], nb * 64, kb * BK);
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            constexpr uint32_t idesc = umma::idesc_bf16(BM, BN, false, true);
            bool ok = true;
            for (int kb = 0; kb < nk && ok; ++kb) {
                const int s = kb % STAGES;
                ok = mbar_wait(&full[s], (kb / STAGES) & 1, a.status);
                if (!ok) break;
                umma::fence_after();
                const uint32_t sa = smem_u32(smem + s * STAGE_BYTES);
                const uint32_t sb = sa + MH * A_BYTES;
#pragma unroll
                for (int kk = 0; kk < BK / 16; ++kk) {
                    // B: MN-major; 64-column groups 8 KB apart, 8-row K groups 1 KB apart;
                    // step 16 K-rows = 2 KB
                    const uint64_t bd = umma::sdesc_sw128(sb + kk * 2048, BK * 128, 1024);
                    for (int h = 0; h < mh; ++h) {
                        // A: K-major rows of 128 B; step 16 elements = 32 B inside the atom
                        const uint64_t ad = umma::sdesc_sw128(sa + h * A_BYTES + kk * 32, 16, 1024);
                        umma::mma_bf16_ss(tmem + h * BN, ad, bd, idesc, (kb | kk) != 0);
                    }
                }
                umma::commit(&empty[s]);
            }
            if (!ok) abort_flag = 1;
            umma::commit(&acc_ready);
        }
    } else {
        // epilogue: warp w reads TMEM lanes 32*(w%4) .. +31 of half (w - 2) / 4 = tile rows
        const int q = warp & 3, h = (warp - 2) >> 2;
        const int row = m0 + h * BM + q * 32 + lane;
        const bool ok = mbar_wait(&acc_ready, 0, a.status);
        umma::fence_after();
        int64_t crow = -1;
        if (row < m1) {
            const int b = row / a.n, t = row % a.n;
            const int p0 = a.pos0[b];
            if (p0 < 0 || static_cast<int64_t>(p0) + a.n > a.cap)
                set_status(a.status, HS2_ERR_INDEX);         // destination outside the cache
            else
                crow = static_cast<int64_t>(b) * a.cap + p0 + t;
        }
        const bool store = crow >= 0 && ok;
        const uint32_t trow = tmem + (static_cast<uint32_t>(q * 32) << 16) + h * BN;
        if (!a.kv8) {
#pragma unroll 1
            for (int c = 0; c < BN / 32; ++c) {
                uint32_t r[32];
                umma::tmem_ld32(trow + c * 32, r);
                umma::tmem_ld_wait();
                if (store) {
                    __nv_bfloat16* dst = reinterpret_cast<__nv_bfloat16*>(c < 4 ? a.k : a.v) + crow * 128 + (c & 3) * 32;
#pragma unroll
                    for (int j = 0; j < 32; j += 8) {
                        uint4 pk;
                        pk.x = pack_bf16(__uint_as_float(r[j + 0]), __uint_as_float(r[j + 1]));
                        pk.y = pack_bf16(__uint_as_float(r[j + 2]), __uint_as_float(r[j + 3]));
                        pk.z = pack_bf16(__uint_as_float(r[j + 4]), __uint_as_float(r[j + 5]));
                        pk.w = pack_bf16(__uint_as_float(r[j + 6]), __uint_as_float(r[j + 7]));
                        *reinterpret_cast<uint4*>(dst + j) = pk;
                    }
                }
            }
        } else {
            // K (columns 0..127) then V (128..255): the row's amax from a first read of its
            // 128 accumulators, the codes from a second
#pragma unroll 1
            for (int part = 0; part < 2; ++part) {
                float amax = 0.f;
#pragma unroll 1
                for (int c = 0; c < 4; ++c) {
                    uint32_t r[32];
                    umma::tmem_ld32(trow + (4 * part + c) * 32, r);
                    umma::tmem_ld_wait();
#pragma unroll
                    for (int j = 0; j < 32; ++j) amax = fmaxf(amax, fabsf(__uint_as_float(r[j])));
                }
                const float sc = amax > 0.f ? __fdiv_rn(amax, 448.f) : 1.f;
#pragma unroll 1
                for (int c = 0; c < 4; ++c) {
                    uint32_t r[32];
                    umma::tmem_ld32(trow + (4 * part + c) * 32, r);
                    umma::tmem_ld_wait();
                    if (store) quant32_e4m3(r, sc, (part ? a.v : a.k) + crow * 128 + c * 32);
                }
                if (store) (part ? a.v_scale : a.k_scale)[crow] = sc;
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

cudaError_t launch_bridge(const BridgeArgs& ba, cudaStream_t st) {
    const int rows = ba.batch * ba.n;
    if (rows <= 0) return cudaSuccess;
    CUtensorMap amap, bmap;
    if (!make_tmap_2d(&amap, ba.hidden, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, ba.d_model, rows,
                      static_cast<uint64_t>(ba.d_model) * 2, BK, BM, true))
        return cudaErrorInvalidValue;
    if (!make_tmap_2d(&bmap, ba.w_kv, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, BN, ba.d_model, BN * 2, 64, BK, true))
        return cudaErrorInvalidValue;
    Params a{};
    a.rows = rows; a.n = ba.n; a.d_model = ba.d_model; a.cap = ba.cap; a.pos0 = ba.pos0;
    a.k = static_cast<uint8_t*>(ba.k);
    a.v = static_cast<uint8_t*>(ba.v);
    a.k_scale = ba.k_scale; a.v_scale = ba.v_scale; a.kv8 = ba.kv8;
    a.status = ba.status;
    const size_t smem = 1024 + STAGES * STAGE_BYTES;
    cudaError_t e = cudaFuncSetAttribute(bridge_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    // one CTA per SM when that gives each CTA BM .. BMC rows (the arithmetic intensity sits
    // just under the HBM ridge, so idle SMs cost bandwidth); fewer, fuller CTAs otherwise
    int grid = num_sms();
    if (grid * BMC < rows) grid = (rows + BMC - 1) / BMC;
    if (grid * BM > rows) grid = (rows + BM - 1) / BM;
    bridge_kernel<<<grid, NT, smem, st>>>(amap, bmap, a);
    return cudaGetLastError();
}

}  // namespace hs2
