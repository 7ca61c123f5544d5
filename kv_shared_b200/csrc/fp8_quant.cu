// fp8_quant.cu -- per-token e4m3 cache quantizer.
//
// "Xiaomi unveils HySparse2, reducing million-token prefill compute to about
// one-fifth of the baseline": the one-million-token figures use FP8 caches.  The
// format is not given; this library stores e4m3 codes with one fp32 scale per
// cache row: s = amax / 448 (IEEE fp32 division, s = 1 for an all-zero row) and
// code = e4m3(x / s) rounded to nearest even, saturating to +-448.  One warp per
// row of head_dim values.
#include "common.cuh"
#include "internal.h"

namespace hs2 {
namespace {

template <int D>
__global__ void __launch_bounds__(256) fp8_quant_kernel(const float* __restrict__ src, int64_t rows,
                                                        uint8_t* __restrict__ codes, float* __restrict__ scales) {
    constexpr int PER = D / 32;                     // values per lane (2 or 4)
    const int64_t row = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (row >= rows) return;
    const float* x = src + row * D + lane * PER;
    float v[PER];
#pragma unroll
    for (int i = 0; i < PER; ++i) v[i] = x[i];
    float amax = 0.f;
#pragma unroll
    for (int i = 0; i < PER; ++i) amax = fmaxf(amax, fabsf(v[i]));
    amax = warp_max(amax);
    const float s = amax > 0.f ? __fdiv_rn(amax, 448.f) : 1.f;
    uint16_t pk[PER / 2];
#pragma unroll
    for (int i = 0; i < PER / 2; ++i) {
        const float y0 = __fdiv_rn(v[2 * i], s), y1 = __fdiv_rn(v[2 * i + 1], s);
        // the second source operand lands in the low byte
        asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(pk[i]) : "f"(y1), "f"(y0));
    }
    uint8_t* c = codes + row * D + lane * PER;
    if (PER == 4) {
        *reinterpret_cast<uint32_t*>(c) = static_cast<uint32_t>(pk[0]) | (static_cast<uint32_t>(pk[PER / 2 - 1]) << 16);
    } else {
        *reinterpret_cast<uint16_t*>(c) = pk[0];
    }
    if (lane == 0) scales[row] = s;
}

}  // namespace

cudaError_t launch_fp8_quantize(const float* src, int64_t rows, int head_dim, uint8_t* codes,
                                float* scales, cudaStream_t st) {
    if (rows <= 0) return cudaSuccess;
    const dim3 grid(static_cast<unsigned>((rows + 7) / 8));
    if (head_dim == 128) fp8_quant_kernel<128><<<grid, 256, 0, st>>>(src, rows, codes, scales);
    else fp8_quant_kernel<64><<<grid, 256, 0, st>>>(src, rows, codes, scales);
    return cudaGetLastError();
}

}  // namespace hs2
