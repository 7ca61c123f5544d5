// common.cuh -- device helpers shared by the hs2 kernels (sm_100a).
//
// Thin inline-PTX wrappers written from the PTX ISA: mbarrier with bounded
// waits, TMA (cp.async.bulk.tensor) loads, cp.async 16-byte gathers, ldmatrix
// and the bf16 mma.sync tile used by the decode and sparse kernels, plus the
// device status word kept at the start of the caller's workspace.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "../../include/hs2.h"

namespace hs2 {

// ---------------------------------------------------------------- status word
// The first 4 KB of every workspace are the status block: the device status word
// at offset 0 and, from byte 256, the semaphore counters of split-K merges (zero
// when idle: hs2_workspace_init clears the block, the last CTA of a merge resets
// its counter).
constexpr size_t kStatusBytes = 4096;
constexpr int kCounterOffsetInts = 64;
constexpr int kMaxCounters = static_cast<int>(kStatusBytes / 4) - kCounterOffsetInts;

// Bound of every wait on an mbarrier: a phase that has not completed within
// kWaitNs nanoseconds of global time (or kWaitPolls polls) is reported as a
// timeout instead of hanging the GPU.
constexpr uint64_t kWaitNs = 2000000000ull;
constexpr uint32_t kWaitPolls = 1u << 26;

__device__ __forceinline__ uint64_t global_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ void set_status(uint32_t* status, uint32_t code) {
    if (status) atomicCAS(status, 0u, code);
}

// Position of a query row checked against the bound the host sized the launch
// for: an out-of-range position is clamped and reported as HS2_ERR_INDEX.
__device__ __forceinline__ int checked_pos(int p, int64_t max_ctx, uint32_t* status) {
    if (p < 0 || p >= max_ctx) {
        set_status(status, HS2_ERR_INDEX);
        p = p < 0 ? 0 : static_cast<int>(max_ctx - 1);
    }
    return p;
}

// ---------------------------------------------------------------- mbarrier
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;"
                 ::"r"(smem_u32(bar)), "r"(bytes) : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok) : "r"(smem_u32(bar)), "r"(parity) : "memory");
    return ok != 0;
}

// Bounded wait for the phase with the given parity; false (and the status word
// set to HS2_ERR_TIMEOUT) if it did not complete in time.  The clock is read only
// every 64 polls so that a phase completing soon costs nothing but the polls.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, uint32_t* status,
                                          uint64_t limit_ns = kWaitNs) {
#pragma unroll 1
    for (int i = 0; i < 64; ++i)
        if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_ns();
#pragma unroll 1
    for (uint32_t i = 0; i < kWaitPolls; ++i) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((i & 63) == 63 && global_ns() - t0 > limit_ns) break;
    }
    set_status(status, HS2_ERR_TIMEOUT);
    return false;
}

__device__ __forceinline__ bool mbar_test_wait(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok) : "r"(smem_u32(bar)), "r"(parity) : "memory");
    return ok != 0;
}

// As mbar_wait, but polling with the non-blocking test_wait, so that the thread
// never sleeps and reacts to the phase change at once.  For a single thread whose
// reaction time is on the critical path (the MMA issuer).
__device__ __forceinline__ bool mbar_wait_spin(uint64_t* bar, uint32_t parity, uint32_t* status,
                                               uint64_t limit_ns = kWaitNs) {
    const uint64_t t0 = global_ns();
#pragma unroll 1
    for (uint64_t i = 0; i < static_cast<uint64_t>(kWaitPolls) * 64u; ++i) {
        if (mbar_test_wait(bar, parity)) return true;
        if ((i & 255) == 255 && global_ns() - t0 > limit_ns) break;
    }
    set_status(status, HS2_ERR_TIMEOUT);
    return false;
}

// ---------------------------------------------------------------- TMA
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, uint64_t* bar,
                                            int32_t x, int32_t y) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3}], [%4];"
        ::"r"(smem_u32(dst)), "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y),
          "r"(smem_u32(bar))
        : "memory");
}

__device__ __forceinline__ void prefetch_tmap(const CUtensorMap* map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// ---------------------------------------------------------------- cp.async (16 B)
__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;"
                 ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async16_zfill(void* dst, const void* src, bool valid) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;"
                 ::"r"(smem_u32(dst)), "l"(src), "r"(valid ? 16 : 0) : "memory");
}
// 4-byte copy (for 4-byte-aligned sources); zero-filled when !valid
__device__ __forceinline__ void cp_async4_zfill(void* dst, const void* src, bool valid) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;"
                 ::"r"(smem_u32(dst)), "l"(src), "r"(valid ? 4 : 0) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// ---------------------------------------------------------------- ldmatrix / mma
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                        uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                          uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr));
}

// D[16x8] += A[16x16] * B[16x8], bf16 inputs, fp32 accumulators.
__device__ __forceinline__ void mma_bf16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
        "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// D[16x8] += A[16x16] * B[16x8], f16 inputs, fp32 accumulators.
__device__ __forceinline__ void mma_f16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 "
        "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// One arrival on `bar` once every cp.async this thread issued before has landed (the
// barrier's expected count includes it: .noinc).
__device__ __forceinline__ void cp_async_arrive_noinc(uint64_t* bar) {
    asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ uint32_t pack_f16(float lo, float hi) {
    __half2 v = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
}

// Four e4m3 bytes (b0 lowest) -> f16 pairs (b0, b1) and (b2, b3); exact (hardware cvt).
__device__ __forceinline__ void e4m3x4_to_f16x2x2(uint32_t v, uint32_t& lo, uint32_t& hi) {
    asm("{\n\t.reg .b16 l, h;\n\t"
        "mov.b32 {l, h}, %2;\n\t"
        "cvt.rn.f16x2.e4m3x2 %0, l;\n\t"
        "cvt.rn.f16x2.e4m3x2 %1, h;\n\t}"
        : "=r"(lo), "=r"(hi) : "r"(v));
}

// Byte permute: result byte i = byte sel_i of the 8 bytes {b (high), a (low)}.
__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
    uint32_t r;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(sel));
    return r;
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
}

// e4m3 pair (low byte = first element) -> bf16 pair, exact: e4m3 -> f16 is exact
// (hardware cvt), f16 -> f32 -> bf16 is exact for values with <= 4 significant bits.
__device__ __forceinline__ uint32_t e4m3x2_to_bf16x2(uint16_t v) {
    uint32_t h2;
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(v));
    __half2 h = *reinterpret_cast<__half2*>(&h2);
    float2 f = __half22float2(h);
    return pack_bf16(f.x, f.y);
}

// ---------------------------------------------------------------- swizzled tiles
// A tile of R rows x 128 bf16 (256 B per row) is stored as two halves of 64
// columns, each R x 128 B, with the 16-byte chunk index XOR-ed by (row % 8): the
// layout a TMA load with 128-byte swizzle writes for a box of 64 x R (half base
// 1024-byte aligned).  Byte offset of 16-byte chunk c (0..15) of row r:
template <int R>
__device__ __forceinline__ uint32_t swz_off(int r, int c) {
    return (c >> 3) * (R * 128) + r * 128 + (((c & 7) ^ (r & 7)) << 4);
}

// ---------------------------------------------------------------- misc
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// 2^x by the hardware approximation (one MUFU op; subnormal results flush to 0,
// which only affects probabilities below 2^-126).
__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// ---------------------------------------------------------------- importance bins
// Coarse bins of a non-negative fp32 importance value, used to find the selection
// cutoff while the values stream out of the prefill kernel: four bins per octave (the
// exponent and the top two mantissa bits), bin 0 holding everything below 2^-28 (zero
// included), the last bin everything from 2^3.75 up (importance never exceeds the head
// count, 16).  Bins are ordered like the values they hold.  (Eight per octave left 17%
// fewer candidates in the agent prefill, but the wider scans made the call slower.)
constexpr int kImpSub = 2;                                   // mantissa bits in a bin index
constexpr int kImpBins = 32 << kImpSub;                      // 32 octaves
constexpr int kImpPerLane = kImpBins / 32;                   // bins per lane in warp scans
constexpr int kImpBinBase = (127 - 28) << kImpSub;

__device__ __forceinline__ int imp_bin(float v) {
    const int b = static_cast<int>(__float_as_uint(v) >> (23 - kImpSub)) - kImpBinBase;
    return b < 0 ? 0 : (b > kImpBins - 1 ? kImpBins - 1 : b);
}

// smallest value of bin b (0 for bin 0)
__device__ __forceinline__ float imp_bin_floor(int b) {
    return b <= 0 ? 0.f : __uint_as_float(static_cast<uint32_t>(b + kImpBinBase) << (23 - kImpSub));
}

// Bin of a decode row's importance for its selection histogram: the fp32 bit pattern's top
// bits (exponent and kDecHistShift's leading mantissa bits; values are non-negative, so the
// bins order like the values), clamped into the histogram.
constexpr int kDecHistShift = 21;                           // 4 bins per octave
constexpr int kDecHistBins = 1 << (31 - kDecHistShift);     // every non-negative fp32 value
constexpr int kDecFineBits = 11;                            // refinement of a cutoff bin
constexpr int kDecFineBins = 1 << kDecFineBits;
constexpr int kDecFineShift = kDecHistShift - kDecFineBits;
constexpr int kDecHistRow = kDecHistBins + kDecFineBins;    // a row's coarse then fine counts
__device__ __forceinline__ int dec_bin(uint32_t bits) {
    const uint32_t b = bits >> kDecHistShift;
    return b < static_cast<uint32_t>(kDecHistBins) ? static_cast<int>(b) : kDecHistBins - 1;
}

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

}  // namespace hs2
