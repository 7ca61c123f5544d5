// e4m3_mma.cuh -- attention on e4m3 K/V rows without a conversion pass: f16
// mma.sync tiles fed straight from the rows as they sit in shared memory (rows of
// 128 B, the 16-byte chunk index XOR-ed by row % 8, the layout a TMA load with
// 128-byte swizzle writes); e4m3 -> f16 is exact, one cvt per pair.  Used by the
// decode passes (TMA tiles) and by the decode sparse layer (gathered rows).
#pragma once

#include "common.cuh"

namespace hs2 {

constexpr int kE4D = 128;          // head dimension of these tiles

// f16 A-fragments of Q for keys from e4m3 tiles.  Within each 16-dim step the k order is
// permuted so that the 4 consecutive dims 4t .. 4t+3 that ldmatrix gives a thread of a key
// (two b16 units = four e4m3 bytes) form its B registers: k = 2t, 2t+1 <-> dims 4t, 4t+1 and
// k = 2t+8, 2t+9 <-> dims 4t+2, 4t+3.  Q is scaled by 2^-e (e > 0 only if max |q| >= 2^14)
// to fit f16; returns 2^e.  Every warp loads all of Q, so all warps find the same e.
__device__ __forceinline__ float load_q_frags_e4m3(const __nv_bfloat16* qb, int g, int t, uint32_t (&qa)[8][4]) {
    uint2 raw[8][2];
    float mx = 0.f;
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
        raw[ks][0] = __ldg(reinterpret_cast<const uint2*>(qb + g * kE4D + 16 * ks + 4 * t));
        raw[ks][1] = __ldg(reinterpret_cast<const uint2*>(qb + (g + 8) * kE4D + 16 * ks + 4 * t));
#pragma unroll
        for (int r = 0; r < 2; ++r) {
            const float2 x = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&raw[ks][r].x));
            const float2 y = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&raw[ks][r].y));
            mx = fmaxf(mx, fmaxf(fmaxf(fabsf(x.x), fabsf(x.y)), fmaxf(fabsf(y.x), fabsf(y.y))));
        }
    }
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
    int e = 0;
    if (mx >= 16384.f) {
        int ex;
        frexpf(mx, &ex);                        // mx < 2^ex
        e = ex - 14;
    }
    const float s = ldexpf(1.f, -e);
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
        uint32_t v[2][2];
#pragma unroll
        for (int r = 0; r < 2; ++r) {
            const float2 x = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&raw[ks][r].x));
            const float2 y = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&raw[ks][r].y));
            v[r][0] = pack_f16(x.x * s, x.y * s);    // dims 4t, 4t+1
            v[r][1] = pack_f16(y.x * s, y.y * s);    // dims 4t+2, 4t+3
        }
        qa[ks][0] = v[0][0];        // row g,     k = 2t, 2t+1
        qa[ks][1] = v[1][0];        // row g + 8
        qa[ks][2] = v[0][1];        // row g,     k = 2t+8, 2t+9
        qa[ks][3] = v[1][1];        // row g + 8
    }
    return ldexpf(1.f, e);
}

// S for 16 heads x this warp's 16 keys (rows row0 .. row0 + 15 of the tile at shared address
// tbase): two n-tiles of 8 keys, 8 k-steps each, K fragments by ldmatrix of the raw tile.
__device__ __forceinline__ void qk_e4m3(uint32_t tbase, int row0, const uint32_t (&qa)[8][4], float (&acc)[2][4],
                                        int lane) {
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[nt][e] = 0.f;
        const int r = row0 + nt * 8 + (lane & 7);
#pragma unroll
        for (int half = 0; half < 2; ++half) {
            const int chunk = 4 * half + (lane >> 3);
            uint32_t k[4];
            ldsm_x4(tbase + r * 128 + ((chunk ^ (r & 7)) << 4), k[0], k[1], k[2], k[3]);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                uint32_t b0, b1;
                e4m3x4_to_f16x2x2(k[j], b0, b1);
                mma_f16(acc[nt], qa[4 * half + j], b0, b1);
            }
        }
    }
}

// O += P V for this warp's 16 keys (rows row0 .. row0 + 15 of the tile at tbase).  ldmatrix
// .trans on b16 units (two dims) gives a thread keys 2t, 2t+1 (and 2t+8, 2t+9) of dims 2g,
// 2g+1 of a 16-dim chunk; a byte permute regroups them into one f16 pair of keys per dim.
// Accumulator o[4 G + 2 h + p] then holds dims 32 G + 16 h + 4 t + p (c0, c2) and that + 2
// (c1, c3), rows g and g + 8.
__device__ __forceinline__ void pv_e4m3(uint32_t tbase, int row0, const uint32_t (&pa)[4], float (&o)[16][4],
                                        int lane) {
    const int j = lane >> 3;
    const int r = row0 + (j & 1) * 8 + (lane & 7);
#pragma unroll
    for (int G = 0; G < 4; ++G) {
        const int chunk = 2 * G + (j >> 1);
        uint32_t v[4];
        ldsm_x4_t(tbase + r * 128 + ((chunk ^ (r & 7)) << 4), v[0], v[1], v[2], v[3]);
#pragma unroll
        for (int hs = 0; hs < 2; ++hs) {
            uint32_t e0, o0, e1, o1;
            e4m3x4_to_f16x2x2(prmt(v[2 * hs], 0u, 0x3120u), e0, o0);        // keys 2t, 2t+1
            e4m3x4_to_f16x2x2(prmt(v[2 * hs + 1], 0u, 0x3120u), e1, o1);    // keys 2t+8, 2t+9
            mma_f16(o[4 * G + 2 * hs], pa, e0, e1);
            mma_f16(o[4 * G + 2 * hs + 1], pa, o0, o1);
        }
    }
}

}  // namespace hs2
