// cand_select.cu -- token-level top-K + forced window of a prefill row, from the
// candidate list that the full-attention kernel streamed out while it computed the
// row's importance ("Xiaomi Unveils HySparse2 Architecture for MiMo-V3", section
// "Two-Level KV Sharing": the full layer picks the positions the later layers keep
// once it has run; section "Token-Level Sparse Selection": 1,024 global positions
// plus the 128 most recent).
//
// The list of a row holds every key of [0, p - W] that can be among its K best
// (importance desc, position asc) -- and usually few others -- in no particular order,
// with one count per importance bin (see imp_bin).  One CTA per row:
//   1. the bins give the bin b* holding the K-th best candidate and the number A of
//      candidates in higher bins (all selected);
//   2. one pass over the list collects the positions above b* and the (value, position)
//      keys of bin b*;
//   3. the K - A best keys of bin b* (bitonic sort in shared memory; a bin too large
//      for shared memory is resolved by radix digits over the list instead);
//   4. the K positions sorted ascending, then the window [max(0, p-W+1), p], then -1.
// Integer work only: the importance values are compared as their fp32 bit patterns
// (non-negative, so they order as unsigned integers).
#include "common.cuh"
#include "internal.h"

namespace hs2 {
namespace {

constexpr int CNT = 256;
constexpr int kBndCap = 4096;                  // bin-b* keys sorted in shared memory

struct Smem {
    unsigned long long bnd[kBndCap];           // keys of bin b*: (value bits << 32) | ~position
    int sel[kFusedSelectMaxBudget];            // selected positions
    uint32_t hist[kImpBins];
    int rh[256];                               // digit counts (large-bin fallback)
    int nsel, nbnd;
    int bstar, above, need, nb;
    unsigned long long prefix, mask;
    int remaining;
};

__device__ __forceinline__ unsigned long long sel_key(uint2 e) {
    return (static_cast<unsigned long long>(e.x) << 32) | static_cast<uint32_t>(~e.y);
}

__device__ __forceinline__ int key_pos(unsigned long long k) { return static_cast<int>(~static_cast<uint32_t>(k)); }

// In-place bitonic sort of n (a power of two) elements in shared memory, descending when
// `desc`; the whole CTA takes part.
template <typename T>
__device__ void bitonic(T* v, int n, bool desc) {
    for (int k = 2; k <= n; k <<= 1) {
        for (int j = k >> 1; j > 0; j >>= 1) {
            for (int i = threadIdx.x; i < n; i += CNT) {
                const int l = i ^ j;
                if (l > i) {
                    const bool up = ((i & k) == 0) != desc;      // ascending block when up
                    const T a = v[i], b = v[l];
                    if ((a > b) == up) { v[i] = b; v[l] = a; }
                }
            }
            __syncthreads();
        }
    }
}

__global__ void __launch_bounds__(CNT) cand_select_kernel(CandSelectArgs a) {
    extern __shared__ uint8_t smem_raw[];
    Smem& sm = *reinterpret_cast<Smem*>(smem_raw);
    const int row = blockIdx.x, tid = threadIdx.x;
    const int b = row / a.n_q, r = row % a.n_q;
    const int p = checked_pos(a.q_pos0[b] + r, a.max_ctx, a.status);
    const int n_cand = max(0, p - a.window + 1);
    const int kg = min(a.budget, n_cand);              // global picks of this row
    const int nwin = min(p + 1, a.window);

    if (kg > 0) {
        const uint2* list = a.cand + static_cast<size_t>(row) * a.cand_ld;
        const int cap = a.cand_ld < n_cand ? static_cast<int>(a.cand_ld) : n_cand;
        const int c = min(a.cand_cnt[row], cap);
        if (tid < kImpBins) sm.hist[tid] = a.hist[static_cast<size_t>(row) * kImpBins + tid];
        if (tid == 0) { sm.nsel = 0; sm.nbnd = 0; }
        __syncthreads();
        if (tid == 0) {
            int cum = 0, bs = -1;
            for (int bin = kImpBins - 1; bin >= 0; --bin) {
                if (cum + static_cast<int>(sm.hist[bin]) >= kg) { bs = bin; break; }
                cum += static_cast<int>(sm.hist[bin]);
            }
            if (bs < 0) {                               // fewer candidates than picks: a bad list
                set_status(a.status, HS2_ERR_INDEX);
                bs = 0;
            }
            sm.bstar = bs;
            sm.above = cum;
            sm.need = kg - cum;
            sm.nb = static_cast<int>(sm.hist[bs]);
        }
        __syncthreads();
        const int bs = sm.bstar, need = sm.need, nb = sm.nb;
        const bool in_smem = nb <= kBndCap;
        // 2. positions above bin b*, keys of bin b*
        for (int base = 0; base < c; base += 4 * CNT) {
            uint2 e[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int i = base + u * CNT + tid;
                e[u] = i < c ? __ldcs(list + i) : make_uint2(0u, 0u);
            }
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                if (base + u * CNT + tid >= c) continue;
                const int bin = imp_bin(__uint_as_float(e[u].x));
                if (bin > bs) {
                    const int s = atomicAdd(&sm.nsel, 1);
                    if (s < kg) sm.sel[s] = static_cast<int>(e[u].y);
                } else if (bin == bs && in_smem) {
                    const int s = atomicAdd(&sm.nbnd, 1);
                    if (s < kBndCap) sm.bnd[s] = sel_key(e[u]);
                }
            }
        }
        __syncthreads();
        // 3. the `need` best keys of bin b*
        if (need >= nb && in_smem) {
            for (int i = tid; i < min(sm.nbnd, kBndCap); i += CNT) {
                const int s = atomicAdd(&sm.nsel, 1);
                if (s < kg) sm.sel[s] = key_pos(sm.bnd[i]);
            }
        } else if (in_smem) {
            const int n = min(sm.nbnd, kBndCap);
            int np = 1;
            while (np < n) np <<= 1;
            for (int i = n + tid; i < np; i += CNT) sm.bnd[i] = 0ull;     // below every real key
            __syncthreads();
            bitonic(sm.bnd, np, true);
            for (int i = tid; i < need; i += CNT) {
                const int s = atomicAdd(&sm.nsel, 1);
                if (s < kg) sm.sel[s] = key_pos(sm.bnd[i]);
            }
        } else {
            // a bin too large for shared memory: the need-th best key of bin b* by 8-bit digits
            // over the list (keys are unique: the position is part of them), then every key of
            // the bin from it up
            if (tid == 0) { sm.prefix = 0ull; sm.mask = 0ull; sm.remaining = need; }
            for (int shift = 56; shift >= 0; shift -= 8) {
                sm.rh[tid] = 0;
                __syncthreads();
                const unsigned long long pre = sm.prefix, msk = sm.mask;
                for (int i = tid; i < c; i += CNT) {
                    const uint2 e = list[i];
                    const unsigned long long k = sel_key(e);
                    if (imp_bin(__uint_as_float(e.x)) == bs && (k & msk) == pre)
                        atomicAdd(&sm.rh[(k >> shift) & 255u], 1);
                }
                __syncthreads();
                if (tid == 0) {
                    int cum = 0;
                    for (int d = 255; d >= 0; --d) {
                        if (cum + sm.rh[d] >= sm.remaining) {
                            sm.prefix |= static_cast<unsigned long long>(d) << shift;
                            sm.mask |= 0xFFull << shift;
                            sm.remaining -= cum;
                            break;
                        }
                        cum += sm.rh[d];
                    }
                }
                __syncthreads();
            }
            const unsigned long long tau = sm.prefix;
            for (int i = tid; i < c; i += CNT) {
                const uint2 e = list[i];
                if (imp_bin(__uint_as_float(e.x)) == bs && sel_key(e) >= tau) {
                    const int s = atomicAdd(&sm.nsel, 1);
                    if (s < kg) sm.sel[s] = static_cast<int>(e.y);
                }
            }
        }
        __syncthreads();
        if (tid == 0 && sm.nsel != kg) set_status(a.status, HS2_ERR_INDEX);    // inconsistent list
        // 4. ascending positions
        int np = 1;
        while (np < kg) np <<= 1;
        for (int i = kg + tid; i < np; i += CNT) sm.sel[i] = 0x7fffffff;
        for (int i = min(sm.nsel, kg) + tid; i < kg; i += CNT) sm.sel[i] = 0x7fffffff;
        __syncthreads();
        bitonic(sm.sel, np, false);
    }
    int32_t* out = a.idx + static_cast<size_t>(row) * a.idx_stride;
    const int win0 = p - nwin + 1;
    for (int j = tid; j < a.idx_stride; j += CNT) {
        int v = -1;
        if (j < kg) v = sm.sel[j];
        else if (j < kg + nwin) v = win0 + (j - kg);
        out[j] = v;
    }
    if (tid == 0) a.cnt[row] = kg + nwin;
}

}  // namespace

cudaError_t launch_cand_select(const CandSelectArgs& a, cudaStream_t st) {
    if (a.rows <= 0) return cudaSuccess;
    if (a.budget > kFusedSelectMaxBudget) return cudaErrorInvalidValue;
    const size_t sm = sizeof(Smem);
    cudaError_t e = cudaFuncSetAttribute(cand_select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(sm));
    if (e != cudaSuccess) return e;
    cand_select_kernel<<<a.rows, CNT, sm, st>>>(a);
    return cudaGetLastError();
}

}  // namespace hs2
