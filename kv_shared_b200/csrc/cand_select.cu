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
//   1. the bins give the bin b* holding the K-th best candidate;
//   2. one pass over the list marks the positions of higher bins in a bitmap of the
//      row's candidate positions and copies the keys of bin b* to shared memory;
//   3. bin b* is narrowed digit by digit (8 bits of the key (value bits, ~position) at a
//      time: a histogram, the digit holding the cutoff, the keys of higher digits
//      marked) until at most 32 keys remain, which one warp ranks exactly;
//   4. a block-wide scan of the bitmap writes the K positions in ascending order, then
//      the window [max(0, p-W+1), p], then -1.
// Rows whose candidate range is too long for the bitmap keep a position list and sort
// it instead; a cutoff bin too large for shared memory is narrowed by passes over the
// list in global memory.  Integer work only: importance values are compared as their
// fp32 bit patterns (non-negative, so they order as unsigned integers).
#include "common.cuh"
#include "internal.h"

namespace hs2 {
namespace {

constexpr int CNT = 256;
constexpr int NWARP = CNT / 32;
constexpr int kBndCap = 2048;                  // cutoff-bin keys held in shared memory
constexpr int kMapWords = 8192;                // bitmap of candidate positions (262144 bits)
constexpr int kFinal = 32;                     // keys ranked by one warp at the end

// Shared memory: this struct, then the bitmap of the longest candidate range of the launch
// (or the position list when that range is too long for a bitmap), sized at launch so that
// more CTAs fit on an SM.
struct Smem {
    unsigned long long bnd[2][kBndCap];        // cutoff keys (ping-pong while narrowing)
    uint32_t hist[kImpBins];
    int dh[256];                               // digit counts
    int wsum[NWARP];
    int nsel, nbnd[2];
    int bstar, need, nb, digit, cur;
    unsigned long long kand, kor;              // AND and OR of the cutoff-bin keys
};

__device__ __forceinline__ unsigned long long sel_key(uint2 e) {
    return (static_cast<unsigned long long>(e.x) << 32) | static_cast<uint32_t>(~e.y);
}

__device__ __forceinline__ int key_pos(unsigned long long k) { return static_cast<int>(~static_cast<uint32_t>(k)); }

// Appends one value per flagged lane to arr at a warp-aggregated offset of *count.
template <typename T>
__device__ __forceinline__ void warp_append(bool flag, T v, T* arr, int* count, int cap) {
    const uint32_t m = __ballot_sync(0xffffffffu, flag);
    if (m == 0u) return;
    const int lane = threadIdx.x & 31;
    int base = 0;
    if (lane == __ffs(m) - 1) base = atomicAdd(count, __popc(m));
    base = __shfl_sync(0xffffffffu, base, __ffs(m) - 1);
    const int s = base + __popc(m & ((1u << lane) - 1u));
    if (flag && s < cap) arr[s] = v;
}

// In-place bitonic sort (ascending) of n (a power of two) ints; the whole CTA takes part.
__device__ void bitonic_asc(int* v, int n) {
    for (int k = 2; k <= n; k <<= 1) {
        for (int j = k >> 1; j > 0; j >>= 1) {
            for (int i = threadIdx.x; i < n; i += CNT) {
                const int l = i ^ j;
                if (l > i) {
                    const bool up = (i & k) == 0;
                    const int a = v[i], b = v[l];
                    if ((a > b) == up) { v[i] = b; v[l] = a; }
                }
            }
            __syncthreads();
        }
    }
}

// Block-wide exclusive scan of one int per thread.
__device__ __forceinline__ int block_excl_scan(int x, Smem& sm) {
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    int incl = x;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
    }
    if (lane == 31) sm.wsum[w] = incl;
    __syncthreads();
    int before = 0;
    for (int i = 0; i < w; ++i) before += sm.wsum[i];
    __syncthreads();
    return before + incl - x;
}

__global__ void __launch_bounds__(CNT, 5) cand_select_kernel(CandSelectArgs a) {
    extern __shared__ __align__(16) uint8_t smem_raw[];
    Smem& sm = *reinterpret_cast<Smem*>(smem_raw);
    uint32_t* map = reinterpret_cast<uint32_t*>(smem_raw + sizeof(Smem));     // bitmap mode
    int* sel = reinterpret_cast<int*>(smem_raw + sizeof(Smem));               // list mode
    const int row = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int b = row / a.n_q, r = row % a.n_q;
    const int p = checked_pos(a.q_pos0[b] + r, a.max_ctx, a.status);
    const int n_cand = max(0, p - a.window + 1);
    const int kg = min(a.budget, n_cand);              // global picks of this row
    const int nwin = min(p + 1, a.window);
    const bool use_map = a.map_words > 0;                  // launch-wide: n_cand <= 32 * map_words
    const int words = (n_cand + 31) >> 5;

    if (kg > 0) {
        // the row's two segments (one per key half of the tiles), read as one list
        const uint2* seg0 = a.cand + static_cast<size_t>(row) * 2 * a.cand_seg;
        const uint2* seg1 = seg0 + a.cand_seg;
        const int segcap = a.cand_seg < n_cand ? static_cast<int>(a.cand_seg) : n_cand;
        const int c0 = max(0, min(a.cand_cnt[2 * row], segcap));
        const int c = c0 + max(0, min(a.cand_cnt[2 * row + 1], segcap));
        auto entry = [&](int i) -> uint2 { return i < c0 ? seg0[i] : seg1[i - c0]; };
        auto entry_cs = [&](int i) -> uint2 { return i < c0 ? __ldcs(seg0 + i) : __ldcs(seg1 + (i - c0)); };
        for (int i = tid; i < kImpBins; i += CNT) sm.hist[i] = a.hist[static_cast<size_t>(row) * kImpBins + i];
        if (use_map)
            for (int i = tid; i < words; i += CNT) map[i] = 0u;
        if (tid == 0) { sm.nsel = 0; sm.nbnd[0] = 0; sm.nbnd[1] = 0; sm.cur = 0; sm.kand = ~0ull; sm.kor = 0ull; }
        __syncthreads();
        if (warp == 0) {                               // 1. the cutoff bin
            uint32_t h[kImpPerLane];
            int mine = 0;
#pragma unroll
            for (int j = 0; j < kImpPerLane; ++j) { h[j] = sm.hist[kImpPerLane * lane + j]; mine += static_cast<int>(h[j]); }
            int above = mine;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_down_sync(0xffffffffu, above, o);
                if (lane + o < 32) above += y;
            }
            int cum = above - mine, best = -1, best_cum = 0;
#pragma unroll
            for (int j = kImpPerLane - 1; j >= 0; --j) {
                if (best < 0 && cum + static_cast<int>(h[j]) >= kg) { best = kImpPerLane * lane + j; best_cum = cum; }
                cum += static_cast<int>(h[j]);
            }
            const int top = __reduce_max_sync(0xffffffffu, best);
            const uint32_t own = __ballot_sync(0xffffffffu, best == top && top >= 0);
            if (top < 0) {                              // fewer candidates than picks: a bad list
                if (lane == 0) {
                    set_status(a.status, HS2_ERR_INDEX);
                    sm.bstar = 0; sm.need = 0; sm.nb = 0;
                }
            } else if (lane == __ffs(own) - 1) {
                sm.bstar = top;
                sm.need = kg - best_cum;
                sm.nb = static_cast<int>(h[top % kImpPerLane]);
            }
        }
        __syncthreads();
        const int bs = sm.bstar, nb = sm.nb;
        const bool bnd_smem = nb <= kBndCap;
        // 2. mark the positions above bin b*, gather bin b*'s keys; a batch's appends take one
        // shared counter update per warp (a per-entry update serialised the warps on it)
        constexpr int kLd = 16;                        // loads in flight per thread
        unsigned long long kand = ~0ull, kor = 0ull;
        for (int base = 0; base < c; base += kLd * CNT) {
            uint2 e[kLd];
#pragma unroll
            for (int u = 0; u < kLd; ++u) {
                const int i = base + u * CNT + tid;
                e[u] = i < c ? entry_cs(i) : make_uint2(0u, 0x7fffffffu);
            }
            uint32_t at_bs = 0u, above = 0u;           // bit u: entry u in bin b* / above it
#pragma unroll
            for (int u = 0; u < kLd; ++u) {
                const bool valid = base + u * CNT + tid < c;
                const int bin = valid ? imp_bin(__uint_as_float(e[u].x)) : -1;
                const int pos = static_cast<int>(e[u].y);
                if (bin > bs) {
                    above |= 1u << u;
                    if (use_map && pos < n_cand) atomicOr(&map[pos >> 5], 1u << (pos & 31));
                }
                if (bin == bs) {
                    at_bs |= 1u << u;
                    kand &= sel_key(e[u]);
                    kor |= sel_key(e[u]);
                }
            }
            auto append = [&](uint32_t flags, int* count, int cap, auto value) {
                const int n = __popc(flags);
                int incl = n;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const int y = __shfl_up_sync(0xffffffffu, incl, o);
                    if (lane >= o) incl += y;
                }
                if (__shfl_sync(0xffffffffu, incl, 31) == 0) return;
                int base_w = 0;
                if (lane == 31) base_w = atomicAdd(count, incl);
                int off = __shfl_sync(0xffffffffu, base_w, 31) + incl - n;
#pragma unroll
                for (int u = 0; u < kLd; ++u)             // static indices: e[] stays in registers
                    if (flags & (1u << u)) {
                        if (off < cap) value(off, u);
                        ++off;
                    }
            };
            if (bnd_smem)
                append(at_bs, &sm.nbnd[0], kBndCap,
                       [&](int off, int u) { sm.bnd[0][off] = sel_key(e[u]); });
            if (!use_map)
                append(above, &sm.nsel, kFusedSelectMaxBudget,
                       [&](int off, int u) { sel[off] = static_cast<int>(e[u].y); });
        }
        atomicAnd(&sm.kand, kand);
        atomicOr(&sm.kor, kor);
        __syncthreads();
        // 3. narrow bin b* to the `need` best keys
        auto take = [&](unsigned long long k) {
            const int pos = key_pos(k);
            if (use_map) {
                if (pos >= 0 && pos < n_cand) atomicOr(&map[pos >> 5], 1u << (pos & 31));
            } else {
                const int s = atomicAdd(&sm.nsel, 1);
                if (s < kFusedSelectMaxBudget) sel[s] = pos;
            }
        };
        if (!bnd_smem) {
            // too many keys for shared memory: digit passes over the list in global memory
            // (8 bits of the key at a time from the top), each keeping bin b*'s keys of the
            // cutoff digit, until they fit
            int shift = 56, need = sm.need;
            unsigned long long pre = 0ull, msk = 0ull;
            for (;;) {
                sm.dh[tid] = 0;
                __syncthreads();
                for (int i = tid; i < c; i += CNT) {
                    const uint2 e = entry(i);
                    const unsigned long long k = sel_key(e);
                    if (imp_bin(__uint_as_float(e.x)) == bs && (k & msk) == pre) atomicAdd(&sm.dh[(k >> shift) & 255u], 1);
                }
                __syncthreads();
                if (tid == 0) {
                    int cum = 0, d = 255;
                    for (; d > 0 && cum + sm.dh[d] < need; --d) cum += sm.dh[d];
                    sm.digit = d;
                    sm.nb = sm.dh[d];
                    sm.need = need - cum;
                }
                __syncthreads();
                const int d = sm.digit;
                for (int i = tid; i < c; i += CNT) {                  // keys of higher digits are in
                    const uint2 e = entry(i);
                    const unsigned long long k = sel_key(e);
                    if (imp_bin(__uint_as_float(e.x)) == bs && (k & msk) == pre &&
                        static_cast<int>((k >> shift) & 255u) > d)
                        take(k);
                }
                pre |= static_cast<unsigned long long>(d) << shift;
                msk |= 0xFFull << shift;
                need = sm.need;
                __syncthreads();
                if (sm.nb <= kBndCap || shift == 0) break;
                shift -= 8;
            }
            for (int base = 0; base < c; base += CNT) {
                const int i = base + tid;
                const uint2 e = i < c ? entry(i) : make_uint2(0u, 0u);
                const unsigned long long k = sel_key(e);
                warp_append(i < c && imp_bin(__uint_as_float(e.x)) == bs && (k & msk) == pre, k, sm.bnd[0],
                            &sm.nbnd[0], kBndCap);
            }
            __syncthreads();
        }
        {
            // narrow the shared-memory keys by 8-bit digits, from the digit holding the highest
            // bit where the cutoff-bin keys differ (bins 0 and 127 hold values of several
            // exponents, so the shared bits are measured, not assumed)
            int cur = 0;
            const unsigned long long diff = sm.kand ^ sm.kor;
            int shift = diff ? ((63 - __clzll(static_cast<long long>(diff))) & ~7) : 0;
            for (;;) {
                const int n = min(sm.nbnd[cur], kBndCap), need = sm.need;
                if (n <= kFinal || need >= n) break;
                sm.dh[tid] = 0;
                __syncthreads();
                for (int i = tid; i < n; i += CNT) atomicAdd(&sm.dh[(sm.bnd[cur][i] >> shift) & 255u], 1);
                __syncthreads();
                if (warp == 0) {
                    int h[8];
                    int mine = 0;
#pragma unroll
                    for (int j = 0; j < 8; ++j) { h[j] = sm.dh[8 * lane + j]; mine += h[j]; }
                    int above = mine;
#pragma unroll
                    for (int o = 1; o < 32; o <<= 1) {
                        const int y = __shfl_down_sync(0xffffffffu, above, o);
                        if (lane + o < 32) above += y;
                    }
                    int cum = above - mine, best = -1, best_cum = 0;
#pragma unroll
                    for (int j = 7; j >= 0; --j) {
                        if (best < 0 && cum + h[j] >= need) { best = 8 * lane + j; best_cum = cum; }
                        cum += h[j];
                    }
                    const int top = __reduce_max_sync(0xffffffffu, best);
                    const uint32_t own = __ballot_sync(0xffffffffu, best == top);
                    if (lane == __ffs(own) - 1) { sm.digit = top; sm.need = need - best_cum; }
                    if (lane == 0) sm.nbnd[cur ^ 1] = 0;
                }
                __syncthreads();
                const int d = sm.digit;
                for (int base = 0; base < n; base += CNT) {
                    const int i = base + tid;
                    const unsigned long long k = i < n ? sm.bnd[cur][i] : 0ull;
                    const int kd = i < n ? static_cast<int>((k >> shift) & 255u) : -1;
                    if (kd > d) take(k);
                    warp_append(kd == d, k, sm.bnd[cur ^ 1], &sm.nbnd[cur ^ 1], kBndCap);
                }
                __syncthreads();
                cur ^= 1;
                if (shift == 0) break;
                shift -= 8;
            }
            // at most kFinal keys left (or all of them taken): one warp ranks them exactly
            const int n = min(sm.nbnd[cur], kBndCap), need = sm.need;
            if (warp == 0 && need > 0) {
                if (need >= n) {
                    for (int i = lane; i < n; i += 32) take(sm.bnd[cur][i]);
                } else {
                    const unsigned long long k = lane < n ? sm.bnd[cur][lane] : 0ull;
                    int rank = 0;
                    for (int j = 0; j < n; ++j) rank += __shfl_sync(0xffffffffu, k, j) > k ? 1 : 0;
                    if (lane < n && rank < need) take(k);
                }
            }
        }
        __syncthreads();
    }
    // 4. the output row: K positions ascending, the window, -1
    int32_t* out = a.idx + static_cast<size_t>(row) * a.idx_stride;
    const int win0 = p - nwin + 1;
    if (kg > 0 && use_map) {
        const int per = (words + CNT - 1) / CNT;
        const int w0 = min(tid * per, words), w1 = min(w0 + per, words);
        int cnt_bits = 0;
        for (int w = w0; w < w1; ++w) cnt_bits += __popc(map[w]);
        int o = block_excl_scan(cnt_bits, sm);
        for (int w = w0; w < w1; ++w) {
            uint32_t m = map[w];
            while (m) {
                const int bit = __ffs(m) - 1;
                m &= m - 1;
                if (o < kg) out[o] = w * 32 + bit;
                ++o;
            }
        }
        if (tid == CNT - 1 && o != kg) set_status(a.status, HS2_ERR_INDEX);   // inconsistent list
    } else if (kg > 0) {
        int np = 1;
        while (np < kg) np <<= 1;
        const int ns = min(sm.nsel, kg);
        if (tid == 0 && sm.nsel != kg) set_status(a.status, HS2_ERR_INDEX);
        for (int i = ns + tid; i < np; i += CNT) sel[i] = 0x7fffffff;
        __syncthreads();
        bitonic_asc(sel, np);
        for (int j = tid; j < kg; j += CNT) out[j] = sel[j];
    }
    for (int j = kg + tid; j < a.idx_stride; j += CNT) out[j] = j < kg + nwin ? win0 + (j - kg) : -1;
    if (tid == 0) a.cnt[row] = kg + nwin;
}

}  // namespace

cudaError_t launch_cand_select(const CandSelectArgs& in, cudaStream_t st) {
    if (in.rows <= 0) return cudaSuccess;
    if (in.budget > kFusedSelectMaxBudget) return cudaErrorInvalidValue;
    CandSelectArgs a = in;
    // the longest candidate range of the launch is [0, max_ctx - 1 - window]
    const int64_t n_cand = a.max_ctx - a.window > 0 ? a.max_ctx - a.window : 0;
    const int64_t words = (n_cand + 31) / 32;
    a.map_words = words <= kMapWords ? static_cast<int>(words > 0 ? words : 1) : 0;
    const size_t sm = sizeof(Smem) + (a.map_words > 0 ? 4 * static_cast<size_t>(a.map_words)
                                                       : 4 * static_cast<size_t>(kFusedSelectMaxBudget));
    cudaError_t e = cudaFuncSetAttribute(cand_select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(sm));
    if (e != cudaSuccess) return e;
    cand_select_kernel<<<a.rows, CNT, sm, st>>>(a);
    return cudaGetLastError();
}

}  // namespace hs2
