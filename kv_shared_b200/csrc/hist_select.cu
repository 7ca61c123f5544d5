// hist_select.cu -- token-level top-K + forced window of decode rows, from the histogram of
// candidate importances that the decode attention kernels fill while they write the rows
// ("Xiaomi Unveils HySparse2 Architecture for MiMo-V3", section "Two-Level KV Sharing": the
// full layer picks the positions the later layers keep once it has run; section
// "Token-Level Sparse Selection": 1,024 global positions plus the 128 most recent).
//
// The histogram of a row counts every candidate key of [0, p - W] in a bin of its fp32 bit
// pattern (bits >> kDecHistShift; importance values are non-negative, so the patterns order
// like the values).  Many CTAs per row:
//   1. each CTA finds the cutoff bin b1 that holds the row's K-th best candidate;
//   2. each CTA passes over its slice of the row: the positions of keys above b1 go to the
//      row's list (fewer than K of them), the keys of b1 (value bits, ~position) to the row's
//      tie list;
//   3. the last CTA of the row (a counter) narrows the tie list by 8-bit digits to its `need`
//      best (value desc, position asc), sorts the K positions (counting sort into buckets of
//      positions, then ranks within a bucket) and writes idx and cnt: the K positions
//      ascending, the window [max(0, p-W+1), p], then -1.
// A cutoff bin with more keys than the tie buffer holds (a nearly flat row) is first refined by
// the next kDecFineBits bits of the values: every CTA of the row counts its keys of the bin in
// fine bins, the row's CTAs wait for one another (a bounded wait on a counter; the launch is
// cooperative, so they are all resident), and the cutoff class becomes (bin, fine bin).  A
// class still too large (values equal to the last bits) is narrowed by passes over the row in
// global memory.  Integer work only after each value's class.
#include "common.cuh"
#include "internal.h"

namespace hs2 {
namespace {

constexpr int HNT = 256;
constexpr int HWARPS = HNT / 32;
constexpr int kSortBuckets = 4096;            // buckets of the final counting sort
static_assert(kDecHistBins % HNT == 0 && kDecFineBins % HNT == 0 && kSortBuckets % HNT == 0,
              "bins and buckets split evenly over the threads");

struct HSmem {
    int wsum[HWARPS];
    int dh[256];
    int b1, above, n1, last, digit, need, cnt, nsel;
    unsigned long long kand, kor;
};

__device__ __forceinline__ unsigned long long tie_key(uint32_t bits, int pos) {
    return (static_cast<unsigned long long>(bits) << 32) | static_cast<uint32_t>(~pos);
}
__device__ __forceinline__ int tie_pos(unsigned long long k) { return static_cast<int>(~static_cast<uint32_t>(k)); }

// Appends v for each flagged lane at a warp-aggregated offset of *count (shared memory);
// entries at or past cap are counted but not stored.
template <typename T>
__device__ __forceinline__ void warp_push(bool flag, T v, T* arr, int* count, int cap) {
    const uint32_t m = __ballot_sync(0xffffffffu, flag);
    if (m == 0u) return;
    const int lane = threadIdx.x & 31;
    int base = 0;
    if (lane == __ffs(m) - 1) base = atomicAdd(count, __popc(m));
    base = __shfl_sync(0xffffffffu, base, __ffs(m) - 1);
    const int s = base + __popc(m & ((1u << lane) - 1u));
    if (flag && s < cap) arr[s] = v;
}

// The 256-bin digit histogram sm.dh read by warp 0: the highest digit d whose keys, with those
// of the higher digits, reach `need`.  Sets sm.digit, sm.need (still to take within d) and
// sm.cnt (keys of d).
__device__ __forceinline__ void pick_digit(HSmem& sm, int need) {
    const int lane = threadIdx.x & 31;
    int h[8], mine = 0;
#pragma unroll
    for (int j = 0; j < 8; ++j) { h[j] = sm.dh[8 * lane + j]; mine += h[j]; }
    int suf = mine;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_down_sync(0xffffffffu, suf, o);
        if (lane + o < 32) suf += y;
    }
    int cum = suf - mine, best = -1, best_cum = 0;
#pragma unroll
    for (int j = 7; j >= 0; --j) {
        if (best < 0 && cum + h[j] >= need) { best = 8 * lane + j; best_cum = cum; }
        cum += h[j];
    }
    const int top = __reduce_max_sync(0xffffffffu, best);
    const uint32_t own = __ballot_sync(0xffffffffu, best == top && top >= 0);
    if (top < 0) {                            // fewer keys than `need`: take them all
        if (lane == 0) { sm.digit = 0; sm.need = 0; sm.cnt = 0; }
    } else if (lane == __ffs(own) - 1) {
        sm.digit = top;
        sm.need = need - best_cum;
        sm.cnt = h[top % 8];
    }
}

// Narrows the keys that for_keys(f) yields (f called once per key, by some thread) to the
// `need` best: afterwards exactly the keys k with (k & mask) >= prefix are taken.  Digits of
// 8 bits from `shift` down (the bits above shift + 7 are the same for every key).
template <typename ForKeys>
__device__ void narrow(HSmem& sm, int need, int shift, ForKeys for_keys, unsigned long long& mask,
                       unsigned long long& prefix) {
    mask = 0ull;
    prefix = 0ull;
    if (need <= 0) {                          // nothing to take: a prefix no key reaches
        mask = ~0ull;
        prefix = ~0ull;
        return;
    }
    for (;;) {
        sm.dh[threadIdx.x] = 0;
        __syncthreads();
        const unsigned long long m = mask, pre = prefix;
        const int sh = shift;
        for_keys([&](unsigned long long k) {
            if ((k & m) == pre) atomicAdd(&sm.dh[(k >> sh) & 255u], 1);
        });
        __syncthreads();
        if (threadIdx.x < 32) pick_digit(sm, need);
        __syncthreads();
        prefix |= static_cast<unsigned long long>(sm.digit) << shift;
        mask |= 0xFFull << shift;
        const bool done = sm.cnt <= sm.need || shift == 0;   // every key of the digit is taken
        need = sm.need;
        __syncthreads();
        if (done) break;
        shift -= 8;
    }
}

// Bounded wait until *p >= target (false, status set, on timeout).
__device__ __forceinline__ bool wait_at_least(const int* p, int target, uint32_t* status) {
    const uint64_t t0 = global_ns();
#pragma unroll 1
    for (uint32_t i = 0; i < kWaitPolls; ++i) {
        int v;
        asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
        if (v >= target) return true;
        if ((i & 15) == 15) {
            if (global_ns() - t0 > kWaitNs) break;
            __nanosleep(64);
        }
    }
    set_status(status, HS2_ERR_TIMEOUT);
    return false;
}

// The highest bin of h[0 .. n) (thread t holding bins per*t .. per*t + per - 1, per = n / HNT)
// whose count, with the counts of the bins above it, reaches `need`: sets sm.b1 (-1 if none),
// sm.above (keys of the higher bins) and sm.n1 (keys of the bin).  All threads call it.
template <int PER, typename Load>
__device__ void cutoff_bin(HSmem& sm, int need, Load load) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    int hb[PER], mine = 0;
#pragma unroll
    for (int j = 0; j < PER; ++j) {
        hb[j] = load(PER * tid + j);
        mine += hb[j];
    }
    int suf = mine;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_down_sync(0xffffffffu, suf, o);
        if (lane + o < 32) suf += y;
    }
    if (tid == 0) sm.b1 = -1;
    if (lane == 0) sm.wsum[warp] = suf;
    __syncthreads();
    int cum = suf - mine;
    for (int w = warp + 1; w < HWARPS; ++w) cum += sm.wsum[w];
    int best = -1, best_cum = 0;
#pragma unroll
    for (int j = PER - 1; j >= 0; --j) {
        if (best < 0 && cum + hb[j] >= need) { best = PER * tid + j; best_cum = cum; }
        cum += hb[j];
    }
    if (best >= 0) atomicMax(&sm.b1, best);
    __syncthreads();
    if (best >= 0 && best == sm.b1) { sm.above = best_cum; sm.n1 = hb[best % PER]; }
    __syncthreads();
}

// class of a value: its coarse bin, or (level 1) the coarse bin and the next kDecFineBits bits
__device__ __forceinline__ uint32_t value_class(uint32_t bits, int level) {
    const uint32_t c = static_cast<uint32_t>(dec_bin(bits));
    return level ? (c << kDecFineBits) | ((bits >> kDecFineShift) & (kDecFineBins - 1)) : c;
}

// Block-wide exclusive scan of one int per thread (wsum: HWARPS ints of shared memory).
__device__ __forceinline__ int block_excl_scan(int x, int* wsum) {
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    int incl = x;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
    }
    if (lane == 31) wsum[w] = incl;
    __syncthreads();
    int before = 0;
    for (int i = 0; i < w; ++i) before += wsum[i];
    __syncthreads();
    return before + incl - x;
}

__global__ void __launch_bounds__(HNT) hist_select_kernel(HistSelectArgs a) {
    extern __shared__ __align__(16) uint8_t dyn[];
    int* pos = reinterpret_cast<int*>(dyn);                   // [budget] staging of the keys above
    unsigned long long* tk = reinterpret_cast<unsigned long long*>(dyn + 4 * kFusedSelectMaxBudget);   // [kDecTieCap]
    int* fh = reinterpret_cast<int*>(tk);                     // refinement: [kDecFineBins] before the ties
    __shared__ HSmem sm;
    __shared__ int s_level, s_tval, s_need, s_na, s_nt, s_base_a, s_base_t;
    const int row = blockIdx.y, tid = threadIdx.x;
    const int p = checked_pos(a.q_pos0[row], a.max_ctx, a.status);
    const int n_cand = max(0, p - a.window + 1);
    const int kg = min(a.budget, n_cand);
    const int nwin = min(p + 1, a.window);
    const int* hist = a.hist + static_cast<size_t>(row) * kDecHistRow;
    int* fine = a.hist + static_cast<size_t>(row) * kDecHistRow + kDecHistBins;
    int* ctl = a.ctl + 4 * row;
    int* above = a.above + static_cast<size_t>(row) * a.budget;
    unsigned long long* tie = a.tie + static_cast<size_t>(row) * kDecTieCap;
    const float* srow = a.scores + static_cast<size_t>(row) * a.score_ld;
    const bool partial = kg > 0 && kg < n_cand;          // otherwise every candidate or none
    const int begin = blockIdx.x * a.slice, end = min(begin + a.slice, n_cand);

    // every key of this CTA's slice (f may see indices at or past end: it checks them); 16
    // keys per thread in flight, as float4 when the rows are 16-byte aligned
    auto for_slice = [&](auto f) {
        if (a.vec4) {
            for (int base = begin; base < end; base += 16 * HNT) {
                float4 v[4];
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int i = base + 4 * (u * HNT + tid);
                    if (i + 4 <= end) {
                        v[u] = __ldcg(reinterpret_cast<const float4*>(srow + i));
                    } else {
                        v[u].x = i < end ? __ldcg(srow + i) : 0.f;
                        v[u].y = i + 1 < end ? __ldcg(srow + i + 1) : 0.f;
                        v[u].z = i + 2 < end ? __ldcg(srow + i + 2) : 0.f;
                        v[u].w = 0.f;
                    }
                }
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int i = base + 4 * (u * HNT + tid);
                    f(i, __float_as_uint(v[u].x));
                    f(i + 1, __float_as_uint(v[u].y));
                    f(i + 2, __float_as_uint(v[u].z));
                    f(i + 3, __float_as_uint(v[u].w));
                }
            }
        } else {
            for (int base = begin; base < end; base += 16 * HNT) {
                float v[16];
#pragma unroll
                for (int u = 0; u < 16; ++u) {
                    const int i = base + u * HNT + tid;
                    v[u] = i < end ? __ldcg(srow + i) : 0.f;
                }
#pragma unroll
                for (int u = 0; u < 16; ++u) f(base + u * HNT + tid, __float_as_uint(v[u]));
            }
        }
    };

    if (tid == 0) {
        sm.nsel = 0; sm.kand = ~0ull; sm.kor = 0ull;
        s_level = 0; s_tval = -1; s_need = 0; s_na = 0; s_nt = 0;
    }
    if (partial) {
        // 1. the cutoff bin of the coarse histogram
        cutoff_bin<kDecHistBins / HNT>(sm, kg, [&](int i) { return __ldcg(hist + i); });
        const int b1 = sm.b1;
        if (b1 >= 0 && tid == 0) { s_tval = b1; s_need = kg - sm.above; }
        __syncthreads();
        if (b1 >= 0 && sm.n1 > kDecTieCap) {
            // 1b. too many keys in it for the tie buffer (a nearly flat row): refine the bin by
            // the next kDecFineBits bits, counted over the whole row by all of its CTAs
            const int need0 = kg - sm.above;
            for (int i = tid; i < kDecFineBins; i += HNT) fh[i] = 0;
            __syncthreads();
            for_slice([&](int i, uint32_t bits) {
                if (i < end && dec_bin(bits) == b1) atomicAdd(&fh[(bits >> kDecFineShift) & (kDecFineBins - 1)], 1);
            });
            __syncthreads();
            for (int i = tid; i < kDecFineBins; i += HNT)
                if (fh[i]) atomicAdd(fine + i, fh[i]);
            __threadfence();
            __syncthreads();
            if (tid == 0) {
                atomicAdd(ctl + 3, 1);
                if (!wait_at_least(ctl + 3, static_cast<int>(gridDim.x), a.status)) s_tval = -1;
            }
            __syncthreads();
            if (s_tval >= 0) {
                cutoff_bin<kDecFineBins / HNT>(sm, need0, [&](int i) { return __ldcg(fine + i); });
                if (tid == 0) {
                    if (sm.b1 < 0) {
                        s_tval = -1;
                    } else {
                        s_level = 1;
                        s_tval = static_cast<int>((static_cast<uint32_t>(b1) << kDecFineBits) | static_cast<uint32_t>(sm.b1));
                        s_need = need0 - sm.above;
                    }
                }
                __syncthreads();
            }
        }
        // 2. this CTA's slice: keys of a higher class, keys of the cutoff class, gathered in
        // shared memory and appended to the row's lists at offsets of one reservation each
        const int level = s_level;
        const int tval = s_tval;
        if (tval >= 0) {
            for_slice([&](int i, uint32_t bits) {
                const int c = static_cast<int>(value_class(bits, level));
                warp_push(i < end && c > tval, i, pos, &s_na, kFusedSelectMaxBudget);
                warp_push(i < end && c == tval, tie_key(bits, i), tk, &s_nt, kDecTieCap);
            });
            __syncthreads();
            if (tid == 0) {
                s_base_a = s_na ? atomicAdd(ctl + 0, s_na) : 0;
                s_base_t = s_nt ? atomicAdd(ctl + 1, s_nt) : 0;
            }
            __syncthreads();
            const int na = min(s_na, kFusedSelectMaxBudget), nt = min(s_nt, kDecTieCap);
            for (int i = tid; i < na; i += HNT)
                if (s_base_a + i < a.budget) above[s_base_a + i] = pos[i];
            for (int i = tid; i < nt; i += HNT)
                if (s_base_t + i < kDecTieCap) tie[s_base_t + i] = tk[i];
        }
    }
    // 3. the last CTA of the row finishes it
    __threadfence();
    __syncthreads();
    if (tid == 0) sm.last = atomicAdd(ctl + 2, 1) == static_cast<int>(gridDim.x) - 1;
    __syncthreads();
    if (!sm.last) return;
    __threadfence();

    int32_t* out = a.idx + static_cast<size_t>(row) * a.idx_stride;
    const int level = s_level, tval = s_tval;
    if (partial && tval < 0) set_status(a.status, HS2_ERR_INDEX);       // fewer counted keys than picks
    const bool picked = partial && tval >= 0;
    if (picked) {
        const int n_above = __ldcg(ctl + 0), n_tie = __ldcg(ctl + 1);
        if (tid == 0 && n_above != kg - s_need) set_status(a.status, HS2_ERR_INDEX);
        const int na = min(n_above, kg);
        const int need = kg - na;
        for (int i = tid; i < na; i += HNT) pos[i] = __ldcg(above + i);
        auto take = [&](unsigned long long k) {
            const int s = atomicAdd(&sm.nsel, 1);
            if (na + s < kFusedSelectMaxBudget) pos[na + s] = tie_pos(k);
        };
        unsigned long long mask, prefix;
        if (n_tie <= kDecTieCap) {
            unsigned long long kand = ~0ull, kor = 0ull;
            for (int i = tid; i < n_tie; i += HNT) {
                const unsigned long long k = __ldcg(tie + i);
                tk[i] = k;
                kand &= k;
                kor |= k;
            }
            atomicAnd(&sm.kand, kand);
            atomicOr(&sm.kor, kor);
            __syncthreads();
            const unsigned long long diff = sm.kand ^ sm.kor;
            const int shift = diff ? ((63 - __clzll(static_cast<long long>(diff))) & ~7) : 0;
            narrow(sm, need, shift,
                   [&](auto f) {
                       for (int i = tid; i < n_tie; i += HNT) f(tk[i]);
                   },
                   mask, prefix);
            for (int i = tid; i < n_tie; i += HNT) {
                const unsigned long long k = tk[i];
                if ((k & mask) >= prefix) take(k);
            }
        } else {
            // a tie class past its buffer (values equal to the last bits): narrow over the row's
            // keys of the class in global memory; above bit 32 + the class's lowest value bit
            // a key's bits are the class's
            auto row_keys = [&](auto f) {
                for (int i = tid; i < n_cand; i += HNT) {
                    const uint32_t bits = __float_as_uint(__ldcg(srow + i));
                    if (static_cast<int>(value_class(bits, level)) == tval) f(tie_key(bits, i));
                }
            };
            const int low = level ? kDecFineShift : kDecHistShift;
            narrow(sm, need, (32 + low - 1) & ~7, row_keys, mask, prefix);
            row_keys([&](unsigned long long k) {
                if ((k & mask) >= prefix) take(k);
            });
        }
        __syncthreads();
        if (tid == 0 && sm.nsel != need) set_status(a.status, HS2_ERR_INDEX);
        __syncthreads();
        // the picks ascending: a counting sort into buckets of 2^sh positions (the tie keys'
        // space is free now), then each pick's rank within its bucket
        const int have = min(na + sm.nsel, kg);
        int* tmp = reinterpret_cast<int*>(tk);                       // [kFusedSelectMaxBudget]
        int* bend = tmp + kFusedSelectMaxBudget;                      // [kSortBuckets]
        int sh = 0;
        while ((n_cand >> sh) >= kSortBuckets) ++sh;
        const int nb = (n_cand >> sh) + 1;
        for (int i = tid; i < nb; i += HNT) bend[i] = 0;
        __syncthreads();
        for (int i = tid; i < have; i += HNT) atomicAdd(&bend[pos[i] >> sh], 1);
        __syncthreads();
        {
            constexpr int PER = kSortBuckets / HNT;
            int c[PER], sum = 0;
#pragma unroll
            for (int j = 0; j < PER; ++j) {
                const int bi = PER * tid + j;
                c[j] = bi < nb ? bend[bi] : 0;
                sum += c[j];
            }
            int o = block_excl_scan(sum, sm.wsum);
#pragma unroll
            for (int j = 0; j < PER; ++j) {
                const int bi = PER * tid + j;
                if (bi < nb) bend[bi] = o;                             // bucket start, for now
                o += c[j];
            }
        }
        __syncthreads();
        for (int i = tid; i < have; i += HNT) tmp[atomicAdd(&bend[pos[i] >> sh], 1)] = pos[i];
        __syncthreads();                                               // bend[b]: end of bucket b
        for (int i = tid; i < have; i += HNT) {
            const int v = tmp[i], bk = v >> sh;
            const int lo = bk ? bend[bk - 1] : 0, hi = bend[bk];
            int r = lo;
            for (int j = lo; j < hi; ++j) r += tmp[j] < v ? 1 : 0;
            out[r] = v;
        }
    } else if (kg > 0 && !partial) {
        for (int j = tid; j < kg; j += HNT) out[j] = j;   // every candidate is a pick
    }
    const int pick = partial && !picked ? 0 : kg;
    const int win0 = p - nwin + 1;
    for (int j = pick + tid; j < a.idx_stride; j += HNT) out[j] = j < pick + nwin ? win0 + (j - pick) : -1;
    if (tid == 0) a.cnt[row] = pick + nwin;
}

}  // namespace

size_t dec_select_ws_bytes(int batch, int budget) {
    auto al = [](size_t x) { return (x + 255) & ~size_t(255); };
    const size_t b = static_cast<size_t>(batch > 0 ? batch : 1);
    return al(sizeof(int) * b * kDecHistRow) + al(sizeof(int) * 4 * b) +
           al(sizeof(int) * b * static_cast<size_t>(budget > 0 ? budget : 1)) +
           al(sizeof(unsigned long long) * b * kDecTieCap);
}

DecSelState dec_select_state(void* ws, int batch, int budget) {
    auto al = [](size_t x) { return (x + 255) & ~size_t(255); };
    const size_t b = static_cast<size_t>(batch > 0 ? batch : 1);
    uint8_t* w = static_cast<uint8_t*>(ws);
    DecSelState s{};
    s.hist = reinterpret_cast<int*>(w);
    w += al(sizeof(int) * b * kDecHistRow);
    s.ctl = reinterpret_cast<int*>(w);
    w += al(sizeof(int) * 4 * b);
    s.above = reinterpret_cast<int*>(w);
    w += al(sizeof(int) * b * static_cast<size_t>(budget > 0 ? budget : 1));
    s.tie = reinterpret_cast<unsigned long long*>(w);
    return s;
}

cudaError_t launch_hist_select(const HistSelectArgs& in, cudaStream_t st) {
    if (in.rows <= 0) return cudaSuccess;
    if (in.budget > kFusedSelectMaxBudget || in.budget < 0) return cudaErrorInvalidValue;
    HistSelectArgs a = in;
    // slices: about two CTAs per SM over all rows, at least 4096 keys each
    const int64_t n_max = a.max_ctx - a.window > 0 ? a.max_ctx - a.window : 1;
    int64_t slices = (2 * static_cast<int64_t>(num_sms()) + a.rows - 1) / a.rows;
    const int64_t cap_slices = (n_max + 4095) / 4096;
    if (slices > cap_slices) slices = cap_slices;
    if (slices < 1) slices = 1;
    if (slices > 65535) slices = 65535;
    int64_t slice = (n_max + slices - 1) / slices;
    slice = (slice + 4 * HNT - 1) / (4 * HNT) * (4 * HNT);
    a.slice = static_cast<int>(slice);
    slices = (n_max + slice - 1) / slice;
    a.vec4 = a.score_ld % 4 == 0;
    const size_t smem = 4 * static_cast<size_t>(kFusedSelectMaxBudget) + 8 * static_cast<size_t>(kDecTieCap);
    cudaError_t e = cudaFuncSetAttribute(hist_select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    // the CTAs of a row may wait on one another (refinement): with several per row, all of
    // the launch's CTAs must be resident at once
    if (slices > 1) {
        int per_sm = 0;
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, hist_select_kernel, HNT, smem);
        if (e != cudaSuccess) return e;
        const int64_t resident = static_cast<int64_t>(per_sm) * num_sms();
        if (static_cast<int64_t>(a.rows) * slices > resident) {
            slices = resident / a.rows;
            if (slices < 1) slices = 1;
            slice = (n_max + slices - 1) / slices;
            slice = (slice + 4 * HNT - 1) / (4 * HNT) * (4 * HNT);
            a.slice = static_cast<int>(slice);
            slices = (n_max + slice - 1) / slice;
        }
    }
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(static_cast<unsigned>(slices), static_cast<unsigned>(a.rows));
    cfg.blockDim = dim3(HNT);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = slices > 1 ? 1 : 0;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, hist_select_kernel, a);
}

}  // namespace hs2
