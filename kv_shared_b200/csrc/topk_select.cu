// topk_select.cu -- token-level (and block-level) selection with the forced window.
//
// Per query row at position p ("Xiaomi Unveils HySparse2 Architecture for
// MiMo-V3", section "Token-Level Sparse Selection: Precision and Efficiency
// Balance": a compulsory window of the latest 128 tokens and 1,024 global picks):
//   window = [max(0, p-W+1), p], candidates = [0, p-W],
//   global = the K best candidates by (importance desc, position asc),
//   idx    = ascending union, -1 padded; cnt = |idx|.
// Block arm (first-generation rule of the MiMo-V3 news flash: a group of 64 is
// kept whole if any of its tokens is important): blocks of `bs` positions from
// 0, block importance = max, floor(K/bs) best blocks (lower block on ties).
//
// Exact selection on order-preserving uint32 images of the fp32 values.  A row
// is handled by a cluster of CS CTAs (CS = 1..16), CTA r owning a contiguous
// slice of the keys, cached in shared memory when it fits.
//   1. the row's key range (reduced over the cluster) gives the bits all keys
//      share; the first radix digit (<= 11 bits) is taken right below them.  Slices
//      too long for shared memory skip this pass (one read of the row saved), ask
//      for the whole slice in L2 up front (it is read twice) and take the top 13
//      bits as the first digit
//   2. one histogram of that digit over every key (summed over the cluster by
//      distributed shared memory) locates the bin b1 holding the K-th best key
//   3. every CTA compacts, in position order, its keys in bins >= b1 into a
//      short candidate list (about K plus the few keys of bin b1 per row); slices
//      read from global memory in one streaming pass, each warp buffering the
//      matches of its own segment
//   4. the remaining digits are resolved on the candidate lists only -> the exact
//      threshold key tau and how many keys equal to it are taken (need_eq)
//   5. each CTA writes its candidates above tau and its share of the first
//      need_eq equal to tau (the lower-position tie rule), already ascending, at
//      offsets from a cluster-wide prefix of the counts.
// If a candidate list would overflow its buffer (adversarial value
// distributions), the cluster falls back to resolving every digit over all keys.
// Integer work only after the key map.
#include <cooperative_groups.h>

#include "common.cuh"
#include "internal.h"

namespace cg = cooperative_groups;

namespace hs2 {
namespace {

constexpr int NT = 512;
constexpr int NW = NT / 32;
constexpr int NBINS = 2048;
constexpr int kMaxCluster = 16;           // 16 is a non-portable cluster size (few long rows)
constexpr int kSmemKeys = 24576;          // keys cached per CTA (96 KB)
constexpr int kCandCap = 2048;            // candidates per CTA (16 KB), a power of two
constexpr int kWarpCap = 512;             // streamed compaction: matches buffered per warp
constexpr int kStreamBits = 13;           // first digit of a streamed slice (fixed: top 13 bits)
constexpr int kMaxBins = 1 << kStreamBits;
static_assert(2 * kMaxBins <= 2 * NW * kWarpCap, "a streamed slice's histograms live in the warp buffers");

__device__ __forceinline__ uint32_t ord_key(float f) {
    const uint32_t u = __float_as_uint(f);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

struct Smem {
    int hist[2][NBINS];         // double-buffered: a digit's histogram may still be read
                                // by the cluster while the next digit's is built
    int warp_tot[NW];
    int total;
    int found_bin;
    int found_above;
    uint32_t wlo[NW], whi[NW];
    uint32_t range[2];          // this CTA's key range (read by the cluster)
    int counts[2];              // published to the cluster: #above, #equal (fallback paths)
    int dec[8];                 // rank 0's decisions: first-digit bin, count above, bin size,
                                // candidate mode; threshold key and equal keys to take
    int pub[2];                 // this CTA's candidate count and bin-b1 key count (read by rank 0)
    int table[kMaxCluster][2];  // rank 0: output offset and equal-key rank base per CTA
    int cnt_gt[kMaxCluster], cnt_eq[kMaxCluster];
    int ncand2, nb1;
    uint32_t bcast[2 * kMaxCluster];   // remote values fetched once and shared with the CTA
    int lhist[256];             // rank 0's digits over the gathered bin-b1 keys
};

// Block-wide exclusive scan of one int per thread; sm.total receives the sum.
__device__ __forceinline__ int block_excl_scan(int v, Smem& sm) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) sm.warp_tot[warp] = x;
    __syncthreads();
    if (warp == 0) {
        const int w = lane < NW ? sm.warp_tot[lane] : 0;
        int s = w;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, s, o);
            if (lane >= o) s += y;
        }
        if (lane < NW) sm.warp_tot[lane] = s - w;
        if (lane == NW - 1) sm.total = s;
    }
    __syncthreads();
    const int r = sm.warp_tot[warp] + x - v;
    __syncthreads();
    return r;
}

// Keys of this CTA's slice: cached in shared memory or recomputed from global.
struct Slice {
    const float* s;            // row scores
    int bs;                    // 1 = token keys, >1 = block maxima
    int n_cand;                // candidate tokens of the row
    int begin, end;            // this CTA's key range (tokens or blocks)
    const uint32_t* cache;     // shared-memory copy or nullptr
    __device__ __forceinline__ uint32_t compute(int i) const {
        if (bs == 1) return ord_key(s[i]);
        float m = -INFINITY;
        const int e = min((i + 1) * bs, n_cand);
        for (int j = i * bs; j < e; ++j) m = fmaxf(m, s[j]);
        return ord_key(m);
    }
    __device__ __forceinline__ uint32_t key(int i) const { return cache ? cache[i - begin] : compute(i); }
    // tokens a selected key expands to
    __device__ __forceinline__ int tokens(int i) const { return min((i + 1) * bs, n_cand) - i * bs; }
};

// Visits every key of the slice as f(i, key, valid) with 8 independent loads in
// flight per thread; all threads make the same number of calls.
constexpr int kBatch = 8;
template <typename F>
__device__ __forceinline__ void for_keys(const Slice& sl, F f) {
    for (int base = sl.begin; base < sl.end; base += NT * kBatch) {
        uint32_t k[kBatch];
#pragma unroll
        for (int u = 0; u < kBatch; ++u) {
            const int i = base + u * NT + threadIdx.x;
            k[u] = i < sl.end ? sl.key(i) : 0u;
        }
#pragma unroll
        for (int u = 0; u < kBatch; ++u) {
            const int i = base + u * NT + threadIdx.x;
            f(i, k[u], i < sl.end);
        }
    }
}

// One radix digit: histogram of bits [shift, shift+width) of the keys that `visit`
// offers and that match prefix under mask, summed over the cluster; leaves the bin
// holding the k_rem-th largest and the count above it in sm.found_bin/found_above.
// Histogram buffer `hb` alternates between digits, so one cluster barrier per digit
// suffices (a buffer is rebuilt only after every CTA has passed the next barrier).
template <int CS, typename Visit>
__device__ __forceinline__ void radix_digit(cg::cluster_group& cluster, Smem& sm, int hbuf, int shift, int width,
                                            uint32_t prefix, uint32_t mask, int k_rem, Visit visit) {
    const int nb = 1 << width;
    int* hist = sm.hist[hbuf];
    for (int i = threadIdx.x; i < nb; i += NT) hist[i] = 0;
    __syncthreads();
    visit([&](uint32_t key) {
        if ((key & mask) == prefix) atomicAdd(&hist[(key >> shift) & (nb - 1)], 1);
    });
    cluster.sync();
    const int bins_per = (nb + NT - 1) / NT;                   // 1..4
    int local[NBINS / NT];
    int tot = 0;
#pragma unroll
    for (int q = 0; q < NBINS / NT; ++q) {
        const int bin = nb - 1 - (threadIdx.x * bins_per + q);
        int c = 0;
        if (q < bins_per && bin >= 0) {
            int v[CS];
#pragma unroll
            for (int rr = 0; rr < CS; ++rr) v[rr] = CS == 1 ? hist[bin] : cluster.map_shared_rank(hist, rr)[bin];
#pragma unroll
            for (int rr = 0; rr < CS; ++rr) c += v[rr];
        }
        local[q] = c;
        tot += c;
    }
    const int above = block_excl_scan(tot, sm);
    if (above < k_rem && above + tot >= k_rem) {
        int acc = above;
        for (int q = 0; q < bins_per; ++q) {
            if (acc + local[q] >= k_rem) {
                sm.found_bin = nb - 1 - (threadIdx.x * bins_per + q);
                sm.found_above = acc;
                break;
            }
            acc += local[q];
        }
    }
    __syncthreads();
}

// Writes, in ascending order from out + written, the selected keys among n entries
// (position pos(e), key keyf(e), already ascending): key > tau, or key == tau while
// the running rank of equal keys (starting at eq_seen) is below need_eq; take_all
// selects every entry.  Returns the new written count.
template <typename Pos, typename Key>
__device__ __forceinline__ int ordered_write(Smem& sm, const Slice& sl, int n, Pos pos, Key keyf, uint32_t tau,
                                             int need_eq, bool take_all, int eq_seen, int written, int32_t* out) {
    for (int base = 0; base < n; base += 4 * NT) {
        const int e0 = base + 4 * threadIdx.x;
        uint32_t keys[4];
        int e_cnt = 0;
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int e = e0 + u;
            keys[u] = (e < n) ? keyf(e) : 0u;
            if (e < n && !take_all) e_cnt += keys[u] == tau;
        }
        const int eq_before = block_excl_scan(e_cnt, sm);
        const int eq_round = sm.total;
        int rank_eq = eq_seen + eq_before, ntok = 0;
        bool sel[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int e = e0 + u;
            sel[u] = false;
            if (e >= n) continue;
            if (take_all || keys[u] > tau) sel[u] = true;
            else if (keys[u] == tau) { sel[u] = rank_eq < need_eq; ++rank_eq; }
            if (sel[u]) ntok += sl.tokens(pos(e));
        }
        const int at = block_excl_scan(ntok, sm);
        const int round_total = sm.total;
        int o = written + at;
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            if (!sel[u]) continue;
            const int i = pos(e0 + u);
            const int e = min((i + 1) * sl.bs, sl.n_cand);
            for (int j = i * sl.bs; j < e; ++j) out[o++] = j;
        }
        written += round_total;
        eq_seen += eq_round;
    }
    return written;
}

// Visits every key of the slice as f(i, key) (any order).  Token keys go through
// 16-byte loads, 4 keys each and 8 loads in flight per thread, whenever the slice
// start is 16-byte aligned (shared-memory cache or score row); otherwise for_keys.
template <typename F>
__device__ __forceinline__ void for_keys_fast(const Slice& sl, F f) {
    const void* base_ptr = sl.cache ? static_cast<const void*>(sl.cache) : static_cast<const void*>(sl.s + sl.begin);
    if (sl.bs != 1 || (reinterpret_cast<uintptr_t>(base_ptr) & 15u) != 0) {
        for_keys(sl, [&](int i, uint32_t key, bool valid) { if (valid) f(i, key); });
        return;
    }
    const int n = sl.end - sl.begin, n4 = n >> 2;
    for (int base = 0; base < n4; base += NT * 8) {
        uint4 v[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int q = base + u * NT + threadIdx.x;
            if (q < n4) {
                if (sl.cache) {
                    v[u] = reinterpret_cast<const uint4*>(sl.cache)[q];
                } else {
                    const float4 x = __ldg(reinterpret_cast<const float4*>(sl.s + sl.begin) + q);
                    v[u] = make_uint4(ord_key(x.x), ord_key(x.y), ord_key(x.z), ord_key(x.w));
                }
            }
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int q = base + u * NT + threadIdx.x;
            if (q < n4) {
                const int i = sl.begin + 4 * q;
                f(i, v[u].x); f(i + 1, v[u].y); f(i + 2, v[u].z); f(i + 3, v[u].w);
            }
        }
    }
    for (int i = sl.begin + 4 * n4 + threadIdx.x; i < sl.end; i += NT) f(i, sl.key(i));
}

// Compacts, in position order, the slice's keys >= thr into (ck, cp); returns their
// number.  Rounds of 4 consecutive keys per thread, one block scan per round.
__device__ __forceinline__ int compact_ordered(const Slice& sl, uint32_t thr, uint32_t* ck, uint32_t* cp, Smem& sm) {
    int n = 0;
    const bool vec = sl.cache != nullptr;                  // cache rows start 16-byte aligned
    for (int base = sl.begin; base < sl.end; base += 4 * NT) {
        const int i0 = base + 4 * threadIdx.x;
        uint32_t k[4];
        if (vec && i0 + 3 < sl.end) {
            const uint4 v = *reinterpret_cast<const uint4*>(sl.cache + (i0 - sl.begin));
            k[0] = v.x; k[1] = v.y; k[2] = v.z; k[3] = v.w;
        } else {
#pragma unroll
            for (int u = 0; u < 4; ++u) k[u] = i0 + u < sl.end ? sl.key(i0 + u) : 0u;
        }
        int c = 0;
#pragma unroll
        for (int u = 0; u < 4; ++u) c += (i0 + u < sl.end) && k[u] >= thr;
        const int at = block_excl_scan(c, sm);
        const int tot = sm.total;
        int o = n + at;
#pragma unroll
        for (int u = 0; u < 4; ++u)
            if (i0 + u < sl.end && k[u] >= thr) { ck[o] = k[u]; cp[o] = static_cast<uint32_t>(i0 + u); ++o; }
        n += tot;
    }
    __syncthreads();                                      // the last round's entries are read next
    return n;
}

// As compact_ordered for a slice cached in shared memory: each warp owns a contiguous
// segment (chunks of 128 keys, 4 per lane), counts its matches, one block scan of
// the warp counts, then a second read writes them in order (warp-level scans only).
__device__ __forceinline__ int compact_cached(const Slice& sl, uint32_t thr, uint32_t* ck, uint32_t* cp, Smem& sm) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int n = sl.end - sl.begin;
    const int seg = ((n + NW * 128 - 1) / (NW * 128)) * 128;
    const int s0 = min(warp * seg, n), s1 = min(s0 + seg, n);
    auto load4 = [&](int e, uint32_t (&k)[4]) {              // keys e .. e+3 of the slice (e % 4 == 0)
        if (e + 3 < n) {
            const uint4 v = *reinterpret_cast<const uint4*>(sl.cache + e);
            k[0] = v.x; k[1] = v.y; k[2] = v.z; k[3] = v.w;
        } else {
#pragma unroll
            for (int u = 0; u < 4; ++u) k[u] = e + u < n ? sl.cache[e + u] : 0u;
        }
    };
    int mine = 0;
    for (int c0 = s0; c0 < s1; c0 += 128) {
        const int e = c0 + 4 * lane;
        uint32_t k[4];
        load4(e, k);
#pragma unroll
        for (int u = 0; u < 4; ++u) mine += (e + u < s1) && k[u] >= thr;
    }
    mine = __reduce_add_sync(0xffffffffu, mine);
    const int wbase = block_excl_scan(lane == 0 ? mine : 0, sm);
    const int total = sm.total;
    int o = __shfl_sync(0xffffffffu, wbase, 0);
    for (int c0 = s0; c0 < s1; c0 += 128) {
        const int e = c0 + 4 * lane;
        uint32_t k[4];
        load4(e, k);
        int c = 0;
#pragma unroll
        for (int u = 0; u < 4; ++u) c += (e + u < s1) && k[u] >= thr;
        int x = c;
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, x, d);
            if (lane >= d) x += y;
        }
        int w = o + x - c;
#pragma unroll
        for (int u = 0; u < 4; ++u)
            if ((e + u < s1) && k[u] >= thr) { ck[w] = k[u]; cp[w] = static_cast<uint32_t>(sl.begin + e + u); ++w; }
        o += __shfl_sync(0xffffffffu, x, 31);
    }
    __syncthreads();
    return total;
}

// As compact_ordered for a slice read from global memory (token keys, 16-byte aligned
// start): one streaming pass, 16-byte loads, 8 in flight per lane.  Warp w takes a
// contiguous segment of the slice and appends its matches, in order, to its own buffer
// (wk, wp: kWarpCap entries per warp) with warp scans only; the buffers are then
// concatenated in warp order.  Returns -1, having written nothing to (ck, cp), if a warp's
// matches would overflow its buffer.
__device__ __forceinline__ int compact_stream(const Slice& sl, uint32_t thr, uint32_t* ck, uint32_t* cp,
                                              uint32_t* wk, uint32_t* wp, Smem& sm) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int n = sl.end - sl.begin, n4 = n >> 2;
    const int seg4 = (n4 + NW - 1) / NW;                     // 16-byte groups per warp
    const int q_begin = min(warp * seg4, n4), q_end = min(q_begin + seg4, n4);
    const float4* src = reinterpret_cast<const float4*>(sl.s + sl.begin);
    uint32_t* mk = wk + warp * kWarpCap;
    uint32_t* mp = wp + warp * kWarpCap;
    int cnt = 0;
    bool over = false;
    auto append = [&](const uint32_t (&k)[4], int first, int valid) {   // keys first .. first+3, in order
        int c = 0;
#pragma unroll
        for (int e = 0; e < 4; ++e) c += (e < valid) && k[e] >= thr;
        int incl = c;
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, incl, d);
            if (lane >= d) incl += y;
        }
        const int tot = __shfl_sync(0xffffffffu, incl, 31);
        if (cnt + tot > kWarpCap) {
            over = true;
        } else if (c) {
            int o = cnt + incl - c;
#pragma unroll
            for (int e = 0; e < 4; ++e)
                if ((e < valid) && k[e] >= thr) { mk[o] = k[e]; mp[o] = static_cast<uint32_t>(first + e); ++o; }
        }
        cnt += tot;
    };
    for (int q0 = q_begin; q0 < q_end && !over; q0 += 8 * 32) {
        float4 x[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int q = q0 + u * 32 + lane;
            x[u] = q < q_end ? __ldg(src + q) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int q = q0 + u * 32 + lane;
            const uint32_t k[4] = {ord_key(x[u].x), ord_key(x[u].y), ord_key(x[u].z), ord_key(x[u].w)};
            append(k, sl.begin + 4 * q, q < q_end ? 4 : 0);
        }
    }
    if (warp == NW - 1 && !over && 4 * n4 < n) {               // the last 1..3 keys, after every segment
        uint32_t k[4] = {0u, 0u, 0u, 0u};
        const int rest = n - 4 * n4;
        if (lane == 0)
            for (int e = 0; e < rest; ++e) k[e] = sl.key(sl.begin + 4 * n4 + e);
        append(k, sl.begin + 4 * n4, lane == 0 ? rest : 0);
    }
    if (threadIdx.x == 0) sm.found_above = 0;                // overflow flag
    __syncthreads();
    if (over && lane == 0) sm.found_above = 1;
    const int wbase = block_excl_scan(lane == 0 ? cnt : 0, sm);
    const int total = sm.total;
    if (sm.found_above) return -1;
    const int base = __shfl_sync(0xffffffffu, wbase, 0);
    for (int e = lane; e < cnt; e += 32) {
        ck[base + e] = mk[e];
        cp[base + e] = mp[e];
    }
    __syncthreads();
    return total;
}

// Bin of h[0..nb) (bins ascending in key) holding the k-th largest key: out[0] = bin,
// out[1] = keys in the bins above it, out[2] = keys in it.  Chunks of 32 bins are summed by
// warps (conflict-free reads), the chunk sums scanned by the block, the chunk found scanned
// by one warp.  Whole CTA; nb a power of two <= kMaxBins; uses sm.lhist as chunk sums.
__device__ __forceinline__ void find_bin(const int* h, int nb, int k, Smem& sm, int* out) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int nch = (nb + 31) / 32;                          // chunk c: bins nb-1-32c-31 .. nb-1-32c
    int* csum = sm.lhist;
    for (int c = warp; c < nch; c += NW) {
        const int bin = nb - 1 - (c * 32 + lane);
        const int v = __reduce_add_sync(0xffffffffu, bin >= 0 ? h[bin] : 0);
        if (lane == 0) csum[c] = v;
    }
    __syncthreads();
    const int cv = static_cast<int>(threadIdx.x) < nch ? csum[threadIdx.x] : 0;
    const int above = block_excl_scan(cv, sm);
    if (static_cast<int>(threadIdx.x) < nch && above < k && above + cv >= k) {
        sm.found_bin = threadIdx.x;
        sm.found_above = above;
    }
    __syncthreads();
    if (warp == 0) {
        const int c = sm.found_bin;
        const int bin = nb - 1 - (c * 32 + lane);
        const int v = bin >= 0 ? h[bin] : 0;
        int incl = v;
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, incl, d);
            if (lane >= d) incl += y;
        }
        const int ab = sm.found_above + incl - v;
        if (v > 0 && ab < k && ab + v >= k) {
            out[0] = bin;
            out[1] = ab;
            out[2] = v;
        }
    }
    __syncthreads();
}

// The k-th largest (k >= 1) of the n keys g[] that match prefix under mask, resolved
// 8 bits at a time (bits below `shift`) with the histogram sm.lhist; whole CTA.
__device__ __forceinline__ uint32_t local_kth(const uint32_t* g, int n, uint32_t prefix, uint32_t mask, int shift,
                                              int k, Smem& sm) {
    int* hist = sm.lhist;
#pragma unroll 1
    for (int top = shift - 1; top >= 0;) {
        const int width = min(8, top + 1);
        const int sh = top - width + 1;
        const int nb = 1 << width;
        for (int i = threadIdx.x; i < nb; i += NT) hist[i] = 0;
        __syncthreads();
        // keys sharing a prefix crowd few bins: lanes with the same bin add once together
        for (int e0 = 0; e0 < n; e0 += NT) {
            const int e = e0 + threadIdx.x;
            const uint32_t key = e < n ? g[e] : 0u;
            const bool in = e < n && (key & mask) == prefix;
            const int bn = in ? static_cast<int>((key >> sh) & (nb - 1)) : -1;
            const uint32_t peers = __match_any_sync(0xffffffffu, bn);
            if (in && (__ffs(peers) - 1) == (threadIdx.x & 31)) atomicAdd(&hist[bn], __popc(peers));
        }
        __syncthreads();
        const int bin = nb - 1 - static_cast<int>(threadIdx.x);        // one bin per thread, descending
        const int c = bin >= 0 ? hist[bin] : 0;
        const int above = block_excl_scan(c, sm);
        if (c > 0 && above < k && above + c >= k) {
            sm.found_bin = bin;
            sm.found_above = above;
        }
        __syncthreads();
        prefix |= static_cast<uint32_t>(sm.found_bin) << sh;
        mask |= static_cast<uint32_t>(nb - 1) << sh;
        k -= sm.found_above;
        __syncthreads();                                   // found_bin is rewritten next digit
        top = sh - 1;
    }
    return prefix;
}

template <int CS>
__global__ void __launch_bounds__(NT, 2) select_kernel(SelectArgs a, int cache_keys) {
    constexpr int cs = CS;
    extern __shared__ uint32_t dsm[];
    uint32_t* key_cache = dsm;                                 // [cache_keys]
    uint32_t* cand_key = dsm + cache_keys;                     // [kCandCap]
    uint32_t* cand_pos = cand_key + kCandCap;                  // [kCandCap]
    uint32_t* warp_buf = cand_pos + kCandCap;                  // [2][NW][kWarpCap] when cache_keys == 0
    __shared__ Smem sm;
    cg::cluster_group cluster = cg::this_cluster();
    const int rank = static_cast<int>(cluster.block_rank());
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int row = blockIdx.x / cs;
    const int b = row / a.n_q, r = row % a.n_q;
    const int p = checked_pos(a.q_pos0[b] + r, a.max_ctx, a.status);
    int32_t* out = a.idx + static_cast<size_t>(row) * a.idx_stride;
    const int W = a.window;
    const int n_cand = max(p - W + 1, 0);
    const int w0 = n_cand;
    const int bs = a.block_size < 1 ? 1 : a.block_size;
    const int n_keys = (n_cand + bs - 1) / bs;                    // tokens or blocks
    const int K = bs == 1 ? min(a.budget, n_cand) : min(a.budget / bs, n_keys);
    const bool take_all = (K >= n_keys);
    const bool take_none = (K <= 0);
    auto remote = [&](auto* ptr, int rr) { return cs == 1 ? ptr : cluster.map_shared_rank(ptr, rr); };

    Slice sl;
    sl.s = a.scores + static_cast<size_t>(row) * a.score_ld;
    sl.bs = bs;
    sl.n_cand = n_cand;
    const int per = ((n_keys + cs - 1) / cs + 3) & ~3;
    sl.begin = min(rank * per, n_keys);
    sl.end = min(sl.begin + per, n_keys);
    sl.cache = nullptr;

    // ---- 1. cache the slice's keys (when they fit) and find the row's key range; a slice
    // read from global memory skips this pass and takes the first digit at the top bits
    uint32_t lo = 0xffffffffu, hi = 0u;
    const bool cached = per <= cache_keys;
    if (!take_all && !take_none && !cached && warp == 0) {
        // a streamed slice is read twice (first digit, then compaction): ask for all of it in
        // L2 at once (bulk prefetch, 16-byte aligned pieces inside the slice) so that the
        // first pass is not limited by the loads this CTA keeps in flight
        const int t0 = sl.begin * bs, t1 = min(sl.end * bs, n_cand);
        const uintptr_t b0 = (reinterpret_cast<uintptr_t>(sl.s + t0) + 15) & ~uintptr_t(15);
        const uintptr_t b1 = reinterpret_cast<uintptr_t>(sl.s + t1) & ~uintptr_t(15);
        if (b1 > b0) {
            const uintptr_t step = ((b1 - b0 + 31) / 32 + 15) & ~uintptr_t(15);
            const uintptr_t c0 = b0 + lane * step;
            if (c0 < b1) {
                const uint32_t n = static_cast<uint32_t>(min(step, b1 - c0));
                asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(c0), "r"(n) : "memory");
            }
        }
    }
    if (!take_all && !take_none && !cached) {
        lo = 0u;
        hi = 0xffffffffu;
    }
    if (!take_all && !take_none && cached) {
        if (cached && bs > 1) {
            // block keys: one warp per block, max over its tokens by shuffles
            for (int bb = sl.begin + warp; bb < sl.end; bb += NW) {
                const int e = min((bb + 1) * bs, n_cand);
                float m = -INFINITY;
                for (int j = bb * bs + lane; j < e; j += 32) m = fmaxf(m, sl.s[j]);
                m = warp_max(m);
                const uint32_t k = ord_key(m);
                if (lane == 0) key_cache[bb - sl.begin] = k;
                lo = min(lo, k);
                hi = max(hi, k);
            }
        } else {
            for_keys_fast(sl, [&](int i, uint32_t key) {
                if (cached) key_cache[i - sl.begin] = key;
                lo = min(lo, key);
                hi = max(hi, key);
            });
        }
        if (cached) sl.cache = key_cache;
        lo = __reduce_min_sync(0xffffffffu, lo);
        hi = __reduce_max_sync(0xffffffffu, hi);
        if (lane == 0) { sm.wlo[warp] = lo; sm.whi[warp] = hi; }
        __syncthreads();
        if (threadIdx.x == 0) {
            uint32_t l = sm.wlo[0], h = sm.whi[0];
            for (int w = 1; w < NW; ++w) { l = min(l, sm.wlo[w]); h = max(h, sm.whi[w]); }
            sm.range[0] = l; sm.range[1] = h;
        }
        cluster.sync();                            // [barrier 1] ranges written once
        // one thread per remote word, then shared: not every thread reading every peer
        if (threadIdx.x < 2 * cs) sm.bcast[threadIdx.x] = remote(sm.range, threadIdx.x >> 1)[threadIdx.x & 1];
        __syncthreads();
        lo = 0xffffffffu; hi = 0u;
#pragma unroll
        for (int rr = 0; rr < cs; ++rr) {
            lo = min(lo, sm.bcast[2 * rr]);
            hi = max(hi, sm.bcast[2 * rr + 1]);
        }
        __syncthreads();                           // bcast is reused
    }

    uint32_t tau = 0;
    int need_eq = 0;
    bool use_cands = false;
    int n_my = 0;                                  // this CTA's candidate count
    int out_base = 0, eq_base = 0;                 // tokens / equal keys before this CTA's
    bool offsets_known = false;
    if (!take_all && !take_none) {
        if (lo == hi) {                            // every key has the same value
            tau = hi;
            need_eq = K;
        } else {
            const int hb = 31 - __clz(lo ^ hi);    // highest bit where the keys differ
            uint32_t mask = ~((2u << hb) - 1u);    // (hb == 31 gives 0: nothing shared)
            uint32_t prefix = hi & mask;
            int k_rem = K;
            // streamed slices (no range pass) take the top 13 bits: importance values span few
            // octaves, so bins of an eighth of an octave keep bin b1 short; the histogram and
            // rank 0's sum live in the warp buffers, which are free until the compaction
            int width = cached ? min(11, hb + 1) : kStreamBits;
            int shift = hb - width + 1;
            const int nb = 1 << width;
            // ---- 2. first digit over every key; rank 0 sums the cluster's histograms
            int* hist = cached ? sm.hist[0] : reinterpret_cast<int*>(warp_buf);
            for (int i = threadIdx.x; i < nb; i += NT) hist[i] = 0;
            __syncthreads();
            for_keys_fast(sl, [&](int, uint32_t key) { atomicAdd(&hist[(key >> shift) & (nb - 1)], 1); });
            cluster.sync();                        // [barrier 2] histograms complete
            if (rank == 0) {
                // the cluster's histogram summed into hist[1] with coalesced remote reads
                // (consecutive threads, consecutive bins), then scanned from there
                int* hsum = cached ? sm.hist[1] : reinterpret_cast<int*>(warp_buf) + kMaxBins;
                if (CS == 1) {
                    hsum = hist;
                } else {
                    for (int bin = threadIdx.x; bin < nb; bin += NT) {
                        int v[CS];
#pragma unroll
                        for (int rr = 0; rr < CS; ++rr) v[rr] = remote(hist, rr)[bin];
                        int c = 0;
#pragma unroll
                        for (int rr = 0; rr < CS; ++rr) c += v[rr];
                        hsum[bin] = c;
                    }
                    __syncthreads();
                }
                find_bin(hsum, nb, k_rem, sm, sm.dec);
                // candidate lists fit when K + |bin b1| <= kCandCap (a CTA holds at most the
                // row's keys above b1 (< K) plus those in b1); the gather buffer holds |b1|
                if (threadIdx.x == 0) sm.dec[3] = (K + sm.dec[2] <= kCandCap && sm.dec[2] <= 2 * NBINS) ? 1 : 0;
            }
            cluster.sync();                        // [barrier 3] decision published
            if (threadIdx.x < 4) sm.bcast[threadIdx.x] = static_cast<uint32_t>(remote(sm.dec, 0)[threadIdx.x]);
            __syncthreads();
            const int b1 = static_cast<int>(sm.bcast[0]), above1 = static_cast<int>(sm.bcast[1]);
            use_cands = sm.bcast[3] != 0;
            __syncthreads();
            prefix |= static_cast<uint32_t>(b1) << shift;
            mask |= static_cast<uint32_t>(nb - 1) << shift;
            k_rem -= above1;
            if (use_cands) {
                // ---- 3. candidates: this CTA's keys at or above bin b1, in position order;
                // its bin-b1 keys (fewer than kCandCap - K on this path) copied to hist[1]
                if (threadIdx.x == 0) { sm.ncand2 = 0; sm.nb1 = 0; }
                if (sl.cache) {
                    n_my = compact_cached(sl, prefix, cand_key, cand_pos, sm);
                } else {
                    n_my = -1;
                    if (cache_keys == 0 && bs == 1 && (reinterpret_cast<uintptr_t>(sl.s + sl.begin) & 15u) == 0)
                        n_my = compact_stream(sl, prefix, cand_key, cand_pos, warp_buf, warp_buf + NW * kWarpCap, sm);
                    if (n_my < 0) n_my = compact_ordered(sl, prefix, cand_key, cand_pos, sm);
                }
                uint32_t* b1k = reinterpret_cast<uint32_t*>(sm.hist[1]);
                for (int e0 = 0; e0 < n_my; e0 += NT) {              // one counter update per warp
                    const int e = e0 + threadIdx.x;
                    const uint32_t key = e < n_my ? cand_key[e] : 0u;
                    const bool in = e < n_my && (key & mask) == prefix;
                    const uint32_t bal = __ballot_sync(0xffffffffu, in);
                    int base = 0;
                    if (lane == 0 && bal) base = atomicAdd(&sm.nb1, __popc(bal));
                    base = __shfl_sync(0xffffffffu, base, 0);
                    if (in) b1k[base + __popc(bal & ((1u << lane) - 1u))] = key;
                }
                __syncthreads();
                if (threadIdx.x == 0) { sm.pub[0] = n_my; sm.pub[1] = sm.nb1; }
                cluster.sync();                    // [barrier 4] candidate lists complete
                // ---- 4. rank 0: the bin-b1 keys of the whole cluster, sorted descending, give
                // tau exactly; then every CTA's counts and output offsets
                if (rank == 0) {
                    uint32_t* g = reinterpret_cast<uint32_t*>(&sm.hist[0][0]);    // the cluster's bin-b1 keys
                    // every CTA's counts in one batch, then one flat copy of all bin-b1 keys
                    int nb1[kMaxCluster], na[kMaxCluster], off[kMaxCluster + 1];
#pragma unroll
                    for (int rr = 0; rr < CS; ++rr) {
                        const int* pb = remote(sm.pub, rr);
                        na[rr] = pb[0];
                        nb1[rr] = pb[1];
                    }
                    off[0] = 0;
#pragma unroll
                    for (int rr = 0; rr < CS; ++rr) off[rr + 1] = off[rr] + nb1[rr];
#pragma unroll
                    for (int rr = 0; rr < CS; ++rr) {
                        const uint32_t* bk = remote(b1k, rr);
                        for (int e = threadIdx.x; e < nb1[rr]; e += NT) g[off[rr] + e] = bk[e];
                    }
                    if (threadIdx.x == 0) sm.ncand2 = off[CS];
                    if (threadIdx.x < kMaxCluster) { sm.cnt_gt[threadIdx.x] = 0; sm.cnt_eq[threadIdx.x] = 0; }
                    __syncthreads();
                    const int n1 = sm.ncand2;
                    const uint32_t t = local_kth(g, n1, prefix, mask, shift, k_rem, sm);
                    // per CTA: its candidates above bin b1, plus its bin-b1 keys (its segment
                    // of g) above / equal to t
#pragma unroll
                    for (int rr = 0; rr < CS; ++rr) {
                        int cg_ = 0, ce = 0;
                        for (int e = off[rr] + threadIdx.x; e < off[rr + 1]; e += NT) {
                            const uint32_t key = g[e];
                            cg_ += key > t;
                            ce += key == t;
                        }
                        cg_ = __reduce_add_sync(0xffffffffu, cg_);
                        ce = __reduce_add_sync(0xffffffffu, ce);
                        if (threadIdx.x == 0) cg_ += na[rr] - nb1[rr];
                        if (lane == 0) {
                            if (cg_) atomicAdd(&sm.cnt_gt[rr], cg_);
                            if (ce) atomicAdd(&sm.cnt_eq[rr], ce);
                        }
                    }
                    __syncthreads();
                    if (threadIdx.x == 0) {
                        int total_gt = 0;
                        for (int rr = 0; rr < cs; ++rr) total_gt += sm.cnt_gt[rr];
                        const int neq = K - total_gt;          // equal keys still to take
                        int ob = 0, eb = 0;
                        for (int rr = 0; rr < cs; ++rr) {
                            sm.table[rr][0] = ob;
                            sm.table[rr][1] = eb;
                            ob += (sm.cnt_gt[rr] + max(0, min(sm.cnt_eq[rr], neq - eb))) * bs;
                            eb += sm.cnt_eq[rr];
                        }
                        sm.dec[4] = static_cast<int>(t);
                        sm.dec[5] = neq;
                    }
                }
                cluster.sync();                    // [barrier 5] threshold and offsets published
                if (threadIdx.x < 2) sm.bcast[threadIdx.x] = static_cast<uint32_t>(remote(sm.dec, 0)[4 + threadIdx.x]);
                else if (threadIdx.x < 4)
                    sm.bcast[threadIdx.x] = static_cast<uint32_t>(remote(&sm.table[0][0], 0)[2 * rank + threadIdx.x - 2]);
                __syncthreads();
                tau = sm.bcast[0];
                need_eq = static_cast<int>(sm.bcast[1]);
                out_base = static_cast<int>(sm.bcast[2]);
                eq_base = static_cast<int>(sm.bcast[3]);
                offsets_known = true;
            } else {
                // ---- 4'. candidate lists would not fit: remaining digits over every key
                int hbuf = 1;
#pragma unroll 1
                for (int top = shift - 1; top >= 0;) {
                    width = min(11, top + 1);
                    shift = top - width + 1;
                    radix_digit<CS>(cluster, sm, hbuf, shift, width, prefix, mask, k_rem, [&](auto add) {
                        for_keys(sl, [&](int, uint32_t key, bool valid) { if (valid) add(key); });
                    });
                    hbuf ^= 1;
                    prefix |= static_cast<uint32_t>(sm.found_bin) << shift;
                    mask |= static_cast<uint32_t>((1 << width) - 1) << shift;
                    k_rem -= sm.found_above;
                    __syncthreads();
                    top = shift - 1;
                }
                tau = prefix;
                need_eq = k_rem;
            }
        }
    }

    // ---- 5. (all-equal and fallback paths) this CTA's counts and cluster-wide offsets
    if (!offsets_known) {
        int gt = 0, eq = 0;
        if (!take_all && !take_none)
            for_keys(sl, [&](int, uint32_t key, bool valid) {
                gt += valid && key > tau;
                eq += valid && key == tau;
            });
        block_excl_scan(gt, sm);
        const int t_gt = sm.total;
        block_excl_scan(eq, sm);
        const int t_eq = sm.total;
        if (threadIdx.x == 0) { sm.counts[0] = t_gt; sm.counts[1] = t_eq; }
        cluster.sync();                            // counts written once; the final barrier
                                                   // keeps them alive while they are read
        for (int rr = 0; rr < rank; ++rr) {
            const int* c = cluster.map_shared_rank(sm.counts, rr);
            int keys_sel;
            if (take_all) {
                const int rb = min(rr * per, n_keys), re = min(rb + per, n_keys);
                keys_sel = re - rb;
            } else if (take_none) {
                keys_sel = 0;
            } else {
                keys_sel = c[0] + max(0, min(c[1], need_eq - eq_base));
            }
            // lower ranks own only whole blocks (a partial last block belongs to the CTA
            // owning the row's last key, and never precedes another CTA's keys)
            out_base += keys_sel * bs;
            eq_base += c[1];
        }
    }

    // ---- 6. ordered write of this CTA's selection
    int written = out_base;
    if (!take_none) {
        if (use_cands) {
            written = ordered_write(
                sm, sl, n_my, [&](int e) { return static_cast<int>(cand_pos[e]); },
                [&](int e) { return cand_key[e]; }, tau, need_eq, false, eq_base, written, out);
        } else {
            written = ordered_write(
                sm, sl, sl.end - sl.begin, [&](int e) { return sl.begin + e; },
                [&](int e) { return sl.key(sl.begin + e); }, tau, need_eq, take_all, eq_base, written, out);
        }
    }

    // the forced window after all global picks (every window position exceeds every
    // candidate), written by the CTA owning the last candidate key: its running count
    // is exact (a partial last block is counted with its true length)
    const int writer = n_keys > 0 ? min((n_keys - 1) / per, cs - 1) : 0;
    if (rank == writer) {
        for (int j = w0 + threadIdx.x; j <= p; j += NT) out[written + (j - w0)] = j;
        const int total = written + (p - w0 + 1);
        for (int i = total + threadIdx.x; i < a.idx_stride; i += NT) out[i] = -1;
        if (threadIdx.x == 0) a.cnt[row] = total;
    }
    cluster.sync();                                // no CTA leaves while its memory may be read
}

int pick_cluster(int rows, int64_t max_keys) {
    // enough rows to fill the GPU: one CTA per row (keys streamed when they do not fit)
    if (rows >= 2 * num_sms()) return 1;
    int cs = 1;
    while (cs < 8 && (max_keys + cs - 1) / cs > kSmemKeys) cs *= 2;
    const int target = 2 * num_sms();
    while (cs < 8 && static_cast<int64_t>(rows) * cs * 2 <= target && max_keys / (cs * 2) >= 1024)
        cs *= 2;
    // a few rows still streamed from global memory by 8 CTAs each: 16 per row
    if (cs == 8 && (max_keys + 7) / 8 > kSmemKeys && rows * 16 <= num_sms()) cs = 16;
    return cs;
}

}  // namespace

cudaError_t launch_select(const SelectArgs& a, cudaStream_t st) {
    if (a.rows <= 0) return cudaSuccess;
    const int bs = a.block_size < 1 ? 1 : a.block_size;
    const int64_t max_keys = (a.max_ctx + bs - 1) / bs;
    int cs = pick_cluster(a.rows, max_keys);
    for (;;) {
        const int64_t per = ((max_keys + cs - 1) / cs + 3) & ~int64_t(3);
        const int cache_keys = per <= kSmemKeys ? static_cast<int>(per) : 0;
        const size_t smem = (static_cast<size_t>(cache_keys) + 2 * kCandCap + (cache_keys == 0 ? 2 * NW * kWarpCap : 0)) *
                            sizeof(uint32_t);
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(static_cast<unsigned>(a.rows) * cs);
        cfg.blockDim = dim3(NT);
        cfg.dynamicSmemBytes = smem;
        cfg.stream = st;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = cs;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        auto prepare = [&](auto kern) {
            cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
            if (e == cudaSuccess && cs > 8) e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
            return e;
        };
        auto launch = [&](auto kern) {
            cudaError_t e = prepare(kern);
            if (e != cudaSuccess) return e;
            return cudaLaunchKernelEx(&cfg, kern, a, cache_keys);
        };
        if (cs == 16) {
            // a 16-CTA cluster must fit a GPC with this shared memory; otherwise 8
            int n = 0;
            if (prepare(select_kernel<16>) != cudaSuccess ||
                cudaOccupancyMaxActiveClusters(&n, select_kernel<16>, &cfg) != cudaSuccess || n < 1) {
                cudaGetLastError();
                cs = 8;
                continue;
            }
            return launch(select_kernel<16>);
        }
        switch (cs) {
            case 1: return launch(select_kernel<1>);
            case 2: return launch(select_kernel<2>);
            case 4: return launch(select_kernel<4>);
            default: return launch(select_kernel<8>);
        }
    }
}

}  // namespace hs2
