// topk_select.cu -- token-level (and block-level) selection with the forced window.
//
// Per query row at position p ("Xiaomi Unveils HySparse2 Architecture for
// MiMo-V3", section "Token-Level Sparse Selection: Precision and Efficiency
// Balance": the most recent 128 tokens are forced, plus 1,024 global tokens):
//   window = [max(0, p-W+1), p], candidates = [0, p-W],
//   global = the K best candidates by (importance desc, position asc),
//   idx    = ascending union, -1 padded; cnt = |idx|.
// Block arm (first-generation rule of the MiMo-V3 news flash: a group of 64 is
// kept whole if any of its tokens is important): blocks of `bs` positions from
// 0, block importance = max, floor(K/bs) best blocks (lower block on ties).
//
// A row is handled by a cluster of CS CTAs (CS = 1..8); CTA r owns a contiguous
// slice of the candidates and keeps their order-preserving uint32 images in
// shared memory when they fit.  The K-th best key is found exactly by a radix
// select over the bits below those every key of the row shares (from the row's
// key range), at most 11 bits per digit: per digit every CTA builds a histogram
// of its slice, the cluster's histograms are summed over distributed shared
// memory and each CTA takes the same decision.  Then every CTA writes,
// in ascending order, its keys above the threshold and its share of the first
// (K - #above) keys equal to it (the lower-index tie rule), at offsets from a
// cluster-wide prefix of the counts.  Integer work only after the key map.
#include <cooperative_groups.h>

#include "common.cuh"
#include "internal.h"

namespace cg = cooperative_groups;

namespace hs2 {
namespace {

constexpr int NT = 512;
constexpr int NW = NT / 32;
constexpr int NBINS = 2048;
constexpr int kMaxCluster = 8;
constexpr int kSmemKeys = 32768;          // keys cached per CTA (128 KB)

__device__ __forceinline__ uint32_t ord_key(float f) {
    const uint32_t u = __float_as_uint(f);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

struct Smem {
    int hist[NBINS];
    int warp_tot[NW];
    int total;
    int found_bin;
    int found_above;
    int counts[2];              // this CTA's (#above, #equal) for the compaction
    uint32_t wlo[NW], whi[NW];  // per-warp key range
    uint32_t range[2];          // this CTA's key range (read by the cluster)
};

// Block-wide exclusive scan of one int per thread; *total receives the sum.
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
    int n_cand;                // candidates of the row
    int begin, end;            // this CTA's key range (tokens or blocks)
    uint32_t* cache;           // shared-memory copy or nullptr
    __device__ __forceinline__ uint32_t compute(int i) const {
        if (bs == 1) return ord_key(s[i]);
        float m = -INFINITY;
        const int e = min((i + 1) * bs, n_cand);
        for (int j = i * bs; j < e; ++j) m = fmaxf(m, s[j]);
        return ord_key(m);
    }
    __device__ __forceinline__ uint32_t key(int i) const { return cache ? cache[i - begin] : compute(i); }
};

// Visits every key of the slice as f(i, key, valid) with 8 independent loads in
// flight per thread; all threads of the block make the same number of calls (keys
// past the slice come with valid = false), so f may use warp-wide primitives.
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

__global__ void __launch_bounds__(NT) select_kernel(SelectArgs a, int cs, int cache_keys) {
    extern __shared__ uint32_t key_cache[];
    __shared__ Smem sm;
    cg::cluster_group cluster = cg::this_cluster();
    const int rank = static_cast<int>(cluster.block_rank());
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

    Slice sl;
    sl.s = a.scores + static_cast<size_t>(row) * a.score_ld;
    sl.bs = bs;
    sl.n_cand = n_cand;
    const int per = ((n_keys + cs - 1) / cs + 3) & ~3;
    sl.begin = min(rank * per, n_keys);
    sl.end = min(sl.begin + per, n_keys);
    sl.cache = nullptr;
    if (per <= cache_keys) {
        if (bs == 1) {
            // token keys: 8 coalesced loads in flight per thread
            for_keys(sl, [&](int i, uint32_t key, bool valid) { if (valid) key_cache[i - sl.begin] = key; });
        } else {
            // block keys: one warp per block, max over its tokens by shuffles
            const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
            for (int bb = sl.begin + warp; bb < sl.end; bb += NW) {
                const int e = min((bb + 1) * bs, n_cand);
                float m = -INFINITY;
                for (int j = bb * bs + lane; j < e; j += 32) m = fmaxf(m, sl.s[j]);
                m = warp_max(m);
                if (lane == 0) key_cache[bb - sl.begin] = ord_key(m);
            }
        }
        sl.cache = key_cache;
    }
    __syncthreads();

    uint32_t tau = 0;
    int need_eq = 0;
    const bool take_all = (K >= n_keys);
    const bool take_none = (K <= 0);
    if (!take_all && K > 0) {
        // key range of the row: the digits start right below the bits every key shares
        // (importance values crowd into a few binades; a fixed top digit would put them
        // into a handful of bins)
        uint32_t lo = 0xffffffffu, hi = 0u;
        for_keys(sl, [&](int, uint32_t key, bool valid) {
            if (valid) { lo = min(lo, key); hi = max(hi, key); }
        });
        lo = __reduce_min_sync(0xffffffffu, lo);
        hi = __reduce_max_sync(0xffffffffu, hi);
        if ((threadIdx.x & 31) == 0) { sm.wlo[threadIdx.x >> 5] = lo; sm.whi[threadIdx.x >> 5] = hi; }
        __syncthreads();
        if (threadIdx.x == 0) {
            uint32_t l = sm.wlo[0], h = sm.whi[0];
            for (int w = 1; w < NW; ++w) { l = min(l, sm.wlo[w]); h = max(h, sm.whi[w]); }
            sm.range[0] = l; sm.range[1] = h;
        }
        cluster.sync();
        lo = 0xffffffffu; hi = 0u;
        for (int rr = 0; rr < cs; ++rr) {
            const uint32_t* rg = cluster.map_shared_rank(sm.range, rr);
            lo = min(lo, rg[0]);
            hi = max(hi, rg[1]);
        }
        cluster.sync();
        if (lo == hi) {                         // every candidate key is the same value
            tau = hi;
            need_eq = K;
        } else {
            const int hb = 31 - __clz(lo ^ hi); // highest bit where the keys differ
            uint32_t mask = ~((2u << hb) - 1u); // (hb == 31 gives 0: nothing shared)
            uint32_t prefix = hi & mask;
            int k_rem = K;
#pragma unroll 1
            for (int top = hb; top >= 0;) {
                const int width = min(11, top + 1);
                const int shift = top - width + 1, nb = 1 << width;
                for (int i = threadIdx.x; i < nb; i += NT) sm.hist[i] = 0;
                __syncthreads();
                for_keys(sl, [&](int, uint32_t key, bool valid) {
                    if (valid && (key & mask) == prefix) atomicAdd(&sm.hist[(key >> shift) & (nb - 1)], 1);
                });
                cluster.sync();
                // counts of the whole row: sum of the cluster's histograms, from the top bin
                const int bins_per = (nb + NT - 1) / NT;               // 1..4
                int local[NBINS / NT];
                int tot = 0;
                for (int q = 0; q < bins_per; ++q) {
                    const int bin = nb - 1 - (threadIdx.x * bins_per + q);
                    int c = 0;
                    if (bin >= 0)
                        for (int rr = 0; rr < cs; ++rr) c += cluster.map_shared_rank(sm.hist, rr)[bin];
                    local[q] = c;
                    tot += c;
                }
                cluster.sync();                 // every CTA has read every histogram
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
                prefix |= static_cast<uint32_t>(sm.found_bin) << shift;
                mask |= static_cast<uint32_t>(nb - 1) << shift;
                k_rem -= sm.found_above;
                __syncthreads();
                top = shift - 1;
            }
            tau = prefix;
            need_eq = k_rem;
        }
    }

    // this CTA's counts, then cluster-wide offsets
    int gt = 0, eq = 0;
    if (!take_all && K > 0) {
        for_keys(sl, [&](int, uint32_t key, bool valid) {
            gt += valid && key > tau;
            eq += valid && key == tau;
        });
    }
    int t_gt = block_excl_scan(gt, sm);
    t_gt = sm.total;
    int t_eq = block_excl_scan(eq, sm);
    t_eq = sm.total;
    (void)t_gt;
    if (threadIdx.x == 0) { sm.counts[0] = t_gt; sm.counts[1] = t_eq; }
    cluster.sync();
    int out_base = 0, eq_base = 0;                   // tokens written / equal keys seen before this CTA
    for (int rr = 0; rr < rank; ++rr) {
        const int* c = cluster.map_shared_rank(sm.counts, rr);
        const int e_before = eq_base;
        const int take_eq = take_all ? 0 : max(0, min(c[1], need_eq - e_before));
        int keys_sel;
        if (take_all) {
            const int rb = min(rr * per, n_keys), re = min(rb + per, n_keys);
            keys_sel = re - rb;
        } else {
            keys_sel = c[0] + take_eq;
        }
        // tokens: blocks expand to bs tokens (only the row's last block is partial, and it
        // belongs to the last CTA, never to a lower rank)
        out_base += keys_sel * bs;
        eq_base += c[1];
    }
    cluster.sync();                                  // remote counts read: they may be reused

    // ascending compaction of this CTA's slice, 4 consecutive keys per thread per round
    int eq_seen = eq_base;
    int written = out_base;
    for (int base = sl.begin; base < (take_none ? sl.begin : sl.end); base += 4 * NT) {
        const int i0 = base + 4 * threadIdx.x;
        uint32_t keys[4];
        int e_cnt = 0;
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int i = i0 + u;
            keys[u] = (i < sl.end) ? sl.key(i) : 0u;
            if (i < sl.end && !take_all) e_cnt += keys[u] == tau;
        }
        const int eq_before = block_excl_scan(e_cnt, sm);
        const int eq_round = sm.total;
        int rank_eq = eq_seen + eq_before, ntok = 0;
        bool sel[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int i = i0 + u;
            sel[u] = false;
            if (i >= sl.end) continue;
            if (take_all || keys[u] > tau) sel[u] = true;
            else if (keys[u] == tau) { sel[u] = rank_eq < need_eq; ++rank_eq; }
            if (sel[u]) ntok += min((i + 1) * bs, n_cand) - i * bs;
        }
        const int pos = block_excl_scan(ntok, sm);
        const int round_total = sm.total;
        int o = written + pos;
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            if (!sel[u]) continue;
            const int i = i0 + u;
            const int e = min((i + 1) * bs, n_cand);
            for (int j = i * bs; j < e; ++j) out[o++] = j;
        }
        written += round_total;
        eq_seen += eq_round;
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
    cluster.sync();                                  // no CTA leaves while its memory may be read
}

int pick_cluster(int rows, int64_t max_keys) {
    int cs = 1;
    while (cs < kMaxCluster && (max_keys + cs - 1) / cs > kSmemKeys) cs *= 2;
    const int target = 2 * num_sms();
    while (cs < kMaxCluster && static_cast<int64_t>(rows) * cs * 2 <= target && max_keys / (cs * 2) >= 1024)
        cs *= 2;
    return cs;
}

}  // namespace

cudaError_t launch_select(const SelectArgs& a, cudaStream_t st) {
    if (a.rows <= 0) return cudaSuccess;
    const int bs = a.block_size < 1 ? 1 : a.block_size;
    const int64_t max_keys = (a.max_ctx + bs - 1) / bs;
    const int cs = pick_cluster(a.rows, max_keys);
    const int64_t per = ((max_keys + cs - 1) / cs + 3) & ~int64_t(3);
    const int cache_keys = per <= kSmemKeys ? static_cast<int>(per) : 0;
    const size_t smem = static_cast<size_t>(cache_keys) * sizeof(uint32_t);
    cudaError_t e = cudaFuncSetAttribute(select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
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
    return cudaLaunchKernelEx(&cfg, select_kernel, a, cs, cache_keys);
}

}  // namespace hs2
