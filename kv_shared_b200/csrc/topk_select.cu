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
// One CTA per row.  The K-th best key is found exactly by a three-digit radix
// select (11 + 11 + 10 bits) on order-preserving uint32 images of the fp32
// values; then one ascending pass writes every candidate above the threshold
// and the first (K - #above) candidates equal to it, which is the lower-index
// tie rule, already in ascending order.  Integer work only after the key map.
#include "common.cuh"
#include "internal.h"

namespace hs2 {
namespace {

constexpr int NT = 1024;
constexpr int NW = NT / 32;

__device__ __forceinline__ uint32_t ord_key(float f) {
    const uint32_t u = __float_as_uint(f);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Block-wide exclusive scan of one int per thread; returns the exclusive prefix
// and writes the total to *total.  All threads must call it.
__device__ __forceinline__ int block_excl_scan(int v, int* warp_tot, int* total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) warp_tot[warp] = x;
    __syncthreads();
    if (warp == 0) {
        int w = lane < NW ? warp_tot[lane] : 0;
        int s = w;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, s, o);
            if (lane >= o) s += y;
        }
        if (lane < NW) warp_tot[lane] = s - w;      // exclusive warp offsets
        if (lane == NW - 1) *total = s;
    }
    __syncthreads();
    const int r = warp_tot[warp] + x - v;
    __syncthreads();
    return r;
}

struct Smem {
    int hist[2048];
    int warp_tot[NW];
    int total;
    int found_bin;
    int found_above;
};

// Exact K-th largest key among n keys given by get(i) (K in [1, n-1]).
// Returns the threshold key; *need_eq = how many keys equal to it are taken.
template <typename Get>
__device__ uint32_t radix_threshold(Get get, int n, int K, Smem& sm, int* need_eq) {
    uint32_t prefix = 0, mask = 0;
    int k_rem = K;
    const int shifts[3] = {21, 10, 0};
    const int widths[3] = {11, 11, 10};
#pragma unroll 1
    for (int pass = 0; pass < 3; ++pass) {
        const int shift = shifts[pass], nb = 1 << widths[pass];
        for (int i = threadIdx.x; i < nb; i += NT) sm.hist[i] = 0;
        __syncthreads();
        for (int i = threadIdx.x; i < n; i += NT) {
            const uint32_t key = get(i);
            if ((key & mask) == prefix) atomicAdd(&sm.hist[(key >> shift) & (nb - 1)], 1);
        }
        __syncthreads();
        // suffix counts from the top: thread j owns bins [j*per, (j+1)*per) counted from the top
        const int per = nb / NT;                       // 2 (first two passes) or 1
        int local = 0;
        for (int q = 0; q < per; ++q) local += sm.hist[nb - 1 - (threadIdx.x * per + q)];
        const int above = block_excl_scan(local, sm.warp_tot, &sm.total);
        if (above < k_rem && above + local >= k_rem) {
            int acc = above;
            for (int q = 0; q < per; ++q) {
                const int bin = nb - 1 - (threadIdx.x * per + q);
                const int c = sm.hist[bin];
                if (acc + c >= k_rem) { sm.found_bin = bin; sm.found_above = acc; break; }
                acc += c;
            }
        }
        __syncthreads();
        prefix |= static_cast<uint32_t>(sm.found_bin) << shift;
        mask |= static_cast<uint32_t>(nb - 1) << shift;
        k_rem -= sm.found_above;
        __syncthreads();
    }
    *need_eq = k_rem;
    return prefix;
}

__global__ void __launch_bounds__(NT) select_kernel(SelectArgs a) {
    __shared__ Smem sm;
    const int row = blockIdx.x;
    const int b = row / a.n_q, r = row % a.n_q;
    const int p = checked_pos(a.q_pos0[b] + r, a.max_ctx, a.status);
    const float* s = a.scores + static_cast<size_t>(row) * a.score_ld;
    int32_t* out = a.idx + static_cast<size_t>(row) * a.idx_stride;
    const int W = a.window;
    const int n_cand = max(p - W + 1, 0);
    const int w0 = max(p - W + 1, 0);
    int written = 0;

    if (a.block_size <= 1) {
        const int K = min(a.budget, n_cand);
        if (K > 0) {
            uint32_t tau = 0;
            int need_eq = 0;
            if (K < n_cand) {
                tau = radix_threshold([&](int i) { return ord_key(s[i]); }, n_cand, K, sm, &need_eq);
            }
            // ascending compaction: 4 consecutive candidates per thread per round
            int eq_seen = 0;
            for (int base = 0; base < n_cand; base += 4 * NT) {
                const int j0 = base + 4 * threadIdx.x;
                int gt = 0, eq = 0;
                uint32_t keys[4];
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int j = j0 + u;
                    keys[u] = (j < n_cand) ? ord_key(s[j]) : 0u;
                    if (j < n_cand && K < n_cand) {
                        gt += keys[u] > tau;
                        eq += keys[u] == tau;
                    }
                }
                const int eq_before = block_excl_scan(eq, sm.warp_tot, &sm.total);
                const int eq_round = sm.total;
                // number selected by this thread
                int rank = eq_seen + eq_before, mine = 0;
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int j = j0 + u;
                    if (j >= n_cand) break;
                    bool sel;
                    if (K == n_cand) sel = true;
                    else if (keys[u] > tau) sel = true;
                    else if (keys[u] == tau) { sel = rank < need_eq; ++rank; }
                    else sel = false;
                    mine += sel;
                }
                (void)gt;
                const int pos = block_excl_scan(mine, sm.warp_tot, &sm.total);
                const int round_total = sm.total;
                rank = eq_seen + eq_before;
                int o = written + pos;
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int j = j0 + u;
                    if (j >= n_cand) break;
                    bool sel;
                    if (K == n_cand) sel = true;
                    else if (keys[u] > tau) sel = true;
                    else if (keys[u] == tau) { sel = rank < need_eq; ++rank; }
                    else sel = false;
                    if (sel) out[o++] = j;
                }
                written += round_total;
                eq_seen += eq_round;
                __syncthreads();
            }
        }
    } else {
        // block arm: block importance = max over its tokens inside the candidates,
        // recomputed on every pass (no scratch)
        const int bs = a.block_size;
        const int nb = (n_cand + bs - 1) / bs;
        const int Kb = min(a.budget / bs, nb);
        auto bkey = [&](int bb) {
            float m = -INFINITY;
            const int e = min((bb + 1) * bs, n_cand);
            for (int j = bb * bs; j < e; ++j) m = fmaxf(m, s[j]);
            return ord_key(m);
        };
        if (Kb > 0) {
            uint32_t tau = 0;
            int need_eq = 0;
            if (Kb < nb) tau = radix_threshold(bkey, nb, Kb, sm, &need_eq);
            int eq_seen = 0;
            for (int base = 0; base < nb; base += NT) {
                const int bb = base + threadIdx.x;
                const uint32_t key = bb < nb ? bkey(bb) : 0u;
                const int eq = (bb < nb && Kb < nb && key == tau) ? 1 : 0;
                const int eq_before = block_excl_scan(eq, sm.warp_tot, &sm.total);
                const int eq_round = sm.total;
                bool sel = false;
                if (bb < nb) {
                    if (Kb == nb || key > tau) sel = true;
                    else if (key == tau) sel = (eq_seen + eq_before) < need_eq;
                }
                const int ntok = sel ? (min((bb + 1) * bs, n_cand) - bb * bs) : 0;
                const int pos = block_excl_scan(ntok, sm.warp_tot, &sm.total);
                const int round_total = sm.total;
                for (int u = 0; u < ntok; ++u) out[written + pos + u] = bb * bs + u;
                written += round_total;
                eq_seen += eq_round;
                __syncthreads();
            }
        }
    }
    // forced window after the global picks (all window positions exceed every candidate)
    for (int j = w0 + threadIdx.x; j <= p; j += NT) out[written + (j - w0)] = j;
    const int total = written + (p - w0 + 1);
    for (int i = total + threadIdx.x; i < a.idx_stride; i += NT) out[i] = -1;
    if (threadIdx.x == 0) a.cnt[row] = total;
}

}  // namespace

cudaError_t launch_select(const SelectArgs& a, cudaStream_t st) {
    if (a.rows <= 0) return cudaSuccess;
    select_kernel<<<a.rows, NT, 0, st>>>(a);
    return cudaGetLastError();
}

}  // namespace hs2
