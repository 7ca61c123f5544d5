/*
 * hs2_oracle.c -- plain, slow CPU oracle for the HySparse2 hybrid-block hot path.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product library links, includes or
 * calls this file; only the tests, the package's smoke check and the CPU
 * baseline leg of the benchmark do.  It shares no code, header or constant table
 * with the CUDA path.
 *
 * Every routine is the plain definition written out as loops in fp64 (fp32 only
 * where a floating-point result decides an integer code, see oracle_fp8_quantize).
 * There is no blocking, no fusion and no reordering beyond what the definition
 * states.  OpenMP is used only to run independent query rows at once.
 *
 * Sources (pages on the web, cited by title and section):
 *   [NF]  "Xiaomi's MiMo-V3 Architecture Reduces Prefill Compute by 80%"
 *         (kucoin.com news flash, single paragraph).
 *   [LB]  "Xiaomi Unveils HySparse2 Architecture for MiMo-V3: Designed to Improve
 *         Long-Context Agent Inference" (blog.lynxflow.co), sections
 *         "Two-Level KV Sharing: Enabling Prefill Early Exit" and
 *         "Token-Level Sparse Selection: Precision and Efficiency Balance".
 *   [AX]  "What HySparse2 is actually optimizing" (frontier.agentik-os.com),
 *         sections "2. Two levels of KV sharing", "3. Token-level selection and
 *         unified KV cache", "What is not documented".
 *   [AN]  "Xiaomi unveils HySparse2, reducing million-token prefill compute to
 *         about one-fifth of the baseline" (ainews.surl.tw), paragraphs on the
 *         self-/cross-decoder split, token-level selection and FP8 caches.
 *
 * Readings where the pages are silent (the pages give no scoring rule, see [AX]
 * "What is not documented"):
 *   - importance of key j for query row i = sum over query heads of the fp32/fp64
 *     softmax probability P_h[i][j] of the full-attention layer;
 *   - ties in importance go to the lower position;
 *   - the forced window holds the W most recent positions including the query's
 *     own, and the global picks come only from positions before the window, so
 *     the selected count is min(p + 1, W + K_sel);
 *   - the sparse layer runs one joint softmax over window and global picks;
 *   - no positional encoding, bias or sink; softmax scale 1/sqrt(D) unless given.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define EXPORT __attribute__((visibility("default")))

/* ------------------------------------------------------------------------- */
/* Full causal MQA attention with per-key importance.                         */
/*                                                                           */
/* [LB] "Two-Level KV Sharing" (KV Reuse paragraph): once the full layer has */
/* run, it picks the positions that matter for the later layers.  [AN]: the  */
/* compared configuration uses MQA: every query head reads one K/V head.     */
/*                                                                           */
/* q     [n_rows][H][D]   query rows of one sequence                          */
/* k, v  [n_keys][D]      the sequence's shared cache                         */
/* pos   [n_rows]         absolute position p of each row; it sees keys 0..p  */
/* o     [n_rows][H][D]   out: sum_j P_h[j] v[j]                              */
/* lse   [n_rows][H]      out: natural log-sum-exp of the scaled logits        */
/* score [n_rows][score_stride] out: score[j] = sum_h P_h[j] for j <= p, 0 else */
/* ------------------------------------------------------------------------- */
EXPORT void oracle_full_attn(int n_rows, int H, int D, int64_t n_keys,
                             const double* q, const double* k, const double* v,
                             const int64_t* pos, double scale,
                             double* o, double* lse, double* score, int64_t score_stride)
{
    #pragma omp parallel for schedule(dynamic, 1)
    for (int r = 0; r < n_rows; ++r) {
        const int64_t p = pos[r];
        const int64_t n = p + 1;                 /* causal: keys 0..p */
        double* s = (double*)malloc(sizeof(double) * (size_t)H * (size_t)n);
        const double* qr = q + (size_t)r * H * D;
        double* orow = o + (size_t)r * H * D;
        double* srow = score ? score + (size_t)r * (size_t)score_stride : NULL;
        if (srow) for (int64_t j = 0; j < score_stride; ++j) srow[j] = 0.0;
        (void)n_keys;

        /* step 1: scaled logits s_h[j] = scale * <q_h, k_j> */
        for (int h = 0; h < H; ++h)
            for (int64_t j = 0; j < n; ++j) {
                double acc = 0.0;
                for (int d = 0; d < D; ++d) acc += qr[h * D + d] * k[(size_t)j * D + d];
                s[(size_t)h * n + j] = scale * acc;
            }

        for (int h = 0; h < H; ++h) {
            const double* sh = s + (size_t)h * n;
            /* step 2: max, log-sum-exp */
            double m = -INFINITY;
            for (int64_t j = 0; j < n; ++j) if (sh[j] > m) m = sh[j];
            double sum = 0.0;
            for (int64_t j = 0; j < n; ++j) sum += exp(sh[j] - m);
            const double L = m + log(sum);
            lse[(size_t)r * H + h] = L;
            /* step 3: normalized probabilities, output, head-summed importance */
            for (int d = 0; d < D; ++d) orow[h * D + d] = 0.0;
            for (int64_t j = 0; j < n; ++j) {
                const double P = exp(sh[j] - L);
                for (int d = 0; d < D; ++d) orow[h * D + d] += P * v[(size_t)j * D + d];
                if (srow) srow[j] += P;
            }
        }
        free(s);
    }
}

/* ------------------------------------------------------------------------- */
/* Selection.                                                                 */
/*                                                                           */
/* [NF]: a budget of 1,024 picked tokens, and the latest 128 tokens are kept */
/* unconditionally by the layers that reuse the pick.  [LB] "Token-Level     */
/* Sparse Selection": a 128-token local window on top of 1,024 global picks; */
/* picks are individual tokens ([AX] section 3).  Output: ascending          */
/* positions, count returned.                                                */
/* ------------------------------------------------------------------------- */
typedef struct { double key; int64_t id; } ranked_t;

/* total order: larger key first, then smaller id */
static int cmp_ranked(const void* a, const void* b)
{
    const ranked_t* x = (const ranked_t*)a;
    const ranked_t* y = (const ranked_t*)b;
    if (x->key > y->key) return -1;
    if (x->key < y->key) return 1;
    return (x->id < y->id) ? -1 : (x->id > y->id);
}

static int cmp_i32(const void* a, const void* b)
{
    const int32_t x = *(const int32_t*)a, y = *(const int32_t*)b;
    return (x > y) - (x < y);
}

/* Token level: window Win = [max(0,p-W+1), p]; candidates Cand = [0, p-W];
 * G = first min(K_sel, |Cand|) of Cand ordered by (score desc, position asc);
 * out = sort_asc(Win u G).  Returns the count. */
EXPORT int oracle_select_tokens(int64_t p, int W, int K_sel, const double* score, int32_t* out)
{
    int c = 0;
    const int64_t n_cand = p - W + 1 > 0 ? p - W + 1 : 0;
    if (n_cand > 0 && K_sel > 0) {
        ranked_t* r = (ranked_t*)malloc(sizeof(ranked_t) * (size_t)n_cand);
        for (int64_t j = 0; j < n_cand; ++j) { r[j].key = score[j]; r[j].id = j; }
        qsort(r, (size_t)n_cand, sizeof(ranked_t), cmp_ranked);
        const int64_t g = n_cand < K_sel ? n_cand : K_sel;
        for (int64_t i = 0; i < g; ++i) out[c++] = (int32_t)r[i].id;
        free(r);
    }
    for (int64_t j = (p - W + 1 > 0 ? p - W + 1 : 0); j <= p; ++j) out[c++] = (int32_t)j;
    qsort(out, (size_t)c, sizeof(int32_t), cmp_i32);
    return c;
}

/* Block level (the first-generation rule, [NF]: importance was decided per group
 * of 64 tokens, and a group with one important member was kept in full): blocks of size bs
 * tile Cand from position 0, a block's score is the max of its tokens' scores,
 * the floor(K_sel/bs) best blocks by (block score desc, block asc) are kept
 * (only their positions inside Cand), plus the window.  Returns the count. */
EXPORT int oracle_select_blocks(int64_t p, int W, int K_sel, int bs, const double* score, int32_t* out)
{
    int c = 0;
    const int64_t n_cand = p - W + 1 > 0 ? p - W + 1 : 0;
    const int64_t nb = (n_cand + bs - 1) / bs;
    const int64_t want = K_sel / bs;
    if (nb > 0 && want > 0) {
        ranked_t* r = (ranked_t*)malloc(sizeof(ranked_t) * (size_t)nb);
        for (int64_t b = 0; b < nb; ++b) {
            double m = -INFINITY;
            for (int64_t j = b * bs; j < (b + 1) * bs && j < n_cand; ++j) if (score[j] > m) m = score[j];
            r[b].key = m; r[b].id = b;
        }
        qsort(r, (size_t)nb, sizeof(ranked_t), cmp_ranked);
        const int64_t g = nb < want ? nb : want;
        for (int64_t i = 0; i < g; ++i)
            for (int64_t j = r[i].id * bs; j < (r[i].id + 1) * bs && j < n_cand; ++j) out[c++] = (int32_t)j;
        free(r);
    }
    for (int64_t j = (p - W + 1 > 0 ? p - W + 1 : 0); j <= p; ++j) out[c++] = (int32_t)j;
    qsort(out, (size_t)c, sizeof(int32_t), cmp_i32);
    return c;
}

/* ------------------------------------------------------------------------- */
/* Sparse attention with KV Reuse.                                            */
/*                                                                           */
/* [AX] section 2: a sparse layer has no cache or selector of its own; it    */
/* reads the full layer's cache at the full layer's picks.  [AX] section 3:  */
/* window and global picks live in the same cache -> one softmax over both.  */
/* q [n_rows][H][D]; k, v [n_keys][D]; idx [n_rows][idx_stride]; cnt [n_rows] */
/* ------------------------------------------------------------------------- */
EXPORT void oracle_sparse_attn(int n_rows, int H, int D, const double* q, const double* k,
                               const double* v, const int32_t* idx, const int32_t* cnt,
                               int idx_stride, double scale, double* o, double* lse)
{
    #pragma omp parallel for schedule(dynamic, 1)
    for (int r = 0; r < n_rows; ++r) {
        const int n = cnt[r];
        const int32_t* id = idx + (size_t)r * idx_stride;
        double* s = (double*)malloc(sizeof(double) * (size_t)(n > 0 ? n : 1));
        for (int h = 0; h < H; ++h) {
            const double* qh = q + ((size_t)r * H + h) * D;
            double* oh = o + ((size_t)r * H + h) * D;
            double m = -INFINITY;
            for (int t = 0; t < n; ++t) {
                double acc = 0.0;
                for (int d = 0; d < D; ++d) acc += qh[d] * k[(size_t)id[t] * D + d];
                s[t] = scale * acc;
                if (s[t] > m) m = s[t];
            }
            double sum = 0.0;
            for (int t = 0; t < n; ++t) sum += exp(s[t] - m);
            const double L = m + log(sum);
            if (lse) lse[(size_t)r * H + h] = L;
            for (int d = 0; d < D; ++d) oh[d] = 0.0;
            for (int t = 0; t < n; ++t) {
                const double P = exp(s[t] - L);
                for (int d = 0; d < D; ++d) oh[d] += P * v[(size_t)id[t] * D + d];
            }
        }
        free(s);
    }
}

/* ------------------------------------------------------------------------- */
/* KV Bridging projection.                                                    */
/*                                                                           */
/* [LB] "Two-Level KV Sharing": the caches of the cross-decoder's full layers */
/* are projections of self-decoder activations, with a separate K/V weight    */
/* per target layer.  Reading: one matrix W [dm][2D], K from                  */
/* columns 0..D-1 and V from columns D..2D-1, no bias, no norm.               */
/* x [n][dm]; w [dm][2D]; kout, vout [n][D] (exact fp64 products)             */
/* ------------------------------------------------------------------------- */
EXPORT void oracle_bridge(int64_t n, int dm, int D, const double* x, const double* w,
                          double* kout, double* vout)
{
    #pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < n; ++t)
        for (int c = 0; c < 2 * D; ++c) {
            double acc = 0.0;
            for (int m = 0; m < dm; ++m) acc += x[(size_t)t * dm + m] * w[(size_t)m * 2 * D + c];
            if (c < D) kout[(size_t)t * D + c] = acc;
            else       vout[(size_t)t * D + (c - D)] = acc;
        }
}

/* ------------------------------------------------------------------------- */
/* Number formats.                                                            */
/* ------------------------------------------------------------------------- */

/* Round a double to the nearest bfloat16 (1 sign, 8 exponent, 7 fraction bits),
 * ties to even, returned as its 16-bit pattern.  Finite inputs within range
 * only (the cache values are O(1)).  Written from the format definition: the
 * value is scaled so that the bf16 ulp is 1, rounded with rint (ties to even in
 * the default rounding mode) and rebuilt. */
EXPORT uint16_t oracle_round_bf16(double x)
{
    if (x == 0.0) return signbit(x) ? 0x8000u : 0u;
    const uint16_t sign = signbit(x) ? 0x8000u : 0u;
    double a = fabs(x);
    int e;
    (void)frexp(a, &e);                     /* a = f * 2^e, f in [0.5, 1) */
    int ue = e - 1;                          /* a in [2^ue, 2^(ue+1)) */
    if (ue < -126) ue = -126;                /* subnormal range: fixed ulp 2^-133 */
    double q = rint(ldexp(a, 7 - ue));       /* integer mantissa incl. hidden bit */
    if (q >= 256.0) { q /= 2.0; ue += 1; }   /* rounding carried into next binade */
    uint32_t biased, frac;
    if (q < 128.0) { biased = 0; frac = (uint32_t)q; }          /* subnormal */
    else           { biased = (uint32_t)(ue + 127); frac = (uint32_t)q - 128u; }
    return (uint16_t)(sign | (biased << 7) | frac);
}

EXPORT void oracle_round_bf16_array(int64_t n, const double* x, uint16_t* out)
{
    for (int64_t i = 0; i < n; ++i) out[i] = oracle_round_bf16(x[i]);
}

/* e4m3 ("fn" variant: no infinities, 0x7F/0xFF are NaN, largest finite 448).
 * value = 2^(E-7) * (1 + M/8) for E in 1..15, and M * 2^-9 for E = 0. */
EXPORT double oracle_e4m3_decode(uint8_t c)
{
    const int E = (c >> 3) & 0xF, M = c & 7;
    double a = (E == 0) ? ldexp((double)M, -9) : ldexp(1.0 + M / 8.0, E - 7);
    return (c & 0x80) ? -a : a;
}

/* Nearest e4m3 value to y, ties to even, saturating to +-448 (finite y). */
EXPORT uint8_t oracle_e4m3_encode(float y)
{
    const uint8_t sign = signbit(y) ? 0x80 : 0;
    const double a = fabs((double)y);
    if (a >= 448.0) return sign | 0x7E;
    if (a < ldexp(1.0, -6)) {                /* subnormal step 2^-9; M = 8 is the */
        const double m = rint(a * 512.0);    /* smallest normal, code 0x08        */
        return sign | (uint8_t)m;
    }
    int e;
    (void)frexp(a, &e);
    int ue = e - 1;                          /* a in [2^ue, 2^(ue+1)), ue >= -6 */
    double m = rint((ldexp(a, -ue) - 1.0) * 8.0);
    if (m >= 8.0) { m = 0.0; ue += 1; }
    return sign | (uint8_t)(((ue + 7) << 3) | (int)m);
}

/* FP8 cache quantizer, one row (token) of D values at a time, done separately
 * for K and V.  [AN]: the 1M-token analysis uses FP8 caches; the format and
 * scaling are not given, reading: e4m3, one fp32 scale per token,
 * s = amax / 448 (s = 1 for an all-zero row), code = e4m3_rne_satfinite(x / s).
 * Both divisions are single-precision IEEE divisions so that the code decision
 * is taken in the same precision as in the kernel. */
EXPORT void oracle_fp8_quantize(int64_t n, int D, const float* x, uint8_t* codes, float* scales)
{
    for (int64_t t = 0; t < n; ++t) {
        const float* xr = x + (size_t)t * D;
        float amax = 0.0f;
        for (int d = 0; d < D; ++d) { float a = fabsf(xr[d]); if (a > amax) amax = a; }
        volatile float s = (amax > 0.0f) ? amax / 448.0f : 1.0f;
        scales[t] = s;
        for (int d = 0; d < D; ++d) {
            volatile float y = xr[d] / s;
            codes[(size_t)t * D + d] = oracle_e4m3_encode(y);
        }
    }
}

/* Dequantized value of every code times its row's scale, in fp64 (exact). */
EXPORT void oracle_fp8_dequantize(int64_t n, int D, const uint8_t* codes, const float* scales, double* out)
{
    for (int64_t t = 0; t < n; ++t)
        for (int d = 0; d < D; ++d)
            out[(size_t)t * D + d] = oracle_e4m3_decode(codes[(size_t)t * D + d]) * (double)scales[t];
}
