/*
 * gnf4_oracle.c -- CPU oracle for the grouped 4-bit MoE expert GEMM.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the plain, slow, obviously
 * correct statement of what the GPU library computes.  Only the test suite,
 * the smoke check and the benchmark's CPU legs (its CPU baseline and its
 * reference arm) may load it.  It shares no code, header, table or constant
 * generator with the CUDA path.
 *
 * Precision: quantise / dequantise in fp32 exactly as the formats define
 * them; every sum (GEMM, combine) is accumulated in fp64.
 *
 * Sources (page title, section):
 *   [README]   grouped-nf4-gemm 0.33.1 on PyPI, opening paragraphs ("LUT decode
 *              to fp32 in registers, blockwise scaling, fp32 accumulation, bf16
 *              epilogue") and "Try it on CPU right now", examples 1 and 2
 *              (NF4 [N,K] -> [N,K/2] u8 + [N,K/64] fp32; MXFP4 [..,K] ->
 *              [..,K/32,16] u8 + [..,K/32] u8 e8m0).
 *   [PATCH]    grouped-nf4-gemm releases, v0.2.6 "The patch point" (argsort of
 *              the top-k ids, gather x[idxs // k], tokens_per_expert = sizes;
 *              weighting and unsorting stay with the caller).
 *   [MOE]      grouped-nf4-gemm releases, v0.2.5 "arena -> kernel"
 *              (moe_layer_forward runs gate -> GLU -> down), and index.json,
 *              system_manifest.owns / entrypoints (swiglu among the decode
 *              glue kernels); reading C17 for the row order and activation.
 *   [ROUTER]   grouped-nf4-gemm index.json, problems_solved[5] ("router softmax
 *              and top-k" among the decode tail folded into one launch) and
 *              entrypoints (int4_b32:router_epilogue); reading C18 for ties,
 *              the optional bias and the softmax over the selected logits.
 *   [DGRAD]    grouped-nf4-gemm index.json, system_manifest.owns ("grouped packed
 *              GEMM (NF4 and native MXFP4) and its dgrad") and entrypoints
 *              (nf4_grouped:dgrad_4bit_grouped): dX = dY . W on the same stacks.
 *   [W4A8]     bw24 v0.9.0 release notes, Features ("f8f4 tile piece 1":
 *              e4m3 activation quantisation; "mixed e4m3xe2m1 mxf8f6f4 probe")
 *              and Documentation ("prefill arc design": W4A8-FP8, native e2m1
 *              weights times e4m3 activations in one block-scaled MMA), with
 *              grouped-nf4-gemm index.json, system_manifest.owns ("native
 *              MXFP4"); reading C19 for the activation scale rule.
 *   [ARENA]    grouped-nf4-gemm releases, v0.2.5 "arena -> kernel" (expert
 *              stacks [E,N,K//2] blocks + [E,N,K//32] e8m0 scales).
 *   [QLORA]    The NF4 codebook itself is not printed on the pages; the values
 *              are the NormalFloat-4 table of Dettmers et al., "QLoRA", 2023,
 *              appendix (reading C1).
 *   [OCP-MX]   OCP Microscaling Formats (MX) v1.0: e2m1 element, e8m0 scale,
 *              shared exponent floor(log2(amax)) - emax_elem (reading C8).
 *
 * Points the pages leave open are taken as numbered readings (C1, C2, ...);
 * each function below names the ones it depends on.
 *
 * PARITY UNPINNED: the NF4 nibble order (reading C2: element 2i in the high
 * nibble, the bitsandbytes convention) has no pin outside this project.  The
 * pages print no packed NF4 bytes and no library that packs NF4 is installed,
 * so only the hand-worked byte examples of the test suite fix the reading.
 * Every other function here has an external pin (closed forms, library
 * routines, brute force or the pages' printed figures).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* ------------------------------------------------------------------ */
/* Threads                                                             */
/* ------------------------------------------------------------------ */
static int g_threads = 1;

void orc_set_threads(int n) { g_threads = n < 1 ? 1 : n; }
int orc_get_threads(void) { return g_threads; }

/* ------------------------------------------------------------------ */
/* Tables                                                              */
/* ------------------------------------------------------------------ */

/* NF4: 16 NormalFloat values, index 0 = -1, index 7 = exact zero,
 * index 15 = +1 [QLORA]. */
static const float NF4_VALUES[16] = {
    -1.0f,
    -0.6961928009986877f,
    -0.5250730514526367f,
    -0.39491748809814453f,
    -0.28444138169288635f,
    -0.18477343022823334f,
    -0.09105003625154495f,
    0.0f,
    0.07958029955625534f,
    0.16093020141124725f,
    0.24611230194568634f,
    0.33791524171829224f,
    0.44070982933044434f,
    0.5626170039176941f,
    0.7229568362236023f,
    1.0f,
};

/* e2m1 magnitudes for the three low bits; bit 3 is the sign [OCP-MX]. */
static const float E2M1_MAGNITUDE[8] = {0.0f, 0.5f, 1.0f, 1.5f, 2.0f, 3.0f, 4.0f, 6.0f};

void orc_nf4_values(float out[16]) { memcpy(out, NF4_VALUES, sizeof(NF4_VALUES)); }

/* Value of a 4-bit e2m1 code: sign = bit 3, magnitude = bits 2..0.  Code 8
 * is negative zero (reading C6). */
static float e2m1_value(unsigned code)
{
    float m = E2M1_MAGNITUDE[code & 7u];
    return (code & 8u) ? -m : m;
}

void orc_e2m1_values(float out[16])
{
    for (unsigned c = 0; c < 16; ++c) out[c] = e2m1_value(c);
}

/* e8m0 scale 2^(e-127); e = 255 is NaN; e = 0 gives the fp32 subnormal
 * 2^-127 (reading C7). */
static float e8m0_value(unsigned e)
{
    if (e == 255u) return NAN;
    return ldexpf(1.0f, (int)e - 127);
}

float orc_e8m0_value(int e) { return e8m0_value((unsigned)e & 255u); }

/* bf16 bit pattern -> float (exact: bf16 is the top half of an fp32). */
static float bf16_to_float(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

/* ------------------------------------------------------------------ */
/* NF4 (bitsandbytes gemm_4bit layout) [README example 1]              */
/* ------------------------------------------------------------------ */

/* Index of the codebook value nearest to x; an exact tie goes to the lower
 * index (reading C4). */
static unsigned nf4_nearest(float x)
{
    unsigned best = 0;
    float bestd = fabsf(x - NF4_VALUES[0]);
    for (unsigned i = 1; i < 16; ++i) {
        float d = fabsf(x - NF4_VALUES[i]);
        if (d < bestd) {
            bestd = d;
            best = i;
        }
    }
    return best;
}

/* Quantise rows x K fp32 weights (row-major) into packed [rows, K/2] bytes
 * and absmax [rows, K/64] fp32.  Blocks are 64 consecutive elements of a row
 * (reading C3).  Within a byte, element 2i sits in the high nibble and
 * element 2i+1 in the low nibble (reading C2).  Requires K % 64 == 0. */
void orc_quant_nf4(const float *w, int64_t rows, int64_t K, uint8_t *packed, float *absmax)
{
    const int64_t nb = K / 64;
#pragma omp parallel for num_threads(g_threads) schedule(static)
    for (int64_t r = 0; r < rows; ++r) {
        for (int64_t b = 0; b < nb; ++b) {
            const float *blk = w + r * K + b * 64;
            float amax = 0.0f;
            for (int i = 0; i < 64; ++i) {
                float a = fabsf(blk[i]);
                if (a > amax) amax = a;
            }
            absmax[r * nb + b] = amax;
            uint8_t *dst = packed + r * (K / 2) + b * 32;
            for (int i = 0; i < 32; ++i) {
                unsigned c0, c1;
                if (amax == 0.0f) {
                    c0 = c1 = 7u; /* the exact zero of the codebook */
                } else {
                    c0 = nf4_nearest(blk[2 * i] / amax);
                    c1 = nf4_nearest(blk[2 * i + 1] / amax);
                }
                dst[i] = (uint8_t)((c0 << 4) | c1);
            }
        }
    }
}

/* Decode: value = NF4_VALUES[code] * absmax, one fp32 multiply. */
void orc_dequant_nf4(const uint8_t *packed, const float *absmax, int64_t rows, int64_t K, float *out)
{
    const int64_t nb = K / 64;
#pragma omp parallel for num_threads(g_threads) schedule(static)
    for (int64_t r = 0; r < rows; ++r) {
        for (int64_t k = 0; k < K; ++k) {
            uint8_t byte = packed[r * (K / 2) + k / 2];
            unsigned code = (k % 2 == 0) ? (byte >> 4) : (byte & 15u);
            out[r * K + k] = NF4_VALUES[code] * absmax[r * nb + k / 64];
        }
    }
}

/* ------------------------------------------------------------------ */
/* MXFP4 (OCP e2m1 + e8m0 per 32) [README example 2], [ARENA]          */
/* ------------------------------------------------------------------ */

/* Round a non-negative magnitude (already divided by the block scale) to
 * the nearest e2m1 magnitude index; ties go to the even index (round to
 * nearest even on the e2m1 mantissa); values above 6 saturate [OCP-MX]. */
static unsigned e2m1_round_magnitude(float m)
{
    if (!(m < 6.0f)) return 7u;
    unsigned best = 0;
    float bestd = fabsf(m - E2M1_MAGNITUDE[0]);
    for (unsigned i = 1; i < 8; ++i) {
        float d = fabsf(m - E2M1_MAGNITUDE[i]);
        if (d < bestd || (d == bestd && (i % 2u) == 0u)) {
            bestd = d;
            best = i;
        }
    }
    return best;
}

/* Quantise rows x K fp32 into blocks [rows, K/2] (element 2i in the LOW
 * nibble, reading C5) and scales [rows, K/32] e8m0.  Shared exponent of a
 * block = floor(log2(amax)) - 2 (e2m1's largest exponent is 2), clamped to
 * the e8m0 range; an all-zero block gets scale byte 0 and zero codes
 * (reading C8).  Requires K % 32 == 0. */
void orc_quant_mxfp4(const float *w, int64_t rows, int64_t K, uint8_t *blocks, uint8_t *scales)
{
    const int64_t nb = K / 32;
#pragma omp parallel for num_threads(g_threads) schedule(static)
    for (int64_t r = 0; r < rows; ++r) {
        for (int64_t b = 0; b < nb; ++b) {
            const float *blk = w + r * K + b * 32;
            float amax = 0.0f;
            for (int i = 0; i < 32; ++i) {
                float a = fabsf(blk[i]);
                if (a > amax) amax = a;
            }
            int sexp;
            if (amax == 0.0f) {
                sexp = -127;
            } else {
                int ex;
                frexpf(amax, &ex); /* amax = m * 2^ex, m in [0.5, 1) */
                sexp = (ex - 1) - 2;
                if (sexp < -127) sexp = -127;
                if (sexp > 127) sexp = 127;
            }
            scales[r * nb + b] = (uint8_t)(sexp + 127);
            float s = ldexpf(1.0f, sexp);
            uint8_t *dst = blocks + r * (K / 2) + b * 16;
            for (int i = 0; i < 16; ++i) {
                unsigned code[2];
                for (int h = 0; h < 2; ++h) {
                    float x = blk[2 * i + h];
                    unsigned mag = (amax == 0.0f) ? 0u : e2m1_round_magnitude(fabsf(x) / s);
                    code[h] = mag | (signbit(x) ? 8u : 0u);
                }
                dst[i] = (uint8_t)(code[0] | (code[1] << 4));
            }
        }
    }
}

/* Decode: value = e2m1(code) * 2^(e-127), one fp32 multiply. */
void orc_dequant_mxfp4(const uint8_t *blocks, const uint8_t *scales, int64_t rows, int64_t K, float *out)
{
    const int64_t nb = K / 32;
#pragma omp parallel for num_threads(g_threads) schedule(static)
    for (int64_t r = 0; r < rows; ++r) {
        for (int64_t k = 0; k < K; ++k) {
            uint8_t byte = blocks[r * (K / 2) + k / 2];
            unsigned code = (k % 2 == 0) ? (byte & 15u) : (byte >> 4);
            out[r * K + k] = e2m1_value(code) * e8m0_value(scales[r * nb + k / 32]);
        }
    }
}

/* ------------------------------------------------------------------ */
/* Routing [PATCH]                                                     */
/* ------------------------------------------------------------------ */

/* Stable counting sort of the M = T*k (token, slot) pairs by expert id.
 * Pair f = t*k + j.  Outputs:
 *   offsets[E+1]      offsets[e] = first sorted row of expert e,
 *                     offsets[E] = number of valid pairs;
 *   sorted_to_flat[M] pair index of each sorted row, -1 past offsets[E];
 *   flat_to_sorted[M] sorted row of each pair, -1 for a dropped pair.
 * Within an expert, pairs keep ascending f (reading C11).  Ids outside
 * [0, E) are counted into *bad and dropped (reading C16).
 * Returns 0. */
int orc_route(const int32_t *topk_ids, int64_t T, int64_t k, int64_t E, int32_t *offsets,
              int32_t *sorted_to_flat, int32_t *flat_to_sorted, int64_t *bad)
{
    const int64_t M = T * k;
    int64_t *count = (int64_t *)calloc((size_t)E, sizeof(int64_t));
    int64_t *cursor = (int64_t *)calloc((size_t)E, sizeof(int64_t));
    int64_t nbad = 0;
    for (int64_t f = 0; f < M; ++f) {
        int32_t e = topk_ids[f];
        if (e >= 0 && e < E)
            count[e] += 1;
        else
            nbad += 1;
    }
    offsets[0] = 0;
    for (int64_t e = 0; e < E; ++e) offsets[e + 1] = offsets[e] + (int32_t)count[e];
    for (int64_t e = 0; e < E; ++e) cursor[e] = offsets[e];
    for (int64_t f = 0; f < M; ++f) {
        int32_t e = topk_ids[f];
        if (e >= 0 && e < E) {
            int64_t p = cursor[e]++;
            sorted_to_flat[p] = (int32_t)f;
            flat_to_sorted[f] = (int32_t)p;
        } else {
            flat_to_sorted[f] = -1;
        }
    }
    for (int64_t p = offsets[E]; p < M; ++p) sorted_to_flat[p] = -1;
    *bad = nbad;
    free(count);
    free(cursor);
    return 0;
}

/* x_sorted[p] = x[sorted_to_flat[p] / k] for p < offsets[E]; later rows are
 * zero.  Rows are K bf16 values moved as raw 16-bit patterns. */
void orc_gather(const uint16_t *x, int64_t K, int64_t k, const int32_t *sorted_to_flat, int64_t M,
                int64_t n_valid, uint16_t *x_sorted)
{
    for (int64_t p = 0; p < M; ++p) {
        if (p < n_valid) {
            int64_t t = sorted_to_flat[p] / k;
            memcpy(x_sorted + p * K, x + t * K, (size_t)K * 2);
        } else {
            memset(x_sorted + p * K, 0, (size_t)K * 2);
        }
    }
}

/* ------------------------------------------------------------------ */
/* Grouped GEMM [README], [ARENA]                                      */
/* ------------------------------------------------------------------ */

/* For every requested sorted row r (rows[i], i < n_rows) of expert e, where
 * offsets[e] <= r < offsets[e+1]:
 *     y[i, n] = sum_k A[r, k] * W_e[n, k]        (fp64 accumulation)
 * with W_e the fp32 dequantised weights of expert e, stored [N, K] (both
 * operands K-major, reading C9).  fmt 0 = NF4 (scales = absmax fp32
 * [E,N,K/64]), fmt 1 = MXFP4 (scales = e8m0 bytes [E,N,K/32]).  Rows outside
 * [0, offsets[E]) give NaN.  Each expert is dequantised only if one of its
 * rows is requested. */
static void grouped_gemm(int fmt, const uint16_t *a, const uint8_t *w, const void *scales,
                         const int32_t *offsets, int64_t E, int64_t N, int64_t K, const int64_t *rows,
                         int64_t n_rows, double *y)
{
    float *wd = (float *)malloc((size_t)(N * K) * sizeof(float));
    int64_t *owner = (int64_t *)malloc((size_t)(n_rows > 0 ? n_rows : 1) * sizeof(int64_t));
    for (int64_t i = 0; i < n_rows; ++i) {
        owner[i] = -1;
        for (int64_t e = 0; e < E; ++e)
            if (rows[i] >= offsets[e] && rows[i] < offsets[e + 1]) owner[i] = e;
        if (owner[i] < 0)
            for (int64_t n = 0; n < N; ++n) y[i * N + n] = NAN;
    }
    for (int64_t e = 0; e < E; ++e) {
        int used = 0;
        for (int64_t i = 0; i < n_rows; ++i)
            if (owner[i] == e) used = 1;
        if (!used) continue;
        if (fmt == 0)
            orc_dequant_nf4(w + e * N * (K / 2), (const float *)scales + e * N * (K / 64), N, K, wd);
        else
            orc_dequant_mxfp4(w + e * N * (K / 2), (const uint8_t *)scales + e * N * (K / 32), N, K, wd);
        for (int64_t i = 0; i < n_rows; ++i) {
            if (owner[i] != e) continue;
            const uint16_t *arow = a + rows[i] * K;
#pragma omp parallel for num_threads(g_threads) schedule(static)
            for (int64_t n = 0; n < N; ++n) {
                const float *wrow = wd + n * K;
                double acc = 0.0;
                for (int64_t kk = 0; kk < K; ++kk) acc += (double)bf16_to_float(arow[kk]) * (double)wrow[kk];
                y[i * N + n] = acc;
            }
        }
    }
    free(owner);
    free(wd);
}

void orc_grouped_gemm_nf4(const uint16_t *a, const uint8_t *w, const float *absmax, const int32_t *offsets,
                          int64_t E, int64_t N, int64_t K, const int64_t *rows, int64_t n_rows, double *y)
{
    grouped_gemm(0, a, w, absmax, offsets, E, N, K, rows, n_rows, y);
}

void orc_grouped_gemm_mxfp4(const uint16_t *a, const uint8_t *w, const uint8_t *scales, const int32_t *offsets,
                            int64_t E, int64_t N, int64_t K, const int64_t *rows, int64_t n_rows, double *y)
{
    grouped_gemm(1, a, w, scales, offsets, E, N, K, rows, n_rows, y);
}

/* ------------------------------------------------------------------ */
/* Top-k combine (the caller's "weighting, unsorting") [PATCH]         */
/* ------------------------------------------------------------------ */

/* out[t, n] = sum_{j<k} weights[t, j] * Y[flat_to_sorted[t*k + j], n] in
 * fp64, j ascending; pairs with flat_to_sorted = -1 contribute nothing.
 * Y holds bf16 patterns. */
void orc_combine(const uint16_t *y, const int32_t *flat_to_sorted, const float *weights, int64_t T, int64_t k,
                 int64_t N, double *out)
{
#pragma omp parallel for num_threads(g_threads) schedule(static)
    for (int64_t t = 0; t < T; ++t) {
        for (int64_t n = 0; n < N; ++n) {
            double acc = 0.0;
            for (int64_t j = 0; j < k; ++j) {
                int32_t p = flat_to_sorted[t * k + j];
                if (p < 0) continue;
                acc += (double)weights[t * k + j] * (double)bf16_to_float(y[(int64_t)p * N + n]);
            }
            out[t * N + n] = acc;
        }
    }
}

/* ------------------------------------------------------------------ */
/* Gated activation between the two projections [MOE]                  */
/* ------------------------------------------------------------------ */

/* SwiGLU over a gate_up projection output (reading C17): row r of gu holds
 * 2I values, the gate half first, then the up half;
 *     h[r, i] = silu(gu[r, i]) * gu[r, I + i],   silu(x) = x / (1 + exp(-x)),
 * all in fp64.  Applied to the fp64 output of orc_grouped_gemm_* this is the
 * plain definition of the fused gate_up + SwiGLU projection. */
void orc_swiglu(const double *gu, int64_t rows, int64_t I, double *h)
{
#pragma omp parallel for num_threads(g_threads) schedule(static)
    for (int64_t r = 0; r < rows; ++r) {
        for (int64_t i = 0; i < I; ++i) {
            const double g = gu[r * 2 * I + i];
            const double u = gu[r * 2 * I + I + i];
            h[r * I + i] = g / (1.0 + exp(-g)) * u;
        }
    }
}

/* ------------------------------------------------------------------ */
/* Router epilogue: top-k selection and softmax weights [ROUTER]       */
/* ------------------------------------------------------------------ */

/* Rank of a score in the selection order: NaN below every number. */
static int score_before(float a, int64_t ia, float b, int64_t ib)
{
    const int na = isnan(a), nb = isnan(b);
    if (na != nb) return nb; /* the non-NaN one comes first */
    if (!na && a != b) return a > b;
    return ia < ib; /* equal (or both NaN): lower expert index first */
}

/* For every token t (reading C18):
 *   score[e] = logits[t, e] + bias[e]  (one fp32 addition, bias may be NULL),
 *   ids[t, 0..k) = the k distinct experts with the largest scores, in
 *                  descending score order, ties to the lower expert index,
 *                  NaN scores ranked below every number;
 *   weights[t, j] = exp(l_j - m) / sum_i exp(l_i - m) over the RAW logits l of
 *                   the k selected experts, m = their maximum (fp64 here).
 * The selection is taken in fp32, the precision of the scores. */
void orc_router_topk(const float *logits, const float *bias, int64_t T, int64_t E, int64_t k, int32_t *ids,
                     double *weights)
{
    for (int64_t t = 0; t < T; ++t) {
        const float *row = logits + t * E;
        for (int64_t j = 0; j < k; ++j) {
            int64_t best = -1;
            float bs = 0.0f;
            for (int64_t e = 0; e < E; ++e) {
                int taken = 0;
                for (int64_t i = 0; i < j; ++i)
                    if (ids[t * k + i] == (int32_t)e) taken = 1;
                if (taken) continue;
                const float s = bias != NULL ? row[e] + bias[e] : row[e];
                if (best < 0 || score_before(s, e, bs, best)) {
                    best = e;
                    bs = s;
                }
            }
            ids[t * k + j] = (int32_t)best;
        }
        double m = -INFINITY;
        for (int64_t j = 0; j < k; ++j) {
            const double l = (double)row[ids[t * k + j]];
            if (l > m || isnan(l)) m = l;
        }
        double sum = 0.0;
        for (int64_t j = 0; j < k; ++j) sum += exp((double)row[ids[t * k + j]] - m);
        for (int64_t j = 0; j < k; ++j) weights[t * k + j] = exp((double)row[ids[t * k + j]] - m) / sum;
    }
}

/* ------------------------------------------------------------------ */
/* Data gradient of the grouped projection [DGRAD]                     */
/* ------------------------------------------------------------------ */

/* For every requested sorted row r (rows[i], i < n_rows) of expert e:
 *     dx[i, k] = sum_n dy[r, n] * W_e[n, k]        (fp64 accumulation)
 * with W_e the fp32 dequantised weights [N, K] of expert e (the same stack
 * the forward call reads) and dy [M, N] bf16 patterns.  fmt 0 = NF4, 1 =
 * MXFP4.  Rows outside [0, offsets[E]) give NaN. */
static void grouped_dgrad(int fmt, const uint16_t *dy, const uint8_t *w, const void *scales,
                          const int32_t *offsets, int64_t E, int64_t N, int64_t K, const int64_t *rows,
                          int64_t n_rows, double *dx)
{
    float *wd = (float *)malloc((size_t)(N * K) * sizeof(float));
    for (int64_t i = 0; i < n_rows; ++i) {
        int64_t owner = -1;
        for (int64_t e = 0; e < E; ++e)
            if (rows[i] >= offsets[e] && rows[i] < offsets[e + 1]) owner = e;
        if (owner < 0)
            for (int64_t kk = 0; kk < K; ++kk) dx[i * K + kk] = NAN;
    }
    for (int64_t e = 0; e < E; ++e) {
        int used = 0;
        for (int64_t i = 0; i < n_rows; ++i)
            if (rows[i] >= offsets[e] && rows[i] < offsets[e + 1]) used = 1;
        if (!used) continue;
        if (fmt == 0)
            orc_dequant_nf4(w + e * N * (K / 2), (const float *)scales + e * N * (K / 64), N, K, wd);
        else
            orc_dequant_mxfp4(w + e * N * (K / 2), (const uint8_t *)scales + e * N * (K / 32), N, K, wd);
        for (int64_t i = 0; i < n_rows; ++i) {
            if (!(rows[i] >= offsets[e] && rows[i] < offsets[e + 1])) continue;
            const uint16_t *grow = dy + rows[i] * N;
#pragma omp parallel for num_threads(g_threads) schedule(static)
            for (int64_t kk = 0; kk < K; ++kk) {
                double acc = 0.0;
                for (int64_t n = 0; n < N; ++n) acc += (double)bf16_to_float(grow[n]) * (double)wd[n * K + kk];
                dx[i * K + kk] = acc;
            }
        }
    }
    free(wd);
}

void orc_grouped_dgrad_nf4(const uint16_t *dy, const uint8_t *w, const float *absmax, const int32_t *offsets,
                           int64_t E, int64_t N, int64_t K, const int64_t *rows, int64_t n_rows, double *dx)
{
    grouped_dgrad(0, dy, w, absmax, offsets, E, N, K, rows, n_rows, dx);
}

void orc_grouped_dgrad_mxfp4(const uint16_t *dy, const uint8_t *w, const uint8_t *scales, const int32_t *offsets,
                             int64_t E, int64_t N, int64_t K, const int64_t *rows, int64_t n_rows, double *dx)
{
    grouped_dgrad(1, dy, w, scales, offsets, E, N, K, rows, n_rows, dx);
}

/* ------------------------------------------------------------------ */
/* Native W4A8: MXFP8 activations x MXFP4 weights [W4A8] [OCP-MX]      */
/* ------------------------------------------------------------------ */

/* Value of an e4m3 code (OCP "E4M3": no infinities): sign = bit 7,
 * exponent = bits 6..3 with bias 7, mantissa = bits 2..0; exponent 0 is
 * subnormal (m/8 * 2^-6); S.1111.111 is NaN; the largest finite magnitude
 * is 448 (code 0x7E). */
static double e4m3_value(unsigned code)
{
    const unsigned e = (code >> 3) & 15u, m = code & 7u;
    double v;
    if (e == 15u && m == 7u) return NAN;
    if (e == 0u)
        v = ldexp((double)m / 8.0, -6);
    else
        v = ldexp(1.0 + (double)m / 8.0, (int)e - 7);
    return (code & 0x80u) ? -v : v;
}

void orc_e4m3_values(double out[256])
{
    for (unsigned c = 0; c < 256; ++c) out[c] = e4m3_value(c);
}

/* Nearest finite e4m3 magnitude code (0x00 .. 0x7E) to a non-negative m,
 * found by comparing against every candidate; an exact tie goes to the even
 * code (round to nearest even on the mantissa).  Everything above 448 ends
 * at 448, the largest candidate (saturation, reading C19). */
static unsigned e4m3_round_magnitude(double m)
{
    unsigned best = 0u;
    double bestd = m; /* distance to code 0 (= 0.0) */
    for (unsigned c = 1u; c <= 0x7Eu; ++c) {
        const double d = fabs(m - e4m3_value(c));
        if (d < bestd || (d == bestd && (c % 2u) == 0u)) {
            bestd = d;
            best = c;
        }
    }
    return best;
}

/* One MXFP8 block: 32 values (exact in fp64) -> 32 e4m3 codes + the e8m0
 * scale byte.  Shared exponent floor(log2(amax)) - top: top = 8 is the OCP
 * rule of reading C19 (the largest element lands in [256, 512) and may
 * saturate at 448); top = 7 leaves one binade of headroom (largest element
 * in [128, 256), nothing saturates), the rule of the two-term split
 * (reading C20). */
static uint8_t mxfp8_block(const double *v, uint8_t *codes, int top)
{
    double amax = 0.0;
    for (int i = 0; i < 32; ++i)
        if (fabs(v[i]) > amax) amax = fabs(v[i]);
    int sexp;
    if (amax == 0.0) {
        sexp = -127;
    } else {
        int ex;
        frexp(amax, &ex); /* amax = f * 2^ex, f in [0.5, 1) */
        sexp = (ex - 1) - top;
        if (sexp < -127) sexp = -127;
        if (sexp > 127) sexp = 127;
    }
    for (int i = 0; i < 32; ++i) {
        const unsigned mag = e4m3_round_magnitude(ldexp(fabs(v[i]), -sexp));
        codes[i] = (uint8_t)(mag | (signbit(v[i]) ? 0x80u : 0u));
    }
    return (uint8_t)(sexp + 127);
}

/* Quantise rows x K bf16 activations to MXFP8: codes [rows, K] e4m3 and
 * scales [rows, K/32] e8m0.  Per block of 32: X = floor(log2(amax)) - 8 (8
 * is e4m3's largest exponent), clamped to [-127, 127]; code = the nearest
 * e4m3 value to x / 2^X (saturating at 448), with x's sign; an all-zero
 * block gets scale byte 0 and zero codes (reading C19).  x / 2^X is exact
 * in fp64.  Requires K % 32 == 0 and finite inputs. */
void orc_quant_mxfp8(const uint16_t *x, int64_t rows, int64_t K, uint8_t *codes, uint8_t *scales)
{
    const int64_t nb = K / 32;
#pragma omp parallel for num_threads(g_threads) schedule(static)
    for (int64_t r = 0; r < rows; ++r) {
        for (int64_t b = 0; b < nb; ++b) {
            double v[32];
            for (int i = 0; i < 32; ++i) v[i] = (double)bf16_to_float(x[r * K + b * 32 + i]);
            scales[r * nb + b] = mxfp8_block(v, codes + r * K + b * 32, 8);
        }
    }
}

/* Decode MXFP8: value = e4m3(code) * 2^(s-127), in fp64. */
void orc_dequant_mxfp8(const uint8_t *codes, const uint8_t *scales, int64_t rows, int64_t K, double *out)
{
    const int64_t nb = K / 32;
#pragma omp parallel for num_threads(g_threads) schedule(static)
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t k = 0; k < K; ++k)
            out[r * K + k] = e4m3_value(codes[r * K + k]) * ldexp(1.0, (int)scales[r * nb + k / 32] - 127);
}

/* Native W4A8 grouped GEMM: y[i, n] = sum_k A[r, k] * W_e[n, k] for the
 * sorted rows r = rows[i] of expert e, with A the MXFP8 activations
 * (e4m3 x 2^(sa-127)) and W the MXFP4 weights (e2m1 x 2^(sw-127)); every
 * product and sum in fp64 [W4A8].  Rows outside [0, offsets[E]) give NaN. */
void orc_grouped_gemm_w4a8(const uint8_t *qa, const uint8_t *sa, const uint8_t *w, const uint8_t *sw,
                           const int32_t *offsets, int64_t E, int64_t N, int64_t K, const int64_t *rows,
                           int64_t n_rows, double *y)
{
    float *wd = (float *)malloc((size_t)(N * K) * sizeof(float));
    double *ad = (double *)malloc((size_t)K * sizeof(double));
    for (int64_t e = 0; e < E; ++e) {
        int used = 0;
        for (int64_t i = 0; i < n_rows; ++i)
            if (rows[i] >= offsets[e] && rows[i] < offsets[e + 1]) used = 1;
        if (!used) continue;
        orc_dequant_mxfp4(w + e * N * (K / 2), sw + e * N * (K / 32), N, K, wd);
        for (int64_t i = 0; i < n_rows; ++i) {
            if (!(rows[i] >= offsets[e] && rows[i] < offsets[e + 1])) continue;
            orc_dequant_mxfp8(qa + rows[i] * K, sa + rows[i] * (K / 32), 1, K, ad);
#pragma omp parallel for num_threads(g_threads) schedule(static)
            for (int64_t n = 0; n < N; ++n) {
                const float *wrow = wd + n * K;
                double acc = 0.0;
                for (int64_t kk = 0; kk < K; ++kk) acc += ad[kk] * (double)wrow[kk];
                y[i * N + n] = acc;
            }
        }
    }
    for (int64_t i = 0; i < n_rows; ++i)
        if (!(rows[i] >= 0 && rows[i] < offsets[E]))
            for (int64_t n = 0; n < N; ++n) y[i * N + n] = NAN;
    free(ad);
    free(wd);
}

/* Two-term MXFP8 split of bf16 activations (reading C20): per block of 32,
 * hi = MXFP8 of x and lo = MXFP8 of the residual r = x - dequant(hi) (exact
 * in fp64), both with the headroom rule (shared exponent
 * floor(log2(amax)) - 7, so no element saturates).  x ~ hi + lo with the
 * error of one e4m3 rounding of the residual. */
void orc_quant_mxfp8_split(const uint16_t *x, int64_t rows, int64_t K, uint8_t *hi_codes, uint8_t *hi_scales,
                           uint8_t *lo_codes, uint8_t *lo_scales)
{
    const int64_t nb = K / 32;
#pragma omp parallel for num_threads(g_threads) schedule(static)
    for (int64_t r = 0; r < rows; ++r) {
        for (int64_t b = 0; b < nb; ++b) {
            double v[32], res[32];
            for (int i = 0; i < 32; ++i) v[i] = (double)bf16_to_float(x[r * K + b * 32 + i]);
            uint8_t *hc = hi_codes + r * K + b * 32, *lc = lo_codes + r * K + b * 32;
            const uint8_t hs = mxfp8_block(v, hc, 7);
            hi_scales[r * nb + b] = hs;
            for (int i = 0; i < 32; ++i) res[i] = v[i] - e4m3_value(hc[i]) * ldexp(1.0, (int)hs - 127);
            lo_scales[r * nb + b] = mxfp8_block(res, lc, 7);
        }
    }
}

/* Two-term native GEMM: y[i, n] = sum_k (hi[r, k] + lo[r, k]) * W_e[n, k] in
 * fp64, hi and lo the dequantised MXFP8 terms of reading C20 [W4A8]. */
void orc_grouped_gemm_w4a8x2(const uint8_t *hc, const uint8_t *hs, const uint8_t *lc, const uint8_t *ls,
                             const uint8_t *w, const uint8_t *sw, const int32_t *offsets, int64_t E, int64_t N,
                             int64_t K, const int64_t *rows, int64_t n_rows, double *y)
{
    double *yl = (double *)malloc((size_t)(n_rows > 0 ? n_rows : 1) * (size_t)N * sizeof(double));
    orc_grouped_gemm_w4a8(hc, hs, w, sw, offsets, E, N, K, rows, n_rows, y);
    orc_grouped_gemm_w4a8(lc, ls, w, sw, offsets, E, N, K, rows, n_rows, yl);
    for (int64_t i = 0; i < n_rows * N; ++i) y[i] += yl[i];
    free(yl);
}

/* ------------------------------------------------------------------ */
/* Native W4A4: MXFP4 activations x MXFP4 weights [W4A8] [OCP-MX]      */
/* ------------------------------------------------------------------ */

/* Quantise rows x K bf16 activations to MXFP4 (blocks [rows, K/2], element
 * 2i in the low nibble; scales [rows, K/32] e8m0) by the same OCP rule as
 * the weights (reading C8, applied to activations: reading C21). */
void orc_quant_mxfp4_act(const uint16_t *x, int64_t rows, int64_t K, uint8_t *blocks, uint8_t *scales)
{
    float *xf = (float *)malloc((size_t)(rows * K > 0 ? rows * K : 1) * sizeof(float));
    for (int64_t i = 0; i < rows * K; ++i) xf[i] = bf16_to_float(x[i]);
    orc_quant_mxfp4(xf, rows, K, blocks, scales);
    free(xf);
}

/* Native W4A4 grouped GEMM: y[i, n] = sum_k A[r, k] * W_e[n, k] with both
 * operands MXFP4 (e2m1 x 2^(s-127)); every product and sum in fp64. */
void orc_grouped_gemm_w4a4(const uint8_t *ab, const uint8_t *as, const uint8_t *w, const uint8_t *sw,
                           const int32_t *offsets, int64_t E, int64_t N, int64_t K, const int64_t *rows,
                           int64_t n_rows, double *y)
{
    float *wd = (float *)malloc((size_t)(N * K) * sizeof(float));
    float *ad = (float *)malloc((size_t)K * sizeof(float));
    for (int64_t e = 0; e < E; ++e) {
        int used = 0;
        for (int64_t i = 0; i < n_rows; ++i)
            if (rows[i] >= offsets[e] && rows[i] < offsets[e + 1]) used = 1;
        if (!used) continue;
        orc_dequant_mxfp4(w + e * N * (K / 2), sw + e * N * (K / 32), N, K, wd);
        for (int64_t i = 0; i < n_rows; ++i) {
            if (!(rows[i] >= offsets[e] && rows[i] < offsets[e + 1])) continue;
            orc_dequant_mxfp4(ab + rows[i] * (K / 2), as + rows[i] * (K / 32), 1, K, ad);
#pragma omp parallel for num_threads(g_threads) schedule(static)
            for (int64_t n = 0; n < N; ++n) {
                const float *wrow = wd + n * K;
                double acc = 0.0;
                for (int64_t kk = 0; kk < K; ++kk) acc += (double)ad[kk] * (double)wrow[kk];
                y[i * N + n] = acc;
            }
        }
    }
    for (int64_t i = 0; i < n_rows; ++i)
        if (!(rows[i] >= 0 && rows[i] < offsets[E]))
            for (int64_t n = 0; n < N; ++n) y[i * N + n] = NAN;
    free(ad);
    free(wd);
}
