/*
 * oracle.c -- plain, slow CPU reference for the NVFP4 routed-expert MoE chain.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or
 * call this file: only the tests, the package's smoke check and the CPU
 * baseline leg of the benchmark use it.  It shares no code, header, table or
 * helper with the CUDA library.
 *
 * What it computes (sources: "nvfp4-megamoe-kernel / CURRENT_BUG.md", three
 * snapshots of one page):
 *   - NVFP4 W4A4 (page 1, "Confirmed working" and page 2, "What the quant
 *     method does"): 4-bit E2M1 values, one FP8-E4M3 scale per 16 elements,
 *     one FP32 global scale per tensor, used as a multiplier on the way in;
 *     the GEMM result is multiplied back by the inverse of both global scales.
 *   - Global scale: 448*6/amax of the tensor (the workload definitions of the
 *     configs; page 2 "What the quant method does" shows what an oversized
 *     multiplier does, so the block-scale conversion saturates).
 *   - The chain (page 1, "Phase 1: CuTeDSL Shared Expert Kernel"):
 *     L1 gate_up GEMM -> SiLU(gate)*up -> re-quantise -> L2 down GEMM, with
 *     gate and up stacked in one weight (gate rows first) and their own global
 *     scales (page 1, "Phase 2", the dual-global-scale challenge).
 *   - Routing (page 3, "Architecture Notes": 384 experts, top-6): every
 *     (token, slot) pair goes to its expert, and the expert outputs are summed
 *     back per token with the top-k weights (page 1, "Phase 3": final scatter).
 *   - Per-expert intermediate global scale fixed by a warmup pass (page 1,
 *     "Phase 1", "Warmup-based gs computation"; page 2 step table, row 8).
 *   - Expert parallelism (page 1, "Config values": 48 of the 384 experts per
 *     rank) may ship the activations already quantised; the chain then starts
 *     from the given codes and scales instead of quantising x.
 *
 * Readings where the pages are silent (each one is also listed in the design
 * notes of the repository):
 *   R1  E2M1 and E4M3 rounding is round-to-nearest, ties to the even code,
 *       saturating to the largest finite value; the sign of a zero E2M1 result
 *       is kept (so -0.1 quantises to code 0x8).
 *   R2  Block quantisation in fp32, in this order: a = max|x_i|;
 *       v = (a / 6) * gs; s = E4M3(v); r = (s == 0) ? 0 : gs / value(s);
 *       q_i = E2M1(x_i * r).  Each fp32 operation rounds to nearest.
 *   R3  Global scale gs = 2688 / amax in fp32; amax == 0 gives gs = 1.
 *   R4  Dequantised value = value(q) * value(s) / gs (fp32); GEMM dot products
 *       accumulate in fp64 and are stored as fp32.
 *   R5  h = g * u / (1 + exp(-g)) evaluated in fp64 from the fp32 g and u,
 *       then rounded to fp32 before it is re-quantised.
 *   R6  Routing is a stable counting sort: slot f = t*k + j of expert e lands
 *       at offsets[e] + #{f' < f : ids[f'] == e}.  Ids < 0 are skipped (the
 *       slot contributes nothing); ids >= E are errors and are also skipped.
 *       Expert segments in the permuted buffers are padded to multiples of
 *       128 rows; the padded position is padded_offsets[e] + rank.
 *   R7  out[t] = sum over j ascending of w[t,j] * y[t,j] (fp64, stored fp32).
 *   R8  Warmup: inter_gs[e] = 2688 / max|h| over expert e's warmup rows;
 *       an expert without warmup rows gets 2688 / (max over experts of that
 *       amax); if no expert has rows, 1.
 *   R12 Router (page 3 "Architecture Notes" names top-6 of 384 but no score
 *       function): the k largest logits, ties to the lower id, weights the
 *       selected softmax terms or sigmoids renormalised to sum 1.
 *   R13 Shared experts folded into the routed chain: rows get k + ns slots,
 *       slot k + i = expert E + i with weight 1, summed with the routed slots
 *       as in R7.
 *   (R9, gate rows first, is stated with the chain above; R10, the packing,
 *   under Layouts below; R11 concerns how the activation global scale is
 *   obtained, which the oracle takes as an input.)
 *
 * Layouts (all row-major): codes [rows, cols/2] uint8, element 2i in the low
 * nibble of byte i, element 2i+1 in the high nibble; scales [rows, cols/16]
 * uint8 E4M3 bytes; bf16 values are passed as their uint16 bit patterns.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

/* ------------------------------------------------------------------ */
/* Element formats                                                     */
/* ------------------------------------------------------------------ */

/* E2M1 magnitudes, indexed by the 3-bit magnitude code (exponent 2 bits,
 * mantissa 1 bit, bias 1; code 1 is the subnormal 0.5). */
static const float E2M1_MAGNITUDE[8] = {0.0f, 0.5f, 1.0f, 1.5f, 2.0f, 3.0f, 4.0f, 6.0f};

float oracle_e2m1_decode(uint8_t code)
{
    float m = E2M1_MAGNITUDE[code & 7];
    return (code & 8) ? -m : m;
}

/* Nearest representable magnitude; on a tie the even code wins; anything
 * beyond 6 is nearest to 6 (saturation).  NaN inputs are out of contract. */
uint8_t oracle_e2m1_encode(float v)
{
    uint8_t sign = signbit(v) ? 8 : 0;
    double a = fabs((double)v);
    int best = 0;
    double best_d = INFINITY;
    for (int i = 0; i < 8; i++) {
        double d = fabs(a - (double)E2M1_MAGNITUDE[i]);
        if (d < best_d || (d == best_d && (i & 1) == 0)) {
            best = i;
            best_d = d;
        }
    }
    return (uint8_t)(sign | best);
}

/* E4M3 "FN": bias 7, no infinity, 0x7F / 0xFF are NaN, largest finite 448. */
float oracle_e4m3_decode(uint8_t b)
{
    int e = (b >> 3) & 15;
    int m = b & 7;
    double v;
    if ((b & 0x7F) == 0x7F)
        return NAN;
    if (e == 0)
        v = ldexp((double)m, -9);              /* subnormal: m * 2^-9 */
    else
        v = ldexp(1.0 + m / 8.0, e - 7);
    return (float)((b & 0x80) ? -v : v);
}

/* Nearest finite E4M3 value, ties to the even code, saturating at 448. */
uint8_t oracle_e4m3_encode(float v)
{
    uint8_t sign = signbit(v) ? 0x80 : 0;
    double a = fabs((double)v);
    int best = 0;
    double best_d = INFINITY;
    for (int c = 0; c <= 0x7E; c++) {
        double d = fabs(a - (double)oracle_e4m3_decode((uint8_t)c));
        if (d < best_d || (d == best_d && (c & 1) == 0)) {
            best = c;
            best_d = d;
        }
    }
    return (uint8_t)(sign | best);
}

static float bf16_to_f32(uint16_t h)
{
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

/* ------------------------------------------------------------------ */
/* Global scale (R3)                                                   */
/* ------------------------------------------------------------------ */

float oracle_global_scale_from_amax(float amax)
{
    if (amax == 0.0f)
        return 1.0f;
    return 2688.0f / amax;
}

float oracle_amax_bf16(const uint16_t *x, int64_t n)
{
    float m = 0.0f;
    for (int64_t i = 0; i < n; i++) {
        float a = fabsf(bf16_to_f32(x[i]));
        if (a > m)
            m = a;
    }
    return m;
}

float oracle_amax_f32(const float *x, int64_t n)
{
    float m = 0.0f;
    for (int64_t i = 0; i < n; i++) {
        float a = fabsf(x[i]);
        if (a > m)
            m = a;
    }
    return m;
}

/* ------------------------------------------------------------------ */
/* Block quantiser (R2) and dequantiser (R4)                           */
/* ------------------------------------------------------------------ */

/* One 16-element block: writes 16 codes (one per byte, unpacked) and
 * returns the E4M3 scale byte. */
static uint8_t quantize_block16(const float *x, float gs, uint8_t *code16)
{
    volatile float a = 0.0f;   /* volatile: keep each fp32 step a separate rounding */
    for (int i = 0; i < 16; i++) {
        float ax = fabsf(x[i]);
        if (ax > a)
            a = ax;
    }
    volatile float a_over_6 = a / 6.0f;
    volatile float v = a_over_6 * gs;
    uint8_t s = oracle_e4m3_encode(v);
    float r = 0.0f;
    if (s != 0) {
        volatile float sv = oracle_e4m3_decode(s);
        r = gs / sv;
    }
    for (int i = 0; i < 16; i++) {
        volatile float p = x[i] * r;
        code16[i] = oracle_e2m1_encode(p);
    }
    return s;
}

static void quantize_row_f32(const float *x, int64_t cols, float gs,
                             uint8_t *codes_row, uint8_t *scales_row)
{
    uint8_t c16[16];
    for (int64_t b = 0; b < cols / 16; b++) {
        scales_row[b] = quantize_block16(x + 16 * b, gs, c16);
        for (int i = 0; i < 8; i++)
            codes_row[8 * b + i] = (uint8_t)(c16[2 * i] | (c16[2 * i + 1] << 4));
    }
}

/* x [rows, ldx] bf16 bits -> codes [rows, cols/2], scales [rows, cols/16].
 * cols must be a multiple of 16. */
void oracle_quantize_bf16(const uint16_t *x, int64_t rows, int64_t cols, int64_t ldx,
                          float gs, uint8_t *codes, uint8_t *scales)
{
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; r++) {
        float *tmp = (float *)malloc(sizeof(float) * (size_t)cols);
        for (int64_t c = 0; c < cols; c++)
            tmp[c] = bf16_to_f32(x[r * ldx + c]);
        quantize_row_f32(tmp, cols, gs, codes + r * (cols / 2), scales + r * (cols / 16));
        free(tmp);
    }
}

void oracle_quantize_f32(const float *x, int64_t rows, int64_t cols, int64_t ldx,
                         float gs, uint8_t *codes, uint8_t *scales)
{
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; r++)
        quantize_row_f32(x + r * ldx, cols, gs, codes + r * (cols / 2), scales + r * (cols / 16));
}

static float dequant_element(const uint8_t *codes_row, const uint8_t *scales_row,
                             int64_t c, float gs)
{
    uint8_t byte = codes_row[c / 2];
    uint8_t q = (c & 1) ? (byte >> 4) : (byte & 15);
    float prod = oracle_e2m1_decode(q) * oracle_e4m3_decode(scales_row[c / 16]); /* exact */
    return prod / gs;
}

void oracle_dequantize(const uint8_t *codes, const uint8_t *scales, int64_t rows,
                       int64_t cols, float gs, float *out)
{
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; r++)
        for (int64_t c = 0; c < cols; c++)
            out[r * cols + c] = dequant_element(codes + r * (cols / 2), scales + r * (cols / 16), c, gs);
}

/* ------------------------------------------------------------------ */
/* Routing (R6)                                                        */
/* ------------------------------------------------------------------ */

/* ids [R]; outputs counts [E], offsets [E+1], padded_offsets [E+1],
 * rank [R] (position of the slot inside its expert, -1 if skipped) and
 * pos_padded [R] (-1 if skipped).  Returns the number of ids >= E. */
int oracle_route(const int32_t *ids, int64_t R, int E, int32_t *counts,
                 int32_t *offsets, int32_t *padded_offsets, int32_t *rank,
                 int32_t *pos_padded)
{
    int bad = 0;
    for (int e = 0; e < E; e++)
        counts[e] = 0;
    for (int64_t f = 0; f < R; f++) {
        int32_t e = ids[f];
        if (e >= E)
            bad++;
        else if (e >= 0)
            counts[e]++;
    }
    offsets[0] = 0;
    padded_offsets[0] = 0;
    for (int e = 0; e < E; e++) {
        offsets[e + 1] = offsets[e] + counts[e];
        padded_offsets[e + 1] = padded_offsets[e] + ((counts[e] + 127) / 128) * 128;
    }
    int32_t *seen = (int32_t *)calloc((size_t)(E > 0 ? E : 1), sizeof(int32_t));
    for (int64_t f = 0; f < R; f++) {
        int32_t e = ids[f];
        if (e < 0 || e >= E) {
            rank[f] = -1;
            pos_padded[f] = -1;
            continue;
        }
        rank[f] = seen[e]++;          /* = #{f' < f : ids[f'] == e} */
        pos_padded[f] = padded_offsets[e] + rank[f];
    }
    free(seen);
    return bad;
}

/* ------------------------------------------------------------------ */
/* Dense NVFP4 GEMM (R4)                                               */
/* ------------------------------------------------------------------ */

/* out[m, n] = sum_k dq(A)[m,k] * dq(B)[n,k]; B rows in segment s (rows
 * below seg_end[s], above the previous end) use global scale b_gs[s]. */
void oracle_gemm(const uint8_t *a_codes, const uint8_t *a_scales, float a_gs, int64_t M,
                 const uint8_t *b_codes, const uint8_t *b_scales, const float *b_gs,
                 const int64_t *seg_end, int nseg, int64_t N, int64_t K, float *out)
{
    float *A = (float *)malloc(sizeof(float) * (size_t)(M * K));
    float *B = (float *)malloc(sizeof(float) * (size_t)(N * K));
    oracle_dequantize(a_codes, a_scales, M, K, a_gs, A);
    int64_t start = 0;
    for (int s = 0; s < nseg; s++) {
        int64_t end = seg_end[s];
        oracle_dequantize(b_codes + start * (K / 2), b_scales + start * (K / 16),
                          end - start, K, b_gs[s], B + start * K);
        start = end;
    }
#pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; m++)
        for (int64_t n = 0; n < N; n++) {
            double acc = 0.0;
            for (int64_t k = 0; k < K; k++)
                acc += (double)A[m * K + k] * (double)B[n * K + k];
            out[m * N + n] = (float)acc;
        }
    free(A);
    free(B);
}

/* ------------------------------------------------------------------ */
/* MoE forward                                                         */
/* ------------------------------------------------------------------ */

typedef struct {
    int64_t T, H, I;
    int32_t E, k;
    const uint16_t *x;             /* [T, H] bf16 bits */
    const int32_t *topk_ids;       /* [T, k] */
    const float *topk_weights;     /* [T, k] */
    float x_gs;
    const uint8_t *w13_codes;      /* [E, 2I, H/2]  gate rows 0..I-1, up rows I..2I-1 */
    const uint8_t *w13_scales;     /* [E, 2I, H/16] */
    const float *w13_gs;           /* [E, 2]  (gate, up) */
    const uint8_t *w2_codes;       /* [E, H, I/2] */
    const uint8_t *w2_scales;      /* [E, H, I/16] */
    const float *w2_gs;            /* [E] */
    const float *inter_gs;         /* [E]; may be NULL when only h is wanted */
    /* outputs (any may be NULL) */
    float *out;                    /* [T, H] */
    float *h;                      /* [R, I]  slot order f = t*k + j */
    uint8_t *h_codes;              /* [R, I/2] slot order */
    uint8_t *h_scales;             /* [R, I/16] slot order */
    float *y;                      /* [R, H]  slot order */
    float *h_amax;                 /* [E] max |h| over each expert's rows */
    /* activations given already quantised (both non-NULL): x is not read and
     * these codes [T, H/2] and scales [T, H/16] stand for quantise(x, x_gs) */
    const uint8_t *x_codes;
    const uint8_t *x_scales;
} oracle_moe_args;

/* The whole chain, expert by expert, over the stable routing order (R6):
 * quantise x (R2), L1 with the gate/up global scales (R4), SiLU*up (R5),
 * re-quantise with inter_gs[e], L2, then the weighted combine (R7). */
int oracle_moe_forward(const oracle_moe_args *p)
{
    const int64_t T = p->T, H = p->H, I = p->I, R = p->T * p->k;
    const int E = p->E, k = p->k;
    int32_t *counts = (int32_t *)malloc(sizeof(int32_t) * (size_t)E);
    int32_t *offsets = (int32_t *)malloc(sizeof(int32_t) * (size_t)(E + 1));
    int32_t *poff = (int32_t *)malloc(sizeof(int32_t) * (size_t)(E + 1));
    int32_t *rank = (int32_t *)malloc(sizeof(int32_t) * (size_t)R);
    int32_t *posp = (int32_t *)malloc(sizeof(int32_t) * (size_t)R);
    int bad = oracle_route(p->topk_ids, R, E, counts, offsets, poff, rank, posp);

    /* expert-major list of slots, in routing order */
    int64_t *slot_of = (int64_t *)malloc(sizeof(int64_t) * (size_t)(R > 0 ? R : 1));
    for (int64_t f = 0; f < R; f++)
        if (rank[f] >= 0)
            slot_of[offsets[p->topk_ids[f]] + rank[f]] = f;

    /* quantised activations, one row per token (or the caller's) */
    uint8_t *xq = (uint8_t *)malloc((size_t)(T * H / 2 > 0 ? T * H / 2 : 1));
    uint8_t *xs = (uint8_t *)malloc((size_t)(T * H / 16 > 0 ? T * H / 16 : 1));
    if (p->x_codes && p->x_scales) {
        memcpy(xq, p->x_codes, (size_t)(T * H / 2));
        memcpy(xs, p->x_scales, (size_t)(T * H / 16));
    } else {
        oracle_quantize_bf16(p->x, T, H, H, p->x_gs, xq, xs);
    }
    float *xd = (float *)malloc(sizeof(float) * (size_t)(T * H));
    oracle_dequantize(xq, xs, T, H, p->x_gs, xd);

    double *y_all = (double *)calloc((size_t)(R * H > 0 ? R * H : 1), sizeof(double));
    float *h_all = (float *)calloc((size_t)(R * I > 0 ? R * I : 1), sizeof(float));
    float *W13 = (float *)malloc(sizeof(float) * (size_t)(2 * I * H));
    float *W2 = (float *)malloc(sizeof(float) * (size_t)(H * I));

    for (int e = 0; e < E; e++) {
        int64_t n_rows = counts[e];
        float amax_e = 0.0f;
        if (n_rows == 0) {
            if (p->h_amax)
                p->h_amax[e] = 0.0f;
            continue;
        }
        const uint8_t *c13 = p->w13_codes + (int64_t)e * 2 * I * (H / 2);
        const uint8_t *s13 = p->w13_scales + (int64_t)e * 2 * I * (H / 16);
        oracle_dequantize(c13, s13, I, H, p->w13_gs[2 * e + 0], W13);
        oracle_dequantize(c13 + I * (H / 2), s13 + I * (H / 16), I, H, p->w13_gs[2 * e + 1], W13 + I * H);
        if (p->inter_gs)
            oracle_dequantize(p->w2_codes + (int64_t)e * H * (I / 2),
                              p->w2_scales + (int64_t)e * H * (I / 16), H, I, p->w2_gs[e], W2);

#pragma omp parallel for schedule(dynamic, 1) reduction(max : amax_e)
        for (int64_t i = 0; i < n_rows; i++) {
            int64_t f = slot_of[offsets[e] + i];
            int64_t t = f / k;
            const float *a = xd + t * H;
            float *hrow = h_all + f * I;
            for (int64_t n = 0; n < I; n++) {
                double g = 0.0, u = 0.0;
                for (int64_t c = 0; c < H; c++) {
                    g += (double)a[c] * (double)W13[n * H + c];
                    u += (double)a[c] * (double)W13[(I + n) * H + c];
                }
                float gf = (float)g, uf = (float)u;
                double hv = (double)gf * (double)uf / (1.0 + exp(-(double)gf));
                hrow[n] = (float)hv;
                if (fabsf(hrow[n]) > amax_e)
                    amax_e = fabsf(hrow[n]);
            }
            if (!p->inter_gs)
                continue;
            uint8_t *hq = (uint8_t *)malloc((size_t)(I / 2));
            uint8_t *hs = (uint8_t *)malloc((size_t)(I / 16));
            float *hd = (float *)malloc(sizeof(float) * (size_t)I);
            quantize_row_f32(hrow, I, p->inter_gs[e], hq, hs);
            for (int64_t c = 0; c < I; c++)
                hd[c] = dequant_element(hq, hs, c, p->inter_gs[e]);
            if (p->h_codes)
                memcpy(p->h_codes + f * (I / 2), hq, (size_t)(I / 2));
            if (p->h_scales)
                memcpy(p->h_scales + f * (I / 16), hs, (size_t)(I / 16));
            for (int64_t n = 0; n < H; n++) {
                double acc = 0.0;
                for (int64_t c = 0; c < I; c++)
                    acc += (double)hd[c] * (double)W2[n * I + c];
                y_all[f * H + n] = (double)(float)acc;
            }
            free(hq);
            free(hs);
            free(hd);
        }
        if (p->h_amax)
            p->h_amax[e] = amax_e;
    }

    if (p->h)
        memcpy(p->h, h_all, sizeof(float) * (size_t)(R * I));
    if (p->y)
        for (int64_t i = 0; i < R * H; i++)
            p->y[i] = (float)y_all[i];
    if (p->out && p->inter_gs) {
#pragma omp parallel for schedule(static)
        for (int64_t t = 0; t < T; t++)
            for (int64_t n = 0; n < H; n++) {
                double acc = 0.0;
                for (int j = 0; j < k; j++) {
                    int64_t f = t * k + j;
                    if (rank[f] < 0)
                        continue;
                    acc += (double)p->topk_weights[f] * y_all[f * H + n];
                }
                p->out[t * H + n] = (float)acc;
            }
    }

    free(counts); free(offsets); free(poff); free(rank); free(posp); free(slot_of);
    free(xq); free(xs); free(xd); free(y_all); free(h_all); free(W13); free(W2);
    return bad;
}

/* Warmup (R8): run the chain up to h on the warmup batch and turn each
 * expert's max |h| into its intermediate global scale. */
int oracle_moe_warmup_inter_gs(const oracle_moe_args *p_in, float *inter_gs_out)
{
    oracle_moe_args p = *p_in;
    float *amax = (float *)malloc(sizeof(float) * (size_t)p.E);
    p.inter_gs = NULL;
    p.out = NULL; p.h = NULL; p.h_codes = NULL; p.h_scales = NULL; p.y = NULL;
    p.h_amax = amax;
    int bad = oracle_moe_forward(&p);
    float gmax = 0.0f;
    for (int e = 0; e < p.E; e++)
        if (amax[e] > gmax)
            gmax = amax[e];
    for (int e = 0; e < p.E; e++)
        inter_gs_out[e] = oracle_global_scale_from_amax(amax[e] > 0.0f ? amax[e] : gmax);
    free(amax);
    return bad;
}

/* ------------------------------------------------------------------ */
/* Top-k router (the step before the path)                             */
/* ------------------------------------------------------------------ */

/* For each token: the k experts with the largest logits, in descending
 * order, ties to the lower expert id (the router's scores -- softmax or
 * sigmoid of the logits -- are increasing functions of the logit, so the
 * same experts).  Weights (R12): scoring 0 = softmax renormalised over the
 * selected experts, w_j = exp(l_j) / sum_i exp(l_i); scoring 1 = sigmoid
 * renormalised, w_j = s_j / sum_i s_i.  Evaluated in fp64, stored fp32.
 * R13: with ns shared experts (page 1 "Phase 1": a shared expert is the
 * routed chain with one expert and no routing), rows hold k + ns slots and slot
 * k + i is expert E + i with weight 1: every token runs every shared expert
 * at full weight, as one more group of the routed chain. */
void oracle_topk_shared(const float *logits, int64_t T, int E, int k, int scoring, int ns, int32_t *ids, float *w)
{
    const int ld = k + ns;
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < T; t++) {
        const float *l = logits + t * E;
        int32_t *id = ids + t * ld;
        for (int j = 0; j < k; j++) {
            int best = -1;
            for (int e = 0; e < E; e++) {
                int taken = 0;
                for (int i = 0; i < j; i++)
                    if (id[i] == e)
                        taken = 1;
                if (taken)
                    continue;
                if (best < 0 || l[e] > l[best])   /* strict: the lower id wins a tie */
                    best = e;
            }
            id[j] = best;
        }
        double sum = 0.0, v[32];
        for (int j = 0; j < k; j++) {
            double x = (double)l[id[j]];
            v[j] = scoring == 0 ? exp(x - (double)l[id[0]]) : 1.0 / (1.0 + exp(-x));
            sum += v[j];
        }
        for (int j = 0; j < k; j++)
            w[t * ld + j] = (float)(v[j] / sum);
        for (int i = 0; i < ns; i++) {
            id[k + i] = E + i;
            w[t * ld + k + i] = 1.0f;
        }
    }
}

void oracle_topk(const float *logits, int64_t T, int E, int k, int scoring, int32_t *ids, float *w)
{
    oracle_topk_shared(logits, T, E, k, scoring, 0, ids, w);
}

int oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
