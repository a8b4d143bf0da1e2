/*
 * moe_oracle.c -- the oracle for the routed-expert MoE FFN whose expert
 * weights are stored compressed (MXFP4 or 8-dim VQ13 with an optional 8-bit
 * residual stage).
 *
 * TEST INFRASTRUCTURE.  This file is a plain, slow, deliberately obvious CPU
 * restatement of what the layer computes, written from the pages' format and
 * layer descriptions.  Only the tests, the package's smoke check and the
 * benchmark's CPU-baseline leg may load it.  It shares no code, header, table
 * or helper with the CUDA library, and the CUDA library never calls it.
 *
 * Sources (page title, section):
 *  [MIX]  "MiMo-V2.6-Flash-RL Mixed-Quant GGUF", "Why this model needs an
 *         asymmetric layout": routed experts are stored as packed MXFP4, two
 *         logical weights per byte; gate/up/down expert projections.
 *  [SPK]  "MiMo-V2.6-Flash-RL GGUF for a single DGX Spark", "Architecture
 *         notes": 256 routed experts, 8 active per token; MXFP4 with one
 *         E8M0 exponent per 32 values.  "Recipe": a 32-value intermediate
 *         sum passes f16's 65504 in layer 47, so intermediates stay in a
 *         wider type (here: double).
 *  [VQ]   "MiMo-V2.6-Flash-RL UNCENSORED VQ GGUF", "Recipe": an expert row
 *         is cut into 8-weight vectors, each stored as an index into the
 *         layer's codebook, the row scaled by an f16 gain; the layer has a
 *         single codebook for all experts and all three projections; an
 *         optional 256-entry second book spends 8 more bits per vector on
 *         the first stage's remainder and leaves the first-stage indices
 *         unchanged.
 *  [IQ3]  "MiMo-V2.6-Flash-RL: calibrated IQ3_XXS", "Calibration": the sum
 *         of the per-projection route counts is eight routes per token.
 *
 * Readings taken where the pages are silent (each also fixed by the
 * workload definitions): the nibble of element k sits in byte k/2, low
 * nibble for even k; E8M0 byte b means 2^(b-127) and 255 is NaN; the 13-bit
 * indices of a row form a little-endian bitstream (index j = bits
 * 13j..13j+12, bit p = (byte[p/8] >> (p%8)) & 1); codebook entries are bf16;
 * dimension i of an 8-vector is K offset 8j+i; the VQ weight is
 * ((base + residual) * gain) in IEEE f32 round-to-nearest-even, in that
 * order, so that a dequantised weight has one exact f32 value; the FFN is
 * SwiGLU, y = W_down (silu(W_gate x) * (W_up x)), silu(z) = z / (1 + e^-z);
 * route ids of -1 mean "no route"; other ids outside [0, E) are skipped and
 * counted as invalid.
 *
 * Build: gcc -O2 -std=c11 -ffp-contract=off -fopenmp -shared -fPIC.
 * (-ffp-contract=off keeps every f32 add and multiply separately rounded.)
 */
#include <math.h>
#include <stddef.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* ------------------------------------------------------------------ */
/* Scalar formats                                                      */
/* ------------------------------------------------------------------ */

/* E2M1 [SPK "Architecture notes" names MXFP4]: bit 3 sign, bits 2..1 the
 * exponent e (bias 1), bit 0 the mantissa m.  e = 0 is subnormal (m * 0.5);
 * otherwise 2^(e-1) * (1 + m/2).  Magnitudes 0, .5, 1, 1.5, 2, 3, 4, 6;
 * code 8 is -0. */
double orc_e2m1(uint32_t code)
{
    int s = (int)((code >> 3) & 1u);
    int e = (int)((code >> 1) & 3u);
    int m = (int)(code & 1u);
    double mag = (e == 0) ? 0.5 * m : ldexp(1.0 + 0.5 * m, e - 1);
    return s ? -mag : mag;
}

/* E8M0 [SPK "Architecture notes"]: an unsigned power-of-two exponent,
 * 2^(b-127); the all-ones byte is NaN. */
double orc_e8m0(uint32_t b)
{
    if (b == 255u) return NAN;
    return ldexp(1.0, (int)b - 127);
}

/* bf16: the upper 16 bits of an IEEE binary32. */
float orc_bf16_to_f32(uint16_t h)
{
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

/* IEEE binary16: 1 sign, 5 exponent (bias 15), 10 mantissa bits. */
double orc_f16_to_f64(uint16_t h)
{
    int s = (h >> 15) & 1;
    int e = (h >> 10) & 31;
    int m = h & 1023;
    double v;
    if (e == 0) v = ldexp((double)m, -24);
    else if (e == 31) v = m ? NAN : INFINITY;
    else v = ldexp(1.0 + m / 1024.0, e - 15);
    return s ? -v : v;
}

/* ------------------------------------------------------------------ */
/* Row decoders                                                        */
/* ------------------------------------------------------------------ */

/* MXFP4 row [MIX "asymmetric layout"; SPK "Architecture notes"]:
 * w[k] = e2m1(nibble k) * e8m0(scale[k/32]).  The product of an E2M1 value
 * and a power of two is exact in f32 (down to f32 subnormals), so the f64
 * value converts to f32 without rounding. */
void orc_row_mxfp4(const uint8_t *codes_row, const uint8_t *scales_row, int K, float *w)
{
    for (int k = 0; k < K; ++k) {
        uint32_t byte = codes_row[k / 2];
        uint32_t nib = (k % 2 == 0) ? (byte & 0xFu) : (byte >> 4);
        w[k] = (float)(orc_e2m1(nib) * orc_e8m0(scales_row[k / 32]));
    }
}

/* 13-bit index j of a row's little-endian bitstream [VQ "Recipe": 13 bits
 * per 8 weights]. */
uint32_t orc_idx13(const uint8_t *row_stream, int64_t j)
{
    uint32_t idx = 0;
    for (int q = 0; q < 13; ++q) {
        int64_t p = 13 * j + q;
        uint32_t bit = (row_stream[p >> 3] >> (p & 7)) & 1u;
        idx |= bit << q;
    }
    return idx;
}

/* VQ row [VQ "Recipe"]: w[8j+i] = (B13[idx13_j][i] + R8[idx8_j][i]) * gain,
 * each step an IEEE f32 operation.  idx8_row / book8 NULL: no residual
 * stage.  gain_bits NULL: gain 1. */
void orc_row_vq(const uint8_t *idx13_row, const uint8_t *idx8_row,
                const uint16_t *book13, const uint16_t *book8,
                const uint16_t *gain_bits, int K, float *w)
{
    float gain = gain_bits ? (float)orc_f16_to_f64(*gain_bits) : 1.0f;
    for (int j = 0; j < K / 8; ++j) {
        uint32_t i13 = orc_idx13(idx13_row, j);
        for (int i = 0; i < 8; ++i) {
            float v = orc_bf16_to_f32(book13[i13 * 8 + i]);
            if (idx8_row && book8) {
                float r = orc_bf16_to_f32(book8[(uint32_t)idx8_row[j] * 8 + i]);
                v = v + r;
            }
            if (gain_bits) v = v * gain;
            w[8 * j + i] = v;
        }
    }
}

/* ------------------------------------------------------------------ */
/* GVQ1-style rows: 12-bit stream + 1-bit plane, 1-byte book entries   */
/* ------------------------------------------------------------------ */

/* E4M3 (the OCP 8-bit float without infinities): bit 7 sign, bits 6..3 the
 * exponent e (bias 7), bits 2..0 the mantissa m.  e = 0: m/8 * 2^-6
 * (subnormal); otherwise (1 + m/8) * 2^(e-7); e = 15 with m = 7 is NaN.
 * Largest magnitude 448.  [Reading: the VQ page gives the books 1-byte
 * entries ("Why 13 bits plus an 8-bit residual": 64 KiB + 2 KiB) without a
 * number format.] */
double orc_e4m3(uint32_t b)
{
    int s = (int)((b >> 7) & 1u);
    int e = (int)((b >> 3) & 15u);
    int m = (int)(b & 7u);
    double v;
    if (e == 15 && m == 7) return NAN;
    if (e == 0) v = ldexp((double)m / 8.0, -6);
    else v = ldexp(1.0 + (double)m / 8.0, e - 7);
    return s ? -v : v;
}

/* Index j of a GVQ1 row [VQ "Recipe": the indices as a 12-bit code stream
 * with a separate plane of one-bit flags]: the low 12 bits are bits 12j..12j+11 of the row's little-endian
 * 12-bit stream, bit 12 is bit j of the row's bit plane (bit q of a stream
 * is bit q%8 of byte q/8, as for the 13-bit stream). */
uint32_t orc_gvq1_idx(const uint8_t *code12_row, const uint8_t *hi_row, int64_t j)
{
    uint32_t idx = 0;
    for (int q = 0; q < 12; ++q) {
        int64_t p = 12 * j + q;
        idx |= ((uint32_t)(code12_row[p >> 3] >> (p & 7)) & 1u) << q;
    }
    idx |= ((uint32_t)(hi_row[j >> 3] >> (j & 7)) & 1u) << 12;
    return idx;
}

/* GVQ1 row: w[8j+i] = (e4m3(B13q[c][i]) * s13 + e4m3(B8q[r][i]) * s8) * gain,
 * every operation an IEEE f32 one in that order (the E4M3 value is exact in
 * f32); idx8_row / book8q NULL: no residual term; gain_bits NULL: gain 1. */
void orc_row_gvq1(const uint8_t *code12_row, const uint8_t *hi_row, const uint8_t *idx8_row,
                  const uint8_t *book13q, const uint8_t *book8q, float s13, float s8,
                  const uint16_t *gain_bits, int K, float *w)
{
    float gain = gain_bits ? (float)orc_f16_to_f64(*gain_bits) : 1.0f;
    for (int j = 0; j < K / 8; ++j) {
        uint32_t c = orc_gvq1_idx(code12_row, hi_row, j);
        for (int i = 0; i < 8; ++i) {
            float v = (float)orc_e4m3(book13q[c * 8 + i]) * s13;
            if (idx8_row && book8q) {
                float r = (float)orc_e4m3(book8q[(uint32_t)idx8_row[j] * 8 + i]) * s8;
                v = v + r;
            }
            if (gain_bits) v = v * gain;
            w[8 * j + i] = v;
        }
    }
}

/* ------------------------------------------------------------------ */
/* Layer description                                                   */
/* ------------------------------------------------------------------ */

enum { ORC_MXFP4 = 0, ORC_VQ13 = 1, ORC_VQ13_R8 = 2, ORC_GVQ1 = 3, ORC_GVQ1_R8 = 4 };

typedef struct {
    int32_t H, I, E, k, fmt;
    /* per projection p (0 gate [I][H], 1 up [I][H], 2 down [H][I]) */
    const uint8_t *codes[3];   /* MXFP4 nibbles   [E][N][K/2]      */
    const uint8_t *scales[3];  /* E8M0 bytes      [E][N][K/32]     */
    const uint8_t *idx13[3];   /* 13-bit stream   [E][N][K*13/64]  */
    const uint8_t *idx8[3];    /* residual index  [E][N][K/8]      */
    const uint16_t *gain[3];   /* f16 row gains   [E][N] or NULL   */
    const uint16_t *book13;    /* bf16 [8192][8]                   */
    const uint16_t *book8;     /* bf16 [256][8] or NULL            */
    /* GVQ1 / GVQ1_R8 (idx8 and gain as above) */
    const uint8_t *code12[3];  /* 12-bit stream   [E][N][K*3/16]   */
    const uint8_t *hi1[3];     /* bit-12 plane    [E][N][K/64]     */
    const uint8_t *gbook13;    /* e4m3 [8192][8]                   */
    const uint8_t *gbook8;     /* e4m3 [256][8] or NULL            */
    float gscale13, gscale8;
} orc_layer;

static void proj_shape(const orc_layer *L, int p, int *N, int *K)
{
    if (p == 2) { *N = L->H; *K = L->I; }
    else        { *N = L->I; *K = L->H; }
}

/* Row n of projection p of expert e, dequantised to f32. */
void orc_dequant_row(const orc_layer *L, int e, int p, int n, float *w)
{
    int N, K;
    proj_shape(L, p, &N, &K);
    int64_t row = (int64_t)e * N + n;
    if (L->fmt == ORC_MXFP4) {
        orc_row_mxfp4(L->codes[p] + row * (K / 2), L->scales[p] + row * (K / 32), K, w);
    } else if (L->fmt == ORC_GVQ1 || L->fmt == ORC_GVQ1_R8) {
        const int r8 = L->fmt == ORC_GVQ1_R8;
        orc_row_gvq1(L->code12[p] + row * ((int64_t)K * 3 / 16), L->hi1[p] + row * (K / 64),
                     r8 ? L->idx8[p] + row * (K / 8) : NULL, L->gbook13, r8 ? L->gbook8 : NULL,
                     L->gscale13, L->gscale8, L->gain[p] ? L->gain[p] + row : NULL, K, w);
    } else {
        int64_t sb = (int64_t)K * 13 / 64;
        const uint8_t *i8 = (L->fmt == ORC_VQ13_R8) ? L->idx8[p] + row * (K / 8) : NULL;
        const uint16_t *b8 = (L->fmt == ORC_VQ13_R8) ? L->book8 : NULL;
        const uint16_t *g = L->gain[p] ? L->gain[p] + row : NULL;
        orc_row_vq(L->idx13[p] + row * sb, i8, L->book13, b8, g, K, w);
    }
}

/* Whole matrix of projection p of expert e, f32 [N][K]. */
void orc_dequant(const orc_layer *L, int e, int p, float *out)
{
    int N, K;
    proj_shape(L, p, &N, &K);
    #pragma omp parallel for schedule(static)
    for (int n = 0; n < N; ++n) orc_dequant_row(L, e, p, n, out + (int64_t)n * K);
}

/* ------------------------------------------------------------------ */
/* The FFN of one route, in f64                                        */
/* ------------------------------------------------------------------ */

/* silu(z) = z / (1 + e^-z).  For very negative z, e^-z is +inf and the
 * quotient is -0, never NaN. */
static double silu(double z) { return z / (1.0 + exp(-z)); }

/* y[H] = W_down,e ( silu(W_gate,e x) * (W_up,e x) ), every product and sum
 * in f64 from the exact f32 weights; h[I] (optional) receives the SwiGLU
 * intermediate [MIX, SPK "Recipe": gate/up/down experts]. */
void orc_expert_ffn(const orc_layer *L, int e, const double *x, double *y, double *h_out)
{
    const int H = L->H, I = L->I;
    double *h = (double *)malloc(sizeof(double) * (size_t)I);
    #pragma omp parallel
    {
        float *wg = (float *)malloc(sizeof(float) * (size_t)H);
        float *wu = (float *)malloc(sizeof(float) * (size_t)H);
        #pragma omp for schedule(static)
        for (int n = 0; n < I; ++n) {
            orc_dequant_row(L, e, 0, n, wg);
            orc_dequant_row(L, e, 1, n, wu);
            double g = 0.0, u = 0.0;
            for (int k = 0; k < H; ++k) {
                g += (double)wg[k] * x[k];
                u += (double)wu[k] * x[k];
            }
            h[n] = silu(g) * u;
        }
        free(wg);
        free(wu);
        float *wd = (float *)malloc(sizeof(float) * (size_t)I);
        #pragma omp for schedule(static)
        for (int m = 0; m < H; ++m) {
            orc_dequant_row(L, e, 2, m, wd);
            double acc = 0.0;
            for (int n = 0; n < I; ++n) acc += (double)wd[n] * h[n];
            y[m] = acc;
        }
        free(wd);
    }
    if (h_out) memcpy(h_out, h, sizeof(double) * (size_t)I);
    free(h);
}

/* ------------------------------------------------------------------ */
/* The routed layer                                                    */
/* ------------------------------------------------------------------ */

/* out[i][:] = sum over slots s of w[t][s] * FFN_{ids[t][s]}(x[t]) for each
 * requested token t = tokens[i] (tokens NULL: t = i for i < n_tok), slots
 * taken in order s = 0..k-1 [SPK "Architecture notes": top-8 of 256].
 * x is [*][H] f64, out is [n_tok][H] f64 (overwritten).  route_counts[p]
 * (optional) counts, per projection, the routes whose expert was applied
 * [IQ3 "Calibration"]; h_out (optional) is [n_tok][k][I], zero for routes
 * not applied.  Returns the number of invalid ids (not -1, not in [0,E)). */
int64_t orc_forward(const orc_layer *L, const double *x, const int32_t *ids,
                    const float *w, const int32_t *tokens, int n_tok,
                    double *out, int64_t *route_counts, double *h_out)
{
    const int H = L->H, I = L->I, k = L->k, E = L->E;
    int64_t invalid = 0;
    double *y = (double *)malloc(sizeof(double) * (size_t)H);
    if (route_counts) route_counts[0] = route_counts[1] = route_counts[2] = 0;
    for (int i = 0; i < n_tok; ++i) {
        int t = tokens ? tokens[i] : i;
        double *o = out + (int64_t)i * H;
        for (int m = 0; m < H; ++m) o[m] = 0.0;
        for (int s = 0; s < k; ++s) {
            int32_t e = ids[(int64_t)t * k + s];
            double *hs = h_out ? h_out + ((int64_t)i * k + s) * I : NULL;
            if (hs) for (int n = 0; n < I; ++n) hs[n] = 0.0;
            if (e == -1) continue;
            if (e < 0 || e >= E) { ++invalid; continue; }
            orc_expert_ffn(L, e, x + (int64_t)t * H, y, hs);
            if (route_counts) { ++route_counts[0]; ++route_counts[1]; ++route_counts[2]; }
            double ws = (double)w[(int64_t)t * k + s];
            for (int m = 0; m < H; ++m) o[m] += ws * y[m];
        }
    }
    free(y);
    return invalid;
}

/* Threads an OpenMP region of this library uses. */
int orc_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* ------------------------------------------------------------------ */
/* Route bucketing                                                     */
/* ------------------------------------------------------------------ */

/* Group the n_routes = T*k routes of a forward by expert [SPK "Speed": the
 * expert matmuls want each expert's tokens together; "Architecture notes":
 * k of E experts per token].  offsets[E+1]: offsets[e] = number of valid
 * routes with an expert below e.  perm: the valid route ids r (= t*k + s)
 * listed expert by expert, ascending r within an expert.  -1 is "no route";
 * other ids outside [0, E) are dropped.  Returns the number of dropped ids
 * other than -1. */
int64_t orc_route_bucket(const int32_t *ids, int64_t n_routes, int32_t E,
                         int32_t *offsets, int32_t *perm)
{
    int64_t invalid = 0, pos = 0;
    for (int64_t r = 0; r < n_routes; ++r)
        if (ids[r] != -1 && (ids[r] < 0 || ids[r] >= E)) ++invalid;
    for (int32_t e = 0; e < E; ++e) {
        offsets[e] = (int32_t)pos;
        for (int64_t r = 0; r < n_routes; ++r)
            if (ids[r] == e) perm[pos++] = (int32_t)r;
    }
    offsets[E] = (int32_t)pos;
    return invalid;
}
