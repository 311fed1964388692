/*
 * mxmoe_oracle.c -- plain, slow, single-threaded float64 CPU oracle for the
 * MXFP4 MoE expert layer of a decode/verify step.
 *
 * TEST INFRASTRUCTURE. Only the tests, the smoke check and the CPU-baseline
 * leg of the benchmark load this library. The CUDA library never calls it and
 * the two share no code, header, table or helper.
 *
 * What the layer is, from the pages:
 *  - "MiMo-V2.5-Pro-FP4-DFlash" model card, section 2 "FP4 Quantization":
 *    only the MoE experts are stored as MXFP4 with block size 32; everything
 *    else stays at higher precision.
 *  - nxbn.cn article on MiMo-V2.5-Pro-FP4-DFlash, section on the FP4 expert
 *    quantisation: quantization_config {store_dtype: mxfp4,
 *    mxfp4_block_size: 32}; section on the architecture: 384 experts,
 *    8 activated per token, hidden size 6144.
 *  - "MiMo-V2.5-Pro-FP4-DFlash" (alphaneural mirror), section 4 "Model
 *    Summary": hidden size 6144, 1.02T total parameters.
 * The pages do not spell out the element bit layout, the scale rule, the
 * rounding, the router function or the expert activation. The readings taken
 * here (OCP MX element/scale encodings, scale exponent floor(log2 amax) - 2,
 * round to nearest with ties to the even mantissa, saturation at 6, softmax
 * over all experts then top-k renormalised, SwiGLU experts with the gate rows
 * first) are stated at each function.
 *
 * Arithmetic: every floating-point step is done in IEEE double with plain
 * loops in the order the definition states; no blocking, no fusion.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define MXO_BLOCK 32 /* elements sharing one scale (model card, section 2) */

/* ------------------------------------------------------------------------ */
/* Element and scale encodings                                               */
/* ------------------------------------------------------------------------ */

/* Value of one E2M1 code (OCP MX element format FP4 E2M1).
 * Bit 3 is the sign, bits 2..1 the exponent field e (bias 1), bit 0 the
 * mantissa m. e == 0 is subnormal: m * 2^-1. Otherwise 2^(e-1) * (1 + m/2).
 * There is no infinity and no NaN. */
double mxo_e2m1_value(int code)
{
    int s = (code >> 3) & 1;
    int e = (code >> 1) & 3;
    int m = code & 1;
    double mag = (e == 0) ? 0.5 * (double)m : ldexp(1.0 + 0.5 * (double)m, e - 1);
    return s ? -mag : mag;
}

/* Value of one E8M0 scale byte (OCP MX shared scale): 2^(S - 127); 255 is NaN. */
double mxo_e8m0_value(int s)
{
    if (s == 255)
        return NAN;
    return ldexp(1.0, s - 127);
}

/* bfloat16 bits -> double (exact: a bf16 value is the top half of a float). */
static double bf16_to_double(uint16_t b)
{
    uint32_t u = ((uint32_t)b) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

double mxo_bf16_to_double(uint16_t b) { return bf16_to_double(b); }

/* Round a non-negative, exactly scaled magnitude q to an E2M1 magnitude code
 * (0..7): the nearest representable value; on a tie, the code whose mantissa
 * bit is 0; anything at or above 6 saturates to 6 (code 7). grid[c] is the
 * value of magnitude code c. */
static int e2m1_round_magnitude(double q, const double grid[8])
{
    if (q >= 6.0)
        return 7;
    int best = 0;
    double bestd = fabs(q - grid[0]);
    for (int c = 1; c < 8; ++c) {
        double d = fabs(q - grid[c]);
        if (d < bestd || (d == bestd && (c & 1) == 0 && (best & 1) == 1)) {
            best = c;
            bestd = d;
        }
    }
    return best;
}

static void e2m1_grid(double grid[8])
{
    for (int c = 0; c < 8; ++c)
        grid[c] = mxo_e2m1_value(c);
}

int mxo_e2m1_round(double q)
{
    double grid[8];
    e2m1_grid(grid);
    return e2m1_round_magnitude(q, grid);
}

/* ------------------------------------------------------------------------ */
/* Quantise / dequantise                                                     */
/* ------------------------------------------------------------------------ */

/* bf16 [rows, K] row-major -> packed [rows, K/2] + scales [rows, K/32].
 *
 * Per 32-element block along K (model card, section 2, "MXFP4 (block size
 * 32)"):
 *   amax = max |x|;
 *   scale exponent e = floor(log2 amax) - 2, clamped to [-127, 127]; a block
 *   whose amax is 0 gets e = -127 (scale byte 0);
 *   scale byte S = e + 127 (E8M0);
 *   each element: q = |x| / 2^e (exact), rounded to the nearest E2M1
 *   magnitude (ties to even mantissa, saturating at 6); the sign bit of x is
 *   kept, also when the magnitude rounds to 0.
 * Packing: element 2j of a row is the low nibble of byte j, element 2j+1 the
 * high nibble. K must be a multiple of 32. */
void mxo_quantize(const uint16_t *w, int64_t rows, int64_t K, uint8_t *packed, uint8_t *scales)
{
    int64_t nblk = K / MXO_BLOCK;
    double grid[8];
    e2m1_grid(grid);
    for (int64_t r = 0; r < rows; ++r) {
        for (int64_t b = 0; b < nblk; ++b) {
            double v[MXO_BLOCK];
            double amax = 0.0;
            for (int i = 0; i < MXO_BLOCK; ++i) {
                v[i] = bf16_to_double(w[r * K + b * MXO_BLOCK + i]);
                if (fabs(v[i]) > amax)
                    amax = fabs(v[i]);
            }
            int e;
            if (amax == 0.0) {
                e = -127;
            } else {
                int ex;
                frexp(amax, &ex); /* amax = f * 2^ex, f in [0.5, 1) */
                e = (ex - 1) - 2; /* floor(log2 amax) - 2 */
                if (e < -127)
                    e = -127;
                if (e > 127)
                    e = 127;
            }
            scales[r * nblk + b] = (uint8_t)(e + 127);
            for (int i = 0; i < MXO_BLOCK; ++i) {
                double q = ldexp(fabs(v[i]), -e);
                int code = e2m1_round_magnitude(q, grid) | (signbit(v[i]) ? 8 : 0);
                int64_t k = b * MXO_BLOCK + i;
                uint8_t *byte = &packed[r * (K / 2) + k / 2];
                if ((k & 1) == 0)
                    *byte = (uint8_t)((*byte & 0xF0) | code);
                else
                    *byte = (uint8_t)((*byte & 0x0F) | (code << 4));
            }
        }
    }
}

/* packed [rows, K/2] + scales [rows, K/32] -> double [rows, K]:
 * element value = E2M1(code) * 2^(S - 127). */
void mxo_dequantize(const uint8_t *packed, const uint8_t *scales, int64_t rows, int64_t K, double *out)
{
    int64_t nblk = K / MXO_BLOCK;
    double value[16];
    for (int c = 0; c < 16; ++c)
        value[c] = mxo_e2m1_value(c);
    for (int64_t r = 0; r < rows; ++r) {
        for (int64_t b = 0; b < nblk; ++b) {
            double s = mxo_e8m0_value(scales[r * nblk + b]);
            for (int64_t k = b * MXO_BLOCK; k < (b + 1) * MXO_BLOCK; ++k) {
                uint8_t byte = packed[r * (K / 2) + k / 2];
                int code = (k & 1) ? (byte >> 4) : (byte & 0x0F);
                out[r * K + k] = value[code] * s;
            }
        }
    }
}

/* ------------------------------------------------------------------------ */
/* Router                                                                    */
/* ------------------------------------------------------------------------ */

/* logits[t, e] = sum_k x[t, k] * Wg[e, k]  (+ bias[e] when bias != NULL).
 * x bf16 [T, H], Wg bf16 [E, H], bias float [E]; the router is the plain
 * linear gate of an MoE layer (384 experts, nxbn.cn article, architecture
 * section); bias is an optional per-expert additive term. */
void mxo_router_logits(const uint16_t *x, const uint16_t *wg, const float *bias, int64_t T, int64_t H,
                       int64_t E, double *logits)
{
    for (int64_t t = 0; t < T; ++t) {
        for (int64_t e = 0; e < E; ++e) {
            double acc = 0.0;
            for (int64_t k = 0; k < H; ++k)
                acc += bf16_to_double(x[t * H + k]) * bf16_to_double(wg[e * H + k]);
            if (bias)
                acc += (double)bias[e];
            logits[t * E + e] = acc;
        }
    }
}

/* Route each token to its top-k experts (8 of 384 in the layer on the pages).
 * Steps, in order: p = softmax over all E logits; take the k largest p, a tie
 * going to the lower expert index; renormalise the k selected p to sum 1.
 * ids int32 [T, k] in selection order (largest first), w double [T, k]. */
void mxo_route(const double *logits, int64_t T, int64_t E, int k, int32_t *ids, double *w)
{
    double *p = (double *)malloc(sizeof(double) * (size_t)E);
    char *taken = (char *)malloc((size_t)E);
    for (int64_t t = 0; t < T; ++t) {
        const double *l = logits + t * E;
        double lmax = l[0];
        for (int64_t e = 1; e < E; ++e)
            if (l[e] > lmax)
                lmax = l[e];
        double z = 0.0;
        for (int64_t e = 0; e < E; ++e) {
            p[e] = exp(l[e] - lmax);
            z += p[e];
        }
        for (int64_t e = 0; e < E; ++e)
            p[e] /= z;
        memset(taken, 0, (size_t)E);
        for (int j = 0; j < k; ++j) {
            int64_t best = -1;
            for (int64_t e = 0; e < E; ++e)
                if (!taken[e] && (best < 0 || p[e] > p[best]))
                    best = e;
            taken[best] = 1;
            ids[t * k + j] = (int32_t)best;
        }
        double s = 0.0;
        for (int j = 0; j < k; ++j)
            s += p[ids[t * k + j]];
        for (int j = 0; j < k; ++j)
            w[t * k + j] = p[ids[t * k + j]] / s;
    }
    free(p);
    free(taken);
}

/* Same routing from float32 logits (converted exactly to double first). */
void mxo_route_f32(const float *logits, int64_t T, int64_t E, int k, int32_t *ids, double *w)
{
    double *l = (double *)malloc(sizeof(double) * (size_t)(T * E));
    for (int64_t i = 0; i < T * E; ++i)
        l[i] = (double)logits[i];
    mxo_route(l, T, E, k, ids, w);
    free(l);
}

/* ------------------------------------------------------------------------ */
/* Permute / combine                                                         */
/* ------------------------------------------------------------------------ */

/* Group the T*k (token, slot) pairs by expert.
 * offsets int32 [E+1]: offsets[e] = number of pairs routed to experts < e.
 * src_row int32 [T*k]: the pair index t*k + j at each grouped position,
 *   experts ascending, and within one expert pairs in ascending (t, j).
 * dst_of int32 [T*k]: the grouped position of pair t*k + j. */
void mxo_permute(const int32_t *ids, int64_t T, int k, int64_t E, int32_t *offsets, int32_t *src_row,
                 int32_t *dst_of)
{
    int64_t n = T * k;
    int64_t *count = (int64_t *)calloc((size_t)E, sizeof(int64_t));
    int64_t *cursor = (int64_t *)calloc((size_t)E, sizeof(int64_t));
    for (int64_t p = 0; p < n; ++p)
        count[ids[p]] += 1;
    offsets[0] = 0;
    for (int64_t e = 0; e < E; ++e)
        offsets[e + 1] = offsets[e] + (int32_t)count[e];
    for (int64_t e = 0; e < E; ++e)
        cursor[e] = offsets[e];
    for (int64_t p = 0; p < n; ++p) {
        int64_t pos = cursor[ids[p]]++;
        src_row[pos] = (int32_t)p;
        dst_of[p] = (int32_t)pos;
    }
    free(count);
    free(cursor);
}

/* y[t, c] = sum over j = 0..k-1, in that order, of w[t, j] * y_perm[dst_of[t*k + j], c]. */
void mxo_combine(const double *y_perm, const int32_t *dst_of, const double *w, int64_t T, int k, int64_t H,
                 double *y)
{
    for (int64_t t = 0; t < T; ++t) {
        for (int64_t c = 0; c < H; ++c) {
            double acc = 0.0;
            for (int j = 0; j < k; ++j)
                acc += w[t * k + j] * y_perm[(int64_t)dst_of[t * k + j] * H + c];
            y[t * H + c] = acc;
        }
    }
}

/* ------------------------------------------------------------------------ */
/* Expert FFN                                                                */
/* ------------------------------------------------------------------------ */

/* One expert applied to n activation rows.
 * w13 double [2I, H]: rows 0..I-1 are the gate projection, rows I..2I-1 the
 * up projection; w2 double [H, I] is the down projection; x bf16 [n, H].
 *   g = W_gate x, u = W_up x, h = silu(g) * u = g / (1 + e^-g) * u,
 *   y = W_down h.
 * No biases and no clamp. h_out (double [n, I]) may be NULL. */
void mxo_expert_ffn(const double *w13, const double *w2, const uint16_t *x, int64_t n, int64_t H, int64_t I,
                    double *h_out, double *y)
{
    double *xd = (double *)malloc(sizeof(double) * (size_t)H);
    double *h = (double *)malloc(sizeof(double) * (size_t)I);
    for (int64_t r = 0; r < n; ++r) {
        for (int64_t k = 0; k < H; ++k)
            xd[k] = bf16_to_double(x[r * H + k]);
        for (int64_t i = 0; i < I; ++i) {
            double g = 0.0, u = 0.0;
            for (int64_t k = 0; k < H; ++k) {
                g += w13[i * H + k] * xd[k];
                u += w13[(I + i) * H + k] * xd[k];
            }
            h[i] = g / (1.0 + exp(-g)) * u;
            if (h_out)
                h_out[r * I + i] = h[i];
        }
        for (int64_t c = 0; c < H; ++c) {
            double acc = 0.0;
            for (int64_t i = 0; i < I; ++i)
                acc += w2[c * I + i] * h[i];
            y[r * H + c] = acc;
        }
    }
    free(xd);
    free(h);
}

/* Decode one expert's MXFP4 weights to double and run it on n rows.
 * packed13 [2I, H/2], sc13 [2I, H/32], packed2 [H, I/2], sc2 [H, I/32]. */
void mxo_expert_ffn_mxfp4(const uint8_t *packed13, const uint8_t *sc13, const uint8_t *packed2,
                          const uint8_t *sc2, const uint16_t *x, int64_t n, int64_t H, int64_t I,
                          double *h_out, double *y)
{
    double *w13 = (double *)malloc(sizeof(double) * (size_t)(2 * I * H));
    double *w2 = (double *)malloc(sizeof(double) * (size_t)(H * I));
    mxo_dequantize(packed13, sc13, 2 * I, H, w13);
    mxo_dequantize(packed2, sc2, H, I, w2);
    mxo_expert_ffn(w13, w2, x, n, H, I, h_out, y);
    free(w13);
    free(w2);
}

/* ------------------------------------------------------------------------ */
/* FP8 expert weights (the pages' quality baseline)                          */
/* ------------------------------------------------------------------------ */

/* The model card's section 2 compares the MXFP4 experts with an FP8 baseline
 * and its introduction says that lowering the bit width per parameter speeds
 * up decoding; the pages give no FP8 layout. The reading here keeps the MX
 * family of the FP4 experts: E4M3 elements with one E8M0 scale per 32
 * elements along K (OCP MX FP8, "MXFP8"), the scale exponent chosen the same
 * way as for E2M1 -- floor(log2 amax) minus the exponent of the element
 * format's largest power of two (2 for E2M1, whose largest value is 1.5 * 2^2;
 * 8 for E4M3, whose largest value is 1.75 * 2^8). */

/* Value of one E4M3 code (OCP 8-bit floating point, E4M3).
 * Bit 7 is the sign, bits 6..3 the exponent field e (bias 7), bits 2..0 the
 * mantissa m. e == 0 is subnormal: (m / 8) * 2^-6. Otherwise
 * 2^(e-7) * (1 + m/8). Codes 0x7F and 0xFF (e = 15, m = 7) are NaN; there is
 * no infinity, so the largest finite magnitude is 2^8 * 1.75 = 448. */
double mxo_e4m3_value(int code)
{
    int s = (code >> 7) & 1;
    int e = (code >> 3) & 15;
    int m = code & 7;
    if (e == 15 && m == 7)
        return NAN;
    double mag = (e == 0) ? ldexp((double)m / 8.0, -6) : ldexp(1.0 + (double)m / 8.0, e - 7);
    return s ? -mag : mag;
}

/* Round a non-negative, exactly scaled magnitude q to an E4M3 magnitude code
 * (0x00 .. 0x7E): the nearest finite E4M3 value; on a tie, the code whose
 * mantissa's lowest bit is 0; anything above 448 saturates to 448 (0x7E).
 * A plain search over the 127 finite magnitudes. */
int mxo_e4m3_round(double q)
{
    if (q >= 448.0)
        return 0x7E;
    int best = 0;
    double bestd = fabs(q - mxo_e4m3_value(0));
    for (int c = 1; c <= 0x7E; ++c) {
        double d = fabs(q - mxo_e4m3_value(c));
        if (d < bestd || (d == bestd && (c & 1) == 0 && (best & 1) == 1)) {
            best = c;
            bestd = d;
        }
    }
    return best;
}

/* bf16 [rows, K] row-major -> E4M3 codes [rows, K] (one byte per element) +
 * scales [rows, K/32].
 * Per 32-element block along K:
 *   amax = max |x|;
 *   scale exponent e = floor(log2 amax) - 8, clamped to [-127, 127]; a block
 *   whose amax is 0 gets e = -127 (scale byte 0);
 *   scale byte S = e + 127 (E8M0);
 *   each element: q = |x| / 2^e (exact), rounded to the nearest E4M3
 *   magnitude (ties to the even mantissa, saturating at 448); the sign bit
 *   of x is kept, also when the magnitude rounds to 0.
 * K must be a multiple of 32. */
void mxo_quantize_fp8(const uint16_t *w, int64_t rows, int64_t K, uint8_t *codes, uint8_t *scales)
{
    int64_t nblk = K / MXO_BLOCK;
    for (int64_t r = 0; r < rows; ++r) {
        for (int64_t b = 0; b < nblk; ++b) {
            double v[MXO_BLOCK];
            double amax = 0.0;
            for (int i = 0; i < MXO_BLOCK; ++i) {
                v[i] = bf16_to_double(w[r * K + b * MXO_BLOCK + i]);
                if (fabs(v[i]) > amax)
                    amax = fabs(v[i]);
            }
            int e;
            if (amax == 0.0) {
                e = -127;
            } else {
                int ex;
                frexp(amax, &ex); /* amax = f * 2^ex, f in [0.5, 1) */
                e = (ex - 1) - 8; /* floor(log2 amax) - 8 */
                if (e < -127)
                    e = -127;
                if (e > 127)
                    e = 127;
            }
            scales[r * nblk + b] = (uint8_t)(e + 127);
            for (int i = 0; i < MXO_BLOCK; ++i) {
                double q = ldexp(fabs(v[i]), -e);
                codes[r * K + b * MXO_BLOCK + i] = (uint8_t)(mxo_e4m3_round(q) | (signbit(v[i]) ? 0x80 : 0));
            }
        }
    }
}

/* codes [rows, K] + scales [rows, K/32] -> double [rows, K]:
 * element value = E4M3(code) * 2^(S - 127). */
void mxo_dequantize_fp8(const uint8_t *codes, const uint8_t *scales, int64_t rows, int64_t K, double *out)
{
    int64_t nblk = K / MXO_BLOCK;
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t b = 0; b < nblk; ++b) {
            double s = mxo_e8m0_value(scales[r * nblk + b]);
            for (int64_t k = b * MXO_BLOCK; k < (b + 1) * MXO_BLOCK; ++k)
                out[r * K + k] = mxo_e4m3_value(codes[r * K + k]) * s;
        }
}

/* Decode one expert's FP8 weights to double and run it on n rows (the same
 * SwiGLU expert as mxo_expert_ffn). codes13 [2I, H], sc13 [2I, H/32],
 * codes2 [H, I], sc2 [H, I/32]. */
void mxo_expert_ffn_fp8(const uint8_t *codes13, const uint8_t *sc13, const uint8_t *codes2, const uint8_t *sc2,
                        const uint16_t *x, int64_t n, int64_t H, int64_t I, double *h_out, double *y)
{
    double *w13 = (double *)malloc(sizeof(double) * (size_t)(2 * I * H));
    double *w2 = (double *)malloc(sizeof(double) * (size_t)(H * I));
    mxo_dequantize_fp8(codes13, sc13, 2 * I, H, w13);
    mxo_dequantize_fp8(codes2, sc2, H, I, w2);
    mxo_expert_ffn(w13, w2, x, n, H, I, h_out, y);
    free(w13);
    free(w2);
}

/* ------------------------------------------------------------------------ */
/* Block verification of a speculative draft                                 */
/* ------------------------------------------------------------------------ */

/* softmax(z / tau) of one row of V float logits into p (double). */
static void softmax_row(const float *z, int64_t V, double tau, double *p)
{
    double zmax = (double)z[0];
    for (int64_t v = 1; v < V; ++v)
        if ((double)z[v] > zmax)
            zmax = (double)z[v];
    double s = 0.0;
    for (int64_t v = 0; v < V; ++v) {
        p[v] = exp(((double)z[v] - zmax) / tau);
        s += p[v];
    }
    for (int64_t v = 0; v < V; ++v)
        p[v] /= s;
}

/* Index of the largest of V float logits, a tie going to the lower index. */
static int64_t argmax_row(const float *z, int64_t V)
{
    int64_t best = 0;
    for (int64_t v = 1; v < V; ++v)
        if (z[v] > z[best])
            best = v;
    return best;
}

/* Verify B blocks of K drafted tokens against the backbone.
 *
 * "MiMo-V2.5-Pro-FP4-DFlash" (alphaneural mirror), section 3 "Block-Diffusion
 * Speculative Decoding (DFlash)": the drafter fills a whole block of masked
 * positions (at most 8) in one forward pass, the backbone verifies the block
 * in one step, and the rejection-sampling verification keeps the output
 * lossless. The pages give no formula; the reading here is the standard
 * speculative-sampling test, taken position by position in block order:
 *   p_i = softmax(z_i / tau) from the backbone's logits z_i at block position
 *   i, q_i = softmax(w_i / tau) from the drafter's logits w_i;
 *   draft token d_i is accepted when u_i * q_i(d_i) < p_i(d_i), u_i uniform
 *   in [0, 1) and passed in;
 *   at the first rejection j the output token is drawn from max(0, p_j - q_j)
 *   normalised, and after K acceptances from p_K, both by inverse CDF in
 *   token order with u_K: the smallest v whose running sum exceeds u_K times
 *   the total (the last v with a non-zero weight if rounding leaves none).
 * tau = 0 is greedy verification: d_i is accepted while it equals the argmax
 * of z_i (a tie going to the lower token index); the output token is the
 * argmax of z_n at the first mismatch n (n = K after K matches).
 * A draft token outside [0, V) is never accepted.
 *
 * target float [B][K+1][V]; draft float [B][K][V] (not read when tau = 0);
 * dtok int32 [B][K]; u float [B][K+1]; accepted int32 [B]; tokens int32
 * [B][K+1]: the accepted drafts, then the output token, then -1.
 * margin_acc, margin_draw (each may be NULL) double [B]: how far the
 * decisions taken lie from their thresholds, for tests that compare with
 * lower-precision arithmetic: the smallest |u q - p| / max(u q, p) over the
 * acceptance tests taken, and the distance of u_K times the total from the
 * nearer running-sum boundary of the drawn token, over the total; infinity for
 * greedy verification, whose comparisons are exact. */
void mxo_verify_block(const float *target, const float *draft, const int32_t *dtok, const float *u, int64_t B, int K,
                      int64_t V, double tau, int32_t *accepted, int32_t *tokens, double *margin_acc,
                      double *margin_draw)
{
    double *p = (double *)malloc(sizeof(double) * (size_t)V);
    double *q = (double *)malloc(sizeof(double) * (size_t)V);
    for (int64_t b = 0; b < B; ++b) {
        const float *zb = target + b * (int64_t)(K + 1) * V;
        const float *wb = draft ? draft + b * (int64_t)K * V : NULL;
        const int32_t *db = dtok + b * K;
        const float *ub = u + b * (K + 1);
        double mg = INFINITY, mgd = INFINITY;
        int n = 0;
        int64_t out = 0;
        if (tau == 0.0) {
            while (n < K && db[n] >= 0 && db[n] < V && argmax_row(zb + (int64_t)n * V, V) == db[n])
                ++n;
            out = argmax_row(zb + (int64_t)n * V, V);
        } else {
            for (n = 0; n < K; ++n) {
                const int32_t d = db[n];
                if (d < 0 || d >= V)
                    break;
                softmax_row(zb + (int64_t)n * V, V, tau, p);
                softmax_row(wb + (int64_t)n * V, V, tau, q);
                const double lhs = (double)ub[n] * q[d], rhs = p[d];
                const double den = lhs > rhs ? lhs : rhs;
                if (den > 0.0 && fabs(lhs - rhs) / den < mg)
                    mg = fabs(lhs - rhs) / den;
                if (!(lhs < rhs))
                    break;
            }
            /* the weights of the draw: residual at a rejection, else p_K */
            softmax_row(zb + (int64_t)n * V, V, tau, p);
            if (n < K) {
                softmax_row(wb + (int64_t)n * V, V, tau, q);
                for (int64_t v = 0; v < V; ++v)
                    p[v] = p[v] > q[v] ? p[v] - q[v] : 0.0;
            }
            double total = 0.0;
            for (int64_t v = 0; v < V; ++v)
                total += p[v];
            const double thr = (double)ub[K] * total;
            double run = 0.0;
            out = -1;
            for (int64_t v = 0; v < V; ++v) {
                const double before = run;
                run += p[v];
                if (run > thr) {
                    out = v;
                    const double gap = (thr - before) < (run - thr) ? (thr - before) : (run - thr);
                    mgd = gap / total;
                    break;
                }
            }
            if (out < 0)
                for (int64_t v = V - 1; v >= 0; --v)
                    if (p[v] > 0.0) {
                        out = v;
                        break;
                    }
        }
        accepted[b] = n;
        for (int i = 0; i <= K; ++i)
            tokens[b * (K + 1) + i] = i < n ? db[i] : (i == n ? (int32_t)out : -1);
        if (margin_acc)
            margin_acc[b] = mg;
        if (margin_draw)
            margin_draw[b] = mgd;
    }
    free(p);
    free(q);
}

/* The interval [lo, hi) that token v covers in the normalised running sum of
 * a draw's weights (the same weights as in mxo_verify_block): the residual
 * max(0, p - q) when a drafter row w is given, else p; p = softmax(z / tau),
 * q = softmax(w / tau). A draw with uniform u yields v exactly when
 * lo <= u < hi. */
void mxo_draw_interval(const float *z, const float *w, int64_t V, double tau, int64_t v, double *lo, double *hi)
{
    double *p = (double *)malloc(sizeof(double) * (size_t)V);
    double *q = (double *)malloc(sizeof(double) * (size_t)V);
    softmax_row(z, V, tau, p);
    if (w) {
        softmax_row(w, V, tau, q);
        for (int64_t i = 0; i < V; ++i)
            p[i] = p[i] > q[i] ? p[i] - q[i] : 0.0;
    }
    double total = 0.0, before = 0.0;
    for (int64_t i = 0; i < V; ++i) {
        if (i == v)
            before = total;
        total += p[i];
    }
    *lo = before / total;
    *hi = (before + p[v]) / total;
    free(p);
    free(q);
}
