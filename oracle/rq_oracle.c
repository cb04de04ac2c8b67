/*
 * rq_oracle.c -- CPU oracle for the ResidualQuant hot path.
 *
 * TEST INFRASTRUCTURE ONLY (see rq_oracle.h).  Plain scalar C, single
 * threaded, compiled with -ffp-contract=off so that every float expression
 * below is evaluated as written: one IEEE binary32 (or binary64) operation
 * at a time, round-to-nearest-even, subnormals kept.
 *
 * Method: "ResidualQuant: KV Cache Quantization for Looped Transformers with
 * 2-Bit Residuals", Abstract: final-loop K/V as the reference, the other
 * loops as rotated, least-squares-scaled low-bit residuals, bit width chosen
 * per loop.  Each function names the step of the method it restates and the
 * reading it takes where the page leaves the step open.
 */
#include "rq_oracle.h"

#include <float.h>
#include <math.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------------ */
/* scalar formats                                                            */
/* ------------------------------------------------------------------------ */

/* bf16 is the upper 16 bits of a binary32: widening is exact. */
float orq_bf16_to_f32(uint16_t h)
{
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

double orq_f16_to_f64(uint16_t h)
{
    _Float16 v;
    memcpy(&v, &h, sizeof v);
    return (double)v;
}

/* Scales are stored as fp16, rounded to nearest even (reading: the page
 * fixes no scale format; fp16 RN is the plainest choice). */
uint16_t orq_f64_to_f16(double x)
{
    _Float16 v = (_Float16)x;
    uint16_t h;
    memcpy(&h, &v, sizeof h);
    return h;
}

/* ------------------------------------------------------------------------ */
/* seeded signs: the random part of the rotation                             */
/* ------------------------------------------------------------------------ */

/* splitmix64 (Steele, Lea and Flood, "Fast splittable pseudorandom number
 * generators", OOPSLA 2014), used as a counter-based generator: output i of
 * the stream started at `seed` is the mix of seed + (i+1)*golden-gamma. */
uint64_t orq_splitmix64(uint64_t seed, uint64_t i)
{
    uint64_t z = seed + (i + 1u) * 0x9E3779B97F4A7C15ull;
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    return z ^ (z >> 31);
}

/* D = diag(+-1): D_i = -1 exactly when the top bit of output i is set.
 * One sign vector per seed, shared by every layer, head, loop, K and V. */
void orq_signs(uint64_t seed, int d, int8_t *D)
{
    for (int i = 0; i < d; ++i)
        D[i] = (orq_splitmix64(seed, (uint64_t)i) >> 63) ? -1 : 1;
}

/* ------------------------------------------------------------------------ */
/* rotation (Abstract: the residuals are rotated before quantisation)        */
/* Reading: Rot = c_d * H_d * D, H_d the Sylvester Hadamard matrix.          */
/* ------------------------------------------------------------------------ */

/* c_d = 1/sqrt(d) rounded once to binary32. */
float orq_cd_f32(int d)
{
    return (float)(1.0 / sqrt((double)d));
}

/* Sylvester Hadamard entry: (-1)^popcount(i & j). */
int orq_hadamard_entry(int i, int j)
{
    unsigned v = (unsigned)(i & j);
    int parity = 0;
    while (v) {
        parity ^= (int)(v & 1u);
        v >>= 1;
    }
    return parity ? -1 : 1;
}

/* R[i][j] = (1/sqrt(d)) * H[i][j] * D[j], in double. */
void orq_rotation_matrix_f64(int d, const int8_t *D, double *R)
{
    double cd = 1.0 / sqrt((double)d);
    for (int i = 0; i < d; ++i)
        for (int j = 0; j < d; ++j)
            R[(size_t)i * d + j] = cd * (double)orq_hadamard_entry(i, j) * (double)D[j];
}

/* Unnormalised fast Walsh-Hadamard transform in double, same stage order as
 * the fp32 path.  Used only to pin the fp32 butterfly against the matrix. */
void orq_fwht_f64(int d, double *v)
{
    for (int h = 1; h < d; h <<= 1)
        for (int i = 0; i < d; i += 2 * h)
            for (int j = i; j < i + h; ++j) {
                double a = v[j], b = v[j + h];
                v[j] = a + b;
                v[j + h] = a - b;
            }
}

/* y = c_d * FWHT(D r) in binary32.  Spec of the arithmetic (reading): flip
 * signs (exact), then butterfly stages h = 1, 2, 4, ..., d/2, each pair
 * (a at the lower index, b at index + h) becoming (a + b, a - b), each one
 * RN binary32 operation; finally one RN multiply by c_d. */
void orq_rotate_f32(int d, const int8_t *D, const float *r, float *y)
{
    float v[ORQ_MAX_D];
    for (int i = 0; i < d; ++i)
        v[i] = D[i] < 0 ? -r[i] : r[i];
    for (int h = 1; h < d; h <<= 1)
        for (int i = 0; i < d; i += 2 * h)
            for (int j = i; j < i + h; ++j) {
                float a = v[j], b = v[j + h];
                v[j] = a + b;
                v[j + h] = a - b;
            }
    float cd = orq_cd_f32(d);
    for (int i = 0; i < d; ++i)
        y[i] = v[i] * cd;
}

/* ------------------------------------------------------------------------ */
/* group quantiser (Abstract: INT2 residuals with a least-squares scale;     */
/* loop-wise mixed precision lets a loop use more bits)                      */
/* ------------------------------------------------------------------------ */

/* One group of g rotated coordinates, b = bits in {2, 4}.
 * Readings:
 *   grid   : symmetric mid-rise, levels l = 2c - (2^b - 1), i.e. odd
 *            integers in [-(2^b-1), 2^b-1]; every code is used.
 *   init   : the outermost level maps to the group's absmax:
 *            inv = (2^(b-1) - 1/2) / amax  (binary32 division);
 *            inv = 0 when amax is zero or subnormal (< FLT_MIN).
 *   code   : u = y * inv (binary32), c = clamp(floor(u) + 2^(b-1), 0, 2^b-1).
 *            A u that is exactly an integer sits on a decision boundary;
 *            floor sends it to the upper level.  These are counted as ties.
 *   scale  : for the fixed codes, s = <y, l> / <l, l> minimises ||y - s l||^2
 *            (the least-squares scale); computed in double here, then
 *            clamped to +-65504 and rounded to fp16.
 * s_exact receives the unrounded double scale. */
void orq_quantize_group_f32(int g, int bits, const float *y, uint8_t *codes,
                            double *s_exact, uint16_t *s_f16, int *ties)
{
    const int nlev = 1 << bits;
    const int half = 1 << (bits - 1);

    float amax = 0.0f;
    for (int i = 0; i < g; ++i) {
        float a = fabsf(y[i]);
        if (a > amax)
            amax = a;
    }
    const float outer = (float)half - 0.5f;        /* 1.5 or 7.5, exact */
    const float inv = (amax < FLT_MIN) ? 0.0f : outer / amax;

    double num = 0.0, den = 0.0;
    int nties = 0;
    for (int i = 0; i < g; ++i) {
        float u = y[i] * inv;
        float fl = floorf(u);
        if (inv != 0.0f && fl == u)
            ++nties;
        int c = (int)fl + half;
        if (c < 0)
            c = 0;
        if (c > nlev - 1)
            c = nlev - 1;
        codes[i] = (uint8_t)c;
        int lvl = 2 * c - (nlev - 1);
        num += (double)y[i] * (double)lvl;
        den += (double)(lvl * lvl);
    }
    double s = num / den;
    if (s > 65504.0)
        s = 65504.0;
    if (s < -65504.0)
        s = -65504.0;
    if (s_exact)
        *s_exact = s;
    *s_f16 = orq_f64_to_f16(s);
    if (ties)
        *ties += nties;
}

/* Packing (reading): element j of a row in word j / (32/b), bit offset
 * b * (j mod 32/b), least significant bits first.  A row takes
 * ceil(d*b/32) words (exactly d*b/32 for the head sizes the library takes). */
void orq_pack_codes(int d, int bits, const uint8_t *codes, uint32_t *words)
{
    const int per = 32 / bits;
    for (int w = 0; w < (d + per - 1) / per; ++w)
        words[w] = 0u;
    for (int j = 0; j < d; ++j)
        words[j / per] |= (uint32_t)codes[j] << (bits * (j % per));
}

void orq_unpack_codes(int d, int bits, const uint32_t *words, uint8_t *codes)
{
    const int per = 32 / bits;
    const uint32_t mask = (1u << bits) - 1u;
    for (int j = 0; j < d; ++j)
        codes[j] = (uint8_t)((words[j / per] >> (bits * (j % per))) & mask);
}

/* ------------------------------------------------------------------------ */
/* encoder                                                                   */
/* ------------------------------------------------------------------------ */

/* Residual against the final-loop reference (Abstract), widened to binary32
 * and subtracted once (RN), then rotated and quantised group by group. */
void orq_encode_row_f32(int d, int g, int bits, const int8_t *D,
                        const uint16_t *x, const uint16_t *ref,
                        uint32_t *words, uint16_t *scales, int *ties)
{
    float r[ORQ_MAX_D], y[ORQ_MAX_D];
    uint8_t c[ORQ_MAX_D];
    for (int i = 0; i < d; ++i)
        r[i] = orq_bf16_to_f32(x[i]) - orq_bf16_to_f32(ref[i]);
    orq_rotate_f32(d, D, r, y);
    for (int k = 0; k < d / g; ++k)
        orq_quantize_group_f32(g, bits, y + k * g, c + k * g, NULL, scales + k, ties);
    orq_pack_codes(d, bits, c, words);
}

long orq_encode_rows_f32(long n_rows, int d, int g, int bits, uint64_t seed,
                         const uint16_t *x, const uint16_t *ref,
                         uint32_t *words, uint16_t *scales)
{
    int8_t D[ORQ_MAX_D];
    orq_signs(seed, d, D);
    const int wpr = (d * bits + 31) / 32;
    long ties = 0;
    for (long row = 0; row < n_rows; ++row) {
        int t = 0;
        orq_encode_row_f32(d, g, bits, D, x + row * d, ref + row * d,
                           words + row * wpr, scales + row * (d / g), &t);
        ties += t;
    }
    return ties;
}

/* ------------------------------------------------------------------------ */
/* least-squares refinement                                                  */
/* ------------------------------------------------------------------------ */

float orq_ls_dot_f32(int g, const float *y, const int *lvl)
{
    if (g < 32) {                       /* a single chain */
        float acc = 0.0f;
        for (int i = 0; i < g; ++i)
            acc = fmaf(y[i], (float)lvl[i], acc);
        return acc;
    }
    float total = 0.0f;
    for (int b = 0; b < g / 32; ++b) {
        float run[2];
        for (int h = 0; h < 2; ++h) {
            float acc = 0.0f;
            for (int i = 0; i < 16; ++i) {
                const int j = 32 * b + 16 * h + i;
                acc = fmaf(y[j], (float)lvl[j], acc);
            }
            run[h] = acc;
        }
        const float blk = run[0] + run[1];
        total = (b == 0) ? blk : total + blk;
    }
    return total;
}

/* codes of one group for the step 1 / (2 inv): nearest odd level, ties up */
static void quantize_with_inv_f32(int g, int bits, const float *y, float inv,
                                  uint8_t *codes, int *lvl)
{
    const int nlev = 1 << bits;
    const int half = 1 << (bits - 1);
    for (int i = 0; i < g; ++i) {
        float fl = floorf(y[i] * inv);
        if (fl < (float)-half)
            fl = (float)-half;
        if (fl > (float)(half - 1))
            fl = (float)(half - 1);
        const int c = (int)fl + half;
        codes[i] = (uint8_t)c;
        lvl[i] = 2 * c - (nlev - 1);
    }
}

static float ls_scale_f32(int g, const float *y, const int *lvl)
{
    int nrm = 0;
    for (int i = 0; i < g; ++i)
        nrm += lvl[i] * lvl[i];
    return orq_ls_dot_f32(g, y, lvl) / (float)nrm;
}

void orq_quantize_group_refined_f32(int g, int bits, const float *y, int iters,
                                    uint8_t *codes, float *s_out, uint16_t *s_f16)
{
    const int half = 1 << (bits - 1);
    int lvl[ORQ_MAX_D];
    float amax = 0.0f;
    for (int i = 0; i < g; ++i) {
        const float a = fabsf(y[i]);
        if (a > amax)
            amax = a;
    }
    const float outer = (float)half - 0.5f;
    const float inv0 = (amax < FLT_MIN) ? 0.0f : outer / amax;
    quantize_with_inv_f32(g, bits, y, inv0, codes, lvl);
    float s = ls_scale_f32(g, y, lvl);
    for (int k = 0; k < iters; ++k) {
        if (!(s >= FLT_MIN))
            break;
        quantize_with_inv_f32(g, bits, y, 0.5f / s, codes, lvl);
        s = ls_scale_f32(g, y, lvl);
    }
    if (s > 65504.0f)
        s = 65504.0f;
    if (s < -65504.0f)
        s = -65504.0f;
    if (s_out)
        *s_out = s;
    *s_f16 = orq_f64_to_f16((double)s);
}

void orq_encode_row_refined_f32(int d, int g, int bits, const int8_t *D, int iters,
                                const uint16_t *x, const uint16_t *ref,
                                uint32_t *words, uint16_t *scales)
{
    float r[ORQ_MAX_D], y[ORQ_MAX_D];
    uint8_t c[ORQ_MAX_D];
    for (int i = 0; i < d; ++i)
        r[i] = orq_bf16_to_f32(x[i]) - orq_bf16_to_f32(ref[i]);
    orq_rotate_f32(d, D, r, y);
    for (int k = 0; k < d / g; ++k)
        orq_quantize_group_refined_f32(g, bits, y + k * g, iters, c + k * g, NULL, scales + k);
    orq_pack_codes(d, bits, c, words);
}

void orq_encode_rows_refined_f32(long n_rows, int d, int g, int bits, uint64_t seed,
                                 int iters, const uint16_t *x, const uint16_t *ref,
                                 uint32_t *words, uint16_t *scales)
{
    int8_t D[ORQ_MAX_D];
    orq_signs(seed, d, D);
    const int wpr = (d * bits + 31) / 32;
    for (long row = 0; row < n_rows; ++row)
        orq_encode_row_refined_f32(d, g, bits, D, iters, x + row * d, ref + row * d,
                                   words + row * wpr, scales + row * (d / g));
}

int orq_quantize_group_refined_f64(int g, int bits, const double *y, int iters,
                                   uint8_t *codes, double *s_out, double *err)
{
    const int nlev = 1 << bits;
    const int half = 1 << (bits - 1);
    double amax = 0.0;
    for (int i = 0; i < g; ++i)
        if (fabs(y[i]) > amax)
            amax = fabs(y[i]);
    double inv = (amax < (double)FLT_MIN) ? 0.0 : ((double)half - 0.5) / amax;
    double s = 0.0;
    int done = 0;
    for (int k = 0; k <= iters; ++k) {
        if (k > 0) {
            if (!(s >= (double)FLT_MIN))
                break;
            inv = 0.5 / s;
            ++done;
        }
        double num = 0.0, den = 0.0;
        for (int i = 0; i < g; ++i) {
            double fl = floor(y[i] * inv);
            if (fl < -half)
                fl = -half;
            if (fl > half - 1)
                fl = half - 1;
            const int c = (int)fl + half;
            codes[i] = (uint8_t)c;
            const int l = 2 * c - (nlev - 1);
            num += y[i] * l;
            den += (double)(l * l);
        }
        s = num / den;
        if (err) {
            double e = 0.0;
            for (int i = 0; i < g; ++i) {
                const double dv = y[i] - s * (2 * codes[i] - (nlev - 1));
                e += dv * dv;
            }
            err[k] = e;
        }
    }
    if (s_out)
        *s_out = s;
    return done;
}

/* ------------------------------------------------------------------------ */
/* compressed reference                                                      */
/* ------------------------------------------------------------------------ */

void orq_encode_rows_cr_f32(long n_rows, int d, int g, int ref_bits, int bits, uint64_t seed,
                            const uint16_t *ref, const uint16_t *x,
                            uint32_t *ref_words, uint16_t *ref_scales,
                            uint32_t *words, uint16_t *scales)
{
    int8_t D[ORQ_MAX_D];
    orq_signs(seed, d, D);
    const int rwpr = (d * ref_bits + 31) / 32;
    const int wpr = (d * bits + 31) / 32;
    const int rtop = (1 << ref_bits) - 1;
    for (long row = 0; row < n_rows; ++row) {
        float r[ORQ_MAX_D], y[ORQ_MAX_D], z[ORQ_MAX_D];
        uint8_t c[ORQ_MAX_D];
        for (int i = 0; i < d; ++i)
            r[i] = orq_bf16_to_f32(ref[row * d + i]);
        orq_rotate_f32(d, D, r, y);
        for (int k = 0; k < d / g; ++k) {
            uint16_t h;
            orq_quantize_group_refined_f32(g, ref_bits, y + k * g, 0, c + k * g, NULL, &h);
            if (ref_scales)
                ref_scales[row * (d / g) + k] = h;
            const float s = (float)orq_f16_to_f64(h);
            for (int i = 0; i < g; ++i)
                z[k * g + i] = s * (float)(2 * c[k * g + i] - rtop);
        }
        if (ref_words)
            orq_pack_codes(d, ref_bits, c, ref_words + row * rwpr);
        if (!x)
            continue;
        for (int i = 0; i < d; ++i)
            r[i] = orq_bf16_to_f32(x[row * d + i]);
        orq_rotate_f32(d, D, r, y);
        for (int i = 0; i < d; ++i)
            y[i] = y[i] - z[i];
        for (int k = 0; k < d / g; ++k)
            orq_quantize_group_refined_f32(g, bits, y + k * g, 0, c + k * g, NULL,
                                           scales + row * (d / g) + k);
        orq_pack_codes(d, bits, c, words + row * wpr);
    }
}

void orq_reconstruct_row_cr_f64(int d, int g, int ref_bits, int bits, const int8_t *D,
                                const uint32_t *ref_words, const uint16_t *ref_scales,
                                const uint32_t *words, const uint16_t *scales, double *out)
{
    uint8_t cr[ORQ_MAX_D], c[ORQ_MAX_D];
    double w[ORQ_MAX_D];
    double *R = (double *)malloc(sizeof(double) * (size_t)d * d);
    orq_rotation_matrix_f64(d, D, R);
    orq_unpack_codes(d, ref_bits, ref_words, cr);
    if (words)
        orq_unpack_codes(d, bits, words, c);
    const int rtop = (1 << ref_bits) - 1, top = (1 << bits) - 1;
    for (int i = 0; i < d; ++i) {
        const int k = i / g;
        w[i] = orq_f16_to_f64(ref_scales[k]) * (2 * cr[i] - rtop);
        if (words)
            w[i] += orq_f16_to_f64(scales[k]) * (2 * c[i] - top);
    }
    /* out = R^T w */
    for (int j = 0; j < d; ++j) {
        double acc = 0.0;
        for (int i = 0; i < d; ++i)
            acc += R[(size_t)i * d + j] * w[i];
        out[j] = acc;
    }
    free(R);
}

/* fp64 definitional encoder: y = R r with the explicit matrix, the same code
 * rule evaluated in double, and the least-squares scale in double. */
void orq_encode_row_f64(int d, int g, int bits, const int8_t *D,
                        const uint16_t *x, const uint16_t *ref,
                        uint8_t *codes, double *scales, double *bdist)
{
    const int nlev = 1 << bits;
    const int half = 1 << (bits - 1);
    double *R = (double *)malloc(sizeof(double) * (size_t)d * d);
    double r[ORQ_MAX_D], y[ORQ_MAX_D];
    orq_rotation_matrix_f64(d, D, R);
    for (int i = 0; i < d; ++i)
        r[i] = (double)orq_bf16_to_f32(x[i]) - (double)orq_bf16_to_f32(ref[i]);
    for (int i = 0; i < d; ++i) {
        double acc = 0.0;
        for (int j = 0; j < d; ++j)
            acc += R[(size_t)i * d + j] * r[j];
        y[i] = acc;
    }
    free(R);
    for (int k = 0; k < d / g; ++k) {
        const double *yg = y + k * g;
        double amax = 0.0;
        for (int i = 0; i < g; ++i)
            if (fabs(yg[i]) > amax)
                amax = fabs(yg[i]);
        double inv = (amax < (double)FLT_MIN) ? 0.0 : ((double)half - 0.5) / amax;
        double num = 0.0, den = 0.0;
        for (int i = 0; i < g; ++i) {
            double u = yg[i] * inv;
            double fl = floor(u);
            int c = (int)fl + half;
            if (c < 0)
                c = 0;
            if (c > nlev - 1)
                c = nlev - 1;
            codes[k * g + i] = (uint8_t)c;
            int lvl = 2 * c - (nlev - 1);
            num += yg[i] * lvl;
            den += (double)(lvl * lvl);
            if (bdist) {
                double dn = fabs(u - floor(u + 0.5));
                /* the outer clamp edges are not decision boundaries */
                bdist[k * g + i] = (inv == 0.0) ? INFINITY : dn;
            }
        }
        scales[k] = num / den;
    }
}

/* ------------------------------------------------------------------------ */
/* reconstruction and attention, fp64                                        */
/* ------------------------------------------------------------------------ */

/* K_hat = ref + Rot^T (s * l): the residual is decoded in the rotated
 * domain with the stored fp16 scale and rotated back with the transpose.
 * R is the explicit rotation matrix of orq_rotation_matrix_f64. */
static void reconstruct_with_matrix(int d, int g, int bits, const double *R,
                                    const uint16_t *ref, const uint32_t *words,
                                    const uint16_t *scales, double *out)
{
    for (int i = 0; i < d; ++i)
        out[i] = (double)orq_bf16_to_f32(ref[i]);
    if (bits == 16)
        return;
    const int nlev = 1 << bits;
    uint8_t c[ORQ_MAX_D];
    double yhat[ORQ_MAX_D];
    orq_unpack_codes(d, bits, words, c);
    for (int i = 0; i < d; ++i)
        yhat[i] = orq_f16_to_f64(scales[i / g]) * (double)(2 * c[i] - (nlev - 1));
    for (int j = 0; j < d; ++j) {
        double acc = 0.0;
        for (int i = 0; i < d; ++i)
            acc += R[(size_t)i * d + j] * yhat[i];     /* (R^T yhat)_j */
        out[j] += acc;
    }
}

void orq_reconstruct_row_f64(int d, int g, int bits, const int8_t *D,
                             const uint16_t *ref, const uint32_t *words,
                             const uint16_t *scales, double *out)
{
    double *R = (double *)malloc(sizeof(double) * (size_t)d * d);
    orq_rotation_matrix_f64(d, D, R);
    reconstruct_with_matrix(d, g, bits, R, ref, words, scales, out);
    free(R);
}

/* Max-subtracted softmax attention in double. */
void orq_attention_f64(int T, int d, int G, const double *q, const double *K,
                       const double *V, double scale, double *out)
{
    double *z = (double *)malloc(sizeof(double) * (size_t)(T > 0 ? T : 1));
    for (int r = 0; r < G; ++r) {
        double m = -INFINITY;
        for (int t = 0; t < T; ++t) {
            double acc = 0.0;
            for (int i = 0; i < d; ++i)
                acc += q[(size_t)r * d + i] * K[(size_t)t * d + i];
            z[t] = scale * acc;
            if (z[t] > m)
                m = z[t];
        }
        double sum = 0.0;
        for (int t = 0; t < T; ++t) {
            z[t] = exp(z[t] - m);
            sum += z[t];
        }
        for (int i = 0; i < d; ++i) {
            double acc = 0.0;
            for (int t = 0; t < T; ++t)
                acc += z[t] * V[(size_t)t * d + i];
            out[(size_t)r * d + i] = acc / sum;
        }
    }
    free(z);
}

/* Decode attention at one loop: every cached row of that loop is rebuilt
 * from the reference plus its residual, then attended exactly.  This is the
 * result the fused GPU kernel must reach (it may only reorder the sums). */
int orq_decode_attention_f64(int T, int d, int g, int G, int bits, uint64_t seed,
                             double scale, const uint16_t *q,
                             const uint16_t *ref_k, const uint16_t *ref_v,
                             const uint32_t *codes_k, const uint32_t *codes_v,
                             const uint16_t *scales_k, const uint16_t *scales_v,
                             double *out)
{
    if (T < 1 || d < 1 || d > ORQ_MAX_D || G < 1)
        return 1;
    if (bits != 16 && (g < 1 || d % g))
        return 1;
    int8_t D[ORQ_MAX_D];
    orq_signs(seed, d, D);
    if (scale <= 0.0)
        scale = 1.0 / sqrt((double)d);
    const int wpr = (bits == 16) ? 0 : (d * bits + 31) / 32;
    const int spr = (bits == 16) ? 0 : d / g;
    double *K = (double *)malloc(sizeof(double) * (size_t)T * d);
    double *V = (double *)malloc(sizeof(double) * (size_t)T * d);
    double *qd = (double *)malloc(sizeof(double) * (size_t)G * d);
    if (!K || !V || !qd) {
        free(K);
        free(V);
        free(qd);
        return 2;
    }
    double *R = (double *)malloc(sizeof(double) * (size_t)d * d);
    if (!R) {
        free(K);
        free(V);
        free(qd);
        return 2;
    }
    orq_rotation_matrix_f64(d, D, R);
    for (int t = 0; t < T; ++t) {
        reconstruct_with_matrix(d, g, bits, R, ref_k + (size_t)t * d,
                                bits == 16 ? NULL : codes_k + (size_t)t * wpr,
                                bits == 16 ? NULL : scales_k + (size_t)t * spr,
                                K + (size_t)t * d);
        reconstruct_with_matrix(d, g, bits, R, ref_v + (size_t)t * d,
                                bits == 16 ? NULL : codes_v + (size_t)t * wpr,
                                bits == 16 ? NULL : scales_v + (size_t)t * spr,
                                V + (size_t)t * d);
    }
    free(R);
    for (int i = 0; i < G * d; ++i)
        qd[i] = (double)orq_bf16_to_f32(q[i]);
    orq_attention_f64(T, d, G, qd, K, V, scale, out);
    free(K);
    free(V);
    free(qd);
    return 0;
}
