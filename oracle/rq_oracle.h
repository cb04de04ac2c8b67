/*
 * rq_oracle.h -- CPU oracle for the ResidualQuant hot path.
 *
 * TEST INFRASTRUCTURE ONLY.  This file and rq_oracle.c are the slow, plain,
 * obviously-correct restatement of the method that the CUDA library is
 * checked against.  Only the test-suite, the smoke check and the CPU-baseline
 * leg of the benchmark may load it.  It shares no code, header, table or
 * constant with the CUDA library under kv_cache_residual_rq_b200/csrc, and
 * the library never loads it.
 *
 * Method source: "ResidualQuant: KV Cache Quantization for Looped
 * Transformers with 2-Bit Residuals" (newx.sg page, Abstract and AI Summary):
 * the final loop's K/V is kept as a reference, every other loop is stored as
 * a low-bit residual against it, the residual is rotated, quantised per group
 * down to INT2 with a least-squares scale, and the bit width may differ per
 * loop.  Everything finer than that (the Walsh-Hadamard rotation, the code
 * grid, the rounding rule, the group size, the packing) is a reading of the
 * pages; each is stated below where the function that implements it is
 * declared.
 *
 * Two levels:
 *   - the fp32 exact-spec path (orq_*_f32): the encoder step by step, in
 *     the fp32 operation order the spec fixes.  Codes from this path are the
 *     bit-exact target for the GPU encoder.
 *   - the fp64 definitional path (orq_*_f64): the rotation as an explicit
 *     d x d matrix, reconstruction and softmax attention in double.  This is
 *     the reference for decode-attention outputs.
 *
 * Data formats (all little-endian, all arrays row-major):
 *   bf16  : uint16_t, the top half of an IEEE binary32
 *   fp16  : uint16_t, IEEE binary16
 *   codes : per row of d elements, ceil(d*bits/32) uint32 words; element j lives
 *           in word j / (32/bits) at bit offset bits * (j % (32/bits))
 *   scales: per row, d/g fp16 values, one per contiguous group of g rotated
 *           coordinates
 */
#ifndef RQ_ORACLE_H
#define RQ_ORACLE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define ORQ_MAX_D 4096

/* ---- scalar formats ---------------------------------------------------- */
float    orq_bf16_to_f32(uint16_t h);
double   orq_f16_to_f64(uint16_t h);
uint16_t orq_f64_to_f16(double x);          /* IEEE round-to-nearest-even */

/* ---- seeded sign vector (counter-based splitmix64) --------------------- */
uint64_t orq_splitmix64(uint64_t seed, uint64_t i);
void     orq_signs(uint64_t seed, int d, int8_t *D);

/* ---- rotation ----------------------------------------------------------- */
float orq_cd_f32(int d);                                 /* RN_f32(1/sqrt(d)) */
int   orq_hadamard_entry(int i, int j);                  /* Sylvester, +-1 */
void  orq_rotation_matrix_f64(int d, const int8_t *D, double *R);
void  orq_rotate_f32(int d, const int8_t *D, const float *r, float *y);
void  orq_fwht_f64(int d, double *v);                    /* in place, unnormalised */

/* ---- quantiser (fp32 exact-spec) ---------------------------------------- */
void orq_quantize_group_f32(int g, int bits, const float *y, uint8_t *codes,
                            double *s_exact, uint16_t *s_f16, int *ties);
void orq_pack_codes(int d, int bits, const uint8_t *codes, uint32_t *words);
void orq_unpack_codes(int d, int bits, const uint32_t *words, uint8_t *codes);

/* ---- encoder ------------------------------------------------------------ */
/* One row: r = x - ref, y = Rot r, per-group codes and scale. */
void orq_encode_row_f32(int d, int g, int bits, const int8_t *D,
                        const uint16_t *x, const uint16_t *ref,
                        uint32_t *words, uint16_t *scales, int *ties);

/* n_rows contiguous rows of d elements. Returns the total tie count. */
long orq_encode_rows_f32(long n_rows, int d, int g, int bits, uint64_t seed,
                         const uint16_t *x, const uint16_t *ref,
                         uint32_t *words, uint16_t *scales);

/* fp64 definitional encoder for one row.  Also returns, per element, the
 * distance of u from the nearest decision boundary (an integer) so that
 * disagreement with the fp32 path can be attributed to boundary proximity. */
void orq_encode_row_f64(int d, int g, int bits, const int8_t *D,
                        const uint16_t *x, const uint16_t *ref,
                        uint8_t *codes, double *scales, double *bdist);

/* ---- least-squares refinement (alternating code / scale refits) --------- */
/* Reading of the pages' "least-squares scaling" taken one step further, as
 * alternating refits: from the absmax codes and their least-squares scale
 * s_0, each refit k = 1..iters re-quantises every coordinate to the nearest
 * level of the current scale (inv = RN(0.5 / s), c = clamp(floor(RN(y inv))
 * + 2^(b-1), 0, 2^b - 1), ties to the upper level) and refits
 * s = <y,l>/<l,l>.  Refits stop early if s falls below FLT_MIN.  Because each
 * scale decides the next codes, the binary32 order of <y,l> is fixed: fused
 * multiply-add chains over runs of 16 consecutive coordinates (first to last,
 * from 0), the two runs of each 32-coordinate block added, then the blocks
 * added in order (a group shorter than 32 is a single chain).  Scales stay in
 * binary32 between refits; the stored scale is the last one, clamped to
 * +-65504 and rounded to fp16. */
float orq_ls_dot_f32(int g, const float *y, const int *lvl);
void orq_quantize_group_refined_f32(int g, int bits, const float *y, int iters,
                                    uint8_t *codes, float *s_out, uint16_t *s_f16);
void orq_encode_row_refined_f32(int d, int g, int bits, const int8_t *D, int iters,
                                const uint16_t *x, const uint16_t *ref,
                                uint32_t *words, uint16_t *scales);
void orq_encode_rows_refined_f32(long n_rows, int d, int g, int bits, uint64_t seed,
                                 int iters, const uint16_t *x, const uint16_t *ref,
                                 uint32_t *words, uint16_t *scales);
/* The same refits in double on given rotated coordinates y; err[k] receives
 * ||y - s_k l_k||^2 after refit k (err[0]: the absmax codes with s_0), so
 * err has iters + 1 entries.  Returns the number of refits done. */
int orq_quantize_group_refined_f64(int g, int bits, const double *y, int iters,
                                   uint8_t *codes, double *s_out, double *err);

/* ---- compressed reference (the reference loop itself as rotated codes) --- */
/* Reading of the pages' storage figure (80.7% less than BF16, beyond what a
 * BF16 reference allows): the final loop is stored as rotated low-bit codes
 * too, and every other loop as its residual against the RECONSTRUCTED
 * reference, taken in the rotated domain.  Per row, in binary32:
 *   y_ref = Rot f32(ref)            (the FWHT specification above)
 *   reference codes/scales          quantiser above with ref_bits (4 or 8),
 *                                   scale in the fixed <y,l> order
 *                                   (refinement section, zero refits)
 *   z_i   = f32(s16_ref) * l_ref,i  (exact: 11 x 9 significant bits)
 *   e_i   = RN(y_i - z_i),  y = Rot f32(x)  for a non-final loop x
 *   residual codes/scales           quantiser with bits (2 or 4), same
 *                                   scale order
 * so codes AND scales are reproducible bit for bit.  Reconstruction:
 *   K_L^ = Rot^T z,   K_l^ = Rot^T (z + s16_l l_l). */
void orq_encode_rows_cr_f32(long n_rows, int d, int g, int ref_bits, int bits, uint64_t seed,
                            const uint16_t *ref, const uint16_t *x,
                            uint32_t *ref_words, uint16_t *ref_scales,
                            uint32_t *words, uint16_t *scales);
/* out[d] in double; words/scales NULL reconstructs the reference loop. */
void orq_reconstruct_row_cr_f64(int d, int g, int ref_bits, int bits, const int8_t *D,
                                const uint32_t *ref_words, const uint16_t *ref_scales,
                                const uint32_t *words, const uint16_t *scales, double *out);

/* ---- reconstruction and attention (fp64 definitional) ------------------- */
/* out[d] = f64(ref) + Rot^T (s16 * level), for one row. bits==16 => ref. */
void orq_reconstruct_row_f64(int d, int g, int bits, const int8_t *D,
                             const uint16_t *ref, const uint32_t *words,
                             const uint16_t *scales, double *out);

/* Softmax attention of G query rows over T keys/values, all in double:
 * out[r] = sum_t softmax_t(scale * <q_r, K_t>) V_t. */
void orq_attention_f64(int T, int d, int G, const double *q, const double *K,
                       const double *V, double scale, double *out);

/* Decode attention at one loop for one (batch, kv-head): reconstruct every
 * cached K/V row of that loop, then exact attention.  q is bf16 [G][d];
 * ref_k/ref_v bf16 [T][d]; codes [T][d*bits/32]; scales fp16 [T][d/g].
 * bits == 16 means the loop is the reference (codes/scales unused).
 * scale <= 0 selects 1/sqrt(d).  out is [G][d] double.  Returns 0 on success. */
int orq_decode_attention_f64(int T, int d, int g, int G, int bits, uint64_t seed,
                             double scale, const uint16_t *q,
                             const uint16_t *ref_k, const uint16_t *ref_v,
                             const uint32_t *codes_k, const uint32_t *codes_v,
                             const uint16_t *scales_k, const uint16_t *scales_v,
                             double *out);

#ifdef __cplusplus
}
#endif
#endif
