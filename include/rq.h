/*
 * rq.h -- C ABI of librq.so, the B200 (sm_100a) hot path of ResidualQuant.
 *
 * Method: "ResidualQuant: KV Cache Quantization for Looped Transformers with
 * 2-Bit Residuals" (newx.sg page, Abstract).  A looped Transformer writes one
 * K/V per loop.  The final loop's K/V is kept in BF16 as the reference; every
 * other loop is stored as its residual against the reference, rotated,
 * quantised per group to INT2 (or INT4 for loops given more bits) with a
 * least-squares fp16 scale.  Decode attention reads the reference plus the
 * codes and rebuilds the loop's K/V on the fly.
 *
 * Conventions for every entry point:
 *   - Data pointers are DEVICE pointers unless a parameter says "host".
 *     The caller allocates and owns every buffer, including the workspace;
 *     the library allocates nothing and never synchronises the stream.
 *   - `stream` is a cudaStream_t passed as void*; NULL means the legacy
 *     default stream.  Work is enqueued in order on that stream and the call
 *     returns before it runs.
 *   - Arguments are validated before anything is enqueued.  A call that
 *     returns an error has enqueued nothing and written nothing.
 *   - Device pointers must be 16-byte aligned (RQ_ERR_ALIGNMENT otherwise).
 *   - Buffers must be at least the size the matching rq_*_bytes() query
 *     returns; those sizes are rounded up to 16 bytes and the kernels may
 *     read (never write) the padding.
 *   - No C++ exception, abort or CUDA error escapes: launch failures come
 *     back as RQ_ERR_CUDA.
 *   - bf16 / fp16 values are passed as uint16_t bit patterns.
 *
 * Layouts (row-major, T = ctx_cap (ctx when 0), d = head_dim, g = group,
 * b = bits):
 *   K/V of one loop, reference : bf16 [rows][kv_heads][T][d]
 *   query                      : bf16 [batch][q_heads][d]
 *   codes of one loop          : uint32 [rows][kv_heads][T][d*b/32];
 *                                element j of a row is in word j/(32/b) at
 *                                bit offset b*(j mod 32/b), LSB first;
 *                                code c stands for level 2c - (2^b - 1)
 *   scales of one loop         : fp16 [rows][kv_heads][T][d/g], one per
 *                                contiguous group of g rotated coordinates
 *   output                     : fp32 [batch][q_heads][d]
 * Query head j attends with kv head j / (q_heads / kv_heads).
 *
 * Rotation: Rot = (1/sqrt(d)) * H_d * D, H_d the Sylvester Hadamard matrix,
 * D = diag(+-1) with D_i = -1 iff bit 63 of splitmix64 output i of `seed`
 * is set (output i = mix(seed + (i+1) * 0x9E3779B97F4A7C15)).  The same seed
 * must be given to rq_encode and rq_decode_attention.
 */
#ifndef RQ_H
#define RQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    RQ_OK = 0,
    RQ_ERR_INVALID_ARG = 1,   /* null pointer, non-positive size, bad shape */
    RQ_ERR_UNSUPPORTED = 2,   /* head_dim, group, bits or GQA ratio not built */
    RQ_ERR_ALIGNMENT = 3,     /* a device pointer is not 16-byte aligned */
    RQ_ERR_WORKSPACE = 4,     /* workspace missing or smaller than required */
    RQ_ERR_CUDA = 5           /* a CUDA launch or query failed */
} rq_status;

#define RQ_MAX_LOOPS 16       /* non-final loops one rq_encode call takes */

typedef struct {
    int32_t batch;      /* leading rows: B for decode; any flattened count
                           (e.g. layers * B) for encode */
    int32_t kv_heads;   /* Hkv >= 1 */
    int32_t q_heads;    /* Hq, a multiple of Hkv (decode only; encode ignores) */
    int32_t ctx;        /* T: tokens per (row, kv head) the call covers */
    int32_t head_dim;   /* d: 64 or 128 */
    int32_t group;      /* g: 32 or 64, divides d */
    int32_t ctx_cap;    /* token capacity (pitch) of the K/V, codes and scales
                           arrays per (row, kv head); 0 means ctx.  A cache
                           allocated for ctx_cap tokens holds its first ctx
                           tokens valid, so it can grow in place. */
} rq_shape;

/* Library version as major*10000 + minor*100 + patch. */
int rq_version(void);

/* Static text for a status code; never NULL. */
const char *rq_status_string(rq_status s);

/* Bytes of the codes of ONE loop at `bits` (2, 4, or 8 for a compressed
 * reference) for `shape`:
 * batch*kv_heads*T*head_dim*bits/8 rounded up to 16, T = ctx_cap (ctx when
 * 0).  0 for bits == 16 or an invalid shape.  Host-only arithmetic. */
size_t rq_codes_bytes(const rq_shape *shape, int bits);

/* Bytes of the fp16 scales of ONE loop: batch*kv_heads*T*(head_dim/group)*2
 * rounded up to 16, T = ctx_cap (ctx when 0).  0 for bits == 16 or an
 * invalid shape. */
size_t rq_scales_bytes(const rq_shape *shape, int bits);

/* Workspace bytes rq_decode_attention needs for `shape` (partial softmax
 * states of the context splits, one arrival counter per (batch, kv head) and
 * a status word).  0 for an invalid shape.  Host-only arithmetic. */
size_t rq_decode_workspace_bytes(const rq_shape *shape);

/*
 * rq_encode -- ResidualQuant encoder (Abstract: the non-final loops are
 * stored as residuals against the final-loop reference, rotated, and
 * quantised per group with a least-squares scale; the bit width is chosen
 * per loop).
 *
 * For every row (r, h, t) and every loop l < n_loops with bits[l] != 16:
 *   e   = f32(kv_loops[l][r,h,t,:]) - f32(ref[r,h,t,:])       (binary32, RN)
 *   y   = RN(c_d * FWHT(D e)), butterfly stages h = 1, 2, ..., d/2, each
 *         (a, b) -> (a + b, a - b) in binary32 RN, c_d = RN(1/sqrt(d))
 *   per group of g coordinates: amax = max |y_i|;
 *         inv = (2^(b-1) - 1/2) / amax (binary32 RN), or 0 if amax < 2^-126;
 *         c_i = clamp(floor(RN(y_i * inv)) + 2^(b-1), 0, 2^b - 1);
 *         l_i = 2 c_i - (2^b - 1);
 *         s = <y, l> / <l, l>, clamped to +-65504, stored as fp16 RN.
 * Codes are bit-identical to that sequence; the scale's dot product is
 * summed in an unspecified order (at most one fp16 ulp from the exact value).
 *
 *   shape          : batch = number of leading rows, kv_heads, ctx, head_dim,
 *                    group used; q_heads ignored.  ctx == 0 is a no-op.
 *   kv_loops       : HOST array of n_loops device pointers, bf16 K (or V) of
 *                    each non-final loop, layout [rows][Hkv][T][d].
 *   n_loops        : 1 .. RQ_MAX_LOOPS.
 *   ref            : device bf16, the final loop, same layout.  Read only.
 *   bits_per_loop  : HOST array of n_loops values, each 2, 4 or 16.
 *                    16 marks a loop kept in BF16 by the caller: nothing is
 *                    written for it and its pointers may be NULL.
 *   seed           : rotation seed.
 *   codes_out      : HOST array of n_loops device pointers, each
 *                    rq_codes_bytes(shape, bits_per_loop[l]) bytes.
 *   scales_out     : HOST array of n_loops device pointers (fp16 bits), each
 *                    rq_scales_bytes(shape, bits_per_loop[l]) bytes.
 * The host arrays are read before the call returns.  Outputs must not
 * overlap inputs.
 */
rq_status rq_encode(const rq_shape *shape, const uint16_t *const *kv_loops, int n_loops,
                    const uint16_t *ref, const uint8_t *bits_per_loop, uint64_t seed,
                    uint32_t *const *codes_out, uint16_t *const *scales_out, void *stream);

/*
 * rq_encode_at -- rq_encode from a token window into a cache position (the
 * encode-on-arrival step of a decode loop: a token's non-final loops can be
 * encoded only once its final loop exists; until then they stay in BF16 in a
 * window, the same constraint the LoopVQ page describes for its serving
 * integration).
 *
 * Same arithmetic as rq_encode.  For every (row r, kv head h) and token
 * t < shape->ctx it reads source token src_offset + t of arrays whose token
 * pitch is src_pitch, and writes destination token dst_offset + t of arrays
 * whose token pitch is dst_pitch:
 *   kv_loops[l], ref   : bf16 [rows][Hkv][src_pitch][d]
 *   codes_out[l]       : [rows][Hkv][dst_pitch][d*b/32]
 *   scales_out[l]      : [rows][Hkv][dst_pitch][d/g]
 *   ref_out (optional) : bf16 [rows][Hkv][dst_pitch][d]; when not NULL the
 *                        final-loop rows are copied there too, so a window
 *                        slot can be retired into the cache in one call.
 * shape->ctx_cap is ignored.  Requires src_offset + ctx <= src_pitch and
 * dst_offset + ctx <= dst_pitch.  Destination tokens outside the written
 * range are not touched.
 */
rq_status rq_encode_at(const rq_shape *shape, int src_pitch, int src_offset, int dst_pitch,
                       int dst_offset, const uint16_t *const *kv_loops, int n_loops,
                       const uint16_t *ref, const uint8_t *bits_per_loop, uint64_t seed,
                       uint32_t *const *codes_out, uint16_t *const *scales_out,
                       uint16_t *ref_out, void *stream);

/*
 * rq_encode_cr_at -- encode into the compressed-reference format: the final
 * loop itself is stored as rotated low-bit codes, and every other loop as its
 * residual against the reconstructed reference, in the rotated domain (the
 * reading of the pages' storage figure under which a decode step reads fewer
 * bytes than BF16: ResidualQuant page, Abstract).  Per row, in binary32:
 *   y_ref = Rot ref;  reference codes/scales: the group quantiser with
 *           ref_bits, its least-squares sum in the fixed order of
 *           rq_encode_at_ex;  z = f32(s16_ref) * l_ref (exact);
 *   e     = RN(Rot x - z) for each non-final loop x, quantised with its bits.
 * Codes and scales are bit-exact.  Reconstruction: K_L = Rot^T z and
 * K_l = Rot^T (z + s16_l l_l); rq_reconstruct_cr and
 * rq_decode_attention_cr read this format.
 *
 *   shape          : rows [batch][Hkv][ctx][d] of contiguous sources;
 *                    ctx_cap ignored.
 *   dst_pitch/offset: token pitch of the outputs and first token written
 *                    (as rq_encode_at), so a step's new token can be retired
 *                    into a cache position.
 *   kv_loops, n_loops (0 .. RQ_MAX_LOOPS), bits_per_loop (2, 4 or 16),
 *   codes_out, scales_out: as rq_encode_at; HOST arrays (may be NULL when
 *                    n_loops is 0).
 *   ref            : device bf16 final loop, contiguous.
 *   ref_bits       : 4 or 8.
 *   ref_codes_out  : rq_codes_bytes(dst shape, ref_bits) bytes.
 *   ref_scales_out : rq_scales_bytes(dst shape, ref_bits) bytes.
 * Errors: as rq_encode_at; RQ_ERR_UNSUPPORTED for other ref_bits.
 */
rq_status rq_encode_cr_at(const rq_shape *shape, int dst_pitch, int dst_offset,
                          const uint16_t *const *kv_loops, int n_loops, const uint16_t *ref,
                          int ref_bits, const uint8_t *bits_per_loop, uint64_t seed,
                          uint32_t *ref_codes_out, uint16_t *ref_scales_out,
                          uint32_t *const *codes_out, uint16_t *const *scales_out,
                          void *stream);

/* Most least-squares refits rq_encode_at_ex accepts. */
#define RQ_MAX_REFINE 8

/*
 * rq_encode_at_ex -- rq_encode_at with least-squares refinement (the pages'
 * least-squares scaling, iterated: ResidualQuant page, Abstract).
 *
 * refine_iters (0 .. RQ_MAX_REFINE): after the absmax codes and their
 * least-squares scale s, each refit re-quantises every coordinate of the
 * group to the nearest level of the current scale (step 2s: inv = RN(0.5/s),
 * c = clamp(floor(RN(y inv)) + 2^(b-1), 0, 2^b - 1), ties to the upper
 * level) and refits s = <y,l>/<l,l>; a group whose scale is below FLT_MIN
 * keeps its codes.  <y,l> is summed in a fixed binary32 order (fma chains
 * over runs of 16 coordinates, the runs of each 32-block added, then the
 * blocks), so codes and scales are reproducible bit for bit.  The error
 * ||y - s l|| never increases from one refit to the next.  The stored
 * format is unchanged: every decoder reads the refined codes as any others.
 * refine_iters = 0 is rq_encode_at.  Other arguments and errors as
 * rq_encode_at; a refine_iters outside 0 .. RQ_MAX_REFINE is
 * RQ_ERR_INVALID_ARG.
 */
rq_status rq_encode_at_ex(const rq_shape *shape, int src_pitch, int src_offset,
                          int dst_pitch, int dst_offset, const uint16_t *const *kv_loops,
                          int n_loops, const uint16_t *ref, const uint8_t *bits_per_loop,
                          uint64_t seed, int refine_iters, uint32_t *const *codes_out,
                          uint16_t *const *scales_out, uint16_t *ref_out, void *stream);

/*
 * rq_encode_paged -- rq_encode_at_ex into paged pools (the layout read by
 * rq_decode_attention_paged): token t of sequence b, head h of the sources
 * is written at position pos = dst_pos[b] + t of that sequence, i.e. row
 * (page_table[b][pos / 64] * Hkv + h) * 64 + pos % 64 of every pool.
 *   kv_loops, ref : contiguous device bf16 [batch][Hkv][ctx][d] (the tokens
 *                   to retire, e.g. one per sequence per decode step).
 *   dst_pos       : DEVICE int32 [batch], first position written per sequence.
 *   page_table    : DEVICE int32 [batch][max_pages]; pools of n_pages pages.
 *   codes_out, scales_out : HOST arrays of device pool pointers, sized by
 *                   rq_codes_bytes / rq_scales_bytes of a shape with batch =
 *                   n_pages and ctx = 64.
 *   ref_out       : optional bf16 reference pool [n_pages][Hkv][64][d].
 * A position past the table or a page id outside the pool writes nothing.
 * Arithmetic, refits and errors as rq_encode_at_ex.
 */
rq_status rq_encode_paged(const rq_shape *shape, const uint16_t *const *kv_loops, int n_loops,
                          const uint16_t *ref, const uint8_t *bits_per_loop, uint64_t seed,
                          int refine_iters, const int32_t *dst_pos, const int32_t *page_table,
                          int max_pages, int n_pages, uint32_t *const *codes_out,
                          uint16_t *const *scales_out, uint16_t *ref_out, void *stream);

/*
 * rq_decode_attention -- fused ResidualQuant decode attention for one loop
 * (Abstract: the reconstruction stays efficient; the reduced KV traffic is
 * what speeds decode up).
 *
 * For each batch b and query head j (kv head h = j / G, G = Hq / Hkv), with
 * K_hat_t = ref_k[b,h,t] + Rot^T (s^K_t * l^K_t) and likewise V_hat:
 *   out[b,j,:] = sum_t softmax_t(sigma * <q[b,j], K_hat_t>) V_hat_t
 * computed without materialising K_hat or V_hat: the query is rotated once
 * (q~ = Rot q), scores are <q, ref_k_t> + sum_groups s_t,g <q~_g, l_t,g>, the
 * V residual is accumulated in the rotated domain and rotated back once per
 * output row.  The context is split across CTAs (split-K) and the partial
 * softmax states are merged in the same launch.
 *
 *   shape          : batch, kv_heads, q_heads (multiple of kv_heads, ratio
 *                    1..8), ctx >= 1, head_dim 64|128, group 32|64.
 *   q              : device bf16 [batch][q_heads][d].
 *   ref_k, ref_v   : device bf16 [batch][Hkv][T][d], the final loop.
 *   codes_k/v      : device, this loop's codes (rq_codes_bytes); ignored and
 *                    may be NULL when bits == 16.
 *   scales_k/v     : device fp16 bits, this loop's scales (rq_scales_bytes);
 *                    ignored and may be NULL when bits == 16.
 *   bits           : 2 or 4 for a residual loop; 16 for the reference loop
 *                    itself (plain attention over ref_k/ref_v).
 *   seed           : the seed the codes were encoded with.
 *   softmax_scale  : sigma; <= 0 selects 1/sqrt(head_dim).
 *   out            : device fp32 [batch][q_heads][d].
 *   workspace      : device, >= rq_decode_workspace_bytes(shape) bytes,
 *                    ZERO-FILLED before its first use.  Every successful call
 *                    leaves it ready for the next; calls sharing a workspace
 *                    must be ordered on one stream.
 * The split of the context depends only on (batch, kv_heads, ctx), never on
 * bits, so a residual loop whose scales are all zero gives bit-for-bit the
 * output of the reference loop.
 */
rq_status rq_decode_attention(const rq_shape *shape, const uint16_t *q,
                              const uint16_t *ref_k, const uint16_t *ref_v,
                              const uint32_t *codes_k, const uint32_t *codes_v,
                              const uint16_t *scales_k, const uint16_t *scales_v,
                              int bits, uint64_t seed, float softmax_scale, float *out,
                              void *workspace, size_t workspace_bytes, void *stream);

/*
 * rq_decode_attention_tail -- rq_decode_attention over the shape->ctx cached
 * tokens plus n_tail BF16 tokens of the same loop that are not encoded yet
 * (the current token and any others still in the window):
 *   out[b,j,:] = softmax over { K_hat_t, t < ctx } U { tail_k[b,h,i], i < n_tail }
 * applied to the matching V rows.  The tail is folded into the merge that
 * finishes each head, in the same launch.
 *   tail_k, tail_v : device bf16 [batch][Hkv][tail_pitch][d], tokens
 *                    0..n_tail-1 used; may be NULL when n_tail == 0.
 *   n_tail         : 0 .. 256 (RQ_MAX_TAIL); tail_pitch >= n_tail.
 * Everything else as rq_decode_attention (which is this call with n_tail 0).
 */
#define RQ_MAX_TAIL 256

rq_status rq_decode_attention_tail(const rq_shape *shape, const uint16_t *q,
                                   const uint16_t *ref_k, const uint16_t *ref_v,
                                   const uint32_t *codes_k, const uint32_t *codes_v,
                                   const uint16_t *scales_k, const uint16_t *scales_v,
                                   int bits, uint64_t seed, float softmax_scale,
                                   const uint16_t *tail_k, const uint16_t *tail_v, int n_tail,
                                   int tail_pitch, float *out, void *workspace,
                                   size_t workspace_bytes, void *stream);

/* Most sequences of one variable-length call. */
#define RQ_MAX_VARLEN_BATCH 1024

/*
 * rq_decode_attention_varlen -- rq_decode_attention_tail for a batch whose
 * sequences hold different numbers of cached tokens (continuous batching;
 * the lengths live on the device, so one captured graph serves every step).
 *
 *   ctx_lens : DEVICE int32 [shape->batch], 4-byte aligned; sequence b
 *              attends over its first ctx_lens[b] cached tokens (plus the
 *              n_tail tail tokens).  Read by the kernel, so it may be written
 *              by the preceding kernel of the stream.  A length outside
 *              0 .. capacity is clamped and sets status bit 16; a sequence
 *              with 0 cached tokens attends over its tail only (with no tail
 *              its output is 0/0, NaN).
 *   shape    : capacity per head = shape->ctx_cap (or shape->ctx when
 *              ctx_cap is 0): the token pitch of ref_k/ref_v/codes/scales.
 *              batch <= RQ_MAX_VARLEN_BATCH.
 *   workspace: rq_decode_workspace_bytes_varlen(shape) bytes, zeroed once.
 * The work is split evenly over the tokens actually present (computed on the
 * device), not over the capacity.  Other arguments as rq_decode_attention_tail.
 * Errors: RQ_ERR_INVALID_ARG for a null ctx_lens or batch above the limit,
 * RQ_ERR_ALIGNMENT for a misaligned ctx_lens, else as the tail variant.
 */
rq_status rq_decode_attention_varlen(const rq_shape *shape, const int32_t *ctx_lens,
                                     const uint16_t *q, const uint16_t *ref_k,
                                     const uint16_t *ref_v, const uint32_t *codes_k,
                                     const uint32_t *codes_v, const uint16_t *scales_k,
                                     const uint16_t *scales_v, int bits, uint64_t seed,
                                     float softmax_scale, const uint16_t *tail_k,
                                     const uint16_t *tail_v, int n_tail, int tail_pitch,
                                     float *out, void *workspace, size_t workspace_bytes,
                                     void *stream);

/*
 * rq_decode_attention_cr -- decode attention of one loop over a cache in the
 * compressed-reference format (rq_encode_cr_at): scores and values are formed
 * from the reference codes plus (bits 2 or 4) the loop's residual codes, all
 * in the rotated domain -- s = sigma <q~, s_ref l_ref + s l>, one Rot^T per
 * output row -- so no BF16 row is read; bits == 16 decodes the final loop
 * from the reference codes alone (codes/scales may then be NULL).
 * Query rows per kv head G = q_heads / kv_heads in {1, 2, 4, 8}.
 *   ctx_lens  : NULL (every sequence has shape->ctx tokens; workspace of
 *               rq_decode_workspace_bytes) or a device int32 [batch] as in
 *               rq_decode_attention_varlen (workspace of
 *               rq_decode_workspace_bytes_varlen).
 *   ref_codes_k/v, ref_scales_k/v, ref_bits (4 or 8): the reference's
 *               codes and fp16 scales, [batch][Hkv][T_cap][...].
 * Tail tokens (BF16 K/V of the current token) and every other argument as
 * rq_decode_attention_tail.  The value weights p s are fp16 after a
 * warp-wide power of two that follows the largest scale of each tile, so
 * every finite fp16 scale is in range; a call whose reference or residual
 * value scales are not finite sets workspace status bit 64 and its output is
 * not valid.
 */
rq_status rq_decode_attention_cr(const rq_shape *shape, const int32_t *ctx_lens,
                                 const uint16_t *q, const uint32_t *ref_codes_k,
                                 const uint32_t *ref_codes_v, const uint16_t *ref_scales_k,
                                 const uint16_t *ref_scales_v, int ref_bits,
                                 const uint32_t *codes_k, const uint32_t *codes_v,
                                 const uint16_t *scales_k, const uint16_t *scales_v, int bits,
                                 uint64_t seed, float softmax_scale, const uint16_t *tail_k,
                                 const uint16_t *tail_v, int n_tail, int tail_pitch, float *out,
                                 void *workspace, size_t workspace_bytes, void *stream);

/*
 * rq_decode_attention_paged -- rq_decode_attention_varlen over paged caches:
 * the cache is a pool of pages of 64 tokens (one decode tile), and each
 * sequence's tokens live in the pages its row of a page table names.
 *   page_table : DEVICE int32 [batch][max_pages], 4-byte aligned: tokens
 *                64 j .. 64 j + 63 of sequence b are page page_table[b][j].
 *                Entries past a sequence's length are not read.  An entry
 *                outside 0 .. n_pages-1 is treated as an empty page and sets
 *                status bit 32 (the pool is never addressed out of range).
 *   ref_k, ref_v : pools bf16 [n_pages][Hkv][64][d];
 *   codes_k/v, scales_k/v : pools [n_pages][Hkv][64][d*b/32] and [...][d/g]
 *                (rq_codes_bytes / rq_scales_bytes of a shape with batch =
 *                n_pages, ctx = 64).
 *   shape      : ctx must equal max_pages * 64 (the capacity per sequence;
 *                ctx_cap 0 or equal); workspace of
 *                rq_decode_workspace_bytes_varlen(shape).
 *   ctx_lens   : as rq_decode_attention_varlen (required).
 * Everything else as rq_decode_attention_varlen; BF16 reference only.
 */
rq_status rq_decode_attention_paged(const rq_shape *shape, const int32_t *ctx_lens,
                                    const int32_t *page_table, int max_pages, int n_pages,
                                    const uint16_t *q, const uint16_t *ref_k,
                                    const uint16_t *ref_v, const uint32_t *codes_k,
                                    const uint32_t *codes_v, const uint16_t *scales_k,
                                    const uint16_t *scales_v, int bits, uint64_t seed,
                                    float softmax_scale, const uint16_t *tail_k,
                                    const uint16_t *tail_v, int n_tail, int tail_pitch, float *out,
                                    void *workspace, size_t workspace_bytes, void *stream);

/* Workspace bytes for rq_decode_attention_varlen with this shape (any
 * lengths up to the capacity); 0 if the shape is unsupported. */
size_t rq_decode_workspace_bytes_varlen(const rq_shape *shape);

/*
 * rq_decode_attention_noalloc -- rq_decode_attention without a workspace
 * argument, for callers that cannot allocate device memory (for example code
 * hosted by an application that owns every allocation, or a path that must
 * not call cudaMalloc because it may synchronise the device).  The paper has
 * no counterpart: this is a property of the library, not of the method.
 *
 * Same arguments, layouts, results and validation as rq_decode_attention,
 * minus `workspace` and `workspace_bytes`.  The scratch is a fixed array of
 * RQ_NOALLOC_SCRATCH_BYTES in the library's own device memory; every GPU on
 * which this entry point is used keeps that much until the process exits.
 *   - Allocates nothing: no cudaMalloc, no cudaFree, no allocating library
 *     routine.  It clears the scratch's status word and arrival counters
 *     (cudaMemsetAsync on `stream`) before each launch.
 *   - A shape needing more than RQ_NOALLOC_SCRATCH_BYTES
 *     (rq_decode_workspace_bytes(shape) > RQ_NOALLOC_SCRATCH_BYTES) is
 *     rejected with RQ_ERR_WORKSPACE before anything is enqueued.
 *   - The first call on a device looks up the array's device address (once
 *     per device, with that device current); make that first call before any
 *     stream capture.
 *   - Every call shares the one array per device and it keeps the last
 *     call's contents: calls whose executions overlap on the GPU (other
 *     streams, other host threads on the same device) race and give wrong
 *     results; order them on one stream.
 *   - There is no status readback for this scratch.
 */
#define RQ_NOALLOC_SCRATCH_BYTES (8u << 20)

rq_status rq_decode_attention_noalloc(const rq_shape *shape, const uint16_t *q,
                                      const uint16_t *ref_k, const uint16_t *ref_v,
                                      const uint32_t *codes_k, const uint32_t *codes_v,
                                      const uint16_t *scales_k, const uint16_t *scales_v,
                                      int bits, uint64_t seed, float softmax_scale, float *out,
                                      void *stream);

/*
 * rq_reconstruct -- the format's decoder: rebuilds one loop's K (or V) rows
 * (Abstract: a non-final loop is the final-loop reference plus its rotated,
 * least-squares-scaled low-bit residual) for consumers that want the loop's
 * values themselves rather than the fused attention:
 *   out[r,h,t,:] = f32(ref[r,h,t,:]) + Rot^T (s_g * l)      (bits 2 or 4)
 *   out[r,h,t,:] = f32(ref[r,h,t,:])                        (bits 16)
 * computed in fp32 (the inverse rotation summed in butterfly order), written
 * as fp32, or as bf16 rounded to nearest when out_bf16 != 0.
 *   shape  : batch, kv_heads, ctx (tokens rebuilt per row and head), head_dim,
 *            group, ctx_cap (token pitch of ref, codes, scales and out).
 *   out    : device [rows][Hkv][T][d], T = ctx_cap (ctx when 0); tokens
 *            beyond ctx are not written.
 * ref and codes must come from the same rq_encode seed.
 */
rq_status rq_reconstruct(const rq_shape *shape, const uint16_t *ref, const uint32_t *codes,
                         const uint16_t *scales, int bits, uint64_t seed, void *out,
                         int out_bf16, void *stream);

/* rq_reconstruct_cr -- rq_reconstruct for the compressed-reference format
 * (rq_encode_cr_at): out = Rot^T (s_ref l_ref + s l), or Rot^T (s_ref l_ref)
 * for bits == 16 (the reference loop; codes/scales may then be NULL).
 * ref_codes/ref_scales as written by rq_encode_cr_at with ref_bits (4 or 8);
 * layout, capacity and errors as rq_reconstruct. */
rq_status rq_reconstruct_cr(const rq_shape *shape, const uint32_t *ref_codes,
                            const uint16_t *ref_scales, int ref_bits, const uint32_t *codes,
                            const uint16_t *scales, int bits, uint64_t seed, void *out,
                            int out_bf16, void *stream);

/* Reads and clears the encoders' sticky status word of the current device
 * (blocking; waits for all work on the device).  0 means every rq_encode /
 * rq_encode_at since the last read ran clean; non-zero means a bounded wait
 * inside the encoder ran out (bit 0: the copy engine's slot was never
 * released, bit 1: a copy never completed, bit 2: a consumer's tile never
 * arrived) and the codes written since then are invalid.  Bit 3 (value 8)
 * exists only in the bounds-checked build of this library (librq_bounds.so,
 * compiled with RQ_BOUNDS_CHECK): an encoder or reconstruction kernel found
 * an index outside its buffer and skipped that access.  The reconstruction
 * entry points report here too. */
rq_status rq_encode_take_status(uint32_t *host_status);

/* Copies the workspace's device status word to *host_status (blocking read
 * on `stream`).  0 means every decode call since the workspace was zeroed
 * ran clean; non-zero means a call's output is invalid and the workspace must
 * be zeroed again: bits 1, 2, 8 a bounded wait inside a kernel ran out, 4 a
 * partial-record slot out of range, 16 a sequence length clamped to the
 * capacity, 32 a page id outside the pool, 64 a compressed-reference value
 * weight not finite; 128, only in the bounds-checked build (librq_bounds.so), an
 * index a decode kernel computed fell outside its buffer or shared-memory
 * area and that access was skipped.  This is the only entry point that
 * synchronises. */
rq_status rq_workspace_status(const void *workspace, size_t workspace_bytes,
                              uint32_t *host_status, void *stream);

#ifdef __cplusplus
}
#endif
#endif /* RQ_H */
