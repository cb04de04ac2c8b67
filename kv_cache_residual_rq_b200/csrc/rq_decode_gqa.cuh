// rq_decode_gqa.cuh -- ResidualQuant decode attention for grouped queries
// (G = q_heads / kv_heads in {2, 4, 8}) on the sm_100a tensor cores.
//
// Method: "ResidualQuant: KV Cache Quantization for Looped Transformers with
// 2-Bit Residuals", Abstract -- decode rebuilds each non-final loop's K/V
// from the BF16 final-loop reference plus the loop's rotated low-bit residual.
//
// With G query rows per kv head every K/V tile is shared by G rows, so the
// four products of the fused attention are small dense contractions and go to
// the tensor cores (mma.sync m16n8k16, fp32 accumulation), per warp and per
// 16 tokens of a 64-token tile:
//   S_ref = Q  K^T              (K from shared memory, ldmatrix)
//   S_res = Q~ C_K^T            per scale group, then x s^K
//   O_ref^T += V^T P^T          (V via ldmatrix.trans)
//   O_res^T += C_V^T (P s^V)^T
// with fp32 accumulation.  S_ref and O_ref are bf16 x bf16.  S_res, INT2
// residual with 64-dim groups: integer MMAs (m16n8k32) of the rows' q~ as
// 16-bit fixed point (signed bytes h | l as A rows g | g + 8) against the
// codes one per byte (a shift and a mask per four), exact integer level sums
// per group until x s^K sig.  S_res otherwise: one f16 MMA per k-step, q~
// scaled by a power of two 2^E per row (max |q~| 2^E in [2^13, 2^14)) and
// rounded to f16 (11 significant bits), against the K codes as the exact f16
// subnormals c 2^-24 (a shift and a mask per two codes, no offset); per scale
// group q~ . l = 2^25 acc - (2^b - 1) sum q~, times s^K 2^-E.  O_res: the V
// codes c are exact bf16 values, and P s^V, not
// a bf16 value, is split into a bf16 high part and a bf16 remainder and
// multiplied twice (~16 significant bits, bf16's range); sum_t p s (2c -
// (2^b-1)) = 2 (C_V^T (P s)^T) - (2^b - 1) sum_t p s is completed when the
// warp flushes.  Rows beyond G are zero and their weights are forced to zero.
//
// Compressed INT8 / INT4 reference (same page, the reference loop itself
// stored as rotated codes): the reference term is one more quantised term in
// the rotated domain, s_ref <q~, l_ref> for the scores and sum_t p s_ref l_ref
// for the values, l_ref = 2c - (2^b - 1).  Scores: integer MMAs (m16n8k32,
// s8 x u8) per 32-dim slice, the rows' q~ as 16-bit fixed point Q = q~ / sig
// split into signed bytes h (rows g) and l (rows g + 8) against the codes one
// per byte (INT8 rows as ldmatrix reads them, INT4 nibbles by one mask or a
// shift and a mask per four); per scale group sig (2 <Q, c> - (2^b - 1) sum
// Q) is exact in integers until the scale.  Values: the codes enter f16 MMAs
// as the exact subnormals c 2^-24 (one byte permute per two INT8 codes, one
// shift and one mask per two INT4 codes) against the weights p s_ref split
// into f16 parts after a lazily updated power of two keeps them in f16's
// range; the 2^24 returns when the warp flushes.  The reference rows (d or
// d/2 bytes) arrive swizzled; the k order of the q~ fragments and the m-row
// order of the value accumulators follow the codes' positions in the 32-bit
// ldmatrix words.
//
// The reference K/V tiles (BF16 rows, or code rows) arrive by TMA
// tensor copies with the swizzle of their line width (conflict-free
// ldmatrix); codes and scales by plain bulk copies, as in the single-query
// kernel.  The work split, the partial records and the
// last-arriving-CTA merge with the single inverse rotation are shared with it
// (rq_decode_common.cuh).  Every mbarrier wait is bounded.
#pragma once

#include "rq_decode_tc.cuh"

namespace rq {

// Launch of the grouped-query kernel for one head size and reference type;
// each is instantiated in a translation unit of its own
// (rq_decode_gqa_d<head_dim>_r<ref bits>.cu) so the builds run in parallel.
cudaError_t launch_gqa_d128_r0(int G, int bits, const TcParams& gp, cudaStream_t stream);
cudaError_t launch_gqa_d128_r4(int G, int bits, const TcParams& gp, cudaStream_t stream);
cudaError_t launch_gqa_d128_r8(int G, int bits, const TcParams& gp, cudaStream_t stream);
cudaError_t launch_gqa_d64_r0(int G, int bits, const TcParams& gp, cudaStream_t stream);
cudaError_t launch_gqa_d64_r4(int G, int bits, const TcParams& gp, cudaStream_t stream);
cudaError_t launch_gqa_d64_r8(int G, int bits, const TcParams& gp, cudaStream_t stream);

#ifdef RQ_GQA_KERNEL_DEFINITIONS
namespace {

template <int D, int G, int BITS, int GROUP, int RB>
struct GCfg {
  static constexpr int TILE = kDecodeTile;                 // 64 tokens
  static constexpr int WTOK = TILE / kConsumerWarps;       // 16 tokens per warp
  static constexpr bool RES = (BITS != 16);
  // INT2 residual: ldmatrix reads the code rows directly.  With 64-dim scale
  // groups a 16-byte row chunk is exactly one group; with 32-dim groups it
  // holds two, and lanes exchange words (one shuffle) so that every k-step
  // and every m-tile stays inside one group.
  static constexpr bool LDM2 = (BITS == 2);
  // INT4 residual: a 16-byte row chunk (32 dims) always lies inside one scale
  // group; ldmatrix words of eight codes, no exchange needed
  static constexpr bool LDM4 = (BITS == 4);
  // INT2 residual with 64-dim groups (a 16-byte chunk of a code row is one
  // group): scores as integer MMAs, the q~ rows as 16-bit fixed point
  static constexpr bool RIM = (BITS == 2 && GROUP == 64);
  static constexpr int NCH = D / 64;                        // 64-dim chunks per row
  static constexpr bool CR = (RB == 8);                    // INT8 compressed reference
  static constexpr bool CR4 = (RB == 4);                   // INT4 compressed reference
  static constexpr bool CRX = (RB != 0);                   // either
  // INT8 compressed reference with an INT2 residual: the residual's value
  // products go into the reference's f16 accumulators (one set of value
  // accumulators; the other combinations keep their own)
  static constexpr bool VSH = (RB == 8 && BITS == 2);
  static constexpr int RROW = CRX ? D * RB / 8 : 0;        // reference code bytes per token
  // f16 operands of the reference codes: the exact subnormals c 2^-24 (the
  // code in the low mantissa bits, no offset).  A sum acc over those operands
  // gives the level sum  sum w (2c - (2^RB - 1)) = 2^25 acc - (2^RB - 1) sum w.
  static constexpr float CSCALE = 33554432.0f;                        // 2^25
  static constexpr float LOFF = (float)((1 << RB) - 1);
  static constexpr int NBOX = D / 64;                      // 64-column boxes per row
  static constexpr int BOX_BYTES = 64 * 128;               // 64 rows x 128 B
  // one K or V reference tile: BF16 boxes, or the INT8 code rows (D bytes each)
  static constexpr int REF_TILE_BYTES = CRX ? TILE * RROW : NBOX * BOX_BYTES;
  static constexpr int KT = D / 16;                        // k-steps of 16 dims
  static constexpr int CROW = RES ? D * BITS / 8 : 0;      // code bytes per token
  static constexpr int CWORDS = CROW / 4;
  static constexpr int SC_BYTES = RES ? TILE * (2 * D / 32) + 32 : 0;
  static constexpr int RSC_BYTES = CRX ? TILE * (2 * D / 32) + 32 : 0;  // reference scales
  static constexpr int OFF_K = 0;
  static constexpr int OFF_V = OFF_K + REF_TILE_BYTES;
  static constexpr int OFF_CK = OFF_V + REF_TILE_BYTES;
  static constexpr int OFF_CV = OFF_CK + TILE * CROW;
  static constexpr int OFF_SK = OFF_CV + TILE * CROW;
  static constexpr int OFF_SV = OFF_SK + SC_BYTES;
  static constexpr int OFF_RSK = OFF_SV + SC_BYTES;
  static constexpr int OFF_RSV = OFF_RSK + RSC_BYTES;
  static constexpr int STAGE_BYTES = (OFF_RSV + RSC_BYTES + 1023) / 1024 * 1024;
  static constexpr int STAGES = 2;

  static constexpr int RING_BYTES = STAGES * STAGE_BYTES;
  static constexpr int MERGE_FLOATS = kConsumerWarps * G * (2 + 2 * D);
  static constexpr int QBUF_FLOATS = 2 * G * D;
  static constexpr int NG = D / GROUP;                      // scale groups per token
  static constexpr int NV = D / 32;                        // 32-dim slices
  static constexpr int SPG = GROUP / 32;                   // slices per scale group
  static constexpr int KSG = GROUP / 16;                   // k-steps per scale group
  static constexpr int SB = 2 * NG;                        // scale bytes per token
  // per warp, row and scale group: sum of p s^V (and of p s_ref^V)
  static constexpr int WSUM_FLOATS = kConsumerWarps * G * NG * (CRX ? 2 : 1);
  // q, q~ high, q~ remainder (bf16); with a compressed reference also
  // q~ 2^E high, remainder (f16, k-permuted for the reference's codes)
  // qfrag regions (32-bit words): kind 0 at QF0 (the bf16 query; BF16
  // reference only), kinds 1 and 2 at QF1, QF1 + KT * 64 (the residual's f16
  // fragments), or at QF1 the residual's integer-MMA fragments (RIM), and the
  // compressed reference's integer-MMA fragments at QFC
  static constexpr int QF0 = 0;
  static constexpr int QF1 = CRX ? 0 : KT * 64;
  static constexpr int QF12_WORDS = RIM ? NCH * 256 : (RES ? 2 * KT * 64 : 0);
  static constexpr int QFC = QF1 + QF12_WORDS;
  static constexpr int QFRAG_WORDS = QFC + (CRX ? NV * 32 * 4 : 0);
  // residual: per (row, scale group) the sum of the q~ fragments' values (f16
  // form) or of Q (integer form), for the levels' 2^b - 1 offset; compressed
  // reference: the same sums of its Q; per row the residual's scale (2^-E or
  // sig) and the compressed reference's sig; even count to keep the barriers
  // 8-byte aligned
  static constexpr int SQ_FLOATS =
      (G * NG * (CRX ? 2 : 1) + ((CRX || RES) ? G : 0) + (CRX ? G : 0) + 1) / 2 * 2;
  static constexpr int SMEM_BYTES = 1024 /* base alignment slack */ + RING_BYTES +
                                    4 * (MERGE_FLOATS + QBUF_FLOATS + WSUM_FLOATS +
                                         QFRAG_WORDS + SQ_FLOATS) +
                                    2 * STAGES * 8 + 16 + STAGES * 8;   // + stage rows
  // resident CTAs per SM: two (168 registers); with one set of value
  // accumulators (VSH, or a compressed reference alone) three (128
  // registers) where their shared memory fits (228 KB per SM, 1 KB of it
  // reserved per CTA)
  static constexpr bool FITS3 = SMEM_BYTES <= 228 * 1024 / 3 - 1024;
  static constexpr int CTAS = ((VSH || (CRX && !RES)) && FITS3) ? 3 : 2;
  static_assert(G == 2 || G == 4 || G == 8, "grouped queries");
  static_assert(MERGE_FLOATS >= kVarlenMaxBatch + 1, "merge area holds the length scan");
  static_assert(GROUP == 32 || GROUP == 64, "scale group");
  static_assert(D == 64 || D == 128, "head_dim");
  static_assert(RB == 0 || RB == 4 || RB == 8, "reference: BF16 rows, INT4 or INT8 codes");
  // the swizzle pattern repeats every 8 lines: 1024 B for 128-byte lines
  static_assert(OFF_V % (CRX ? 8 * RROW : 1024) == 0, "swizzled tiles start on the period");
};


template <int D, int G, int BITS, int GROUP, int RB>
__global__ void __launch_bounds__(kDecodeThreads, GCfg<D, G, BITS, GROUP, RB>::CTAS)
decode_gqa_kernel(const __grid_constant__ TcParams gp) {
  using C = GCfg<D, G, BITS, GROUP, RB>;
  const DecodeParams& p = gp.p;
  constexpr int STAGES = C::STAGES, TILE = C::TILE, KT = C::KT;
  constexpr unsigned FULL = 0xffffffffu;
  constexpr int TOPLVL = C::RES ? (1 << BITS) - 1 : 0;
  constexpr int NG = C::NG, KSG = C::KSG, SB = C::SB;

  extern __shared__ unsigned char smem_raw[];
  // the swizzled boxes need 1024-byte alignment
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  unsigned char* ring = smem;
  float* merge = reinterpret_cast<float*>(smem + C::RING_BYTES);
  float* qbuf = merge + C::MERGE_FLOATS;
  float* wsum_s = qbuf + C::QBUF_FLOATS;
  uint32_t* qfrag = reinterpret_cast<uint32_t*>(wsum_s + C::WSUM_FLOATS);  // [3][KT][32][2]
  float* sq_s = reinterpret_cast<float*>(qfrag + C::QFRAG_WORDS);           // [G][NG]
  float* sqh_s = sq_s + G * NG;              // CR: [G][NG] sums of Q per scale group
  // [G] the residual's per-row scale: 2^-E of the f16 q~ fragments, or sig
  // of the integer form's Q
  float* rsig_s = sq_s + G * NG * (C::CRX ? 2 : 1);
  float* rsigc_s = rsig_s + G;               // CR: [G] sig of each row's Q
  float* wsumR_s = wsum_s + kConsumerWarps * G * NG;   // CR: sums of p s_ref^V
  uint64_t* full_bar = reinterpret_cast<uint64_t*>(sq_s + C::SQ_FLOATS);
  uint64_t* empty_bar = full_bar + STAGES;
  volatile int* flags = reinterpret_cast<volatile int*>(empty_bar + STAGES);
  volatile unsigned long long* stage_row = reinterpret_cast<volatile unsigned long long*>(
      reinterpret_cast<unsigned char*>(empty_bar + STAGES) + 16);    // [STAGES], paged

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int cta = blockIdx.x;
  pdl_allow_next();
  if (cta >= p.ctas) return;

  if (tid == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], kConsumerWarps);
    }
    flags[0] = 0;
    flags[1] = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (warp == kConsumerWarps && lane == 0) prefetch_first_tiles<C, D>(p, cta);
  pdl_wait_prev();     // inputs and workspace may come from the previous kernel

  // this CTA's run of tiles (the merge area is free scratch until the first head)
  CallSplit split;
  long long tile_begin, tile_end;
  TileCursor first_cur;
  if (!plan_cta(p, cta, reinterpret_cast<int*>(merge), split, tile_begin, tile_end, first_cur))
    return;
  const int n_my = (int)(tile_end - tile_begin);
  // scale bytes a stage holds (per array), for the bounds-checked build
  constexpr int SCAP = C::RES ? C::SC_BYTES : (C::CRX ? C::RSC_BYTES : 0);
  // ========================= producer warp ================================
  if (warp == kConsumerWarps) {
    if (lane == 0)
      tile_producer<C>(gp, ring, full_bar, empty_bar, flags, stage_row, first_cur, n_my, SCAP);
    return;
  }

  // ========================= consumer warps ===============================
  const int g = lane >> 2;            // fragment row group
  const int q = lane & 3;             // fragment column pair
  const int wtok = warp * C::WTOK;    // this warp's first token in a tile
  const bool row_ok = g < G;          // lanes whose S/P row is a real query row
  const float score_scale = p.score_scale;

  // The per-head Q A-fragments live in shared memory (qfrag): for k-step kk
  // and lane, {a0, a2} of the bf16 query (kind 0) and, with a residual, of
  // the rotated query as f16 q~ 2^E (kind 1; kind 2 is unused): rows g, dims
  // in the k order of the residual's code words; rows g >= G are zero, and
  // a1 = a3 = 0 (rows g + 8).  With a compressed reference, the region after
  // kind 2 holds per 32-dim slice and lane the four s8 A words {a0, a1, a2,
  // a3} of the reference's integer MMAs (rows g: bytes h of Q, rows g + 8:
  // bytes l, in the k order of the reference's code words).
  // softmax state of row g (lanes with row_ok), and the output accumulators
  // (O^T fragments: dims 16mt + g (+8), rows 2q, 2q + 1)
  float m_run = kNegInf, l_run = 0.0f;
  float wsum[NG], wsumR[NG];
  float vscale = 1.0f;     // INT8 reference: power of two applied to the V weights
  float oref[KT][4], ores[KT][4];

  auto reset_state = [&]() {
    m_run = kNegInf;
    l_run = 0.0f;
    vscale = 1.0f;
#pragma unroll
    for (int j = 0; j < NG; ++j) {
      wsum[j] = 0.0f;
      wsumR[j] = 0.0f;
    }
#pragma unroll
    for (int mt = 0; mt < KT; ++mt)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        oref[mt][e] = 0.0f;
        ores[mt][e] = 0.0f;
      }
  };

  auto setup_head = [&](long long hd) {
    float* qs = qbuf;
    float* qt = qbuf + G * D;
    load_rotate_queries<D, G>(p, hd, qs, qt, tid);
    const float cd = rot_scale<D>();
    if constexpr (C::CRX) {
      if (warp == 0) {
        // row g of q~ as 16-bit fixed point Q = q~ / sig (sig = max |q~| /
        // 32639, so Q = 256 h + l with signed bytes h, l), as the A fragments
        // of the compressed reference's integer MMAs: per 32-dim slice j,
        // rows g carry the h bytes and rows g + 8 the l bytes; the k
        // positions 4q + b and 16 + 4q + b carry the dims of the codes the
        // ldmatrix words hold there (INT8: 32j + 4q + b, + 16; INT4: nibbles
        // 0 and 1 of byte 4q + b of chunk j, dims 32j + 8q + 2b, + 1)
        float mx = 0.0f;
        if (row_ok)
          for (int d = q; d < D; d += 4) mx = fmaxf(mx, fabsf(cd * qt[g * D + d]));
        mx = fmaxf(mx, __shfl_xor_sync(FULL, mx, 1));
        mx = fmaxf(mx, __shfl_xor_sync(FULL, mx, 2));
        const float sig = mx > 0.0f ? mx * (1.0f / 32639.0f) : 1.0f;
        const float inv = 1.0f / sig;
        if (row_ok && q == 0) rsigc_s[g] = sig;
        int sq = 0;          // sum of Q over the lane's dims of the current scale group
#pragma unroll 1
        for (int j = 0; j < C::NV; ++j) {
          uint32_t a[4] = {0u, 0u, 0u, 0u};
          if (row_ok) {
#pragma unroll
            for (int h2 = 0; h2 < 2; ++h2)
#pragma unroll
              for (int b = 0; b < 4; ++b) {
                const int dim = C::CR ? 32 * j + 16 * h2 + 4 * q + b : 32 * j + 8 * q + 2 * b + h2;
                const int Q = min(max(__float2int_rn(cd * qt[g * D + dim] * inv), -32639), 32639);
                const int lo = ((Q + 128) & 255) - 128;
                const int hi = (Q - lo) >> 8;
                a[2 * h2] |= (uint32_t)(hi & 0xFF) << (8 * b);
                a[2 * h2 + 1] |= (uint32_t)(lo & 0xFF) << (8 * b);
                sq += Q;
              }
          }
          *reinterpret_cast<uint4*>(qfrag + C::QFC + (j * 32 + lane) * 4) =
              make_uint4(a[0], a[1], a[2], a[3]);
          if ((j + 1) % C::SPG == 0) {                // end of a scale group
            sq += __shfl_xor_sync(FULL, sq, 1);
            sq += __shfl_xor_sync(FULL, sq, 2);
            if (row_ok && q == 0) sqh_s[g * NG + j / C::SPG] = (float)sq;
            sq = 0;
          }
        }
      }
    }
    float upR = 1.0f;        // 2^E of the residual's f16 q~ fragments (row g)
    if constexpr (C::RIM) {
      if (warp == (C::CRX ? 1 : kConsumerWarps - 1)) {   // beside warp 0's fragments
        // row g of q~ as 16-bit fixed point Q = q~ / sig, as the s8 A
        // fragments of the residual's integer MMAs: per 64-dim chunk c and
        // code pair pp, rows g carry the h bytes and rows g + 8 the l bytes;
        // k positions 4q + b | 16 + 4q + b carry dims 64c + 16q + 2pp + 4b | +1
        // (codes 2pp + 4b | 2pp + 1 + 4b of the word holding dims 16q .. 16q+15)
        float mx = 0.0f;
        if (row_ok)
          for (int d = q; d < D; d += 4) mx = fmaxf(mx, fabsf(cd * qt[g * D + d]));
        mx = fmaxf(mx, __shfl_xor_sync(FULL, mx, 1));
        mx = fmaxf(mx, __shfl_xor_sync(FULL, mx, 2));
        const float sig = mx > 0.0f ? mx * (1.0f / 32639.0f) : 1.0f;
        const float inv = 1.0f / sig;
        if (row_ok && q == 0) rsig_s[g] = sig;
#pragma unroll 1
        for (int c = 0; c < C::NCH; ++c) {
          int sq = 0;
#pragma unroll
          for (int pp = 0; pp < 2; ++pp) {
            uint32_t a[4] = {0u, 0u, 0u, 0u};
            if (row_ok) {
#pragma unroll
              for (int h2 = 0; h2 < 2; ++h2)
#pragma unroll
                for (int b = 0; b < 4; ++b) {
                  const int dim = 64 * c + 16 * q + 2 * pp + h2 + 4 * b;
                  const int Q =
                      min(max(__float2int_rn(cd * qt[g * D + dim] * inv), -32639), 32639);
                  const int lo = ((Q + 128) & 255) - 128;
                  const int hi = (Q - lo) >> 8;
                  a[2 * h2] |= (uint32_t)(hi & 0xFF) << (8 * b);
                  a[2 * h2 + 1] |= (uint32_t)(lo & 0xFF) << (8 * b);
                  sq += Q;
                }
            }
            *reinterpret_cast<uint4*>(qfrag + C::QF1 + ((2 * c + pp) * 32 + lane) * 4) =
                make_uint4(a[0], a[1], a[2], a[3]);
          }
          sq += __shfl_xor_sync(FULL, sq, 1);
          sq += __shfl_xor_sync(FULL, sq, 2);
          if (row_ok && q == 0) sq_s[g * NG + c] = (float)sq;     // chunk c = scale group c
        }
      }
    } else if constexpr (C::RES) {
      if (warp == 0) {
        float mx = 0.0f;
        if (row_ok)
          for (int d = q; d < D; d += 4) mx = fmaxf(mx, fabsf(cd * qt[g * D + d]));
        mx = fmaxf(mx, __shfl_xor_sync(FULL, mx, 1));
        mx = fmaxf(mx, __shfl_xor_sync(FULL, mx, 2));
        const int ex = (int)((__float_as_uint(mx) >> 23) & 0xFFu) - 127;
        const int E = min(13 - ex, 126);
        upR = __uint_as_float((uint32_t)(127 + E) << 23);
        if (row_ok && q == 0) rsig_s[g] = __uint_as_float((uint32_t)(127 - E) << 23);
      }
    }
    if (warp == 0) {
      float sqj = 0.0f;      // running sum of the current scale group (INT2)
#pragma unroll 1
      for (int kk = 0; kk < KT; ++kk) {
        // (kind 0 only for a BF16 reference, kinds 1 and 2 only for the f16
        // residual form; the others' regions hold other fragments or none)
        uint32_t* fa = qfrag + C::QF0 + (kk * 32 + lane) * 2;
        uint32_t* fh = qfrag + C::QF1 + (kk * 32 + lane) * 2;
        uint32_t* fl = qfrag + C::QF1 + KT * 64 + (kk * 32 + lane) * 2;
        if (row_ok) {
          const float* qrow = qs + g * D + 16 * kk + 2 * q;
          // INT2 with ldmatrix words: k-step kk = 4c + t of chunk c carries
          // dims 64c + 16q + 2t + {0, 8 | 1, 9} (codes 2t, 2t+8 | 2t+1, 2t+9
          // of the word holding the chunk's dims 16q .. 16q+15)
          // (32-dim groups: k-step kk is half t = kk & 1 of group (kk >> 1) & 1 of
          // chunk kk >> 2; lane q reads the word of dims 16 (q & 1) .. of that
          // group and takes its codes 2u, 2u+8 | 2u+1, 2u+9, u = 2t + (q >> 1))
          const int lo2 = GROUP == 64 ? 16 * q + 2 * (kk & 3)
                                      : 32 * ((kk >> 1) & 1) + 16 * (q & 1) +
                                            2 * (2 * (kk & 1) + (q >> 1));
          const float* trow = qt + g * D + (C::LDM2 ? 64 * (kk >> 2) + lo2 : 16 * kk + 2 * q);
          if constexpr (!C::CRX) {
            fa[0] = pack_bf16(qrow[0], qrow[1]);     // exact: q is bf16
            fa[1] = pack_bf16(qrow[8], qrow[9]);
          }
          if constexpr (C::RIM || !C::RES) {
            // (the residual's fragments are the integer MMAs' above)
          } else if constexpr (BITS == 2) {
            // k positions 2q, 2q+1 | 2q+8, 2q+9 carry dims 2q, 2q+8 | 2q+1, 2q+9,
            // so the two codes of a B register sit 16 bits apart
            fh[0] = pack_f16(cd * trow[0] * upR, cd * trow[8] * upR);
            fh[1] = pack_f16(cd * trow[1] * upR, cd * trow[9] * upR);
            fl[0] = fl[1] = 0u;
            sqj += (f16_lo_f(fh[0]) + f16_hi_f(fh[0])) + (f16_lo_f(fh[1]) + f16_hi_f(fh[1]));
          } else if constexpr (C::LDM4) {
            // k-step kk = half h of 32-dim chunk kk >> 1: k positions 2q, 2q+1 |
            // 2q+8, 2q+9 carry dims 8q + 2h + {0, 4 | 1, 5} (the word's codes
            // 2h, 2h+4 | 2h+1, 2h+5, each register's two codes 16 bits apart)
            const float* t4 = qt + g * D + 32 * (kk >> 1) + 8 * q + 2 * (kk & 1);
            fh[0] = pack_f16(cd * t4[0] * upR, cd * t4[4] * upR);
            fh[1] = pack_f16(cd * t4[1] * upR, cd * t4[5] * upR);
            fl[0] = fl[1] = 0u;
            sqj += (f16_lo_f(fh[0]) + f16_hi_f(fh[0])) + (f16_lo_f(fh[1]) + f16_hi_f(fh[1]));
          }
        } else {
          if constexpr (!C::CRX) fa[0] = fa[1] = 0u;
          if constexpr (C::RES && !C::RIM) fh[0] = fh[1] = fl[0] = fl[1] = 0u;
        }
        if ((BITS == 2 || C::LDM4) && !C::RIM && (kk + 1) % KSG == 0) {   // end of a scale group
          sqj += __shfl_xor_sync(FULL, sqj, 1);
          sqj += __shfl_xor_sync(FULL, sqj, 2);
          if (row_ok && q == 0) sq_s[g * NG + kk / KSG] = sqj;
          sqj = 0.0f;
        }
      }
    }
    named_bar_sync(1, kConsumerThreads);
  };

  auto flush_head = [&](long long hd, long long first_tile, int nt_h) {
    // l and the V weight sums of row g over the four lanes of its row group
    l_run += __shfl_xor_sync(FULL, l_run, 1);
    l_run += __shfl_xor_sync(FULL, l_run, 2);
#pragma unroll
    for (int j = 0; j < NG; ++j) {
      wsum[j] += __shfl_xor_sync(FULL, wsum[j], 1);
      wsum[j] += __shfl_xor_sync(FULL, wsum[j], 2);
      if constexpr (C::CRX) {
        wsumR[j] += __shfl_xor_sync(FULL, wsumR[j], 1);
        wsumR[j] += __shfl_xor_sync(FULL, wsumR[j], 2);
      }
    }
    named_bar_sync(1, kConsumerThreads);          // merge area free
    float* mw = merge + warp * G * (2 + 2 * D);
    if constexpr (C::CRX) {
      // non-finite reference weights (invalid scales): the output is not valid
      bool bad = false;
#pragma unroll
      for (int j = 0; j < NG; ++j) bad |= !isfinite(wsumR[j]);
      if (row_ok && q == 0 && bad) flag_error(p.status, 64u);
    }
    if (row_ok && q == 0) {
      mw[g * (2 + 2 * D)] = m_run;
      mw[g * (2 + 2 * D) + 1] = l_run;
#pragma unroll
      for (int j = 0; j < NG; ++j) {
        if constexpr (C::RES) wsum_s[(warp * G + g) * NG + j] = wsum[j] * (C::VSH ? 1.0f / vscale : 1.0f);
        if constexpr (C::CRX) wsumR_s[(warp * G + g) * NG + j] = wsumR[j] * (1.0f / vscale);
      }
    }
    // O^T fragments: c0 (dim 16mt+g, row 2q), c1 (.., row 2q+1), c2/c3 dim +8;
    // the INT8 reference's m-rows g, g + 8 are dims 16mt + 2g, 16mt + 2g + 1,
    // the INT4 reference's 32 (mt / 2) + 4g + 2 (mt & 1) (+ 1)
#pragma unroll
    for (int mt = 0; mt < KT; ++mt) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int r = 2 * q + (e & 1);
        const int dim = 16 * mt + g + 8 * (e >> 1);
        const int dim_res =
            C::LDM4       ? 32 * (mt >> 1) + 4 * g + 2 * (mt & 1) + (e >> 1)
            : !C::LDM2    ? dim
            : GROUP == 64 ? 64 * (mt >> 2) + 8 * g + 2 * (mt & 3) + (e >> 1)
                          : 64 * (mt >> 2) + 32 * ((mt >> 1) & 1) + 8 * (g & 3) + 4 * (mt & 1) +
                                2 * (g >> 2) + (e >> 1);
        const int dim_ref = C::CR    ? 16 * mt + 2 * g + (e >> 1)
                            : C::CR4 ? 32 * (mt >> 1) + 4 * g + 2 * (mt & 1) + (e >> 1)
                                     : dim;
        if (r < G) {
          // (INT4 reference: m-rows g + 8 hold 16 x their codes' products)
          if constexpr (C::CRX)
            mw[r * (2 + 2 * D) + 2 + dim_ref] =
                oref[mt][e] * (C::CSCALE / vscale) * ((C::CR4 && (e >> 1)) ? 0.0625f : 1.0f);
          else mw[r * (2 + 2 * D) + 2 + dim_ref] = oref[mt][e];
          if constexpr (C::RES && !C::VSH) mw[r * (2 + 2 * D) + 2 + D + dim_res] = 2.0f * ores[mt][e];
          else mw[r * (2 + 2 * D) + 2 + D + dim] = 0.0f;
        }
      }
    }
    named_bar_sync(1, kConsumerThreads);
    if constexpr (C::RES || C::CRX) {
      // complete sum_t p s (2c - top) = 2 sum p s c - top sum p s; the
      // compressed reference's sum_t p s_ref (2c - (2^RB - 1)) = CSCALE acc -
      // LOFF sum p s_ref (acc over the f16 code operands, written as
      // CSCALE acc), moved to the rotated part
      for (int e = tid; e < kConsumerWarps * G * D; e += kConsumerThreads) {
        const int w = e / (G * D), r = (e / D) % G, dim = e % D;
        float* rec = merge + (w * G + r) * (2 + 2 * D);
        const int wi = (w * G + r) * NG + dim / GROUP;
        float z = rec[2 + D + dim];
        if constexpr (C::RES) z -= (float)TOPLVL * wsum_s[wi];
        if constexpr (C::CRX) {
          z += rec[2 + dim] - C::LOFF * wsumR_s[wi];
          rec[2 + dim] = 0.0f;
        }
        rec[2 + D + dim] = z;
      }
      named_bar_sync(1, kConsumerThreads);
    }
    // compressed references: four records per merge batch (more registers for the token loop)
    finish_head<D, G, C::RES || C::CRX, C::CRX ? 4 : kMergeFew>(p, hd, first_tile, nt_h, split,
                                                                 cta, merge, qbuf, flags, tid);
  };

  // ---- one tile ----
  auto tile_mma = [&](const unsigned char* st, int n, int sc_off) {
    if (!C::CRX && n < TILE) {
      // rows past the head's last token (spare capacity, the next head, or
      // nothing ever written) are not part of the context: their weights are
      // 0, and zeroing this warp's such V rows keeps a non-finite value there
      // out of the products
      unsigned char* vrows = const_cast<unsigned char*>(st) + C::OFF_V;
      for (int e = lane; e < C::WTOK * C::NBOX * 8; e += 32) {
        const int tok = wtok + e / (C::NBOX * 8), c = e % (C::NBOX * 8);
        if (tok >= n)
          *reinterpret_cast<uint4*>(vrows + (c >> 3) * C::BOX_BYTES + tok * 128 + (c & 7) * 16) =
              make_uint4(0u, 0u, 0u, 0u);
      }
      __syncwarp();
    }
    const uint32_t sK = smem_u32(st + C::OFF_K);
    const uint32_t sV = smem_u32(st + C::OFF_V);
    // ldmatrix row order: the row addressed by lane r (of a matrix's eight)
    // is token (r >> 1) + 4 (r & 1) of its 8-token half, so n / k positions
    // 2q, 2q + 1 carry tokens q, q + 4 (the four lanes of a row group then
    // read four consecutive rows of the plainly loaded code rows)
    const int pr7 = ((lane & 7) >> 1) | ((lane & 1) << 2);
    // ---- scores for the warp's two 8-token tiles, k-steps outermost ----
    // c[nt]: S_ref (then + s x S_res) fragments, row g, tokens q, q + 4 of nt
    float cref[2][4] = {{0.0f, 0.0f, 0.0f, 0.0f}, {0.0f, 0.0f, 0.0f, 0.0f}};
    // BF16 reference: the odd k-steps' products in a second accumulator (two
    // chains of KT / 2 MMAs instead of one of KT), added before the softmax
    float cref2[2][4] = {{0.0f, 0.0f, 0.0f, 0.0f}, {0.0f, 0.0f, 0.0f, 0.0f}};
    float ct[2][4] = {{0.0f, 0.0f, 0.0f, 0.0f}, {0.0f, 0.0f, 0.0f, 0.0f}};
    const int tok0[2] = {wtok + q, wtok + 8 + q};     // tokens of c0 per tile (c1: + 4)
    // ldmatrix: matrices (tile 0, dims +0..7), (tile 0, +8..15), (tile 1, ..), (tile 1, ..)
    const int ktr = wtok + ((lane >> 4) & 1) * 8 + pr7;
    const int kch = (lane >> 3) & 1;
    if constexpr (C::CRX) {
      // ---- compressed reference: S_ref = Q C_ref^T per 32-dim slice j as
      // integer MMAs: A = the rows' Q bytes (rows g: h, rows g + 8: l; kind
      // 3 of qfrag), B = the codes of the n-tile's 8 tokens (ldmatrix words,
      // one code per byte: INT8 as stored, INT4 nibble 0 | nibble 1) ----
      int ci[2][4] = {{0, 0, 0, 0}, {0, 0, 0, 0}};
      uint32_t b8[4];      // (nt 0, chunk), (nt 1, chunk), (nt 0, chunk + 1), (nt 1, chunk + 1)
      const int m = lane >> 3;
#pragma unroll
      for (int j = 0; j < C::NV; ++j) {
        if constexpr (C::CR) {
          ldsm_x4(sK + swz_offset<C::RROW>(wtok + (m & 1) * 8 + pr7, 2 * j + (m >> 1)), b8);
        } else if ((j & 1) == 0) {
          ldsm_x4(sK + swz_offset<C::RROW>(wtok + (m & 1) * 8 + pr7, j + (m >> 1)), b8);
        }
        const uint4 af = *reinterpret_cast<const uint4*>(qfrag + C::QFC + (j * 32 + lane) * 4);
        const uint32_t a[4] = {af.x, af.y, af.z, af.w};
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
          uint32_t b0, b1;
          if constexpr (C::CR) {
            b0 = b8[nt];
            b1 = b8[2 + nt];
          } else {
            const uint32_t w = b8[2 * (j & 1) + nt];
            b0 = w & 0x0F0F0F0Fu;
            b1 = (w >> 4) & 0x0F0F0F0Fu;
          }
          mma_s8u8(ci[nt], a, b0, b1);
        }
        if ((j + 1) % C::SPG == 0) {
          // end of scale group jg: S += s_ref[t, jg] sig (2 <Q, c> - (2^RB - 1) sum Q)
          const int jg = j / C::SPG;
          const float sg = row_ok ? rsigc_s[g] : 0.0f;
          const int off = row_ok ? (int)((1 << RB) - 1) * __float2int_rn(sqh_s[g * NG + jg]) : 0;
#pragma unroll
          for (int nt = 0; nt < 2; ++nt) {
            const float r0 = half_at(st + C::OFF_RSK + sc_off + tok0[nt] * SB + 2 * jg);
            const float r1 = half_at(st + C::OFF_RSK + sc_off + (tok0[nt] + 4) * SB + 2 * jg);
            const int x0 = 512 * ci[nt][0] + 2 * ci[nt][2] - off;
            const int x1 = 512 * ci[nt][1] + 2 * ci[nt][3] - off;
            cref[nt][0] = fmaf(r0 * sg, (float)x0, cref[nt][0]);
            cref[nt][1] = fmaf(r1 * sg, (float)x1, cref[nt][1]);
#pragma unroll
            for (int e = 0; e < 4; ++e) ci[nt][e] = 0;
          }
        }
      }
    }
    uint32_t ck4[4];         // INT2 residual: the tile's K code words
    uint32_t ckp[4];         // 32-dim groups: the same words of lane ^ 2
#pragma unroll
    for (int kk = 0; kk < KT; ++kk) {
      if constexpr (!C::CRX) {
        const int chunk = 2 * kk + kch;
        uint32_t b[4];
        ldsm_x4(sK + (chunk >> 3) * C::BOX_BYTES + ktr * 128 + (((chunk & 7) ^ pr7) << 4), b);
        uint32_t a[4] = {0u, 0u, 0u, 0u};
        {
          const uint2 f = *reinterpret_cast<const uint2*>(qfrag + C::QF0 + (kk * 32 + lane) * 2);
          a[0] = f.x;
          a[2] = f.y;
        }
        mma_bf16((kk & 1) ? cref2[0] : cref[0], a, b[0], b[1]);
        mma_bf16((kk & 1) ? cref2[1] : cref[1], a, b[2], b[3]);
      }
      if constexpr (C::RES && !C::RIM) {
        const uint2 fh = *reinterpret_cast<const uint2*>(qfrag + C::QF1 + (kk * 32 + lane) * 2);
        const uint32_t ah[4] = {fh.x, 0u, fh.y, 0u};
        if constexpr (C::LDM4) {
          // every fourth k-step: words (nt 0, chunk), (nt 1, chunk), (nt 0,
          // chunk + 1), (nt 1, chunk + 1) of two 32-dim chunks
          if ((kk & 3) == 0) {
            const int m = lane >> 3;
            ldsm_x4(smem_u32(st + C::OFF_CK + (wtok + (m & 1) * 8 + pr7) * C::CROW +
                             ((kk >> 1) + (m >> 1)) * 16),
                    ck4);
          }
        }
        if constexpr (C::LDM2) {
          // the whole warp tile's K codes in one ldmatrix: words (nt 0, chunk
          // 0), (nt 1, chunk 0)[, (nt 0, chunk 1), (nt 1, chunk 1)]
          if (kk == 0) {
            const int m = (lane >> 3) & (2 * C::NCH - 1);
            const uint32_t a = smem_u32(st + C::OFF_CK + (wtok + (m & 1) * 8 + pr7) * C::CROW +
                                        (m >> 1) * 16);
            if constexpr (C::NCH == 2) {
              ldsm_x4(a, ck4);
            } else {
              uint32_t r2[2];
              ldsm_x2(a, r2);
              ck4[0] = r2[0];
              ck4[1] = r2[1];
            }
            if constexpr (GROUP == 32) {
#pragma unroll
              for (int m = 0; m < 2 * C::NCH; ++m) ckp[m] = __shfl_xor_sync(FULL, ck4[m], 2);
            }
          }
        }
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
          uint32_t b0, b1;
          if constexpr (C::LDM2) {
            // codes 2u, 2u+8 | 2u+1, 2u+9 of the word in the low mantissa
            // bits: the exact f16 subnormals c 2^-24 (the q~ fragments' k
            // permutation puts the two codes of a B register 16 bits apart)
            uint32_t w;
            int u;
            if constexpr (GROUP == 64) {
              w = ck4[2 * (kk >> 2) + nt];
              u = kk & 3;
            } else {
              const int idx = 2 * (kk >> 2) + nt;
              w = ((q >> 1) == ((kk >> 1) & 1)) ? ck4[idx] : ckp[idx];
              u = 2 * (kk & 1) + (q >> 1);
            }
            b0 = (w >> (4 * u)) & 0x00030003u;
            b1 = (w >> (4 * u + 2)) & 0x00030003u;
          } else {
            static_assert(C::LDM4, "residual codes are INT2 or INT4");
            // codes 2h, 2h+4 | 2h+1, 2h+5 as f16 subnormals c 2^-24, exact
            const uint32_t w = ck4[2 * ((kk >> 1) & 1) + nt];
            const int h = kk & 1;
            b0 = (w >> (8 * h)) & 0x000F000Fu;
            b1 = (w >> (8 * h + 4)) & 0x000F000Fu;
          }
          mma_f16(ct[nt], ah, b0, b1);
        }
        if ((kk + 1) % KSG == 0) {
          // end of scale group j: S += s^K_{t, j} x (q~_j . l_j) for c0, c1
          const int j = kk / KSG;
          const float rsR = row_ok ? rsig_s[g] : 0.0f;
          const float offR = row_ok ? (float)TOPLVL * sq_s[g * NG + j] : 0.0f;
#pragma unroll
          for (int nt = 0; nt < 2; ++nt) {
            const float sk0 = half_at(st + C::OFF_SK + sc_off + tok0[nt] * SB + 2 * j);
            const float sk1 = half_at(st + C::OFF_SK + sc_off + (tok0[nt] + 4) * SB + 2 * j);
            cref[nt][0] = fmaf(sk0 * rsR, fmaf(C::CSCALE, ct[nt][0], -offR), cref[nt][0]);
            cref[nt][1] = fmaf(sk1 * rsR, fmaf(C::CSCALE, ct[nt][1], -offR), cref[nt][1]);
#pragma unroll
            for (int e = 0; e < 4; ++e) ct[nt][e] = 0.0f;
          }
        }
      }
    }
    if constexpr (C::RIM) {
      // ---- residual scores as integer MMAs per 64-dim chunk (one scale
      // group): A = the rows' Q bytes (h | l), B = the n-tile's code words
      // (ldmatrix: lane q holds dims 16q .. 16q+15 of the chunk), one code
      // per byte by a shift and a mask per four codes ----
      uint32_t w4[4];        // (nt 0, chunk 0), (nt 1, chunk 0)[, (nt 0, chunk 1), (nt 1, chunk 1)]
      {
        const int m = (lane >> 3) & (2 * C::NCH - 1);
        const uint32_t a = smem_u32(st + C::OFF_CK + (wtok + (m & 1) * 8 + pr7) * C::CROW +
                                    (m >> 1) * 16);
        if constexpr (C::NCH == 2) {
          ldsm_x4(a, w4);
        } else {
          uint32_t r2[2];
          ldsm_x2(a, r2);
          w4[0] = r2[0];
          w4[1] = r2[1];
        }
      }
      const float sg = row_ok ? rsig_s[g] : 0.0f;
#pragma unroll
      for (int c = 0; c < C::NCH; ++c) {
        int ci[2][4] = {{0, 0, 0, 0}, {0, 0, 0, 0}};
#pragma unroll
        for (int pp = 0; pp < 2; ++pp) {
          const uint4 af = *reinterpret_cast<const uint4*>(qfrag + C::QF1 +
                                                           ((2 * c + pp) * 32 + lane) * 4);
          const uint32_t a[4] = {af.x, af.y, af.z, af.w};
#pragma unroll
          for (int nt = 0; nt < 2; ++nt) {
            const uint32_t w = w4[2 * c + nt];
            mma_s8u8(ci[nt], a, (w >> (4 * pp)) & 0x03030303u, (w >> (4 * pp + 2)) & 0x03030303u);
          }
        }
        // scale group c: S += s^K[t, c] sig (2 <Q, c> - 3 sum Q)
        const int off = row_ok ? TOPLVL * __float2int_rn(sq_s[g * NG + c]) : 0;
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
          const float sk0 = half_at(st + C::OFF_SK + sc_off + tok0[nt] * SB + 2 * c);
          const float sk1 = half_at(st + C::OFF_SK + sc_off + (tok0[nt] + 4) * SB + 2 * c);
          const int x0 = 512 * ci[nt][0] + 2 * ci[nt][2] - off;
          const int x1 = 512 * ci[nt][1] + 2 * ci[nt][3] - off;
          cref[nt][0] = fmaf(sk0 * sg, (float)x0, cref[nt][0]);
          cref[nt][1] = fmaf(sk1 * sg, (float)x1, cref[nt][1]);
        }
      }
    }
    if constexpr (!C::CRX) {
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) cref[nt][e] += cref2[nt][e];
    }
    float sc[2][2];          // row g, tokens q, q + 4 of tile nt
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
      sc[nt][0] = (row_ok && tok0[nt] < n) ? score_scale * cref[nt][0] : kNegInf;
      sc[nt][1] = (row_ok && tok0[nt] + 4 < n) ? score_scale * cref[nt][1] : kNegInf;
    }
    // ---- online softmax of row g (four lanes per row), rescaled lazily ----
    float mc = fmaxf(fmaxf(sc[0][0], sc[0][1]), fmaxf(sc[1][0], sc[1][1]));
    float alpha = 1.0f;
    if (__any_sync(FULL, mc > m_run + kLazyMax)) {
      mc = fmaxf(mc, __shfl_xor_sync(FULL, mc, 1));
      mc = fmaxf(mc, __shfl_xor_sync(FULL, mc, 2));
      const float m_new = fmaxf(m_run, mc);
      alpha = (m_new == m_run) ? 1.0f : (m_run == kNegInf ? 0.0f : exp2f(m_run - m_new));
      m_run = m_new;
    }
    float pr[2][2];
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int e = 0; e < 2; ++e) pr[nt][e] = (sc[nt][e] == kNegInf) ? 0.0f : exp2f(sc[nt][e] - m_run);
    l_run = l_run * alpha + (pr[0][0] + pr[0][1]) + (pr[1][0] + pr[1][1]);
    if (!__all_sync(FULL, alpha == 1.0f)) {
      // rows 2q and 2q+1 of the O^T fragments: their alphas live in lanes 8q, 8q+4
      const float a0 = __shfl_sync(FULL, alpha, 8 * q);
      const float a1 = __shfl_sync(FULL, alpha, 8 * q + 4);
      const float2 a01 = make_float2(a0, a1);
#pragma unroll
      for (int mt = 0; mt < KT; ++mt) {
        float2 x = __fmul2_rn(make_float2(oref[mt][0], oref[mt][1]), a01);
        float2 y = __fmul2_rn(make_float2(oref[mt][2], oref[mt][3]), a01);
        oref[mt][0] = x.x; oref[mt][1] = x.y; oref[mt][2] = y.x; oref[mt][3] = y.y;
        if constexpr (C::RES && !C::VSH) {
          x = __fmul2_rn(make_float2(ores[mt][0], ores[mt][1]), a01);
          y = __fmul2_rn(make_float2(ores[mt][2], ores[mt][3]), a01);
          ores[mt][0] = x.x; ores[mt][1] = x.y; ores[mt][2] = y.x; ores[mt][3] = y.y;
        }
      }
#pragma unroll
      for (int j = 0; j < NG; ++j) {
        wsum[j] *= alpha;
        wsumR[j] *= alpha;
      }
    }
    // P^T fragments (k = tokens q, q + 4 / + 8, n = row g): bf16 hi + lo
    const uint32_t ph0 = pack_bf16(pr[0][0], pr[0][1]);
    const uint32_t ph1 = pack_bf16(pr[1][0], pr[1][1]);
    const uint32_t pl0 = pack_bf16(pr[0][0] - bf16_lo_f(ph0), pr[0][1] - bf16_hi_f(ph0));
    const uint32_t pl1 = pack_bf16(pr[1][0] - bf16_lo_f(ph1), pr[1][1] - bf16_hi_f(ph1));
    if constexpr (C::CRX) {
      // ---- O_ref^T += C_ref^T (P s_ref^V 2^Ev)^T, codes as f16 subnormals ----
      // ldmatrix.trans of the code rows.  INT8: word = codes (token q: dims
      // 2g, 2g+1; token q + 4: dims 2g, 2g+1) of a 16-dim chunk; m-row g is
      // dim 2g, m-row g + 8 dim 2g + 1.  INT4: word = codes of dims 4g .. 4g+3
      // of a 32-dim chunk (token q low half, q + 4 high half, code i at bits
      // 4i); m-tile 2 chunk has m-rows g, g + 8 = dims 4g, 4g + 1, m-tile
      // 2 chunk + 1 dims 4g + 2, 4g + 3.  The weights p s_ref are f16 high parts
      // and remainders after a warp-wide power of two vscale that keeps the
      // tile's largest scale in [1, 2^7): with p < 2^kLazyMax = 2^8 (the
      // lazy softmax max) no weight reaches 2^15, below f16's largest value,
      // and the remainders stay far above its subnormals for every weight
      // that matters.  vscale changes lazily; the accumulators follow it
      // exactly.
      const int tk[4] = {wtok + q, wtok + q + 4, wtok + q + 8, wtok + q + 12};
      auto s_ref_v = [&](int k, int j) {               // 0 beyond the tile
        const float v = half_at(st + C::OFF_RSV + sc_off + tk[k] * SB + 2 * j);
        return (tk[k] < n) ? v : 0.0f;
      };
      // the residual's value products land in the same accumulators, with
      // the same power of two on their weights p s^V
      auto s_res_v = [&](int k, int j) {
        if constexpr (C::VSH) {
          const float v = half_at(st + C::OFF_SV + sc_off + tk[k] * SB + 2 * j);
          return (tk[k] < n) ? v : 0.0f;
        } else {
          return 0.0f;
        }
      };
      float smax = 0.0f;
#pragma unroll
      for (int j = 0; j < NG; ++j)
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          smax = fmaxf(smax, fabsf(s_ref_v(k, j)));
          if constexpr (C::VSH) smax = fmaxf(smax, fabsf(s_res_v(k, j)));
        }
      smax = fmaxf(smax, __shfl_xor_sync(FULL, smax, 1));
      smax = fmaxf(smax, __shfl_xor_sync(FULL, smax, 2));
      {
        const float big = smax * vscale;                 // the same in every lane
        static_assert(kLazyMax <= 8.0f, "p s_ref vscale < 2^(kLazyMax + 7) must fit f16");
        if (smax > 0.0f && !(big >= 1.0f && big < 128.0f)) {
          const int ex = (int)((__float_as_uint(smax) >> 23) & 0xFFu) - 127;
          const float nv = __uint_as_float((uint32_t)(127 + 3 - ex) << 23);   // [2^3, 2^4)
          const float f = nv / vscale;                     // a power of two, exact
#pragma unroll
          for (int mt = 0; mt < KT; ++mt)
#pragma unroll
            for (int e = 0; e < 4; ++e) oref[mt][e] *= f;
#pragma unroll
          for (int j = 0; j < NG; ++j) {
            wsumR[j] *= f;
            if constexpr (C::VSH) wsum[j] *= f;
          }
          vscale = nv;
        }
      }
      const float pk[4] = {pr[0][0] * vscale, pr[0][1] * vscale, pr[1][0] * vscale,
                           pr[1][1] * vscale};
      // The residual's V codes on the reference's m-rows, as f16 subnormals:
      // m-row g (+ 8) of m-tile mt is dim d0 (+ 1), d0 = 16mt + 2g (INT8
      // reference) or 32 (mt / 2) + 4g + 2 (mt & 1) (INT4 reference); one
      // byte permute puts the byte holding d0's code of tokens q, q + 4
      // (and q + 8, q + 12) into halves 0 and 1, a shift brings d0's code to
      // bit 0 and d0 + 1's follows at bit BITS.
      auto res_frag = [&](int mt, uint32_t (&a)[4]) {
        if constexpr (C::VSH) {
          const int d0 = C::CR ? 16 * mt + 2 * g : 32 * (mt >> 1) + 4 * g + 2 * (mt & 1);
          const int wi = d0 * BITS / 32;                       // word holding d0's code
          const int bit = (d0 * BITS) & 31;                    // its bit in the word
          const uint32_t bs = (uint32_t)(bit >> 3);             // byte of the word
          const uint32_t psel = bs | (bs << 4) | ((4u + bs) << 8) | ((4u + bs) << 12);
          const int sh = bit & 7;
          const unsigned char* cvb = st + C::OFF_CV + wi * 4;
          const uint32_t x01 =
              __byte_perm(*reinterpret_cast<const uint32_t*>(cvb + tk[0] * C::CROW),
                          *reinterpret_cast<const uint32_t*>(cvb + tk[1] * C::CROW), psel) >> sh;
          const uint32_t x23 =
              __byte_perm(*reinterpret_cast<const uint32_t*>(cvb + tk[2] * C::CROW),
                          *reinterpret_cast<const uint32_t*>(cvb + tk[3] * C::CROW), psel) >> sh;
          constexpr uint32_t M = (BITS == 2) ? 0x00030003u : 0x000F000Fu;
          a[0] = x01 & M;
          a[1] = (x01 >> BITS) & M;
          a[2] = x23 & M;
          a[3] = (x23 >> BITS) & M;
        }
      };
#pragma unroll
      for (int j = 0; j < NG; ++j) {
        float wv[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) wv[k] = pk[k] * s_ref_v(k, j);
        wsumR[j] += (wv[0] + wv[1]) + (wv[2] + wv[3]);
        uint32_t bh0, bl0, bh1, bl1;
        split_f16(wv[0], wv[1], bh0, bl0);
        split_f16(wv[2], wv[3], bh1, bl1);
        uint32_t rh0 = 0u, rl0 = 0u, rh1 = 0u, rl1 = 0u;   // the residual's weights
        if constexpr (C::VSH) {
          float wr[4];
#pragma unroll
          for (int k = 0; k < 4; ++k) wr[k] = pk[k] * s_res_v(k, j);
          wsum[j] += (wr[0] + wr[1]) + (wr[2] + wr[3]);
          split_f16(wr[0], wr[1], rh0, rl0);
          split_f16(wr[2], wr[3], rh1, rl1);
        }
        auto residual_mma = [&](int mt) {
          if constexpr (C::VSH) {
            uint32_t a[4];
            res_frag(mt, a);
            mma_f16(oref[mt], a, rh0, rh1);
            mma_f16(oref[mt], a, rl0, rl1);
          }
        };
        if constexpr (C::CR4) {
#pragma unroll
          for (int ch = j * GROUP / 32; ch < (j + 1) * GROUP / 32; ++ch) {
            const int m = (lane >> 3) & 1;
            uint32_t v[2];   // (tokens 0-7, chunk ch), (tokens 8-15, chunk ch)
            ldsm_x2_trans(sV + swz_offset<C::RROW>(wtok + m * 8 + pr7, ch), v);
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              // nibbles 2h (m-rows g) and 2h + 1 (m-rows g + 8) of each half:
              // the odd one masked in place as 16 c (an exact subnormal), its
              // m-rows scaled back by 1/16 at the flush
              const uint32_t v0 = h ? v[0] >> 8 : v[0], v1 = h ? v[1] >> 8 : v[1];
              const uint32_t a[4] = {v0 & 0x000F000Fu, v0 & 0x00F000F0u, v1 & 0x000F000Fu,
                                     v1 & 0x00F000F0u};
              mma_f16(oref[2 * ch + h], a, bh0, bh1);
              mma_f16(oref[2 * ch + h], a, bl0, bl1);
              residual_mma(2 * ch + h);
            }
          }
        } else {
#pragma unroll
          for (int mt2 = j * KSG / 2; mt2 < (j + 1) * KSG / 2; ++mt2) {
            const int m = lane >> 3;
            uint32_t v[4];   // (tokens 0-7, chunk 2mt2), (8-15, 2mt2), (0-7, 2mt2+1), (8-15, ..)
            ldsm_x4_trans(sV + swz_offset<C::RROW>(wtok + (m & 1) * 8 + pr7, 2 * mt2 + (m >> 1)),
                          v);
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              const int mt = 2 * mt2 + h;
              const uint32_t R0 = v[2 * h], R1 = v[2 * h + 1];
              // bytes 0, 2 (dim 2g) and bytes 1, 3 (dim 2g + 1) as f16 subnormals
              const uint32_t a[4] = {
                  __byte_perm(R0, 0u, 0x4240), __byte_perm(R0, 0u, 0x4341),
                  __byte_perm(R1, 0u, 0x4240), __byte_perm(R1, 0u, 0x4341)};
              mma_f16(oref[mt], a, bh0, bh1);
              mma_f16(oref[mt], a, bl0, bl1);
              residual_mma(mt);
            }
          }
        }
      }
    } else {
      // ---- O_ref^T += V^T P^T ----
#pragma unroll
      for (int mt = 0; mt < KT; ++mt) {
        const int m = lane >> 3;                         // matrix this lane addresses
        const int tr = wtok + (m >> 1) * 8 + pr7;
        const int chunk = 2 * mt + (m & 1);
        const uint32_t addr = sV + (chunk >> 3) * C::BOX_BYTES + tr * 128 +
                              ((((chunk & 7) ^ pr7)) << 4);
        uint32_t a[4];
        ldsm_x4_trans(addr, a);
        mma_bf16(oref[mt], a, ph0, ph1);
        mma_bf16(oref[mt], a, pl0, pl1);
      }
    }
    // ---- O_res^T += C_V^T (P s^V)^T (an INT8 compressed reference with an
    // INT2 residual takes these products into its accumulators above) ----
    if constexpr (C::RES && !C::VSH) {
      const int tk[4] = {wtok + q, wtok + q + 4, wtok + q + 8, wtok + q + 12};
      const float pk[4] = {pr[0][0], pr[0][1], pr[1][0], pr[1][1]};
      // INT2, 64-dim groups: the warp tile's V code words by one
      // ldmatrix.trans: word = codes of dims 8g .. 8g+7 of a 64-dim chunk
      // (token q low half, q + 4 high half, code i at bits 2i); (tokens 0-7,
      // chunk 0), (8-15, chunk 0)[, (0-7, chunk 1), (8-15, chunk 1)]
      uint32_t cv4[4], cvp[4];   // cvp (32-dim groups): the words of lane ^ 16
      if constexpr (C::LDM2) {
        const int m = (lane >> 3) & (2 * C::NCH - 1);
        const uint32_t a = smem_u32(st + C::OFF_CV + (wtok + (m & 1) * 8 + pr7) * C::CROW +
                                    (m >> 1) * 16);
        if constexpr (C::NCH == 2) {
          ldsm_x4_trans(a, cv4);
        } else {
          uint32_t r2[2];
          ldsm_x2_trans(a, r2);
          cv4[0] = r2[0];
          cv4[1] = r2[1];
        }
        if constexpr (GROUP == 32) {
#pragma unroll
          for (int m2 = 0; m2 < 2 * C::NCH; ++m2) cvp[m2] = __shfl_xor_sync(FULL, cv4[m2], 16);
        }
      }
#pragma unroll
      for (int j = 0; j < NG; ++j) {
        float wv[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const float sv = half_at(st + C::OFF_SV + sc_off + tk[k] * SB + 2 * j);
          wv[k] = (tk[k] < n) ? pk[k] * sv : 0.0f;       // weight 0 beyond the tile
        }
        wsum[j] += (wv[0] + wv[1]) + (wv[2] + wv[3]);
        uint32_t bh0, bl0, bh1, bl1;
        split_bf16(wv[0], wv[1], bh0, bl0);
        split_bf16(wv[2], wv[3], bh1, bl1);
        if constexpr (C::LDM2) {
          // operands (128 + c) - 128 = c, exact (the accumulator carries no
          // offset across the head's tiles)
          const uint32_t m128 = 0xC300C300u;   // {-128, -128}
          if constexpr (GROUP == 64) {
            // chunk j: m-tile 4j + i has m-rows g, g + 8 = dims 64j + 8g + 2i (+ 1)
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const uint32_t R0 = cv4[2 * j], R1 = cv4[2 * j + 1];
              const uint32_t a[4] = {badd2_u(((R0 >> (4 * i)) & 0x00030003u) | kMagic, m128),
                                     badd2_u(((R0 >> (4 * i + 2)) & 0x00030003u) | kMagic, m128),
                                     badd2_u(((R1 >> (4 * i)) & 0x00030003u) | kMagic, m128),
                                     badd2_u(((R1 >> (4 * i + 2)) & 0x00030003u) | kMagic, m128)};
              mma_bf16(ores[4 * j + i], a, bh0, bh1);
              mma_bf16(ores[4 * j + i], a, bl0, bl1);
            }
          } else {
            // group j = half gc of chunk c: lanes g and g ^ 4 both hold the
            // word of dims 8 (g & 3) .. +7 of the group; m-tile 2j + i has
            // m-rows g, g + 8 = dims 64c + 32gc + 8 (g & 3) + 4i + 2 (g >> 2) (+ 1)
            const int c = j >> 1, gc = j & 1;
            const bool own = (g >> 2) == gc;
            const uint32_t R0 = own ? cv4[2 * c] : cvp[2 * c];
            const uint32_t R1 = own ? cv4[2 * c + 1] : cvp[2 * c + 1];
#pragma unroll
            for (int i = 0; i < 2; ++i) {
              const int sh = 2 * (4 * i + 2 * (g >> 2));
              const uint32_t a[4] = {badd2_u(((R0 >> sh) & 0x00030003u) | kMagic, m128),
                                     badd2_u(((R0 >> (sh + 2)) & 0x00030003u) | kMagic, m128),
                                     badd2_u(((R1 >> sh) & 0x00030003u) | kMagic, m128),
                                     badd2_u(((R1 >> (sh + 2)) & 0x00030003u) | kMagic, m128)};
              mma_bf16(ores[2 * j + i], a, bh0, bh1);
              mma_bf16(ores[2 * j + i], a, bl0, bl1);
            }
          }
        } else {
          static_assert(C::LDM4, "residual codes are INT2 or INT4");
          // the group's 32-dim chunks by ldmatrix.trans: word = codes of dims
          // 4g .. 4g+3 of the chunk (token q low half, q + 4 high half, code i
          // at bits 4i); m-tile 2 ch has m-rows g, g + 8 = dims 4g, 4g + 1,
          // m-tile 2 ch + 1 dims 4g + 2, 4g + 3; operands (128 + c) - 128 = c
          const uint32_t m128 = 0xC300C300u;   // {-128, -128}
#pragma unroll
          for (int ch = j * GROUP / 32; ch < (j + 1) * GROUP / 32; ++ch) {
            const int m = (lane >> 3) & 1;
            uint32_t v[2];   // (tokens 0-7, chunk ch), (tokens 8-15, chunk ch)
            ldsm_x2_trans(smem_u32(st + C::OFF_CV + (wtok + m * 8 + pr7) * C::CROW + ch * 16), v);
#pragma unroll
            for (int xy = 0; xy < 2; ++xy) {
              const int sh = 8 * xy;
              const uint32_t a[4] = {badd2_u(((v[0] >> sh) & 0x000F000Fu) | kMagic, m128),
                                     badd2_u(((v[0] >> (sh + 4)) & 0x000F000Fu) | kMagic, m128),
                                     badd2_u(((v[1] >> sh) & 0x000F000Fu) | kMagic, m128),
                                     badd2_u(((v[1] >> (sh + 4)) & 0x000F000Fu) | kMagic, m128)};
              mma_bf16(ores[2 * ch + xy], a, bh0, bh1);
              mma_bf16(ores[2 * ch + xy], a, bl0, bl1);
            }
          }
        }
      }
    }
  };

  // ---- main loop over this CTA's tiles ----
  consume_tiles<C>(p, ring, full_bar, empty_bar, flags, stage_row, first_cur, n_my, SCAP,
                   setup_head, flush_head, reset_state, tile_mma);
}

// ---- host side ---------------------------------------------------------------

template <int D, int G, int BITS, int GROUP, int RB>
cudaError_t launch_gqa_t(const TcParams& gp, cudaStream_t stream) {
  using C = GCfg<D, G, BITS, GROUP, RB>;
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(decode_gqa_kernel<D, G, BITS, GROUP, RB>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         C::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  TcParams g2 = gp;
  if constexpr (C::CTAS != kDecodeCtasPerSm) {
    // the call's CTAs: CTAS per SM, no more than its tiles (uniform calls)
    long long P = (long long)device_sm_count() * C::CTAS;
    if (P > kDecodeMaxCtas) P = kDecodeMaxCtas;
    if (!g2.p.ctx_lens && P > g2.p.n_tiles) P = g2.p.n_tiles;
    if (P < 1) P = 1;
    g2.p.ctas = (int)P;
  }
  return launch_pdl(decode_gqa_kernel<D, G, BITS, GROUP, RB>, g2.p.ctas, kDecodeThreads,
                    C::SMEM_BYTES, stream, g2);
}

template <int D, int G, int RB>
cudaError_t launch_gqa_g(int bits, const TcParams& gp, cudaStream_t stream) {
  const int group = gp.p.group;
  if (bits == 16) {
    if constexpr (RB == 0) {
      return launch_gqa_t<D, G, 16, 32, RB>(gp, stream);   // no scales are read
    } else {
      return group == 32 ? launch_gqa_t<D, G, 16, 32, RB>(gp, stream)
                         : launch_gqa_t<D, G, 16, 64, RB>(gp, stream);
    }
  }
  if (bits == 2)
    return group == 32 ? launch_gqa_t<D, G, 2, 32, RB>(gp, stream)
                       : launch_gqa_t<D, G, 2, 64, RB>(gp, stream);
  if (bits == 4)
    return group == 32 ? launch_gqa_t<D, G, 4, 32, RB>(gp, stream)
                       : launch_gqa_t<D, G, 4, 64, RB>(gp, stream);
  return cudaErrorInvalidValue;
}

template <int D, int RB>
cudaError_t launch_gqa_d(int G, int bits, const TcParams& gp, cudaStream_t stream) {
  switch (G) {
    case 2: return launch_gqa_g<D, 2, RB>(bits, gp, stream);
    case 4: return launch_gqa_g<D, 4, RB>(bits, gp, stream);
    case 8: return launch_gqa_g<D, 8, RB>(bits, gp, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace
#endif

}  // namespace rq
