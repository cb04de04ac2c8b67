// rq_decode_cr1.cu -- ResidualQuant decode attention with one query row per
// kv head over a compressed reference, on the sm_100a tensor cores.
//
// Method: "ResidualQuant: KV Cache Quantization for Looped Transformers with
// 2-Bit Residuals", Abstract -- the final loop's reference itself stored as
// rotated INT8 / INT4 codes with fp16 scales per group, every non-final loop
// as rotated INT2 / INT4 residuals against the reconstructed reference.
//
// All of a head's products live in the rotated domain.  With q~ the rotated
// query, j(d) the scale group of dim d and l = 2c - (2^b - 1) the level of a
// code c of b bits:
//   score_t = sum_j s_ref[t, j] <q~_j, l_ref[t]_j> + s^K[t, j] <q~_j, l^K[t]_j>
//   o~[d]   = sum_t p_t (s_ref^V[t, j(d)] l_ref[t, d] + s^V[t, j(d)] l^V[t, d])
// and o~ is inverse-rotated once per head when the CTAs' records are merged
// (rq_decode_common.cuh).  Per warp and 16-token tile:
//
// Scores: integer MMAs (mma.sync m16n8k32, u8 codes x s8 query), tokens as
//   the M rows.  q~ is held as 16-bit fixed point per 32-dim slice v (Q = q~ /
//   sig_v rounded, |Q| <= 32639, Q = 256 h + l with h, l signed bytes).  The
//   B operand's eight columns are (slice v, byte h or l), so one accumulator
//   holds every token's exact integer <Q_v, c_v> for all slices; the level
//   sum is 2 <Q, c> - (2^b - 1) sum Q, then x sig_v and the token's scale.
//   INT8 reference rows are the A operand straight from ldmatrix; INT4 and
//   INT2 codes get one code per byte by a shift and a mask per four codes
//   (the k order of an MMA follows the codes' positions in their words, and
//   the B fragments are built in the same order).
// Values: f16 MMAs (m16n8k16), tokens as the k dimension and dims as the M
//   rows.  Codes enter as the exact f16 subnormals c 2^-24: the reference's
//   by ldmatrix.trans and one byte permute per two codes, the residual's by
//   one byte permute per two tokens and a shift and a mask per two codes,
//   placed on the reference's m-rows so that both share the accumulators.
//   The weights w = p s 2^Ev are split into an f16 high part (column v) and
//   remainder (column v + D/32) per slice v; 2^Ev is a warp-wide power of two,
//   updated lazily, that keeps the tile's largest value scale in [1, 2^7) so
//   that no weight (p < 2^8 under the lazy softmax) leaves f16's range.  The
//   2^25 and the (2^b - 1) sum w offsets are applied when the warp flushes.
//
// Tiles come through the pipeline of rq_decode_tc.cuh (reference code rows
// by TMA tensor copies with the swizzle of their width, residual codes and
// scales by bulk copies); the work split, records and merge are shared with
// the other decode kernels.
#include "rq_decode_tc.cuh"

namespace rq {
namespace {

template <int D, int BITS, int GROUP, int RB>
struct C1Cfg {
  static constexpr int TILE = kDecodeTile;                 // 64 tokens
  static constexpr int WTOK = TILE / kConsumerWarps;       // 16 tokens per warp
  static constexpr bool RES = (BITS != 16);
  static constexpr bool CRX = true;
  static constexpr int RROW = D * RB / 8;                  // reference code bytes per token
  static constexpr int REF_TILE_BYTES = TILE * RROW;
  static constexpr int NBOX = 0, BOX_BYTES = 0;            // (BF16 reference boxes: unused)
  static constexpr int CROW = RES ? D * BITS / 8 : 0;      // residual code bytes per token
  static constexpr int CWORDS = CROW / 4;
  static constexpr int NG = D / GROUP;                     // scale groups per token
  static constexpr int SB = 2 * NG;                        // scale bytes per token
  static constexpr int NV = D / 32;                        // 32-dim slices
  static constexpr int MT = D / 16;                        // value m-tiles
  static constexpr int SC_BYTES = RES ? TILE * (2 * D / 32) + 32 : 0;
  static constexpr int RSC_BYTES = TILE * (2 * D / 32) + 32;
  static constexpr int OFF_K = 0;
  static constexpr int OFF_V = OFF_K + REF_TILE_BYTES;
  static constexpr int OFF_CK = OFF_V + REF_TILE_BYTES;
  static constexpr int OFF_CV = OFF_CK + TILE * CROW;
  static constexpr int OFF_SK = OFF_CV + TILE * CROW;
  static constexpr int OFF_SV = OFF_SK + SC_BYTES;
  static constexpr int OFF_RSK = OFF_SV + SC_BYTES;
  static constexpr int OFF_RSV = OFF_RSK + RSC_BYTES;
  static constexpr int STAGE_BYTES = (OFF_RSV + RSC_BYTES + 1023) / 1024 * 1024;
  // resident CTAs per SM (registers: 65536 / (CTAS x 160 threads), rounded to
  // whole warps per scheduler)
  static constexpr int CTAS = 3;
  // per consumer warp {m, l, o_ref[D], o~[D]}; also the scratch of the
  // sequence-length scan of a variable-length call
  static constexpr int MERGE_0 = kConsumerWarps * (2 + 2 * D);
  static constexpr int MERGE_FLOATS = MERGE_0 > kVarlenMaxBatch + 4 ? MERGE_0 : kVarlenMaxBatch + 4;
  static constexpr int QBUF_FLOATS = 2 * D;                // q and FWHT(D q)
  static constexpr int QI_WORDS = D + 2 * NV;              // Q[D], sig[NV], sum Q[NV]
  // score B fragments per lane: reference MMAs [NV], residual MMAs [4]
  static constexpr int KFRAG_WORDS = (NV + 4) * 32 * 2;
  static constexpr int WSUM_FLOATS = kConsumerWarps * NV * 2;
  static constexpr int MAX_STAGES = 4;
  static constexpr int OTHER_BYTES = 1024 /* base alignment slack */ +
                                     4 * (MERGE_FLOATS + QBUF_FLOATS + QI_WORDS + WSUM_FLOATS +
                                          KFRAG_WORDS) +
                                     2 * MAX_STAGES * 8 + 16 + MAX_STAGES * 8;   // + stage rows
  // the ring: as many stages (2 .. 4) as the CTAS resident CTAs' shared
  // memory allows (228 KB per SM, 1 KB of it reserved per CTA)
  static constexpr int SMEM_PER_CTA = 228 * 1024 / CTAS - 1024;
  static constexpr int FIT = (SMEM_PER_CTA - OTHER_BYTES) / STAGE_BYTES;
  static constexpr int STAGES = FIT > MAX_STAGES ? MAX_STAGES : FIT;
  static constexpr int RING_BYTES = STAGES * STAGE_BYTES;
  static constexpr int SMEM_BYTES = OTHER_BYTES + RING_BYTES;
  static_assert(STAGES >= 2, "a double-buffered ring fits");
  static_assert(D == 64 || D == 128, "head_dim");
  static_assert(GROUP == 32 || GROUP == 64, "scale group");
  static_assert(RB == 4 || RB == 8, "compressed reference: INT4 or INT8 codes");
  static_assert(BITS == 2 || BITS == 4 || BITS == 16, "residual INT2 / INT4, or none");
  // the swizzle pattern repeats every 8 lines
  static_assert(OFF_V % (8 * RROW) == 0, "swizzled tiles start on the period");
  static_assert((WSUM_FLOATS + QI_WORDS + QBUF_FLOATS + MERGE_FLOATS + KFRAG_WORDS) % 2 == 0,
                "barriers 8-byte aligned");
};

// Dim of k position k16 + 4 t + b (k16 = 0 or 16) of score MMA i.
// Reference, INT8: MMA j covers slice j in order (the ldmatrix bytes).
// Reference, INT4: MMA 2 cq + s takes nibble s of chunks 2 cq, 2 cq + 1.
template <int RB>
__device__ __forceinline__ int kdim_ref(int i, int k16, int t, int b) {
  if constexpr (RB == 8) return 32 * i + k16 + 4 * t + b;
  else return 64 * (i >> 1) + 2 * k16 + 8 * t + 2 * b + (i & 1);
}
// Residual, INT2: MMA m takes codes m + 4 b of words 2 t (k16 0) and 2 t + 1.
// Residual, INT4: MMA m takes nibbles (m & 1) + 2 b of words 4 t + (m >> 1)
// (k16 0) and 4 t + 2 + (m >> 1).
template <int BITS>
__device__ __forceinline__ int kdim_res(int m, int k16, int t, int b) {
  if constexpr (BITS == 2) return 32 * t + k16 + m + 4 * b;
  else return 32 * t + k16 + 8 * (m >> 1) + (m & 1) + 2 * b;
}
// Dim of value m-tile mt's m-row r (0..15).
template <int RB>
__device__ __forceinline__ int vdim(int mt, int r) {
  const int hi = r >> 3, g = r & 7;
  if constexpr (RB == 8) return 32 * (mt >> 1) + 16 * hi + 2 * g + (mt & 1);
  else return 64 * (mt >> 2) + 32 * hi + 4 * g + (mt & 3);
}

template <int D, int BITS, int GROUP, int RB>
__global__ void __launch_bounds__(kDecodeThreads, C1Cfg<D, BITS, GROUP, RB>::CTAS)
decode_cr1_kernel(const __grid_constant__ TcParams gp) {
  using C = C1Cfg<D, BITS, GROUP, RB>;
  const DecodeParams& p = gp.p;
  constexpr int STAGES = C::STAGES, NV = C::NV, MT = C::MT, SB = C::SB;
  constexpr unsigned FULL = 0xffffffffu;
  constexpr int TOP = C::RES ? (1 << BITS) - 1 : 0;
  constexpr int RT = (1 << RB) - 1;
  constexpr int RSH = (GROUP == 64) ? 1 : 0;               // slice -> scale group
  constexpr float CSCALE = 33554432.0f;                    // 2^25

  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  unsigned char* ring = smem;
  float* merge = reinterpret_cast<float*>(smem + C::RING_BYTES);
  float* qbuf = merge + C::MERGE_FLOATS;
  int* qi = reinterpret_cast<int*>(qbuf + C::QBUF_FLOATS);          // Q[D]
  float* qsig_s = reinterpret_cast<float*>(qi + D);                 // [NV]
  int* qsum_s = qi + D + NV;                                         // [NV]
  float* wsum_s = reinterpret_cast<float*>(qi + C::QI_WORDS);       // [warp][NV][2]
  uint32_t* kfrag = reinterpret_cast<uint32_t*>(wsum_s + C::WSUM_FLOATS);   // [NV + 4][32][2]
  uint64_t* full_bar = reinterpret_cast<uint64_t*>(kfrag + C::KFRAG_WORDS);
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

  CallSplit split;
  long long tile_begin, tile_end;
  TileCursor first_cur;
  if (!plan_cta(p, cta, reinterpret_cast<int*>(merge), split, tile_begin, tile_end, first_cur))
    return;
  const int n_my = (int)(tile_end - tile_begin);
  constexpr int SCAP = C::RES ? C::SC_BYTES : C::RSC_BYTES;   // scale bytes per array

  // ========================= producer warp ================================
  if (warp == kConsumerWarps) {
    if (lane == 0)
      tile_producer<C>(gp, ring, full_bar, empty_bar, flags, stage_row, first_cur, n_my, SCAP);
    return;
  }

  // ========================= consumer warps ===============================
  const int g = lane >> 2;            // fragment row group
  const int t = lane & 3;             // fragment column pair / k group
  const int tv = (NV == 4 || t < NV) ? t : 0;   // t as a slice (head_dim 64: t < 2)
  const int wtok = warp * C::WTOK;
  const int r7 = lane & 7;
  const int mrow = lane >> 3;         // ldmatrix: the matrix this lane addresses
  // value B columns of this lane: slice cv = g % NV, part g / NV (0 high
  // part, 1 remainder, else an unused column)
  const int cv = g % NV, cpart = g / NV;

  // per-head constants of the lane: sig_t x score scale and the levels'
  // offsets; the score B fragments (Q bytes in the k order of the codes) are
  // in kfrag, written by warp 0
  float ksig = 0.0f;
  int koffR = 0, koffK = 0;
  // running state: softmax max and sum (base 2), V weight power of two, the
  // lane's sums of reference / residual weights (slice cv, part 0 lanes),
  // and the value accumulators (m-rows = dims, columns = slice x part)
  float m_run = kNegInf, l_run = 0.0f, vscale = 1.0f, wr_sum = 0.0f, wv_sum = 0.0f;
  float acc[MT][4];

  auto reset_state = [&]() {
    m_run = kNegInf;
    l_run = 0.0f;
    vscale = 1.0f;
    wr_sum = 0.0f;
    wv_sum = 0.0f;
#pragma unroll
    for (int mt = 0; mt < MT; ++mt)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[mt][e] = 0.0f;
  };

  auto setup_head = [&](long long hd) {
    float* qs = qbuf;
    float* qt = qbuf + D;
    load_rotate_queries<D, 1>(p, hd, qs, qt, tid);
    const float cd = rot_scale<D>();
    if (warp < NV) {
      // slice v = warp of q~ as 16-bit fixed point, one dim per lane: Q =
      // q~ / sig, |Q| <= 32639 so that Q = 256 h + l has signed-byte h and l
      const float x = cd * qt[32 * warp + lane];
      float mx = fabsf(x);
#pragma unroll
      for (int m = 1; m < 32; m <<= 1) mx = fmaxf(mx, __shfl_xor_sync(FULL, mx, m));
      const float sig = mx > 0.0f ? mx * (1.0f / 32639.0f) : 1.0f;
      const float inv = 1.0f / sig;
      const int Q = min(max(__float2int_rn(x * inv), -32639), 32639);
      qi[32 * warp + lane] = Q;
      int sum = Q;
#pragma unroll
      for (int m = 1; m < 32; m <<= 1) sum += __shfl_xor_sync(FULL, sum, m);
      if (lane == 0) {
        qsig_s[warp] = sig;
        qsum_s[warp] = sum;
      }
    }
    named_bar_sync(1, kConsumerThreads);
    // byte (0: h, 1: l) of Q[dim] for this lane's B column (slice g / 2),
    // zero for the other slices' k positions
    auto qbyte = [&](int dim) -> uint32_t {
      if (dim >= D || (dim >> 5) != (g >> 1)) return 0u;
      const int Q = qi[dim];
      const int lo = ((Q + 128) & 255) - 128;
      const int hi = (Q - lo) >> 8;
      return (uint32_t)(((g & 1) ? lo : hi) & 0xFF);
    };
    // the MMAs' fragments, spread over the consumer warps
#pragma unroll 1
    for (int i = warp; i < NV + 4; i += kConsumerWarps) {
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        uint32_t w = 0u;
#pragma unroll
        for (int b = 0; b < 4; ++b) {
          const int dim = i < NV ? kdim_ref<RB>(i, 16 * h, t, b)
                                 : kdim_res<BITS == 4 ? 4 : 2>(i - NV, 16 * h, t, b);
          w |= qbyte(dim) << (8 * b);
        }
        kfrag[(i * 32 + lane) * 2 + h] = w;
      }
    }
    const bool slice_ok = t < NV;
    ksig = slice_ok ? qsig_s[tv] * p.score_scale : 0.0f;
    koffR = slice_ok ? -RT * qsum_s[tv] : 0;
    koffK = slice_ok ? -TOP * qsum_s[tv] : 0;
    named_bar_sync(1, kConsumerThreads);      // fragments written, Q free for the next head
  };

  auto flush_head = [&](long long hd, long long first_tile, int nt_h) {
    // l over the 8 row groups (the four lanes of a group hold the same tokens)
    l_run += __shfl_xor_sync(FULL, l_run, 4);
    l_run += __shfl_xor_sync(FULL, l_run, 8);
    l_run += __shfl_xor_sync(FULL, l_run, 16);
    // weight sums of slice cv over the lanes' tokens
    wr_sum += __shfl_xor_sync(FULL, wr_sum, 1);
    wr_sum += __shfl_xor_sync(FULL, wr_sum, 2);
    wv_sum += __shfl_xor_sync(FULL, wv_sum, 1);
    wv_sum += __shfl_xor_sync(FULL, wv_sum, 2);
    // remainder columns (v + NV) onto the high ones (v): lane t ^ NV/2
#pragma unroll
    for (int mt = 0; mt < MT; ++mt)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[mt][e] += __shfl_xor_sync(FULL, acc[mt][e], NV / 2);
    named_bar_sync(1, kConsumerThreads);          // merge area free
    float* mw = merge + warp * (2 + 2 * D);
    if (lane == 0) {
      mw[0] = m_run;
      mw[1] = l_run;
    }
    const float inv_vs = 1.0f / vscale;           // a power of two
    if (t == 0 && cpart == 0) {
      // non-finite weights (invalid scales): the output is not valid
      if (!isfinite(wr_sum) || !isfinite(wv_sum)) flag_error(p.status, 64u);
      wsum_s[(warp * NV + cv) * 2] = wr_sum * inv_vs;
      wsum_s[(warp * NV + cv) * 2 + 1] = wv_sum * inv_vs;
    }
    // lane (g, t) holds columns 2t, 2t+1 of m-rows g, g + 8: the slice-vg
    // value of a dim sits in lane t = vg / 2, column parity vg & 1
#pragma unroll
    for (int mt = 0; mt < MT; ++mt)
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int dim = vdim<RB>(mt, g + 8 * h);
        const int vg = dim >> 5;
        if ((vg >> 1) == t) {
          const float a = (vg & 1) ? acc[mt][2 * h + 1] : acc[mt][2 * h];
          mw[2 + D + dim] = a * (CSCALE * inv_vs);
        }
      }
    named_bar_sync(1, kConsumerThreads);
    // o~ = 2^25 acc - (2^RB - 1) sum w_ref - (2^b - 1) sum w_res per slice;
    // the BF16 part of the record is empty
    for (int e = tid; e < kConsumerWarps * D; e += kConsumerThreads) {
      const int w = e / D, dim = e % D;
      float* rec = merge + w * (2 + 2 * D);
      const float* ws = wsum_s + (w * NV + (dim >> 5)) * 2;
      rec[2 + D + dim] -= (float)RT * ws[0] + (float)TOP * ws[1];
      rec[2 + dim] = 0.0f;
    }
    named_bar_sync(1, kConsumerThreads);
    // four records per batch: the smaller merge leaves the token loop more registers
    finish_head<D, 1, true, 4>(p, hd, first_tile, nt_h, split, cta, merge, qbuf, flags, tid);
  };

  auto kfrag_at = [&](int i) {
    return *reinterpret_cast<const uint2*>(kfrag + (i * 32 + lane) * 2);
  };

  // ---- one tile: 16 tokens per warp ----
  auto tile_cr1 = [&](const unsigned char* st, int n, int sc_off) {
    const uint32_t sK = smem_u32(st + C::OFF_K);
    const uint32_t sV = smem_u32(st + C::OFF_V);
    // ---- scores of tokens wtok + g (c0, c1) and wtok + g + 8 (c2, c3) ----
    // two accumulators per chain (even / odd MMAs), summed after
    int cr[4] = {0, 0, 0, 0}, cr2[4] = {0, 0, 0, 0};
    {
      const int trow = wtok + (mrow & 1) * 8 + r7;
      if constexpr (RB == 8) {
        // matrices (tokens 0-7, chunk 2j), (8-15, 2j), (0-7, 2j + 1), (8-15, 2j + 1)
#pragma unroll
        for (int j = 0; j < NV; ++j) {
          uint32_t a[4];
          ldsm_x4(sK + swz_offset<C::RROW>(trow, 2 * j + (mrow >> 1)), a);
          const uint2 b = kfrag_at(j);
          mma_u8s8((j & 1) ? cr2 : cr, a, b.x, b.y);
        }
      } else {
#pragma unroll
        for (int cq = 0; cq < NV / 2; ++cq) {
          uint32_t r[4];
          ldsm_x4(sK + swz_offset<C::RROW>(trow, 2 * cq + (mrow >> 1)), r);
          // low nibbles, and the high ones masked in place as bytes 16 c (cr2
          // then holds 16 x their sums, divided out below)
#pragma unroll
          for (int s = 0; s < 2; ++s) {
            const uint32_t mk = s ? 0xF0F0F0F0u : 0x0F0F0F0Fu;
            const uint32_t a[4] = {r[0] & mk, r[1] & mk, r[2] & mk, r[3] & mk};
            const uint2 b = kfrag_at(2 * cq + s);
            mma_u8s8(s ? cr2 : cr, a, b.x, b.y);
          }
        }
      }
    }
    int ck[4] = {0, 0, 0, 0}, ck2[4] = {0, 0, 0, 0};
    if constexpr (C::RES) {
      // lane t: the words of slice t of tokens g and g + 8, one code per byte
      const unsigned char* r0 = st + C::OFF_CK + (wtok + g) * C::CROW;
      const unsigned char* r1 = r0 + 8 * C::CROW;
      if constexpr (BITS == 2) {
        const uint2 w0 = *reinterpret_cast<const uint2*>(r0 + 8 * tv);
        const uint2 w1 = *reinterpret_cast<const uint2*>(r1 + 8 * tv);
#pragma unroll
        for (int m = 0; m < 4; ++m) {
          const uint32_t a[4] = {(w0.x >> (2 * m)) & 0x03030303u, (w1.x >> (2 * m)) & 0x03030303u,
                                 (w0.y >> (2 * m)) & 0x03030303u, (w1.y >> (2 * m)) & 0x03030303u};
          const uint2 b = kfrag_at(NV + m);
          mma_u8s8((m & 1) ? ck2 : ck, a, b.x, b.y);
        }
      } else {
        const uint4 w0 = *reinterpret_cast<const uint4*>(r0 + 16 * tv);
        const uint4 w1 = *reinterpret_cast<const uint4*>(r1 + 16 * tv);
        const uint32_t x0[4] = {w0.x, w0.y, w0.z, w0.w};
        const uint32_t x1[4] = {w1.x, w1.y, w1.z, w1.w};
        // odd m: the high nibbles masked in place (ck2 holds 16 x their sums)
#pragma unroll
        for (int m = 0; m < 4; ++m) {
          const int wi = m >> 1;
          const uint32_t mk = (m & 1) ? 0xF0F0F0F0u : 0x0F0F0F0Fu;
          const uint32_t a[4] = {x0[wi] & mk, x1[wi] & mk, x0[2 + wi] & mk, x1[2 + wi] & mk};
          const uint2 b = kfrag_at(NV + m);
          mma_u8s8((m & 1) ? ck2 : ck, a, b.x, b.y);
        }
      }
    }
    float f0, f1;
    {
      // level sums 2 <Q, c> - (2^b - 1) sum Q of slice t, exact in integers
      const int rg = tv >> RSH;
      const int tok0 = wtok + g, tok1 = tok0 + 8;
      // (exact: an INT4 chain's second accumulator holds multiples of 16)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        cr[e] += (RB == 4) ? (cr2[e] >> 4) : cr2[e];
        ck[e] += (BITS == 4) ? (ck2[e] >> 4) : ck2[e];
      }
      const int xr0 = 512 * cr[0] + 2 * cr[1] + koffR;
      const int xr1 = 512 * cr[2] + 2 * cr[3] + koffR;
      const unsigned char* rs = st + C::OFF_RSK + sc_off + 2 * rg;
      f0 = half_at(rs + tok0 * SB) * (float)xr0;
      f1 = half_at(rs + tok1 * SB) * (float)xr1;
      if constexpr (C::RES) {
        const int xk0 = 512 * ck[0] + 2 * ck[1] + koffK;
        const int xk1 = 512 * ck[2] + 2 * ck[3] + koffK;
        const unsigned char* ks = st + C::OFF_SK + sc_off + 2 * rg;
        f0 = fmaf(half_at(ks + tok0 * SB), (float)xk0, f0);
        f1 = fmaf(half_at(ks + tok1 * SB), (float)xk1, f1);
      }
      f0 *= ksig;
      f1 *= ksig;
      if (NV != 4 && t >= NV) f0 = f1 = 0.0f;
      f0 += __shfl_xor_sync(FULL, f0, 1);
      f1 += __shfl_xor_sync(FULL, f1, 1);
      f0 += __shfl_xor_sync(FULL, f0, 2);
      f1 += __shfl_xor_sync(FULL, f1, 2);
      if (n < C::TILE) {               // a partial tile: tokens from n on are not cached
        if (tok0 >= n) f0 = kNegInf;
        if (tok1 >= n) f1 = kNegInf;
      }
    }
    // ---- online softmax, one row per warp, rescaled lazily ----
    {
      float mc = fmaxf(f0, f1);
      if (__any_sync(FULL, mc > m_run + kLazyMax)) {
        mc = fmaxf(mc, __shfl_xor_sync(FULL, mc, 4));
        mc = fmaxf(mc, __shfl_xor_sync(FULL, mc, 8));
        mc = fmaxf(mc, __shfl_xor_sync(FULL, mc, 16));
        const float m_new = fmaxf(m_run, mc);
        const float alpha = (m_run == kNegInf) ? 0.0f : exp2f(m_run - m_new);
        m_run = m_new;
        l_run *= alpha;
        wr_sum *= alpha;
        wv_sum *= alpha;
#pragma unroll
        for (int mt = 0; mt < MT; ++mt)
#pragma unroll
          for (int e = 0; e < 4; ++e) acc[mt][e] *= alpha;
      }
    }
    const float p0 = (f0 == kNegInf) ? 0.0f : exp2f(f0 - m_run);
    const float p1 = (f1 == kNegInf) ? 0.0f : exp2f(f1 - m_run);
    l_run += p0 + p1;

    // ---- value weights ----
    // k positions 2t, 2t+1 (b0) and 2t+8, 2t+9 (b1) of the value MMAs carry
    // tokens t, t + 4 and t + 8, t + 12: the four lanes t then read four
    // consecutive code rows (no bank conflict), and the ldmatrix row order
    // below follows the same permutation
    const int tk[4] = {t, t + 4, t + 8, t + 12};
    float pk[4] = {__shfl_sync(FULL, p0, 4 * t), __shfl_sync(FULL, p0, 4 * t + 16),
                   __shfl_sync(FULL, p1, 4 * t), __shfl_sync(FULL, p1, 4 * t + 16)};
    float sr[4], sv[4] = {0.0f, 0.0f, 0.0f, 0.0f};
    {
      const int rg = cv >> RSH;
      float smax = 0.0f;
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int tok = wtok + tk[k];
        sr[k] = half_at(st + C::OFF_RSV + sc_off + tok * SB + 2 * rg);
        if constexpr (C::RES) sv[k] = half_at(st + C::OFF_SV + sc_off + tok * SB + 2 * rg);
      }
      if (n < C::TILE) {                 // weight 0 beyond the tile
#pragma unroll
        for (int k = 0; k < 4; ++k)
          if (wtok + tk[k] >= n) sr[k] = sv[k] = 0.0f;
      }
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        smax = fmaxf(smax, fabsf(sr[k]));
        if constexpr (C::RES) smax = fmaxf(smax, fabsf(sv[k]));
      }
      // 2^Ev moves only when the tile's largest value scale times 2^Ev leaves
      // [1, 2^7): one vote decides, the warp's max is formed only then
      const float big_l = smax * vscale;
      const uint32_t code = (big_l >= 128.0f ? 1u : 0u) | (big_l >= 1.0f ? 2u : 0u) |
                            (smax > 0.0f ? 4u : 0u);
      const uint32_t any = __reduce_or_sync(FULL, code);
      static_assert(kLazyMax <= 8.0f, "p s vscale < 2^(kLazyMax + 7) must fit f16");
      if ((any & 1u) || ((any & 4u) && !(any & 2u))) {
        // lanes differ in tokens (t) and slice (g % NV)
        smax = fmaxf(smax, __shfl_xor_sync(FULL, smax, 1));
        smax = fmaxf(smax, __shfl_xor_sync(FULL, smax, 2));
        smax = fmaxf(smax, __shfl_xor_sync(FULL, smax, 4));
        if constexpr (NV == 4) smax = fmaxf(smax, __shfl_xor_sync(FULL, smax, 8));
        const int ex = (int)((__float_as_uint(smax) >> 23) & 0xFFu) - 127;
        const float nv = __uint_as_float((uint32_t)(127 + 3 - ex) << 23);   // [2^3, 2^4)
        const float f = nv / vscale;                     // a power of two, exact
#pragma unroll
        for (int mt = 0; mt < MT; ++mt)
#pragma unroll
          for (int e = 0; e < 4; ++e) acc[mt][e] *= f;
        wr_sum *= f;
        wv_sum *= f;
        vscale = nv;
      }
    }
#pragma unroll
    for (int k = 0; k < 4; ++k) pk[k] *= vscale;
    // B fragments: the high part (part 0), the remainder (part 1) or zero
    auto weight_frags = [&](const float (&s)[4], uint32_t& b0, uint32_t& b1, float& wsum) {
      const float w0 = pk[0] * s[0], w1 = pk[1] * s[1], w2 = pk[2] * s[2], w3 = pk[3] * s[3];
      uint32_t h0, l0, h1, l1;
      split_f16(w0, w1, h0, l0);
      split_f16(w2, w3, h1, l1);
      b0 = cpart == 0 ? h0 : (cpart == 1 ? l0 : 0u);
      b1 = cpart == 0 ? h1 : (cpart == 1 ? l1 : 0u);
      if (cpart == 0) wsum += (w0 + w1) + (w2 + w3);
    };
    uint32_t br0, br1, bv0 = 0u, bv1 = 0u;
    weight_frags(sr, br0, br1, wr_sum);
    if constexpr (C::RES) weight_frags(sv, bv0, bv1, wv_sum);
    // INT8 reference: the residual codes of the odd m-tiles enter masked in
    // place (4c for INT2, 16c for INT4; exact subnormals), their weights
    // scaled down by the same power of two (exact)
    uint32_t bv0o = bv0, bv1o = bv1;
    if constexpr (C::RES && RB == 8) {
      const uint32_t f = (BITS == 2) ? 0x34003400u : 0x2C002C00u;   // {1/4, 1/4} / {1/16, 1/16}
      bv0o = hmul2_u(bv0, f);
      bv1o = hmul2_u(bv1, f);
    }

    // ---- values: o~^T += C^T W^T, reference then residual codes ----
    const unsigned char* cvb = st + C::OFF_CV;
    // ldmatrix.trans: matrix row r (this lane's address) is token
    // (r >> 1) + 4 (r & 1) of its 8-token half, so lane t receives tokens t, t + 4
    const int vrow = wtok + (mrow >> 1) * 8 + ((r7 >> 1) | ((r7 & 1) << 2));
    if constexpr (RB == 8) {
      // residual byte of m-row g: INT2 byte g / 2 (bits 4 (g & 1) + 2e),
      // INT4 byte g & 3 (bits 4e) of word (g >> 2)
      const uint32_t bsel = (BITS == 2) ? (uint32_t)(g >> 1) : (uint32_t)(g & 3);
      const uint32_t psel = bsel | (bsel << 4) | ((4u + bsel) << 8) | ((4u + bsel) << 12);
#pragma unroll
      for (int cp = 0; cp < NV; ++cp) {
        uint32_t R[4];   // (tokens 0-7, chunk 2cp), (0-7, 2cp + 1), (8-15, 2cp), (8-15, 2cp + 1)
        ldsm_x4_trans(sV + swz_offset<C::RROW>(vrow, 2 * cp + (mrow & 1)), R);
        uint32_t X[4];   // residual: (tokens t, t+4 | t+8, t+12) x (m-rows g | g + 8)
        if constexpr (C::RES) {
          if constexpr (BITS == 2) {
            // words 2cp (m-rows g) and 2cp + 1 (m-rows g + 8) of the four tokens
            uint2 w[4];
#pragma unroll
            for (int k = 0; k < 4; ++k)
              w[k] = *reinterpret_cast<const uint2*>(cvb + (wtok + tk[k]) * C::CROW + 8 * cp);
            // the nibble of m-row g down to bit 0
            const int sh = 4 * (g & 1);
            X[0] = __byte_perm(w[0].x, w[1].x, psel) >> sh;
            X[1] = __byte_perm(w[0].y, w[1].y, psel) >> sh;
            X[2] = __byte_perm(w[2].x, w[3].x, psel) >> sh;
            X[3] = __byte_perm(w[2].y, w[3].y, psel) >> sh;
          } else {
            // words 4cp + (g >> 2) (m-rows g) and 4cp + 2 + (g >> 2)
            const int wo = 4 * (4 * cp + (g >> 2));
            uint32_t w[4][2];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              const unsigned char* rr = cvb + (wtok + tk[k]) * C::CROW + wo;
              w[k][0] = *reinterpret_cast<const uint32_t*>(rr);
              w[k][1] = *reinterpret_cast<const uint32_t*>(rr + 8);
            }
            X[0] = __byte_perm(w[0][0], w[1][0], psel);
            X[1] = __byte_perm(w[0][1], w[1][1], psel);
            X[2] = __byte_perm(w[2][0], w[3][0], psel);
            X[3] = __byte_perm(w[2][1], w[3][1], psel);
          }
        }
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          // bytes 0, 2 (dim 2g + e of tokens t, t + 4) as f16 subnormals
          const uint32_t sel = e ? 0x4341u : 0x4240u;
          const uint32_t a[4] = {__byte_perm(R[0], 0u, sel), __byte_perm(R[1], 0u, sel),
                                 __byte_perm(R[2], 0u, sel), __byte_perm(R[3], 0u, sel)};
          mma_f16(acc[2 * cp + e], a, br0, br1);
          if constexpr (C::RES) {
            // m-rows g: INT2 bits 2e of the nibble (Y), INT4 nibble e of the byte
            constexpr uint32_t M = (BITS == 2) ? 0x00030003u : 0x000F000Fu;
            const uint32_t Me = e ? (BITS == 2 ? M << 2 : M << 4) : M;
            const uint32_t c[4] = {X[0] & Me, X[1] & Me, X[2] & Me, X[3] & Me};
            if (e) mma_f16(acc[2 * cp + e], c, bv0o, bv1o);
            else mma_f16(acc[2 * cp + e], c, bv0, bv1);
          }
        }
      }
    } else {
      // residual of m-row g (dims 64cq + 4g + s): INT2 byte g & 3 (bits 2s) of
      // word 4cq + (g >> 2); INT4 half g & 1 (bits 4s) of word 8cq + (g >> 1)
      const uint32_t h2 = (uint32_t)(g & 1);
      const uint32_t psel =
          (BITS == 2)
              ? ((uint32_t)(g & 3) | ((uint32_t)(g & 3) << 4) | ((4u + (g & 3)) << 8) |
                 ((4u + (g & 3)) << 12))
              : ((2u * h2) | ((2u * h2 + 1u) << 4) | ((4u + 2u * h2) << 8) |
                 ((5u + 2u * h2) << 12));
      // codes are masked in place where they sit in the low 10 bits of a
      // half (exact subnormals 2^k c 2^-24), their weights scaled by 2^-k
      // (exact): the reference's odd nibbles (k = 4), the INT2 residual's
      // fields 1-3 (k = 2, 4, 6), the INT4 residual's odd nibbles (k = 4);
      // nibbles 2 and 3 of a half are first moved down by one shift of 8
      const uint32_t br0q = hmul2_u(br0, 0x2C002C00u), br1q = hmul2_u(br1, 0x2C002C00u);
      uint32_t bvs0[4] = {bv0, bv0, bv0, bv0}, bvs1[4] = {bv1, bv1, bv1, bv1};
      if constexpr (C::RES) {
        if constexpr (BITS == 2) {
#pragma unroll
          for (int s = 1; s < 4; ++s) {
            const uint32_t f = s == 1 ? 0x34003400u : (s == 2 ? 0x2C002C00u : 0x24002400u);
            bvs0[s] = hmul2_u(bv0, f);
            bvs1[s] = hmul2_u(bv1, f);
          }
        } else {
          bvs0[1] = bvs0[3] = hmul2_u(bv0, 0x2C002C00u);
          bvs1[1] = bvs1[3] = hmul2_u(bv1, 0x2C002C00u);
        }
      }
#pragma unroll
      for (int cq = 0; cq < NV / 2; ++cq) {
        uint32_t R[4];   // (tokens 0-7, chunk 2cq), (0-7, 2cq + 1), (8-15, 2cq), (8-15, 2cq + 1)
        ldsm_x4_trans(sV + swz_offset<C::RROW>(vrow, 2 * cq + (mrow & 1)), R);
        uint32_t X[4];
        if constexpr (C::RES) {
          // words of m-rows g and g + 8 (32 dims further)
          const int wo = (BITS == 2) ? 4 * (4 * cq + (g >> 2)) : 4 * (8 * cq + (g >> 1));
          constexpr int WHI = (BITS == 2) ? 8 : 16;    // bytes from m-row g's word to g + 8's
          uint32_t w[4][2];
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const unsigned char* rr = cvb + (wtok + tk[k]) * C::CROW + wo;
            w[k][0] = *reinterpret_cast<const uint32_t*>(rr);
            w[k][1] = *reinterpret_cast<const uint32_t*>(rr + WHI);
          }
          X[0] = __byte_perm(w[0][0], w[1][0], psel);
          X[1] = __byte_perm(w[0][1], w[1][1], psel);
          X[2] = __byte_perm(w[2][0], w[3][0], psel);
          X[3] = __byte_perm(w[2][1], w[3][1], psel);
        }
        uint32_t R8[4], X8[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          R8[i] = R[i] >> 8;
          X8[i] = (BITS == 4) ? X[i] >> 8 : X[i];
        }
#pragma unroll
        for (int s = 0; s < 4; ++s) {
          // nibble s of each half: dim 4g + s of tokens t, t + 4
          const uint32_t* Rs = s < 2 ? R : R8;
          const uint32_t Mr = (s & 1) ? 0x00F000F0u : 0x000F000Fu;
          const uint32_t a[4] = {Rs[0] & Mr, Rs[1] & Mr, Rs[2] & Mr, Rs[3] & Mr};
          mma_f16(acc[4 * cq + s], a, (s & 1) ? br0q : br0, (s & 1) ? br1q : br1);
          if constexpr (C::RES) {
            const uint32_t* Xs = (BITS == 4 && s >= 2) ? X8 : X;
            const uint32_t M = (BITS == 2) ? (0x00030003u << (2 * s))
                                           : ((s & 1) ? 0x00F000F0u : 0x000F000Fu);
            const uint32_t c[4] = {Xs[0] & M, Xs[1] & M, Xs[2] & M, Xs[3] & M};
            mma_f16(acc[4 * cq + s], c, bvs0[s], bvs1[s]);
          }
        }
      }
    }
  };

  consume_tiles<C>(p, ring, full_bar, empty_bar, flags, stage_row, first_cur, n_my, SCAP,
                   setup_head, flush_head, reset_state, tile_cr1);
}

template <int D, int BITS, int GROUP, int RB>
cudaError_t launch_cr1_t(const TcParams& gp, cudaStream_t stream) {
  using C = C1Cfg<D, BITS, GROUP, RB>;
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(decode_cr1_kernel<D, BITS, GROUP, RB>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         C::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  // the call's CTAs: CTAS per SM, no more than its tiles (uniform calls)
  TcParams g2 = gp;
  long long P = (long long)device_sm_count() * C::CTAS;
  if (P > kDecodeMaxCtas) P = kDecodeMaxCtas;
  if (!g2.p.ctx_lens && P > g2.p.n_tiles) P = g2.p.n_tiles;
  if (P < 1) P = 1;
  g2.p.ctas = (int)P;
  return launch_pdl(decode_cr1_kernel<D, BITS, GROUP, RB>, g2.p.ctas, kDecodeThreads,
                    C::SMEM_BYTES, stream, g2);
}

template <int D, int RB>
cudaError_t launch_cr1_b(int bits, const TcParams& gp, cudaStream_t stream) {
  const bool g32 = gp.p.group == 32;
  if (bits == 2) return g32 ? launch_cr1_t<D, 2, 32, RB>(gp, stream) : launch_cr1_t<D, 2, 64, RB>(gp, stream);
  if (bits == 4) return g32 ? launch_cr1_t<D, 4, 32, RB>(gp, stream) : launch_cr1_t<D, 4, 64, RB>(gp, stream);
  if (bits == 16) return g32 ? launch_cr1_t<D, 16, 32, RB>(gp, stream) : launch_cr1_t<D, 16, 64, RB>(gp, stream);
  return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_decode_cr1(int head_dim, int bits, const DecodeParams& p,
                              cudaStream_t stream) {
  TcParams gp;
  gp.p = p;
  const unsigned long long rows =
      p.page_table ? (unsigned long long)p.n_pages * p.kv_heads * kDecodeTile
                   : (unsigned long long)p.batch * p.kv_heads * p.ctx_pitch;
  // tensor-copy row coordinates are 32-bit signed
  if (rows > 0x7FFFFFFFull) return cudaErrorInvalidValue;
  if (p.ref_bits != 8 && p.ref_bits != 4) return cudaErrorInvalidValue;
  const int rrow = head_dim * p.ref_bits / 8;
  if (!encode_bytes_map(&gp.tmap_k, p.rcodes_k, rows, rrow, kDecodeTile) ||
      !encode_bytes_map(&gp.tmap_v, p.rcodes_v, rows, rrow, kDecodeTile))
    return cudaErrorInvalidValue;
  if (p.ref_bits == 8) {
    if (head_dim == 128) return launch_cr1_b<128, 8>(bits, gp, stream);
    if (head_dim == 64) return launch_cr1_b<64, 8>(bits, gp, stream);
  } else {
    if (head_dim == 128) return launch_cr1_b<128, 4>(bits, gp, stream);
    if (head_dim == 64) return launch_cr1_b<64, 4>(bits, gp, stream);
  }
  return cudaErrorInvalidValue;
}

}  // namespace rq
