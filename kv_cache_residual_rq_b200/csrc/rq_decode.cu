// rq_decode.cu -- fused ResidualQuant decode attention for sm_100a.
//
// Method: "ResidualQuant: KV Cache Quantization for Looped Transformers with
// 2-Bit Residuals", Abstract -- decode reads the BF16 final-loop reference
// plus each other loop's low-bit rotated residual and rebuilds that loop's
// K/V efficiently; the saving is KV memory traffic.
//
// For one loop the kernel computes, per (batch b, query head j, kv head h):
//   score_t = sigma * ( <q, refK_t> + sum_g s^K_t,g <q~_g, l^K_t,g> ),  q~ = Rot q
//   out     = ( sum_t p_t refV_t + Rot^T sum_t p_t s^V_t l^V_t ) / sum_t p_t
// so K_hat and V_hat are never built: the query is rotated once per head
// and the V residual is accumulated in the rotated domain and rotated back
// once per output row.
//
// Structure (one launch per call):
//   - P = 2 x SMs persistent CTAs.  The (head, tile) space -- heads are
//     (b, h) pairs, tiles are 64-token runs of the context -- is numbered
//     head-major and cut into P equal runs, one per CTA, so each CTA streams
//     the same number of tiles.
//   - Warp 4 is the producer: one lane issues cp.async.bulk copies of a
//     tile's reference K/V rows, codes and scales (all contiguous runs in
//     HBM) into a ring of shared-memory stages, completion tracked by
//     mbarrier transaction counts.
//   - Warps 0-3 consume: lanes split head_dim, so one 16- or 8-byte shared
//     load per lane reads a token row.  Base-2 online softmax per warp.
//   - At the end of a head's run the consumer warps merge their states and
//     write one partial record; the last CTA to arrive for that head (an
//     atomic ticket, no waiting) merges all records, applies the inverse
//     rotation once and writes the output.
//
// Arithmetic per token is what limits this kernel once the copies stream, so
// the single-query (G = 1) path is shaped to issue few instructions:
//   - INT2 K residual: per head, a shared-memory table holds, for every
//     4-dim slice of q~ and every byte of 4 codes, the partial product
//     sum_k q~_k l(c_k); a lane's 8 dims cost two table reads.
//   - Codes become floats with one AND/OR each and one paired subtract per
//     two codes (the 2^23 exponent trick, the code left at its bit
//     position, `sub.rn.f32x2`); the position's
//     power of two is folded into the query constants or applied once when
//     the V accumulator is flushed.
//   - Scores are reduce-scattered across the lanes of a token (one shuffle
//     per value instead of four), so each lane evaluates one exp per chunk.
//   - <q, refK> uses the sm_100 fp32 += bf16 x bf16 fused multiply-add on
//     the packed rows (no unpacking; the products are exact), and the V
//     accumulators are packed fp32 pairs updated with the paired FMA.
// Every mbarrier wait is bounded; a wait that runs out raises the workspace
// status word, and the kernel still finishes (its output is then invalid).
#include "rq_decode_common.cuh"

namespace rq {
namespace {

constexpr int kThreads = kDecodeThreads;

template <int D, int G, int BITS>
struct Cfg {
  static constexpr int DPL = (G >= 4) ? 4 : 8;              // dims per lane
  static constexpr int LPT = D / DPL;                       // lanes per token
  static constexpr int TPS = 32 / LPT;                      // tokens per warp step
  static constexpr int TILE = kDecodeTile;
  static constexpr int TPW = TILE / kConsumerWarps;         // tokens per warp per tile
  static constexpr int STEPS = TPW / TPS;                   // warp steps per tile
  // G == 1 reduce-scatters LPT/2 partial scores per chunk
  static constexpr int CH = (G == 1) ? LPT / 2 : (STEPS < 4 ? STEPS : 4);
  static constexpr bool RES = (BITS != 16);
  static constexpr bool LUT = (G == 1 && BITS == 2);
  static constexpr int KROW = D * 2;                        // BF16 reference row bytes
  static constexpr int CROW = RES ? D * BITS / 8 : 0;       // code bytes per token
  static constexpr int CWORDS = CROW / 4;
  static constexpr int SC_BYTES = RES ? TILE * (2 * D / 32) + 32 : 0;
  static constexpr int OFF_K = 0;
  static constexpr int OFF_V = OFF_K + TILE * KROW;
  static constexpr int OFF_CK = OFF_V + TILE * KROW;
  static constexpr int OFF_CV = OFF_CK + TILE * CROW;
  static constexpr int OFF_SK = OFF_CV + TILE * CROW;
  static constexpr int OFF_SV = OFF_SK + SC_BYTES;
  static constexpr int STAGE_BYTES = OFF_SV + SC_BYTES;
  static constexpr int STAGES = RES ? 2 : 3;
  static constexpr int RING_BYTES = STAGES * STAGE_BYTES;
  // K-residual table: [256 byte values][32 slices] floats
  static constexpr int LUT_FLOATS = LUT ? 256 * 32 : 0;
  // merge area: per warp and query row {m, l} + accRef[D] + accRes[D]; it
  // shares the table's space when there is one (never live at once)
  static constexpr int MERGE_FLOATS = kConsumerWarps * G * (2 + 2 * D);
  // ... and serves as scratch for the sequence-length scan of a
  // variable-length call before the first head
  static constexpr int AREA_0 = LUT_FLOATS > MERGE_FLOATS ? LUT_FLOATS : MERGE_FLOATS;
  static constexpr int AREA_FLOATS = AREA_0 > kVarlenMaxBatch + 4 ? AREA_0 : kVarlenMaxBatch + 4;
  static constexpr int QBUF_FLOATS = 2 * G * D;             // q and q~
  // bf16 query rows of the first heads of a CTA's run, fetched at the start
  static constexpr int QPRE_HEADS = 4;
  static constexpr int QPRE_BYTES = QPRE_HEADS * G * D * 2;
  static constexpr int SMEM_BYTES =
      RING_BYTES + 4 * (AREA_FLOATS + QBUF_FLOATS) + 2 * STAGES * 8 + 16 + QPRE_BYTES +
      STAGES * 8;   // + the stages' resolved rows
  static_assert(TPW % TPS == 0 && STEPS % CH == 0, "tile split");
  static_assert(G != 1 || CH == STEPS, "G == 1 processes a whole tile per chunk");
  static_assert(STAGE_BYTES % 16 == 0, "stage alignment");
};

// code c (already masked, left at its bit position) -> exact float
__device__ __forceinline__ float code_at(uint32_t masked) {
  return __uint_as_float(0x4B000000u | masked) - 8388608.0f;
}

// {a.x - b.x, a.y - b.y}, one paired instruction
__device__ __forceinline__ float2 sub2_rn(float2 a, float2 b) {
  float2 r;
  asm("{\n\t.reg .b64 ra, rb, rr;\n\tmov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "sub.rn.f32x2 rr, ra, rb;\n\tmov.b64 {%0, %1}, rr;\n\t}"
      : "=f"(r.x), "=f"(r.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return r;
}

// The lane's DPL codes as floats c_k * 2^pos_k (pos_k = the bit position the
// code sits at inside `x`, the lane's bits already shifted down to bit 0):
// each masked code ORed into the bit pattern of 2^23, then 2^23 subtracted
// (exact), two codes per paired subtraction.
template <int BITS, int DPL>
__device__ __forceinline__ void codes_positional(uint32_t x, float (&f)[DPL]) {
  constexpr uint32_t M = (1u << BITS) - 1u;
  uint32_t m[DPL];
  if constexpr (BITS * DPL > 16) {
    // 8 INT4 codes: split so no code sits above bit 16 (exactness needs < 2^23)
    const uint32_t lo = x & 0xFFFFu, hi = x >> 16;
#pragma unroll
    for (int k = 0; k < DPL / 2; ++k) {
      m[k] = lo & (M << (BITS * k));
      m[k + DPL / 2] = hi & (M << (BITS * k));
    }
  } else {
#pragma unroll
    for (int k = 0; k < DPL; ++k) m[k] = x & (M << (BITS * k));
  }
  const float2 big = make_float2(8388608.0f, 8388608.0f);
#pragma unroll
  for (int j = 0; j < DPL / 2; ++j) {
    const float2 v = sub2_rn(make_float2(__uint_as_float(0x4B000000u | m[2 * j]),
                                         __uint_as_float(0x4B000000u | m[2 * j + 1])),
                             big);
    f[2 * j] = v.x;
    f[2 * j + 1] = v.y;
  }
}

// 2^-pos of code k in codes_positional
template <int BITS, int DPL>
__host__ __device__ constexpr float pos_factor(int k) {
  return (BITS * DPL > 16) ? 1.0f / (float)(1u << (BITS * (k % (DPL / 2))))
                           : 1.0f / (float)(1u << (BITS * k));
}

template <int D, int G, int BITS>
__global__ void __launch_bounds__(kThreads, 2)
decode_kernel(const DecodeParams p) {
  using C = Cfg<D, G, BITS>;
  constexpr int DPL = C::DPL, LPT = C::LPT, TPS = C::TPS, TILE = C::TILE;
  constexpr int STAGES = C::STAGES, CH = C::CH;
  constexpr unsigned FULL = 0xffffffffu;
  constexpr int TOPLVL = C::RES ? (1 << BITS) - 1 : 0;
  constexpr int PB = C::RES ? BITS : 2;     // bit width used for position factors

  extern __shared__ __align__(128) unsigned char smem[];
  unsigned char* ring = smem;
  float* area = reinterpret_cast<float*>(smem + C::RING_BYTES);  // table / merge
  float* merge = area;
  float* lut = area;
  float* qbuf = area + C::AREA_FLOATS;
  uint64_t* full_bar = reinterpret_cast<uint64_t*>(qbuf + C::QBUF_FLOATS);
  uint64_t* empty_bar = full_bar + STAGES;
  volatile int* flags = reinterpret_cast<volatile int*>(empty_bar + STAGES);  // [0] abort, [1] last
  uint16_t* qpre = reinterpret_cast<uint16_t*>(
      reinterpret_cast<unsigned char*>(empty_bar + STAGES) + 16);      // [QPRE_HEADS][G][D]
  volatile unsigned long long* stage_row = reinterpret_cast<volatile unsigned long long*>(
      reinterpret_cast<unsigned char*>(qpre) + C::QPRE_BYTES);          // [STAGES], paged

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
  // dense calls of uniform length (the run depends on the arguments alone):
  // the first tiles of this CTA's run go into L2 while the previous grid
  // finishes, so that the ring fills from L2 once the wait returns
  if (warp == kConsumerWarps && lane == 0 && !p.ctx_lens && !p.page_table) {
    CallSplit sp;
    long long tb, te;
    TileCursor c;
    if (plan_cta(p, cta, nullptr, sp, tb, te, c)) {
      const int sb = (D / p.group) * 2;
      const long long npf = min(te - tb, (long long)kPrefetchTiles);
      for (long long i = 0; i < npf; ++i) {
        size_t row;
        const int n = c.n();
        if (n > 0 && tile_row(p, c, row)) {
          const size_t lo = (row * sb) & ~(size_t)15;
          const uint32_t nb = (uint32_t)(((row * sb + (size_t)n * sb + 15) & ~(size_t)15) - lo);
          if (tile_in_bounds(p, row, n, lo, nb, sb)) {
            bulk_prefetch_l2(p.ref_k + row * D, n * C::KROW);
            bulk_prefetch_l2(p.ref_v + row * D, n * C::KROW);
            if constexpr (C::RES) {
              bulk_prefetch_l2(p.codes_k + row * C::CWORDS, n * C::CROW);
              bulk_prefetch_l2(p.codes_v + row * C::CWORDS, n * C::CROW);
              bulk_prefetch_l2(reinterpret_cast<const unsigned char*>(p.scales_k) + lo, nb);
              bulk_prefetch_l2(reinterpret_cast<const unsigned char*>(p.scales_v) + lo, nb);
            }
          }
        }
        c.next(p);
      }
    }
  }
  pdl_wait_prev();     // inputs and workspace may come from the previous kernel

  // this CTA's run of tiles (the merge area is free scratch until the first head)
  CallSplit split;
  long long tile_begin, tile_end;
  TileCursor first_cur;
  if (!plan_cta(p, cta, reinterpret_cast<int*>(area), split, tile_begin, tile_end, first_cur))
    return;
  const int n_my = (int)(tile_end - tile_begin);
  const int SB = (D / p.group) * 2;     // scale bytes per token
  // bytes of the 16-byte-aligned run holding the scales of tokens [row, row + n)
  auto sc_bytes_ref = [&](size_t row, int n) {
    const size_t start = row * SB;
    return (uint32_t)(((start + (size_t)n * SB + 15) & ~(size_t)15) - (start & ~(size_t)15));
  };
  // scale bytes a stage holds (per array), for the bounds-checked build
  constexpr int SCAP = C::RES ? C::SC_BYTES : 0;
  // a tile's copies stay inside the call's arrays and the stage
  auto copies_in_bounds = [&](size_t row, int n) {
    const size_t lo = (row * SB) & ~(size_t)15;
    const uint32_t nb = sc_bytes_ref(row, n);
    return tile_in_bounds(p, row, n, lo, nb, SB) &&
           RQ_IN_BOUNDS(SCAP == 0 || (int)nb <= SCAP, p.status, kStatusBounds);
  };

  // ========================= producer warp ================================
  if (warp == kConsumerWarps) {
    if (lane == 0) {
      int issued = 0;
      TileCursor cur = first_cur;
      // paged caches: the next tile's page id is read one tile ahead, so its
      // latency overlaps the wait for a free stage
      int page_next = (p.page_table && n_my > 0) ? tile_page(p, cur) : 0;
      for (int i = 0; i < n_my; ++i) {
        const int s = i % STAGES;
        const TileCursor tc = cur;
        const int page = page_next;
        cur.next(p);
        if (p.page_table && i + 1 < n_my) page_next = tile_page(p, cur);
        if (i >= STAGES) {
          if (!mbar_wait_bounded(&empty_bar[s], ((i / STAGES) - 1) & 1)) {
            flag_error(p.status, 1u);
            flags[0] = 1;
            break;
          }
        }
        if (flags[0]) break;
        size_t row;
        const bool page_ok = p.page_table ? tile_row_page(p, tc, page, row) : tile_row(p, tc, row);
        if (!page_ok && tc.n() > 0) flag_error(p.status, 32u);
        const int n = page_ok ? tc.n() : 0;
        if (p.page_table) stage_row[s] = page_ok ? (unsigned long long)row : kBadRow;
        unsigned char* st = ring + s * C::STAGE_BYTES;
        if (n <= 0 || !copies_in_bounds(row, n)) {   // the empty tile of an empty sequence
          if (n > 0 && p.page_table) stage_row[s] = kBadRow;
          mbar_arrive(&full_bar[s]);
          ++issued;
          continue;
        }
        uint32_t bytes = 2u * n * C::KROW;
        size_t sc_lo = 0;
        uint32_t sc_bytes = 0;
        if constexpr (C::RES) {
          const size_t start = row * SB;
          sc_lo = start & ~(size_t)15;
          sc_bytes = (uint32_t)(((start + (size_t)n * SB + 15) & ~(size_t)15) - sc_lo);
          bytes += 2u * n * C::CROW + 2u * sc_bytes;
        }
        mbar_arrive_expect_tx(&full_bar[s], bytes);
        bulk_g2s(st + C::OFF_K, p.ref_k + row * D, n * C::KROW, &full_bar[s]);
        bulk_g2s(st + C::OFF_V, p.ref_v + row * D, n * C::KROW, &full_bar[s]);
        if constexpr (C::RES) {
          bulk_g2s(st + C::OFF_CK, p.codes_k + row * C::CWORDS, n * C::CROW, &full_bar[s]);
          bulk_g2s(st + C::OFF_CV, p.codes_v + row * C::CWORDS, n * C::CROW, &full_bar[s]);
          bulk_g2s(st + C::OFF_SK, reinterpret_cast<const unsigned char*>(p.scales_k) + sc_lo,
                   sc_bytes, &full_bar[s]);
          bulk_g2s(st + C::OFF_SV, reinterpret_cast<const unsigned char*>(p.scales_v) + sc_lo,
                   sc_bytes, &full_bar[s]);
        }
        ++issued;
      }
      // never leave with copies in flight into this CTA's shared memory
      for (int j = (issued > STAGES ? issued - STAGES : 0); j < issued; ++j)
        if (!mbar_wait_bounded(&full_bar[j % STAGES], (j / STAGES) & 1)) flag_error(p.status, 2u);
    }
    return;
  }

  // ========================= consumer warps ===============================
  // the query rows of the first heads of the run, while the first tiles are
  // in flight (made visible by the barrier that starts load_rotate_queries)
  const long long h_first = first_cur.hd;
  const int n_pre =
      (int)min((long long)C::QPRE_HEADS, (long long)p.batch * p.kv_heads - h_first);
  for (int e = tid; e < n_pre * G * D / 8; e += kConsumerThreads) {
    const int hh = e / (G * D / 8), rem = e % (G * D / 8);
    const long long hd = h_first + hh;
    const int b = (int)(hd / p.kv_heads), h = (int)(hd % p.kv_heads);
    if (RQ_IN_BOUNDS(hd >= 0 && hd < (long long)p.batch * p.kv_heads &&
                         (size_t)h * G + G <= (size_t)p.q_heads,
                     p.status, kStatusBounds))
      reinterpret_cast<uint4*>(qpre)[e] =
          reinterpret_cast<const uint4*>(p.q + ((size_t)b * p.q_heads + (size_t)h * G) * D)[rem];
  }

  const int li = lane % LPT;          // lane within its token
  const int slot = lane / LPT;        // token slot within a warp step
  const int dim0 = li * DPL;          // first dim this lane owns
  const float score_scale = p.score_scale;
  const int cw = (dim0 * PB) / 32;    // code word of this lane
  const int csh = (dim0 * PB) % 32;   // bit offset of the lane's codes in it
  constexpr int NP = DPL / 2;         // packed pairs per lane

  // table slices and byte selectors of this lane (G == 1, INT2): the lane's
  // 16 code bits are bytes 2*(li&1) and 2*(li&1)+1 of word cw, for slices
  // 2li and 2li+1.  The two token slots of a warp step read the slices in
  // opposite order so the 32 lanes hit 32 different banks.
  const int slice_a = 2 * li + (slot & 1);
  const int slice_b = 2 * li + 1 - (slot & 1);
  const uint32_t sel_a = 0x4440u | (uint32_t)(2 * (li & 1) + (slot & 1));
  const uint32_t sel_b = 0x4440u | (uint32_t)(2 * (li & 1) + 1 - (slot & 1));
  // with head_dim 64 there are 16 slices; slots 2 and 3 read a second copy
  const int lut_copy = (D == 64) ? 16 * ((slot >> 1) & 1) : 0;

  // per-lane constants of the current head (scores are accumulated without
  // the softmax scale, which multiplies each reduced score once)
  uint32_t qbf[G][NP];                // q as packed bf16 pairs
  float2 qc[G][NP];                   // 2 q~ 2^-pos (codes at their bit position)
  float qoff[G];                      // (2^b - 1) * sum q~ over the lane's dims
  // running state
  float m_run[G], l_run[G], wsum[G];
  float2 accV[G][NP], accC[G][NP];

  auto reset_state = [&]() {
#pragma unroll
    for (int r = 0; r < G; ++r) {
      m_run[r] = kNegInf;
      l_run[r] = 0.0f;
      wsum[r] = 0.0f;
#pragma unroll
      for (int j = 0; j < NP; ++j) {
        accV[r][j] = make_float2(0.0f, 0.0f);
        accC[r][j] = make_float2(0.0f, 0.0f);
      }
    }
  };

  // load and rotate the G query rows of head hd (and fill the K table);
  // all consumer threads
  auto setup_head = [&](long long hd) {
    float* qs = qbuf;              // [G][D] raw q
    float* qt = qbuf + G * D;      // [G][D] FWHT(D q)
    load_rotate_queries<D, G>(p, hd, qs, qt, tid,
                              hd - h_first < n_pre ? qpre + (hd - h_first) * G * D : nullptr);
    const float cd = rot_scale<D>();
    if constexpr (C::LUT) {
      // lut[byte][slice] = sum_k q~[4 slice + k] * l(c_k(byte)), l(c) = 2c - 3,
      // c_k = bits 2k..2k+1 of the byte.  Thread: slice = tid % S and
      // c0 = (tid / S) % 4 fixed; it writes the 64 bytes with that c0 (and,
      // for head_dim 64, a second copy at slice + 16).
      constexpr int S = D / 4;
      const int slice = tid % S;
      const int c0 = (tid / S) & 3;
      const int copy = (D == 64) ? 16 * ((tid / (4 * S)) & 1) : 0;
      float lv[4][4];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float qk = cd * qt[4 * slice + k];
#pragma unroll
        for (int c = 0; c < 4; ++c) lv[k][c] = qk * (float)(2 * c - 3);
      }
      const float base = (c0 == 0) ? lv[0][0] : (c0 == 1) ? lv[0][1] : (c0 == 2) ? lv[0][2] : lv[0][3];
#pragma unroll
      for (int n = 0; n < 64; ++n) {
        const float e = base + lv[1][n & 3] + lv[2][(n >> 2) & 3] + lv[3][n >> 4];
        lut[(c0 + 4 * n) * 32 + copy + slice] = e;
      }
      named_bar_sync(1, kConsumerThreads);
    }
#pragma unroll
    for (int r = 0; r < G; ++r) {
      float sum = 0.0f;
#pragma unroll
      for (int j = 0; j < NP; ++j) {
        const float q0 = qs[r * D + dim0 + 2 * j], q1 = qs[r * D + dim0 + 2 * j + 1];
        qbf[r][j] = (__float_as_uint(q0) >> 16) | (__float_as_uint(q1) & 0xFFFF0000u);
        const float t0 = cd * qt[r * D + dim0 + 2 * j];
        const float t1 = cd * qt[r * D + dim0 + 2 * j + 1];
        qc[r][j] = make_float2(2.0f * t0 * pos_factor<PB, DPL>(2 * j),
                               2.0f * t1 * pos_factor<PB, DPL>(2 * j + 1));
        sum += t0 + t1;
      }
      qoff[r] = (float)TOPLVL * sum;
    }
  };

  // merge the 4 warps' states, write the head's partial record, and if this
  // CTA is the last contributor, finish the head
  auto flush_head = [&](long long hd, long long first_tile, int nt_h) {
    // fold the token slots of the warp together
#pragma unroll
    for (int r = 0; r < G; ++r) {
      if constexpr (G == 1) {
        // every token's weight sits in two lanes (li, li ^ 1)
#pragma unroll
        for (int m = 1; m < 32; m <<= 1) l_run[r] += __shfl_xor_sync(FULL, l_run[r], m);
        l_run[r] *= 0.5f;
      } else {
#pragma unroll
        for (int m = LPT; m < 32; m <<= 1) l_run[r] += __shfl_xor_sync(FULL, l_run[r], m);
      }
#pragma unroll
      for (int m = LPT; m < 32; m <<= 1) {
        if constexpr (C::RES) wsum[r] += __shfl_xor_sync(FULL, wsum[r], m);
#pragma unroll
        for (int j = 0; j < NP; ++j) {
          accV[r][j].x += __shfl_xor_sync(FULL, accV[r][j].x, m);
          accV[r][j].y += __shfl_xor_sync(FULL, accV[r][j].y, m);
          if constexpr (C::RES) {
            accC[r][j].x += __shfl_xor_sync(FULL, accC[r][j].x, m);
            accC[r][j].y += __shfl_xor_sync(FULL, accC[r][j].y, m);
          }
        }
      }
    }
    named_bar_sync(1, kConsumerThreads);          // merge area (and table) free
    float* mw = merge + warp * G * (2 + 2 * D);
    if (slot == 0) {
#pragma unroll
      for (int r = 0; r < G; ++r) {
        float* rec = mw + r * (2 + 2 * D);
        if (li == 0) {
          rec[0] = m_run[r];
          rec[1] = l_run[r];
        }
#pragma unroll
        for (int j = 0; j < NP; ++j) {
          float z0 = 0.0f, z1 = 0.0f;        // rotated-domain part
          if constexpr (C::RES) {
            z0 = 2.0f * pos_factor<PB, DPL>(2 * j) * accC[r][j].x - (float)TOPLVL * wsum[r];
            z1 = 2.0f * pos_factor<PB, DPL>(2 * j + 1) * accC[r][j].y - (float)TOPLVL * wsum[r];
          }
          rec[2 + dim0 + 2 * j] = accV[r][j].x;
          rec[2 + dim0 + 2 * j + 1] = accV[r][j].y;
          rec[2 + D + dim0 + 2 * j] = z0;
          rec[2 + D + dim0 + 2 * j + 1] = z1;
        }
      }
    }
    named_bar_sync(1, kConsumerThreads);

    finish_head<D, G, C::RES>(p, hd, first_tile, nt_h, split, cta, merge, qbuf, flags, tid);
  };

  // <q, K row> of the lane's dims, straight from the packed bf16 row
  auto ref_dot = [&](const unsigned char* kp, int r) {
    float dot = 0.0f;
    if constexpr (DPL == 8) {
      const uint4 w = *reinterpret_cast<const uint4*>(kp);
      dot = fma_bf16x2(qbf[r][0], w.x, dot);
      dot = fma_bf16x2(qbf[r][1], w.y, dot);
      dot = fma_bf16x2(qbf[r][2], w.z, dot);
      dot = fma_bf16x2(qbf[r][3], w.w, dot);
    } else {
      const uint2 w = *reinterpret_cast<const uint2*>(kp);
      dot = fma_bf16x2(qbf[r][0], w.x, dot);
      dot = fma_bf16x2(qbf[r][1], w.y, dot);
    }
    return dot;
  };

  // the V row of the lane's dims as NP float pairs
  auto v_pairs = [&](const unsigned char* vp, float2 (&vf)[NP]) {
    if constexpr (DPL == 8) {
      const uint4 w = *reinterpret_cast<const uint4*>(vp);
      vf[0] = make_float2(bf16lo(w.x), bf16hi(w.x));
      vf[1] = make_float2(bf16lo(w.y), bf16hi(w.y));
      vf[2] = make_float2(bf16lo(w.z), bf16hi(w.z));
      vf[3] = make_float2(bf16lo(w.w), bf16hi(w.w));
    } else {
      const uint2 w = *reinterpret_cast<const uint2*>(vp);
      vf[0] = make_float2(bf16lo(w.x), bf16hi(w.x));
      vf[1] = make_float2(bf16lo(w.y), bf16hi(w.y));
    }
  };

  // the lane's codes as float pairs c * 2^pos
  auto code_pairs = [&](uint32_t word, float2 (&cf)[NP]) {
    float f[DPL];
    codes_positional<PB, DPL>(word >> csh, f);
#pragma unroll
    for (int j = 0; j < NP; ++j) cf[j] = make_float2(f[2 * j], f[2 * j + 1]);
  };

  auto rescale = [&](int r, float alpha) {
    const float2 a2 = make_float2(alpha, alpha);
    l_run[r] *= alpha;
    if constexpr (C::RES) wsum[r] *= alpha;
#pragma unroll
    for (int j = 0; j < NP; ++j) {
      accV[r][j] = __fmul2_rn(accV[r][j], a2);
      if constexpr (C::RES) accC[r][j] = __fmul2_rn(accC[r][j], a2);
    }
  };

  // adds weight pw of one token (lane's V row vf, codes word, scale s_v)
  auto accumulate_v = [&](int r, float pw, const float2 (&vf)[NP], const float2 (&cf)[NP],
                          float s_v) {
    const float2 p2 = make_float2(pw, pw);
#pragma unroll
    for (int j = 0; j < NP; ++j) accV[r][j] = __ffma2_rn(p2, vf[j], accV[r][j]);
    if constexpr (C::RES) {
      const float wv = pw * s_v;
      const float2 w2 = make_float2(wv, wv);
      wsum[r] += wv;
#pragma unroll
      for (int j = 0; j < NP; ++j) accC[r][j] = __ffma2_rn(w2, cf[j], accC[r][j]);
    }
  };

  // ---- one tile, single query row per kv head ----
  auto tile_g1 = [&](const unsigned char* st, int n, int sc_off, int grp) {
    float part[CH];
#pragma unroll
    for (int u = 0; u < CH; ++u) {
      const int tok = warp * C::TPW + u * TPS + slot;
      float dot = ref_dot(st + C::OFF_K + tok * C::KROW + dim0 * 2, 0);
      if constexpr (C::RES) {
        const uint32_t word = reinterpret_cast<const uint32_t*>(st + C::OFF_CK)[tok * C::CWORDS + cw];
        const float s_k = half_at(st + C::OFF_SK + sc_off + tok * SB + grp * 2);
        float res;
        if constexpr (C::LUT) {
          const uint32_t ba = __byte_perm(word, 0u, sel_a);
          const uint32_t bb = __byte_perm(word, 0u, sel_b);
          res = lut[ba * 32 + lut_copy + slice_a] + lut[bb * 32 + lut_copy + slice_b];
        } else {
          float2 cf[NP];
          code_pairs(word, cf);
          float2 acc = make_float2(-qoff[0], 0.0f);
#pragma unroll
          for (int j = 0; j < NP; ++j) acc = __ffma2_rn(qc[0][j], cf[j], acc);
          res = acc.x + acc.y;
        }
        dot = fmaf(s_k, res, dot);
      }
      part[u] = dot;
    }
    // reduce-scatter over the LPT lanes of a token: afterwards lane li holds
    // the full score of step li >> 1 (lanes li and li ^ 1 agree)
#pragma unroll
    for (int half = CH / 2, m = LPT / 2; half >= 1; half >>= 1, m >>= 1) {
      const bool upper = (li & m) != 0;
#pragma unroll
      for (int i = 0; i < half; ++i) {
        const float send = upper ? part[i] : part[i + half];
        const float keep = upper ? part[i + half] : part[i];
        part[i] = keep + __shfl_xor_sync(FULL, send, m);
      }
    }
    float sc = score_scale * (part[0] + __shfl_xor_sync(FULL, part[0], 1));
    const int own_tok = warp * C::TPW + (li >> 1) * TPS + slot;
    if (own_tok >= n) sc = kNegInf;
    // online softmax, base 2, rescaled lazily: the running max moves only when
    // a score exceeds it by more than kLazyMax, so weights stay <= 2^kLazyMax
    // and most tiles need one vote instead of a shuffle-max chain
    if (__any_sync(FULL, sc > m_run[0] + kLazyMax)) {
      float mc = sc;
#pragma unroll
      for (int m = 2; m < 32; m <<= 1) mc = fmaxf(mc, __shfl_xor_sync(FULL, mc, m));
      const float m_new = fmaxf(m_run[0], mc);
      rescale(0, (m_run[0] == kNegInf) ? 0.0f : exp2f(m_run[0] - m_new));
      m_run[0] = m_new;
    }
    const float pme = (sc == kNegInf) ? 0.0f : exp2f(sc - m_run[0]);
    l_run[0] += pme;
    // values
#pragma unroll
    for (int u = 0; u < CH; ++u) {
      const float pu = __shfl_sync(FULL, pme, slot * LPT + 2 * u);
      const int tok = warp * C::TPW + u * TPS + slot;
      if (tok < n) {
        float2 vf[NP], cf[NP];
        v_pairs(st + C::OFF_V + tok * C::KROW + dim0 * 2, vf);
        float s_v = 0.0f;
        if constexpr (C::RES) {
          code_pairs(reinterpret_cast<const uint32_t*>(st + C::OFF_CV)[tok * C::CWORDS + cw], cf);
          s_v = half_at(st + C::OFF_SV + sc_off + tok * SB + grp * 2);
        }
        accumulate_v(0, pu, vf, cf, s_v);
      }
    }
  };

  // ---- one tile, G query rows per kv head ----
  auto tile_gn = [&](const unsigned char* st, int n, int sc_off, int grp) {
#pragma unroll 1
    for (int c0 = 0; c0 < C::STEPS; c0 += CH) {
      float sc[G][CH];
#pragma unroll
      for (int u = 0; u < CH; ++u) {
        const int tok = warp * C::TPW + (c0 + u) * TPS + slot;
        const unsigned char* kp = st + C::OFF_K + tok * C::KROW + dim0 * 2;
        float dot[G];
#pragma unroll
        for (int r = 0; r < G; ++r) dot[r] = ref_dot(kp, r);
        if constexpr (C::RES) {
          const uint32_t word =
              reinterpret_cast<const uint32_t*>(st + C::OFF_CK)[tok * C::CWORDS + cw];
          const float s_k = half_at(st + C::OFF_SK + sc_off + tok * SB + grp * 2);
          float2 cf[NP];
          code_pairs(word, cf);
#pragma unroll
          for (int r = 0; r < G; ++r) {
            float2 acc = make_float2(-qoff[r], 0.0f);
#pragma unroll
            for (int j = 0; j < NP; ++j) acc = __ffma2_rn(qc[r][j], cf[j], acc);
            dot[r] = fmaf(s_k, acc.x + acc.y, dot[r]);
          }
        }
#pragma unroll
        for (int r = 0; r < G; ++r) {
#pragma unroll
          for (int m = 1; m < LPT; m <<= 1) dot[r] += __shfl_xor_sync(FULL, dot[r], m);
          sc[r][u] = (tok < n) ? score_scale * dot[r] : kNegInf;
        }
      }
      float pw[G][CH];
#pragma unroll
      for (int r = 0; r < G; ++r) {
        float mc = sc[r][0];
#pragma unroll
        for (int u = 1; u < CH; ++u) mc = fmaxf(mc, sc[r][u]);
#pragma unroll
        for (int m = LPT; m < 32; m <<= 1) mc = fmaxf(mc, __shfl_xor_sync(FULL, mc, m));
        const float m_new = fmaxf(m_run[r], mc);
        if (m_new != m_run[r]) {
          rescale(r, (m_run[r] == kNegInf) ? 0.0f : exp2f(m_run[r] - m_new));
          m_run[r] = m_new;
        }
#pragma unroll
        for (int u = 0; u < CH; ++u) {
          pw[r][u] = (sc[r][u] == kNegInf) ? 0.0f : exp2f(sc[r][u] - m_new);
          l_run[r] += pw[r][u];
        }
      }
#pragma unroll
      for (int u = 0; u < CH; ++u) {
        const int tok = warp * C::TPW + (c0 + u) * TPS + slot;
        if (tok < n) {
          float2 vf[NP], cf[NP];
          v_pairs(st + C::OFF_V + tok * C::KROW + dim0 * 2, vf);
          float s_v = 0.0f;
          if constexpr (C::RES) {
            code_pairs(reinterpret_cast<const uint32_t*>(st + C::OFF_CV)[tok * C::CWORDS + cw],
                       cf);
            s_v = half_at(st + C::OFF_SV + sc_off + tok * SB + grp * 2);
          }
#pragma unroll
          for (int r = 0; r < G; ++r) accumulate_v(r, pw[r][u], vf, cf, s_v);
        }
      }
    }
  };

  // ---- main loop over this CTA's tiles ----
  long long cur_head = -1, cur_first = 0;
  int cur_nt = 0;
  bool aborted = false;
  reset_state();
  TileCursor cur = first_cur;
  for (int i = 0; i < n_my; ++i) {
    const long long hd = cur.hd;
    size_t row = 0;
    int n = cur.n();
    if (!p.page_table) tile_row(p, cur, row);   // paged: the stage's row, below
    if (hd != cur_head) {
      if (cur_head >= 0) {
        flush_head(cur_head, cur_first, cur_nt);
        reset_state();
      }
      cur_head = hd;
      cur_first = cur.head_first();
      cur_nt = cur.nt;
      setup_head(hd);
    }
    cur.next(p);
    const int s = i % STAGES;
    bool ok = !aborted && !flags[0];
    if (ok) ok = mbar_wait_bounded(&full_bar[s], (i / STAGES) & 1);
    ok = __all_sync(FULL, ok);            // one decision per warp
    if (!ok) {
      if (!aborted && lane == 0) flag_error(p.status, 8u);
      aborted = true;
      flags[0] = 1;
    }
    if (!aborted && p.page_table) {
      const unsigned long long r = stage_row[s];   // written before the stage's arrive
      if (r == kBadRow) n = 0;
      else row = (size_t)r;
    }
    if (!aborted && n > 0) {
      const unsigned char* st = ring + s * C::STAGE_BYTES;
      const int sc_off = (int)((row * SB) & 15);
      const int grp = dim0 / p.group;
      // the consumers' stage reads: token rows < n, scales of n tokens
      if (!RQ_IN_BOUNDS(n <= TILE && (SCAP == 0 || sc_off + n * SB <= SCAP), p.status,
                        kStatusBounds))
        n = 0;
    }
    if (!aborted && n > 0) {
      const unsigned char* st = ring + s * C::STAGE_BYTES;
      const int sc_off = (int)((row * SB) & 15);
      const int grp = dim0 / p.group;
      if constexpr (G == 1) tile_g1(st, n, sc_off, grp);
      else tile_gn(st, n, sc_off, grp);
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty_bar[s]);
  }
  // After an abort the flush still runs (on whatever the state holds) so that
  // every consumer thread takes the same barrier sequence; the status word
  // marks the output invalid.
  if (cur_head >= 0) flush_head(cur_head, cur_first, cur_nt);
}

template <int D, int G, int BITS>
cudaError_t launch_decode_t(const DecodeParams& p, cudaStream_t stream) {
  using C = Cfg<D, G, BITS>;
  static bool attr_set = false;   // per process; harmless to repeat
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(decode_kernel<D, G, BITS>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         C::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  return launch_pdl(decode_kernel<D, G, BITS>, p.ctas, kThreads, C::SMEM_BYTES, stream, p);
}

template <int D, int G>
cudaError_t launch_decode_b(int bits, const DecodeParams& p, cudaStream_t stream) {
  if (bits == 2) return launch_decode_t<D, G, 2>(p, stream);
  if (bits == 4) return launch_decode_t<D, G, 4>(p, stream);
  if (bits == 16) return launch_decode_t<D, G, 16>(p, stream);
  return cudaErrorInvalidValue;
}

template <int D, int G>
cudaError_t launch_decode_g(int bits, const DecodeParams& p, cudaStream_t stream) {
  if (p.ref_bits == 0) return launch_decode_b<D, G>(bits, p, stream);
  // a compressed reference: the tensor-core kernel (rq_decode_cr1.cu)
  if (p.ref_bits == 8 || p.ref_bits == 4) return launch_decode_cr1(D, bits, p, stream);
  return cudaErrorInvalidValue;
}

template <int D>
cudaError_t launch_decode_d(int G, int bits, const DecodeParams& p, cudaStream_t stream) {
  if (G == 1) return launch_decode_g<D, 1>(bits, p, stream);
  return cudaErrorInvalidValue;     // grouped queries: rq_decode_gqa.cu
}

}  // namespace

cudaError_t launch_decode(int head_dim, int G, int bits, const DecodeParams& p,
                          cudaStream_t stream) {
  if (head_dim == 128) return launch_decode_d<128>(G, bits, p, stream);
  if (head_dim == 64) return launch_decode_d<64>(G, bits, p, stream);
  return cudaErrorInvalidValue;
}

}  // namespace rq
