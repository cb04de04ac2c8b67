// rq_decode_tc.cuh -- pieces shared by the tensor-core decode kernels: the
// grouped-query kernel (rq_decode_gqa.cuh) and the single-query kernel over a
// compressed reference (rq_decode_cr1.cu).
//
// Both run the same tile pipeline: one producer warp fills a ring of stages
// (reference K/V tiles by TMA tensor copies with the swizzle of their line
// width, codes and scales by bulk copies), four consumer warps take a stage
// each per tile, 16 tokens per warp, and hand it back.  Every mbarrier wait
// is bounded; a wait that runs out raises the workspace status word and the
// kernel still finishes (its output is then invalid).
#pragma once

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>

#include "rq_decode_common.cuh"

namespace rq {

struct alignas(64) TcParams {
  CUtensorMap tmap_k;        // reference K: BF16 rows (box 64 x 64) or code rows (whole rows)
  CUtensorMap tmap_v;
  DecodeParams p;
};

// ---- PTX wrappers -----------------------------------------------------------


__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int x, int y,
                                            uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

__device__ __forceinline__ void ldsm_x2(uint32_t addr, uint32_t (&r)[2]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.shared.b16 {%0, %1}, [%2];"
               : "=r"(r[0]), "=r"(r[1])
               : "r"(addr));
}

__device__ __forceinline__ void ldsm_x2_trans(uint32_t addr, uint32_t (&r)[2]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.trans.shared.b16 {%0, %1}, [%2];"
               : "=r"(r[0]), "=r"(r[1])
               : "r"(addr));
}

__device__ __forceinline__ void ldsm_x4_trans(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

// D(16x8, f32) += A(16x16) B(16x8); A row-major, B column-major fragments.
__device__ __forceinline__ void mma_bf16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, "
      "{%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// the same with f16 operands
__device__ __forceinline__ void mma_f16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                        uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, "
      "{%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Byte offset of 16-byte chunk `chunk` of row `row` in a tile of rows of
// RROW bytes (32, 64 or 128) written by a TMA copy with the swizzle of that
// width: address bits 4.. are XORed with bits 7.. (3 bits for 128 B, 2 for
// 64 B, 1 for 32 B).
template <int RROW>
__device__ __forceinline__ uint32_t swz_offset(int row, int chunk) {
  static_assert(RROW == 32 || RROW == 64 || RROW == 128, "swizzle width");
  const uint32_t o = (uint32_t)(row * RROW + chunk * 16);
  constexpr uint32_t mask = RROW / 16 - 1;
  return o ^ (((o >> 7) & mask) << 4);
}


// {lo, hi} -> packed bf16x2 / f16x2 (round to nearest)
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}
__device__ __forceinline__ uint32_t badd2_u(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("add.rn.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}
__device__ __forceinline__ float bf16_lo_f(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi_f(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// {lo, hi} as a bf16 pair h plus a bf16 pair of remainders r, lo ~ h.lo + r.lo
__device__ __forceinline__ void split_bf16(float lo, float hi, uint32_t& h, uint32_t& r) {
  h = pack_bf16(lo, hi);
  r = pack_bf16(lo - bf16_lo_f(h), hi - bf16_hi_f(h));
}

__device__ __forceinline__ uint32_t pack_f16(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}
__device__ __forceinline__ float f16_lo_f(uint32_t w) {
  return __half2float(__ushort_as_half((unsigned short)(w & 0xFFFFu)));
}
__device__ __forceinline__ float f16_hi_f(uint32_t w) {
  return __half2float(__ushort_as_half((unsigned short)(w >> 16)));
}
// {lo, hi} as an f16 pair h plus an f16 pair of remainders r
__device__ __forceinline__ void split_f16(float lo, float hi, uint32_t& h, uint32_t& r) {
  h = pack_f16(lo, hi);
  r = pack_f16(lo - f16_lo_f(h), hi - f16_hi_f(h));
}

constexpr uint32_t kMagic = 0x43004300u;   // bf16 128.0 in both halves (mantissa unit 1)

// D(16x8, s32) += A(16x32, u8) B(32x8, s8); A row-major, B column-major
// fragments (a0: row g, bytes k = 4t .. 4t+3; a1: row g + 8; a2, a3: k + 16;
// b0: k = 4t .. 4t+3 of column g, b1: k + 16; g = lane / 4, t = lane % 4).
__device__ __forceinline__ void mma_u8s8(int (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0, %1, %2, %3}, "
      "{%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
      : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// The same with a signed A (s8) and an unsigned B (u8).
__device__ __forceinline__ void mma_s8u8(int (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.s8.u8.s32 {%0, %1, %2, %3}, "
      "{%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
      : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// {a.lo * b.lo, a.hi * b.hi} in f16
__device__ __forceinline__ uint32_t hmul2_u(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}

// ---- the tile pipeline --------------------------------------------------------

// Dense calls of uniform length (the CTA's run depends on the arguments
// alone): the first tiles of the run go into L2 before the grid-dependency
// wait, so that the ring fills from L2 once the previous grid has finished.
// Called by one lane.
template <class C, int D>
__device__ __forceinline__ void prefetch_first_tiles(const DecodeParams& p, int cta) {
  if (p.ctx_lens || p.page_table) return;
  CallSplit sp;
  long long tb, te;
  TileCursor c;
  if (!plan_cta(p, cta, nullptr, sp, tb, te, c)) return;
  constexpr int SB = C::SB;
  const long long npf = min(te - tb, (long long)kPrefetchTiles);
  for (long long i = 0; i < npf; ++i, c.next(p)) {
    size_t row;
    const int n = c.n();
    if (n <= 0 || !tile_row(p, c, row)) continue;
    const size_t lo = (row * SB) & ~(size_t)15;
    const uint32_t nb = (uint32_t)(((row * SB + (size_t)n * SB + 15) & ~(size_t)15) - lo);
    if (!tile_in_bounds(p, row, n, lo, nb, SB)) continue;
    if constexpr (C::CRX) {
      bulk_prefetch_l2(reinterpret_cast<const unsigned char*>(p.rcodes_k) + row * C::RROW,
                       n * C::RROW);
      bulk_prefetch_l2(reinterpret_cast<const unsigned char*>(p.rcodes_v) + row * C::RROW,
                       n * C::RROW);
      bulk_prefetch_l2(reinterpret_cast<const unsigned char*>(p.rscales_k) + lo, nb);
      bulk_prefetch_l2(reinterpret_cast<const unsigned char*>(p.rscales_v) + lo, nb);
    } else {
      bulk_prefetch_l2(p.ref_k + row * D, n * 2 * D);
      bulk_prefetch_l2(p.ref_v + row * D, n * 2 * D);
    }
    if constexpr (C::RES) {
      bulk_prefetch_l2(p.codes_k + row * C::CWORDS, n * C::CROW);
      bulk_prefetch_l2(p.codes_v + row * C::CWORDS, n * C::CROW);
      bulk_prefetch_l2(reinterpret_cast<const unsigned char*>(p.scales_k) + lo, nb);
      bulk_prefetch_l2(reinterpret_cast<const unsigned char*>(p.scales_v) + lo, nb);
    }
  }
}

// Producer warp (lane 0 issues): fills stage i % STAGES with tile i of the
// CTA's run once the consumers have released it.  C: the kernel's stage
// layout (STAGES, STAGE_BYTES, REF_TILE_BYTES, OFF_*, CROW, CWORDS, SB, RES,
// CRX, NBOX, BOX_BYTES).  scap: scale bytes a stage holds per array.
template <class C>
__device__ __forceinline__ void tile_producer(const TcParams& gp, unsigned char* ring,
                                              uint64_t* full_bar, uint64_t* empty_bar,
                                              volatile int* flags,
                                              volatile unsigned long long* stage_row,
                                              TileCursor cur, int n_my, int scap) {
  const DecodeParams& p = gp.p;
  constexpr int STAGES = C::STAGES, SB = C::SB;
  int issued = 0;
  // paged caches: the next tile's page id is read one tile ahead
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
    // a tile's copies stay inside the call's arrays and the stage
    bool in_bounds = false;
    if (n > 0) {
      const size_t start = row * SB;
      const size_t lo = start & ~(size_t)15;
      const uint32_t nb = (uint32_t)(((start + (size_t)n * SB + 15) & ~(size_t)15) - lo);
      in_bounds = tile_in_bounds(p, row, n, lo, nb, SB) &&
                  RQ_IN_BOUNDS(scap == 0 || (int)nb <= scap, p.status, kStatusBounds);
    }
    if (n <= 0 || !in_bounds) {   // the empty tile of an empty sequence
      if (n > 0 && p.page_table) stage_row[s] = kBadRow;
      mbar_arrive(&full_bar[s]);
      ++issued;
      continue;
    }
    uint32_t bytes = 2u * C::REF_TILE_BYTES;          // full boxes, OOB rows zero-filled
    size_t sc_lo = 0;
    uint32_t sc_bytes = 0;
    if constexpr (C::RES || C::CRX) {
      const size_t start = row * SB;
      sc_lo = start & ~(size_t)15;
      sc_bytes = (uint32_t)(((start + (size_t)n * SB + 15) & ~(size_t)15) - sc_lo);
    }
    if constexpr (C::RES) bytes += 2u * n * C::CROW + 2u * sc_bytes;
    if constexpr (C::CRX) bytes += 2u * sc_bytes;
    mbar_arrive_expect_tx(&full_bar[s], bytes);
    if constexpr (C::CRX) {
      // one box of whole code rows each
      tma_load_2d(st + C::OFF_K, &gp.tmap_k, 0, (int)row, &full_bar[s]);
      tma_load_2d(st + C::OFF_V, &gp.tmap_v, 0, (int)row, &full_bar[s]);
      bulk_g2s(st + C::OFF_RSK, reinterpret_cast<const unsigned char*>(p.rscales_k) + sc_lo,
               sc_bytes, &full_bar[s]);
      bulk_g2s(st + C::OFF_RSV, reinterpret_cast<const unsigned char*>(p.rscales_v) + sc_lo,
               sc_bytes, &full_bar[s]);
    } else {
#pragma unroll
      for (int bx = 0; bx < C::NBOX; ++bx) {
        tma_load_2d(st + C::OFF_K + bx * C::BOX_BYTES, &gp.tmap_k, 64 * bx, (int)row,
                    &full_bar[s]);
        tma_load_2d(st + C::OFF_V + bx * C::BOX_BYTES, &gp.tmap_v, 64 * bx, (int)row,
                    &full_bar[s]);
      }
    }
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
  for (int j = (issued > STAGES ? issued - STAGES : 0); j < issued; ++j)
    if (!mbar_wait_bounded(&full_bar[j % STAGES], (j / STAGES) & 1)) flag_error(p.status, 2u);
}

// Consumer warps: walk the CTA's run of tiles.  At a head change the
// previous head is flushed (flush_head(hd, first_tile, nt)), the state reset
// and the new head set up (setup_head(hd)); each stage is waited for (bounded;
// after a wait that runs out the warp stops computing but keeps the barrier
// sequence), its row resolved (paged caches), its reads checked, and
// tile(stage, n, sc_off) called for a non-empty tile; the stage is then
// released.  The last head is flushed at the end, after an abort too, so
// that every consumer thread takes the same barrier sequence.
template <class C, class Setup, class Flush, class Reset, class Tile>
__device__ __forceinline__ void consume_tiles(const DecodeParams& p, unsigned char* ring,
                                              uint64_t* full_bar, uint64_t* empty_bar,
                                              volatile int* flags,
                                              volatile unsigned long long* stage_row,
                                              TileCursor cur, int n_my, int scap,
                                              Setup&& setup_head, Flush&& flush_head,
                                              Reset&& reset_state, Tile&& tile) {
  constexpr int STAGES = C::STAGES, SB = C::SB;
  const int lane = threadIdx.x & 31;
  long long cur_head = -1, cur_first = 0;
  int cur_nt = 0;
  bool aborted = false;
  reset_state();
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
    ok = __all_sync(0xffffffffu, ok);      // one decision per warp
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
    // the consumers' stage reads: token rows < n, scales of n tokens
    if (!aborted && n > 0 &&
        !RQ_IN_BOUNDS(n <= C::TILE && (scap == 0 || (int)((row * SB) & 15) + n * SB <= scap),
                      p.status, kStatusBounds))
      n = 0;
    if (!aborted && n > 0) tile(ring + s * C::STAGE_BYTES, n, (int)((row * SB) & 15));
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty_bar[s]);
  }
  if (cur_head >= 0) flush_head(cur_head, cur_first, cur_nt);
}

}  // namespace rq
