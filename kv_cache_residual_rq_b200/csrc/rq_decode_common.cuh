// rq_decode_common.cuh -- pieces shared by the decode-attention kernels.
//
// Both decode kernels (the CUDA-core kernel for one query row per kv head and
// the tensor-core kernel for grouped queries) split a call the same way: the
// (head, tile) space is cut into equal runs, one per persistent CTA; at the
// end of a head's run the CTA's consumer warps leave their softmax states in
// shared memory and call finish_head, which writes the CTA's partial record
// and, in the last CTA to arrive for the head, merges all records and applies
// the inverse rotation once per output row.
#pragma once

#include <cmath>

#include "rq_device.cuh"
#include "rq_internal.h"

namespace rq {

constexpr int kConsumerWarps = 4;
constexpr int kConsumerThreads = kConsumerWarps * 32;
constexpr int kMergeChunk = 64;   // records whose weights the head merge stages at once
constexpr int kMergeFew = 8;      // default: up to this many records a head merge loads in one batch
constexpr int kPrefetchTiles = 2;   // tiles a CTA fetches into L2 before the grid-dependency wait
constexpr int kDecodeThreads = kConsumerThreads + 32;   // + one producer warp
constexpr float kNegInf = -INFINITY;
// lazy rescaling threshold of the online softmax (base-2 units)
constexpr float kLazyMax = 8.0f;

__device__ __forceinline__ void flag_error(uint32_t* status, uint32_t bit) {
  atomicOr(status, bit);
}

// fp16 value (bits in shared memory) as float
__device__ __forceinline__ float half_at(const unsigned char* p) {
  return __half2float(__ushort_as_half(*reinterpret_cast<const uint16_t*>(p)));
}

// ---------------------------------------------------------------------------
// Tile numbering of a call: heads hd = b * kv_heads + h in order, each head's
// tiles in token order.  A head of sequence b has nt_b tiles: p.nt for every
// sequence of a uniform call; max(1, ceil(len_b / 64)) with len_b =
// p.ctx_lens[b] clamped to [0, ctx_pitch] in a variable-length call (an empty
// sequence keeps one empty tile, so its heads are still finished from the
// tail).  A CTA walks its run of tiles with a cursor.
// ---------------------------------------------------------------------------
__device__ __forceinline__ int seq_len(const DecodeParams& p, int b) {
  if (!p.ctx_lens) return p.ctx;
  return min(max(p.ctx_lens[b], 0), p.ctx_pitch);
}

__device__ __forceinline__ int seq_tiles(const DecodeParams& p, int len) {
  return p.ctx_lens ? max(1, (len + kDecodeTile - 1) / kDecodeTile) : p.nt;
}

struct TileCursor {
  long long seq_first;   // number of the first tile of sequence b
  long long hd;          // head: b * kv_heads + h
  int b, h, j;           // sequence, kv head, tile within the head
  int nt, len;           // tiles per head and cached tokens of sequence b

  __device__ int t0() const { return j * kDecodeTile; }
  // tokens of the tile (0 for the empty tile of an empty sequence)
  __device__ int n() const { return min(kDecodeTile, len - j * kDecodeTile); }
  __device__ long long head_first() const { return seq_first + (long long)h * nt; }
  __device__ void next(const DecodeParams& p) {
    if (++j < nt) return;
    j = 0;
    ++hd;
    if (++h < p.kv_heads) return;
    h = 0;
    seq_first += (long long)p.kv_heads * nt;
    if (++b < p.batch) {
      len = seq_len(p, b);
      nt = seq_tiles(p, len);
    }
  }
};

// First row of the cursor's tile in the K/V, code and scale arrays.  Dense
// caches: head hd's token t0 is row hd * ctx_pitch + t0.  Paged caches (page
// = one 64-token tile): sequence b's tile j is page page_table[b][j] of a pool
// [pages][kv_heads][64][...], rows (page * kv_heads + h) * 64 ...  Returns
// false for a page id outside the pool; the caller then treats the tile as
// empty (and the producer raises status bit 32), so a bad table entry cannot
// address memory outside the pool.
// Paged caches: the page id of the cursor's tile (read ahead by the
// producer), and the row of a page id already read.
__device__ __forceinline__ int tile_page(const DecodeParams& p, const TileCursor& c) {
  if (!RQ_IN_BOUNDS(c.b < p.batch && c.j < p.max_pages, p.status, kStatusBounds)) return -1;
  return p.page_table[(size_t)c.b * p.max_pages + c.j];
}
__device__ __forceinline__ bool tile_row_page(const DecodeParams& p, const TileCursor& c,
                                              int page, size_t& row) {
  if (page < 0 || page >= p.n_pages) {
    row = 0;
    return false;
  }
  row = ((size_t)page * p.kv_heads + c.h) * kDecodeTile;
  return true;
}

__device__ __forceinline__ bool tile_row(const DecodeParams& p, const TileCursor& c,
                                         size_t& row) {
  if (!p.page_table) {
    row = (size_t)c.hd * p.ctx_pitch + c.t0();
    return true;
  }
  return tile_row_page(p, c, tile_page(p, c), row);
}

// Rows of the call's K/V, code and scale arrays: heads * ctx_pitch for dense
// caches, the pool's n_pages * kv_heads * 64 for paged ones.
__device__ __forceinline__ size_t call_rows(const DecodeParams& p) {
  return p.page_table ? (size_t)p.n_pages * p.kv_heads * kDecodeTile
                      : (size_t)p.batch * p.kv_heads * p.ctx_pitch;
}

// A tile's copies stay inside the call's arrays: tokens [row, row + n) and
// the 16-byte-aligned scale bytes [sc_lo, sc_lo + sc_bytes) of arrays of
// call_rows(p) rows of sb scale bytes each (sizes rounded up to 16 bytes).
__device__ __forceinline__ bool tile_in_bounds(const DecodeParams& p, size_t row, int n,
                                               size_t sc_lo, uint32_t sc_bytes, int sb) {
  const size_t rows = call_rows(p);
  const size_t sc_total = (rows * (size_t)sb + 15) / 16 * 16;
  return RQ_IN_BOUNDS(n >= 0 && n <= kDecodeTile && row + (size_t)n <= rows &&
                          sc_lo + sc_bytes <= sc_total,
                      p.status, kStatusBounds);
}

// A stage's row as the producer resolved it (paged caches), kBadRow for a
// page id outside the pool; the consumers read it after the stage's barrier
// instead of the page table.
constexpr unsigned long long kBadRow = ~0ull;

// The split of a call over its CTAs: n_tiles tiles in `ctas` equal runs.
struct CallSplit {
  long long n_tiles;
  int ctas;
};

// Work split and start cursor of this CTA.  Uniform calls: from the host's
// plan.  Variable-length calls: every CTA scans the sequence lengths (one
// warp, into `scratch`, which must hold batch + 1 ints and is free until the
// caller's next barrier-protected use), uses min(p.ctas, n_tiles) CTAs and
// finds the sequence of its first tile by binary search.  All threads of the
// CTA call it (it contains __syncthreads); returns false for a CTA without
// work.  Lengths outside [0, ctx_pitch] are clamped and raise status bit 16.
__device__ __forceinline__ bool plan_cta(const DecodeParams& p, int cta, int* scratch,
                                         CallSplit& split, long long& tile_begin,
                                         long long& tile_end, TileCursor& cur) {
  if (!p.ctx_lens) {
    split.n_tiles = p.n_tiles;
    split.ctas = p.ctas;
  } else {
    const int tid = threadIdx.x;
    // the scan writes batch + 1 ints of scratch (sized for kVarlenMaxBatch + 1)
    if (!RQ_IN_BOUNDS(p.batch <= kVarlenMaxBatch, p.status, kStatusBounds)) return false;
    if (tid < 32) {
      // exclusive prefix of per-head tile counts over the sequences
      const int per = (p.batch + 31) / 32;
      const int b0 = tid * per, b1 = min(p.batch, b0 + per);
      int sum = 0;
      bool bad = false;
      for (int b = b0; b < b1; ++b) {
        const int raw = p.ctx_lens[b];
        bad |= raw < 0 || raw > p.ctx_pitch;
        sum += seq_tiles(p, seq_len(p, b));
      }
      int incl = sum;
#pragma unroll
      for (int m = 1; m < 32; m <<= 1) {
        const int o = __shfl_up_sync(0xffffffffu, incl, m);
        if (tid >= m) incl += o;
      }
      int run = incl - sum;
      for (int b = b0; b < b1; ++b) {
        scratch[b] = run;
        run += seq_tiles(p, seq_len(p, b));
      }
      if (tid == 31) scratch[p.batch] = incl;
      if (__any_sync(0xffffffffu, bad) && tid == 0 && cta == 0) flag_error(p.status, 16u);
    }
    __syncthreads();
    split.n_tiles = (long long)p.kv_heads * scratch[p.batch];
    split.ctas = (int)min((long long)p.ctas, split.n_tiles);
  }
  if (cta >= split.ctas) return false;
  tile_begin = (long long)cta * split.n_tiles / split.ctas;
  tile_end = (long long)(cta + 1) * split.n_tiles / split.ctas;
  int b;
  long long seq_first;
  if (!p.ctx_lens) {
    const long long per_seq = (long long)p.kv_heads * p.nt;
    b = (int)(tile_begin / per_seq);
    seq_first = (long long)b * per_seq;
  } else {
    // last sequence whose first tile is <= tile_begin (prefixes strictly increase)
    int lo = 0, hi = p.batch - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if ((long long)p.kv_heads * scratch[mid] <= tile_begin) lo = mid; else hi = mid - 1;
    }
    b = lo;
    seq_first = (long long)p.kv_heads * scratch[b];
  }
  cur.b = b;
  cur.seq_first = seq_first;
  cur.len = seq_len(p, b);
  cur.nt = seq_tiles(p, cur.len);
  const long long rel = tile_begin - seq_first;
  cur.h = (int)(rel / cur.nt);
  cur.j = (int)(rel % cur.nt);
  cur.hd = (long long)b * p.kv_heads + cur.h;
  if (p.ctx_lens) __syncthreads();   // scratch free again
  return true;
}

// Walsh-Hadamard transform (no scaling) of a D-vector spread over a warp:
// lane owns coordinates lane*E .. lane*E+E-1, E = D/32.  Strides below E in
// registers, the rest by shfl.xor; ascending strides, butterfly (a+b, a-b).
template <int D>
__device__ __forceinline__ void warp_fwht(float (&v)[D / 32], int lane) {
  constexpr int E = D / 32;
#pragma unroll
  for (int h = 1; h < E; h <<= 1) {
#pragma unroll
    for (int k = 0; k < E; ++k) {
      if (!(k & h)) {
        const float a = v[k], c = v[k + h];
        v[k] = a + c;
        v[k + h] = a - c;
      }
    }
  }
#pragma unroll
  for (int m = 1; m < 32; m <<= 1) {
    const float sg = (lane & m) ? -1.0f : 1.0f;
#pragma unroll
    for (int k = 0; k < E; ++k) v[k] = fmaf(sg, v[k], __shfl_xor_sync(0xffffffffu, v[k], m));
  }
}

// Loads the G query rows of head hd into qs[G][D] (fp32) and FWHT(D q) into
// qt[G][D]: the rotation q~ = Rot q without its 1/sqrt(d) factor, which the
// caller applies.  qrows: the head's G bf16 rows if already in shared memory,
// else null (read from p.q).  One warp per row; all consumer threads call
// it, and it ends with a consumer barrier.
template <int D, int G>
__device__ __forceinline__ void load_rotate_queries(const DecodeParams& p, long long hd,
                                                    float* qs, float* qt, int tid,
                                                    const uint16_t* qrows = nullptr) {
  constexpr int E = D / 32;
  const int b = (int)(hd / p.kv_heads);
  const int h = (int)(hd % p.kv_heads);
  const int warp = tid >> 5, lane = tid & 31;
  // rows b * q_heads + h * G + r of q: inside the call's batch * q_heads rows
  const bool hd_ok = qrows || RQ_IN_BOUNDS(hd >= 0 && hd < (long long)p.batch * p.kv_heads &&
                                               (size_t)h * G + G <= (size_t)p.q_heads,
                                           p.status, kStatusBounds);
  named_bar_sync(1, kConsumerThreads);          // previous users of the buffers done
  const uint16_t* qbase = qrows ? qrows : p.q + ((size_t)b * p.q_heads + (size_t)h * G) * D;
  for (int r = warp; r < G; r += kConsumerWarps) {
    const uint16_t* qr = qbase + (size_t)r * D + lane * E;
    float v[E];
#pragma unroll
    for (int k = 0; k < E; ++k) {
      const float x = hd_ok ? __uint_as_float((uint32_t)qr[k] << 16) : 0.0f;
      qs[r * D + lane * E + k] = x;
      v[k] = flip_sign(x, sign_bit(p.seed, lane * E + k));
    }
    warp_fwht<D>(v, lane);
#pragma unroll
    for (int k = 0; k < E; ++k) qt[r * D + lane * E + k] = v[k];
  }
  named_bar_sync(1, kConsumerThreads);
}

// merge[w][r] = {m, l, accRef[D], accRes[D]} of consumer warp w and query row
// r (m in base-2 units, accRes in the rotated domain) must be complete and
// visible to all consumer threads.  Writes this CTA's record of head hd and,
// if it is the last CTA of the head to arrive, the head's output, after
// folding in the head's BF16 tail tokens (if any).  qs holds the head's raw
// query rows [G][D] as floats.  All consumer threads call it; `merge` is
// reused as scratch (it holds at least 4 G (2 + 2 D) floats).
template <int D, int G, bool RES, int FEW = kMergeFew>
__device__ __forceinline__ void finish_head(const DecodeParams& p, long long hd,
                                            long long first_tile, int nt_h,
                                            const CallSplit& split, int cta, float* merge,
                                            const float* qs, volatile int* flags, int tid) {
  static_assert(2 * G * D + 3 * G + G * RQ_MAX_TAIL <= 4 * G * (2 + 2 * D),
                "merge area too small for the tail scratch");
  const int b = (int)(hd / p.kv_heads);
  const int h = (int)(hd % p.kv_heads);
  // which records belong to this head, and which one is ours
  const long long f = first_tile, e = f + nt_h - 1;
  const int c_first = (int)(((f + 1) * split.ctas - 1) / split.n_tiles);
  const int c_last = (int)(((e + 1) * split.ctas - 1) / split.n_tiles);
  const int ncontrib = c_last - c_first + 1;
  const int j = cta - c_first;
  if (j < 0 || j >= p.max_contrib || ncontrib > p.max_contrib) {
    if (tid == 0) flag_error(p.status, 4u);
    return;
  }
  // head hd's records and counter, its output rows, its tail tokens and the
  // tail scratch (G * n_tail floats of the merge area)
  {
    const bool ok = hd >= 0 && hd < (long long)p.batch * p.kv_heads &&
                    (size_t)h * G + G <= (size_t)p.q_heads && p.n_tail >= 0 &&
                    p.n_tail <= RQ_MAX_TAIL && (p.n_tail == 0 || p.n_tail <= p.tail_pitch);
    if (!RQ_IN_BOUNDS(ok, p.status, kStatusBounds)) return;
  }
  float* recs = p.records + (size_t)hd * p.max_contrib * G * (4 + 2 * D);
  // per query row: the warps' common max and each warp's weight, once
  float* wts = const_cast<float*>(qs) + G * D;    // [G][1 + warps], the rotated-query buffer
  if (tid < G) {
    const int r = tid;
    float M = kNegInf;
#pragma unroll
    for (int w = 0; w < kConsumerWarps; ++w) M = fmaxf(M, merge[(w * G + r) * (2 + 2 * D)]);
    wts[r * (1 + kConsumerWarps)] = M;
#pragma unroll
    for (int w = 0; w < kConsumerWarps; ++w) {
      const float mw = merge[(w * G + r) * (2 + 2 * D)];
      wts[r * (1 + kConsumerWarps) + 1 + w] = (mw == kNegInf) ? 0.0f : exp2f(mw - M);
    }
  }
  named_bar_sync(1, kConsumerThreads);
  for (int eidx = tid; eidx < G * (2 * D + 2); eidx += kConsumerThreads) {
    const int r = eidx / (2 * D + 2), q = eidx % (2 * D + 2);
    const float* wr = wts + r * (1 + kConsumerWarps);
    float* out_rec = recs + ((size_t)j * G + r) * (4 + 2 * D);
    if (q == 0) {
      out_rec[0] = wr[0];
    } else {
      float acc = 0.0f;
#pragma unroll
      for (int w = 0; w < kConsumerWarps; ++w) acc += wr[1 + w] * merge[(w * G + r) * (2 + 2 * D) + q];
      out_rec[q == 1 ? 1 : q + 2] = acc;   // l at 1; accRef/accRes from 4
    }
  }
  named_bar_sync(1, kConsumerThreads);      // every record store of the CTA issued
  if (tid == 0) {
    // the barrier orders the other threads' record stores before this fence,
    // which makes them visible at GPU scope before the ticket (cumulativity)
    __threadfence();
    const uint32_t old = atomicAdd(&p.counters[hd], 1u);
    const int last = (old == (uint32_t)(ncontrib - 1));
    if (last) {
      p.counters[hd] = 0u;      // ready for the next call
      __threadfence();
    }
    flags[1] = last;
  }
  named_bar_sync(1, kConsumerThreads);
  if (!flags[1]) return;

  // ---- last contributor: merge all records of the head, finish ----
  // Every record load of a pass is independent of the others, so each pass
  // costs about one L2 round trip per batch of loads instead of one per
  // record.  Up to FEW records: each thread loads all of them for its
  // element at once (one round trip).  More: (1) the rows' maxima M_r over
  // the records, (2) per chunk of records their weights exp2(m_c - M_r) and
  // weighted sums l_c, (3) the weighted sums of the accumulators, eight
  // records per batch.
  float* zres = merge;               // [G][D] rotated-domain residual sums
  float* zref = merge + G * D;       // [G][D]
  float* lsum = merge + 2 * G * D;   // [G]
  float* mrow = lsum + G;            // [G] running max (base 2)
  float* arow = mrow + G;            // [G] rescale of the cached part
  float* tsc = arow + G;             // [G][n_tail] tail scores, then weights
  float* red = tsc + G * RQ_MAX_TAIL;            // [warps][G] partial maxima / sums
  float* wch = red + kConsumerWarps * G;         // [kMergeChunk][G] record weights
  float* lch = wch + kMergeChunk * G;            // [kMergeChunk][G] weight x l_c
  static_assert(2 * G * D + 3 * G + G * RQ_MAX_TAIL + kConsumerWarps * G + 2 * kMergeChunk * G <=
                    4 * G * (2 + 2 * D),
                "merge area too small for the merge scratch");
  static_assert(kConsumerThreads % G == 0, "a thread keeps one query row");
  const int warp_m = tid >> 5, lane_m = tid & 31;
  const int rr = tid % G;                        // the row of this thread's records
  constexpr int RSTEP = kConsumerThreads / G;    // records per pass of the threads
  auto rec = [&](int c, int r) { return recs + ((size_t)c * G + r) * (4 + 2 * D); };
  if (ncontrib <= FEW) {
#pragma unroll 1
    for (int eidx = tid; eidx < G * D; eidx += kConsumerThreads) {
      const int r = eidx / D, i = eidx % D;
      float mc[FEW], lc[FEW], va[FEW], vr[FEW];
#pragma unroll
      for (int u = 0; u < FEW; ++u) {
        mc[u] = kNegInf;
        lc[u] = va[u] = vr[u] = 0.0f;
        if (u < ncontrib) {
          const float* rc = rec(u, r);
          mc[u] = __ldcg(rc);
          lc[u] = __ldcg(rc + 1);
          va[u] = __ldcg(rc + 4 + i);
          if constexpr (RES) vr[u] = __ldcg(rc + 4 + D + i);
        }
      }
      float M = kNegInf;
#pragma unroll
      for (int u = 0; u < FEW; ++u) M = fmaxf(M, mc[u]);
      float l = 0.0f, aref = 0.0f, ares = 0.0f;
#pragma unroll
      for (int u = 0; u < FEW; ++u) {
        if (mc[u] != kNegInf) {          // a record without tokens weighs 0
          const float wgt = exp2f(mc[u] - M);
          l = fmaf(wgt, lc[u], l);
          aref = fmaf(wgt, va[u], aref);
          if constexpr (RES) ares = fmaf(wgt, vr[u], ares);
        }
      }
      zref[eidx] = aref;
      zres[eidx] = ares;
      if (i == 0) {
        lsum[r] = l;
        mrow[r] = M;
      }
    }
  } else {
    // (1) M_r
    {
      float pm = kNegInf;
      for (int c = tid / G; c < ncontrib; c += RSTEP) pm = fmaxf(pm, __ldcg(rec(c, rr)));
  #pragma unroll
      for (int m = G; m < 32; m <<= 1) pm = fmaxf(pm, __shfl_xor_sync(0xffffffffu, pm, m));
      if (lane_m < G) red[warp_m * G + lane_m] = pm;
      named_bar_sync(1, kConsumerThreads);
      if (tid < G) {
        float M = kNegInf;
  #pragma unroll
        for (int w = 0; w < kConsumerWarps; ++w) M = fmaxf(M, red[w * G + tid]);
        mrow[tid] = M;
      }
      named_bar_sync(1, kConsumerThreads);
    }
    float lpart = 0.0f;                            // threads tid < G: l of row tid
    for (int c0 = 0; c0 < ncontrib; c0 += kMergeChunk) {
      const int nc = min(kMergeChunk, ncontrib - c0);
      // (2) the chunk's weights; a record without tokens (m = -inf) weighs 0
      for (int e = tid; e < nc * G; e += kConsumerThreads) {
        const int c = c0 + e / G, r = e % G;
        const float* rc = rec(c, r);
        const float mc = __ldcg(rc), lc = __ldcg(rc + 1);
        const float wgt = (mc == kNegInf) ? 0.0f : exp2f(mc - mrow[r]);
        wch[e] = wgt;
        lch[e] = (mc == kNegInf) ? 0.0f : wgt * lc;
      }
      named_bar_sync(1, kConsumerThreads);
      if (tid < G)
        for (int cc = 0; cc < nc; ++cc) lpart += lch[cc * G + tid];
      // (3) the accumulators, eight records per batch of loads
  #pragma unroll 1
      for (int eidx = tid; eidx < G * D; eidx += kConsumerThreads) {
        const int r = eidx / D, i = eidx % D;
        float aref = 0.0f, ares = 0.0f;
        int cc = 0;
        for (; cc + 8 <= nc; cc += 8) {
          float va[8], vr[8];
  #pragma unroll
          for (int u = 0; u < 8; ++u) {
            const float* rc = rec(c0 + cc + u, r);
            va[u] = __ldcg(rc + 4 + i);
            vr[u] = RES ? __ldcg(rc + 4 + D + i) : 0.0f;
          }
  #pragma unroll
          for (int u = 0; u < 8; ++u) {
            const float wgt = wch[(cc + u) * G + r];
            if (wgt != 0.0f) {
              aref = fmaf(wgt, va[u], aref);
              if constexpr (RES) ares = fmaf(wgt, vr[u], ares);
            }
          }
        }
        for (; cc < nc; ++cc) {
          const float* rc = rec(c0 + cc, r);
          const float wgt = wch[cc * G + r];
          const float va = __ldcg(rc + 4 + i);
          const float vr = RES ? __ldcg(rc + 4 + D + i) : 0.0f;
          if (wgt != 0.0f) {
            aref = fmaf(wgt, va, aref);
            if constexpr (RES) ares = fmaf(wgt, vr, ares);
          }
        }
        zref[eidx] = c0 ? zref[eidx] + aref : aref;
        zres[eidx] = c0 ? zres[eidx] + ares : ares;
      }
      named_bar_sync(1, kConsumerThreads);      // the chunk's weights may be overwritten
    }
    if (tid < G) lsum[tid] = lpart;
  }
  const int nt = p.n_tail;
  if (nt > 0) {
    // BF16 tail tokens of this head (not encoded yet): same base-2 scores,
    // merged into the running state before the normalisation
    const size_t tail0 = (size_t)hd * p.tail_pitch;
    named_bar_sync(1, kConsumerThreads);
    {
      // one warp per (query row, tail token): lane-parallel dot product
      constexpr int E = D / 32;
      const int warp = tid >> 5, lane = tid & 31;
      for (int e = warp; e < G * nt; e += kConsumerWarps) {
        const int r = e / nt, jt = e % nt;
        const uint16_t* kr = p.tail_k + (tail0 + jt) * D + lane * E;
        float acc = 0.0f;
#pragma unroll
        for (int k = 0; k < E; ++k)
          acc = fmaf(qs[r * D + lane * E + k], __uint_as_float((uint32_t)kr[k] << 16), acc);
#pragma unroll
        for (int m = 16; m >= 1; m >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, m);
        if (lane == 0) tsc[e] = p.score_scale * acc;
      }
    }
    named_bar_sync(1, kConsumerThreads);
    if (tid < G) {
      const int r = tid;
      float mt = mrow[r];
      for (int jt = 0; jt < nt; ++jt) mt = fmaxf(mt, tsc[r * nt + jt]);
      const float alpha = (mrow[r] == kNegInf) ? 0.0f : exp2f(mrow[r] - mt);
      float l = lsum[r] * alpha;
      for (int jt = 0; jt < nt; ++jt) {
        const float w = exp2f(tsc[r * nt + jt] - mt);
        tsc[r * nt + jt] = w;
        l += w;
      }
      lsum[r] = l;
      mrow[r] = mt;
      arow[r] = alpha;
    }
    named_bar_sync(1, kConsumerThreads);
    for (int eidx = tid; eidx < G * D; eidx += kConsumerThreads) {
      const int r = eidx / D, i = eidx % D;
      float aref = zref[eidx] * arow[r];
      for (int jt = 0; jt < nt; ++jt)
        aref = fmaf(tsc[r * nt + jt], __uint_as_float((uint32_t)p.tail_v[(tail0 + jt) * D + i] << 16),
                    aref);
      zref[eidx] = aref;
      if constexpr (RES) zres[eidx] *= arow[r];
    }
  }
  // out = (zref + Rot^T zres) / l, Rot^T z = D (c_d H z): one warp per row
  named_bar_sync(1, kConsumerThreads);
  {
    constexpr int E = D / 32;
    const int warp = tid >> 5, lane = tid & 31;
    const float cd = rot_scale<D>();
    for (int r = warp; r < G; r += kConsumerWarps) {
      float z[E];
#pragma unroll
      for (int k = 0; k < E; ++k) z[k] = RES ? zres[r * D + lane * E + k] : 0.0f;
      if constexpr (RES) warp_fwht<D>(z, lane);
      const float inv_l = 1.0f / lsum[r];
      float o[E];
#pragma unroll
      for (int k = 0; k < E; ++k) {
        float num = zref[r * D + lane * E + k];
        if constexpr (RES) num += flip_sign(cd * z[k], sign_bit(p.seed, lane * E + k));
        o[k] = num * inv_l;
      }
      float* dst = p.out + ((size_t)b * p.q_heads + (size_t)h * G + r) * D + lane * E;
      if constexpr (E == 4)
        *reinterpret_cast<float4*>(dst) = make_float4(o[0], o[1], o[2], o[3]);
      else
        *reinterpret_cast<float2*>(dst) = make_float2(o[0], o[1]);
    }
  }
}

}  // namespace rq
