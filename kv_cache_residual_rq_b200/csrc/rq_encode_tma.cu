// rq_encode_tma.cu -- ResidualQuant encoder fed by the tensor-copy engine.
//
// Method: "ResidualQuant: KV Cache Quantization for Looped Transformers with
// 2-Bit Residuals", Abstract -- each non-final loop is stored as its residual
// against the final-loop reference, rotated, and quantised per group to INT2
// (INT4 where the loop is given more bits) with a least-squares scale.  The
// codes are the same bits as those of the streaming encoder (rq_encode.cu):
// identical binary32 operations in the identical order.
//
// Used when every source array is a contiguous [rows][head_dim] block (the
// whole-cache encode).  This file holds the plain mode (absmax codes, one
// least-squares scale); the refit and compressed-reference modes, whose
// scales must follow the specification's summation order, are in
// rq_encode_tma_fixed.cu.  One CTA per SM:
//   * a producer warp streams tiles of R rows -- the reference tile, then the
//     same rows of every quantised loop -- into a ring of shared-memory slots
//     with 2-D tensor copies (128-byte swizzle), completion on mbarriers;
//   * a consumer lane owns 64 consecutive coordinates of a row (two lanes per
//     row at head_dim 128, one at 64), as 32 packed pairs {c_m, c_m+32}.
// Per lane and loop: residual and seeded sign in one mixed bf16 x bf16 + f32
// fma per coordinate (D_i x_i + (-D_i ref_i), exact product, one rounding);
// the Walsh-Hadamard strides 1..16 as packed fp32x2 adds and subtracts,
// stride 32 inside each pair, stride 64 (head_dim 128) by shfl.xor; the
// lane's two 32-wide blocks are the two scale groups of 32 (or together one
// of 64), quantised side by side as packed pairs; codes from floor(u)
// obtained as (u + 1.5*2^23) rounded down, whose bit pattern is 0x4B400000 +
// floor(u), packed by shifted adds with one constant correction per word;
// the least-squares numerator <y, l> = 2 <y, floor(u)> + sum y, the block's
// sum y taken from four unrotated coordinates (no level per coordinate).
// Every wait is bounded; on a timeout the kernel raises a bit in the encoder
// status word and stops.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <cstring>
#include <mutex>

#include "rq_device.cuh"
#include "rq_encode_tma_common.cuh"
#include "rq_internal.h"

namespace rq {

// sticky encoder error bits of this device (read and cleared by the host)
__device__ uint32_t g_encode_status;

namespace {

using namespace enc;

// consumer warps per CTA (+ 1 producer warp) and ring slots
template <int D>
constexpr int consumer_warps() { return D == 128 ? 11 : 8; }
template <int D>
constexpr int ring_slots() { return D == 128 ? 5 : 6; }

template <int D, int CW>
struct ECfg {
  static constexpr int LPR = D / 64;                // lanes per row, 64 coordinates each
  static constexpr int RPW = 32 / LPR;              // rows per consumer warp
  static constexpr int R = CW * RPW;                // rows per tile
  static constexpr int NBOX = D / 64;               // 64-column boxes per row
  static constexpr int BOX_BYTES = R * 128;
  static constexpr int SLOT_BYTES = NBOX * BOX_BYTES;
  static constexpr int SLOTS = ring_slots<D>();
  static constexpr int THREADS = (CW + 1) * 32;
  static constexpr int SMEM = 1024 + SLOTS * SLOT_BYTES + 2 * (D / 2) * 4 + 2 * SLOTS * 8;
  static_assert(R <= 256, "tensor-copy box is at most 256 rows");
  static_assert(SMEM <= 232448, "shared memory of one CTA");
};

// The lane's 64 coordinates of row r (q: which half of a 128-wide row), as
// P[m] = {c_m, c_{m+32}}: chunk c of the row's 128-byte box line holds
// coordinates 8c .. 8c+7, so P[m].x comes from chunk m/8 and P[m].y from
// chunk m/8 + 4.  For each coordinate i: out_i = a_i * b_i + add_i, a the
// slot's bf16 row, b the lane's bf16 sign words (word k = coordinates 2k,
// 2k+1), add the float2 addends in the same layout (or zero).
template <int D, int CW, bool ADD>
__device__ __forceinline__ void row_fma(const uint8_t* slot, const uint32_t* signs, int r, int q,
                                        const float2 (&add)[32], float2 (&P)[32]) {
  using C = ECfg<D, CW>;
  const uint8_t* rp = slot + q * C::BOX_BYTES + r * 128;
  const uint4* s4 = reinterpret_cast<const uint4*>(signs + 32 * q);
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    const uint4 v = *reinterpret_cast<const uint4*>(rp + ((c ^ (r & 7)) << 4));
    const uint4 dd = s4[c];
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    const uint32_t dw[4] = {dd.x, dd.y, dd.z, dd.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int i = 8 * c + 2 * k + h;            // coordinate within the lane's 64
        const int m = i & 31;
        const float a = ADD ? ((i < 32) ? add[m].x : add[m].y) : 0.0f;
        const float o = h ? fma_bf16<1>(w[k], dw[k], a) : fma_bf16<0>(w[k], dw[k], a);
        if (i < 32) P[m].x = o; else P[m].y = o;
      }
    }
  }
}

// The lane's 64 coordinates (signs applied) rotated in place: Walsh-Hadamard
// strides ascending, each butterfly (a + b, a - b) one rounded operation --
// strides 1..16 as packed pairs, 32 inside each pair, 64 (head_dim 128) with
// the partner lane -- then x c_d.
template <int D, int RPW>
__device__ __forceinline__ void rotate64(float2 (&P)[32], int q) {
#pragma unroll
  for (int h = 1; h < 32; h <<= 1) {
#pragma unroll
    for (int m = 0; m < 32; ++m) {
      if (!(m & h)) {
        const float2 a = P[m], b = P[m + h];
        P[m] = __fadd2_rn(a, b);
        P[m + h] = fsub2(a, b);
      }
    }
  }
#pragma unroll
  for (int m = 0; m < 32; ++m) {
    const float a = P[m].x, b = P[m].y;
    P[m] = make_float2(__fadd_rn(a, b), __fsub_rn(a, b));
  }
  if constexpr (D == 128) {
    // the lower partner keeps a + b, the upper one a - b (fma with +-1 is
    // exactly one rounded add or subtract)
    const float sg = q ? -1.0f : 1.0f;
    const float2 sg2 = make_float2(sg, sg);
#pragma unroll
    for (int m = 0; m < 32; ++m) {
      float2 o;
      o.x = __shfl_xor_sync(kFull, P[m].x, RPW);
      o.y = __shfl_xor_sync(kFull, P[m].y, RPW);
      P[m] = __ffma2_rn(sg2, P[m], o);
    }
  }
  const float cd = rot_scale<D>();
  const float2 cd2 = make_float2(cd, cd);
#pragma unroll
  for (int m = 0; m < 32; ++m) P[m] = __fmul2_rn(P[m], cd2);
}

// Sum of the rotated coordinates over each of the lane's two 32-wide blocks,
// taken from the unrotated ones.  In the Sylvester Hadamard matrix H the rows
// 32a .. 32a + 31 (block a) sum to 32 (-1)^popcount(a & (j >> 5)) in the
// columns j that are multiples of 32 and to zero in every other column, so
// sum over block a of y = 32 c_d sum_j' (-1)^popcount(a & j') x_(32 j'): the
// lane's x_0 and x_32 and, at head_dim 128, its partner's.  It differs from
// the sum of the computed y by the rotation's roundings (a few units in the
// last place of sum |y|), which the least-squares scale, kept as fp16, does
// not see.
template <int D, int RPW>
__device__ __forceinline__ float2 block_sums(const float2 (&P)[32], int q) {
  float2 a = make_float2(P[0].x + P[0].y, P[0].x - P[0].y);
  if constexpr (D == 128) {
    const float sg = q ? -1.0f : 1.0f;
    float2 o;
    o.x = __shfl_xor_sync(kFull, a.x, RPW);
    o.y = __shfl_xor_sync(kFull, a.y, RPW);
    a = make_float2(fmaf(sg, a.x, o.x), fmaf(sg, a.y, o.y));
  }
  const float k = 32.0f * rot_scale<D>();
  return make_float2(k * a.x, k * a.y);
}

// One quantisation pass over the lane's two 32-coordinate blocks, A = P[].x
// and B = P[].y, with steps 1/(2 inv.x), 1/(2 inv.y): code words (A's BITS
// words, then B's), <y,f> with f = floor(u) and <l,l> of each block (.x,
// .y).  With l = 2 f + 1, <y,l> = 2 <y,f> + sum y, and the caller supplies
// sum y; the scale is kept only as its fp16 rounding, so <y,f> runs as four
// interleaved chains; code words are integer sums (any order).
template <int BITS>
__device__ __forceinline__ void quant_pass(const float2 (&P)[32], float2 inv2,
                                           uint32_t (&w)[2 * BITS], float2& dot_out,
                                           float2& nrm_out) {
  constexpr int PER = 32 / BITS;                    // codes per word
  const float2 mg = make_float2(kFloorMagic, kFloorMagic);
  constexpr int NC = 4;                             // independent chains
  float2 dot[NC], nrm[NC];
#pragma unroll
  for (int c = 0; c < NC; ++c) {
    dot[c] = make_float2(0.0f, 0.0f);
    nrm[c] = make_float2(0.0f, 0.0f);
  }
#pragma unroll
  for (int k = 0; k < 2 * BITS; ++k) w[k] = 0;
#pragma unroll
  for (int m = 0; m < 32; ++m) {
    const int c = m % NC;
    const float2 u = __fmul2_rn(P[m], inv2);
    const float2 t = __fadd2_rd(u, mg);             // 1.5*2^23 + floor(u), exact
    w[m / PER] += __float_as_uint(t.x) << (BITS * (m % PER));
    w[BITS + m / PER] += __float_as_uint(t.y) << (BITS * (m % PER));
    const float2 fl = fsub2(t, mg);                 // floor(u); level 2 floor(u) + 1
    dot[c] = __ffma2_rn(P[m], fl, dot[c]);
    if constexpr (BITS != 2) nrm[c] = __ffma2_rn(fl, fl, nrm[c]);
  }
  // every field received (0x4B400000 + floor(u)); code c = floor(u) + 2^(b-1)
  constexpr uint32_t kOff = kFloorMagicBits - (1u << (BITS - 1));
  constexpr uint32_t kSpread = BITS == 2 ? 0x55555555u : 0x11111111u;
#pragma unroll
  for (int k = 0; k < 2 * BITS; ++k) w[k] -= kOff * kSpread;
  dot_out = __fadd2_rn(__fadd2_rn(dot[0], dot[1]), __fadd2_rn(dot[2], dot[3]));
  if constexpr (BITS == 2) {
    // <l, l> = 32 + 8 * (number of outer levels +-3, i.e. codes 0 and 3,
    // whose two bits are equal): an exact integer
    const uint32_t ea = __popc(~(w[0] ^ (w[0] >> 1)) & 0x55555555u) +
                        __popc(~(w[1] ^ (w[1] >> 1)) & 0x55555555u);
    const uint32_t eb = __popc(~(w[2] ^ (w[2] >> 1)) & 0x55555555u) +
                        __popc(~(w[3] ^ (w[3] >> 1)) & 0x55555555u);
    nrm_out = make_float2((float)(32u + 8u * ea), (float)(32u + 8u * eb));
  } else {
    // <l, l> = 4 (sum f^2 + sum f) + 32, sum f = sum c - 8 * 32 from the code
    // words; integers below 2^24 in every partial sum: exact in any order
    auto csum = [](uint32_t x) {
      const uint32_t b = (x & 0x0F0F0F0Fu) + ((x >> 4) & 0x0F0F0F0Fu);
      return (b * 0x01010101u) >> 24;
    };
    const int fa = (int)(csum(w[0]) + csum(w[1]) + csum(w[2]) + csum(w[3])) - 256;
    const int fb = (int)(csum(w[4]) + csum(w[5]) + csum(w[6]) + csum(w[7])) - 256;
    const float2 sq = __fadd2_rn(__fadd2_rn(nrm[0], nrm[1]), __fadd2_rn(nrm[2], nrm[3]));
    nrm_out = make_float2(4.0f * (sq.x + (float)fa) + 32.0f, 4.0f * (sq.y + (float)fb) + 32.0f);
  }
}

__device__ __forceinline__ float2 f2(float x) { return make_float2(x, x); }

// Codes and scales of the lane's 64 rotated coordinates: blocks A (P[].x)
// and B (P[].y) are one 32-wide scale group each, or together one group of
// 64; ysum = sum y over each block.  The absmax step, then the least-squares
// scale of those codes.
template <int BITS, int GROUP>
__device__ __forceinline__ void quantize_store(const float2 (&P)[32], float2 ysum,
                                               uint32_t* codes_row, uint16_t* scales_row, int q,
                                               bool valid) {
  // absmax of each block as four interleaved chains (max is exact in any order)
  float ax[4], ay[4];
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    ax[c] = fmax3_abs(0.0f, P[2 * c].x, P[2 * c + 1].x);
    ay[c] = fmax3_abs(0.0f, P[2 * c].y, P[2 * c + 1].y);
  }
#pragma unroll
  for (int m = 8; m < 32; m += 2) {
    const int c = (m / 2) % 4;
    ax[c] = fmax3_abs(ax[c], P[m].x, P[m + 1].x);
    ay[c] = fmax3_abs(ay[c], P[m].y, P[m + 1].y);
  }
  float amx = fmaxf(fmaxf(ax[0], ax[1]), fmaxf(ax[2], ax[3]));
  float amy = fmaxf(fmaxf(ay[0], ay[1]), fmaxf(ay[2], ay[3]));
  if constexpr (GROUP == 64) amx = amy = fmaxf(amx, amy);
  constexpr float outer = (float)(1 << (BITS - 1)) - 0.5f;
  float2 inv;
  inv.x = (amx < 1.17549435e-38f) ? 0.0f : __fdiv_rn(outer, amx);
  inv.y = (GROUP == 64) ? inv.x : ((amy < 1.17549435e-38f) ? 0.0f : __fdiv_rn(outer, amy));
  uint32_t w[2 * BITS];
  float2 d, n;
  quant_pass<BITS>(P, inv, w, d, n);
  d = make_float2(fmaf(2.0f, d.x, ysum.x), fmaf(2.0f, d.y, ysum.y));   // <y, l>
  if constexpr (GROUP == 64) {
    d = f2(d.x + d.y);                              // block A + block B
    n = f2(n.x + n.y);
  }
  // least-squares scale; only its fp16 rounding is kept, so the fast
  // reciprocal division serves
  float2 s;
  s.x = __fdividef(d.x, n.x);
  s.y = (GROUP == 64) ? s.x : __fdividef(d.y, n.y);
  s.x = fminf(fmaxf(s.x, -65504.0f), 65504.0f);
  s.y = fminf(fmaxf(s.y, -65504.0f), 65504.0f);
  const __half hx = __float2half_rn(s.x), hy = __float2half_rn(s.y);
  if (!valid) return;
  uint4* o = reinterpret_cast<uint4*>(codes_row + 2 * BITS * q);
#pragma unroll
  for (int k = 0; k < 2 * BITS / 4; ++k)
    o[k] = make_uint4(w[4 * k], w[4 * k + 1], w[4 * k + 2], w[4 * k + 3]);
  if constexpr (GROUP == 32)
    *reinterpret_cast<uint32_t*>(scales_row + 2 * q) =
        (uint32_t)__half_as_ushort(hx) | ((uint32_t)__half_as_ushort(hy) << 16);
  else
    scales_row[q] = __half_as_ushort(hx);
}

// The plain mode: BF16 reference, absmax codes, one least-squares scale.
template <int D, int GROUP, int CW>
__global__ void __launch_bounds__(ECfg<D, CW>::THREADS, 1)
encode_tma_kernel(const __grid_constant__ EncodeTmaParams tp) {
  using C = ECfg<D, CW>;
  constexpr int SLOTS = C::SLOTS;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* ring = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint32_t* dtab = reinterpret_cast<uint32_t*>(ring + SLOTS * C::SLOT_BYTES);  // D_i as bf16 pairs
  uint32_t* ndtab = dtab + D / 2;                                            // -D_i
  uint64_t* full = reinterpret_cast<uint64_t*>(ndtab + D / 2);
  uint64_t* empty = full + SLOTS;
  const EncodeParams& p = tp.p;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  pdl_allow_next();

  for (int i = threadIdx.x; i < D / 2; i += blockDim.x) {
    const uint32_t lo = sign_bit(p.seed, 2 * i) ? 0xBF80u : 0x3F80u;
    const uint32_t hi = sign_bit(p.seed, 2 * i + 1) ? 0xBF80u : 0x3F80u;
    dtab[i] = lo | (hi << 16);
    ndtab[i] = dtab[i] ^ 0x80008000u;
  }
  if (threadIdx.x == 0) {
    for (int s = 0; s < SLOTS; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], CW);
    }
    fence_mbar_init();
  }
  __syncthreads();
  pdl_wait_prev();     // the sources may come from the previous kernel

  const int per_tile = 1 + tp.n_active;
  if (warp == CW) {
    // ---------------- producer ----------------
    if (lane != 0) return;
    long long it = 0;
    bool ok = true;
    for (int t = blockIdx.x; ok && t < tp.n_tiles; t += gridDim.x) {
      for (int j = 0; j < per_tile; ++j, ++it) {
        const int s = (int)(it % SLOTS);
        // the tile's first row lies inside the sources (the tensor maps zero-fill
        // the rows of a partial tile past the end)
        (void)RQ_IN_BOUNDS((long long)t * C::R < p.n_rows && j < RQ_MAX_LOOPS + 1, p.status,
                           kEncodeStatusBounds);
        if (it >= SLOTS && !mbar_wait_bounded(&empty[s], (uint32_t)((it / SLOTS - 1) & 1))) {
          atomicOr(&g_encode_status, 1u);
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(&full[s], C::SLOT_BYTES);
#pragma unroll
        for (int b = 0; b < C::NBOX; ++b)
          tma_load_2d(ring + s * C::SLOT_BYTES + b * C::BOX_BYTES, &tp.maps[j], 64 * b,
                      t * C::R, &full[s]);
      }
    }
    // do not leave while copies into this CTA's shared memory are in flight
    for (long long k = (it > SLOTS ? it - SLOTS : 0); k < it; ++k)
      if (!mbar_wait_bounded(&full[k % SLOTS], (uint32_t)((k / SLOTS) & 1)))
        atomicOr(&g_encode_status, 2u);
    return;
  }

  // ---------------- consumers ----------------
  const int rw = lane % C::RPW;          // row within the warp
  const int q = lane / C::RPW;           // which 64 coordinates of the row
  const int r = warp * C::RPW + rw;      // row within the tile
  // shared-memory reads of this lane: line r of box q of a slot
  if (!RQ_IN_BOUNDS(r < C::R && q < C::NBOX, p.status, kEncodeStatusBounds)) return;
  long long it = 0;
  for (int t = blockIdx.x; t < tp.n_tiles; t += gridDim.x) {
    const long long idx = (long long)t * C::R + r;
    // idx < n_tiles * R <= kEncodeTmaMaxRows + R < 2^31: a 32-bit division
    const uint32_t hd32 = (uint32_t)idx / (uint32_t)p.ctx;
    const long long hd = hd32, tok = idx - (long long)hd32 * p.ctx;
    long long row = 0;
    bool valid = idx < p.n_rows && enc_dst_row(p, hd, tok, row);
    // every output of the row (codes, scales, reference copy) is written at
    // destination row `row`
    if (valid)
      valid = RQ_IN_BOUNDS(row >= 0 && row < p.n_dst_rows, p.status, kEncodeStatusBounds);

    // reference: -D_i ref_i, kept for every loop of these rows
    int s = (int)(it % SLOTS);
    if (!mbar_wait_bounded(&full[s], (uint32_t)((it / SLOTS) & 1))) {
      atomicOr(&g_encode_status, 4u);
      return;
    }
    const uint8_t* slot = ring + s * C::SLOT_BYTES;
    if (valid && p.ref_out) {
      const uint8_t* rp = slot + q * C::BOX_BYTES + r * 128;
      uint4* o = reinterpret_cast<uint4*>(p.ref_out + (size_t)row * D + q * 64);
#pragma unroll
      for (int c = 0; c < 8; ++c) o[c] = *reinterpret_cast<const uint4*>(rp + ((c ^ (r & 7)) << 4));
    }
    float2 zr[32];
    row_fma<D, CW, false>(slot, ndtab, r, q, zr, zr);
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);
    ++it;

    for (int j = 0; j < tp.n_active; ++j) {
      s = (int)(it % SLOTS);
      if (!mbar_wait_bounded(&full[s], (uint32_t)((it / SLOTS) & 1))) {
        atomicOr(&g_encode_status, 4u);
        return;
      }
      // y = D_i x_i + (-D_i ref_i), one rounding, then rotated
      float2 P[32];
      row_fma<D, CW, true>(ring + s * C::SLOT_BYTES, dtab, r, q, zr, P);
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);
      ++it;
      const float2 ysum = block_sums<D, C::RPW>(P, q);
      rotate64<D, C::RPW>(P, q);
      const int l = tp.active[j];
      if (p.bits[l] == 2)
        quantize_store<2, GROUP>(P, ysum, p.codes[l] + (size_t)row * (D / 16),
                                 p.scales[l] + (size_t)row * (D / GROUP), q, valid);
      else
        quantize_store<4, GROUP>(P, ysum, p.codes[l] + (size_t)row * (D / 8),
                                 p.scales[l] + (size_t)row * (D / GROUP), q, valid);
    }
  }
}

template <int D, int GROUP>
cudaError_t launch_t(const EncodeTmaParams& tp, int num_sms, cudaStream_t stream) {
  constexpr int CW = consumer_warps<D>();
  using C = ECfg<D, CW>;
  cudaError_t e = cudaFuncSetAttribute(encode_tma_kernel<D, GROUP, CW>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
  if (e != cudaSuccess) return e;
  const int grid = tp.n_tiles < num_sms ? tp.n_tiles : num_sms;
  return launch_pdl(encode_tma_kernel<D, GROUP, CW>, (unsigned)grid, C::THREADS, C::SMEM, stream,
                    tp);
}

}  // namespace

int encode_tma_rows_per_tile(int head_dim) {
  return head_dim == 128 ? ECfg<128, consumer_warps<128>()>::R : ECfg<64, consumer_warps<64>()>::R;
}

cudaError_t launch_encode_tma(int head_dim, int group, const EncodeParams& p, int num_sms,
                              cudaStream_t stream) {
  // least-squares refits and the compressed reference: rq_encode_tma_fixed.cu
  if (p.ref_bits != 0 || p.refine_iters > 0)
    return launch_encode_tma_fixed(head_dim, group, p, num_sms, stream);
  EncodeTmaParams tp;
  std::memset(&tp, 0, sizeof tp);
  tp.p = p;
  const int R = encode_tma_rows_per_tile(head_dim);
  tp.n_tiles = (int)((p.n_rows + R - 1) / R);
  if (!encode_rows_map(&tp.maps[0], p.ref, (unsigned long long)p.n_rows, head_dim, R))
    return cudaErrorInvalidValue;
  for (int l = 0; l < p.n_loops; ++l) {
    if (p.bits[l] == 16) continue;
    if (!encode_rows_map(&tp.maps[1 + tp.n_active], p.x[l], (unsigned long long)p.n_rows,
                         head_dim, R))
      return cudaErrorInvalidValue;
    tp.active[tp.n_active++] = l;
  }
  if (head_dim == 128 && group == 32) return launch_t<128, 32>(tp, num_sms, stream);
  if (head_dim == 128 && group == 64) return launch_t<128, 64>(tp, num_sms, stream);
  if (head_dim == 64 && group == 32) return launch_t<64, 32>(tp, num_sms, stream);
  if (head_dim == 64 && group == 64) return launch_t<64, 64>(tp, num_sms, stream);
  return cudaErrorInvalidValue;
}

uint32_t* encode_status_ptr() {
  constexpr int kMaxDevices = 64;
  static uint32_t* addr[kMaxDevices] = {nullptr};
  static std::mutex mu;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (!addr[dev]) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_encode_status) != cudaSuccess) return nullptr;
    addr[dev] = static_cast<uint32_t*>(ptr);
  }
  return addr[dev];
}

cudaError_t encode_take_status(uint32_t* bits) {
  uint32_t zero = 0;
  cudaError_t e = cudaMemcpyFromSymbol(bits, g_encode_status, sizeof(uint32_t));
  if (e != cudaSuccess) return e;
  return cudaMemcpyToSymbol(g_encode_status, &zero, sizeof(uint32_t));
}

}  // namespace rq
