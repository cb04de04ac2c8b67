// rq_encode_tma_fixed.cu -- the tensor-copy encoder's least-squares-refit
// and compressed-reference modes.
//
// Method: "ResidualQuant: KV Cache Quantization for Looped Transformers with
// 2-Bit Residuals", Abstract -- each non-final loop is stored as its residual
// against the final-loop reference, rotated, and quantised per group with a
// least-squares scale.  In these two modes a scale's bits decide later bits
// (the next refit's codes; the reconstruction every loop's residual is taken
// against), so every <y,l> is summed in the fixed order of the specification
// and divided in IEEE binary32.  The plain mode (rq_encode_tma.cu) gives each
// lane 64 coordinates; these modes hold more state per lane and measure
// faster with 32, on 15 consumer warps:
//   * a producer warp streams tiles of R rows -- the reference tile, then the
//     same rows of every quantised loop -- into a ring of shared-memory slots
//     with 2-D tensor copies (128-byte swizzle), completion on mbarriers;
//   * each consumer warp owns 8 rows (head_dim 128; 16 rows for 64) of the
//     tile, 4 (2) lanes per row, 32 consecutive coordinates per lane, so a
//     scale group of 32 is one lane and needs no cross-lane reduction.
// Per lane and loop: residual and seeded sign in one mixed bf16 x bf16 + f32
// fma per coordinate; the Walsh-Hadamard stages 1..16 in registers as packed
// fp32x2 adds and subtracts (stage 16 scalar), stages 32 and 64 by shfl.xor;
// codes from floor(u) obtained as (u + 1.5*2^23) rounded down.  Every wait is
// bounded; on a timeout the kernel raises a bit in the encoders' status word
// (p.status) and stops.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <cstring>

#include "rq_device.cuh"
#include "rq_encode_tma_common.cuh"
#include "rq_internal.h"

namespace rq {

namespace {

constexpr int kSlots = 6;
using namespace enc;

template <int D, int CW>
struct ECfg {
  static constexpr int LPR = D / 32;                // lanes per row
  static constexpr int RPW = 32 / LPR;              // rows per consumer warp
  static constexpr int R = CW * RPW;                // rows per tile
  static constexpr int NBOX = D / 64;               // 64-column boxes per row
  static constexpr int BOX_BYTES = R * 128;
  static constexpr int SLOT_BYTES = NBOX * BOX_BYTES;
  static constexpr int THREADS = (CW + 1) * 32;
  static constexpr int SMEM = 1024 + kSlots * SLOT_BYTES + 2 * (D / 2) * 4 + 2 * kSlots * 8;
  static_assert(R <= 256, "tensor-copy box is at most 256 rows");
};

// 32 bf16 of one lane: row r of the slot, 16-byte chunks c0 .. c0+3 of box b
template <int D, int CW>
__device__ __forceinline__ void load_row(const uint8_t* slot, int r, int q, uint32_t (&w)[16]) {
  using C = ECfg<D, CW>;
  const int b = (D == 128) ? (q >> 1) : 0;
  const int c0 = (D == 128) ? (q & 1) * 4 : q * 4;
  const uint8_t* rp = slot + b * C::BOX_BYTES + r * 128;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint4 v = *reinterpret_cast<const uint4*>(rp + (((c0 + i) ^ (r & 7)) << 4));
    w[4 * i] = v.x;
    w[4 * i + 1] = v.y;
    w[4 * i + 2] = v.z;
    w[4 * i + 3] = v.w;
  }
}

// One quantisation pass of a lane's 32 rotated coordinates P[m] = {y_m,
// y_{m+16}} with step 1/(2 inv): packed code words, <y,l> in the fixed order
// (fma chains over coordinates 0..15 and 16..31, the two runs added; the
// partner lane's block added for groups of 64) and <l,l> (exact).
template <int BITS, int GROUP, int RPW, bool CLAMP, bool WANT_LV = false>
__device__ __forceinline__ void quant_pass(const float2 (&P)[16], float inv, uint32_t (&w)[BITS],
                                           float& dot_out, float& nrm_out,
                                           float2* lv_out = nullptr) {
  const float2 inv2 = make_float2(inv, inv);
  const float2 mg = make_float2(kFloorMagic, kFloorMagic);
  const float2 two = make_float2(2.0f, 2.0f), one = make_float2(1.0f, 1.0f);
  constexpr float lo = kFloorMagic - (float)(1 << (BITS - 1));
  constexpr float hi = kFloorMagic + (float)((1 << (BITS - 1)) - 1);
  float2 dot = make_float2(0.0f, 0.0f), nrm = make_float2(0.0f, 0.0f);
#pragma unroll
  for (int k = 0; k < BITS; ++k) w[k] = 0;
#pragma unroll
  for (int m = 0; m < 16; ++m) {
    const float2 u = __fmul2_rn(P[m], inv2);
    float2 t = __fadd2_rd(u, mg);                   // 1.5*2^23 + floor(u), exact
    if constexpr (CLAMP) {
      t.x = fminf(fmaxf(t.x, lo), hi);
      t.y = fminf(fmaxf(t.y, lo), hi);
    }
    if constexpr (BITS == 2) {
      w[0] += __float_as_uint(t.x) << (2 * m);
      w[1] += __float_as_uint(t.y) << (2 * m);
    } else if constexpr (BITS == 4) {
      w[m / 8] += __float_as_uint(t.x) << (4 * (m % 8));
      w[2 + m / 8] += __float_as_uint(t.y) << (4 * (m % 8));
    } else {
      w[m / 4] += __float_as_uint(t.x) << (8 * (m % 4));
      w[4 + m / 4] += __float_as_uint(t.y) << (8 * (m % 4));
    }
    const float2 fl = fsub2(t, mg);                 // floor(u)
    const float2 lv = __ffma2_rn(fl, two, one);     // level 2 floor(u) + 1 = 2c - (2^b - 1)
    if constexpr (WANT_LV) lv_out[m] = lv;
    dot = __ffma2_rn(P[m], lv, dot);
    if constexpr (BITS != 2) nrm = __ffma2_rn(lv, lv, nrm);
  }
  // every field received (0x4B400000 + floor(u)); code c = floor(u) + 2^(b-1)
  constexpr uint32_t kOff = kFloorMagicBits - (1u << (BITS - 1));
  constexpr uint32_t kSpread =
      BITS == 2 ? 0x55555555u : (BITS == 4 ? 0x11111111u : 0x01010101u);
#pragma unroll
  for (int k = 0; k < BITS; ++k) w[k] -= kOff * kSpread;
  float d = dot.x + dot.y, n;
  if constexpr (BITS == 2) {
    // <l, l> = 32 + 8 * (number of outer levels +-3, i.e. codes 0 and 3,
    // whose two bits are equal): an exact integer either way
    const uint32_t e = __popc(~(w[0] ^ (w[0] >> 1)) & 0x55555555u) +
                       __popc(~(w[1] ^ (w[1] >> 1)) & 0x55555555u);
    n = (float)(32u + 8u * e);
  } else {
    n = nrm.x + nrm.y;
  }
  if (GROUP == 64) {
    d += __shfl_xor_sync(kFull, d, RPW);
    n += __shfl_xor_sync(kFull, n, RPW);
  }
  dot_out = d;
  nrm_out = n;
}

// codes and scale of one lane's 32 rotated coordinates: the absmax step,
// then `iters` least-squares refits (nearest level of the current scale,
// then the scale refitted); a group whose scale is below FLT_MIN keeps its
// codes.  The loop runs the same number of times in every lane.
template <int BITS, int GROUP, int RPW, bool WANT_Z = false>
__device__ __forceinline__ void quantize_store(const float2 (&P)[16], uint32_t* codes_row,
                                               uint16_t* scales_row, int q, bool valid,
                                               int iters, float2* z = nullptr) {
  float amax = 0.0f;
#pragma unroll
  for (int m = 0; m < 16; ++m) amax = fmax3_abs(amax, P[m].x, P[m].y);
  if (GROUP == 64) amax = fmaxf(amax, __shfl_xor_sync(kFull, amax, RPW));
  constexpr float outer = (float)(1 << (BITS - 1)) - 0.5f;
  const float inv = (amax < 1.17549435e-38f) ? 0.0f : __fdiv_rn(outer, amax);
  uint32_t w[BITS];
  float d, n;
  quant_pass<BITS, GROUP, RPW, false, WANT_Z>(P, inv, w, d, n, z);
  float s = d / n;                                  // least-squares scale
  for (int k = 0; k < iters; ++k) {
    const bool live = s >= 1.17549435e-38f;
    uint32_t w2[BITS];
    float d2, n2;
    quant_pass<BITS, GROUP, RPW, true>(P, live ? __fdiv_rn(0.5f, s) : 0.0f, w2, d2, n2);
    if (live) {
#pragma unroll
      for (int j = 0; j < BITS; ++j) w[j] = w2[j];
      s = d2 / n2;
    }
  }
  s = fminf(fmaxf(s, -65504.0f), 65504.0f);
  const __half s16 = __float2half_rn(s);
  if constexpr (WANT_Z) {
    // the reconstructed rotated row s16 * l (exact: 11 x 9 significant bits)
    const float sf = __half2float(s16);
    const float2 s2 = make_float2(sf, sf);
#pragma unroll
    for (int m = 0; m < 16; ++m) z[m] = __fmul2_rn(z[m], s2);
  }
  if (!valid) return;
  if constexpr (BITS == 2) {
    *reinterpret_cast<uint2*>(codes_row + 2 * q) = make_uint2(w[0], w[1]);
  } else if constexpr (BITS == 4) {
    *reinterpret_cast<uint4*>(codes_row + 4 * q) = make_uint4(w[0], w[1], w[2], w[3]);
  } else {
    uint4* o = reinterpret_cast<uint4*>(codes_row + 8 * q);
    o[0] = make_uint4(w[0], w[1], w[2], w[3]);
    o[1] = make_uint4(w[4], w[5], w[6], w[7]);
  }
  if (GROUP == 32)
    scales_row[q] = __half_as_ushort(s16);
  else if (!(q & 1))
    scales_row[q >> 1] = __half_as_ushort(s16);
}

// the row's 32 coordinates of this lane, v (signs applied), rotated in place
// into P[m] = {y_m, y_{m+16}}: Walsh-Hadamard strides ascending, a butterfly
// (a + b, a - b), then x c_d
template <int D, int LPR, int RPW>
__device__ __forceinline__ void rotate_lane(const float (&v)[32], float2 (&P)[16], int q) {
#pragma unroll
  for (int m = 0; m < 16; ++m) P[m] = make_float2(v[m], v[m + 16]);
#pragma unroll
  for (int h = 1; h < 16; h <<= 1) {
#pragma unroll
    for (int m = 0; m < 16; ++m) {
      if (!(m & h)) {
        const float2 a = P[m], b = P[m + h];
        P[m] = __fadd2_rn(a, b);
        P[m + h] = fsub2(a, b);
      }
    }
  }
#pragma unroll
  for (int m = 0; m < 16; ++m) {
    const float a = P[m].x, b = P[m].y;
    P[m] = make_float2(__fadd_rn(a, b), __fsub_rn(a, b));
  }
#pragma unroll
  for (int k = 1; k < LPR; k <<= 1) {
    // the lower partner keeps a + b, the upper one a - b (fma with +-1 is
    // exactly one rounded add or subtract)
    const float sg = (q & k) ? -1.0f : 1.0f;
    const float2 sg2 = make_float2(sg, sg);
#pragma unroll
    for (int m = 0; m < 16; ++m) {
      float2 o;
      o.x = __shfl_xor_sync(kFull, P[m].x, RPW * k);
      o.y = __shfl_xor_sync(kFull, P[m].y, RPW * k);
      P[m] = __ffma2_rn(sg2, P[m], o);
    }
  }
  const float cd = rot_scale<D>();
  const float2 cd2 = make_float2(cd, cd);
#pragma unroll
  for (int m = 0; m < 16; ++m) P[m] = __fmul2_rn(P[m], cd2);
}

// MODE 1: BF16 reference with least-squares refits; 2: compressed reference.
template <int D, int GROUP, int CW, int MODE>
__global__ void __launch_bounds__(ECfg<D, CW>::THREADS, 1)
encode_tma_kernel(const __grid_constant__ EncodeTmaParams tp) {
  using C = ECfg<D, CW>;
  static_assert(MODE == 1 || MODE == 2, "the refit and compressed-reference modes");
  const int iters = tp.p.refine_iters;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* ring = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint32_t* dtab = reinterpret_cast<uint32_t*>(ring + kSlots * C::SLOT_BYTES);  // D_i as bf16 pairs
  uint32_t* ndtab = dtab + D / 2;                                            // -D_i
  uint64_t* full = reinterpret_cast<uint64_t*>(ndtab + D / 2);
  uint64_t* empty = full + kSlots;
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
    for (int s = 0; s < kSlots; ++s) {
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
        const int s = (int)(it % kSlots);
        // the tile's first row lies inside the sources (the tensor maps zero-fill
        // the rows of a partial tile past the end)
        (void)RQ_IN_BOUNDS((long long)t * C::R < p.n_rows && j < RQ_MAX_LOOPS + 1, p.status,
                           kEncodeStatusBounds);
        if (it >= kSlots && !mbar_wait_bounded(&empty[s], (uint32_t)((it / kSlots - 1) & 1))) {
          atomicOr(p.status, 1u);
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
    for (long long k = (it > kSlots ? it - kSlots : 0); k < it; ++k)
      if (!mbar_wait_bounded(&full[k % kSlots], (uint32_t)((k / kSlots) & 1)))
        atomicOr(p.status, 2u);
    return;
  }

  // ---------------- consumers ----------------
  const int rw = lane % C::RPW;          // row within the warp
  const int q = lane / C::RPW;           // which 32 coordinates of the row
  const int r = warp * C::RPW + rw;      // row within the tile
  // shared-memory reads of this lane: line r of a slot, chunks 4q .. 4q+3 of
  // box q / 2 (head_dim 128) or box 0 (64)
  if (!RQ_IN_BOUNDS(r < C::R && q < C::LPR, p.status, kEncodeStatusBounds)) return;
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
    int s = (int)(it % kSlots);
    if (!mbar_wait_bounded(&full[s], (uint32_t)((it / kSlots) & 1))) {
      atomicOr(p.status, 4u);
      return;
    }
    uint32_t wv[16];
    load_row<D, CW>(ring + s * C::SLOT_BYTES, r, q, wv);
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);
    ++it;
    if (valid && p.ref_out) {
      uint4* o = reinterpret_cast<uint4*>(p.ref_out + (size_t)row * D + q * 32);
#pragma unroll
      for (int i = 0; i < 4; ++i)
        o[i] = make_uint4(wv[4 * i], wv[4 * i + 1], wv[4 * i + 2], wv[4 * i + 3]);
    }
    // BF16 reference: -D_i ref_i for the residual fma of every loop.
    // Compressed reference: the rotated reference is quantised (its codes
    // stored) and zr holds its reconstruction s16 * l, subtracted from every
    // loop's rotated row.
    float zr[32];
    constexpr bool cr = (MODE == 2);
    if constexpr (!cr) {
      const uint4* nd4 = reinterpret_cast<const uint4*>(ndtab + q * 16);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const uint4 nd = nd4[i];
        const uint32_t ndw[4] = {nd.x, nd.y, nd.z, nd.w};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          zr[8 * i + 2 * k] = fma_bf16<0>(wv[4 * i + k], ndw[k], 0.0f);
          zr[8 * i + 2 * k + 1] = fma_bf16<1>(wv[4 * i + k], ndw[k], 0.0f);
        }
      }
    } else {
      float v[32];
      const uint4* d4 = reinterpret_cast<const uint4*>(dtab + q * 16);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const uint4 dd = d4[i];
        const uint32_t dw[4] = {dd.x, dd.y, dd.z, dd.w};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          v[8 * i + 2 * k] = fma_bf16<0>(wv[4 * i + k], dw[k], 0.0f);        // D_i ref_i
          v[8 * i + 2 * k + 1] = fma_bf16<1>(wv[4 * i + k], dw[k], 0.0f);
        }
      }
      float2 P[16], Z[16];
      rotate_lane<D, C::LPR, C::RPW>(v, P, q);
      if (p.ref_bits == 8)
        quantize_store<8, GROUP, C::RPW, true>(P, p.ref_codes + (size_t)row * (D / 4),
                                               p.ref_scales + (size_t)row * (D / GROUP), q,
                                               valid, 0, Z);
      else
        quantize_store<4, GROUP, C::RPW, true>(P, p.ref_codes + (size_t)row * (D / 8),
                                               p.ref_scales + (size_t)row * (D / GROUP), q,
                                               valid, 0, Z);
#pragma unroll
      for (int m = 0; m < 16; ++m) {
        zr[m] = Z[m].x;
        zr[m + 16] = Z[m].y;
      }
    }

    for (int j = 0; j < tp.n_active; ++j) {
      s = (int)(it % kSlots);
      if (!mbar_wait_bounded(&full[s], (uint32_t)((it / kSlots) & 1))) {
        atomicOr(p.status, 4u);
        return;
      }
      load_row<D, CW>(ring + s * C::SLOT_BYTES, r, q, wv);
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);
      ++it;

      // BF16 reference: y = D_i x_i + (-D_i ref_i), one rounding, then rotated.
      // Compressed reference: D_i x_i (exact), rotated, then e = RN(y - zr).
      float v[32];
      {
        const uint4* d4 = reinterpret_cast<const uint4*>(dtab + q * 16);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const uint4 dd = d4[i];
          const uint32_t dw[4] = {dd.x, dd.y, dd.z, dd.w};
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const float a0 = cr ? 0.0f : zr[8 * i + 2 * k];
            const float a1 = cr ? 0.0f : zr[8 * i + 2 * k + 1];
            v[8 * i + 2 * k] = fma_bf16<0>(wv[4 * i + k], dw[k], a0);
            v[8 * i + 2 * k + 1] = fma_bf16<1>(wv[4 * i + k], dw[k], a1);
          }
        }
      }
      float2 P[16];
      rotate_lane<D, C::LPR, C::RPW>(v, P, q);
      if constexpr (cr) {
#pragma unroll
        for (int m = 0; m < 16; ++m) P[m] = fsub2(P[m], make_float2(zr[m], zr[m + 16]));
      }

      const int l = tp.active[j];
      if (p.bits[l] == 2)
        quantize_store<2, GROUP, C::RPW>(P, p.codes[l] + (size_t)row * (D / 16),
                                         p.scales[l] + (size_t)row * (D / GROUP), q, valid,
                                         iters);
      else
        quantize_store<4, GROUP, C::RPW>(P, p.codes[l] + (size_t)row * (D / 8),
                                         p.scales[l] + (size_t)row * (D / GROUP), q, valid,
                                         iters);
    }
  }
}

constexpr int kConsumerWarps = 15;   // + 1 producer = 16 warps, 4 per scheduler

template <int D, int GROUP, int MODE>
cudaError_t launch_tm(const EncodeTmaParams& tp, int num_sms, cudaStream_t stream) {
  using C = ECfg<D, kConsumerWarps>;
  cudaError_t e = cudaFuncSetAttribute(encode_tma_kernel<D, GROUP, kConsumerWarps, MODE>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
  if (e != cudaSuccess) return e;
  const int grid = tp.n_tiles < num_sms ? tp.n_tiles : num_sms;
  return launch_pdl(encode_tma_kernel<D, GROUP, kConsumerWarps, MODE>, (unsigned)grid,
                    C::THREADS, C::SMEM, stream, tp);
}

template <int D, int GROUP>
cudaError_t launch_t(const EncodeTmaParams& tp, int num_sms, cudaStream_t stream) {
  if (tp.p.ref_bits != 0) return launch_tm<D, GROUP, 2>(tp, num_sms, stream);
  return launch_tm<D, GROUP, 1>(tp, num_sms, stream);
}

}  // namespace

cudaError_t launch_encode_tma_fixed(int head_dim, int group, const EncodeParams& p, int num_sms,
                                    cudaStream_t stream) {
  EncodeTmaParams tp;
  std::memset(&tp, 0, sizeof tp);
  tp.p = p;
  const int R = head_dim == 128 ? ECfg<128, kConsumerWarps>::R : ECfg<64, kConsumerWarps>::R;
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

}  // namespace rq
