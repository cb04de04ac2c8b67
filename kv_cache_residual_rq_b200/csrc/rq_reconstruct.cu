// rq_reconstruct.cu -- rebuild a loop's K/V rows from the stored format.
//
// Method: "ResidualQuant: KV Cache Quantization for Looped Transformers with
// 2-Bit Residuals", Abstract -- a non-final loop is the final-loop reference
// plus a rotated low-bit residual with a least-squares scale.  This kernel
// applies that definition row by row, for consumers that want the loop's K/V
// itself (any attention kernel, a prefill over the cache, quality studies):
//   out = f32(ref) + Rot^T (s * l),  Rot^T z = D (c_d H z)
// Mapping as in the encoder: 16 lanes (head_dim 128) or 8 (64) per row,
// 8 coordinates per lane; butterflies in registers for strides 1-4 and by
// shfl.xor across lanes for the rest.  Plain streaming kernel, no waits.
#include "rq_device.cuh"
#include "rq_internal.h"

namespace rq {
namespace {

constexpr int kThreads = 256;

// RB: 0 = BF16 reference rows; 4 or 8 = compressed reference (codes and
// scales in the rotated domain: out = Rot^T (s_ref l_ref + s l))
template <int D, int GROUP, int BITS, bool OUT_BF16, int RB>
__global__ void __launch_bounds__(kThreads)
reconstruct_kernel(const ReconstructParams p) {
  constexpr int DPL = 8;
  constexpr int LPR = D / DPL;       // lanes per row
  constexpr int RPW = 32 / LPR;      // rows per warp
  constexpr int LPG = GROUP / DPL;   // lanes per scale group
  constexpr unsigned FULL = 0xffffffffu;
  constexpr int TOP = (1 << BITS) - 1;

  const int lane = threadIdx.x & 31;
  const int li = lane % LPR;
  const int slot = lane / LPR;
  const long long warp = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const long long nwarps = ((long long)gridDim.x * blockDim.x) >> 5;

  uint32_t neg = 0;
#pragma unroll
  for (int k = 0; k < DPL; ++k) neg |= sign_bit(p.seed, li * DPL + k) << k;
  const float cd = rot_scale<D>();

  for (long long row0 = warp * RPW; row0 < p.n_rows; row0 += nwarps * RPW) {
    const long long idx = row0 + slot;
    const long long hd = idx / p.ctx, t = idx % p.ctx;
    const long long row = hd * p.pitch + t;
    // every array of the call holds heads * pitch rows
    const bool valid = idx < p.n_rows &&
                       RQ_IN_BOUNDS(row >= 0 && row < (p.n_rows / p.ctx) * p.pitch, p.status,
                                    kEncodeStatusBounds);
    const size_t eoff = (size_t)row * D + li * DPL;
    uint4 rw = make_uint4(0, 0, 0, 0);
    if constexpr (RB == 0) {
      if (valid) rw = __ldcs(reinterpret_cast<const uint4*>(p.ref + eoff));
    }
    float v[DPL];
    float vr[DPL];                    // compressed reference: s_ref l_ref
#pragma unroll
    for (int k = 0; k < DPL; ++k) vr[k] = 0.0f;
    if constexpr (RB != 0) {
      constexpr int RTOP = (1 << RB) - 1;
      uint32_t rc[2] = {0u, 0u};
      float sr = 0.0f;
      if (valid) {
        const uint32_t* cw = p.ref_codes + (size_t)row * (D * RB / 32) + li * DPL * RB / 32;
        rc[0] = cw[0];
        if constexpr (RB == 8) rc[1] = cw[1];
        sr = __half2float(__ushort_as_half(p.ref_scales[(size_t)row * (D / GROUP) + li / LPG]));
      }
#pragma unroll
      for (int k = 0; k < DPL; ++k) {
        const int c = (int)((rc[(k * RB) / 32] >> ((k * RB) % 32)) & (uint32_t)RTOP);
        vr[k] = sr * (float)(2 * c - RTOP);
      }
    }
    if constexpr (BITS != 16 || RB != 0) {
      uint32_t x = 0;
      float s = 0.0f;
      if constexpr (BITS != 16) {
        if (valid) {
          const int bit0 = li * DPL * BITS;
          x = p.codes[(size_t)row * (D * BITS / 32) + bit0 / 32] >> (bit0 % 32);
          s = __half2float(__ushort_as_half(p.scales[(size_t)row * (D / GROUP) + li / LPG]));
        }
      }
#pragma unroll
      for (int k = 0; k < DPL; ++k) {
        const int c = (int)((x >> (BITS * k)) & (uint32_t)TOP);
        v[k] = (BITS == 16) ? vr[k] : vr[k] + s * (float)(2 * c - TOP);
      }
      // Rot^T: butterflies (strides 1, 2, 4 in registers, the rest across lanes)
#pragma unroll
      for (int h = 1; h < DPL; h <<= 1) {
#pragma unroll
        for (int k = 0; k < DPL; ++k) {
          if (!(k & h)) {
            const float a = v[k], b = v[k + h];
            v[k] = a + b;
            v[k + h] = a - b;
          }
        }
      }
#pragma unroll
      for (int m = 1; m < LPR; m <<= 1) {
        const float sg = (li & m) ? -1.0f : 1.0f;
#pragma unroll
        for (int k = 0; k < DPL; ++k) {
          const float other = __shfl_xor_sync(FULL, v[k], m);
          v[k] = fmaf(sg, v[k], other);
        }
      }
#pragma unroll
      for (int k = 0; k < DPL; ++k) v[k] = flip_sign(cd * v[k], (neg >> k) & 1u);
    } else {
#pragma unroll
      for (int k = 0; k < DPL; ++k) v[k] = 0.0f;
    }
    const uint32_t rs[4] = {rw.x, rw.y, rw.z, rw.w};
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      v[2 * c] += bf16lo(rs[c]);
      v[2 * c + 1] += bf16hi(rs[c]);
    }
    if (valid) {
      if constexpr (OUT_BF16) {
        uint4 o;
        uint32_t* op = &o.x;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const __nv_bfloat162 b2 = __floats2bfloat162_rn(v[2 * c], v[2 * c + 1]);
          op[c] = *reinterpret_cast<const uint32_t*>(&b2);
        }
        reinterpret_cast<uint4*>(p.out)[eoff / 8] = o;
      } else {
        float4* o = reinterpret_cast<float4*>(reinterpret_cast<float*>(p.out) + eoff);
        o[0] = make_float4(v[0], v[1], v[2], v[3]);
        o[1] = make_float4(v[4], v[5], v[6], v[7]);
      }
    }
  }
}

template <int D, int GROUP, int BITS, int RB = 0>
cudaError_t launch_t(const ReconstructParams& p, int num_sms, cudaStream_t stream) {
  constexpr int rows_per_block = kThreads / 32 * (32 / (D / 8));
  long long blocks = (p.n_rows + rows_per_block - 1) / rows_per_block;
  const long long cap = (long long)num_sms * 8;
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  if (p.out_bf16)
    reconstruct_kernel<D, GROUP, BITS, true, RB><<<(unsigned)blocks, kThreads, 0, stream>>>(p);
  else
    reconstruct_kernel<D, GROUP, BITS, false, RB><<<(unsigned)blocks, kThreads, 0, stream>>>(p);
  return cudaGetLastError();
}

template <int D, int GROUP>
cudaError_t launch_g(int bits, const ReconstructParams& p, int num_sms, cudaStream_t stream) {
  if (bits == 2) return launch_t<D, GROUP, 2>(p, num_sms, stream);
  if (bits == 4) return launch_t<D, GROUP, 4>(p, num_sms, stream);
  if (bits == 16) return launch_t<D, GROUP, 16>(p, num_sms, stream);
  return cudaErrorInvalidValue;
}

template <int D, int GROUP, int RB>
cudaError_t launch_cr_b(int bits, const ReconstructParams& p, int num_sms, cudaStream_t stream) {
  if (bits == 2) return launch_t<D, GROUP, 2, RB>(p, num_sms, stream);
  if (bits == 4) return launch_t<D, GROUP, 4, RB>(p, num_sms, stream);
  if (bits == 16) return launch_t<D, GROUP, 16, RB>(p, num_sms, stream);
  return cudaErrorInvalidValue;
}

template <int D, int GROUP>
cudaError_t launch_cr_g(int ref_bits, int bits, const ReconstructParams& p, int num_sms,
                        cudaStream_t stream) {
  if (ref_bits == 8) return launch_cr_b<D, GROUP, 8>(bits, p, num_sms, stream);
  if (ref_bits == 4) return launch_cr_b<D, GROUP, 4>(bits, p, num_sms, stream);
  return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_reconstruct_cr(int head_dim, int group, int ref_bits, int bits,
                                  const ReconstructParams& p, int num_sms, cudaStream_t stream) {
  if (head_dim == 128 && group == 32) return launch_cr_g<128, 32>(ref_bits, bits, p, num_sms, stream);
  if (head_dim == 128 && group == 64) return launch_cr_g<128, 64>(ref_bits, bits, p, num_sms, stream);
  if (head_dim == 64 && group == 32) return launch_cr_g<64, 32>(ref_bits, bits, p, num_sms, stream);
  if (head_dim == 64 && group == 64) return launch_cr_g<64, 64>(ref_bits, bits, p, num_sms, stream);
  return cudaErrorInvalidValue;
}

cudaError_t launch_reconstruct(int head_dim, int group, int bits, const ReconstructParams& p,
                               int num_sms, cudaStream_t stream) {
  if (head_dim == 128 && group == 32) return launch_g<128, 32>(bits, p, num_sms, stream);
  if (head_dim == 128 && group == 64) return launch_g<128, 64>(bits, p, num_sms, stream);
  if (head_dim == 64 && group == 32) return launch_g<64, 32>(bits, p, num_sms, stream);
  if (head_dim == 64 && group == 64) return launch_g<64, 64>(bits, p, num_sms, stream);
  return cudaErrorInvalidValue;
}

}  // namespace rq
