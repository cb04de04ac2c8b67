// rq_encode.cu -- ResidualQuant encoder for sm_100a.
//
// Method: "ResidualQuant: KV Cache Quantization for Looped Transformers with
// 2-Bit Residuals", Abstract -- each non-final loop is stored as its residual
// against the final-loop reference, rotated, and quantised per group to INT2
// (INT4 where the loop is given more bits) with a least-squares scale.
//
// Mapping: a row is one (row, kv head, token) vector of head_dim elements;
// source and destination rows may sit in arrays of different token pitch
// (encoding a window slot into a cache position).
// 16 lanes (head_dim 128) or 8 lanes (64) own a row, 8 consecutive elements
// per lane, so each lane moves its slice of every loop with one 16-byte
// load.  The reference slice is loaded once and reused for every loop.  The
// Walsh-Hadamard butterflies run in registers for strides 1, 2, 4 and across
// lanes (shfl.xor) for the larger strides, in ascending stride order, each
// butterfly one round-to-nearest binary32 add or subtract -- the sequence the
// codes are specified by, so codes are bit-identical to that specification.
// The kernel is a plain streaming kernel: no shared memory, no waits.
#include "rq_device.cuh"
#include "rq_internal.h"

namespace rq {
namespace {

constexpr int kEncodeThreads = 256;
constexpr int kLoopBatch = 4;   // loops whose loads are in flight together

__device__ __forceinline__ uint4 ld_stream(const uint16_t* p) {
  return __ldcs(reinterpret_cast<const uint4*>(p));
}

template <int D, int GROUP>
__global__ void __launch_bounds__(kEncodeThreads)
encode_kernel(const EncodeParams p) {
  constexpr int DPL = 8;             // elements per lane
  constexpr int LPR = D / DPL;       // lanes per row
  constexpr int RPW = 32 / LPR;      // rows per warp
  constexpr int LPG = GROUP / DPL;   // lanes per group
  constexpr unsigned FULL = 0xffffffffu;

  const int lane = threadIdx.x & 31;
  const int li = lane % LPR;
  const int slot = lane / LPR;
  const long long warp = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const long long nwarps = ((long long)gridDim.x * blockDim.x) >> 5;

  uint32_t neg = 0;                  // bit k: coordinate li*8+k has sign -1
#pragma unroll
  for (int k = 0; k < DPL; ++k) neg |= sign_bit(p.seed, li * DPL + k) << k;
  const float cd = rot_scale<D>();

  for (long long row0 = warp * RPW; row0 < p.n_rows; row0 += nwarps * RPW) {
    const long long idx = row0 + slot;             // (head, token) index of this call
    const long long hd = idx / p.ctx, t = idx % p.ctx;
    const long long src_row = hd * p.src_pitch + p.src_offset + t;
    const bool valid = idx < p.n_rows &&
                       RQ_IN_BOUNDS(src_row >= 0 && src_row < p.n_src_rows, p.status,
                                    kEncodeStatusBounds);
    long long row = 0;                                             // destination row
    const bool wvalid = valid && enc_dst_row(p, hd, t, row) &&
                        RQ_IN_BOUNDS(row >= 0 && row < p.n_dst_rows, p.status,
                                     kEncodeStatusBounds);
    const size_t eoff = (size_t)src_row * D + li * DPL;
    const uint4 rw = valid ? ld_stream(p.ref + eoff) : make_uint4(0, 0, 0, 0);
    if (wvalid && p.ref_out)
      *reinterpret_cast<uint4*>(p.ref_out + (size_t)row * D + li * DPL) = rw;

    for (int lb = 0; lb < p.n_loops; lb += kLoopBatch) {
      uint4 xw[kLoopBatch];
#pragma unroll
      for (int j = 0; j < kLoopBatch; ++j) {
        const int l = lb + j;
        xw[j] = make_uint4(0, 0, 0, 0);
        if (valid && l < p.n_loops && p.bits[l] != 16) xw[j] = ld_stream(p.x[l] + eoff);
      }
#pragma unroll
      for (int j = 0; j < kLoopBatch; ++j) {
        const int l = lb + j;
        if (l >= p.n_loops) break;          // uniform over the grid
        const int bits = p.bits[l];
        if (bits == 16) continue;           // uniform over the grid

        // residual against the reference, sign flip (exact)
        const uint32_t xs[4] = {xw[j].x, xw[j].y, xw[j].z, xw[j].w};
        const uint32_t rs[4] = {rw.x, rw.y, rw.z, rw.w};
        float v[DPL];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          v[2 * c] = __fsub_rn(bf16lo(xs[c]), bf16lo(rs[c]));
          v[2 * c + 1] = __fsub_rn(bf16hi(xs[c]), bf16hi(rs[c]));
        }
#pragma unroll
        for (int k = 0; k < DPL; ++k) v[k] = flip_sign(v[k], (neg >> k) & 1u);

        // butterflies, strides 1, 2, 4 inside the lane
#pragma unroll
        for (int h = 1; h < DPL; h <<= 1) {
#pragma unroll
          for (int k = 0; k < DPL; ++k) {
            if (!(k & h)) {
              const float a = v[k], b = v[k + h];
              v[k] = __fadd_rn(a, b);
              v[k + h] = __fsub_rn(a, b);
            }
          }
        }
        // strides 8 .. D/2 across lanes: the lower partner keeps a + b, the
        // upper one a - b; fma with +-1 is exactly one rounded add/subtract
#pragma unroll
        for (int m = 1; m < LPR; m <<= 1) {
          const float sg = (li & m) ? -1.0f : 1.0f;
#pragma unroll
          for (int k = 0; k < DPL; ++k) {
            const float other = __shfl_xor_sync(FULL, v[k], m);
            v[k] = __fmaf_rn(sg, v[k], other);
          }
        }
#pragma unroll
        for (int k = 0; k < DPL; ++k) v[k] = __fmul_rn(v[k], cd);

        // group absmax over LPG lanes
        float amax = 0.0f;
#pragma unroll
        for (int k = 0; k < DPL; ++k) amax = fmaxf(amax, fabsf(v[k]));
#pragma unroll
        for (int m = 1; m < LPG; m <<= 1) amax = fmaxf(amax, __shfl_xor_sync(FULL, amax, m));

        const int half = 1 << (bits - 1);
        const int top = (1 << bits) - 1;
        const float outer = (float)half - 0.5f;
        const float inv = (amax < 1.17549435e-38f) ? 0.0f : __fdiv_rn(outer, amax);

        // one quantisation pass with step 1/(2 iv): codes (clamped), the
        // lane's levels, and <l,l> of the group
        float lvl[DPL];
        auto pass = [&](float iv, uint32_t& packed, int& nrm) {
          packed = 0;
          nrm = 0;
#pragma unroll
          for (int k = 0; k < DPL; ++k) {
            const float u = __fmul_rn(v[k], iv);
            int c = __float2int_rd(u) + half;     // floor(u) + 2^(b-1)
            c = min(max(c, 0), top);
            const int l2 = 2 * c - top;
            lvl[k] = (float)l2;
            nrm += l2 * l2;
            packed |= (uint32_t)c << (bits * k);
          }
#pragma unroll
          for (int m = 1; m < LPG; m <<= 1) nrm += __shfl_xor_sync(FULL, nrm, m);
        };
        // <y,l> of the group in the order that refits depend on: fma chains
        // over runs of 16 coordinates (lanes 2j, 2j+1: the odd lane continues
        // its even neighbour's chain), the two runs of each 32-block added,
        // then the blocks of a 64-group added; the total is broadcast from
        // the group's last lane
        auto fixed_dot = [&]() {
          float a = 0.0f;
#pragma unroll
          for (int k = 0; k < DPL; ++k) a = fmaf(v[k], lvl[k], a);
          const float prev = __shfl_up_sync(FULL, a, 1);
          if (li & 1) {
            a = prev;
#pragma unroll
            for (int k = 0; k < DPL; ++k) a = fmaf(v[k], lvl[k], a);
          }
          const float run0 = __shfl_up_sync(FULL, a, 2);
          float tot = ((li & 3) == 3) ? run0 + a : a;
          if (GROUP == 64) {
            const float blk0 = __shfl_up_sync(FULL, tot, 4);
            if ((li & 7) == 7) tot = blk0 + tot;
          }
          return __shfl_sync(FULL, tot, lane | (LPG - 1));
        };

        uint32_t packed;
        int nrm;
        pass(inv, packed, nrm);
        float dot;
        if (p.refine_iters == 0) {
          dot = 0.0f;
#pragma unroll
          for (int k = 0; k < DPL; ++k) dot = fmaf(v[k], lvl[k], dot);
#pragma unroll
          for (int m = 1; m < LPG; m <<= 1) dot += __shfl_xor_sync(FULL, dot, m);
        } else {
          dot = fixed_dot();
        }
        float s = dot / (float)nrm;               // least-squares scale
        for (int it = 0; it < p.refine_iters; ++it) {
          // refit: nearest level of the current scale, then the scale
          const bool live = s >= 1.17549435e-38f;   // the same in every lane of the group
          uint32_t packed2;
          int nrm2;
          pass(live ? __fdiv_rn(0.5f, s) : 0.0f, packed2, nrm2);
          const float dot2 = fixed_dot();
          if (live) {
            packed = packed2;
            s = dot2 / (float)nrm2;
          }
        }
        s = fminf(fmaxf(s, -65504.0f), 65504.0f);

        if (bits == 2) {
          // 16 codes per word: lanes 2w and 2w+1 of a row share word w
          const uint32_t upper = __shfl_down_sync(FULL, packed, 1);
          if (wvalid && !(li & 1))
            p.codes[l][(size_t)row * (D / 16) + (li >> 1)] = packed | (upper << 16);
        } else {
          if (wvalid) p.codes[l][(size_t)row * (D / 8) + li] = packed;
        }
        if (wvalid && (li % LPG) == 0)
          p.scales[l][(size_t)row * (D / GROUP) + li / LPG] =
              __half_as_ushort(__float2half_rn(s));
      }
    }
  }
}

template <int D, int GROUP>
cudaError_t launch_encode_t(const EncodeParams& p, int num_sms, cudaStream_t stream) {
  constexpr int rows_per_block = kEncodeThreads / 32 * (32 / (D / 8));
  long long blocks = (p.n_rows + rows_per_block - 1) / rows_per_block;
  const long long cap = (long long)num_sms * 8;
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  encode_kernel<D, GROUP><<<(unsigned)blocks, kEncodeThreads, 0, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_encode(int head_dim, int group, const EncodeParams& p, int num_sms,
                          cudaStream_t stream) {
  if (head_dim == 128 && group == 32) return launch_encode_t<128, 32>(p, num_sms, stream);
  if (head_dim == 128 && group == 64) return launch_encode_t<128, 64>(p, num_sms, stream);
  if (head_dim == 64 && group == 32) return launch_encode_t<64, 32>(p, num_sms, stream);
  if (head_dim == 64 && group == 64) return launch_encode_t<64, 64>(p, num_sms, stream);
  return cudaErrorInvalidValue;
}

}  // namespace rq
