// rq_encode_tma_common.cuh -- pieces shared by the two tensor-copy encoder
// kernels (rq_encode_tma.cu: the plain mode; rq_encode_tma_fixed.cu: the
// least-squares-refit and compressed-reference modes): the launch parameter
// block, the 2-D tensor copy, and the few arithmetic primitives both use.
#pragma once

#include <cuda.h>

#include "rq_device.cuh"
#include "rq_internal.h"

namespace rq {
namespace enc {

// floor(u) as the round-down add u + 1.5*2^23, whose bit pattern is
// 0x4B400000 + floor(u) for |u| < 2^22
constexpr float kFloorMagic = 12582912.0f;          // 1.5 * 2^23
constexpr uint32_t kFloorMagicBits = 0x4B400000u;
constexpr unsigned kFull = 0xffffffffu;

struct alignas(64) EncodeTmaParams {
  CUtensorMap maps[RQ_MAX_LOOPS + 1];   // [0] the reference, then each quantised loop
  EncodeParams p;
  int active[RQ_MAX_LOOPS];             // loop index of each quantised loop, in order
  int n_active;
  int n_tiles;
};

__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int x, int y,
                                            uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar))
      : "memory");
}

// a.half(H) * b.half(H) + c, bf16 operands, one rounding
template <int H>
__device__ __forceinline__ float fma_bf16(uint32_t a2, uint32_t b2, float c) {
  float d;
  if constexpr (H == 0)
    asm("{\n\t.reg .b16 al, ah, bl, bh;\n\tmov.b32 {al, ah}, %1;\n\tmov.b32 {bl, bh}, %2;\n\t"
        "fma.rn.f32.bf16 %0, al, bl, %3;\n\t}"
        : "=f"(d) : "r"(a2), "r"(b2), "f"(c));
  else
    asm("{\n\t.reg .b16 al, ah, bl, bh;\n\tmov.b32 {al, ah}, %1;\n\tmov.b32 {bl, bh}, %2;\n\t"
        "fma.rn.f32.bf16 %0, ah, bh, %3;\n\t}"
        : "=f"(d) : "r"(a2), "r"(b2), "f"(c));
  return d;
}

// max(m, |a|, |b|) for m >= 0
__device__ __forceinline__ float fmax3_abs(float m, float a, float b) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(m), "f"(fabsf(a)), "f"(fabsf(b)));
  return r;
}

__device__ __forceinline__ float2 fsub2(float2 a, float2 b) {
  float2 r;
  asm("{\n\t.reg .b64 ra, rb, rr;\n\tmov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "sub.rn.f32x2 rr, ra, rb;\n\tmov.b64 {%0, %1}, rr;\n\t}"
      : "=f"(r.x), "=f"(r.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return r;
}

}  // namespace enc
}  // namespace rq
