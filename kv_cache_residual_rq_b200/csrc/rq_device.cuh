// rq_device.cuh -- device helpers shared by the encoder and the decode kernel.
//
// Rotation signs (splitmix64), bf16 unpacking, and the mbarrier / bulk-copy
// (TMA, non-tensor, one destination CTA) primitives of sm_100a as inline PTX.  Every
// mbarrier wait is bounded: after kWaitLimitCycles it gives up and reports
// failure instead of spinning forever.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

namespace rq {

// ---------------------------------------------------------------------------
// seeded signs of the rotation: D_i = -1 iff bit 63 of splitmix64 output i
// (Steele, Lea and Flood, OOPSLA 2014; output i = mix(seed + (i+1) * gamma))
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint64_t splitmix64_at(uint64_t seed, uint64_t i) {
  uint64_t z = seed + (i + 1ull) * 0x9E3779B97F4A7C15ull;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

// 1 when the sign of coordinate i is negative.
__device__ __forceinline__ uint32_t sign_bit(uint64_t seed, int i) {
  return (uint32_t)(splitmix64_at(seed, (uint64_t)i) >> 63);
}

// c_d = RN_f32(1/sqrt(d)) for the two head sizes the library builds.
template <int D>
__device__ __forceinline__ float rot_scale() {
  static_assert(D == 64 || D == 128, "head_dim 64 or 128");
  return D == 64 ? 0.125f : 0.0883883476483184405f;  // 0x3DB504F3
}

// bf16 pair packed in a uint32 -> two floats (exact widening).
__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// acc + a.lo * b.lo + a.hi * b.hi for two packed bf16 pairs, each step one
// fused multiply-add with an fp32 accumulator (bf16 x bf16 products are exact
// in fp32, so this equals widening both operands and using fmaf).
__device__ __forceinline__ float fma_bf16x2(uint32_t a2, uint32_t b2, float acc) {
  asm("{\n\t.reg .b16 al, ah, bl, bh;\n\t"
      "mov.b32 {al, ah}, %1;\n\t"
      "mov.b32 {bl, bh}, %2;\n\t"
      "fma.rn.f32.bf16 %0, al, bl, %0;\n\t"
      "fma.rn.f32.bf16 %0, ah, bh, %0;\n\t}"
      : "+f"(acc)
      : "r"(a2), "r"(b2));
  return acc;
}

__device__ __forceinline__ float flip_sign(float x, uint32_t neg) {
  return __uint_as_float(__float_as_uint(x) ^ (neg << 31));
}

// ---------------------------------------------------------------------------
// Bounds-checked builds (nvcc -DRQ_BOUNDS_CHECK: librq_bounds.so).  Before
// an access whose index a kernel computes at run time, RQ_IN_BOUNDS(ok,
// status, bit) tests that index against the extent of its buffer -- the
// sizes the C ABI's size queries give for the call's shape -- or of its
// shared-memory area.  A failed test raises `bit` in the call's status word
// and the access is skipped; nothing traps.  In normal builds the test is
// the constant true and the condition is never evaluated.
// ---------------------------------------------------------------------------
#ifdef RQ_BOUNDS_CHECK
__device__ __forceinline__ bool rq_in_bounds(bool ok, uint32_t* status, uint32_t bit) {
  if (!ok) atomicOr(status, bit);
  return ok;
}
#define RQ_IN_BOUNDS(ok, status, bit) (::rq::rq_in_bounds((ok), (status), (bit)))
#else
#define RQ_IN_BOUNDS(ok, status, bit) (true)
#endif
constexpr uint32_t kStatusBounds = 128u;         // decode workspace status word
constexpr uint32_t kEncodeStatusBounds = 8u;     // encoder status word

// ---------------------------------------------------------------------------
// mbarrier + bulk async copy (global -> shared, completion via mbarrier tx)
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
               : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 _, [%0], %1;" ::"r"(
                   smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(done)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return done != 0;
}

// About 2 s at the B200's top clock: far beyond any legitimate wait.
constexpr long long kWaitLimitCycles = 4000000000ll;

// Bounded wait for the phase with the given parity to complete.
// Returns false when the limit ran out.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity)) {
    if (clock64() - t0 > kWaitLimitCycles) return false;
  }
  return true;
}

// cp.async.bulk global -> this CTA's own shared memory,
// completion counted on `bar`.
// dst, src 16-byte aligned; bytes a multiple of 16.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes,
                                         uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// cp.async.bulk prefetch of global memory into L2 (no data returned, no
// completion to wait for).  src 16-byte aligned; bytes a multiple of 16.
__device__ __forceinline__ void bulk_prefetch_l2(const void* src, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}

// Programmatic dependent launch (sm_90 and later).  pdl_allow_next lets the
// next kernel of the stream be scheduled once every CTA of this grid has
// started; pdl_wait_prev blocks until the grids before this one have
// completed and their writes are visible.  A kernel launched with the
// programmatic-serialization attribute must call pdl_wait_prev before its
// first global memory read whose value it uses.  An L2 prefetch may come
// earlier: it returns no data, and L2 is where the previous grid's writes
// land, so every read after the wait sees them.
__device__ __forceinline__ void pdl_allow_next() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void pdl_wait_prev() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// named barrier over `nthreads` threads (a multiple of 32)
__device__ __forceinline__ void named_bar_sync(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

}  // namespace rq
