// rq_noalloc.cu -- decode attention for callers that cannot allocate memory.
//
// rq_decode_attention needs a caller-provided workspace.  Some callers have
// no way to provide one: code that runs inside a host application which owns
// every device allocation and hands out none, code on a latency-critical
// path that must not call cudaMalloc (it can synchronise the device), or a
// plug-in whose memory budget was fixed before it was loaded.  This file
// gives them rq_decode_attention_noalloc: the same kernel, with its scratch
// in a fixed-size array that lives in the library's own device memory.
//
// The array is a file-scope __device__ variable, so every GPU on which the
// library is used holds RQ_NOALLOC_SCRATCH_BYTES of it until the process
// exits.  Host code never dereferences the symbol: on first use per device
// it asks the runtime for the array's device address (cudaGetSymbolAddress,
// with that device current) and caches it.  No call here allocates memory.
#include <cmath>
#include <mutex>

#include "rq_internal.h"

namespace {

__device__ __align__(256) unsigned char g_noalloc_scratch[RQ_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
void* g_scratch_addr[kMaxDevices] = {nullptr};
std::mutex g_scratch_mu;

// Device address of the scratch array on the current device (set up once
// per device).  Returns false if the runtime cannot provide it.
bool scratch_address(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return false;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return false;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return true;
}

bool a16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" rq_status rq_decode_attention_noalloc(
    const rq_shape* shape, const uint16_t* q, const uint16_t* ref_k, const uint16_t* ref_v,
    const uint32_t* codes_k, const uint32_t* codes_v, const uint16_t* scales_k,
    const uint16_t* scales_v, int bits, uint64_t seed, float softmax_scale, float* out,
    void* stream) {
  // Anything rq_decode_attention would reject is handed to it unchanged, so
  // the caller gets the same status and nothing is enqueued.
  const size_t need = rq_decode_workspace_bytes(shape);
  const bool res = bits != 16;
  const bool args_ok =
      need != 0 && (bits == 2 || bits == 4 || bits == 16) && q && ref_k && ref_v && out &&
      a16(q) && a16(ref_k) && a16(ref_v) && a16(out) &&
      (!res || (codes_k && codes_v && scales_k && scales_v && a16(codes_k) && a16(codes_v) &&
                a16(scales_k) && a16(scales_v))) &&
      (softmax_scale <= 0.0f || std::isfinite(softmax_scale));
  if (!args_ok)
    return rq_decode_attention(shape, q, ref_k, ref_v, codes_k, codes_v, scales_k, scales_v, bits,
                               seed, softmax_scale, out, nullptr, 0, stream);
  if (need > RQ_NOALLOC_SCRATCH_BYTES) return RQ_ERR_WORKSPACE;

  void* scratch = nullptr;
  if (!scratch_address(&scratch)) return RQ_ERR_CUDA;

  // The status word and the per-head arrival counters must start at zero;
  // the partial records need no clearing.
  const long long heads = (long long)shape->batch * shape->kv_heads;
  const size_t zero_bytes = rq::kWsHeaderBytes + rq::ws_counters_bytes(heads);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(scratch, 0, zero_bytes, st) != cudaSuccess) return RQ_ERR_CUDA;
  return rq_decode_attention(shape, q, ref_k, ref_v, codes_k, codes_v, scales_k, scales_v, bits,
                             seed, softmax_scale, out, scratch, RQ_NOALLOC_SCRATCH_BYTES, stream);
}
