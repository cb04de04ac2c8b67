// rq_api.cu -- the C ABI of librq.so (declared in include/rq.h).
//
// Host side only: argument validation (before anything is enqueued), the
// size queries, the work plan of a decode call, and dispatch to the kernels.
// Nothing here allocates device memory or synchronises, except
// rq_workspace_status and rq_encode_take_status, whose job is to read a
// status word back.
#include <climits>
#include <cmath>
#include <cstring>

#include "rq_internal.h"

namespace rq {

namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
size_t round16(size_t n) { return (n + 15) / 16 * 16; }

bool supported_dims(int head_dim, int group) {
  return (head_dim == 64 || head_dim == 128) && (group == 32 || group == 64) &&
         head_dim % group == 0;
}

// token pitch of the arrays a shape describes
int pitch_of(const rq_shape* s) { return s->ctx_cap ? s->ctx_cap : s->ctx; }

// basic shape check shared by the size queries; false for anything invalid
bool shape_ok(const rq_shape* s, bool need_ctx) {
  if (!s) return false;
  if (s->batch < 1 || s->kv_heads < 1 || s->ctx < 0) return false;
  if (s->ctx_cap != 0 && s->ctx_cap < s->ctx) return false;
  if (need_ctx && s->ctx < 1) return false;
  return supported_dims(s->head_dim, s->group);
}

// Extents and status word every encoder launch carries (the bounds-checked
// build tests its indices against them); false if the status word's device
// address is not available.
bool finish_encode_params(EncodeParams& p, const rq_shape& s) {
  const long long heads = (long long)s.batch * s.kv_heads;
  p.n_src_rows = heads * p.src_pitch;
  p.n_dst_rows = p.page_table ? (long long)p.n_pages * s.kv_heads * 64 : heads * p.dst_pitch;
  p.status = encode_status_ptr();
  return p.status != nullptr;
}

bool decode_shape_ok(const rq_shape* s) {
  if (!shape_ok(s, true)) return false;
  if (s->q_heads < s->kv_heads || s->q_heads % s->kv_heads) return false;
  const int G = s->q_heads / s->kv_heads;
  return G == 1 || G == 2 || G == 4 || G == 8;
}

}  // namespace

int device_sm_count() {
  static int cache[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return 0;
  if (dev < 64 && cache[dev] > 0) return cache[dev];
  int sms = 0;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  if (dev < 64) cache[dev] = sms;
  return sms;
}

DecodePlan plan_decode(const rq_shape& s, int num_sms, bool varlen) {
  DecodePlan pl;
  pl.heads = (long long)s.batch * s.kv_heads;
  if (varlen) {
    // tiles are counted on the device; a head of a sequence at full
    // capacity has nt tiles and can meet at most one CTA run per tile
    const int cap = s.ctx_cap ? s.ctx_cap : s.ctx;
    pl.nt = cap > 0 ? (cap + kDecodeTile - 1) / kDecodeTile : 1;
    pl.n_tiles = 0;
    long long P = (long long)num_sms * kDecodeCtasPerSm;
    if (P > kDecodeMaxCtas) P = kDecodeMaxCtas;
    if (P < 1) P = 1;
    pl.ctas = (int)P;
    pl.max_contrib = pl.nt < kDecodeMaxCtas ? pl.nt : kDecodeMaxCtas;
    return pl;
  }
  pl.nt = (s.ctx + kDecodeTile - 1) / kDecodeTile;
  pl.n_tiles = pl.heads * pl.nt;
  long long P = (long long)num_sms * kDecodeCtasPerSm;
  if (P > kDecodeMaxCtas) P = kDecodeMaxCtas;
  if (P > pl.n_tiles) P = pl.n_tiles;
  if (P < 1) P = 1;
  pl.ctas = (int)P;
  // a head spans at most floor(P / heads) + 2 CTA runs; bound with the
  // largest P any device can get so the workspace size is device independent
  long long mc = kDecodeMaxCtas / pl.heads + 2;
  if (mc > pl.nt) mc = pl.nt;
  pl.max_contrib = (int)mc;
  return pl;
}

size_t decode_workspace_bytes(const rq_shape& s, bool varlen) {
  const DecodePlan pl = plan_decode(s, 1, varlen);
  const int G = s.q_heads / s.kv_heads;
  return kWsHeaderBytes + ws_counters_bytes(pl.heads) +
         (size_t)pl.heads * pl.max_contrib * G * ws_record_floats(s.head_dim) * sizeof(float);
}

}  // namespace rq

using namespace rq;

extern "C" {

int rq_version(void) { return 100; }   // 0.1.0

const char* rq_status_string(rq_status s) {
  switch (s) {
    case RQ_OK: return "ok";
    case RQ_ERR_INVALID_ARG: return "invalid argument";
    case RQ_ERR_UNSUPPORTED: return "unsupported head_dim, group, bits or GQA ratio";
    case RQ_ERR_ALIGNMENT: return "device pointer not 16-byte aligned";
    case RQ_ERR_WORKSPACE: return "workspace missing or too small";
    case RQ_ERR_CUDA: return "CUDA launch or query failed";
  }
  return "unknown status";
}

size_t rq_codes_bytes(const rq_shape* shape, int bits) {
  if (!shape_ok(shape, false) || (bits != 2 && bits != 4 && bits != 8)) return 0;
  const size_t elems =
      (size_t)shape->batch * shape->kv_heads * pitch_of(shape) * (size_t)shape->head_dim;
  return round16(elems * bits / 8);
}

size_t rq_scales_bytes(const rq_shape* shape, int bits) {
  if (!shape_ok(shape, false) || (bits != 2 && bits != 4 && bits != 8)) return 0;
  const size_t groups = (size_t)shape->batch * shape->kv_heads * pitch_of(shape) *
                        (size_t)(shape->head_dim / shape->group);
  return round16(groups * 2);
}

size_t rq_decode_workspace_bytes(const rq_shape* shape) {
  if (!decode_shape_ok(shape)) return 0;
  return decode_workspace_bytes(*shape);
}

rq_status rq_encode_at_ex(const rq_shape* shape, int src_pitch, int src_offset,
                          int dst_pitch, int dst_offset, const uint16_t* const* kv_loops,
                          int n_loops, const uint16_t* ref, const uint8_t* bits_per_loop,
                          uint64_t seed, int refine_iters, uint32_t* const* codes_out,
                          uint16_t* const* scales_out, uint16_t* ref_out, void* stream) {
  if (!shape || !kv_loops || !bits_per_loop || !codes_out || !scales_out)
    return RQ_ERR_INVALID_ARG;
  if (refine_iters < 0 || refine_iters > RQ_MAX_REFINE) return RQ_ERR_INVALID_ARG;
  if (shape->batch < 1 || shape->kv_heads < 1 || shape->ctx < 0) return RQ_ERR_INVALID_ARG;
  if (src_offset < 0 || dst_offset < 0 || src_pitch < 1 || dst_pitch < 1 ||
      (long long)src_offset + shape->ctx > src_pitch ||
      (long long)dst_offset + shape->ctx > dst_pitch)
    return RQ_ERR_INVALID_ARG;
  if (n_loops < 1 || n_loops > RQ_MAX_LOOPS) return RQ_ERR_INVALID_ARG;
  if (!supported_dims(shape->head_dim, shape->group)) return RQ_ERR_UNSUPPORTED;
  if (!ref) return RQ_ERR_INVALID_ARG;
  if (!aligned16(ref) || (ref_out && !aligned16(ref_out))) return RQ_ERR_ALIGNMENT;
  EncodeParams p;
  std::memset(&p, 0, sizeof p);
  int active = 0;
  for (int l = 0; l < n_loops; ++l) {
    const int b = bits_per_loop[l];
    if (b != 2 && b != 4 && b != 16) return RQ_ERR_UNSUPPORTED;
    p.bits[l] = b;
    if (b == 16) continue;
    if (!kv_loops[l] || !codes_out[l] || !scales_out[l]) return RQ_ERR_INVALID_ARG;
    if (!aligned16(kv_loops[l]) || !aligned16(codes_out[l]) || !aligned16(scales_out[l]))
      return RQ_ERR_ALIGNMENT;
    p.x[l] = kv_loops[l];
    p.codes[l] = codes_out[l];
    p.scales[l] = scales_out[l];
    ++active;
  }
  p.ref = ref;
  p.ref_out = ref_out;
  p.n_loops = n_loops;
  p.refine_iters = refine_iters;
  p.kv_heads = shape->kv_heads;
  p.seed = seed;
  p.ctx = shape->ctx;
  p.src_pitch = src_pitch;
  p.src_offset = src_offset;
  p.dst_pitch = dst_pitch;
  p.dst_offset = dst_offset;
  p.n_rows = (long long)shape->batch * shape->kv_heads * shape->ctx;
  if (p.n_rows == 0 || (active == 0 && !ref_out)) return RQ_OK;
  if (!finish_encode_params(p, *shape)) return RQ_ERR_CUDA;
  const int sms = device_sm_count();
  if (sms <= 0) return RQ_ERR_CUDA;
  const bool contiguous = src_pitch == shape->ctx && src_offset == 0 &&
                          p.n_rows <= kEncodeTmaMaxRows;
  cudaError_t e = contiguous ? launch_encode_tma(shape->head_dim, shape->group, p, sms,
                                                 static_cast<cudaStream_t>(stream))
                             : launch_encode(shape->head_dim, shape->group, p, sms,
                                             static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? RQ_OK : RQ_ERR_CUDA;
}

rq_status rq_encode_cr_at(const rq_shape* shape, int dst_pitch, int dst_offset,
                          const uint16_t* const* kv_loops, int n_loops, const uint16_t* ref,
                          int ref_bits, const uint8_t* bits_per_loop, uint64_t seed,
                          uint32_t* ref_codes_out, uint16_t* ref_scales_out,
                          uint32_t* const* codes_out, uint16_t* const* scales_out,
                          void* stream) {
  if (!shape || (n_loops > 0 && (!kv_loops || !bits_per_loop || !codes_out || !scales_out)))
    return RQ_ERR_INVALID_ARG;
  if (shape->batch < 1 || shape->kv_heads < 1 || shape->ctx < 0) return RQ_ERR_INVALID_ARG;
  if (dst_offset < 0 || dst_pitch < 1 || (long long)dst_offset + shape->ctx > dst_pitch)
    return RQ_ERR_INVALID_ARG;
  if (n_loops < 0 || n_loops > RQ_MAX_LOOPS) return RQ_ERR_INVALID_ARG;
  if (ref_bits != 4 && ref_bits != 8) return RQ_ERR_UNSUPPORTED;
  if (!supported_dims(shape->head_dim, shape->group)) return RQ_ERR_UNSUPPORTED;
  if (!ref || !ref_codes_out || !ref_scales_out) return RQ_ERR_INVALID_ARG;
  if (!aligned16(ref) || !aligned16(ref_codes_out) || !aligned16(ref_scales_out))
    return RQ_ERR_ALIGNMENT;
  EncodeParams p;
  std::memset(&p, 0, sizeof p);
  for (int l = 0; l < n_loops; ++l) {
    const int b = bits_per_loop[l];
    if (b != 2 && b != 4 && b != 16) return RQ_ERR_UNSUPPORTED;
    p.bits[l] = b;
    if (b == 16) continue;
    if (!kv_loops[l] || !codes_out[l] || !scales_out[l]) return RQ_ERR_INVALID_ARG;
    if (!aligned16(kv_loops[l]) || !aligned16(codes_out[l]) || !aligned16(scales_out[l]))
      return RQ_ERR_ALIGNMENT;
    p.x[l] = kv_loops[l];
    p.codes[l] = codes_out[l];
    p.scales[l] = scales_out[l];
  }
  p.ref = ref;
  p.ref_bits = ref_bits;
  p.ref_codes = ref_codes_out;
  p.ref_scales = ref_scales_out;
  p.n_loops = n_loops;
  p.kv_heads = shape->kv_heads;
  p.seed = seed;
  p.ctx = shape->ctx;
  p.src_pitch = shape->ctx;
  p.src_offset = 0;
  p.dst_pitch = dst_pitch;
  p.dst_offset = dst_offset;
  p.n_rows = (long long)shape->batch * shape->kv_heads * shape->ctx;
  if (p.n_rows == 0) return RQ_OK;
  if (p.n_rows > kEncodeTmaMaxRows) return RQ_ERR_UNSUPPORTED;
  if (!finish_encode_params(p, *shape)) return RQ_ERR_CUDA;
  const int sms = device_sm_count();
  if (sms <= 0) return RQ_ERR_CUDA;
  cudaError_t e = launch_encode_tma(shape->head_dim, shape->group, p, sms,
                                    static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? RQ_OK : RQ_ERR_CUDA;
}

rq_status rq_encode_paged(const rq_shape* shape, const uint16_t* const* kv_loops, int n_loops,
                          const uint16_t* ref, const uint8_t* bits_per_loop, uint64_t seed,
                          int refine_iters, const int32_t* dst_pos, const int32_t* page_table,
                          int max_pages, int n_pages, uint32_t* const* codes_out,
                          uint16_t* const* scales_out, uint16_t* ref_out, void* stream) {
  if (!shape || !kv_loops || !bits_per_loop || !codes_out || !scales_out || !dst_pos ||
      !page_table)
    return RQ_ERR_INVALID_ARG;
  if (shape->batch < 1 || shape->kv_heads < 1 || shape->ctx < 0) return RQ_ERR_INVALID_ARG;
  if (max_pages < 1 || n_pages < 1) return RQ_ERR_INVALID_ARG;
  if (refine_iters < 0 || refine_iters > RQ_MAX_REFINE) return RQ_ERR_INVALID_ARG;
  if (n_loops < 1 || n_loops > RQ_MAX_LOOPS) return RQ_ERR_INVALID_ARG;
  if (!supported_dims(shape->head_dim, shape->group)) return RQ_ERR_UNSUPPORTED;
  if (!ref) return RQ_ERR_INVALID_ARG;
  if (!aligned16(ref) || (ref_out && !aligned16(ref_out))) return RQ_ERR_ALIGNMENT;
  if ((reinterpret_cast<uintptr_t>(dst_pos) & 3u) || (reinterpret_cast<uintptr_t>(page_table) & 3u))
    return RQ_ERR_ALIGNMENT;
  EncodeParams p;
  std::memset(&p, 0, sizeof p);
  int active = 0;
  for (int l = 0; l < n_loops; ++l) {
    const int b = bits_per_loop[l];
    if (b != 2 && b != 4 && b != 16) return RQ_ERR_UNSUPPORTED;
    p.bits[l] = b;
    if (b == 16) continue;
    if (!kv_loops[l] || !codes_out[l] || !scales_out[l]) return RQ_ERR_INVALID_ARG;
    if (!aligned16(kv_loops[l]) || !aligned16(codes_out[l]) || !aligned16(scales_out[l]))
      return RQ_ERR_ALIGNMENT;
    p.x[l] = kv_loops[l];
    p.codes[l] = codes_out[l];
    p.scales[l] = scales_out[l];
    ++active;
  }
  p.ref = ref;
  p.ref_out = ref_out;
  p.n_loops = n_loops;
  p.refine_iters = refine_iters;
  p.kv_heads = shape->kv_heads;
  p.page_table = page_table;
  p.dst_pos = dst_pos;
  p.max_pages = max_pages;
  p.n_pages = n_pages;
  p.seed = seed;
  p.ctx = shape->ctx;
  p.src_pitch = shape->ctx;
  p.src_offset = 0;
  p.n_rows = (long long)shape->batch * shape->kv_heads * shape->ctx;
  if (p.n_rows == 0 || (active == 0 && !ref_out)) return RQ_OK;
  if (!finish_encode_params(p, *shape)) return RQ_ERR_CUDA;
  const int sms = device_sm_count();
  if (sms <= 0) return RQ_ERR_CUDA;
  cudaError_t e = p.n_rows <= kEncodeTmaMaxRows
                      ? launch_encode_tma(shape->head_dim, shape->group, p, sms,
                                          static_cast<cudaStream_t>(stream))
                      : launch_encode(shape->head_dim, shape->group, p, sms,
                                      static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? RQ_OK : RQ_ERR_CUDA;
}

rq_status rq_encode_at(const rq_shape* shape, int src_pitch, int src_offset, int dst_pitch,
                       int dst_offset, const uint16_t* const* kv_loops, int n_loops,
                       const uint16_t* ref, const uint8_t* bits_per_loop, uint64_t seed,
                       uint32_t* const* codes_out, uint16_t* const* scales_out,
                       uint16_t* ref_out, void* stream) {
  return rq_encode_at_ex(shape, src_pitch, src_offset, dst_pitch, dst_offset, kv_loops, n_loops,
                         ref, bits_per_loop, seed, 0, codes_out, scales_out, ref_out, stream);
}

rq_status rq_encode(const rq_shape* shape, const uint16_t* const* kv_loops, int n_loops,
                    const uint16_t* ref, const uint8_t* bits_per_loop, uint64_t seed,
                    uint32_t* const* codes_out, uint16_t* const* scales_out, void* stream) {
  if (!shape) return RQ_ERR_INVALID_ARG;
  if (shape->ctx_cap != 0 && shape->ctx_cap < shape->ctx) return RQ_ERR_INVALID_ARG;
  const int pitch = pitch_of(shape) > 0 ? pitch_of(shape) : 1;
  return rq_encode_at(shape, pitch, 0, pitch, 0, kv_loops, n_loops, ref, bits_per_loop, seed,
                      codes_out, scales_out, nullptr, stream);
}

}  // extern "C"

namespace {

// Shared body of the decode entry points; ctx_lens null: every sequence has
// shape->ctx cached tokens.
struct Paged {                 // paged cache (table null: dense arrays)
  const int32_t* table = nullptr;
  int max_pages = 0;
  int n_pages = 0;
};

struct CrRef {                 // compressed reference (ref_bits 0: BF16 rows)
  int ref_bits = 0;
  const uint32_t* codes_k = nullptr;
  const uint32_t* codes_v = nullptr;
  const uint16_t* scales_k = nullptr;
  const uint16_t* scales_v = nullptr;
};

rq_status decode_impl(const rq_shape* shape, const int32_t* ctx_lens, const uint16_t* q,
                      const uint16_t* ref_k, const uint16_t* ref_v, const uint32_t* codes_k,
                      const uint32_t* codes_v, const uint16_t* scales_k,
                      const uint16_t* scales_v, int bits, uint64_t seed, float softmax_scale,
                      const uint16_t* tail_k, const uint16_t* tail_v, int n_tail,
                      int tail_pitch, float* out, void* workspace, size_t workspace_bytes,
                      void* stream, const CrRef& cr = CrRef(), const Paged& pg = Paged()) {
  const bool varlen = ctx_lens != nullptr;
  if (pg.table) {
    if (!varlen || !shape) return RQ_ERR_INVALID_ARG;
    if (pg.max_pages < 1 || pg.n_pages < 1) return RQ_ERR_INVALID_ARG;
    if ((long long)pg.max_pages * kDecodeTile != shape->ctx ||
        (shape->ctx_cap != 0 && shape->ctx_cap != shape->ctx))
      return RQ_ERR_INVALID_ARG;
    if (reinterpret_cast<uintptr_t>(pg.table) & 3u) return RQ_ERR_ALIGNMENT;
  }
  if (cr.ref_bits != 0) {
    if (cr.ref_bits != 4 && cr.ref_bits != 8) return RQ_ERR_UNSUPPORTED;
    if (!shape) return RQ_ERR_INVALID_ARG;
    if (!cr.codes_k || !cr.codes_v || !cr.scales_k || !cr.scales_v) return RQ_ERR_INVALID_ARG;
    if (!aligned16(cr.codes_k) || !aligned16(cr.codes_v) || !aligned16(cr.scales_k) ||
        !aligned16(cr.scales_v))
      return RQ_ERR_ALIGNMENT;
    // the reference rows are not read: stand-ins keep the checks below uniform
    ref_k = reinterpret_cast<const uint16_t*>(cr.codes_k);
    ref_v = reinterpret_cast<const uint16_t*>(cr.codes_v);
  }
  if (!shape) return RQ_ERR_INVALID_ARG;
  if (shape->batch < 1 || shape->kv_heads < 1 || shape->ctx < 1 ||
      shape->q_heads < shape->kv_heads)
    return RQ_ERR_INVALID_ARG;
  if (varlen && shape->batch > RQ_MAX_VARLEN_BATCH) return RQ_ERR_INVALID_ARG;
  if (varlen && (reinterpret_cast<uintptr_t>(ctx_lens) & 3u)) return RQ_ERR_ALIGNMENT;
  if (shape->ctx_cap != 0 && shape->ctx_cap < shape->ctx) return RQ_ERR_INVALID_ARG;
  if (n_tail < 0 || n_tail > RQ_MAX_TAIL) return RQ_ERR_INVALID_ARG;
  if (n_tail > 0 && (!tail_k || !tail_v || tail_pitch < n_tail)) return RQ_ERR_INVALID_ARG;
  if (n_tail > 0 && (!aligned16(tail_k) || !aligned16(tail_v))) return RQ_ERR_ALIGNMENT;
  if (shape->q_heads % shape->kv_heads) return RQ_ERR_INVALID_ARG;
  if (!decode_shape_ok(shape)) return RQ_ERR_UNSUPPORTED;
  if (bits != 2 && bits != 4 && bits != 16) return RQ_ERR_UNSUPPORTED;
  if (!q || !ref_k || !ref_v || !out) return RQ_ERR_INVALID_ARG;
  if (bits != 16 && (!codes_k || !codes_v || !scales_k || !scales_v)) return RQ_ERR_INVALID_ARG;
  if (!(softmax_scale <= 0.0f || std::isfinite(softmax_scale))) return RQ_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(ref_k) || !aligned16(ref_v) || !aligned16(out))
    return RQ_ERR_ALIGNMENT;
  if (bits != 16 && (!aligned16(codes_k) || !aligned16(codes_v) || !aligned16(scales_k) ||
                     !aligned16(scales_v)))
    return RQ_ERR_ALIGNMENT;
  if (!workspace || workspace_bytes < decode_workspace_bytes(*shape, varlen))
    return RQ_ERR_WORKSPACE;
  if (!aligned16(workspace)) return RQ_ERR_ALIGNMENT;

  const int sms = device_sm_count();
  if (sms <= 0) return RQ_ERR_CUDA;
  const DecodePlan pl = plan_decode(*shape, sms, varlen);
  const int G = shape->q_heads / shape->kv_heads;
  DecodeParams p;
  p.q = q;
  p.ref_k = ref_k;
  p.ref_v = ref_v;
  p.codes_k = bits == 16 ? nullptr : codes_k;
  p.codes_v = bits == 16 ? nullptr : codes_v;
  p.scales_k = bits == 16 ? nullptr : scales_k;
  p.scales_v = bits == 16 ? nullptr : scales_v;
  p.out = out;
  unsigned char* ws = static_cast<unsigned char*>(workspace);
  p.status = reinterpret_cast<uint32_t*>(ws);
  p.counters = reinterpret_cast<uint32_t*>(ws + kWsHeaderBytes);
  p.records = reinterpret_cast<float*>(ws + kWsHeaderBytes + ws_counters_bytes(pl.heads));
  p.batch = shape->batch;
  p.kv_heads = shape->kv_heads;
  p.q_heads = shape->q_heads;
  p.ctx = shape->ctx;
  p.group = shape->group;
  p.ctx_pitch = pitch_of(shape);
  p.tail_k = n_tail > 0 ? tail_k : nullptr;
  p.tail_v = n_tail > 0 ? tail_v : nullptr;
  p.n_tail = n_tail;
  p.tail_pitch = n_tail > 0 ? tail_pitch : 0;
  p.ctx_lens = ctx_lens;
  if (varlen) p.ctx = pitch_of(shape);
  p.page_table = pg.table;
  p.max_pages = pg.max_pages;
  p.n_pages = pg.n_pages;
  p.ref_bits = cr.ref_bits;
  p.rcodes_k = cr.codes_k;
  p.rcodes_v = cr.codes_v;
  p.rscales_k = cr.scales_k;
  p.rscales_v = cr.scales_v;
  p.nt = pl.nt;
  p.n_tiles = pl.n_tiles;
  p.ctas = pl.ctas;
  p.max_contrib = pl.max_contrib;
  p.seed = seed;
  const float sigma =
      softmax_scale > 0.0f ? softmax_scale : 1.0f / std::sqrt((float)shape->head_dim);
  p.score_scale = sigma * 1.4426950408889634f;   // log2(e)
  cudaError_t e = (G == 1)
                      ? launch_decode(shape->head_dim, G, bits, p, static_cast<cudaStream_t>(stream))
                      : launch_decode_gqa(shape->head_dim, G, bits, p,
                                          static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? RQ_OK : RQ_ERR_CUDA;
}

}  // namespace

extern "C" {

rq_status rq_decode_attention_tail(const rq_shape* shape, const uint16_t* q,
                                   const uint16_t* ref_k, const uint16_t* ref_v,
                                   const uint32_t* codes_k, const uint32_t* codes_v,
                                   const uint16_t* scales_k, const uint16_t* scales_v, int bits,
                                   uint64_t seed, float softmax_scale, const uint16_t* tail_k,
                                   const uint16_t* tail_v, int n_tail, int tail_pitch,
                                   float* out, void* workspace, size_t workspace_bytes,
                                   void* stream) {
  return decode_impl(shape, nullptr, q, ref_k, ref_v, codes_k, codes_v, scales_k, scales_v, bits,
                     seed, softmax_scale, tail_k, tail_v, n_tail, tail_pitch, out, workspace,
                     workspace_bytes, stream);
}

rq_status rq_decode_attention_varlen(const rq_shape* shape, const int32_t* ctx_lens,
                                     const uint16_t* q, const uint16_t* ref_k,
                                     const uint16_t* ref_v, const uint32_t* codes_k,
                                     const uint32_t* codes_v, const uint16_t* scales_k,
                                     const uint16_t* scales_v, int bits, uint64_t seed,
                                     float softmax_scale, const uint16_t* tail_k,
                                     const uint16_t* tail_v, int n_tail, int tail_pitch,
                                     float* out, void* workspace, size_t workspace_bytes,
                                     void* stream) {
  if (!ctx_lens) return RQ_ERR_INVALID_ARG;
  return decode_impl(shape, ctx_lens, q, ref_k, ref_v, codes_k, codes_v, scales_k, scales_v,
                     bits, seed, softmax_scale, tail_k, tail_v, n_tail, tail_pitch, out,
                     workspace, workspace_bytes, stream);
}

rq_status rq_decode_attention_cr(const rq_shape* shape, const int32_t* ctx_lens,
                                 const uint16_t* q, const uint32_t* ref_codes_k,
                                 const uint32_t* ref_codes_v, const uint16_t* ref_scales_k,
                                 const uint16_t* ref_scales_v, int ref_bits,
                                 const uint32_t* codes_k, const uint32_t* codes_v,
                                 const uint16_t* scales_k, const uint16_t* scales_v, int bits,
                                 uint64_t seed, float softmax_scale, const uint16_t* tail_k,
                                 const uint16_t* tail_v, int n_tail, int tail_pitch, float* out,
                                 void* workspace, size_t workspace_bytes, void* stream) {
  CrRef cr;
  cr.ref_bits = ref_bits;
  cr.codes_k = ref_codes_k;
  cr.codes_v = ref_codes_v;
  cr.scales_k = ref_scales_k;
  cr.scales_v = ref_scales_v;
  if (ref_bits != 4 && ref_bits != 8) return RQ_ERR_UNSUPPORTED;
  return decode_impl(shape, ctx_lens, q, nullptr, nullptr, codes_k, codes_v, scales_k, scales_v,
                     bits, seed, softmax_scale, tail_k, tail_v, n_tail, tail_pitch, out,
                     workspace, workspace_bytes, stream, cr);
}

rq_status rq_decode_attention_paged(const rq_shape* shape, const int32_t* ctx_lens,
                                    const int32_t* page_table, int max_pages, int n_pages,
                                    const uint16_t* q, const uint16_t* ref_k,
                                    const uint16_t* ref_v, const uint32_t* codes_k,
                                    const uint32_t* codes_v, const uint16_t* scales_k,
                                    const uint16_t* scales_v, int bits, uint64_t seed,
                                    float softmax_scale, const uint16_t* tail_k,
                                    const uint16_t* tail_v, int n_tail, int tail_pitch, float* out,
                                    void* workspace, size_t workspace_bytes, void* stream) {
  if (!ctx_lens || !page_table) return RQ_ERR_INVALID_ARG;
  Paged pg;
  pg.table = page_table;
  pg.max_pages = max_pages;
  pg.n_pages = n_pages;
  return decode_impl(shape, ctx_lens, q, ref_k, ref_v, codes_k, codes_v, scales_k, scales_v, bits,
                     seed, softmax_scale, tail_k, tail_v, n_tail, tail_pitch, out, workspace,
                     workspace_bytes, stream, CrRef(), pg);
}

size_t rq_decode_workspace_bytes_varlen(const rq_shape* shape) {
  if (!decode_shape_ok(shape) || shape->batch > RQ_MAX_VARLEN_BATCH) return 0;
  return decode_workspace_bytes(*shape, true);
}

rq_status rq_decode_attention(const rq_shape* shape, const uint16_t* q, const uint16_t* ref_k,
                              const uint16_t* ref_v, const uint32_t* codes_k,
                              const uint32_t* codes_v, const uint16_t* scales_k,
                              const uint16_t* scales_v, int bits, uint64_t seed,
                              float softmax_scale, float* out, void* workspace,
                              size_t workspace_bytes, void* stream) {
  return rq_decode_attention_tail(shape, q, ref_k, ref_v, codes_k, codes_v, scales_k, scales_v,
                                  bits, seed, softmax_scale, nullptr, nullptr, 0, 0, out,
                                  workspace, workspace_bytes, stream);
}

rq_status rq_reconstruct(const rq_shape* shape, const uint16_t* ref, const uint32_t* codes,
                         const uint16_t* scales, int bits, uint64_t seed, void* out, int out_bf16,
                         void* stream) {
  if (!shape || !ref || !out) return RQ_ERR_INVALID_ARG;
  if (shape->batch < 1 || shape->kv_heads < 1 || shape->ctx < 0) return RQ_ERR_INVALID_ARG;
  if (shape->ctx_cap != 0 && shape->ctx_cap < shape->ctx) return RQ_ERR_INVALID_ARG;
  if (!supported_dims(shape->head_dim, shape->group)) return RQ_ERR_UNSUPPORTED;
  if (bits != 2 && bits != 4 && bits != 16) return RQ_ERR_UNSUPPORTED;
  if (bits != 16 && (!codes || !scales)) return RQ_ERR_INVALID_ARG;
  if (!aligned16(ref) || !aligned16(out) ||
      (bits != 16 && (!aligned16(codes) || !aligned16(scales))))
    return RQ_ERR_ALIGNMENT;
  ReconstructParams p;
  std::memset(&p, 0, sizeof p);
  p.ref = ref;
  p.codes = bits == 16 ? nullptr : codes;
  p.scales = bits == 16 ? nullptr : scales;
  p.out = out;
  p.ctx = shape->ctx;
  p.pitch = pitch_of(shape);
  p.n_rows = (long long)shape->batch * shape->kv_heads * shape->ctx;
  p.out_bf16 = out_bf16 ? 1 : 0;
  p.seed = seed;
  if (p.n_rows == 0) return RQ_OK;
  p.status = encode_status_ptr();
  if (!p.status) return RQ_ERR_CUDA;
  const int sms = device_sm_count();
  if (sms <= 0) return RQ_ERR_CUDA;
  cudaError_t e = launch_reconstruct(shape->head_dim, shape->group, bits, p, sms,
                                     static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? RQ_OK : RQ_ERR_CUDA;
}

rq_status rq_reconstruct_cr(const rq_shape* shape, const uint32_t* ref_codes,
                            const uint16_t* ref_scales, int ref_bits, const uint32_t* codes,
                            const uint16_t* scales, int bits, uint64_t seed, void* out,
                            int out_bf16, void* stream) {
  if (!shape || !ref_codes || !ref_scales || !out) return RQ_ERR_INVALID_ARG;
  if (shape->batch < 1 || shape->kv_heads < 1 || shape->ctx < 0) return RQ_ERR_INVALID_ARG;
  if (shape->ctx_cap != 0 && shape->ctx_cap < shape->ctx) return RQ_ERR_INVALID_ARG;
  if (!supported_dims(shape->head_dim, shape->group)) return RQ_ERR_UNSUPPORTED;
  if (ref_bits != 4 && ref_bits != 8) return RQ_ERR_UNSUPPORTED;
  if (bits != 2 && bits != 4 && bits != 16) return RQ_ERR_UNSUPPORTED;
  if (bits != 16 && (!codes || !scales)) return RQ_ERR_INVALID_ARG;
  if (!aligned16(ref_codes) || !aligned16(ref_scales) || !aligned16(out) ||
      (bits != 16 && (!aligned16(codes) || !aligned16(scales))))
    return RQ_ERR_ALIGNMENT;
  ReconstructParams p;
  std::memset(&p, 0, sizeof p);
  p.ref_codes = ref_codes;
  p.ref_scales = ref_scales;
  p.codes = bits == 16 ? nullptr : codes;
  p.scales = bits == 16 ? nullptr : scales;
  p.out = out;
  p.ctx = shape->ctx;
  p.pitch = pitch_of(shape);
  p.n_rows = (long long)shape->batch * shape->kv_heads * shape->ctx;
  p.out_bf16 = out_bf16 ? 1 : 0;
  p.seed = seed;
  if (p.n_rows == 0) return RQ_OK;
  p.status = encode_status_ptr();
  if (!p.status) return RQ_ERR_CUDA;
  const int sms = device_sm_count();
  if (sms <= 0) return RQ_ERR_CUDA;
  cudaError_t e = launch_reconstruct_cr(shape->head_dim, shape->group, ref_bits, bits, p, sms,
                                        static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? RQ_OK : RQ_ERR_CUDA;
}

rq_status rq_encode_take_status(uint32_t* host_status) {
  if (!host_status) return RQ_ERR_INVALID_ARG;
  if (cudaDeviceSynchronize() != cudaSuccess) return RQ_ERR_CUDA;
  return encode_take_status(host_status) == cudaSuccess ? RQ_OK : RQ_ERR_CUDA;
}

rq_status rq_workspace_status(const void* workspace, size_t workspace_bytes,
                              uint32_t* host_status, void* stream) {
  if (!workspace || !host_status || workspace_bytes < kWsHeaderBytes) return RQ_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaMemcpyAsync(host_status, workspace, sizeof(uint32_t), cudaMemcpyDeviceToHost, st) !=
      cudaSuccess)
    return RQ_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return RQ_ERR_CUDA;
  return RQ_OK;
}

}  // extern "C"
