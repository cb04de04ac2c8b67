// rq_internal.h -- launch parameters shared by the C ABI layer and the kernels.
#pragma once

#include <cstddef>
#include <cstdint>
#include <utility>
#include <cuda.h>
#include <cuda_runtime.h>

#include "rq.h"

namespace rq {

// Launch with programmatic stream serialization: the kernel may be scheduled
// while the previous kernel of the stream is finishing, and waits for it
// (pdl_wait_prev) before touching global memory.  Only for kernels that call
// pdl_wait_prev first.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), unsigned grid, unsigned block, size_t smem,
                       cudaStream_t stream, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(block);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, args...);
  if (e == cudaErrorNotSupported || e == cudaErrorInvalidValue) {
    // a stream that cannot take the attribute: plain stream order (the
    // kernel's wait then returns at once)
    (void)cudaGetLastError();
    cfg.numAttrs = 0;
    e = cudaLaunchKernelEx(&cfg, kernel, args...);
  }
  return e;
}

// ---------------------------------------------------------------------------
// encoder
// ---------------------------------------------------------------------------
struct EncodeParams {
  const uint16_t* x[RQ_MAX_LOOPS];   // bf16 rows of each non-final loop
  uint32_t* codes[RQ_MAX_LOOPS];
  uint16_t* scales[RQ_MAX_LOOPS];
  int bits[RQ_MAX_LOOPS];
  const uint16_t* ref;               // bf16 rows of the final loop
  uint16_t* ref_out;                 // optional copy of the reference rows
  long long n_rows;                  // (head, token) rows to encode = heads * ctx
  int ctx;                           // tokens per head in this call
  int src_pitch, src_offset;         // token pitch / first token of the inputs
  int dst_pitch, dst_offset;         // token pitch / first token of the outputs
  int n_loops;
  int refine_iters;                  // least-squares refits after the absmax codes
  int kv_heads;                      // heads per row of the shape (paged destinations)
  const int* page_table;             // paged destination pools: page of token block j of
  const int* dst_pos;                //   sequence b at [b * max_pages + j]; first position
  int max_pages, n_pages;            //   written per sequence; null for dense outputs
  int ref_bits;                      // 0: BF16 reference; 4 or 8: compressed reference
  uint32_t* ref_codes;               // compressed reference: codes and scales out
  uint16_t* ref_scales;
  uint64_t seed;
  // extents the bounds-checked build tests indices against: rows of the
  // sources (heads * src_pitch) and of the outputs (heads * dst_pitch, or a
  // paged pool's n_pages * kv_heads * 64), and the encoders' status word
  long long n_src_rows, n_dst_rows;
  uint32_t* status;
};

#ifdef __CUDACC__
// Destination row of token t of head hd (hd = b * kv_heads + h).  Dense
// outputs: hd * dst_pitch + dst_offset + t.  Paged pools of 64-token pages:
// position pos = dst_pos[b] + t of sequence b lives in page page_table[b][pos / 64]
// at row (page * kv_heads + h) * 64 + pos % 64.  Returns false -- nothing is
// written -- for a position past the table or a page id outside the pool.
__device__ __forceinline__ bool enc_dst_row(const EncodeParams& p, long long hd, long long t,
                                            long long& row) {
  if (!p.page_table) {
    row = hd * p.dst_pitch + p.dst_offset + t;
    return true;
  }
  const long long b = hd / p.kv_heads, h = hd - b * p.kv_heads;
  const long long pos = (long long)p.dst_pos[b] + t;
  if (pos < 0 || pos >= (long long)p.max_pages * 64) return false;
  const int page = p.page_table[b * p.max_pages + pos / 64];
  if (page < 0 || page >= p.n_pages) return false;
  row = ((long long)page * p.kv_heads + h) * 64 + pos % 64;
  return true;
}
#endif

// streaming encoder: any token pitch and offset (rq_encode.cu)
cudaError_t launch_encode(int head_dim, int group, const EncodeParams& p, int num_sms,
                          cudaStream_t stream);
// encoder fed by tensor copies: every source a contiguous [n_rows][head_dim]
// block (src_pitch == ctx, src_offset == 0), n_rows <= kEncodeTmaMaxRows
// (rq_encode_tma.cu)
constexpr long long kEncodeTmaMaxRows = (1ll << 31) - 512;
cudaError_t launch_encode_tma(int head_dim, int group, const EncodeParams& p, int num_sms,
                              cudaStream_t stream);
// its least-squares-refit and compressed-reference modes (called by
// launch_encode_tma; rq_encode_tma_fixed.cu)
cudaError_t launch_encode_tma_fixed(int head_dim, int group, const EncodeParams& p, int num_sms,
                                    cudaStream_t stream);
// read and clear the sticky error bits of the encoders on the current device
cudaError_t encode_take_status(uint32_t* bits);
// device address of that status word on the current device (looked up once
// per device); null if the runtime cannot provide it
uint32_t* encode_status_ptr();

// ---------------------------------------------------------------------------
// reconstruction (the format's decoder)
// ---------------------------------------------------------------------------
struct ReconstructParams {
  const uint16_t* ref;        // BF16 reference rows (null for a compressed reference)
  const uint32_t* ref_codes;  // compressed reference: codes and fp16 scales
  const uint16_t* ref_scales;
  const uint32_t* codes;      // unused for bits 16
  const uint16_t* scales;
  void* out;                  // fp32 or bf16 rows
  long long n_rows;           // heads * ctx
  int ctx, pitch;
  int out_bf16;
  uint64_t seed;
  uint32_t* status;           // the encoders' status word (bounds-checked build)
};

cudaError_t launch_reconstruct(int head_dim, int group, int bits, const ReconstructParams& p,
                               int num_sms, cudaStream_t stream);
// compressed reference with ref_bits (4 or 8); bits 16 = the reference loop
cudaError_t launch_reconstruct_cr(int head_dim, int group, int ref_bits, int bits,
                                  const ReconstructParams& p, int num_sms, cudaStream_t stream);

// ---------------------------------------------------------------------------
// decode attention
// ---------------------------------------------------------------------------

// Work split of one decode call.  The context of each (batch, kv head) --
// a "head" -- is cut into tiles of kDecodeTile tokens; the heads' tiles are
// numbered head-major and the P CTAs take equal contiguous runs of that
// numbering, so every CTA streams the same number of tiles whatever the
// shape.  A head touched by several CTAs is merged by the last to finish.
constexpr int kDecodeTile = 64;
constexpr int kDecodeCtasPerSm = 2;
constexpr int kDecodeMaxCtas = 1024;     // bound used to size the workspace
constexpr int kVarlenMaxBatch = 1024;    // sequences of a variable-length call
static_assert(kVarlenMaxBatch == RQ_MAX_VARLEN_BATCH, "one limit");

struct DecodePlan {
  long long heads;      // batch * kv_heads
  int nt;               // tiles per head
  long long n_tiles;    // heads * nt
  int ctas;             // P
  int max_contrib;      // partial records reserved per head
};

// Host arithmetic shared by the size query and the launch.
// varlen: the tile count is known only on the device; the plan then holds
// the CTA count and a record bound that holds for any lengths <= capacity.
DecodePlan plan_decode(const rq_shape& s, int num_sms, bool varlen = false);
size_t decode_workspace_bytes(const rq_shape& s, bool varlen = false);

// Workspace layout: [status u32, pad to 16][counters u32 per head, pad to 16]
//                   [partial records: heads * max_contrib * G records]
// A record is {m, l, pad, pad, accRef[d], accRes[d]} as fp32.
constexpr size_t kWsHeaderBytes = 16;
inline size_t ws_counters_bytes(long long heads) {
  return ((size_t)heads * 4 + 15) / 16 * 16;
}
inline size_t ws_record_floats(int head_dim) { return 4 + 2 * (size_t)head_dim; }

struct DecodeParams {
  const uint16_t* q;
  const uint16_t* ref_k;
  const uint16_t* ref_v;
  const uint32_t* codes_k;
  const uint32_t* codes_v;
  const uint16_t* scales_k;
  const uint16_t* scales_v;
  float* out;
  uint32_t* status;
  uint32_t* counters;
  float* records;
  int batch, kv_heads, q_heads, ctx, group;
  int ctx_pitch;         // token pitch of ref/codes/scales per head (>= ctx)
  const uint16_t* tail_k;   // optional BF16 tail tokens [heads][tail_pitch][d]
  const uint16_t* tail_v;
  int n_tail, tail_pitch;
  int ref_bits;          // 0: BF16 reference rows; 4 or 8: compressed reference
  const uint32_t* rcodes_k;   // compressed reference: codes and fp16 scales
  const uint32_t* rcodes_v;
  const uint16_t* rscales_k;
  const uint16_t* rscales_v;
  const int* page_table; // paged cache: page of tile j of sequence b at
  int max_pages, n_pages; //   [b * max_pages + j], pool of n_pages pages; else null
  const int* ctx_lens;   // variable-length call: cached tokens per sequence
                         // [batch] (device int32), else null (ctx for all)
  int nt;
  long long n_tiles;
  int ctas;
  int max_contrib;
  uint64_t seed;
  float score_scale;     // softmax scale * log2(e)
};

// one query row per kv head (CUDA cores)
cudaError_t launch_decode(int head_dim, int G, int bits, const DecodeParams& p,
                          cudaStream_t stream);
// grouped queries, G in {2, 4, 8} (tensor cores, TMA tensor copies)
cudaError_t launch_decode_gqa(int head_dim, int G, int bits, const DecodeParams& p,
                              cudaStream_t stream);
// one query row per kv head over a compressed reference (p.ref_bits 4 or 8):
// the tensor-core kernel (rq_decode_cr1.cu)
cudaError_t launch_decode_cr1(int head_dim, int bits, const DecodeParams& p, cudaStream_t stream);

int device_sm_count();   // SMs of the current device, cached per device

// TMA map of a row-major [rows][d] bf16 array: box 64 columns x box_rows
// rows, 128-byte swizzle, rows past the end read as zeros (rq_tma.cu).
bool encode_rows_map(CUtensorMap* map, const void* base, unsigned long long rows, int d,
                     int box_rows);
// TMA map of a row-major [rows][row_bytes] byte array (row_bytes 32, 64 or
// 128): box = whole rows x box_rows, swizzle of the row's width.
bool encode_bytes_map(CUtensorMap* map, const void* base, unsigned long long rows, int row_bytes,
                      int box_rows);

}  // namespace rq
