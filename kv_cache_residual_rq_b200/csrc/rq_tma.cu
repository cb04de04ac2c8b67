// rq_tma.cu -- TMA tensor maps for the kernels that stream [rows][head_dim]
// bf16 arrays through the tensor-copy engine.
//
// The encode entry point of the driver is looked up once through the
// runtime (no link-time dependency on libcuda).  A map views a row-major
// [rows][d] bf16 array as 2-D (x = dimension, y = row), box = 64 columns x
// box_rows rows (one 128-byte line per row), with the 128-byte swizzle so
// that threads reading 16-byte chunks of eight consecutive rows hit eight
// different bank groups.  Rows past the end of the array read as zeros.
// A byte map views [rows][row_bytes] bytes (row_bytes 32, 64 or 128) the same way,
// one whole row per box line, with the swizzle of the line's width.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "rq_internal.h"

namespace rq {
namespace {

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult qres;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &qres) ==
            cudaSuccess &&
        qres == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
  });
  return fn;
}

}  // namespace

bool encode_rows_map(CUtensorMap* map, const void* base, unsigned long long rows, int d,
                     int box_rows) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
  if (!enc || rows == 0 || box_rows < 1 || box_rows > 256) return false;
  cuuint64_t dims[2] = {(cuuint64_t)d, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)d * 2};
  cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims,
                   strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool encode_bytes_map(CUtensorMap* map, const void* base, unsigned long long rows, int row_bytes,
                      int box_rows) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
  if (!enc || rows == 0 || box_rows < 1 || box_rows > 256) return false;
  if (row_bytes != 32 && row_bytes != 64 && row_bytes != 128) return false;
  cuuint64_t dims[2] = {(cuuint64_t)row_bytes, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)row_bytes};
  cuuint32_t box[2] = {(cuuint32_t)row_bytes, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides,
                   box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   row_bytes == 128  ? CU_TENSOR_MAP_SWIZZLE_128B
                   : row_bytes == 64 ? CU_TENSOR_MAP_SWIZZLE_64B
                                     : CU_TENSOR_MAP_SWIZZLE_32B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

}  // namespace rq
