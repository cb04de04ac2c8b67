// rq_decode_gqa_d64_r8.cu -- the grouped-query decode kernel's instances for
// head_dim 64 and an INT8 compressed reference (one translation unit each, compiled in
// parallel).
#define RQ_GQA_KERNEL_DEFINITIONS
#include "rq_decode_gqa.cuh"

namespace rq {

cudaError_t launch_gqa_d64_r8(int G, int bits, const TcParams& gp, cudaStream_t stream) {
  return launch_gqa_d<64, 8>(G, bits, gp, stream);
}

}  // namespace rq
