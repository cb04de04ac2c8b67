// rq_decode_gqa_d128_r4.cu -- the grouped-query decode kernel's instances for
// head_dim 128 and an INT4 compressed reference (one translation unit each, compiled in
// parallel).
#define RQ_GQA_KERNEL_DEFINITIONS
#include "rq_decode_gqa.cuh"

namespace rq {

cudaError_t launch_gqa_d128_r4(int G, int bits, const TcParams& gp, cudaStream_t stream) {
  return launch_gqa_d<128, 4>(G, bits, gp, stream);
}

}  // namespace rq
