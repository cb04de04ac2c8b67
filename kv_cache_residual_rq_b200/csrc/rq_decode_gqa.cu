// rq_decode_gqa.cu -- host entry of the grouped-query decode kernel
// (rq_decode_gqa.cuh): tensor maps of the call's reference rows, then the
// launch of the instance for its head size and reference type.
#include "rq_decode_gqa.cuh"

namespace rq {

cudaError_t launch_decode_gqa(int head_dim, int G, int bits, const DecodeParams& p,
                              cudaStream_t stream) {
  TcParams gp;
  gp.p = p;
  const unsigned long long rows =
      p.page_table ? (unsigned long long)p.n_pages * p.kv_heads * kDecodeTile
                   : (unsigned long long)p.batch * p.kv_heads * p.ctx_pitch;
  // tensor-copy row coordinates are 32-bit signed
  if (rows > 0x7FFFFFFFull) return cudaErrorInvalidValue;
  if (p.ref_bits == 8 || p.ref_bits == 4) {
    // the reference is code rows of head_dim * ref_bits / 8 bytes
    const int rrow = head_dim * p.ref_bits / 8;
    if (!encode_bytes_map(&gp.tmap_k, p.rcodes_k, rows, rrow, kDecodeTile) ||
        !encode_bytes_map(&gp.tmap_v, p.rcodes_v, rows, rrow, kDecodeTile))
      return cudaErrorInvalidValue;
    if (p.ref_bits == 8) {
      if (head_dim == 128) return launch_gqa_d128_r8(G, bits, gp, stream);
      if (head_dim == 64) return launch_gqa_d64_r8(G, bits, gp, stream);
    } else {
      if (head_dim == 128) return launch_gqa_d128_r4(G, bits, gp, stream);
      if (head_dim == 64) return launch_gqa_d64_r4(G, bits, gp, stream);
    }
    return cudaErrorInvalidValue;
  }
  if (p.ref_bits != 0) return cudaErrorInvalidValue;
  if (!encode_rows_map(&gp.tmap_k, p.ref_k, rows, head_dim, kDecodeTile) ||
      !encode_rows_map(&gp.tmap_v, p.ref_v, rows, head_dim, kDecodeTile))
    return cudaErrorInvalidValue;
  if (head_dim == 128) return launch_gqa_d128_r0(G, bits, gp, stream);
  if (head_dim == 64) return launch_gqa_d64_r0(G, bits, gp, stream);
  return cudaErrorInvalidValue;
}

}  // namespace rq
