// Decode partition-kernel variants for bf16 pools with head_dim 256.
#include "pkv_decode_kernels.cuh"

namespace pkv {

int run_bf16_256(const Geometry& geo, const DecodeArgs& args, const void* k, const void* v,
                 cudaStream_t stream) {
  return run_decode<__nv_bfloat16, 256>(geo, args, k, v, stream);
}

}  // namespace pkv
