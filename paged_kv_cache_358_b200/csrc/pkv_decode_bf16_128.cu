// Decode partition-kernel variants for bf16 pools with head_dim 128.
#include "pkv_decode_kernels.cuh"

namespace pkv {

int run_bf16_128(const Geometry& geo, const DecodeArgs& args, const void* k, const void* v,
                 cudaStream_t stream) {
  return run_decode<__nv_bfloat16, 128>(geo, args, k, v, stream);
}

}  // namespace pkv
