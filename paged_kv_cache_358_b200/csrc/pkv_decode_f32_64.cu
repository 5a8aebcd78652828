// Decode partition-kernel variants for f32 pools with head_dim 64.
#include "pkv_decode_kernels.cuh"

namespace pkv {

int run_f32_64(const Geometry& geo, const DecodeArgs& args, const void* k, const void* v,
                 cudaStream_t stream) {
  return run_decode<float, 64>(geo, args, k, v, stream);
}

}  // namespace pkv
