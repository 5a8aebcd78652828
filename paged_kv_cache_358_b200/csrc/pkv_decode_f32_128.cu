// Decode partition-kernel variants for f32 pools with head_dim 128.
#include "pkv_decode_kernels.cuh"

namespace pkv {

int run_f32_128(const Geometry& geo, const DecodeArgs& args, const void* k, const void* v,
                 cudaStream_t stream) {
  return run_decode<float, 128>(geo, args, k, v, stream);
}

}  // namespace pkv
