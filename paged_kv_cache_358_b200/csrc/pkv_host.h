// Host-side helpers shared by the libpkv translation units: per-thread error
// text and CUDA error mapping.
#pragma once

#include <cuda_runtime.h>

namespace host {

void set_error(const char* msg);
const char* last_error();
// Record the CUDA error text and return PKV_ERR_CUDA.
int cuda_fail(cudaError_t e);
// Check the last kernel launch: PKV_OK or PKV_ERR_CUDA.
int check_launch();

}  // namespace host
