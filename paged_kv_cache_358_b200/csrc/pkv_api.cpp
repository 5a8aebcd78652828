// Version, status strings and per-thread CUDA error text of libpkv.
#include <cuda_runtime.h>

#include <cstdio>
#include <cstring>

#include "../../include/pkv.h"
#include "pkv_host.h"

namespace host {

namespace {
thread_local char g_err[256] = {0};
}

void set_error(const char* msg) {
  std::snprintf(g_err, sizeof(g_err), "%s", msg ? msg : "");
}

const char* last_error() { return g_err; }

int cuda_fail(cudaError_t e) {
  std::snprintf(g_err, sizeof(g_err), "%s: %s", cudaGetErrorName(e), cudaGetErrorString(e));
  return PKV_ERR_CUDA;
}

int check_launch() {
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? PKV_OK : cuda_fail(e);
}

}  // namespace host

extern "C" {

const char* pkv_version(void) { return "pkv 0.1.0 sm_100a"; }

const char* pkv_status_string(int status) {
  switch (status) {
    case PKV_OK: return "ok";
    case PKV_ERR_NO_BLOCKS: return "no free blocks";
    case PKV_ERR_INVALID: return "invalid argument";
    case PKV_ERR_CUDA: return "cuda error";
    case PKV_ERR_DEVICE_TIMEOUT: return "device wait timed out";
    case PKV_ERR_BAD_TABLE: return "block table entry out of range";
    case PKV_ERR_PLAN_MISMATCH: return "plan made for other sizes";
  }
  return "unknown status";
}

const char* pkv_last_cuda_error(void) { return host::last_error(); }

}  // extern "C"
