// Host plumbing of libhpcdecode: error messages, status strings, device queries.
#include <stdarg.h>
#include <stdio.h>

#include <mutex>

#include "hpc_common.cuh"

namespace hpc {

namespace {
thread_local char g_last_error[512] = "";
}

void set_error(const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_last_error, sizeof(g_last_error), fmt, ap);
  va_end(ap);
}

int fail(int code, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_last_error, sizeof(g_last_error), fmt, ap);
  va_end(ap);
  return code;
}

int check_launch(const char* what) {
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return fail(HPC_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
  return HPC_OK;
}

int device_sm_count() {
  static int cache[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (dev >= 0 && dev < 64 && cache[dev] > 0) return cache[dev];
  int n = 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  if (dev >= 0 && dev < 64) cache[dev] = n;
  return n;
}

}  // namespace hpc

extern "C" const char* hpc_status_string(int status) {
  switch (status) {
    case HPC_OK: return "ok";
    case HPC_ERR_ARG: return "invalid argument";
    case HPC_ERR_SHAPE: return "unsupported shape";
    case HPC_ERR_DTYPE: return "unsupported dtype";
    case HPC_ERR_ALIGN: return "misaligned pointer";
    case HPC_ERR_CUDA: return "CUDA error";
    case HPC_ERR_CAPACITY: return "buffer too small";
    default: return "unknown status";
  }
}

extern "C" const char* hpc_last_error(void) { return hpc::g_last_error; }

extern "C" int hpc_abi_version(void) { return HPC_DECODE_ABI_VERSION; }
