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

// ---- diagnostic of the bounded waits
// Every pipeline wait in the library is mbar_wait with a time limit. This kernel runs that same
// wait on a barrier phase that either completes at once (arrive != 0) or never completes
// (arrive == 0), so that a caller can see the give-up path work on its device: the wait
// returns false after limit_ns, HPC_DEV_TIMEOUT lands in the status word, and the kernel ends
// normally. No trap, no fault; the context stays usable.
namespace hpc {
namespace {
__global__ void __launch_bounds__(32, 1)
    wait_selftest_kernel(uint64_t limit_ns, int arrive, uint32_t* status, uint64_t* waited_ns) {
  __shared__ uint64_t bar;
  const uint32_t b = smem_u32(&bar);
  if (threadIdx.x == 0) {
    mbar_init(b, 1);
    fence_barrier_init();
  }
  __syncthreads();
  if (arrive && threadIdx.x == 0) mbar_arrive(b);
  __syncthreads();
  const uint64_t t0 = global_timer_ns();
  const bool ok = mbar_wait(b, 0, limit_ns);
  const uint64_t t1 = global_timer_ns();
  const bool all_ok = __all_sync(0xffffffffu, ok);
  if (threadIdx.x == 0) {
    if (!all_ok) atomicOr(status, HPC_DEV_TIMEOUT);
    if (waited_ns) *waited_ns = t1 - t0;
  }
}
}  // namespace
}  // namespace hpc

extern "C" int hpc_wait_selftest(uint64_t limit_ns, int32_t arrive, uint32_t* status, uint64_t* waited_ns,
                                 void* stream) {
  using namespace hpc;
  if (!status) return fail(HPC_ERR_ARG, "null pointer argument");
  if (limit_ns == 0 || limit_ns > kWaitLimitNs)
    return fail(HPC_ERR_ARG, "limit_ns must be in 1 .. %llu", static_cast<unsigned long long>(kWaitLimitNs));
  wait_selftest_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(limit_ns, arrive != 0, status, waited_ns);
  return check_launch("wait_selftest_kernel");
}
