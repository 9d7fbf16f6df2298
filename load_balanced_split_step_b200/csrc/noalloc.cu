// hpc_decode_step_noalloc: one decode step (plan -> attention -> merge) whose scratch
// memory is a fixed array compiled into this library, for callers that cannot allocate
// device memory.
//
// Who needs it. Some callers are not allowed to call cudaMalloc:
//  * code that runs inside a CUDA graph capture, where allocation is not captured;
//  * serving loops that reserve all device memory up front and must not stall, since
//    cudaMalloc can synchronise the device and can fail under memory pressure;
//  * plugins hosted by a framework whose allocator owns the device memory.
// The normal entry points take a plan workspace and partial-state buffers from the caller.
// This one takes them from g_noalloc_scratch instead. The caller passes only inputs and
// outputs.
//
// Rules that follow from one shared array:
//  * Its size is fixed at HPC_NOALLOC_SCRATCH_BYTES (16 MiB). Every GPU that loads the
//    library holds it until the process exits. A shape that needs more is rejected with
//    HPC_ERR_CAPACITY before anything is launched.
//  * Every call uses the same array and leaves its contents behind. Nothing in it needs
//    to start at zero: the planner rewrites every plan field on each call, and a partial
//    slot is always written before it is read. Calls that overlap on the GPU race on the
//    array. Issue them on one stream, or order them with events.
//  * Host code cannot use the array's name as a device address. The first call in each CUDA
//    context (per device, and again after that device's context was reset and recreated) asks
//    the runtime for the address (cudaGetSymbolAddress) with that device current, and caches
//    it under the context's unique id. Make that first call before any stream capture begins.
//  * Every host check (shapes, dtypes, alignment, sizes, the stream's device) runs before the
//    first of the three launches, so a non-zero return means nothing was launched.
#include <mutex>

#include "hpc_common.cuh"

namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[HPC_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
void* g_scratch_ptr[kMaxDevices] = {nullptr};
unsigned long long g_scratch_ctx[kMaxDevices] = {0};  // unique id of the context the address belongs to

// Unique id of the current CUDA context (never reused within the process), or 0 if the driver
// does not report one; then the cache is keyed on the device ordinal alone.
unsigned long long current_context_id() {
  static PFN_cuCtxGetCurrent_v4000 get_current = nullptr;
  static PFN_cuCtxGetId_v12000 get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(f);
    f = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(f);
  });
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (!get_current || !get_id || get_current(&ctx) != CUDA_SUCCESS || !ctx || get_id(ctx, &id) != CUDA_SUCCESS)
    return 0;
  return id;
}

// Device address of g_noalloc_scratch in the current context (looked up on first use there).
// The stream must belong to the current device: the address is only valid in its context.
int scratch_address(cudaStream_t stream, void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return hpc::fail(HPC_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
  if (dev < 0 || dev >= kMaxDevices) return hpc::fail(HPC_ERR_ARG, "device ordinal %d out of range", dev);
  if (stream) {
    int sdev = -1;
    e = cudaStreamGetDevice(stream, &sdev);
    if (e != cudaSuccess) return hpc::fail(HPC_ERR_CUDA, "cudaStreamGetDevice: %s", cudaGetErrorString(e));
    if (sdev != dev)
      return hpc::fail(HPC_ERR_ARG, "the stream belongs to device %d but device %d is current", sdev, dev);
  }
  // the caller's buffers live in the current context, so it exists (no cudaFree(0) here: that
  // call is not allowed while a stream is being captured)
  const unsigned long long ctx = current_context_id();
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_ptr[dev] || g_scratch_ctx[dev] != ctx) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || !p)
      return hpc::fail(HPC_ERR_CUDA, "cudaGetSymbolAddress(g_noalloc_scratch): %s", cudaGetErrorString(e));
    g_scratch_ptr[dev] = p;
    g_scratch_ctx[dev] = ctx;
  }
  *out = g_scratch_ptr[dev];
  return HPC_OK;
}

inline size_t up256(size_t x) { return (x + 255) & ~size_t(255); }

}  // namespace

extern "C" int hpc_decode_step_noalloc(const void* q, const void* k_pages, const void* v_pages, hpc_dtype kv_dtype,
                                       const float* k_scale, const float* v_scale, int32_t num_pages,
                                       int32_t page_size, int32_t num_heads, int32_t kv_heads, int32_t head_dim,
                                       const int32_t* block_table, int32_t max_pages_per_req,
                                       const int32_t* seq_lens, int32_t batch, int32_t tile_len, int32_t num_ctas,
                                       float sm_scale, void* out, hpc_dtype out_dtype, uint32_t* status,
                                       void* stream) {
  if (batch < 1 || kv_heads < 1 || num_heads < 1 || num_ctas < 1 || head_dim < 1)
    return hpc::fail(HPC_ERR_ARG, "batch, heads, head_dim and num_ctas must be >= 1");
  if (num_heads % kv_heads) return hpc::fail(HPC_ERR_SHAPE, "num_heads %% kv_heads != 0");
  if (max_pages_per_req < 1 || page_size < 1 ||
      static_cast<int64_t>(max_pages_per_req) * static_cast<int64_t>(page_size) > INT32_MAX)
    return hpc::fail(HPC_ERR_SHAPE, "max_pages_per_req * page_size must lie in 1 .. INT32_MAX");
  const size_t plan_bytes = hpc_plan_workspace_bytes(batch, kv_heads, num_ctas);
  if (plan_bytes == 0) return hpc::fail(HPC_ERR_ARG, "bad plan shape");
  const size_t max_items = static_cast<size_t>(num_ctas) + static_cast<size_t>(batch) * kv_heads;
  const size_t group = static_cast<size_t>(num_heads / kv_heads);
  const size_t po_bytes = max_items * group * head_dim * sizeof(float);
  const size_t pml_bytes = max_items * group * 2 * sizeof(float);
  const size_t need = up256(plan_bytes) + up256(po_bytes) + up256(pml_bytes);
  if (need > HPC_NOALLOC_SCRATCH_BYTES)
    return hpc::fail(HPC_ERR_CAPACITY,
                     "hpc_decode_step_noalloc needs %zu bytes of scratch, the built-in array holds %zu; "
                     "use the entry points with caller-owned buffers",
                     need, static_cast<size_t>(HPC_NOALLOC_SCRATCH_BYTES));
  void* base = nullptr;
  int rc = scratch_address(static_cast<cudaStream_t>(stream), &base);
  if (rc) return rc;
  char* s = static_cast<char*>(base);
  float* partial_o = reinterpret_cast<float*>(s + up256(plan_bytes));
  float* partial_ml = reinterpret_cast<float*>(s + up256(plan_bytes) + up256(po_bytes));
  return hpc::step_three_launch(q, k_pages, v_pages, kv_dtype, k_scale, v_scale, num_pages, page_size, num_heads,
                                kv_heads, head_dim, block_table, max_pages_per_req, seq_lens, batch, tile_len,
                                num_ctas, sm_scale, out, out_dtype, status, s, plan_bytes, partial_o, po_bytes,
                                partial_ml, pml_bytes, stream);
}
