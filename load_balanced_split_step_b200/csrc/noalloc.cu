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
//  * Host code cannot use the array's name as a device address. The first call on each
//    device, with that device current, asks the runtime for the address
//    (cudaGetSymbolAddress) and caches it. Make that first call before any stream
//    capture begins.
#include <mutex>

#include "hpc_common.cuh"

namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[HPC_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
void* g_scratch_ptr[kMaxDevices] = {nullptr};

// Device address of g_noalloc_scratch on the current device (set-up on first use).
int scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return hpc::fail(HPC_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
  if (dev < 0 || dev >= kMaxDevices) return hpc::fail(HPC_ERR_ARG, "device ordinal %d out of range", dev);
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || !p)
      return hpc::fail(HPC_ERR_CUDA, "cudaGetSymbolAddress(g_noalloc_scratch): %s", cudaGetErrorString(e));
    g_scratch_ptr[dev] = p;
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
  int rc = scratch_address(&base);
  if (rc) return rc;
  char* s = static_cast<char*>(base);
  void* plan_ws = s;
  float* partial_o = reinterpret_cast<float*>(s + up256(plan_bytes));
  float* partial_ml = reinterpret_cast<float*>(s + up256(plan_bytes) + up256(po_bytes));

  hpc_plan plan;
  rc = hpc_decode_plan(seq_lens, batch, num_heads, kv_heads, tile_len, num_ctas, max_pages_per_req * page_size,
                       plan_ws, plan_bytes, &plan, status, stream);
  if (rc) return rc;
  rc = hpc_decode_attention(q, k_pages, v_pages, kv_dtype, HPC_HND, k_scale, v_scale, num_pages, page_size, num_heads,
                            kv_heads, head_dim, block_table, max_pages_per_req, seq_lens, &plan, sm_scale, partial_o,
                            partial_ml, out, out_dtype, status, stream);
  if (rc) return rc;
  return hpc_merge_states(partial_o, partial_ml, &plan, num_heads, head_dim, out, out_dtype, status, stream);
}
