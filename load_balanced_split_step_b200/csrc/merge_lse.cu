// Log-sum-exp merge of attention outputs over disjoint parts of the same keys.
//
// When one request's KV is split across GPUs (request-sharded placement of a decode batch,
// with a request longer than one GPU's share cut into token ranges), each part yields a
// normalised output o_i and its log-sum-exp lse_i = log sum_j exp(s_j) over the part's keys.
// The whole is
//     LSE = log sum_i exp(lse_i),   out = sum_i exp(lse_i - LSE) o_i,
// the same log-sum-exp combine that merges a request split across CTAs inside one GPU. The
// pages describe the split of a request's tiles across processing units ("腾讯混元三算子杀入
// SGLang" (AREX), Dynamic Attention paragraph) but no merge step and no multi-GPU placement;
// this entry point extends the in-GPU merge to parts computed on different GPUs. One warp per
// output row; lanes split head_dim.
#include "hpc_common.cuh"

namespace hpc {
namespace {

constexpr int kMergeLseThreads = 256;

__global__ void __launch_bounds__(kMergeLseThreads)
    merge_lse_kernel(const float* __restrict__ outs, const float* __restrict__ lses, int32_t parts, int64_t rows,
                     int32_t head_dim, float* __restrict__ out, float* __restrict__ lse_out) {
  pdl_wait();
  pdl_launch_dependents();
  const int lane = threadIdx.x & 31;
  const int64_t warps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  for (int64_t r = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5); r < rows; r += warps) {
    float M = -INFINITY;
    for (int i = 0; i < parts; ++i) M = fmaxf(M, lses[static_cast<int64_t>(i) * rows + r]);
    float S = 0.f;
    if (M != -INFINITY)
      for (int i = 0; i < parts; ++i) S += expf(lses[static_cast<int64_t>(i) * rows + r] - M);
    const float inv = S > 0.f ? 1.f / S : 0.f;
    for (int d = lane; d < head_dim; d += 32) {
      float acc = 0.f;
      if (M != -INFINITY)
        for (int i = 0; i < parts; ++i) {
          const int64_t k = static_cast<int64_t>(i) * rows + r;
          acc += expf(lses[k] - M) * outs[k * head_dim + d];
        }
      out[r * head_dim + d] = acc * inv;
    }
    if (lse_out && lane == 0) lse_out[r] = S > 0.f ? M + logf(S) : -INFINITY;
  }
}

// The same merge, with each output row's parts found through an index: row (r, h) combines
// rows part_index[r][k] (k < max_parts, index >= 0) of outs / lses at head h. One part is copied
// exactly (its weight is exp(0) = 1 and the sum is 1); no part gives zeros and -inf. An index
// at or past part_rows is skipped and sets HPC_DEV_BAD_INDEX.
__global__ void __launch_bounds__(kMergeLseThreads)
    merge_lse_gather_kernel(const float* __restrict__ outs, const float* __restrict__ lses,
                            const int32_t* __restrict__ part_index, int32_t max_parts, int64_t part_rows,
                            int32_t batch, int32_t num_heads, int32_t head_dim, float* __restrict__ out,
                            float* __restrict__ lse_out, uint32_t* __restrict__ status) {
  pdl_wait();
  pdl_launch_dependents();
  const int lane = threadIdx.x & 31;
  const int64_t rows = static_cast<int64_t>(batch) * num_heads;
  const int64_t warps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  for (int64_t row = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5); row < rows;
       row += warps) {
    const int64_t r = row / num_heads;
    const int h = static_cast<int>(row - r * num_heads);
    const int32_t* idx = part_index + r * max_parts;
    float M = -INFINITY;
    bool bad = false;
    for (int k = 0; k < max_parts; ++k) {
      const int32_t i = idx[k];
      if (i < 0) continue;
      if (i >= part_rows) {
        bad = true;
        continue;
      }
      M = fmaxf(M, lses[static_cast<int64_t>(i) * num_heads + h]);
    }
    float S = 0.f;
    if (M != -INFINITY)
      for (int k = 0; k < max_parts; ++k) {
        const int32_t i = idx[k];
        if (i >= 0 && i < part_rows) S += expf(lses[static_cast<int64_t>(i) * num_heads + h] - M);
      }
    const float inv = S > 0.f ? 1.f / S : 0.f;
    for (int d = lane; d < head_dim; d += 32) {
      float acc = 0.f;
      if (M != -INFINITY)
        for (int k = 0; k < max_parts; ++k) {
          const int32_t i = idx[k];
          if (i < 0 || i >= part_rows) continue;
          const int64_t pr = static_cast<int64_t>(i) * num_heads + h;
          acc += expf(lses[pr] - M) * outs[pr * head_dim + d];
        }
      out[row * head_dim + d] = acc * inv;
    }
    if (lane == 0) {
      if (lse_out) lse_out[row] = S > 0.f ? M + logf(S) : -INFINITY;
      if (bad && status) atomicOr(status, HPC_DEV_BAD_INDEX);
    }
  }
}

// dst row j = src row index[j], rows of row_bytes (a multiple of 16) bytes. An index outside
// [0, src_rows) gives a zero row and sets HPC_DEV_BAD_INDEX.
__global__ void __launch_bounds__(kMergeLseThreads)
    gather_rows_kernel(const uint4* __restrict__ src, int64_t src_rows, const int32_t* __restrict__ index,
                       int64_t n, int64_t row_vecs, uint4* __restrict__ dst, uint32_t* __restrict__ status) {
  pdl_wait();
  pdl_launch_dependents();
  const int64_t total = n * row_vecs;
  for (int64_t t = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; t < total;
       t += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t j = t / row_vecs, v = t - j * row_vecs;
    const int32_t i = index[j];
    if (i < 0 || i >= src_rows) {
      dst[t] = make_uint4(0u, 0u, 0u, 0u);
      if (v == 0 && status) atomicOr(status, HPC_DEV_BAD_INDEX);
      continue;
    }
    dst[t] = src[static_cast<int64_t>(i) * row_vecs + v];
  }
}

// Block-table view of the parts a request-sharded rank runs: row i holds the pages of request
// req[i] from column col0[i] on, -1 past the table. One thread per entry.
__global__ void __launch_bounds__(kMergeLseThreads)
    gather_pages_kernel(const int32_t* __restrict__ src, int32_t src_rows, int32_t src_cols,
                        const int32_t* __restrict__ req, const int32_t* __restrict__ col0, int32_t n, int32_t width,
                        int32_t* __restrict__ dst, uint32_t* __restrict__ status) {
  pdl_wait();
  pdl_launch_dependents();
  const int64_t total = static_cast<int64_t>(n) * width;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  bool bad = false;
  for (int64_t k = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; k < total; k += stride) {
    const int64_t i = k / width, j = k - i * width;
    const int32_t r = req[i], c0 = col0[i];
    int32_t v = -1;
    if (r < 0 || r >= src_rows || c0 < 0) {
      bad = true;
    } else if (c0 + j < src_cols) {
      v = src[static_cast<int64_t>(r) * src_cols + c0 + j];
    }
    dst[k] = v;
  }
  if (bad && status) atomicOr(status, HPC_DEV_BAD_INDEX);
}

}  // namespace
}  // namespace hpc

using namespace hpc;

extern "C" int hpc_merge_lse(const float* outs, const float* lses, int32_t parts, int64_t rows, int32_t head_dim,
                             float* out, float* lse_out, void* stream) {
  if (!outs || !lses || !out) return fail(HPC_ERR_ARG, "null pointer argument");
  if (parts < 1 || rows < 0 || head_dim < 1) return fail(HPC_ERR_ARG, "parts, rows and head_dim must be positive");
  if (rows == 0) return HPC_OK;
  const int64_t per_block = kMergeLseThreads / 32;
  int64_t blocks = (rows + per_block - 1) / per_block;
  const int sms = device_sm_count();
  const int64_t cap = sms > 0 ? static_cast<int64_t>(sms) * 8 : 1024;
  if (blocks > cap) blocks = cap;
  const cudaError_t e = launch_pdl(merge_lse_kernel, dim3(static_cast<unsigned>(blocks)), dim3(kMergeLseThreads), 0,
                                   static_cast<cudaStream_t>(stream), outs, lses, parts, rows, head_dim, out, lse_out);
  if (e != cudaSuccess) return fail(HPC_ERR_CUDA, "merge_lse_kernel: %s", cudaGetErrorString(e));
  return check_launch("merge_lse_kernel");
}

extern "C" int hpc_merge_lse_gather(const float* outs, const float* lses, int64_t part_rows, const int32_t* part_index,
                                    int32_t max_parts, int32_t batch, int32_t num_heads, int32_t head_dim, float* out,
                                    float* lse_out, uint32_t* status, void* stream) {
  if (!outs || !lses || !part_index || !out) return fail(HPC_ERR_ARG, "null pointer argument");
  if (part_rows < 0 || max_parts < 1 || batch < 0 || num_heads < 1 || head_dim < 1)
    return fail(HPC_ERR_ARG, "part_rows, max_parts, batch, num_heads and head_dim must be in range");
  if (batch == 0) return HPC_OK;
  const int64_t rows = static_cast<int64_t>(batch) * num_heads;
  const int64_t per_block = kMergeLseThreads / 32;
  int64_t blocks = (rows + per_block - 1) / per_block;
  const int sms = device_sm_count();
  const int64_t cap = sms > 0 ? static_cast<int64_t>(sms) * 8 : 1024;
  if (blocks > cap) blocks = cap;
  const cudaError_t e =
      launch_pdl(merge_lse_gather_kernel, dim3(static_cast<unsigned>(blocks)), dim3(kMergeLseThreads), 0,
                 static_cast<cudaStream_t>(stream), outs, lses, part_index, max_parts, part_rows, batch, num_heads,
                 head_dim, out, lse_out, status);
  if (e != cudaSuccess) return fail(HPC_ERR_CUDA, "merge_lse_gather_kernel: %s", cudaGetErrorString(e));
  return check_launch("merge_lse_gather_kernel");
}

extern "C" int hpc_gather_rows(const void* src, int64_t src_rows, int64_t row_bytes, const int32_t* index, int64_t n,
                               void* dst, uint32_t* status, void* stream) {
  if (!src || !index || !dst) return fail(HPC_ERR_ARG, "null pointer argument");
  if (src_rows < 0 || n < 0 || row_bytes <= 0) return fail(HPC_ERR_ARG, "src_rows, n and row_bytes must be in range");
  if (row_bytes % 16) return fail(HPC_ERR_SHAPE, "row_bytes must be a multiple of 16");
  if ((reinterpret_cast<uintptr_t>(src) | reinterpret_cast<uintptr_t>(dst)) & 15)
    return fail(HPC_ERR_ALIGN, "src and dst must be 16-byte aligned");
  if (n == 0) return HPC_OK;
  const int64_t row_vecs = row_bytes / 16, total = n * row_vecs;
  int64_t blocks = (total + kMergeLseThreads - 1) / kMergeLseThreads;
  const int sms = device_sm_count();
  const int64_t cap = sms > 0 ? static_cast<int64_t>(sms) * 8 : 1024;
  if (blocks > cap) blocks = cap;
  const cudaError_t e =
      launch_pdl(gather_rows_kernel, dim3(static_cast<unsigned>(blocks)), dim3(kMergeLseThreads), 0,
                 static_cast<cudaStream_t>(stream), static_cast<const uint4*>(src), src_rows, index, n, row_vecs,
                 static_cast<uint4*>(dst), status);
  if (e != cudaSuccess) return fail(HPC_ERR_CUDA, "gather_rows_kernel: %s", cudaGetErrorString(e));
  return check_launch("gather_rows_kernel");
}

extern "C" int hpc_gather_pages(const int32_t* src, int32_t src_rows, int32_t src_cols, const int32_t* req,
                                const int32_t* col0, int32_t n, int32_t width, int32_t* dst, uint32_t* status,
                                void* stream) {
  if (!src || !req || !col0 || !dst) return fail(HPC_ERR_ARG, "null pointer argument");
  if (src_rows < 0 || src_cols < 1 || n < 0 || width < 1) return fail(HPC_ERR_ARG, "sizes out of range");
  if (n == 0) return HPC_OK;
  const int64_t total = static_cast<int64_t>(n) * width;
  int64_t blocks = (total + kMergeLseThreads - 1) / kMergeLseThreads;
  const int sms = device_sm_count();
  const int64_t cap = sms > 0 ? static_cast<int64_t>(sms) * 8 : 1024;
  if (blocks > cap) blocks = cap;
  const cudaError_t e = launch_pdl(gather_pages_kernel, dim3(static_cast<unsigned>(blocks)), dim3(kMergeLseThreads), 0,
                                   static_cast<cudaStream_t>(stream), src, src_rows, src_cols, req, col0, n, width,
                                   dst, status);
  if (e != cudaSuccess) return fail(HPC_ERR_CUDA, "gather_pages_kernel: %s", cudaGetErrorString(e));
  return check_launch("gather_pages_kernel");
}
