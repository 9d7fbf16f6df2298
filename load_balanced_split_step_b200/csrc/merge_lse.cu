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
