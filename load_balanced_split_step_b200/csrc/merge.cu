// Log-sum-exp merge of split (request, kv head) pairs.
//
// The plan cuts a long request's tiles across several CTAs ("Tencent HPC llega a SGLang …",
// remio.ai, section "Por qué Tencent HPC importa para el serving de modelos en línea":
// uniform tiles spread over CTAs). Each CTA left a partial softmax state per query head,
// in natural-log units: m = max score, l = sum exp(s - m), o = sum exp(s - m) v. The exact
// result is
//     M = max_i m_i,  L = sum_i exp(m_i - M) l_i,  out = sum_i exp(m_i - M) o_i / L.
// The plan's merge_list names the (request, kv head) segments with an item count != 1:
// at most num_ctas - 1 split segments, plus the empty ones (L_r = 0), which get zeros.
// A grid-stride loop over that device-side list needs no host knowledge of its length.
//
// One CTA per segment. Every per-(item, head) weight exp(m_i - M) / L is computed once
// into shared memory. The output loop is then a weighted sum of independent loads, so its
// latency is one round of loads rather than a chain per item.
#include "hpc_common.cuh"

namespace hpc {
namespace {

constexpr int kMergeThreads = 256;
constexpr int kMergeSmemPairs = 2048;  // (item, head) weights held in shared memory per segment

__global__ void __launch_bounds__(kMergeThreads)
    merge_states_kernel(const float* __restrict__ partial_o, const float* __restrict__ partial_ml,
                        const int32_t* __restrict__ merge_list, const int32_t* __restrict__ merge_indptr,
                        const int64_t* __restrict__ counts, int32_t kv_heads, int32_t group, int32_t head_dim,
                        int32_t num_heads, void* out, int out_bf16) {
  __shared__ float s_m[kMergeSmemPairs];
  __shared__ float s_w[kMergeSmemPairs];
  __shared__ float s_M[8], s_invL[8];
  pdl_wait();  // partial states come from the attention kernel just before
  pdl_launch_dependents();
  const int64_t n_merge = counts[1];
  for (int64_t m = blockIdx.x; m < n_merge; m += gridDim.x) {
    const int32_t s = merge_list[m];
    const int32_t r = s / kv_heads, kvh = s - r * kv_heads;
    const int32_t i0 = merge_indptr[s], i1 = merge_indptr[s + 1];
    const int n = i1 - i0;
    const int64_t orow = (static_cast<int64_t>(r) * num_heads + kvh * group) * head_dim;
    const bool fast = n * group <= kMergeSmemPairs && group <= 8;
    if (fast && n > 0) {
      const float* ml = partial_ml + 2 * static_cast<int64_t>(i0) * group;
      for (int k = threadIdx.x; k < n * group; k += blockDim.x) {
        s_m[k] = ml[2 * k];
        s_w[k] = ml[2 * k + 1];  // l for now
      }
      __syncthreads();
      if (threadIdx.x < group) {
        const int h = threadIdx.x;
        float M = -INFINITY;
        for (int i = 0; i < n; ++i) M = fmaxf(M, s_m[i * group + h]);
        float L = 0.f;  // M = -inf: no part saw a live token (bad pages); the row is zero
        for (int i = 0; i < n && M != -INFINITY; ++i) L += expf(s_m[i * group + h] - M) * s_w[i * group + h];
        s_M[h] = M;
        s_invL[h] = L > 0.f ? 1.f / L : 0.f;
      }
      __syncthreads();
      for (int k = threadIdx.x; k < n * group; k += blockDim.x) {
        const int h = k % group;
        s_w[k] = s_invL[h] > 0.f ? expf(s_m[k] - s_M[h]) * s_invL[h] : 0.f;
      }
      __syncthreads();
      const float* po = partial_o + static_cast<int64_t>(i0) * group * head_dim;
      const int64_t stride = static_cast<int64_t>(group) * head_dim;
      for (int idx = threadIdx.x; idx < group * head_dim; idx += blockDim.x) {
        const int h = idx / head_dim;
        float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
        int i = 0;
        for (; i + 4 <= n; i += 4) {
          a0 += s_w[(i + 0) * group + h] * po[(i + 0) * stride + idx];
          a1 += s_w[(i + 1) * group + h] * po[(i + 1) * stride + idx];
          a2 += s_w[(i + 2) * group + h] * po[(i + 2) * stride + idx];
          a3 += s_w[(i + 3) * group + h] * po[(i + 3) * stride + idx];
        }
        for (; i < n; ++i) a0 += s_w[i * group + h] * po[i * stride + idx];
        const float val = (a0 + a1) + (a2 + a3);
        if (out_bf16) reinterpret_cast<__nv_bfloat16*>(out)[orow + idx] = __float2bfloat16_rn(val);
        else reinterpret_cast<float*>(out)[orow + idx] = val;
      }
      __syncthreads();  // shared arrays are reused by the next segment
      continue;
    }
    // no items (L_r = 0), or more (item, head) pairs than shared memory holds
    for (int idx = threadIdx.x; idx < group * head_dim; idx += blockDim.x) {
      const int h = idx / head_dim, d = idx - h * head_dim;
      float val = 0.f;
      if (n > 0) {
        float M = -INFINITY;
        for (int i = i0; i < i1; ++i) M = fmaxf(M, partial_ml[2 * (static_cast<int64_t>(i) * group + h)]);
        float L = 0.f, acc = 0.f;
        for (int i = i0; i < i1 && M != -INFINITY; ++i) {
          const int64_t pi = static_cast<int64_t>(i) * group + h;
          const float e = expf(partial_ml[2 * pi] - M);
          L += e * partial_ml[2 * pi + 1];
          acc += e * partial_o[pi * head_dim + d];
        }
        val = L > 0.f ? acc / L : 0.f;
      }
      if (out_bf16) reinterpret_cast<__nv_bfloat16*>(out)[orow + idx] = __float2bfloat16_rn(val);
      else reinterpret_cast<float*>(out)[orow + idx] = val;
    }
  }
}

}  // namespace
}  // namespace hpc

using namespace hpc;

extern "C" int hpc_merge_states(const float* partial_o, const float* partial_ml, const hpc_plan* plan,
                                int32_t num_heads, int32_t head_dim, void* out, hpc_dtype out_dtype, uint32_t* status,
                                void* stream) {
  if (!partial_o || !partial_ml || !plan || !out || !status) return fail(HPC_ERR_ARG, "null pointer argument");
  if (out_dtype != HPC_FP32 && out_dtype != HPC_BF16) return fail(HPC_ERR_DTYPE, "out_dtype must be FP32 or BF16");
  if (plan->kv_heads < 1 || num_heads % plan->kv_heads) return fail(HPC_ERR_SHAPE, "num_heads %% kv_heads != 0");
  if (head_dim < 1) return fail(HPC_ERR_ARG, "head_dim must be >= 1");
  const int group = num_heads / plan->kv_heads;
  int sms = device_sm_count();
  if (sms < 1) sms = 148;
  int grid = plan->is_static ? plan->merge_capacity : plan->num_ctas;
  if (grid > 2 * sms) grid = 2 * sms;
  if (grid < 1) grid = 1;
  const cudaError_t e =
      launch_pdl(merge_states_kernel, dim3(grid), dim3(kMergeThreads), 0, static_cast<cudaStream_t>(stream), partial_o,
                 partial_ml, plan->merge_list, plan->merge_indptr, plan->counts, plan->kv_heads, group, head_dim,
                 num_heads, out, static_cast<int>(out_dtype == HPC_BF16));
  if (e != cudaSuccess) return fail(HPC_ERR_CUDA, "merge_states_kernel: %s", cudaGetErrorString(e));
  return check_launch("merge_states_kernel");
}
