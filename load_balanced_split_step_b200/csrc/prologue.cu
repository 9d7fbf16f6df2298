// Fused decode prologue: QK-RMSNorm + RoPE on the new token, and its K/V page write.
//
// "vLLM × HPC-Ops: High-Performance Attention and MoE Backends from Tencent Hunyuan" (8sync
// News summary) names a fused RoPE + QK-Norm + KV-write prologue in front of the attention
// backend. One CTA handles one request; the cache may be HND or NHD. The NeoX rotation angles pos * theta^(-2i/D) are
// evaluated once per request in fp64, because pos reaches 1e5 and an fp32 angle would lose
// ~1e-3 rad. They are shared through shared memory. Each warp takes one head at a time:
// q and k heads are RMS-normalised and rotated, v heads copied. q goes out as bf16; k and
// v go into page block_table[r][pos / P], slot pos % P, as bf16 or as E4M3 codes of
// x / scale (round to nearest even, saturating).
#include "hpc_common.cuh"

namespace hpc {
namespace {

constexpr int kProWarps = 8;

template <int D>
__global__ void __launch_bounds__(kProWarps * 32)
    prologue_kernel(const __nv_bfloat16* __restrict__ qkv, const float* __restrict__ q_norm_w,
                    const float* __restrict__ k_norm_w, float eps, double theta, __nv_bfloat16* __restrict__ q_out,
                    void* __restrict__ k_pages, void* __restrict__ v_pages, int fp8, const float* __restrict__ k_scale,
                    const float* __restrict__ v_scale, int32_t num_pages, int32_t P, const int32_t* __restrict__ block_table,
                    int64_t max_pages, const int32_t* __restrict__ seq_lens, int32_t Hq, int32_t Hkv, int nhd,
                    uint32_t* status) {
  constexpr int PER = D / 32;  // elements per lane: d = lane + 32 k
  constexpr int HALF = PER / 2;
  __shared__ float s_cos[D / 2], s_sin[D / 2];
  const int r = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  pdl_wait();
  pdl_launch_dependents();
  const int32_t L = seq_lens[r];
  const bool len_ok = L >= 1 && static_cast<int64_t>(L) <= max_pages * P;
  const int64_t pos = len_ok ? L - 1 : 0;
  int32_t page = -1;
  if (len_ok) page = block_table[r * max_pages + pos / P];
  const bool page_ok = len_ok && page >= 0 && page < num_pages;
  if (threadIdx.x == 0) {
    if (!len_ok) atomicOr(status, HPC_DEV_BAD_SEQLEN);
    else if (!page_ok) atomicOr(status, HPC_DEV_BAD_PAGE);
  }
  for (int i = threadIdx.x; i < D / 2; i += blockDim.x) {
    const double ang = static_cast<double>(pos) * pow(theta, -2.0 * i / D);
    double sn, cs;
    sincos(ang, &sn, &cs);
    s_cos[i] = static_cast<float>(cs);
    s_sin[i] = static_cast<float>(sn);
  }
  __syncthreads();
  const int slot = static_cast<int>(pos % P);
  const int heads = Hq + 2 * Hkv;
  for (int h = warp; h < heads; h += kProWarps) {
    const __nv_bfloat16* src = qkv + (static_cast<int64_t>(r) * heads + h) * D;
    float x[PER];
#pragma unroll
    for (int k = 0; k < PER; ++k) x[k] = __bfloat162float(src[lane + 32 * k]);
    if (h < Hq + Hkv) {
      const float* w = h < Hq ? q_norm_w : k_norm_w;
      float ss = 0.f;
#pragma unroll
      for (int k = 0; k < PER; ++k) ss += x[k] * x[k];
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
      const float inv = 1.f / sqrtf(ss / D + eps);
#pragma unroll
      for (int k = 0; k < PER; ++k) x[k] = x[k] * inv * w[lane + 32 * k];
#pragma unroll
      for (int k = 0; k < HALF; ++k) {  // pair (i, i + D/2), i = lane + 32 k
        const float cs = s_cos[lane + 32 * k], sn = s_sin[lane + 32 * k];
        const float x1 = x[k], x2 = x[k + HALF];
        x[k] = x1 * cs - x2 * sn;
        x[k + HALF] = x2 * cs + x1 * sn;
      }
    }
    if (h < Hq) {
      __nv_bfloat16* dst = q_out + (static_cast<int64_t>(r) * Hq + h) * D;
#pragma unroll
      for (int k = 0; k < PER; ++k) dst[lane + 32 * k] = len_ok ? __float2bfloat16_rn(x[k]) : __float2bfloat16_rn(0.f);
      continue;
    }
    if (!page_ok) continue;
    const bool is_k = h < Hq + Hkv;
    const int g = is_k ? h - Hq : h - Hq - Hkv;
    const int64_t base = nhd ? ((static_cast<int64_t>(page) * P + slot) * Hkv + g) * D
                             : ((static_cast<int64_t>(page) * Hkv + g) * P + slot) * D;
    if (fp8) {
      const float sc = is_k ? k_scale[g] : v_scale[g];
      uint8_t* dst = static_cast<uint8_t*>(is_k ? k_pages : v_pages) + base;
#pragma unroll
      for (int k = 0; k < PER; ++k) dst[lane + 32 * k] = f32_to_e4m3(x[k] / sc);
    } else {
      __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(is_k ? k_pages : v_pages) + base;
#pragma unroll
      for (int k = 0; k < PER; ++k) dst[lane + 32 * k] = __float2bfloat16_rn(x[k]);
    }
  }
}

}  // namespace
}  // namespace hpc

using namespace hpc;

extern "C" int hpc_decode_prologue(const void* qkv, const float* q_norm_w, const float* k_norm_w, float eps,
                                   float rope_theta, void* q_out, void* k_pages, void* v_pages, hpc_dtype kv_dtype,
                                   hpc_kv_layout kv_layout, const float* k_scale, const float* v_scale, int32_t num_pages, int32_t page_size,
                                   const int32_t* block_table, int32_t max_pages_per_req, const int32_t* seq_lens,
                                   int32_t batch, int32_t num_heads, int32_t kv_heads, int32_t head_dim,
                                   uint32_t* status, void* stream) {
  if (!qkv || !q_norm_w || !k_norm_w || !q_out || !k_pages || !v_pages || !block_table || !seq_lens || !status)
    return fail(HPC_ERR_ARG, "null pointer argument");
  if (kv_dtype != HPC_BF16 && kv_dtype != HPC_E4M3) return fail(HPC_ERR_DTYPE, "kv_dtype must be BF16 or E4M3");
  if (kv_layout != HPC_HND && kv_layout != HPC_NHD) return fail(HPC_ERR_ARG, "kv_layout must be HND or NHD");
  const bool fp8 = kv_dtype == HPC_E4M3;
  if (fp8 && (!k_scale || !v_scale)) return fail(HPC_ERR_ARG, "E4M3 cache needs k_scale and v_scale");
  if (batch < 1 || num_heads < 1 || kv_heads < 1 || num_pages < 1 || page_size < 1 || max_pages_per_req < 1)
    return fail(HPC_ERR_ARG, "sizes must be >= 1");
  if (num_heads % kv_heads) return fail(HPC_ERR_SHAPE, "num_heads %% kv_heads != 0");
  if (head_dim != 64 && head_dim != 128) return fail(HPC_ERR_SHAPE, "head_dim must be 64 or 128");
  if (!(rope_theta > 0.f) || !(eps >= 0.f)) return fail(HPC_ERR_ARG, "rope_theta must be > 0 and eps >= 0");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const auto* x = static_cast<const __nv_bfloat16*>(qkv);
  auto* qo = static_cast<__nv_bfloat16*>(q_out);
  auto kern = head_dim == 128 ? prologue_kernel<128> : prologue_kernel<64>;
  const cudaError_t e = launch_pdl(kern, dim3(batch), dim3(kProWarps * 32), 0, st, x, q_norm_w, k_norm_w, eps,
                                   static_cast<double>(rope_theta), qo, k_pages, v_pages, static_cast<int>(fp8),
                                   k_scale, v_scale, num_pages, page_size, block_table,
                                   static_cast<int64_t>(max_pages_per_req), seq_lens, num_heads, kv_heads,
                                   static_cast<int>(kv_layout == HPC_NHD), status);
  if (e != cudaSuccess) return fail(HPC_ERR_CUDA, "prologue_kernel: %s", cudaGetErrorString(e));
  return check_launch("prologue_kernel");
}
