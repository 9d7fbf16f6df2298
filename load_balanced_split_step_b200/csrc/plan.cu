// Per-step tile planner: the load-balanced ("dynamic") plan and the static split-k plan.
//
// "Tencent HPC llega a SGLang …" (remio.ai), section "Por qué Tencent HPC importa para el
// serving de modelos en línea": KV work is cut into uniform tiles and spread over CTAs by
// current load, and the mapping is rebuilt as request lengths change. "腾讯混元三算子杀入
// SGLang" (AREX), Dynamic Attention paragraph: tiles are assigned every decode step by the
// actual KV length. This file builds that mapping on the device from seq_lens, so a
// step needs no host round trip.
//
// Dynamic plan. nt_r = ceil(L_r / tile_len). Segment s = r*Hkv + kvh holds units
// [U_s, U_s + nt_r), where U_s = Hkv * sum_{r' < r} nt_r' + kvh * nt_r. With chunk =
// ceil(T / G), the CTA boundaries are the multiples of chunk. Segment s is cut into
//     pieces_s = nt_r == 0 ? 0 : floor((U_s + nt_r - 1) / chunk) - floor(U_s / chunk) + 1
// items. Piece j starts at U_s (j = 0) or at (floor(U_s/chunk) + j) * chunk, and ends at the
// next boundary or at U_s + nt_r. Item offsets are a prefix sum of pieces_s over segments,
// in request order. The piece that starts on a multiple g*chunk is the first item of CTA g.
// The closed form is evaluated independently per segment, so the kernel is one CTA of
// scans, with no serial walk over units. Its output is byte-identical to the host twin
// hpc_plan_cpu below.
#include <stdarg.h>
#include <stdio.h>
#include <string.h>

#include <algorithm>
#include <vector>

#include "hpc_common.cuh"

namespace hpc {

namespace {

constexpr int kPlanThreads = 1024;

__host__ __device__ inline int64_t ceil_div64(int64_t a, int64_t b) { return (a + b - 1) / b; }

__host__ __device__ inline int32_t tiles_of(int32_t L, int32_t tl) {
  return L > 0 ? static_cast<int32_t>(static_cast<uint32_t>(L - 1) / static_cast<uint32_t>(tl) + 1) : 0;
}

__host__ __device__ inline bool len_ok(int32_t L, int32_t max_seq_len) {
  return L >= 0 && (max_seq_len <= 0 || L <= max_seq_len);
}

// number of items (r, kvh) is cut into
__host__ __device__ inline int32_t pieces_of(int64_t U, int32_t nt, int64_t chunk) {
  if (nt == 0) return 0;
  return static_cast<int32_t>((U + nt - 1) / chunk - U / chunk + 1);
}

// a / b for non-negative operands; 32-bit hardware path when the whole plan fits in 31 bits
// (the flag is uniform across the block).
__device__ __forceinline__ int64_t udiv(int64_t a, int64_t b, bool small) {
  return small ? static_cast<int64_t>(static_cast<uint32_t>(a) / static_cast<uint32_t>(b)) : a / b;
}

// Block-wide exclusive scan of one int64 per thread (kPlanThreads threads).
__device__ int64_t block_exclusive_scan(int64_t v, int64_t* total, int64_t* warp_sums) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int64_t x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int64_t y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) warp_sums[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int64_t w = (lane < kPlanThreads / 32) ? warp_sums[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int64_t y = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += y;
    }
    warp_sums[lane] = w;  // inclusive prefix over warps
  }
  __syncthreads();
  const int64_t warp_prefix = warp > 0 ? warp_sums[warp - 1] : 0;
  *total = warp_sums[kPlanThreads / 32 - 1];
  __syncthreads();  // warp_sums is reused by the next scan
  return warp_prefix + x - v;
}

struct PlanPtrs {
  int64_t* counts;
  hpc_work_item* items;
  int32_t* cta_indptr;
  int32_t* merge_indptr;
  int32_t* merge_list;
};

__global__ void __launch_bounds__(kPlanThreads, 1)
    dynamic_plan_kernel(const int32_t* __restrict__ seq_lens, int32_t B, int32_t Hkv, int32_t tl, int32_t G,
                        int32_t max_seq_len, int32_t max_items, PlanPtrs out, uint32_t* status) {
  __shared__ int64_t warp_sums[32];
  __shared__ int64_t s_total;
  const int tid = threadIdx.x;
  pdl_wait();  // seq_lens may come from the previous kernel; the plan buffers may still be read by it
  pdl_launch_dependents();

  // pass 1: total units
  int64_t local = 0;
  uint32_t bad = 0;
  for (int r = tid; r < B; r += kPlanThreads) {
    int32_t L = seq_lens[r];
    if (!len_ok(L, max_seq_len)) {
      bad |= HPC_DEV_BAD_SEQLEN;
      L = 0;
    }
    local += tiles_of(L, tl);
  }
  if (bad) atomicOr(status, bad);
  for (int o = 16; o > 0; o >>= 1) local += __shfl_xor_sync(0xffffffffu, local, o);
  if ((tid & 31) == 0) warp_sums[tid >> 5] = local;
  __syncthreads();
  if (tid == 0) {
    int64_t t = 0;
    for (int w = 0; w < kPlanThreads / 32; ++w) t += warp_sums[w];
    s_total = t;
  }
  __syncthreads();
  const int64_t T = s_total * Hkv;
  const int64_t chunk = T > 0 ? ceil_div64(T, G) : 0;
  const bool small = T < (int64_t(1) << 31);

  // pass 2: items, in blocks of kPlanThreads requests with running carries
  int64_t carry_nt = 0, carry_items = 0, carry_merge = 0;
  bool overflow = false;
  for (int base = 0; base < B; base += kPlanThreads) {
    const int r = base + tid;
    int32_t nt = 0;
    if (r < B) {
      int32_t L = seq_lens[r];
      nt = len_ok(L, max_seq_len) ? tiles_of(L, tl) : 0;
    }
    int64_t tot_nt, tot_items, tot_merge;
    const int64_t nt_before = carry_nt + block_exclusive_scan(nt, &tot_nt, warp_sums);
    const int64_t U_r = nt_before * Hkv;
    int64_t n_pieces = 0, n_merge = 0;
    if (r < B && nt > 0) {
      for (int kvh = 0; kvh < Hkv; ++kvh) {
        const int64_t U = U_r + static_cast<int64_t>(kvh) * nt;
        const int64_t pc = udiv(U + nt - 1, chunk, small) - udiv(U, chunk, small) + 1;
        n_pieces += pc;
        n_merge += (pc != 1);
      }
    } else if (r < B) {
      n_merge = Hkv;  // an empty request: every kv head is zero-filled by the merge step
    }
    int64_t idx = carry_items + block_exclusive_scan(n_pieces, &tot_items, warp_sums);
    int64_t midx = carry_merge + block_exclusive_scan(n_merge, &tot_merge, warp_sums);
    if (r < B) {
      for (int kvh = 0; kvh < Hkv; ++kvh) {
        const int64_t s = static_cast<int64_t>(r) * Hkv + kvh;
        out.merge_indptr[s] = static_cast<int32_t>(idx);
        if (nt == 0) {
          out.merge_list[midx++] = static_cast<int32_t>(s);
          continue;
        }
        const int64_t U = U_r + static_cast<int64_t>(kvh) * nt;
        const int64_t q0 = udiv(U, chunk, small);
        const int64_t pc = udiv(U + nt - 1, chunk, small) - q0 + 1;
        if (pc != 1) out.merge_list[midx++] = static_cast<int32_t>(s);
        // piece j starts at U (j = 0) or at the CTA boundary (q0 + j) * chunk, and ends at the
        // next boundary or at the end of the segment; piece j belongs to CTA q0 + j
        for (int64_t j = 0; j < pc; ++j, ++idx) {
          const int64_t start = j == 0 ? U : (q0 + j) * chunk;
          const int64_t end = min((q0 + j + 1) * chunk, U + nt);
          if (idx >= max_items) {
            overflow = true;
            continue;
          }
          hpc_work_item w;
          w.req = r;
          w.kv_head = static_cast<int16_t>(kvh);
          w.flags = pc == 1 ? HPC_ITEM_DIRECT : 0;
          w.tile_begin = static_cast<int32_t>(start - U);
          w.tile_end = static_cast<int32_t>(end - U);
          out.items[idx] = w;
          if (j > 0 || start == q0 * chunk) out.cta_indptr[q0 + j] = static_cast<int32_t>(idx);
        }
      }
    }
    carry_nt += tot_nt;
    carry_items += tot_items;
    carry_merge += tot_merge;
  }
  if (overflow) atomicOr(status, HPC_DEV_CAPACITY);
  const int64_t n_items = min(carry_items, static_cast<int64_t>(max_items));
  const int64_t n_active = chunk > 0 ? ceil_div64(T, chunk) : 0;
  for (int64_t g = n_active + tid; g <= G; g += kPlanThreads) out.cta_indptr[g] = static_cast<int32_t>(n_items);
  if (tid == 0) {
    out.merge_indptr[static_cast<int64_t>(B) * Hkv] = static_cast<int32_t>(n_items);
    out.counts[0] = n_items;
    out.counts[1] = carry_merge;
    out.counts[2] = T;
    out.counts[3] = chunk;
  }
}

__global__ void __launch_bounds__(kPlanThreads, 1)
    static_plan_kernel(const int32_t* __restrict__ seq_lens, int32_t B, int32_t Hkv, int32_t tl, int32_t S,
                       int32_t max_seq_len, PlanPtrs out, uint32_t* status) {
  __shared__ int64_t warp_sums[32];
  const int tid = threadIdx.x;
  pdl_wait();
  pdl_launch_dependents();
  int64_t carry_items = 0, carry_merge = 0, carry_nt = 0;
  uint32_t bad = 0;
  for (int base = 0; base < B; base += kPlanThreads) {
    const int r = base + tid;
    int32_t nt = 0;
    if (r < B) {
      const int32_t L = seq_lens[r];
      if (len_ok(L, max_seq_len)) nt = tiles_of(L, tl);
      else bad |= HPC_DEV_BAD_SEQLEN;
    }
    const int32_t per = nt > 0 ? static_cast<int32_t>(ceil_div64(nt, S)) : 0;
    const int32_t pc = nt > 0 ? static_cast<int32_t>(ceil_div64(nt, per)) : 0;  // non-empty splits
    int64_t tot_items, tot_merge, tot_nt;
    block_exclusive_scan(nt, &tot_nt, warp_sums);
    int64_t idx = carry_items + block_exclusive_scan(r < B ? static_cast<int64_t>(pc) * Hkv : 0, &tot_items, warp_sums);
    int64_t midx = carry_merge + block_exclusive_scan(r < B && pc != 1 ? Hkv : 0, &tot_merge, warp_sums);
    if (r < B) {
      for (int kvh = 0; kvh < Hkv; ++kvh) {
        const int64_t s = static_cast<int64_t>(r) * Hkv + kvh;
        out.merge_indptr[s] = static_cast<int32_t>(idx);
        if (pc != 1) out.merge_list[midx++] = static_cast<int32_t>(s);
        for (int32_t j = 0; j < S; ++j) {
          out.cta_indptr[s * S + j] = static_cast<int32_t>(idx + std::min(j, pc));
        }
        for (int32_t j = 0; j < pc; ++j) {
          hpc_work_item w;
          w.req = r;
          w.kv_head = static_cast<int16_t>(kvh);
          w.flags = pc == 1 ? HPC_ITEM_DIRECT : 0;
          w.tile_begin = j * per;
          w.tile_end = std::min((j + 1) * per, nt);
          out.items[idx + j] = w;
        }
        idx += pc;
      }
    }
    carry_items += tot_items;
    carry_merge += tot_merge;
    carry_nt += tot_nt;
  }
  if (bad) atomicOr(status, bad);
  if (tid == 0) {
    const int64_t G = static_cast<int64_t>(B) * Hkv * S;
    out.cta_indptr[G] = static_cast<int32_t>(carry_items);
    out.merge_indptr[static_cast<int64_t>(B) * Hkv] = static_cast<int32_t>(carry_items);
    out.counts[0] = carry_items;
    out.counts[1] = carry_merge;
    out.counts[2] = carry_nt * Hkv;
    out.counts[3] = 0;
  }
}

inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

}  // namespace

int check_plan_args(const void* seq_lens, int32_t batch, int32_t num_heads, int32_t kv_heads, int32_t tile_len,
                    int32_t ctas, const void* workspace, const void* plan, const void* status) {
  if (!seq_lens || !workspace || !plan || !status) return fail(HPC_ERR_ARG, "null pointer argument");
  if (batch < 1 || kv_heads < 1 || num_heads < 1 || ctas < 1)
    return fail(HPC_ERR_ARG, "batch, heads and CTA count must be >= 1");
  if (num_heads % kv_heads != 0) return fail(HPC_ERR_SHAPE, "num_heads %% kv_heads != 0");
  if (kv_heads > 32767) return fail(HPC_ERR_SHAPE, "kv_heads must fit int16");
  if (tile_len < 16 || tile_len % 16 != 0) return fail(HPC_ERR_SHAPE, "tile_len must be a positive multiple of 16");
  if (static_cast<int64_t>(batch) * kv_heads > (1ll << 30) || ctas > (1 << 28))
    return fail(HPC_ERR_SHAPE, "plan too large");
  if ((reinterpret_cast<uintptr_t>(workspace) & 255) != 0) return fail(HPC_ERR_ALIGN, "workspace must be 256-byte aligned");
  return HPC_OK;
}

namespace {

void bind_plan(void* ws, const PlanLayout& L, int32_t batch, int32_t kv_heads, int32_t tile_len, int32_t ctas,
               int32_t max_items, int32_t is_static, hpc_plan* plan) {
  char* base = static_cast<char*>(ws);
  plan->batch = batch;
  plan->kv_heads = kv_heads;
  plan->tile_len = tile_len;
  plan->num_ctas = ctas;
  plan->max_items = max_items;
  plan->merge_capacity = batch * kv_heads;
  plan->is_static = is_static;
  plan->reserved = 0;
  plan->counts = reinterpret_cast<int64_t*>(base + L.counts);
  plan->items = reinterpret_cast<hpc_work_item*>(base + L.items);
  plan->cta_indptr = reinterpret_cast<int32_t*>(base + L.cta_indptr);
  plan->merge_indptr = reinterpret_cast<int32_t*>(base + L.merge_indptr);
  plan->merge_list = reinterpret_cast<int32_t*>(base + L.merge_list);
}

PlanPtrs ptrs_of(const hpc_plan* p) {
  return PlanPtrs{p->counts, p->items, p->cta_indptr, p->merge_indptr, p->merge_list};
}

}  // namespace

PlanLayout plan_layout(int32_t batch, int32_t kv_heads, int32_t num_ctas, int32_t max_items) {
  PlanLayout L;
  const size_t segs = static_cast<size_t>(batch) * kv_heads;
  size_t o = 0;
  L.counts = o;
  o = align256(o + 4 * sizeof(int64_t));
  L.items = o;
  o = align256(o + static_cast<size_t>(max_items) * sizeof(hpc_work_item));
  L.cta_indptr = o;
  o = align256(o + (static_cast<size_t>(num_ctas) + 1) * sizeof(int32_t));
  L.merge_indptr = o;
  o = align256(o + (segs + 1) * sizeof(int32_t));
  L.merge_list = o;
  o = align256(o + segs * sizeof(int32_t));
  L.total = o;
  return L;
}

}  // namespace hpc

using namespace hpc;

extern "C" size_t hpc_plan_workspace_bytes(int32_t batch, int32_t kv_heads, int32_t num_ctas) {
  if (batch < 1 || kv_heads < 1 || num_ctas < 1) return 0;
  const int64_t max_items = static_cast<int64_t>(num_ctas) + static_cast<int64_t>(batch) * kv_heads;
  return plan_layout(batch, kv_heads, num_ctas, static_cast<int32_t>(max_items)).total;
}

extern "C" size_t hpc_plan_static_workspace_bytes(int32_t batch, int32_t kv_heads, int32_t splits) {
  if (batch < 1 || kv_heads < 1 || splits < 1) return 0;
  const int64_t G = static_cast<int64_t>(batch) * kv_heads * splits;
  return plan_layout(batch, kv_heads, static_cast<int32_t>(G), static_cast<int32_t>(G)).total;
}

extern "C" int hpc_decode_plan(const int32_t* seq_lens, int32_t batch, int32_t num_heads, int32_t kv_heads,
                               int32_t tile_len, int32_t num_ctas, int32_t max_seq_len, void* workspace,
                               size_t workspace_bytes, hpc_plan* plan, uint32_t* status, void* stream) {
  int rc = check_plan_args(seq_lens, batch, num_heads, kv_heads, tile_len, num_ctas, workspace, plan, status);
  if (rc) return rc;
  const int64_t max_items = static_cast<int64_t>(num_ctas) + static_cast<int64_t>(batch) * kv_heads;
  if (max_items > (1ll << 30)) return fail(HPC_ERR_SHAPE, "plan too large");
  const PlanLayout L = plan_layout(batch, kv_heads, num_ctas, static_cast<int32_t>(max_items));
  if (workspace_bytes < L.total) return fail(HPC_ERR_CAPACITY, "plan workspace %zu < %zu bytes", workspace_bytes, L.total);
  bind_plan(workspace, L, batch, kv_heads, tile_len, num_ctas, static_cast<int32_t>(max_items), 0, plan);
  const cudaError_t e = launch_pdl(dynamic_plan_kernel, dim3(1), dim3(kPlanThreads), 0, static_cast<cudaStream_t>(stream),
                                   seq_lens, batch, kv_heads, tile_len, num_ctas, max_seq_len,
                                   static_cast<int32_t>(max_items), ptrs_of(plan), status);
  if (e != cudaSuccess) return fail(HPC_ERR_CUDA, "dynamic_plan_kernel: %s", cudaGetErrorString(e));
  return check_launch("dynamic_plan_kernel");
}

extern "C" int hpc_decode_plan_static(const int32_t* seq_lens, int32_t batch, int32_t num_heads, int32_t kv_heads,
                                      int32_t tile_len, int32_t splits, int32_t max_seq_len, void* workspace,
                                      size_t workspace_bytes, hpc_plan* plan, uint32_t* status, void* stream) {
  if (splits < 1) return fail(HPC_ERR_ARG, "splits must be >= 1");
  const int64_t G = static_cast<int64_t>(batch) * kv_heads * splits;
  if (G > (1 << 28)) return fail(HPC_ERR_SHAPE, "static plan too large");
  int rc = check_plan_args(seq_lens, batch, num_heads, kv_heads, tile_len, static_cast<int32_t>(G), workspace, plan,
                           status);
  if (rc) return rc;
  const PlanLayout L = plan_layout(batch, kv_heads, static_cast<int32_t>(G), static_cast<int32_t>(G));
  if (workspace_bytes < L.total) return fail(HPC_ERR_CAPACITY, "plan workspace %zu < %zu bytes", workspace_bytes, L.total);
  bind_plan(workspace, L, batch, kv_heads, tile_len, static_cast<int32_t>(G), static_cast<int32_t>(G), 1, plan);
  const cudaError_t e = launch_pdl(static_plan_kernel, dim3(1), dim3(kPlanThreads), 0, static_cast<cudaStream_t>(stream),
                                   seq_lens, batch, kv_heads, tile_len, splits, max_seq_len, ptrs_of(plan), status);
  if (e != cudaSuccess) return fail(HPC_ERR_CUDA, "static_plan_kernel: %s", cudaGetErrorString(e));
  return check_launch("static_plan_kernel");
}

// Host twin: the same closed form, evaluated sequentially.
extern "C" int hpc_plan_cpu(const int32_t* seq_lens, int32_t batch, int32_t num_heads, int32_t kv_heads,
                            int32_t tile_len, int32_t num_ctas, int32_t max_seq_len, void* workspace,
                            size_t workspace_bytes, hpc_plan* plan, uint32_t* status) {
  int rc = check_plan_args(seq_lens, batch, num_heads, kv_heads, tile_len, num_ctas, workspace, plan, status);
  if (rc) return rc;
  const int64_t max_items = static_cast<int64_t>(num_ctas) + static_cast<int64_t>(batch) * kv_heads;
  const PlanLayout L = plan_layout(batch, kv_heads, num_ctas, static_cast<int32_t>(max_items));
  if (workspace_bytes < L.total) return fail(HPC_ERR_CAPACITY, "plan workspace %zu < %zu bytes", workspace_bytes, L.total);
  memset(workspace, 0, L.total);
  bind_plan(workspace, L, batch, kv_heads, tile_len, num_ctas, static_cast<int32_t>(max_items), 0, plan);
  std::vector<int32_t> nt(batch);
  int64_t total = 0;
  for (int r = 0; r < batch; ++r) {
    int32_t Lr = seq_lens[r];
    if (!len_ok(Lr, max_seq_len)) {
      *status |= HPC_DEV_BAD_SEQLEN;
      Lr = 0;
    }
    nt[r] = tiles_of(Lr, tile_len);
    total += nt[r];
  }
  const int64_t T = total * kv_heads;
  const int64_t chunk = T > 0 ? ceil_div64(T, num_ctas) : 0;
  int64_t idx = 0, midx = 0, U = 0;
  for (int r = 0; r < batch; ++r) {
    for (int kvh = 0; kvh < kv_heads; ++kvh, U += nt[r]) {
      const int64_t s = static_cast<int64_t>(r) * kv_heads + kvh;
      const int32_t pc = pieces_of(U, nt[r], chunk);
      plan->merge_indptr[s] = static_cast<int32_t>(idx);
      if (pc != 1) plan->merge_list[midx++] = static_cast<int32_t>(s);
      for (int32_t j = 0; j < pc; ++j, ++idx) {
        const int64_t start = j == 0 ? U : (U / chunk + j) * chunk;
        const int64_t end = std::min((U / chunk + j + 1) * chunk, U + nt[r]);
        if (idx >= max_items) {
          *status |= HPC_DEV_CAPACITY;
          continue;
        }
        hpc_work_item& w = plan->items[idx];
        w.req = r;
        w.kv_head = static_cast<int16_t>(kvh);
        w.flags = pc == 1 ? HPC_ITEM_DIRECT : 0;
        w.tile_begin = static_cast<int32_t>(start - U);
        w.tile_end = static_cast<int32_t>(end - U);
        if (start % chunk == 0) plan->cta_indptr[start / chunk] = static_cast<int32_t>(idx);
      }
    }
  }
  const int64_t n_items = std::min<int64_t>(idx, max_items);
  const int64_t n_active = chunk > 0 ? ceil_div64(T, chunk) : 0;
  for (int64_t g = n_active; g <= num_ctas; ++g) plan->cta_indptr[g] = static_cast<int32_t>(n_items);
  plan->merge_indptr[static_cast<int64_t>(batch) * kv_heads] = static_cast<int32_t>(n_items);
  plan->counts[0] = n_items;
  plan->counts[1] = midx;
  plan->counts[2] = T;
  plan->counts[3] = chunk;
  return HPC_OK;
}
