// Several new tokens per request on the 5th-generation tensor cores (bf16 cache, head_dim 128).
//
// Same work as the single-launch step of attention.cu with q_len > 1: "腾讯混元三算子杀入 SGLang"
// (AREX), Dynamic Attention paragraph under "Router GEMM：精度不丢，速度翻三倍": a persistent kernel
// runs the tiles that the per-step plan assigns by actual KV length. Items that cover a whole
// (request, kv head) write the output; the others write partial softmax states, merged by the CTA
// that finishes a split (request, kv head) last.
//
// Why another consumer. With mma.sync each query token's warp re-reads the stage's K and V
// fragments from shared memory and runs its own products, and the accumulators of several tokens
// do not fit the register file: four new tokens ran at about half the copy bandwidth, bound by
// per-warp latency. Here the q_len x group query rows of an item (at most 32) are the N of one
// product per stage, the accumulators live in tensor memory, and the operands are read by the
// tensor cores straight from the TMA tiles:
//     S^T[128 tokens x 32 rows] = K[128 x 128 d] . Q^T            (tensor memory, buffer n % 2)
//     O^T[128 d x 32 rows]      = V^T[128 d x 128 tokens] . P^T   (tensor memory, buffer n % 2)
// K and Q^T are K-major with the 128-byte swizzle (two 64-element planes per row); V^T is read as
// an MN-major operand from the same swizzled V tile (leading byte offset = the plane stride); P^T
// is MN-major without swizzle, in core matrices of 8 tokens x 8 rows. P goes in as a bf16 high
// part plus a bf16 residual (two products into the same accumulator), the split that "Tencent HPC
// llega a SGLang …" (remio.ai), section "Dynamic Attention y Fused MoE atacan distintos cuellos de
// botella", describes for an FP32 operand of the Router GEMM.
//
// Roles (320 threads):
//  * warp 9, producer: 128-token stages. K and V have rings of their own (2 and 3 slots of 32 KB),
//    so that a K slot is refilled as soon as its S^T product is done. Boxes of up to 64 tokens never
//    cross a page. Boxes past an item's last token are not loaded, and a page id outside the pool
//    is never handed to TMA (page 0 stands in; the softmax reads the page ids of its own tokens and
//    leaves those tokens out).
//  * warp 8, one lane issues the products in a non-blocking loop (mbarrier.test_wait).
//  * warps 0-7, softmax: two warpgroups take alternate stages, each with its own running state
//    for the item (row maxima, sums and rescale factors in shared memory, output in registers);
//    the two states combine by log-sum-exp at the item end. Thread i owns token row i of S^T and d
//    row i of O^T. Per stage a warpgroup reads S, masks tokens past the item, outside the pool and
//    (per query token) past its causal limit, takes each row's maximum over the 128 tokens (a
//    reduce-scatter over the warp, then shared memory), writes P^T, and folds its previous stage's
//    O^T into registers with the running-maximum correction. O is never rescaled in tensor memory.
// Every wait is bounded (2 s) and ends in HPC_DEV_TIMEOUT; tensor memory is freed on every path.
#include "attention_common.cuh"

namespace hpc {
namespace attn {
namespace {

constexpr int kTmWarps = 10;
constexpr int kTmThreads = kTmWarps * 32;
constexpr int kTmTok = 128;                   // tokens per stage: the M of the S^T product
constexpr int kTmD = 128;                     // head_dim
constexpr int kTmN = 32;                      // query rows per product (q_len x group <= 32)
constexpr int kTmPlane = kTmTok * 128;        // one 64-element plane of a stage's K or V: 16 KB
constexpr int kTmKV = 2 * kTmPlane;           // K (or V) of a stage: 32 KB
constexpr int kTmKS = 2, kTmVS = 3;           // ring slots of K and of V
constexpr int kTmQPlane = kTmN * 128;         // one plane of the Q^T tile: 4 KB
constexpr int kTmQ = 2 * kTmQPlane;           // Q^T tile: 8 KB
constexpr int kTmP = kTmTok * kTmN * 2;       // one P^T matrix (bf16): 8 KB; high + residual per buffer
constexpr uint32_t kTmCols = 128;             // tensor memory: S[2] then O[2], 32 columns each
constexpr int kTmSoftmax = 128;
constexpr int kTmMmaWarp = 8, kTmProducerWarp = 9;
// instruction descriptors: fp32 accumulate, bf16 x bf16, M = 128, N = 32
constexpr uint32_t kTmIdS = (1u << 4) | (1u << 7) | (1u << 10) | ((32u >> 3) << 17) | ((128u >> 4) << 24);
constexpr uint32_t kTmIdO = kTmIdS | (1u << 15) | (1u << 16);  // A and B MN-major

// D (tensor memory, fp32) = A * B (+ D), A and B bf16 in shared memory. Issued by one thread.
__device__ __forceinline__ void umma_bf16(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate));
}

// Whole warp: 32 consecutive 32-bit columns of the warp's 32 lanes (lane = row). Waits for the load.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
        "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]),
        "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

// Reduce v[32] (one value per query row) over the 32 lanes of a warp: five exchange levels each
// keep half of the remaining rows. Lane l returns row l.
template <bool MAX>
__device__ __forceinline__ float warp_reduce32(const float (&v)[32], int lane) {
  auto op = [](float a, float b) { return MAX ? fmaxf(a, b) : a + b; };
  float w16[16], w8[8], w4[4], w2[2];
  const bool b4 = lane & 16, b3 = lane & 8, b2 = lane & 4, b1 = lane & 2, b0 = lane & 1;
#pragma unroll
  for (int k = 0; k < 16; ++k) {
    const float send = b4 ? v[k] : v[k + 16], keep = b4 ? v[k + 16] : v[k];
    w16[k] = op(keep, __shfl_xor_sync(0xffffffffu, send, 16));
  }
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const float send = b3 ? w16[k] : w16[k + 8], keep = b3 ? w16[k + 8] : w16[k];
    w8[k] = op(keep, __shfl_xor_sync(0xffffffffu, send, 8));
  }
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const float send = b2 ? w8[k] : w8[k + 4], keep = b2 ? w8[k + 4] : w8[k];
    w4[k] = op(keep, __shfl_xor_sync(0xffffffffu, send, 4));
  }
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    const float send = b1 ? w4[k] : w4[k + 2], keep = b1 ? w4[k + 2] : w4[k];
    w2[k] = op(keep, __shfl_xor_sync(0xffffffffu, send, 2));
  }
  const float send = b0 ? w2[0] : w2[1], keep = b0 ? w2[1] : w2[0];
  return op(keep, __shfl_xor_sync(0xffffffffu, send, 1));
}

struct TmBars {
  uint32_t base;
  __device__ uint32_t at(int k) const { return base + 8 * k; }
  __device__ uint32_t k_full(int s) const { return at(s); }
  __device__ uint32_t k_empty(int s) const { return at(kTmKS + s); }
  __device__ uint32_t v_full(int s) const { return at(2 * kTmKS + s); }
  __device__ uint32_t v_empty(int s) const { return at(2 * kTmKS + kTmVS + s); }
  static constexpr int kRing = 2 * kTmKS + 2 * kTmVS;
  __device__ uint32_t s_full(int b) const { return at(kRing + b); }
  __device__ uint32_t s_free(int b) const { return at(kRing + 2 + b); }
  __device__ uint32_t p_full(int b) const { return at(kRing + 4 + b); }
  __device__ uint32_t o_full(int b) const { return at(kRing + 6 + b); }
  __device__ uint32_t o_free(int b) const { return at(kRing + 8 + b); }
  __device__ uint32_t q_full(int b) const { return at(kRing + 10 + b); }
  __device__ uint32_t q_free(int b) const { return at(kRing + 12 + b); }
  __device__ uint32_t done() const { return at(kRing + 14); }
  static constexpr int kCount = kRing + 15;
};

// Dynamic shared memory (1024-byte aligned): K ring, V ring, Q^T[2], P^T[2] (high, residual).
constexpr int kTmOffV = kTmKS * kTmKV;
constexpr int kTmOffQ = kTmOffV + kTmVS * kTmKV;
constexpr int kTmOffP = kTmOffQ + 2 * kTmQ;
constexpr int kTmOffBar = kTmOffP + 2 * 2 * kTmP;
constexpr int kTmSmem = kTmOffBar + TmBars::kCount * 8 + 1024;  // + alignment slack

__device__ __forceinline__ int64_t tm_stages(const ItemInfo& x) {
  return x.tok1 > x.tok0 ? (x.tok1 - x.tok0 + kTmTok - 1) / kTmTok : 0;
}

__global__ void __launch_bounds__(kTmThreads, 1)
    decode_attention_tcm_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                                const AttnParams p) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ int64_t s_scan[16], s_walk[9];
  __shared__ int s_flag;
  __shared__ int s_rec_n;
  __shared__ int32_t s_pages[32];
  __shared__ __align__(16) float s_redmax[2][4][kTmN];  // per warpgroup: per-warp row maxima of a stage
  __shared__ __align__(16) float s_redsum[2][4][kTmN];  // per warpgroup: per-warp row sums of a stage
  __shared__ __align__(16) float s_m[2][kTmN];          // per warpgroup: running row maxima (log2 units)
  __shared__ __align__(16) float s_l[2][kTmN];          // per warpgroup: running row sums
  __shared__ __align__(16) float s_a[2][2][kTmN];       // per warpgroup, stage parity: rescale factors
  __shared__ uint32_t s_tmem;
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* kring = smem;
  uint8_t* vring = smem + kTmOffV;
  uint8_t* qt = smem + kTmOffQ;
  uint8_t* pt = smem + kTmOffP;
  const TmBars bar{smem_u32(smem + kTmOffBar)};
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int q_len = p.q_len, group = p.group, rows = q_len * group;  // rows <= kTmN (checked on the host)

  if (threadIdx.x == 0) {
    s_rec_n = 0;
    for (int s = 0; s < kTmKS; ++s) {
      mbar_init(bar.k_full(s), 1);
      mbar_init(bar.k_empty(s), 1);
    }
    for (int s = 0; s < kTmVS; ++s) {
      mbar_init(bar.v_full(s), 1);
      mbar_init(bar.v_empty(s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar.s_full(b), 1);
      mbar_init(bar.s_free(b), 4);
      mbar_init(bar.p_full(b), 4);
      mbar_init(bar.o_full(b), 1);
      mbar_init(bar.o_free(b), 4);
      mbar_init(bar.q_full(b), 4);
      mbar_init(bar.q_free(b), 1);
    }
    mbar_init(bar.done(), 1);
    fence_barrier_init();
  }
  if (warp == kTmMmaWarp) tmem_alloc(smem_u32(&s_tmem), kTmCols);
  if (warp == kTmProducerWarp && lane == 0) {
    prefetch_tensormap(&tm_k);
    prefetch_tensormap(&tm_v);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s_tmem;
  pdl_wait();
  pdl_launch_dependents();

  WalkCursor cursor;
  int64_t chunk = 0;
  // the per-request tile prefix lives in the K ring until the first TMA copy is issued
  plan_in_kernel<kTmD>(p, reinterpret_cast<int64_t*>(kring), s_scan, s_walk, cursor, chunk);
  const int C = p.chunk_tokens;
  const int P = p.page_size;
  const int p_shift = __ffs(P) - 1;
  const int cps = kTmTok / C;  // boxes per stage

  if (warp == kTmProducerWarp) {
    // ------------------------------------------------------------------ producer
    const uint64_t policy = l2_policy_evict_first();
    int64_t n = 0;                  // stages begun
    int64_t filled[2] = {0, 0};     // fills issued: K, V
    bool ok = true;
    uint32_t bad = 0;
    ItemInfo x;
    while (ok && cursor.next(p, x)) {
      const int32_t* bt = p.block_table + static_cast<int64_t>(x.req) * p.max_pages + (x.tok0 >> p_shift);
      const int off0 = static_cast<int>(x.tok0 & (P - 1));
      const int64_t nreal = x.tok1 > x.tok0 ? (x.tok1 - x.tok0 + C - 1) / C : 0;  // boxes with item tokens
      const int64_t nbox = tm_stages(x) * cps;
      for (int64_t cb = 0; cb < nbox && ok; cb += 32) {
        const int nk = static_cast<int>(nbox - cb < 32 ? nbox - cb : 32);
        __syncwarp();
        if (lane < nk) s_pages[lane] = cb + lane < nreal ? bt[(off0 + (cb + lane) * C) >> p_shift] : 0;
        __syncwarp();
        if (lane == 0) {
          // the stage's boxes lie in this batch of page ids (cps divides 32)
          for (int k = 0; k < nk && ok; k += cps, ++n) {
            const int64_t bi = cb + k;
            const int nb = static_cast<int>(nreal - bi < cps ? nreal - bi : cps);
            const uint32_t tx = static_cast<uint32_t>(nb) * 2u * C * 128u;
            for (int kk = 0; kk < nb; ++kk) {
              const int32_t pg = s_pages[k + kk];
              if (pg < 0 || pg >= p.num_pages) bad |= HPC_DEV_BAD_PAGE;
            }
            for (int half = 0; half < 2 && ok; ++half) {  // K, then V
              const int slot = static_cast<int>(half ? n % kTmVS : n % kTmKS);
              const int depth = half ? kTmVS : kTmKS;
              const uint32_t empty = half ? bar.v_empty(slot) : bar.k_empty(slot);
              const uint32_t full = half ? bar.v_full(slot) : bar.k_full(slot);
              if (!mbar_wait(empty, static_cast<uint32_t>(((n / depth) & 1) ^ 1))) {
                ok = false;
                bad |= HPC_DEV_TIMEOUT;
                break;
              }
              mbar_arrive_expect_tx(full, tx);
              const uint32_t base = smem_u32(half ? vring : kring) + slot * kTmKV;
              for (int kk = 0; kk < nb; ++kk) {
                int32_t page = s_pages[k + kk];
                if (page < 0 || page >= p.num_pages) page = 0;  // stand-in; the softmax leaves its tokens out
                const int off = static_cast<int>((off0 + (bi + kk) * C) & (P - 1));
                const int c1 = p.nhd ? x.kvh : off, c2 = p.nhd ? off : x.kvh;
                const uint32_t dst = base + kk * C * 128;
                tma_load_4d(dst, half ? &tm_v : &tm_k, full, 0, c1, c2, page, policy);
                tma_load_4d(dst + kTmPlane, half ? &tm_v : &tm_k, full, 64, c1, c2, page, policy);
              }
              ++filled[half];
            }
          }
        }
        ok = __shfl_sync(0xffffffffu, ok, 0);
        n = __shfl_sync(0xffffffffu, n, 0);
      }
    }
    // Drain: every fill must have landed before the CTA exits. Fill f of a ring went to slot
    // f % depth and completes that slot's full-barrier phase f / depth.
    if (lane == 0) {
      const int64_t nk = filled[0], nv = filled[1];
      for (int64_t f = nk > kTmKS ? nk - kTmKS : 0; f < nk; ++f)
        if (!mbar_wait(bar.k_full(static_cast<int>(f % kTmKS)), static_cast<uint32_t>((f / kTmKS) & 1)))
          bad |= HPC_DEV_TIMEOUT;
      for (int64_t f = nv > kTmVS ? nv - kTmVS : 0; f < nv; ++f)
        if (!mbar_wait(bar.v_full(static_cast<int>(f % kTmVS)), static_cast<uint32_t>((f / kTmVS) & 1)))
          bad |= HPC_DEV_TIMEOUT;
      if (bad) atomicOr(p.status, bad);
    }
  } else if (warp == kTmMmaWarp) {
    // ------------------------------------------------------------------ products
    // One lane issues both streams: S^T of stage nq as soon as its K tile has landed (and its S
    // buffer and the item's Q^T are ready), and O^T of stage npv as soon as its P^T is written and
    // its V tile has landed. A K slot is released by the commit after its S^T product, a V slot by
    // the commit after its O^T products.
    if (lane == 0) {
      WalkCursor qc = cursor;
      ItemInfo xq;
      bool have_q = qc.next(p, xq);
      int64_t q_left = have_q ? tm_stages(xq) : 0;
      int jq = 0;
      bool q_ready = false;
      int64_t nq = 0, npv = 0;
      uint32_t bad = 0;
      uint64_t t_last = global_timer_ns();
      while (true) {
        bool progress = false;
        while (have_q && q_left == 0) {  // items without tokens (cannot occur for a valid plan)
          umma_commit(bar.q_free(jq & 1));
          have_q = qc.next(p, xq);
          q_left = have_q ? tm_stages(xq) : 0;
          ++jq;
        }
        if (have_q) {
          if (!q_ready) q_ready = mbar_test(bar.q_full(jq & 1), static_cast<uint32_t>((jq >> 1) & 1));
          const int ks = static_cast<int>(nq % kTmKS);
          const int b = static_cast<int>(nq & 1);
          if (q_ready && mbar_test(bar.k_full(ks), static_cast<uint32_t>((nq / kTmKS) & 1)) &&
              (nq < 2 || mbar_test(bar.s_free(b), static_cast<uint32_t>(((nq >> 1) - 1) & 1)))) {
            tc_fence_after();
            const uint32_t kbase = smem_u32(kring) + ks * kTmKV;
            const uint32_t qbase = smem_u32(qt) + (jq & 1) * kTmQ;
#pragma unroll
            for (int kk = 0; kk < kTmD / 16; ++kk) {
              const int pl = kk >> 2, sub = kk & 3;
              umma_bf16(tmem + 32 * b, umma_desc(kbase + pl * kTmPlane + 32 * sub, 16, 1024, 2),
                        umma_desc(qbase + pl * kTmQPlane + 32 * sub, 16, 1024, 2), kTmIdS, kk > 0);
            }
            umma_commit(bar.s_full(b));
            umma_commit(bar.k_empty(ks));  // the stage's K is no longer read
            if (--q_left == 0) {
              umma_commit(bar.q_free(jq & 1));  // the item's last read of its Q^T
              have_q = qc.next(p, xq);
              q_left = have_q ? tm_stages(xq) : 0;
              ++jq;
              q_ready = false;
            }
            ++nq;
            progress = true;
          }
        }
        if (npv < nq) {
          const int b = static_cast<int>(npv & 1);
          const int vs = static_cast<int>(npv % kTmVS);
          if (mbar_test(bar.p_full(b), static_cast<uint32_t>((npv >> 1) & 1)) &&
              mbar_test(bar.v_full(vs), static_cast<uint32_t>((npv / kTmVS) & 1)) &&
              (npv < 2 || mbar_test(bar.o_free(b), static_cast<uint32_t>(((npv >> 1) - 1) & 1)))) {
            tc_fence_after();
            const uint32_t vbase = smem_u32(vring) + vs * kTmKV;
            const uint32_t pbase = smem_u32(pt) + b * 2 * kTmP;
#pragma unroll
            for (int kk = 0; kk < kTmTok / 16; ++kk)  // 16 tokens per product: high part of P
              umma_bf16(tmem + 64 + 32 * b, umma_desc(vbase + 2048 * kk, kTmPlane, 1024, 2),
                        umma_desc(pbase + 1024 * kk, 512, 128, 0), kTmIdO, kk > 0);
#pragma unroll
            for (int kk = 0; kk < kTmTok / 16; ++kk)  // residual of P
              umma_bf16(tmem + 64 + 32 * b, umma_desc(vbase + 2048 * kk, kTmPlane, 1024, 2),
                        umma_desc(pbase + kTmP + 1024 * kk, 512, 128, 0), kTmIdO, 1);
            umma_commit(bar.o_full(b));
            umma_commit(bar.v_empty(vs));  // the stage's V is no longer read
            ++npv;
            progress = true;
          }
        } else if (!have_q) {
          break;  // every product issued
        }
        if (progress) {
          t_last = global_timer_ns();
        } else if (global_timer_ns() - t_last > kWaitLimitNs) {
          bad |= HPC_DEV_TIMEOUT;
          break;
        } else {
          __nanosleep(32);
        }
      }
      umma_commit(bar.done());
      if (!mbar_wait(bar.done(), 0)) bad |= HPC_DEV_TIMEOUT;
      if (bad) atomicOr(p.status, bad);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------------ softmax warpgroups
    // Warpgroup w (warps 4w .. 4w+3) takes the stages n with n % 2 == w and keeps its own running
    // state for the item. Control flow is uniform within a warpgroup: loops never end early, and
    // every named barrier is reached by all its threads (barrier 1 + w within a warpgroup, 3 across
    // both). A failed wait (HPC_DEV_TIMEOUT) is made warp-uniform and later waits return at once,
    // so the kernel runs to the end and tensor memory is freed.
    const int w = warp >> 2;
    const int wq = warp & 3;
    const int i = threadIdx.x & (kTmSoftmax - 1);  // token row of S^T, d row of O^T
    const int wbar = 1 + w;
    const uint32_t lrow = static_cast<uint32_t>(wq * 32) << 16;
    zero_empty_requests<kTmD>(p, w * kTmSoftmax + i, 2 * kTmSoftmax);
    int64_t n = 0;  // stage counter over this CTA's items (both warpgroups count every stage)
    int j = 0;
    bool ok = true;
    auto wait = [&](uint32_t b, uint32_t par) -> bool {
      const bool got = __all_sync(0xffffffffu, ok && mbar_wait(b, par));
      if (!got && ok) {
        ok = false;
        if (lane == 0) atomicOr(p.status, HPC_DEV_TIMEOUT);
      }
      return got;
    };
    // Warpgroup 0: Q^T of item y into buffer jy % 2. Row c = t * group + h holds query token t of
    // head kv_head * group + h; rows past q_len * group are zero. Thread i writes 16-byte chunks
    // i, i + 128, i + 256, i + 384 of the 32 x 256-byte tile.
    auto build_q = [&](const ItemInfo& y, int jy) {
      const int qb = jy & 1;
      if (jy >= 2) wait(bar.q_free(qb), static_cast<uint32_t>(((jy >> 1) - 1) & 1));
      uint8_t* qtile = qt + qb * kTmQ;
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int qi = i + kTmSoftmax * k, c = qi >> 4, cc = qi & 15;
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        if (c < rows) {
          const int t = c / group, h = c - t * group;
          v = *reinterpret_cast<const uint4*>(
              p.q + ((static_cast<int64_t>(y.req) * q_len + t) * p.num_heads + y.kvh * group + h) * kTmD + cc * 8);
        }
        *reinterpret_cast<uint4*>(qtile + (cc >> 3) * kTmQPlane + c * 128 + (((cc & 7) ^ (c & 7)) << 4)) = v;
      }
      fence_proxy_async_shared();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar.q_full(qb));
    };

    WalkCursor cur = cursor;
    ItemInfo x;
    bool have = cur.next(p, x);
    if (w == 0 && have) build_q(x, 0);
    while (have) {
      if (w == 0 && i == 0) {
        if (p.record) record_item(p, s_rec_n, x);
        ++s_rec_n;
      }
      const int64_t nst = tm_stages(x);
      const int64_t n0 = n, n_end = n + nst;
      const int64_t L = p.seq_lens[x.req];
      const bool have_next = cur.u < cur.u_end;  // this CTA has another item
      bool built_next = false;
      // the next item's Q^T, written right after warpgroup 0's last P^T of this item
      auto build_next = [&]() {
        WalkCursor a2 = cur;
        ItemInfo y;
        a2.next(p, y);
        build_q(y, j + 1);
        built_next = true;
      };
      if (i < kTmN) {
        s_m[w][i] = -INFINITY;
        s_l[w][i] = 0.f;
      }
      float o_acc[kTmN];
#pragma unroll
      for (int c = 0; c < kTmN; ++c) o_acc[c] = 0.f;
      named_barrier_sync(wbar, kTmSoftmax);  // s_m and s_l are reset for this item
      // fold O^T of stage k into o_acc with that stage's rescale factors (16 columns at a time)
      auto fold = [&](int64_t k) {
        const int b = static_cast<int>(k & 1);
        const bool got = wait(bar.o_full(b), static_cast<uint32_t>((k >> 1) & 1));
        if (got) tc_fence_after();
        const float* a = s_a[w][(k >> 1) & 1];
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          float ov[16];
          if (got) {
            tmem_ld16(tmem + lrow + 64 + 32 * b + 16 * half, ov);
          } else {
#pragma unroll
            for (int c = 0; c < 16; ++c) ov[c] = 0.f;
          }
#pragma unroll
          for (int c = 0; c < 16; ++c) o_acc[16 * half + c] = o_acc[16 * half + c] * a[16 * half + c] + ov[c];
        }
        if (got) tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar.o_free(b));
      };

      int64_t last_own = -1;
      for (int64_t k = n0 + ((n0 & 1) != w ? 1 : 0); k < n_end; k += 2) {
        const int b = w;  // k % 2
        // P buffer b was last read by the O^T products of this warpgroup's previous stage, which
        // the issuing lane may start after this stage's S^T product: fold that stage first (its
        // wait covers the products' completion), before the buffer is overwritten below
        // this thread's token: past the item, or on a page outside the pool, it is dead (the page id
        // is read here, ahead of the waits, so that its latency is hidden)
        const int64_t t = x.tok0 + (k - n0) * kTmTok + i;
        bool tok_ok = t < x.tok1;
        if (tok_ok) {
          const int32_t pg = p.block_table[static_cast<int64_t>(x.req) * p.max_pages + (t >> p_shift)];
          tok_ok = pg >= 0 && pg < p.num_pages;
        }
        if (last_own >= 0) fold(last_own);
        float sv[kTmN];
        if (wait(bar.s_full(b), static_cast<uint32_t>((k >> 1) & 1))) {
          tc_fence_after();
          tmem_ld32(tmem + lrow + 32 * b, sv);
          tc_fence_before();
        } else {
#pragma unroll
          for (int c = 0; c < kTmN; ++c) sv[c] = 0.f;
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(bar.s_free(b));
        // A dead token's V row may hold anything (even NaN): it is zeroed, so that 0 * v stays 0.
        // Only a warp with a dead token waits for the stage's V fill (its slot is refilled only after
        // this stage's O^T product, which waits for the P^T written below, so the phase cannot have
        // moved on); the others never wait on V.
        if (__any_sync(0xffffffffu, !tok_ok)) {
          const int vs = static_cast<int>(k % kTmVS);
          if (wait(bar.v_full(vs), static_cast<uint32_t>((k / kTmVS) & 1)) && !tok_ok) {
            uint8_t* vrow = vring + vs * kTmKV + i * 128;
#pragma unroll
            for (int c = 0; c < 8; ++c) {
              reinterpret_cast<uint4*>(vrow)[c] = make_uint4(0u, 0u, 0u, 0u);
              reinterpret_cast<uint4*>(vrow + kTmPlane)[c] = make_uint4(0u, 0u, 0u, 0u);
            }
          }
        }
        // row c is query token c / group: it sits at L - q_len + c / group and sees tokens up to
        // it, so token t is live for the rows c in [c_lo, rows) with c_lo = group * (t - (L - q_len))
        {
          const int64_t behind = t - (L - q_len);  // query tokens this token is ahead of (<= 0: all see it)
          const int c_lo = behind <= 0 ? 0 : (behind >= q_len ? kTmN : static_cast<int>(behind) * group);
          const int c_hi = tok_ok ? rows : 0;
#pragma unroll
          for (int c = 0; c < kTmN; ++c) sv[c] = (c >= c_lo && c < c_hi) ? sv[c] * p.score_scale : -INFINITY;
        }
        // row maxima over the warpgroup's 128 tokens; lane c of warp 0 sets row c's new maximum
        // and rescale factor
        s_redmax[w][wq][lane] = warp_reduce32<true>(sv, lane);
        named_barrier_sync(wbar, kTmSoftmax);
        float* a_k = s_a[w][(k >> 1) & 1];
        if (wq == 0) {
          if (last_own >= 0)  // the previous own stage's row sums, with that stage's rescale factor
            s_l[w][lane] = s_l[w][lane] * s_a[w][(last_own >> 1) & 1][lane] +
                           ((s_redsum[w][0][lane] + s_redsum[w][1][lane]) + (s_redsum[w][2][lane] + s_redsum[w][3][lane]));
          const float mx = fmaxf(fmaxf(s_redmax[w][0][lane], s_redmax[w][1][lane]),
                                 fmaxf(s_redmax[w][2][lane], s_redmax[w][3][lane]));
          const float mo = s_m[w][lane], mn = fmaxf(mo, mx);
          const float mr = mn == -INFINITY ? 0.f : mn;  // no live token yet: adds nothing
          a_k[lane] = exp2f(mo - mr);
          s_m[w][lane] = mn;
        }
        named_barrier_sync(wbar, kTmSoftmax);
        // P^T, MN-major without swizzle: token i, rows 8m .. 8m + 7 at (i/8)*512 + m*128 + (i%8)*16,
        // as a bf16 high part and a bf16 residual; sv takes p
        uint8_t* pb = pt + b * 2 * kTmP + (i >> 3) * 512 + (i & 7) * 16;
#pragma unroll
        for (int m = 0; m < kTmN / 8; ++m) {
          uint32_t hi[4], lo[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int c = 8 * m + 2 * e;
            const float m0 = s_m[w][c], m1 = s_m[w][c + 1];
            const float p0 = exp2f(sv[c] - (m0 == -INFINITY ? 0.f : m0));
            const float p1 = exp2f(sv[c + 1] - (m1 == -INFINITY ? 0.f : m1));
            sv[c] = p0;
            sv[c + 1] = p1;
            const uint32_t hh = pack_bf16x2(p0, p1);
            hi[e] = hh;
            lo[e] = pack_bf16x2(p0 - __uint_as_float(hh << 16), p1 - __uint_as_float(hh & 0xffff0000u));
          }
          *reinterpret_cast<uint4*>(pb + m * 128) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
          *reinterpret_cast<uint4*>(pb + kTmP + m * 128) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
        }
        fence_proxy_async_shared();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar.p_full(b));
        // row sums of p over the 128 tokens; warp 0 folds them into the running sums during this
        // warpgroup's next stage (or at the item end)
        s_redsum[w][wq][lane] = warp_reduce32<false>(sv, lane);
        if (w == 0 && have_next && k + 2 >= n_end) build_next();
        last_own = k;
      }
      if (w == 0 && have_next && !built_next) build_next();  // no stage of this item here
      if (last_own >= 0) {
        fold(last_own);
        named_barrier_sync(wbar, kTmSoftmax);  // the last stage's row sums are written
        if (wq == 0)
          s_l[w][lane] = s_l[w][lane] * s_a[w][(last_own >> 1) & 1][lane] +
                         ((s_redsum[w][0][lane] + s_redsum[w][1][lane]) + (s_redsum[w][2][lane] + s_redsum[w][3][lane]));
      }
      n = n_end;

      // ---- item end: the two warpgroups' states combined by log-sum-exp. The exchange and merge
      // buffers alias the P^T buffers: both warpgroups have folded their last stage (its products
      // are done), and no P^T is written until the item end is over.
      float* xo = reinterpret_cast<float*>(pt + 2 * kTmP);  // P buffer 1: warpgroup 1's O rows
      if (w == 1) {
#pragma unroll
        for (int c = 0; c < kTmN; c += 4)
          *reinterpret_cast<float4*>(xo + i * kTmN + c) = make_float4(o_acc[c], o_acc[c + 1], o_acc[c + 2], o_acc[c + 3]);
      }
      named_barrier_sync(3, 2 * kTmSoftmax);  // s_m, s_l of both warpgroups and xo are complete
      if (w == 0) {
        const int head0 = x.kvh * group;
        int tq = 0, h = 0;
#pragma unroll
        for (int c = 0; c < kTmN; ++c) {  // unrolled: o_acc stays in registers
          if (c < rows) {
            const float m0 = s_m[0][c], m1 = s_m[1][c], M = fmaxf(m0, m1);
            const float Mr = M == -INFINITY ? 0.f : M;  // neither warpgroup saw a live token
            const float f0 = exp2f(m0 - Mr), f1 = exp2f(m1 - Mr);
            const float Lc = s_l[0][c] * f0 + s_l[1][c] * f1;
            const float oc = o_acc[c] * f0 + xo[i * kTmN + c] * f1;
            if (x.direct) {
              const float val = Lc > 0.f ? oc / Lc : 0.f;
              const int64_t oi = ((static_cast<int64_t>(x.req) * q_len + tq) * p.num_heads + head0 + h) * kTmD + i;
              if (p.out_bf16) reinterpret_cast<__nv_bfloat16*>(p.out)[oi] = __float2bfloat16_rn(val);
              else reinterpret_cast<float*>(p.out)[oi] = val;
            } else {
              const int64_t pi = (x.slot * q_len + tq) * group + h;
              p.partial_o[pi * kTmD + i] = oc;
              if (i == 0) {
                p.partial_ml[2 * pi] = M * kLn2;  // natural-log units
                p.partial_ml[2 * pi + 1] = Lc;
              }
            }
          }
          if (++h == group) {
            h = 0;
            ++tq;
          }
        }
        if (!x.direct) {
          // the CTA that completes the last piece of this (request, kv head) merges it
          __threadfence();
          named_barrier_sync(1, kTmSoftmax);
          if (i == 0) {
            int64_t g1, g2, first_slot;
            segment_ctas(x, p.item_cost, chunk, g1, g2, first_slot);
            const int64_t pieces = g2 - g1 + 1;
            int32_t* ticket = p.tickets + static_cast<int64_t>(x.req) * p.kv_heads + x.kvh;
            const int old = atomicAdd(ticket, 1);
            const int last = old == pieces - 1;
            if (last) {
              __threadfence();
              *ticket = 0;  // ready for the next step
            }
            s_flag = last;
          }
          named_barrier_sync(1, kTmSoftmax);
          if (s_flag) merge_segment<kTmD>(p, x, chunk, i, kTmSoftmax, reinterpret_cast<float*>(pt), 2 * kTmP / 4);
        }
      }
      named_barrier_sync(3, 2 * kTmSoftmax);  // the exchange and merge buffers are P^T again
      ++j;
      have = cur.next(p, x);
    }
    if (p.record && w == 0 && i == 0) record_header(p, s_walk[0], s_walk[1], s_walk[7], s_rec_n);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kTmMmaWarp) {
    tc_fence_after();
    tmem_free(tmem, kTmCols);
  }
}

}  // namespace

bool tcm_supported(int head_dim, bool fp8, int group, int q_len, bool pro) {
  return !fp8 && !pro && head_dim == kTmD && group >= 1 && q_len >= 1 && q_len * group <= kTmN;
}

int launch_attention_tcm(const CUtensorMap& mk, const CUtensorMap& mv, const AttnParams& prm, int grid,
                         cudaStream_t stream) {
  if (prm.chunk_tokens < 16 || kTmTok % prm.chunk_tokens) return fail(HPC_ERR_SHAPE, "box of %d tokens", prm.chunk_tokens);
  if (prm.q_len * prm.group > kTmN) return fail(HPC_ERR_SHAPE, "q_len x group above %d", kTmN);
  static int configured[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !configured[dev]) {
    if (cudaFuncSetAttribute(decode_attention_tcm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kTmSmem) !=
        cudaSuccess)
      return check_launch("cudaFuncSetAttribute(decode_attention_tcm_kernel)");
    configured[dev] = 1;
  }
  const cudaError_t e = launch_pdl(decode_attention_tcm_kernel, dim3(grid), dim3(kTmThreads),
                                   static_cast<size_t>(kTmSmem), stream, mk, mv, prm);
  if (e != cudaSuccess) return fail(HPC_ERR_CUDA, "decode_attention_tcm_kernel: %s", cudaGetErrorString(e));
  return check_launch("decode_attention_tcm_kernel");
}

}  // namespace attn
}  // namespace hpc
