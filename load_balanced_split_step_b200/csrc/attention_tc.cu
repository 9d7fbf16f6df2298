// Persistent split-KV decode attention for an E4M3 cache on the 5th-generation tensor cores.
//
// Same work as decode_attention_kernel in attention.cu: "腾讯混元三算子杀入 SGLang" (AREX), the
// Dynamic Attention paragraph under "Router GEMM：精度不丢，速度翻三倍": a persistent kernel
// runs the tiles that the per-step plan assigns by actual KV length. Items that cover a whole
// (request, kv head) write the output; the others write partial softmax states for the
// log-sum-exp merge (a ticket merge in the single-launch step).
//
// Why another consumer for E4M3. With mma.sync, every E4M3 code has to be widened to f16 in
// registers before the product; on the large-batch workload that widening keeps the SMs busy
// enough to draw the 1 kW cap. tcgen05.mma kind::f8f6f4 reads the codes where TMA put them.
//
// Roles (320 threads):
//  * warp 9, producer: streams 128-token stages (K then V, 16 KB each) into a ring by TMA,
//    as the mma.sync kernel does, in boxes of up to 64 tokens that never cross a page.
//    Boxes past an item's last token are not loaded: their rows hold whatever the slot held
//    before, and the softmax masks those tokens and zeroes their V rows. A page id outside the
//    pool is never handed to TMA either: page 0 stands in, and the box's tokens are masked.
//  * warp 8, one lane issues the products. Per stage n:
//      S^T[128 tokens x 16] = K[128 x 128] . Qhl^T          (tensor memory, buffer n % 2)
//      O^T[128 d x 16]      = V^T[128 x 128 tokens] . Phl    (tensor memory, buffer n % 2)
//    Qhl holds the item's 8 query heads twice: E4M3 codes of q scaled by a power of two,
//    then the codes of the exact residual; S = S_high + S_low recovers ~8 significant bits
//    of q. Phl likewise holds the E4M3 high and residual codes of p for the 8 heads. K is
//    K-major with the 128-byte swizzle TMA wrote; V is read as an MN-major A operand from the
//    same layout; Phl is MN-major without swizzle, 16 bytes per token.
//  * warps 0-7, softmax: two warpgroups take alternate stages, each with its own running state
//    for the item, combined by log-sum-exp at the item end. In a warpgroup, thread i owns token
//    row i of S^T and d row i of O^T. Per stage a warpgroup reads S, takes the row max of each
//    head across the 128 tokens (a reduce-scatter over the warp, then shared memory), folds its
//    previous stage's O^T into registers with the running-max correction, and writes Phl for
//    p = 2^(s - m + 8) (the 2^8 keeps the E4M3 codes of p away from underflow; p <= 256 < 448).
//    O is never rescaled in tensor memory.
// Each stage is a separate pair of products with its own buffers (two of each), so the softmax
// of one stage overlaps the products of the next. Tensor memory: 64 columns (S[2], O[2]).
// Measured, this kernel is slower than the mma.sync one for one new token per request (each
// stage chains two product round trips through mbarriers, with N = 16), so it is opt-in.
// Every wait is bounded (2 s) and ends in HPC_DEV_TIMEOUT; tensor memory is freed on every
// path.
#include "attention_common.cuh"

namespace hpc {
namespace attn {
namespace {

constexpr int kTcWarps = 10;
constexpr int kTcThreads = kTcWarps * 32;
constexpr int kTcTok = 128;                    // tokens per stage: the M of the QK product
constexpr int kTcD = 128;                      // head_dim: one 128-byte row per token
constexpr int kTcHalf = kTcTok * kTcD;         // K (or V) codes of a stage: 16 KB
constexpr int kTcStage = 2 * kTcHalf;
constexpr int kTcQ = 16 * 128;                 // Qhl tile
constexpr int kTcP = kTcTok * 16;              // Phl tile
constexpr int kTcMerge = 1024;                 // floats for the ticket merge
constexpr uint32_t kTmemCols = 64;
constexpr int kSoftmax = 128;                  // threads of one softmax warpgroup
constexpr int kMmaWarp = 8, kProducerWarp = 9;
// instruction descriptors: fp32 accumulate, E4M3 x E4M3, M = 128, N = 16
constexpr uint32_t kIdQK = (1u << 4) | ((16u >> 3) << 17) | ((128u >> 4) << 24);  // A, B K-major
constexpr uint32_t kIdPV = kIdQK | (1u << 15) | (1u << 16);                       // A, B MN-major

// Reduce v[8] (one value per head) over the 32 lanes of a warp: three exchange levels each
// keep half the heads, then two plain levels. Lane l returns head (l >> 2) & 7.
template <bool MAX>
__device__ __forceinline__ float warp_reduce8(const float (&v)[8], int lane) {
  auto op = [](float a, float b) { return MAX ? fmaxf(a, b) : a + b; };
  const bool b4 = lane & 16, b3 = lane & 8, b2 = lane & 4;
  float w4[4], w2[2];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const float send = b4 ? v[k] : v[k + 4];
    const float keep = b4 ? v[k + 4] : v[k];
    w4[k] = op(keep, __shfl_xor_sync(0xffffffffu, send, 16));
  }
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    const float send = b3 ? w4[k] : w4[k + 2];
    const float keep = b3 ? w4[k + 2] : w4[k];
    w2[k] = op(keep, __shfl_xor_sync(0xffffffffu, send, 8));
  }
  const float send = b2 ? w2[0] : w2[1];
  const float keep = b2 ? w2[1] : w2[0];
  float w = op(keep, __shfl_xor_sync(0xffffffffu, send, 4));
  w = op(w, __shfl_xor_sync(0xffffffffu, w, 2));
  w = op(w, __shfl_xor_sync(0xffffffffu, w, 1));
  return w;
}

// v[8] reduced over the 128 softmax threads into out[8] (every thread gets all 8). scratch
// holds 32 floats; it contains one barrier, so a caller that reuses scratch must separate the
// uses by another barrier.
template <bool MAX>
__device__ __forceinline__ void wg_reduce8(const float (&v)[8], float (&out)[8], float* scratch, int warp, int lane,
                                           int barrier) {
  const float w = warp_reduce8<MAX>(v, lane);
  if ((lane & 3) == 0) scratch[((lane >> 2) & 7) * 4 + warp] = w;
  named_barrier_sync(barrier, kSoftmax);
#pragma unroll
  for (int h = 0; h < 8; ++h) {
    const float4 r = reinterpret_cast<const float4*>(scratch)[h];
    out[h] = MAX ? fmaxf(fmaxf(r.x, r.y), fmaxf(r.z, r.w)) : (r.x + r.y) + (r.z + r.w);
  }
}

__device__ __forceinline__ float wg_max1(float v, float* scratch, int warp, int barrier) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, off));
  if ((threadIdx.x & 31) == 0) scratch[warp] = v;
  named_barrier_sync(barrier, kSoftmax);
  return fmaxf(fmaxf(scratch[0], scratch[1]), fmaxf(scratch[2], scratch[3]));
}

// E4M3 codes of 8 values and of their exact residuals: (high codes, residual codes).
__device__ __forceinline__ void split_e4m3x8(const float (&v)[8], uint2& hi, uint2& lo) {
  hi.x = f32x4_to_e4m3x4(v[0], v[1], v[2], v[3]);
  hi.y = f32x4_to_e4m3x4(v[4], v[5], v[6], v[7]);
  float a[4], b[4];
  e4m3x4_to_f32x4(hi.x, a);
  e4m3x4_to_f32x4(hi.y, b);
  lo.x = f32x4_to_e4m3x4(v[0] - a[0], v[1] - a[1], v[2] - a[2], v[3] - a[3]);
  lo.y = f32x4_to_e4m3x4(v[4] - b[0], v[5] - b[1], v[6] - b[2], v[7] - b[3]);
}

struct TcBars {
  uint32_t base;
  int stages;
  __device__ uint32_t full(int s) const { return base + 8 * s; }
  __device__ uint32_t empty(int s) const { return base + 8 * (stages + s); }
  __device__ uint32_t at(int k) const { return base + 8 * (2 * stages + k); }
  __device__ uint32_t s_full(int b) const { return at(0 + b); }
  __device__ uint32_t s_free(int b) const { return at(2 + b); }
  __device__ uint32_t p_full(int b) const { return at(4 + b); }
  __device__ uint32_t o_full(int b) const { return at(6 + b); }
  __device__ uint32_t o_free(int b) const { return at(8 + b); }
  __device__ uint32_t q_full(int b) const { return at(10 + b); }
  __device__ uint32_t q_free(int b) const { return at(12 + b); }
  __device__ uint32_t done() const { return at(14); }
  static constexpr int kExtra = 15;
};

__device__ __forceinline__ int64_t stages_of(const ItemInfo& x) {
  return x.tok1 > x.tok0 ? (x.tok1 - x.tok0 + kTcTok - 1) / kTcTok : 0;
}

template <bool FUSED>
__global__ void __launch_bounds__(kTcThreads, 1)
    decode_attention_tc_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                               const AttnParams p) {
  using Cursor = typename CursorOf<FUSED>::type;
  extern __shared__ uint8_t smem_raw[];
  __shared__ int64_t s_scan[16], s_walk[9];
  __shared__ int s_flag;
  __shared__ int32_t s_pages[32];
  __shared__ uint32_t s_tmem;
  __shared__ __align__(16) float s_red[2][2][32];  // per warpgroup: per-stage head maxima (double buffered)
  __shared__ __align__(16) float s_red2[2][32];    // per warpgroup: item-level sums
  __shared__ float s_qmax[4];                      // q amax of the warpgroup that writes Qhl
  __shared__ float s_sq[2];                        // q scale of each Qhl buffer
  __shared__ float s_xm[8], s_xl[8];               // warpgroup 1's (m, l) at an item end
  __shared__ uint8_t s_badbox[16];                 // per ring slot: boxes whose page id was out of range
  __shared__ int s_rec_n;                          // items this CTA has run (single-launch record)
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int stages = p.stages;
  uint8_t* ring = smem;
  uint8_t* qt = ring + static_cast<size_t>(stages) * kTcStage;
  uint8_t* pt = qt + 2 * kTcQ;
  float* mrg = reinterpret_cast<float*>(pt + 2 * kTcP);
  const TcBars bar{smem_u32(mrg + kTcMerge), stages};
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t ring_u32 = smem_u32(ring);

  if (threadIdx.x == 0) {
    s_rec_n = 0;
    for (int s = 0; s < stages; ++s) {
      mbar_init(bar.full(s), 1);
      mbar_init(bar.empty(s), 1);
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
  if (warp == kMmaWarp) tmem_alloc(smem_u32(&s_tmem), kTmemCols);
  if (warp == kProducerWarp && lane == 0) {
    prefetch_tensormap(&tm_k);
    prefetch_tensormap(&tm_v);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s_tmem;
  // the single launch's plan reads seq_lens alone: before the wait on the previous kernel when
  // that kernel does not write them (plan_early), after it otherwise
  const bool early = FUSED && p.plan_early;
  if (!early) {
    pdl_wait();
    pdl_launch_dependents();
  }

  Cursor cursor;
  int64_t chunk = 0;
  if constexpr (FUSED) {
    // the per-request tile prefix lives in the ring until the first TMA copy is issued
    plan_in_kernel<kTcD>(p, reinterpret_cast<int64_t*>(ring), s_scan, s_walk, cursor, chunk);
    if (early) {
      pdl_wait();
      pdl_launch_dependents();
    }
  } else {
    cursor.it = p.cta_indptr[blockIdx.x];
    cursor.it_end = p.cta_indptr[blockIdx.x + 1];
  }
  const int C = p.chunk_tokens;
  const int P = p.page_size;
  const int cps = kTcTok / C;  // boxes per stage

  if (warp == kProducerWarp) {
    // ------------------------------------------------------------------ producer
    const uint64_t policy = l2_policy_evict_first();
    const int p_shift = __ffs(P) - 1;
    int slot = 0;
    uint32_t phase = 0;
    int64_t issued = 0;
    bool ok = true;
    uint32_t bad = 0;
    ItemInfo x;
    while (ok && cursor.next(p, x)) {
      const int32_t* bt = p.block_table + x.req * p.max_pages + (x.tok0 >> p_shift);
      const int off0 = static_cast<int>(x.tok0 & (P - 1));
      const int64_t nreal = x.tok1 > x.tok0 ? (x.tok1 - x.tok0 + C - 1) / C : 0;  // boxes that hold item tokens
      const int64_t nbox = stages_of(x) * cps;
      for (int64_t cb = 0; cb < nbox && ok; cb += 32) {
        const int nk = static_cast<int>(nbox - cb < 32 ? nbox - cb : 32);
        __syncwarp();
        if (lane < nk) s_pages[lane] = cb + lane < nreal ? bt[(off0 + (cb + lane) * C) >> p_shift] : 0;
        __syncwarp();
        if (lane == 0) {
          for (int k = 0; k < nk; ++k) {
            const int64_t bi = cb + k;
            const int kc = static_cast<int>(bi % cps);
            if (kc == 0) {
              if (!mbar_wait(bar.empty(slot), phase ^ 1)) {
                ok = false;
                bad |= HPC_DEV_TIMEOUT;
                break;
              }
              // boxes of this stage that hold item tokens (the stage's boxes lie in this batch
              // of page ids, as cps divides 32), and those whose page id is out of range
              const int nb = static_cast<int>(nreal - bi < cps ? nreal - bi : cps);
              uint32_t mask = 0;
              for (int kk = 0; kk < nb; ++kk) {
                const int32_t pg = s_pages[k + kk];
                if (pg < 0 || pg >= p.num_pages) mask |= 1u << kk;
              }
              if (mask) bad |= HPC_DEV_BAD_PAGE;
              s_badbox[slot] = static_cast<uint8_t>(mask);
              mbar_arrive_expect_tx(bar.full(slot), static_cast<uint32_t>(nb) * 2u * C * 128u);
            }
            if (bi < nreal) {
              int32_t page = s_pages[k];
              if (page < 0 || page >= p.num_pages) page = 0;  // stand-in; the softmax masks the box
              const int off = static_cast<int>((off0 + bi * C) & (P - 1));
              const int c1 = p.nhd ? x.kvh : off, c2 = p.nhd ? off : x.kvh;
              const uint32_t dst = ring_u32 + slot * kTcStage + kc * C * 128;
              tma_load_4d(dst, &tm_k, bar.full(slot), 0, c1, c2, page, policy);
              tma_load_4d(dst + kTcHalf, &tm_v, bar.full(slot), 0, c1, c2, page, policy);
            }
            if (kc == cps - 1) {
              ++issued;
              if (++slot == stages) {
                slot = 0;
                phase ^= 1;
              }
            }
          }
        }
        ok = __shfl_sync(0xffffffffu, ok, 0);
      }
    }
    // Drain: every fill must have landed before the CTA exits. Fill f went to slot f % stages
    // and completes that slot's full-barrier phase f / stages.
    if (lane == 0) {
      for (int64_t f = issued > stages ? issued - stages : 0; f < issued; ++f)
        if (!mbar_wait(bar.full(static_cast<int>(f % stages)), static_cast<uint32_t>((f / stages) & 1)))
          bad |= HPC_DEV_TIMEOUT;
      if (bad) atomicOr(p.status, bad);
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------------ products
    // One lane issues both streams of products in a polling loop: S^T of stage nq as soon as
    // its K tile has landed (and its S buffer and the item's Qhl are ready), and O^T of stage
    // npv as soon as its P is written. Neither waits for the other, so a ring slot is released
    // (by the commit after its O^T product) as soon as its own softmax is done.
    if (lane == 0) {
      Cursor qc = cursor;
      ItemInfo xq;
      bool have_q = qc.next(p, xq);
      int64_t q_left = have_q ? stages_of(xq) : 0;  // stages of the current item still to issue
      int jq = 0;                                    // item of stage nq
      bool q_ready = false;                          // its Qhl is written
      int64_t nq = 0, npv = 0;
      bool ok = true;
      uint32_t bad = 0;
      uint64_t t_last = global_timer_ns();
      while (true) {
        bool progress = false;
        while (have_q && q_left == 0) {  // items without tokens (cannot occur for a valid plan)
          umma_commit(bar.q_free(jq & 1));  // keep one q_free completion per item
          have_q = qc.next(p, xq);
          q_left = have_q ? stages_of(xq) : 0;
          ++jq;
        }
        if (have_q) {
          if (!q_ready) q_ready = mbar_test(bar.q_full(jq & 1), static_cast<uint32_t>((jq >> 1) & 1));
          const int slot = static_cast<int>(nq % stages);
          const int b = static_cast<int>(nq & 1);
          if (q_ready && mbar_test(bar.full(slot), static_cast<uint32_t>((nq / stages) & 1)) &&
              (nq < 2 || mbar_test(bar.s_free(b), static_cast<uint32_t>(((nq >> 1) - 1) & 1)))) {
            tc_fence_after();
            const uint32_t kbase = ring_u32 + slot * kTcStage;
            const uint32_t qbase = smem_u32(qt) + (jq & 1) * kTcQ;
#pragma unroll
            for (int kk = 0; kk < kTcD / 32; ++kk)
              umma_e4m3(tmem + 16 * b, umma_desc(kbase + 32 * kk, 16, 1024, 2), umma_desc(qbase + 32 * kk, 16, 1024, 2),
                        kIdQK, kk > 0);
            umma_commit(bar.s_full(b));
            if (--q_left == 0) {
              umma_commit(bar.q_free(jq & 1));  // the item's last read of its Qhl
              have_q = qc.next(p, xq);
              q_left = have_q ? stages_of(xq) : 0;
              ++jq;
              q_ready = false;
            }
            ++nq;
            progress = true;
          }
        }
        if (npv < nq) {
          const int b = static_cast<int>(npv & 1);
          if (mbar_test(bar.p_full(b), static_cast<uint32_t>((npv >> 1) & 1)) &&
              (npv < 2 || mbar_test(bar.o_free(b), static_cast<uint32_t>(((npv >> 1) - 1) & 1)))) {
            tc_fence_after();
            const int sl = static_cast<int>(npv % stages);
            const uint32_t vbase = ring_u32 + sl * kTcStage + kTcHalf;
            const uint32_t pbase = smem_u32(pt) + b * kTcP;
#pragma unroll
            for (int kk = 0; kk < kTcTok / 32; ++kk)
              umma_e4m3(tmem + 32 + 16 * b, umma_desc(vbase + 4096 * kk, 16, 1024, 2),
                        umma_desc(pbase + 512 * kk, 128, 16, 0), kIdPV, kk > 0);
            umma_commit(bar.o_full(b));
            umma_commit(bar.empty(sl));  // the stage's K and V are no longer read
            ++npv;
            progress = true;
          }
        } else if (!have_q) {
          break;  // every product issued
        }
        if (progress) {
          t_last = global_timer_ns();
        } else if (global_timer_ns() - t_last > kWaitLimitNs) {
          ok = false;
          bad |= HPC_DEV_TIMEOUT;
          break;
        } else {
          __nanosleep(32);
        }
      }
      umma_commit(bar.done());
      if (!mbar_wait(bar.done(), 0)) bad |= HPC_DEV_TIMEOUT;
      if (bad) atomicOr(p.status, bad);
      (void)ok;
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------------ softmax warpgroups
    // Warpgroup w (warps 4w .. 4w+3) takes the stages n with n % 2 == w, and keeps its own
    // running (m, l, O) for the item; the two states are combined by log-sum-exp at the item
    // end. Warpgroup 0 also writes each item's Qhl.
    // Control flow is uniform within a warpgroup: loops never end early, and every named
    // barrier is reached by all its threads (barrier 1 + w within a warpgroup, 3 across both).
    // A failed wait (HPC_DEV_TIMEOUT) is made warp-uniform and later waits return at once, so
    // the kernel runs to the end and tensor memory is freed.
    const int w = warp >> 2;    // warpgroup
    const int wq = warp & 3;    // warp within the warpgroup: tensor-memory lanes 32 wq ..
    const int i = threadIdx.x & (kSoftmax - 1);  // token row of S^T, d row of O^T
    const int wbar = 1 + w;
    const uint32_t lrow = static_cast<uint32_t>(wq * 32) << 16;
    float* xo = mrg;  // warpgroup 1's O rows at an item end (the merge buffer is free then)
    if constexpr (FUSED) {
      if (w == 0) zero_empty_requests<kTcD>(p, i, kSoftmax);
    }
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
    // Warpgroup 0: Qhl of item y into buffer jy % 2. Thread i holds head i / 16,
    // d = 8 (i % 16) .. + 7. The power of two that scaled q goes to s_sq.
    auto build_q = [&](const ItemInfo& y, int jy) {
      const int qb = jy & 1;
      if (jy >= 2) wait(bar.q_free(qb), static_cast<uint32_t>(((jy >> 1) - 1) & 1));
      const int h = i >> 4, d0 = (i & 15) * 8;
      const bool live = h < p.group;
      float v[8];
      uint4 raw = make_uint4(0u, 0u, 0u, 0u);
      if (live)
        raw = *reinterpret_cast<const uint4*>(
            p.q + (static_cast<int64_t>(y.req) * p.num_heads + y.kvh * p.group + h) * kTcD + d0);
      const uint32_t wd[4] = {raw.x, raw.y, raw.z, raw.w};
      float amax = 0.f;
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        v[2 * k] = __uint_as_float(wd[k] << 16);
        v[2 * k + 1] = __uint_as_float(wd[k] & 0xffff0000u);
        amax = fmaxf(amax, fmaxf(fabsf(v[2 * k]), fabsf(v[2 * k + 1])));
      }
      amax = wg_max1(amax, s_qmax, wq, wbar);
      // a power of two that puts the group's largest |q| in [128, 256)
      int se = 7 - (static_cast<int>((__float_as_uint(amax) >> 23) & 0xffu) - 127);
      se = se < -126 ? -126 : (se > 127 ? 127 : se);
      const float sq = __uint_as_float(static_cast<uint32_t>(se + 127) << 23);
#pragma unroll
      for (int k = 0; k < 8; ++k) v[k] *= sq;
      uint2 hi, lo;
      split_e4m3x8(v, hi, lo);
      // K-major tile, 128-byte swizzle: row r, 16-byte chunk c at r * 128 + ((c ^ (r & 7)) << 4)
      uint8_t* qtile = qt + qb * kTcQ;
      const int c = d0 >> 4, half = d0 & 15;
      *reinterpret_cast<uint2*>(qtile + h * 128 + ((c ^ h) << 4) + half) = hi;
      *reinterpret_cast<uint2*>(qtile + (8 + h) * 128 + ((c ^ h) << 4) + half) = lo;
      if (i == 0) s_sq[qb] = sq;
      fence_proxy_async_shared();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar.q_full(qb));
      named_barrier_sync(wbar, kSoftmax);  // s_qmax is free again
    };

    ItemInfo x;
    bool have = cursor.next(p, x);
    if (w == 0 && have) build_q(x, 0);
    while (have) {
      const int kvh = x.kvh, head0 = kvh * p.group;
      if (w == 0 && i == 0) {
        if (FUSED && p.record) record_item(p, s_rec_n, x);
        ++s_rec_n;
      }
      const int64_t nst = stages_of(x);
      const int64_t n0 = n, n_end = n + nst;
      // the next item's Qhl is written right after warpgroup 0's last P of this item, so that
      // the next item's first product can run while this one ends
      Cursor ahead = cursor;
      ItemInfo y;
      const bool have_next = ahead.next(p, y);
      bool built_next = false;
      // this item's q scale (warpgroup 1 reads it once Qhl is complete)
      if (w == 1) wait(bar.q_full(j & 1), static_cast<uint32_t>((j >> 1) & 1));
      const float score_scale = p.score_scale * p.k_scale[kvh] / s_sq[j & 1];

      float m_run[8], l_part[8], o_acc[8], a_prev[8];
#pragma unroll
      for (int h = 0; h < 8; ++h) {
        m_run[h] = -INFINITY;
        l_part[h] = 0.f;
        o_acc[h] = 0.f;
        a_prev[h] = 0.f;
      }
      // fold O^T of stage k into o_acc with the factor that moves o_acc to that stage's max
      auto fold = [&](int64_t k, const float (&a)[8]) {
        const int b = static_cast<int>(k & 1);
        float ov[16];
        if (wait(bar.o_full(b), static_cast<uint32_t>((k >> 1) & 1))) {
          tc_fence_after();
          tmem_ld16(tmem + lrow + 32 + 16 * b, ov);
          tc_fence_before();
        } else {
#pragma unroll
          for (int c = 0; c < 16; ++c) ov[c] = 0.f;
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(bar.o_free(b));
#pragma unroll
        for (int h = 0; h < 8; ++h) o_acc[h] = o_acc[h] * a[h] + (ov[h] + ov[8 + h]);
      };

      int64_t last_own = -1;
      for (int64_t k = n0 + ((n0 & 1) != w ? 1 : 0); k < n_end; k += 2) {
        const int b = w;  // k % 2
        float sv[16];
        if (wait(bar.s_full(b), static_cast<uint32_t>((k >> 1) & 1))) {
          tc_fence_after();
          tmem_ld16(tmem + lrow + 16 * b, sv);
          tc_fence_before();
        } else {
#pragma unroll
          for (int c = 0; c < 16; ++c) sv[c] = 0.f;
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(bar.s_free(b));
        // boxes with an out-of-range page id: the producer wrote the mask before the fill's
        // arrive; this wait on the fill (already complete, since the S^T product read it) makes
        // the mask visible. The slot cannot be refilled before this stage's P is written.
        uint32_t badm = 0;
        if (wait(bar.full(static_cast<int>(k % stages)), static_cast<uint32_t>((k / stages) & 1)))
          badm = s_badbox[k % stages];
        const int64_t t = x.tok0 + (k - n0) * kTcTok + i;
        const bool valid = t < x.tok1 && !((badm >> (i / C)) & 1u);
        if (!valid) {
          // this token's V row may hold anything (even NaN codes): zero it, so 0 * v stays 0
          uint4* vrow = reinterpret_cast<uint4*>(ring + static_cast<size_t>(k % stages) * kTcStage + kTcHalf + i * 128);
#pragma unroll
          for (int c = 0; c < 8; ++c) vrow[c] = make_uint4(0u, 0u, 0u, 0u);
        }
        float sc[8], mx[8], a[8], pv[8];
#pragma unroll
        for (int h = 0; h < 8; ++h) sc[h] = valid ? (sv[h] + sv[8 + h]) * score_scale : -INFINITY;
        wg_reduce8<true>(sc, mx, s_red[w][(k >> 1) & 1], wq, lane, wbar);
#pragma unroll
        for (int h = 0; h < 8; ++h) {
          const float mn = fmaxf(m_run[h], mx[h]);
          const float mr = mn == -INFINITY ? 0.f : mn;  // no live token yet (bad pages): adds nothing
          a[h] = exp2f(m_run[h] - mr);
          pv[h] = exp2f(sc[h] - mr + 8.f);
          l_part[h] = l_part[h] * a[h] + pv[h];
          m_run[h] = mn;
        }
        uint2 hi, lo;
        split_e4m3x8(pv, hi, lo);
        // P buffer b was last read by the O^T product of this warpgroup's previous stage, which
        // the issuing lane may start after this stage's S^T product: fold that stage first (its
        // wait covers the product's completion), then overwrite the buffer
        if (last_own >= 0) fold(last_own, a_prev);
        *reinterpret_cast<uint4*>(pt + b * kTcP + i * 16) = make_uint4(hi.x, hi.y, lo.x, lo.y);
        fence_proxy_async_shared();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar.p_full(b));
        if (w == 0 && have_next && k + 2 >= n_end) {
          build_q(y, j + 1);
          built_next = true;
        }
#pragma unroll
        for (int h = 0; h < 8; ++h) a_prev[h] = a[h];
        last_own = k;
      }
      if (w == 0 && have_next && !built_next) build_q(y, j + 1);  // no stage of this item here
      if (last_own >= 0) fold(last_own, a_prev);
      n = n_end;

      // ---- item end: l over each warpgroup's 128 token rows, then the two states combined
      float L[8];
      wg_reduce8<false>(l_part, L, s_red2[w], wq, lane, wbar);
      if (w == 1) {
#pragma unroll
        for (int h = 0; h < 8; ++h) xo[i * 8 + h] = o_acc[h];
        if (i == 0) {
#pragma unroll
          for (int h = 0; h < 8; ++h) {
            s_xm[h] = m_run[h];
            s_xl[h] = L[h];
          }
        }
      }
      named_barrier_sync(3, 2 * kSoftmax);
      if (w == 0) {
        const float vs = p.v_scale[kvh];
#pragma unroll
        for (int h = 0; h < 8; ++h) {
          if (h >= p.group) break;
          // a warpgroup without stages in this item has m = -inf and weighs 0
          const float m1 = s_xm[h], M = fmaxf(m_run[h], m1);
          const float Mr = M == -INFINITY ? 0.f : M;  // neither warpgroup saw a live token
          const float f0 = exp2f(m_run[h] - Mr), f1 = exp2f(m1 - Mr);
          const float Lh = L[h] * f0 + s_xl[h] * f1;
          const float oh = o_acc[h] * f0 + xo[i * 8 + h] * f1;
          if (x.direct) {
            const float val = Lh > 0.f ? oh * vs / Lh : 0.f;
            const int64_t oi = (static_cast<int64_t>(x.req) * p.num_heads + head0 + h) * kTcD + i;
            if (p.out_bf16) reinterpret_cast<__nv_bfloat16*>(p.out)[oi] = __float2bfloat16_rn(val);
            else reinterpret_cast<float*>(p.out)[oi] = val;
            if (p.lse && i == 0)  // natural-log units; l carries 2^8
              p.lse[static_cast<int64_t>(x.req) * p.num_heads + head0 + h] =
                  Lh > 0.f ? M * kLn2 + logf(Lh * (1.f / 256.f)) : -INFINITY;
          } else {
            // partial state in natural-log units, without the 2^8 that p carries
            const int64_t pi = x.slot * p.group + h;
            p.partial_o[pi * kTcD + i] = oh * vs * (1.f / 256.f);
            if (i == 0) {
              p.partial_ml[2 * pi] = M * kLn2;
              p.partial_ml[2 * pi + 1] = Lh * (1.f / 256.f);
            }
          }
        }
        if constexpr (FUSED) {
          if (!x.direct) {
            // the CTA that completes the last piece of this (request, kv head) merges it
            __threadfence();
            named_barrier_sync(1, kSoftmax);
            if (i == 0) {
              int64_t g1, g2, first_slot;
              segment_ctas(x, p.item_cost, chunk, g1, g2, first_slot);
              const int64_t pieces = g2 - g1 + 1;
              int32_t* ticket = p.tickets + static_cast<int64_t>(x.req) * p.kv_heads + kvh;
              const int old = atomicAdd(ticket, 1);
              const int last = old == pieces - 1;
              if (last) {
                __threadfence();
                *ticket = 0;  // ready for the next step
              }
              s_flag = last;
            }
            named_barrier_sync(1, kSoftmax);
            if (s_flag) merge_segment<kTcD>(p, x, chunk, i, kSoftmax, mrg, kTcMerge);
          }
        }
      }
      named_barrier_sync(3, 2 * kSoftmax);  // the exchange, merge and scratch buffers are reused
      ++j;
      have = cursor.next(p, x);
    }
    if constexpr (FUSED) {
      // s_walk still holds this CTA's unit run and the chunk from plan_in_kernel
      if (p.record && w == 0 && i == 0) record_header(p, s_walk[0], s_walk[1], s_walk[7], s_rec_n);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_free(tmem, kTmemCols);
  }
}

int tc_stages(int ctas_per_sm, int* smem_bytes) {
  // ring, Qhl[2], Phl[2], merge buffer, barriers; 1 KB alignment slack; static shared memory
  const int budget = kSmemLimit / (ctas_per_sm < 1 ? 1 : ctas_per_sm) - 2048;
  auto need = [](int st) {
    return st * kTcStage + 2 * kTcQ + 2 * kTcP + kTcMerge * 4 + (2 * st + TcBars::kExtra) * 8 + 1024;
  };
  int st = 8;
  while (st > 2 && need(st) > budget) --st;
  if (need(st) > budget) return 0;
  *smem_bytes = need(st);
  return st;
}

}  // namespace

bool tc_supported(int head_dim, bool fp8, int group, int q_len, bool pro) {
  return fp8 && head_dim == kTcD && group >= 1 && group <= 8 && q_len == 1 && !pro;
}

int tc_threads() { return kTcThreads; }

int tc_smem_bytes(int ctas_per_sm) {
  int smem = 0;
  return tc_stages(ctas_per_sm, &smem) ? smem : 0;
}

int launch_attention_tc(bool fused, const CUtensorMap& mk, const CUtensorMap& mv, const AttnParams& prm, int grid,
                        cudaStream_t stream) {
  int smem = 0;
  const int sms = device_sm_count();
  int ctas_per_sm = (sms > 0) ? (grid + sms - 1) / sms : 1;
  if (ctas_per_sm < 1) ctas_per_sm = 1;
  const int st = tc_stages(ctas_per_sm, &smem);
  if (!st) return fail(HPC_ERR_SHAPE, "tensor-core E4M3 attention does not fit shared memory");
  if (prm.chunk_tokens < 16 || kTcTok % prm.chunk_tokens) return fail(HPC_ERR_SHAPE, "box of %d tokens", prm.chunk_tokens);
  AttnParams p = prm;
  p.stages = st;
  auto kern = fused ? decode_attention_tc_kernel<true> : decode_attention_tc_kernel<false>;
  static int configured[2][64] = {{0}};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && configured[fused][dev] < smem) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
      return check_launch("cudaFuncSetAttribute(decode_attention_tc_kernel)");
    configured[fused][dev] = smem;
  }
  const cudaError_t e = launch_pdl(kern, dim3(grid), dim3(kTcThreads), static_cast<size_t>(smem), stream, mk, mv, p);
  if (e != cudaSuccess) return fail(HPC_ERR_CUDA, "decode_attention_tc_kernel: %s", cudaGetErrorString(e));
  return check_launch("decode_attention_tc_kernel");
}

}  // namespace attn
}  // namespace hpc
