// Several new tokens per request on the 5th-generation tensor cores (bf16 cache, head_dim 128).
//
// Same work as the single-launch step of attention.cu with q_len > 1: "腾讯混元三算子杀入 SGLang"
// (AREX), Dynamic Attention paragraph under "Router GEMM：精度不丢，速度翻三倍": a persistent kernel
// runs the tiles that the per-step plan assigns by actual KV length. Items that cover a whole
// (request, kv head) write the output; the others write partial softmax states, merged by the CTA
// that finishes a split (request, kv head) last.
//
// Why another consumer. With mma.sync each query token's warp re-reads the stage's K and V
// fragments from shared memory and runs its own products; four new tokens ran at about half the
// copy bandwidth, bound by per-warp latency. Here the q_len x group query rows of an item (at most
// 32) are the rows of one product per stage, in the orientation that keeps P out of shared memory
// (shared memory is better spent on K and V in flight):
//     S[64 rows x 128 tokens] = Q[64 x 128 d] . K^T        (tensor memory)
//     O[64 rows x 128 d]     += P[64 x 128 tokens] . V     (P read from tensor memory)
// M = 64 is the smallest product; rows 32..63 are padding that is computed and never read. An
// M = 64 accumulator takes the lower half of each 32-lane subpartition (row m at lane
// m % 16 + 32 (m / 16)); the upper halves hold a second one. Stages therefore go in pairs: the
// even stage of a pair in the lower halves, the odd one in the upper halves, both in the same
// columns. Query rows 0..15 live in subpartition 0 and rows 16..31 in subpartition 1; each of
// the two is worked by two warps (warp % 4 is the subpartition a warp reaches), one per half of
// the 128 token columns, so a thread holds one (row, stage) with 64 scores and only the two
// warps' row maxima and sums are exchanged. P (a bf16 high part and residual, two bf16 per
// 32-bit column) is written over the stage's own S columns and is the A operand of the O product
// straight from tensor memory; V is an MN-major B operand read from its swizzled TMA tile.
// Shared memory then holds only Q and the K and V rings (three 32 KB slots each), the bytes a CTA
// keeps in flight. A new S is issued into a buffer only once the O products that read the P
// there have completed: the tensor pipe does not hold a later product's write to those columns
// behind an earlier product's read of them.
//
// The running maximum per (row, half) moves only when a stage's maximum exceeds it by more than
// 2^8 (log2 units); p = 2^(s - m) then stays below 256, and O in tensor memory is rescaled only on
// such a move. The two halves of an item keep separate running states, combined by log-sum-exp at
// the item end. The softmax reads a stage's scores twice, 32 columns at a time (the maximum, then
// p), and computes every exponential and then selects: a branch per token cost several times the
// whole pass.
//
// Roles (224 threads): warps 0, 1, 4, 5 softmax (and Q tiles, item ends, merges); warp 2, one lane
// issues the products in a non-blocking loop; warps 3 and 6 the TMA producers of K and of V. Every
// wait is bounded (2 s) and ends in HPC_DEV_TIMEOUT; tensor memory is freed on every path.
#include "attention_common.cuh"

namespace hpc {
namespace attn {
namespace {

constexpr int kTmThreads = 224;
constexpr int kTmTok = 128;               // tokens per stage: N of the S product, K of the O product
constexpr int kTmD = 128;                 // head_dim
constexpr int kTmN = 32;                  // query rows read back (q_len x group <= 32)
constexpr int kTmPlane = kTmTok * 128;    // one 64-element plane of a stage's K or V: 16 KB
constexpr int kTmKV = 2 * kTmPlane;       // K (or V) of a stage: 32 KB
constexpr int kTmKS = 3, kTmVS = 3;       // ring slots of K and of V
constexpr int kTmQPlane = kTmN * 128;     // one plane of the Q tile: 4 KB
constexpr int kTmQ = 2 * kTmQPlane;       // Q tile: 8 KB
constexpr uint32_t kTmCols = 512;         // S[2] at 0 and 128 (P over S), O at 256
constexpr int kTmSB = 2;                  // S buffers: pair p uses buffer p % 2
constexpr int kTmSoftThreads = 128;       // warps 0, 1, 4, 5
constexpr int kTmMmaWarp = 2, kTmProducerK = 3, kTmProducerV = 6;
constexpr float kTmMove = 8.f;            // the running maximum moves when exceeded by more (log2 units)
// instruction descriptors: fp32 accumulate, bf16 x bf16, M = 64, N = 128; the O product reads V
// (its B) MN-major
constexpr uint32_t kTmIdS = (1u << 4) | (1u << 7) | (1u << 10) | ((128u >> 3) << 17) | ((64u >> 4) << 24);
constexpr uint32_t kTmIdO = kTmIdS | (1u << 16);

// D (tensor memory, fp32) = A * B (+ D), A and B bf16 in shared memory. Issued by one thread.
__device__ __forceinline__ void umma_bf16(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate));
}

// D (tensor memory, fp32) = A * B (+ D), A bf16 in tensor memory, B bf16 in shared memory.
__device__ __forceinline__ void umma_bf16_ts(uint32_t tmem_d, uint32_t tmem_a, uint64_t bdesc, uint32_t idesc,
                                             uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(tmem_d),
      "r"(tmem_a), "l"(bdesc), "r"(idesc), "r"(accumulate));
}

// Whole warp: 32 consecutive 32-bit columns of the warp's 32 lanes (lane = thread). Waits for the load.
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

// Whole warp: store 16 consecutive 32-bit columns of the warp's 32 lanes (not waited for).
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(
          taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]),
      "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}

__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

struct TmBars {
  uint32_t base;
  __device__ uint32_t at(int k) const { return base + 8 * k; }
  __device__ uint32_t k_full(int s) const { return at(s); }
  __device__ uint32_t k_empty(int s) const { return at(kTmKS + s); }
  __device__ uint32_t v_full(int s) const { return at(2 * kTmKS + s); }
  __device__ uint32_t v_empty(int s) const { return at(2 * kTmKS + kTmVS + s); }
  static constexpr int kRing = 2 * kTmKS + 2 * kTmVS;
  __device__ uint32_t s_full(int b) const { return at(kRing + b); }      // S of a pair (commit)
  __device__ uint32_t p_full(int b) const { return at(kRing + 2 + b); }  // P of a pair (2 warps)
  __device__ uint32_t o_done(int h) const { return at(kRing + 4 + h); }  // an O product of half h (commit)
  __device__ uint32_t q_full(int b) const { return at(kRing + 6 + b); }
  __device__ uint32_t q_free(int b) const { return at(kRing + 8 + b); }
  __device__ uint32_t done() const { return at(kRing + 10); }
  __device__ uint32_t buf_free(int b) const { return at(kRing + 11 + b); }  // O products of a pair done (commit)
  static constexpr int kCount = kRing + 11 + kTmSB;
};

// Dynamic shared memory (1024-byte aligned): Q[2], K ring, V ring, barriers. Q comes first: the
// M = 64 product reads 64 rows of a 32-row Q tile, and rows 32..63 fall on the next 4 KB (the
// other Q buffer or the K ring). Their products land in accumulator rows that are never read.
constexpr int kTmOffK = 2 * kTmQ;
constexpr int kTmOffV = kTmOffK + kTmKS * kTmKV;
constexpr int kTmOffBar = kTmOffV + kTmVS * kTmKV;
constexpr int kTmSmem = kTmOffBar + TmBars::kCount * 8 + 1024;  // + alignment slack
static_assert(kTmVS >= 2, "the softmax's wait on a V fill needs the slot's previous fill landed");

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
  __shared__ int32_t s_pages[2][32];
  __shared__ __align__(16) float s_merge[1024];
  __shared__ float s_px[2][2][2][32];  // softmax: [pair parity][subpartition][column half][lane] partial maxima
  __shared__ float s_pl[2][2][32];     // softmax, item end: [subpartition][column half][lane] partial sums
  __shared__ uint32_t s_tmem;
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* qt = smem;
  uint8_t* kring = smem + kTmOffK;
  uint8_t* vring = smem + kTmOffV;
  const TmBars bar{smem_u32(smem + kTmOffBar)};
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int q_len = p.q_len, group = p.group, rows = q_len * group;  // rows <= kTmN (checked on the host)
#ifdef HPC_TRACE
  uint64_t* trace = p.trace ? p.trace + static_cast<size_t>(blockIdx.x) * HPC_TRACE_WORDS : nullptr;
  if (trace && threadIdx.x == 0) {
    trace[0] = global_timer_ns();
    uint32_t smid;
    asm volatile("mov.u32 %0, %%smid;" : "=r"(smid));
    trace[7] = smid;
    trace[2] = trace[3] = 0;
  }
#endif

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
    for (int b = 0; b < kTmSB; ++b) mbar_init(bar.buf_free(b), 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar.s_full(b), 1);
      mbar_init(bar.p_full(b), 4);
      mbar_init(bar.o_done(b), 1);
      mbar_init(bar.q_full(b), 4);
      mbar_init(bar.q_free(b), 1);
    }
    mbar_init(bar.done(), 1);
    fence_barrier_init();
  }
  if (warp == kTmMmaWarp) tmem_alloc(smem_u32(&s_tmem), kTmCols);
  if (warp == kTmProducerK && lane == 0) {
    prefetch_tensormap(&tm_k);
    prefetch_tensormap(&tm_v);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s_tmem;
  // the plan reads seq_lens alone: before the wait on the previous kernel when that kernel does
  // not write them (plan_early), after it otherwise
  if (!p.plan_early) {
    pdl_wait();
    pdl_launch_dependents();
  }

  WalkCursor cursor;
  int64_t chunk = 0;
  // the per-request tile prefix lives in the K ring until the first TMA copy is issued
  plan_in_kernel<kTmD>(p, reinterpret_cast<int64_t*>(kring), s_scan, s_walk, cursor, chunk);
  if (p.plan_early) {
    pdl_wait();
    pdl_launch_dependents();
  }
#ifdef HPC_TRACE
  if (trace && threadIdx.x == 0) trace[1] = global_timer_ns();
#endif
  const int C = p.chunk_tokens;
  const int P = p.page_size;
  const int p_shift = __ffs(P) - 1;
  const int cps = kTmTok / C;  // boxes per stage
  const int c_shift = __ffs(C) - 1;

  if (warp == kTmProducerK || warp == kTmProducerV) {
    // ------------------------------------------------------------------ producers
    // Warp 3 fills the K ring and warp 4 the V ring, each on its own, so that a K fill never waits
    // behind a V slot (a V slot is held until its stage's O product, after the softmax).
    const int half = warp == kTmProducerV ? 1 : 0;  // 0: K, 1: V
    const int depth = half ? kTmVS : kTmKS;
    const CUtensorMap* tmap = half ? &tm_v : &tm_k;
    uint8_t* ring = half ? vring : kring;
    int32_t* pages = s_pages[half];
    const uint64_t policy = l2_policy_evict_first();
    int64_t n = 0;  // stages begun
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
        if (lane < nk) pages[lane] = cb + lane < nreal ? bt[(off0 + (cb + lane) * C) >> p_shift] : 0;
        __syncwarp();
        if (lane == 0) {
          // the stage's boxes lie in this batch of page ids (cps divides 32)
          for (int k = 0; k < nk && ok; k += cps, ++n) {
            const int64_t bi = cb + k;
            const int nb = static_cast<int>(nreal - bi < cps ? nreal - bi : cps);
            const uint32_t tx = static_cast<uint32_t>(nb) * 2u * C * 128u;
            const int slot = static_cast<int>(n % depth);
            const uint32_t empty = half ? bar.v_empty(slot) : bar.k_empty(slot);
            const uint32_t full = half ? bar.v_full(slot) : bar.k_full(slot);
            if (!mbar_wait(empty, static_cast<uint32_t>(((n / depth) & 1) ^ 1))) {
              ok = false;
              bad |= HPC_DEV_TIMEOUT;
              break;
            }
            mbar_arrive_expect_tx(full, tx);
            const uint32_t base = smem_u32(ring) + slot * kTmKV;
            for (int kk = 0; kk < nb; ++kk) {
              int32_t page = pages[k + kk];
              if (page < 0 || page >= p.num_pages) {
                page = 0;  // stand-in; the softmax leaves its tokens out
                if (!half) bad |= HPC_DEV_BAD_PAGE;
              }
              const int off = static_cast<int>((off0 + (bi + kk) * C) & (P - 1));
              const int c1 = p.nhd ? x.kvh : off, c2 = p.nhd ? off : x.kvh;
              const uint32_t dst = base + kk * C * 128;
              tma_load_4d(dst, tmap, full, 0, c1, c2, page, policy);
              tma_load_4d(dst + kTmPlane, tmap, full, 64, c1, c2, page, policy);
            }
          }
        }
        ok = __shfl_sync(0xffffffffu, ok, 0);
        n = __shfl_sync(0xffffffffu, n, 0);
      }
    }
    // Drain: every fill must have landed before the CTA exits. Fill f went to slot f % depth and
    // completes that slot's full-barrier phase f / depth.
    if (lane == 0) {
      for (int64_t f = n > depth ? n - depth : 0; f < n; ++f) {
        const int sl = static_cast<int>(f % depth);
        if (!mbar_wait(half ? bar.v_full(sl) : bar.k_full(sl), static_cast<uint32_t>((f / depth) & 1)))
          bad |= HPC_DEV_TIMEOUT;
      }
      if (bad) atomicOr(p.status, bad);
#ifdef HPC_TRACE
      if (trace && !half) {  // the K producer: its end and the 128-token stages it filled
        trace[4] = global_timer_ns();
        trace[6] = static_cast<uint64_t>(n);
      }
#endif
    }
  } else if (warp == kTmMmaWarp) {
    // ------------------------------------------------------------------ products
    // One lane issues both streams in a non-blocking loop. Stage i of an item is half i % 2 of pair
    // i / 2; pairs are counted over the CTA's items and use S buffer pair % 2.
    //  * S of a stage: when its K tile has landed, the item's Q tile is ready and every O product
    //    of the pair that last used its S buffer has completed (a new S must not overwrite a P that
    //    an O product still reads). The commit after the pair's
    //    last S releases the softmax; each S releases its K slot.
    //  * O of a stage: when its pair's P is written and its V tile has landed. Each O commit
    //    releases the V slot and signals its half.
    if (lane == 0) {
      WalkCursor qc = cursor, vc = cursor;
      ItemInfo xq, xv;
      bool have_q = qc.next(p, xq), have_v = vc.next(p, xv);
      int64_t nst_q = have_q ? tm_stages(xq) : 0, nst_v = have_v ? tm_stages(xv) : 0;
      int64_t iq = 0, iv = 0;      // stage index inside the current S item / O item
      int64_t pq0 = 0, pv0 = 0;    // pairs before the current S item / O item
      int64_t pairs_o = 0;         // pairs whose O products are all issued
      int64_t nq = 0, npv = 0;     // stages with S / O issued
      int jq = 0;
      bool q_ready = false;
      uint32_t bad = 0;
      uint64_t t_last = global_timer_ns();
      while (true) {
        bool progress = false;
        while (have_q && nst_q == 0) {  // items without tokens (cannot occur for a valid plan)
          umma_commit(bar.q_free(jq & 1));
          have_q = qc.next(p, xq);
          nst_q = have_q ? tm_stages(xq) : 0;
          ++jq;
        }
        while (have_v && nst_v == 0) {
          have_v = vc.next(p, xv);
          nst_v = have_v ? tm_stages(xv) : 0;
        }
        if (have_q) {
          if (!q_ready) q_ready = mbar_test(bar.q_full(jq & 1), static_cast<uint32_t>((jq >> 1) & 1));
          const int64_t pair = pq0 + (iq >> 1);
          const int ks = static_cast<int>(nq % kTmKS);
          if (q_ready && pair < pairs_o + 2 &&
              (pair < kTmSB || mbar_test(bar.buf_free(static_cast<int>(pair % kTmSB)),
                                         static_cast<uint32_t>((pair / kTmSB - 1) & 1))) &&
              mbar_test(bar.k_full(ks), static_cast<uint32_t>((nq / kTmKS) & 1))) {
            tc_fence_after();
            const int half = static_cast<int>(iq & 1);
            const uint32_t d = tmem + (static_cast<uint32_t>(16 * half) << 16) + 128u * static_cast<uint32_t>(pair & 1);
            const uint32_t kbase = smem_u32(kring) + ks * kTmKV;
            const uint32_t qbase = smem_u32(qt) + (jq & 1) * kTmQ;
#pragma unroll
            for (int kk = 0; kk < kTmD / 16; ++kk) {
              const int pl = kk >> 2, sub = kk & 3;
              umma_bf16(d, umma_desc(qbase + pl * kTmQPlane + 32 * sub, 16, 1024, 2),
                        umma_desc(kbase + pl * kTmPlane + 32 * sub, 16, 1024, 2), kTmIdS, kk > 0);
            }
            umma_commit(bar.k_empty(ks));  // the stage's K is no longer read
            if (half == 1 || iq + 1 == nst_q) umma_commit(bar.s_full(static_cast<int>(pair & 1)));
            ++nq;
            if (++iq == nst_q) {
              umma_commit(bar.q_free(jq & 1));  // the item's last read of its Q tile
              pq0 += (nst_q + 1) >> 1;
              have_q = qc.next(p, xq);
              nst_q = have_q ? tm_stages(xq) : 0;
              iq = 0;
              ++jq;
              q_ready = false;
            }
            progress = true;
          }
        }
        if (have_v && npv < nq) {
          const int64_t pair = pv0 + (iv >> 1);
          const int vs = static_cast<int>(npv % kTmVS);
          if (mbar_test(bar.p_full(static_cast<int>(pair & 1)), static_cast<uint32_t>((pair >> 1) & 1)) &&
              mbar_test(bar.v_full(vs), static_cast<uint32_t>((npv / kTmVS) & 1))) {
            tc_fence_after();
            const int half = static_cast<int>(iv & 1);
            const uint32_t lo = static_cast<uint32_t>(16 * half) << 16;
            const uint32_t pa = tmem + lo + 128u * static_cast<uint32_t>(pair & 1);
            const uint32_t od = tmem + lo + 256u;
            const uint32_t vbase = smem_u32(vring) + vs * kTmKV;
#pragma unroll
            for (int kk = 0; kk < kTmTok / 16; ++kk)  // 16 tokens per product: high part of P
              umma_bf16_ts(od, pa + 32 * (kk >> 1) + 8 * (kk & 1), umma_desc(vbase + 2048 * kk, kTmPlane, 1024, 2),
                           kTmIdO, (iv >= 2 || kk > 0) ? 1u : 0u);
#pragma unroll
            for (int kk = 0; kk < kTmTok / 16; ++kk)  // residual of P
              umma_bf16_ts(od, pa + 32 * (kk >> 1) + 16 + 8 * (kk & 1), umma_desc(vbase + 2048 * kk, kTmPlane, 1024, 2),
                           kTmIdO, 1u);
            umma_commit(bar.o_done(half));
            umma_commit(bar.v_empty(vs));  // the stage's V is no longer read
            ++npv;
            if (half == 1 || iv + 1 == nst_v) {
              // the pair's P has been read once these products complete: its S buffer is free
              umma_commit(bar.buf_free(static_cast<int>(pair % kTmSB)));
              ++pairs_o;
            }
            if (++iv == nst_v) {
              pv0 += (nst_v + 1) >> 1;
              have_v = vc.next(p, xv);
              nst_v = have_v ? tm_stages(xv) : 0;
              iv = 0;
            }
            progress = true;
          }
        } else if (!have_q && !have_v) {
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
    // ------------------------------------------------------------------ softmax (warps 0, 1, 4, 5)
    // Warp w works on subpartition sp = w % 4 and on column half hb = w / 4 of every stage (tokens
    // 64 hb .. 64 hb + 63, and the same d columns of O). Thread (w, lane l) owns query row
    // r = 16 sp + l % 16 of the stages of half h = l / 16: tensor-memory lane 32 sp + l. The two
    // warps of a subpartition exchange their row maxima once per pair (shared memory and a named
    // barrier of 64 threads) and their row sums at the item end. Control flow is uniform within
    // each warp; per-lane waits (a half's O product) are bounded and do not diverge the collective
    // calls.
    const int sp = warp & 3, hb = warp >> 2, h = lane >> 4;
    const int r = 16 * sp + (lane & 15);
    const int tid = 64 * hb + 32 * sp + lane;  // 0 .. 127
    const int pbar = 2 + sp;                   // named barrier of the subpartition's two warps
    const bool row_live = r < rows;
    const int tq = r / group, hd = r - tq * group;
    const uint32_t tl = tmem + (static_cast<uint32_t>(32 * sp) << 16);  // this warp's lanes
    zero_empty_requests<kTmD>(p, tid, kTmSoftThreads);
    bool ok = true;
    auto fail_wait = [&]() {
      if (ok) {
        ok = false;
        atomicOr(p.status, HPC_DEV_TIMEOUT);
      }
    };
    auto wait_warp = [&](uint32_t b, uint32_t par) -> bool {  // whole warp, same barrier
      const bool got = __all_sync(0xffffffffu, ok && mbar_wait(b, par));
      if (!got && ok) {
        ok = false;
        if (lane == 0) atomicOr(p.status, HPC_DEV_TIMEOUT);
      }
      ok = __all_sync(0xffffffffu, ok);
      return got;
    };
    // Q tile of item y into buffer jy % 2 (the four softmax warps). Row c = t * group + g holds
    // query token t of head kv_head * group + g; rows past q_len * group are zero. Thread tid
    // writes 16-byte chunks tid, tid + 128, tid + 256, tid + 384 of the 32 x 256-byte tile.
    auto build_q = [&](const ItemInfo& y, int jy) {
      const int qb = jy & 1;
      if (jy >= 2) wait_warp(bar.q_free(qb), static_cast<uint32_t>(((jy >> 1) - 1) & 1));
      uint8_t* qtile = qt + qb * kTmQ;
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int qi = tid + kTmSoftThreads * k, c = qi >> 4, cc = qi & 15;
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        if (c < rows) {
          const int t = c / group, g = c - t * group;
          v = *reinterpret_cast<const uint4*>(
              p.q + ((static_cast<int64_t>(y.req) * q_len + t) * p.num_heads + y.kvh * group + g) * kTmD + cc * 8);
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
    if (have) build_q(x, 0);
    int j = 0;            // items
    int64_t n = 0;        // stages before the current item
    int64_t pair0 = 0;    // pairs before the current item
    int64_t pv_cnt = 0;   // O products of this thread's half so far (o_done phases)
    while (have) {
      if (tid == 0) {
        if (p.record) record_item(p, s_rec_n, x);
        ++s_rec_n;
      }
      if (cur.u < cur.u_end) {  // the next item's Q tile (its buffer was last read two items ago)
        WalkCursor a2 = cur;
        ItemInfo y;
        a2.next(p, y);
        build_q(y, j + 1);
      }
      const int64_t nst = tm_stages(x);
      const int64_t npairs = (nst + 1) >> 1;
      const int64_t L = p.seq_lens[x.req];
      // tokens this row may see: before the item's end and up to its own query position
      const int64_t last_vis = L - q_len + tq + 1;
      const int64_t lim = row_live ? (last_vis < x.tok1 ? last_vis : x.tok1) : x.tok0;
      float m_used = -INFINITY, l_sum = 0.f;
      bool had = false;  // this half had a stage in this item
      for (int64_t pi = 0; pi < npairs; ++pi) {
        const int64_t gp = pair0 + pi;
        const int buf = static_cast<int>(gp & 1);
        const int64_t i = 2 * pi + h;  // stage index in the item
        const bool has = i < nst;
        const int64_t k = n + i;
        const int64_t t0 = x.tok0 + i * kTmTok;
        // live tokens of this (row, stage): [0, cb), minus boxes on pages outside the pool
        int cb = 0;
        uint32_t badm = 0;
        bool dead_any = false;  // some token of this stage is dead for every row (its V row is zeroed)
        if (has) {
          const int64_t e = lim - t0;
          cb = e <= 0 ? 0 : (e >= kTmTok ? kTmTok : static_cast<int>(e));
          const int32_t* btr = p.block_table + static_cast<int64_t>(x.req) * p.max_pages;
          for (int b = 0; b < cps; ++b) {
            const int64_t tb = t0 + static_cast<int64_t>(b) * C;
            if (tb < x.tok1) {
              const int32_t pg = btr[tb >> p_shift];
              if (pg < 0 || pg >= p.num_pages) badm |= 1u << b;
            }
          }
          dead_any = badm != 0 || t0 + kTmTok > x.tok1;
        }
        // live tokens of 32-token chunk c4 as a bit mask
        auto chunk_live = [&](int c4) -> uint32_t {
          const int in = cb - 32 * c4;
          uint32_t m = in <= 0 ? 0u : (in >= 32 ? 0xffffffffu : ((1u << in) - 1u));
          if (badm) {
            for (int b = 0; b < cps; ++b) {
              const int lo = max(b * C - 32 * c4, 0), hi = min((b + 1) * C - 32 * c4, 32);
              if (((badm >> b) & 1u) && lo < hi) m &= ~((hi - lo >= 32 ? 0xffffffffu : ((1u << (hi - lo)) - 1u)) << lo);
            }
          }
          return m;
        };
        wait_warp(bar.s_full(buf), static_cast<uint32_t>((gp >> 1) & 1));
        tc_fence_after();
#ifdef HPC_TRACE
        if (trace && tid == 0 && trace[2] == 0) trace[2] = global_timer_ns();
#endif
        // two passes over this warp's 64 scores of the stage (32 at a time): the maximum (combined
        // with the other column half's through shared memory), then p
        float mx = -INFINITY;
#pragma unroll 1
        for (int c4 = 2 * hb; c4 < 2 * hb + 2; ++c4) {
          const uint32_t lv = chunk_live(c4);
          float v[32];
          tmem_ld32(tl + 128u * buf + 32 * c4, v);
#pragma unroll
          for (int c = 0; c < 32; ++c) mx = fmaxf(mx, ((lv >> c) & 1u) ? v[c] * p.score_scale : -INFINITY);
        }
        s_px[gp & 1][sp][hb][lane] = mx;
        named_barrier_sync(pbar, 64);
        mx = fmaxf(mx, s_px[gp & 1][sp][hb ^ 1][lane]);
        // the running maximum: set by the first stage of the half, or by a live stage before which
        // the half saw no live token (its O holds zeros); afterwards moved only past the margin,
        // with O and the sum rescaled
        bool rescale = false;
        float a = 1.f;
        if (has && mx != -INFINITY) {
          if (i < 2 || m_used == -INFINITY) {
            m_used = mx;
          } else if (mx > m_used + kTmMove) {
            a = exp2f(m_used - mx);
            m_used = mx;
            l_sum *= a;
            rescale = true;
          }
        }
        // p = 2^(s - m), written over S: for tokens 32 c .. 32 c + 31 (columns 32 c .. 32 c + 31 of S)
        // a bf16 high part in columns 32 c .. 32 c + 15 and the residual in the next 16, two tokens
        // per column, the even token in the low half
        const float mr = m_used == -INFINITY ? 0.f : m_used;
        float add = 0.f;
#pragma unroll 1
        for (int c4 = 2 * hb; c4 < 2 * hb + 2; ++c4) {
          const uint32_t lv = chunk_live(c4);
          float v[32];
          tmem_ld32(tl + 128u * buf + 32 * c4, v);
          uint32_t hi[16], lo[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            // computed for every token, then selected: no branch (a dead token's score may be anything)
            const float e0 = exp2f(fmaf(v[2 * e], p.score_scale, -mr));
            const float e1 = exp2f(fmaf(v[2 * e + 1], p.score_scale, -mr));
            const float p0 = ((lv >> (2 * e)) & 1u) ? e0 : 0.f;
            const float p1 = ((lv >> (2 * e + 1)) & 1u) ? e1 : 0.f;
            add += p0 + p1;
            const uint32_t hh = pack_bf16x2(p0, p1);
            hi[e] = hh;
            lo[e] = pack_bf16x2(p0 - __uint_as_float(hh << 16), p1 - __uint_as_float(hh & 0xffff0000u));
          }
          // within the chunk's own 32 columns, all read above: high part, then residual
          tmem_st16(tl + 128u * buf + 32 * c4, hi);
          tmem_st16(tl + 128u * buf + 32 * c4 + 16, lo);
        }
        if (has) l_sum += add;
        if (__any_sync(0xffffffffu, rescale)) {
          // O rescaled in tensor memory (after P, so that the scores are no longer held). The load and
          // store take the whole warp, both halves (the other lanes write back their values times 1),
          // so every lane first waits for its own half's previous O product.
          if (pv_cnt > 0 && !mbar_wait(bar.o_done(h), static_cast<uint32_t>((pv_cnt - 1) & 1))) fail_wait();
          ok = __all_sync(0xffffffffu, ok);
          tc_fence_after();
#pragma unroll
          for (int c4 = 2 * hb; c4 < 2 * hb + 2; ++c4) {  // this warp's 64 columns of O
            float v[32];
            tmem_ld32(tl + 256 + 32 * c4, v);
            uint32_t o0[16], o1[16];
#pragma unroll
            for (int c = 0; c < 16; ++c) {
              o0[c] = __float_as_uint(v[c] * a);
              o1[c] = __float_as_uint(v[16 + c] * a);
            }
            tmem_st16(tl + 256 + 32 * c4, o0);
            tmem_st16(tl + 256 + 32 * c4 + 16, o1);
          }
        }
        // tokens dead for every row (past the item, or on a page outside the pool): their V rows
        // may hold anything (even NaN) and are zeroed, so that 0 * v stays 0. The 64 threads of a
        // half take tokens q and q + 64 (q = 16 (2 hb + sp) + l % 16) of their stage.
        if (__any_sync(0xffffffffu, dead_any)) {
          // The wait on the stage's V fill is by phase parity, which is exact only once the slot's
          // previous fill (stage k - kTmVS) has landed. Nothing orders that before this point (the
          // S of this pair implies only the O products of pair gp - 2), so the O products of pair
          // gp - 1 are waited for first: they read every V fill through stage k - 2. Their commit
          // is buf_free, whose phase before (pair gp - 3) completed before this pair's S was written.
          if (dead_any && gp >= 1 &&
              !mbar_wait(bar.buf_free(static_cast<int>((gp - 1) % kTmSB)),
                         static_cast<uint32_t>(((gp - 1) / kTmSB) & 1)))
            fail_wait();
          if (dead_any && ok) {
            const int vs = static_cast<int>(k % kTmVS);
            if (mbar_wait(bar.v_full(vs), static_cast<uint32_t>((k / kTmVS) & 1))) {
              const int q0 = 16 * (2 * hb + sp) + (lane & 15);
#pragma unroll
              for (int u = 0; u < 2; ++u) {
                const int c = q0 + 64 * u;
                if (t0 + c >= x.tok1 || ((badm >> (c >> c_shift)) & 1u)) {
                  uint8_t* vrow = vring + vs * kTmKV + c * 128;
#pragma unroll
                  for (int z = 0; z < 8; ++z) {
                    reinterpret_cast<uint4*>(vrow)[z] = make_uint4(0u, 0u, 0u, 0u);
                    reinterpret_cast<uint4*>(vrow + kTmPlane)[z] = make_uint4(0u, 0u, 0u, 0u);
                  }
                }
              }
            } else {
              fail_wait();
            }
          }
          fence_proxy_async_shared();
          ok = __all_sync(0xffffffffu, ok);
        }
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar.p_full(buf));
        if (has) {
          ++pv_cnt;
          had = true;
        }
      }
      n += nst;
      pair0 += npairs;

      // ---- item end: the two halves combined by log-sum-exp (lanes l and l ^ 16 hold the same
      // row), once every O product of the item is complete. A row's sum is split over the two
      // column halves' warps.
      s_pl[sp][hb][lane] = l_sum;
      named_barrier_sync(pbar, 64);
      l_sum += s_pl[sp][hb ^ 1][lane];
      // The item's last pair gp = pair0 - 1: its buf_free commit follows every O product through
      // it. Its phase before, pair gp - 2, completed before the S of pair gp was written, so the
      // parity wait is exact. (A half's own o_done would not do: its phase before is the O
      // product of pair gp - 1, which nothing here orders.)
      if (npairs > 0 && !mbar_wait(bar.buf_free(static_cast<int>((pair0 - 1) % kTmSB)),
                                   static_cast<uint32_t>(((pair0 - 1) / kTmSB) & 1)))
        fail_wait();
      ok = __all_sync(0xffffffffu, ok);
      tc_fence_after();
      const float m_o = __shfl_xor_sync(0xffffffffu, m_used, 16);
      const float l_o = __shfl_xor_sync(0xffffffffu, l_sum, 16);
      const bool had_o = __shfl_xor_sync(0xffffffffu, had, 16);
      const float m_s = had ? m_used : -INFINITY, m_p = had_o ? m_o : -INFINITY;
      const float M = fmaxf(m_s, m_p);
      const float f_s = m_s == -INFINITY ? 0.f : exp2f(m_s - M), f_p = m_p == -INFINITY ? 0.f : exp2f(m_p - M);
      const float Lt = (had ? l_sum * f_s : 0.f) + (had_o ? l_o * f_p : 0.f);
      const int64_t head = static_cast<int64_t>(x.kvh) * group + hd;
#pragma unroll
      for (int c4 = 2 * hb; c4 < 2 * hb + 2; ++c4) {  // this warp's 64 columns of O
        float v[32];
        tmem_ld32(tl + 256 + 32 * c4, v);
        float mine[16];
#pragma unroll
        for (int c = 0; c < 16; ++c) {
          // this lane writes columns 16 h .. 16 h + 15 of the chunk; it sends the partner the others
          const float keep = h ? v[16 + c] : v[c], send = h ? v[c] : v[16 + c];
          const float got = __shfl_xor_sync(0xffffffffu, send, 16);
          mine[c] = (f_s > 0.f ? keep * f_s : 0.f) + (f_p > 0.f ? got * f_p : 0.f);
        }
        if (row_live) {
          const int d0 = 32 * c4 + 16 * h;
          if (x.direct) {
            const int64_t oi = ((static_cast<int64_t>(x.req) * q_len + tq) * p.num_heads + head) * kTmD + d0;
            if (p.out_bf16) {
              __nv_bfloat16* o = reinterpret_cast<__nv_bfloat16*>(p.out) + oi;
#pragma unroll
              for (int c = 0; c < 16; ++c) o[c] = __float2bfloat16_rn(Lt > 0.f ? mine[c] / Lt : 0.f);
            } else {
              float* o = reinterpret_cast<float*>(p.out) + oi;
#pragma unroll
              for (int c = 0; c < 16; c += 4)
                *reinterpret_cast<float4*>(o + c) =
                    Lt > 0.f ? make_float4(mine[c] / Lt, mine[c + 1] / Lt, mine[c + 2] / Lt, mine[c + 3] / Lt)
                             : make_float4(0.f, 0.f, 0.f, 0.f);
            }
          } else {
            const int64_t pi = (x.slot * q_len + tq) * group + hd;
            float* o = p.partial_o + pi * kTmD + d0;
#pragma unroll
            for (int c = 0; c < 16; c += 4)
              *reinterpret_cast<float4*>(o + c) = make_float4(mine[c], mine[c + 1], mine[c + 2], mine[c + 3]);
            if (h == 0 && c4 == 0) {
              p.partial_ml[2 * pi] = M * kLn2;  // natural-log units
              p.partial_ml[2 * pi + 1] = Lt;
            }
          }
        }
      }
      tc_fence_before();
      if (!x.direct) {
        // the CTA that completes the last piece of this (request, kv head) merges it
        __threadfence();
        named_barrier_sync(1, kTmSoftThreads);
        if (tid == 0) {
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
        named_barrier_sync(1, kTmSoftThreads);
        if (s_flag) merge_segment<kTmD>(p, x, chunk, tid, kTmSoftThreads, s_merge, 1024);
        named_barrier_sync(1, kTmSoftThreads);  // s_flag and s_merge are free again
      }
      ++j;
      have = cur.next(p, x);
    }
    if (p.record && tid == 0) record_header(p, s_walk[0], s_walk[1], s_walk[7], s_rec_n);
#ifdef HPC_TRACE
    if (trace && tid == 0) {
      if (s_rec_n > 0) trace[3] = global_timer_ns();
      trace[5] = static_cast<uint64_t>(s_rec_n);
    }
#endif
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
  if (prm.chunk_tokens < 16 || kTmTok % prm.chunk_tokens)
    return fail(HPC_ERR_SHAPE, "box of %d tokens", prm.chunk_tokens);
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
