// Persistent split-KV decode attention for sm_100a.
//
// "腾讯混元三算子杀入 SGLang" (AREX), Dynamic Attention paragraph under "Router GEMM：精度不丢，
// 速度翻三倍": a persistent kernel takes the tiles that the per-step plan assigns by actual KV
// length. Each CTA runs its items (request, kv head, tile range) back to back. An item
// that covers a whole (request, kv head) writes the final output. Any other item writes
// its partial softmax state (m, l, o) for the log-sum-exp merge.
//
// Design for B200. The kernel is bound by HBM bandwidth: 8 flop per byte of bf16 K+V,
// against a tensor-core ridge near 250 flop/B.
//  * Warp 8 is the producer. One lane streams each (page, kv head) block of K and V into
//    a ring of shared-memory stages with 4-D TMA tensor loads (SWIZZLE_128B). Each stage
//    completes on an mbarrier with the transferred byte count. Whole pages travel as a
//    few bulk copies, with an evict-first L2 policy: each byte is read once.
//  * Warps 0..7 are consumers, in groups that take whole stages round-robin. Inside a stage,
//    each warp takes two consecutive 16-token blocks, which gives two independent MMA chains.
//    Each warp keeps its own online-softmax state for the GQA group of the item's kv head.
//  * QK^T runs as S^T = K * Q^T on mma.m16n8k16: M = 16 tokens, N = 8 query heads, K = head
//    dim. PV runs as O^T = V^T * P^T: M = 16 head-dim rows, N = 8 heads, K = 16 tokens. Both
//    shapes fit the group without padding. The S^T accumulator becomes the P^T operand
//    through two movmatrix transposes. The 128-byte swizzle keeps ldmatrix free of bank
//    conflicts.
//  * With a bf16 cache, P goes into the PV product as a bf16 high part plus a bf16
//    residual: two products accumulated in fp32. "Tencent HPC llega a SGLang …" (remio.ai),
//    section "Dynamic Attention y Fused MoE atacan distintos cuellos de botella", describes
//    this split for an FP32 operand of the Router GEMM. Here it carries P at ~16 significant
//    bits for a few percent of tensor-pipe time.
//  * E4M3 cache: codes are widened to f16 in registers (cvt.f16x2.e4m3x2, exact). V needs
//    the k = token orientation: ldmatrix.trans moves byte pairs, and one byte permute per
//    register regroups them into token pairs before widening. k_scale folds into the score
//    scale, v_scale into the output.
//  * At the end of an item, the 8 consumer warps merge their states through shared memory.
//  * Every wait is bounded (2 s). On expiry the kernel sets HPC_DEV_TIMEOUT, stops waiting,
//    drains its outstanding copies (bounded too) and returns.
#include <math.h>

#include <mutex>

#include "attention_common.cuh"

namespace hpc {
namespace {

using namespace attn;

// Online-softmax update of one warp's state with NB consecutive 16-token blocks of a stage.
// K and V rows rb.. rb + 16*NB of the stage sit at kbase / vbase, in 128-byte swizzled
// planes. Tokens tb.. of the request; tokens >= tok1 are masked, and so is the whole stage when
// `bad` is set (its page id was out of range and page 0 stood in). The flag is applied with the
// tail mask, after the QK^T products, so its shared-memory load does not hold them up. The NB
// blocks give independent MMA chains, so the warp hides latency without more warps.
template <int D, bool FP8, int NB>
__device__ __forceinline__ void consume_blocks(uint32_t kbase, uint32_t vbase, uint32_t plane_bytes, int rb,
                                               int64_t tb, int64_t tok1, bool bad, const uint32_t (&qf)[D / 16][2],
                                               float score_scale, float& m0, float& m1, float& l0, float& l1,
                                               float (&o)[D / 16][4], int lane) {
  constexpr int KSTEPS = D / 16;
  const int g = lane >> 2, c = lane & 3;

  // ---- S^T = K * Q^T, one 16x8 tile per block
  float s[NB][4];
#pragma unroll
  for (int b = 0; b < NB; ++b) s[b][0] = s[b][1] = s[b][2] = s[b][3] = 0.f;
  {
    const int row0 = rb + (lane & 7) + ((lane >> 3) & 1) * 8;
    if (!FP8) {
#pragma unroll
      for (int ks = 0; ks < KSTEPS; ++ks) {
        const int chunk = 2 * ks + (lane >> 4);
#pragma unroll
        for (int b = 0; b < NB; ++b) {
          const int row = row0 + 16 * b;
          uint32_t a0, a1, a2, a3;
          ldsm_x4(kbase + (chunk >> 3) * plane_bytes + swz128(row, chunk & 7), a0, a1, a2, a3);
          mma_bf16_16816(s[b], a0, a1, a2, a3, qf[ks][0], qf[ks][1]);
        }
      }
    } else {
#pragma unroll
      for (int kp = 0; kp < KSTEPS / 2; ++kp) {
        const int chunk = 2 * kp + (lane >> 4);
#pragma unroll
        for (int b = 0; b < NB; ++b) {
          uint32_t x0, x1, x2, x3;  // rows 0-7 / 8-15 of chunk 2kp, then of chunk 2kp+1
          ldsm_x4(kbase + swz128(row0 + 16 * b, chunk), x0, x1, x2, x3);
          uint32_t f0l, f0h, f1l, f1h, f2l, f2h, f3l, f3h;
          e4m3x4_to_f16x4(x0, f0l, f0h);
          e4m3x4_to_f16x4(x1, f1l, f1h);
          e4m3x4_to_f16x4(x2, f2l, f2h);
          e4m3x4_to_f16x4(x3, f3l, f3h);
          mma_f16_16816(s[b], f0l, f1l, f0h, f1h, qf[2 * kp][0], qf[2 * kp][1]);
          mma_f16_16816(s[b], f2l, f3l, f2h, f3h, qf[2 * kp + 1][0], qf[2 * kp + 1][1]);
        }
      }
    }
  }

  // ---- online softmax (base 2) over these NB blocks, per head
  const bool tail = bad || tb + 16 * NB > tok1;
  const int64_t lim = bad ? tb : tok1;  // a masked stage: no token is live
#pragma unroll
  for (int b = 0; b < NB; ++b) {
#pragma unroll
    for (int i = 0; i < 4; ++i) s[b][i] *= score_scale;
    if (tail) {
      if (tb + 16 * b + g >= lim) s[b][0] = s[b][1] = -INFINITY;
      if (tb + 16 * b + g + 8 >= lim) s[b][2] = s[b][3] = -INFINITY;
    }
  }
  float mx0 = fmaxf(s[0][0], s[0][2]), mx1 = fmaxf(s[0][1], s[0][3]);
#pragma unroll
  for (int b = 1; b < NB; ++b) {
    mx0 = fmaxf(mx0, fmaxf(s[b][0], s[b][2]));
    mx1 = fmaxf(mx1, fmaxf(s[b][1], s[b][3]));
  }
#pragma unroll
  for (int off = 4; off < 32; off <<= 1) {
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, off));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, off));
  }
  const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);
  // -inf only when no token has been live yet (a masked stage): the reference 0 keeps every
  // exponential at 0 instead of NaN
  float mr0 = mn0, mr1 = mn1;
  if (tail) {  // only a tail call can have no live token at all
    if (mn0 == -INFINITY) mr0 = 0.f;
    if (mn1 == -INFINITY) mr1 = 0.f;
  }
  const float al0 = exp2f(m0 - mr0), al1 = exp2f(m1 - mr1);
  float pr[NB][4];
  float add0 = 0.f, add1 = 0.f;
#pragma unroll
  for (int b = 0; b < NB; ++b) {
    pr[b][0] = exp2f(s[b][0] - mr0);
    pr[b][1] = exp2f(s[b][1] - mr1);
    pr[b][2] = exp2f(s[b][2] - mr0);
    pr[b][3] = exp2f(s[b][3] - mr1);
    add0 += pr[b][0] + pr[b][2];
    add1 += pr[b][1] + pr[b][3];
  }
  l0 = l0 * al0 + add0;
  l1 = l1 * al1 + add1;
  m0 = mn0;
  m1 = mn1;
  // a factor of exactly 1 leaves O unchanged, so the rescale is skipped when no row max moved
  if (__any_sync(0xffffffffu, al0 != 1.f || al1 != 1.f)) {
#pragma unroll
    for (int i = 0; i < KSTEPS; ++i) {
      o[i][0] *= al0;
      o[i][1] *= al1;
      o[i][2] *= al0;
      o[i][3] *= al1;
    }
  }

  // ---- P^T operands: rows = tokens, cols = heads, transposed to (k = token, n = head).
  // bf16 keeps 8 significant bits, too few for P on short, peaked rows, so a bf16 cache
  // sends P as a bf16 high part plus a bf16 residual (two products summed in fp32). f16 P
  // (E4M3 cache) keeps 11 bits and goes as one product.
  uint32_t ph0[NB], ph1[NB], pl0[NB], pl1[NB];
#pragma unroll
  for (int b = 0; b < NB; ++b) {
    const uint32_t pa = FP8 ? pack_f16x2(pr[b][0], pr[b][1]) : pack_bf16x2(pr[b][0], pr[b][1]);
    const uint32_t pb = FP8 ? pack_f16x2(pr[b][2], pr[b][3]) : pack_bf16x2(pr[b][2], pr[b][3]);
    ph0[b] = movmatrix_trans(pa);
    ph1[b] = movmatrix_trans(pb);
    if (!FP8) {
      pl0[b] = movmatrix_trans(pack_bf16x2(pr[b][0] - __uint_as_float(pa << 16),
                                           pr[b][1] - __uint_as_float(pa & 0xffff0000u)));
      pl1[b] = movmatrix_trans(pack_bf16x2(pr[b][2] - __uint_as_float(pb << 16),
                                           pr[b][3] - __uint_as_float(pb & 0xffff0000u)));
    }
  }
  // V rows past the end may hold anything (even NaN): zero them so 0 * v stays 0.
  // The A-operand halves hold tokens (2c, 2c+1) and (8+2c, 9+2c) of each block.
  uint32_t mlo[NB], mhi[NB];
#pragma unroll
  for (int b = 0; b < NB; ++b) {
    mlo[b] = mhi[b] = 0xffffffffu;
    if (tail) {
      const int64_t t0 = tb + 16 * b;
      mlo[b] = (t0 + 2 * c < lim ? 0x0000ffffu : 0u) | (t0 + 2 * c + 1 < lim ? 0xffff0000u : 0u);
      mhi[b] = (t0 + 2 * c + 8 < lim ? 0x0000ffffu : 0u) | (t0 + 2 * c + 9 < lim ? 0xffff0000u : 0u);
    }
  }

  // ---- O^T += V^T * P^T
  if (!FP8) {
    const int row0 = rb + (lane & 7) + (lane >> 4) * 8;
#pragma unroll
    for (int mi = 0; mi < KSTEPS; ++mi) {
      const int chunk = 2 * mi + ((lane >> 3) & 1);
#pragma unroll
      for (int b = 0; b < NB; ++b) {
        const int row = row0 + 16 * b;
        uint32_t a0, a1, a2, a3;
        ldsm_x4_trans(vbase + (chunk >> 3) * plane_bytes + swz128(row, chunk & 7), a0, a1, a2, a3);
        if (tail) {
          a0 &= mlo[b];
          a1 &= mlo[b];
          a2 &= mhi[b];
          a3 &= mhi[b];
        }
        mma_bf16_16816(o[mi], a0, a1, a2, a3, ph0[b], ph1[b]);
        mma_bf16_16816(o[mi], a0, a1, a2, a3, pl0[b], pl1[b]);
      }
    }
  } else {
    // ldmatrix.trans on byte pairs: lane (g, c) receives bytes (d 2g, 2g+1) of tokens 2c and
    // 2c+1. One byte permute regroups them into the token pairs (2c, 2c+1) at d = 2g and at
    // d = 2g+1, which widen to the f16 A-operand halves of output rows 2g and 2g+1.
    const int row0 = rb + (lane & 7) + ((lane >> 3) & 1) * 8;
#pragma unroll
    for (int kp = 0; kp < KSTEPS / 2; ++kp) {
      const int chunk = 2 * kp + (lane >> 4);
#pragma unroll
      for (int b = 0; b < NB; ++b) {
        uint32_t x0, x1, x2, x3;  // tokens 0-7 / 8-15 of chunk 2kp, then of chunk 2kp+1
        ldsm_x4_trans(vbase + swz128(row0 + 16 * b, chunk), x0, x1, x2, x3);
        uint32_t a0, a1, a2, a3, c0, c1, c2, c3;
        e4m3x4_to_f16x4(__byte_perm(x0, 0, 0x3120), a0, a1);
        e4m3x4_to_f16x4(__byte_perm(x1, 0, 0x3120), a2, a3);
        e4m3x4_to_f16x4(__byte_perm(x2, 0, 0x3120), c0, c1);
        e4m3x4_to_f16x4(__byte_perm(x3, 0, 0x3120), c2, c3);
        if (tail) {
          a0 &= mlo[b];
          a1 &= mlo[b];
          a2 &= mhi[b];
          a3 &= mhi[b];
          c0 &= mlo[b];
          c1 &= mlo[b];
          c2 &= mhi[b];
          c3 &= mhi[b];
        }
        mma_f16_16816(o[2 * kp], a0, a1, a2, a3, ph0[b], ph1[b]);
        mma_f16_16816(o[2 * kp + 1], c0, c1, c2, c3, ph0[b], ph1[b]);
      }
    }
  }
}

// ---- prologue folded into the single-launch step
// "vLLM × HPC-Ops" (8sync News summary) puts a RoPE + QK-Norm + KV-write prologue in front of
// attention. Folded in, it costs no launch and no pass over q through HBM:
//  * The CTA that owns the last tile of a (request, kv head) writes that request's new token
//    (position L - 1) into the cache for this kv head: k through RMSNorm and RoPE, v as is,
//    both as bf16 or E4M3 codes of x / scale. No other CTA reads that token. Its consumer
//    warps do these writes when the kernel starts, fence them against the async proxy and
//    arrive on an mbarrier; the producer waits on it before it requests the chunk that holds
//    the token. (Done by the producer itself, the write's loads and fp64 angles would stall
//    the TMA stream at every segment end.)
//  * Each item's consumers form q from qkv in registers: RMSNorm, NeoX RoPE at L - 1, rounded
//    to bf16 as the prologue kernel's q_out. The rotation table of an item (cos, sin of
//    pos * theta^(-2i/D), evaluated in fp64) is built by 64 consumer threads during the item
//    before, so it is ready when the item starts.
// Arithmetic follows hpc_decode_prologue (same formulas; the new K/V bytes use its lane order).

// Rotation table of position pos into cs / sn (D/2 floats each), by threads t < D/2.
template <int D>
__device__ __forceinline__ void rope_table(int64_t pos, const double* inv_freq, float* cs, float* sn, int t) {
  if (t < D / 2) {
    double a, b;
    sincos(static_cast<double>(pos) * inv_freq[t], &a, &b);
    sn[t] = static_cast<float>(a);
    cs[t] = static_cast<float>(b);
  }
}

// New token of request r, kv head kvh: one warp. Lane holds d = lane + 32 j, as in
// hpc_decode_prologue, and the arithmetic is the same.
template <int D, bool FP8>
__device__ void write_new_token(const AttnParams& p, int r, int kvh, const double* inv_freq, int lane) {
  constexpr int PER = D / 32, HALF = PER / 2;
  const int64_t pos = static_cast<int64_t>(p.seq_lens[r]) - 1;  // >= 0: the request owns tiles
  const int32_t page = p.block_table[r * p.max_pages + pos / p.page_size];
  if (page < 0 || page >= p.num_pages) {
    if (lane == 0) atomicOr(p.status, HPC_DEV_BAD_PAGE);
    return;
  }
  const int slot = static_cast<int>(pos % p.page_size);
  const int64_t heads = p.num_heads + 2 * p.kv_heads;
  const __nv_bfloat16* kx = p.qkv + (static_cast<int64_t>(r) * heads + p.num_heads + kvh) * D;
  const __nv_bfloat16* vx = kx + static_cast<int64_t>(p.kv_heads) * D;
  float k[PER], v[PER];
#pragma unroll
  for (int j = 0; j < PER; ++j) {
    k[j] = __bfloat162float(kx[lane + 32 * j]);
    v[j] = __bfloat162float(vx[lane + 32 * j]);
  }
  float ss = 0.f;
#pragma unroll
  for (int j = 0; j < PER; ++j) ss += k[j] * k[j];
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
  const float inv = 1.f / sqrtf(ss / D + p.eps);
#pragma unroll
  for (int j = 0; j < PER; ++j) k[j] = k[j] * inv * p.k_norm_w[lane + 32 * j];
#pragma unroll
  for (int j = 0; j < HALF; ++j) {
    double a, b;
    sincos(static_cast<double>(pos) * inv_freq[lane + 32 * j], &a, &b);
    const float cs = static_cast<float>(b), sn = static_cast<float>(a);
    const float x1 = k[j], x2 = k[j + HALF];
    k[j] = x1 * cs - x2 * sn;
    k[j + HALF] = x2 * cs + x1 * sn;
  }
  const int64_t base = p.nhd ? ((static_cast<int64_t>(page) * p.page_size + slot) * p.kv_heads + kvh) * D
                             : ((static_cast<int64_t>(page) * p.kv_heads + kvh) * p.page_size + slot) * D;
  if (FP8) {
    const float ks = p.k_scale[kvh], vs = p.v_scale[kvh];
    uint8_t* kd = static_cast<uint8_t*>(p.k_pages_w) + base;
    uint8_t* vd = static_cast<uint8_t*>(p.v_pages_w) + base;
#pragma unroll
    for (int j = 0; j < PER; ++j) {
      kd[lane + 32 * j] = f32_to_e4m3(k[j] / ks);
      vd[lane + 32 * j] = f32_to_e4m3(v[j] / vs);
    }
  } else {
    __nv_bfloat16* kd = static_cast<__nv_bfloat16*>(p.k_pages_w) + base;
    __nv_bfloat16* vd = static_cast<__nv_bfloat16*>(p.v_pages_w) + base;
#pragma unroll
    for (int j = 0; j < PER; ++j) {
      kd[lane + 32 * j] = __float2bfloat16_rn(k[j]);
      vd[lane + 32 * j] = __float2bfloat16_rn(v[j]);
    }
  }
}

// Element index d of q fragment element (ks, e), e = 0..3, for lane column c: the bf16 path
// holds pairs (16ks + 2c, +1) and (16ks + 8 + 2c, +1); the E4M3 path (16ks + 4c, +1, +2, +3).
// Element (ks + KSTEPS/2, e) is d + D/2: each lane holds both halves of its RoPE pairs.
template <bool FP8>
__device__ __forceinline__ int q_elem_d(int ks, int e, int c) {
  if (FP8) return 16 * ks + 4 * c + e;
  return 16 * ks + 2 * c + (e & 1) + 8 * (e >> 1);
}

// q fragments of an item from qkv: RMSNorm (q_norm_w, eps), RoPE from the item's table,
// rounded to bf16 (then to f16 for an E4M3 cache). Lanes of rows g >= group get zeros.
template <int D, bool FP8>
__device__ __forceinline__ void q_from_qkv(const AttnParams& p, int req, int head, bool live, const float* qw,
                                           const float* cs, const float* sn, int c, uint32_t (&qf)[D / 16][2]) {
  constexpr int KSTEPS = D / 16;
  const int64_t heads = p.num_heads + 2 * p.kv_heads;
  const __nv_bfloat16* src = p.qkv + (static_cast<int64_t>(req) * heads + (live ? head : 0)) * D;
  float x[KSTEPS][4];
  float ss = 0.f;
#pragma unroll
  for (int ks = 0; ks < KSTEPS; ++ks) {
#pragma unroll
    for (int e = 0; e < 4; e += 2) {
      const uint32_t w = live ? *reinterpret_cast<const uint32_t*>(src + q_elem_d<FP8>(ks, e, c)) : 0u;
      x[ks][e] = __uint_as_float(w << 16);
      x[ks][e + 1] = __uint_as_float(w & 0xffff0000u);
    }
#pragma unroll
    for (int e = 0; e < 4; ++e) ss += x[ks][e] * x[ks][e];
  }
  ss += __shfl_xor_sync(0xffffffffu, ss, 1);  // the four lanes of one row hold the whole head
  ss += __shfl_xor_sync(0xffffffffu, ss, 2);
  const float inv = 1.f / sqrtf(ss / D + p.eps);
#pragma unroll
  for (int ks = 0; ks < KSTEPS; ++ks)
#pragma unroll
    for (int e = 0; e < 4; ++e) x[ks][e] = x[ks][e] * inv * qw[q_elem_d<FP8>(ks, e, c)];
#pragma unroll
  for (int ks = 0; ks < KSTEPS / 2; ++ks)
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int i = q_elem_d<FP8>(ks, e, c);
      const float x1 = x[ks][e], x2 = x[ks + KSTEPS / 2][e];
      x[ks][e] = x1 * cs[i] - x2 * sn[i];
      x[ks + KSTEPS / 2][e] = x2 * cs[i] + x1 * sn[i];
    }
#pragma unroll
  for (int ks = 0; ks < KSTEPS; ++ks) {
    const uint32_t lo = live ? pack_bf16x2(x[ks][0], x[ks][1]) : 0u;
    const uint32_t hi = live ? pack_bf16x2(x[ks][2], x[ks][3]) : 0u;
    qf[ks][0] = FP8 ? bf16x2_to_f16x2(lo) : lo;
    qf[ks][1] = FP8 ? bf16x2_to_f16x2(hi) : hi;
  }
}

template <int D, bool FP8, bool FUSED, bool PRO, bool MULTI>
__global__ void __launch_bounds__(kThreads, 1)
    decode_attention_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                            const AttnParams p) {
  static_assert(FUSED || !PRO, "the prologue is folded into the single-launch step only");
  static_assert(FUSED || !MULTI, "several new tokens per request run in the single-launch step only");
  static_assert(!(PRO && MULTI), "the folded prologue takes one new token per request");
  // query tokens per request: a compile-time 1 unless this is the several-new-tokens kernel
  const int q_len = MULTI ? p.q_len : 1;
  using S = Shape<D, FP8>;
  using Cursor = typename CursorOf<FUSED>::type;
  extern __shared__ uint8_t smem_raw[];
  __shared__ int64_t s_scan[16], s_walk[9];
  __shared__ int s_flag;
  __shared__ int32_t s_pages[32];
  // per ring slot: the stage's page id was outside the pool, so page 0 stood in for it and the
  // consumers skip the stage (written before the fill's arrive, read after its wait)
  __shared__ uint8_t s_bad[kMaxStages];
  __shared__ int s_rec_n;  // items this CTA has run (written by consumer thread 0)
  // folded prologue: q_norm_w, theta^(-2i/D), two rotation tables [cos | sin], new-token barrier
  __shared__ float s_qw[PRO ? D : 1];
  __shared__ double s_invf[PRO ? D / 2 : 1];
  __shared__ float s_rope[PRO ? 2 * D : 1];
  __shared__ uint64_t s_pro_bar;
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int stages = p.stages;
  uint8_t* ring = smem;
  float* red_o = reinterpret_cast<float*>(smem + static_cast<size_t>(stages) * p.stage_bytes);
  float* red_m = red_o + kConsumerWarps * 8 * S::kRedStride;
  float* red_l = red_m + kConsumerWarps * 8;
  // Barriers: full[stages][groups], then empty[stages]. Stage n (counted over this CTA's items)
  // lives in slot n % stages and is read by warp group n % groups. Its fill completes on
  // full[n % stages][n % groups]. Each group therefore waits on every phase of its own full
  // barriers in order, and a parity wait can never match a phase two behind.
  uint64_t* bars = reinterpret_cast<uint64_t*>(red_l + kConsumerWarps * 8);
  const int bpc = p.chunk_tokens / 16;          // 16-token blocks per stage
  const int q_pad = MULTI ? q_pad_of(q_len) : 1;  // warp slots per block range: one per query token
  const int nb = blocks_per_warp(bpc, FP8, q_pad);  // 16-token blocks per warp per stage
  const int wtok = bpc / nb;                    // warps that split a stage's blocks
  const int wps = wtok * q_pad;                 // warps per stage
  const int groups = kConsumerWarps / wps;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t ring_u32 = smem_u32(ring);
  const uint32_t full0 = smem_u32(bars), empty0 = smem_u32(bars + stages * groups);

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
    for (int s = 0; s < stages * groups; ++s) mbar_init(full0 + 8 * s, 1);
    for (int s = 0; s < stages; ++s) mbar_init(empty0 + 8 * s, wps);
    if (PRO) mbar_init(smem_u32(&s_pro_bar), kConsumerWarps);
    fence_barrier_init();
  }
  if (threadIdx.x == kConsumerWarps * 32) {
    prefetch_tensormap(&tm_k);
    prefetch_tensormap(&tm_v);
  }
  __syncthreads();
  // Everything above overlaps the previous kernel's tail under programmatic dependent launch;
  // seq_lens, q, the cache and the output buffers are touched only after it has finished. The
  // single launch's plan reads seq_lens alone, and runs before the wait when the caller says
  // the previous kernel does not write them (plan_early).
  const bool early = FUSED && p.plan_early;
  if (!early) {
    pdl_wait();
    pdl_launch_dependents();
  }

  Cursor cursor;
  int64_t chunk = 0;
  if constexpr (FUSED) {
    plan_in_kernel<D>(p, reinterpret_cast<int64_t*>(red_o), s_scan, s_walk, cursor, chunk);
    if (early) {
      pdl_wait();
      pdl_launch_dependents();
    }
  } else {
    cursor.it = p.cta_indptr[blockIdx.x];
    cursor.it_end = p.cta_indptr[blockIdx.x + 1];
  }
#ifdef HPC_TRACE
  if (trace && threadIdx.x == 0) trace[1] = global_timer_ns();
#endif
  const int C = p.chunk_tokens;
  const int P = p.page_size;

  if (warp == kConsumerWarps) {
    // ------------------------------------------------------------------ producer
    // The warp loads the page ids of the next 32 chunks in one coalesced load into shared
    // memory; lane 0 then issues the TMA copies on its own. Per stage, lane 0 does only
    // register work: the page offset is a mask (page sizes are powers of two), and the fill
    // parities of the full[slot][group] barriers live in two 64-bit words.
    const uint64_t policy = l2_policy_evict_first();
    const int p_shift = __ffs(P) - 1;
    int stage = 0, gidx = 0;
    uint32_t phase = 0;
    uint64_t par_lo = 0, par_hi = 0;  // bit slot * groups + group: parity of that barrier's next fill
    int64_t issued = 0;
    bool ok = true;
    uint32_t bad = 0;
    bool pro_done = !PRO;  // the new tokens of this CTA's segments are in the cache
    ItemInfo x;
    while (ok && cursor.next(p, x)) {
      const bool has_new = PRO && x.tok1 == p.seq_lens[x.req];  // the item holds token L - 1
      const int32_t* bt = p.block_table + x.req * p.max_pages + (x.tok0 >> p_shift);
      const int off0 = static_cast<int>(x.tok0 & (P - 1));
      const int64_t nchunks = x.tok1 > x.tok0 ? (x.tok1 - x.tok0 + C - 1) / C : 0;
      // Lane 0 requests chunk cb + k: waits for its slot, then issues the K and V boxes.
      auto issue = [&](int64_t cb, int k) -> bool {
        if (!mbar_wait(empty0 + 8 * stage, phase ^ 1)) {
          bad |= HPC_DEV_TIMEOUT;
          return false;
        }
        int32_t page = s_pages[k];
        const int off = static_cast<int>((off0 + (cb + k) * C) & (P - 1));
        // a page id outside the pool is never handed to the copy engine: page 0 stands in, and
        // the consumers leave the stage's tokens out (a stage never spans two pages)
        const bool page_ok = page >= 0 && page < p.num_pages;
        if (!page_ok) {
          bad |= HPC_DEV_BAD_PAGE;
          page = 0;
        }
        s_bad[stage] = page_ok ? 0 : 1;
        const int bi = stage * groups + gidx;
        const uint32_t full = full0 + 8 * bi;
        if (bi < 64) par_lo ^= uint64_t(1) << bi;
        else par_hi ^= uint64_t(1) << (bi - 64);
        const uint32_t dst = ring_u32 + stage * p.stage_bytes;
        // tensor-map coordinates: (d, token, kv head, page) for HND, (d, kv head, token, page) for NHD
        const int c1 = p.nhd ? x.kvh : off, c2 = p.nhd ? off : x.kvh;
        mbar_arrive_expect_tx(full, p.stage_bytes);
#pragma unroll
        for (int pl = 0; pl < S::kPlanes; ++pl)
          tma_load_4d(dst + pl * p.plane_bytes, &tm_k, full, pl * (128 / S::kElt), c1, c2, page, policy);
#pragma unroll
        for (int pl = 0; pl < S::kPlanes; ++pl)
          tma_load_4d(dst + (S::kPlanes + pl) * p.plane_bytes, &tm_v, full, pl * (128 / S::kElt), c1, c2, page,
                      policy);
        ++issued;
        if (++stage == stages) {
          stage = 0;
          phase ^= 1;
        }
        if (++gidx == groups) gidx = 0;
        return true;
      };
      for (int64_t cb = 0; cb < nchunks && ok; cb += 32) {
        const int nk = static_cast<int>(nchunks - cb < 32 ? nchunks - cb : 32);
        __syncwarp();  // lane 0 has finished with the previous batch of page ids
        if (lane < nk) s_pages[lane] = bt[(off0 + (cb + lane) * C) >> p_shift];
        __syncwarp();
        if (lane == 0) {
          for (int k = 0; k < nk && ok; ++k) {
            // with the folded prologue, the chunk that holds the new token waits for its write
            if (PRO && has_new && !pro_done && cb + k == nchunks - 1) {
              if (!mbar_wait(smem_u32(&s_pro_bar), 0)) {
                bad |= HPC_DEV_TIMEOUT;
                ok = false;
                break;
              }
              pro_done = true;
            }
            ok = issue(cb, k);
          }
        }
        ok = __shfl_sync(0xffffffffu, ok, 0);
      }
    }
    // Drain: the last fill of every slot must have landed before the CTA may exit (the
    // consumers stop waiting after a timeout). Slot s was last filled by stage
    // n = last - ((last - s) mod stages), for group n % groups, with the parity before its flip.
    if (lane == 0) {
      const int64_t last = issued - 1;
      for (int s = 0; s < stages && s <= last; ++s) {
        const int64_t n = last - ((last - s) % stages);
        const int bi = s * groups + static_cast<int>(n % groups);
        const uint32_t par = static_cast<uint32_t>(((bi < 64 ? par_lo >> bi : par_hi >> (bi - 64)) & 1u) ^ 1u);
        if (!mbar_wait(full0 + 8 * bi, par)) bad |= HPC_DEV_TIMEOUT;
      }
      if (bad) atomicOr(p.status, bad);
#ifdef HPC_TRACE
      if (trace) {
        trace[4] = global_timer_ns();
        trace[6] = static_cast<uint64_t>(issued);
      }
#endif
    }
    return;
  }

  // -------------------------------------------------------------------- consumers
  // Stage n is read by the warps of group n % groups: wps warps, each taking nb consecutive
  // 16-token blocks. Only those warps wait on it and release it (empty-barrier count = wps).
  const int g = lane >> 2, c = lane & 3;  // MMA fragment row / column pair
  constexpr int KSTEPS = D / 16;
  // warp = (group, query token, block range): group * wps + my_t * wtok + block range
  const int my_group = warp / wps, my_t = MULTI ? (warp % wps) / wtok : 0, my_first = (warp % wtok) * nb;
  const bool t_live = !MULTI || my_t < q_len;
  const uint32_t my_full0 = full0 + 8 * my_group;  // + 8 * groups * slot
  const int ctid = threadIdx.x, cthreads = kConsumerWarps * 32;
  int stage = 0, gidx = 0;
  uint32_t wait_par = 0;  // bit s: parity of this group's next wait on slot s
  bool ok = true;
  if constexpr (FUSED) zero_empty_requests<D>(p, ctid, cthreads);
  int it_par = 0;  // parity of the item count: selects the rotation table
  if constexpr (PRO) {
    for (int i = ctid; i < D; i += cthreads) s_qw[i] = p.q_norm_w[i];
    if (ctid < D / 2) s_invf[ctid] = pow(p.rope_theta, -2.0 * ctid / D);
    if (ctid == 0)
      for (int r = blockIdx.x; r < p.batch; r += gridDim.x)
        if (p.seq_lens[r] == 0) atomicOr(p.status, HPC_DEV_BAD_SEQLEN);  // no token to decode
    named_barrier_sync(1, cthreads);
    {
      // the new token of every segment that ends in this CTA, one warp per segment
      Cursor c2 = cursor;
      ItemInfo y;
      int j = 0;
      while (c2.next(p, y)) {
        if (y.tok1 != p.seq_lens[y.req]) continue;
        if (j++ % kConsumerWarps == warp) write_new_token<D, FP8>(p, y.req, y.kvh, s_invf, lane);
      }
      fence_proxy_async_global();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&s_pro_bar));
      // the first item's rotation table
      c2 = cursor;
      if (c2.next(p, y)) rope_table<D>(static_cast<int64_t>(p.seq_lens[y.req]) - 1, s_invf, s_rope, s_rope + D / 2, ctid);
    }
    named_barrier_sync(1, cthreads);
  }

  ItemInfo x;
  while (cursor.next(p, x)) {
    const int kvh = x.kvh;
    const int head0 = kvh * p.group;
    if (ctid == 0) {  // items this CTA ran (its record, and the trace's count)
      if (FUSED && p.record) record_item(p, s_rec_n, x);
      ++s_rec_n;
    }
    const int64_t tok0 = x.tok0, tok1 = x.tok1;
    // causal limit of this warp's query token: it sits at position L - q_len + my_t
    int64_t lim = tok1;
    if (MULTI) {
      const int64_t last = static_cast<int64_t>(p.seq_lens[x.req]) - q_len + my_t + 1;
      lim = last < tok1 ? last : tok1;
    }

    // Q^T fragments (B operand): lane (g, c) holds query head head0 + g.
    uint32_t qf[KSTEPS][2];
    if constexpr (PRO) {
      const float* tab = s_rope + it_par * D;
      q_from_qkv<D, FP8>(p, x.req, head0 + g, g < p.group, s_qw, tab, tab + D / 2, c, qf);
      // the next item's rotation table goes into the other buffer; the item-end barrier
      // publishes it, and nobody reads that buffer until then
      Cursor c2 = cursor;
      ItemInfo y;
      if (ctid < D / 2 && c2.next(p, y)) {
        float* nt = s_rope + (it_par ^ 1) * D;
        rope_table<D>(static_cast<int64_t>(p.seq_lens[y.req]) - 1, s_invf, nt, nt + D / 2, ctid);
      }
    } else {
      const bool live = g < p.group && t_live;
      const uint32_t* qrow = reinterpret_cast<const uint32_t*>(
          p.q + ((static_cast<int64_t>(x.req) * q_len + (t_live ? my_t : 0)) * p.num_heads + head0 +
                 (live ? g : 0)) * D);
#pragma unroll
      for (int ks = 0; ks < KSTEPS; ++ks) {
        if (!FP8) {
          qf[ks][0] = live ? qrow[8 * ks + c] : 0u;
          qf[ks][1] = live ? qrow[8 * ks + 4 + c] : 0u;
        } else {
          // k-slots (2c, 2c+1) and (8+2c, 9+2c) of chunk ks hold d = 16ks + 4c + {0,1} and {2,3}
          qf[ks][0] = live ? bf16x2_to_f16x2(qrow[8 * ks + 2 * c]) : 0u;
          qf[ks][1] = live ? bf16x2_to_f16x2(qrow[8 * ks + 2 * c + 1]) : 0u;
        }
      }
    }
    float score_scale = p.score_scale;
    if (FP8) score_scale *= p.k_scale[kvh];

    float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;  // heads 2c, 2c+1
    float o[KSTEPS][4];
#pragma unroll
    for (int i = 0; i < KSTEPS; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;

    for (int64_t t = tok0; t < tok1; t += C) {
      if (gidx == my_group) {
        if (ok && !mbar_wait(my_full0 + 8 * groups * stage, (wait_par >> stage) & 1u)) {
          ok = false;
          if (lane == 0) atomicOr(p.status, HPC_DEV_TIMEOUT);
        }
        wait_par ^= 1u << stage;
#ifdef HPC_TRACE
        if (trace && warp == 0 && lane == 0 && trace[2] == 0) trace[2] = global_timer_ns();
#endif
        const int64_t tb = t + 16 * my_first;
        if (ok && t_live && tb < lim) {
          const uint32_t kbase = ring_u32 + stage * p.stage_bytes;
          const uint32_t vbase = kbase + S::kPlanes * p.plane_bytes;
          const bool bad_stage = s_bad[stage] != 0;
          if (nb == 4)
            consume_blocks<D, FP8, 4>(kbase, vbase, p.plane_bytes, 16 * my_first, tb, lim, bad_stage, qf, score_scale,
                                      m0, m1, l0, l1, o, lane);
          else if (nb == 2)
            consume_blocks<D, FP8, 2>(kbase, vbase, p.plane_bytes, 16 * my_first, tb, lim, bad_stage, qf, score_scale,
                                      m0, m1, l0, l1, o, lane);
          else
            consume_blocks<D, FP8, 1>(kbase, vbase, p.plane_bytes, 16 * my_first, tb, lim, bad_stage, qf, score_scale,
                                      m0, m1, l0, l1, o, lane);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(empty0 + 8 * stage);
      }
      if (++stage == stages) stage = 0;
      if (++gidx == groups) gidx = 0;
    }

    // ---- merge the 8 warps' states for this item
#pragma unroll
    for (int off = 4; off < 32; off <<= 1) {
      l0 += __shfl_xor_sync(0xffffffffu, l0, off);
      l1 += __shfl_xor_sync(0xffffffffu, l1, off);
    }
    if (g == 0) {
      red_m[warp * 8 + 2 * c] = m0;
      red_m[warp * 8 + 2 * c + 1] = m1;
      red_l[warp * 8 + 2 * c] = l0;
      red_l[warp * 8 + 2 * c + 1] = l1;
    }
    {
      // rows of heads 2c and 2c+1; column d is stored at d ^ (4 * head)
      float* r0 = red_o + (warp * 8 + 2 * c) * S::kRedStride;
      float* r1 = r0 + S::kRedStride;
      const int x0 = 8 * c, x1 = 8 * c + 4;
#pragma unroll
      for (int i = 0; i < KSTEPS; ++i) {
        const int d0 = 16 * i + out_row<FP8>(g, 0), d1 = 16 * i + out_row<FP8>(g, 1);
        r0[d0 ^ x0] = o[i][0];
        r1[d0 ^ x1] = o[i][1];
        r0[d1 ^ x0] = o[i][2];
        r1[d1 ^ x1] = o[i][3];
      }
    }
    named_barrier_sync(1, cthreads);
    const float vs = FP8 ? p.v_scale[kvh] : 1.f;
    // output row (query token tq, head h) combines the warps that computed query token tq
    for (int idx = ctid; idx < q_len * p.group * D; idx += cthreads) {
      const int row = idx / D, d = idx - row * D;
      const int tq = MULTI ? row / p.group : 0, h = row - tq * p.group;
      float M = -INFINITY;
#pragma unroll
      for (int wq = 0; wq < kConsumerWarps; ++wq)
        if (!MULTI || (wq % wps) / wtok == tq) M = fmaxf(M, red_m[wq * 8 + h]);
      float Ls = 0.f, acc = 0.f;
      if (M != -INFINITY) {
#pragma unroll
        for (int wq = 0; wq < kConsumerWarps; ++wq) {
          if (MULTI && (wq % wps) / wtok != tq) continue;
          const float e = exp2f(red_m[wq * 8 + h] - M);
          Ls += e * red_l[wq * 8 + h];
          acc += e * red_o[(wq * 8 + h) * S::kRedStride + (d ^ (4 * h))];
        }
      }
      acc *= vs;
      if (x.direct) {
        const float val = Ls > 0.f ? acc / Ls : 0.f;
        const int64_t oi = ((static_cast<int64_t>(x.req) * q_len + tq) * p.num_heads + head0 + h) * D + d;
        if (p.out_bf16) reinterpret_cast<__nv_bfloat16*>(p.out)[oi] = __float2bfloat16_rn(val);
        else reinterpret_cast<float*>(p.out)[oi] = val;
        if (!MULTI && p.lse && d == 0)  // log-sum-exp in natural-log units (M is in log2 units)
          p.lse[static_cast<int64_t>(x.req) * p.num_heads + head0 + h] = Ls > 0.f ? M * kLn2 + logf(Ls) : -INFINITY;
      } else {
        const int64_t pi = (x.slot * q_len + tq) * p.group + h;
        p.partial_o[pi * D + d] = acc;
        if (d == 0) {
          p.partial_ml[2 * pi] = M * kLn2;  // natural-log units
          p.partial_ml[2 * pi + 1] = Ls;
        }
      }
    }
    if constexpr (FUSED) {
      if (!x.direct) {
        // the CTA that completes the last piece of this (request, kv head) merges it
        __threadfence();
        named_barrier_sync(1, cthreads);
        if (ctid == 0) {
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
        named_barrier_sync(1, cthreads);
        if (s_flag) merge_segment<D>(p, x, chunk, ctid, cthreads, red_o, kConsumerWarps * 8 * S::kRedStride);
      }
    }
    named_barrier_sync(1, cthreads);  // reduce buffers are reused by the next item
    it_par ^= 1;
  }
  if constexpr (FUSED) {
    // s_walk still holds this CTA's unit run and the chunk from plan_in_kernel
    if (p.record && ctid == 0) record_header(p, s_walk[0], s_walk[1], s_walk[7], s_rec_n);
  }
#ifdef HPC_TRACE
  if (trace && ctid == 0) {
    if (s_rec_n > 0) trace[3] = global_timer_ns();
    trace[5] = static_cast<uint64_t>(s_rec_n);
  }
#endif
}

// ----------------------------------------------------------------------------- host side

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  });
  return fn;
}

// Tensor map of a page pool, HND [num_pages][Hkv][P][D] or NHD [num_pages][P][Hkv][D]. Each box
// is 128 bytes of one token row x `box_tokens` tokens of one (page, kv head), stored with the
// 128-byte swizzle. Dimensions are listed innermost first: (D, P, Hkv, pages) for HND and
// (D, Hkv, P, pages) for NHD, so the same box lands in shared memory in the same layout.
int make_pool_map(CUtensorMap* map, const void* base, bool fp8, bool nhd, int D, int P, int Hkv, int num_pages,
                  int box_tokens) {
  auto fn = encode_fn();
  if (!fn) return fail(HPC_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
  const int elt = fp8 ? 1 : 2;
  const cuuint64_t row = static_cast<cuuint64_t>(D) * elt;
  cuuint64_t dims[4], strides[3];
  cuuint32_t box[4];
  dims[0] = static_cast<cuuint64_t>(D);
  dims[3] = static_cast<cuuint64_t>(num_pages);
  box[0] = static_cast<cuuint32_t>(128 / elt);
  box[3] = 1;
  if (nhd) {
    dims[1] = static_cast<cuuint64_t>(Hkv);
    dims[2] = static_cast<cuuint64_t>(P);
    strides[0] = row;
    strides[1] = row * Hkv;
    strides[2] = row * Hkv * P;
    box[1] = 1;
    box[2] = static_cast<cuuint32_t>(box_tokens);
  } else {
    dims[1] = static_cast<cuuint64_t>(P);
    dims[2] = static_cast<cuuint64_t>(Hkv);
    strides[0] = row;
    strides[1] = row * P;
    strides[2] = row * P * Hkv;
    box[1] = static_cast<cuuint32_t>(box_tokens);
    box[2] = 1;
  }
  cuuint32_t estr[4] = {1, 1, 1, 1};
  // L2 fetch granularity: 256 B when a box row is followed in memory by data the same stream
  // reads (HND rows are contiguous, and a bf16 NHD row is 256 B read as two 128 B boxes).
  // An E4M3 NHD row is 128 B followed by another kv head's row, so 128 B.
  const CUtensorMapL2promotion promo =
      (nhd && row <= 128) ? CU_TENSOR_MAP_L2_PROMOTION_L2_128B : CU_TENSOR_MAP_L2_PROMOTION_L2_256B;
  CUresult r = fn(map, fp8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4,
                  const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  CU_TENSOR_MAP_SWIZZLE_128B, promo, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(HPC_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", static_cast<int>(r));
  return HPC_OK;
}

struct LaunchShape {
  int stages, smem, plane_bytes, stage_bytes;
};

// Static shared memory of the kernel: the walk and page-id arrays, plus the folded prologue's
// norm weights, frequencies and rotation tables.
inline int static_smem_bytes(int D, bool pro) { return 512 + (pro ? D * 4 + D / 2 * 8 + 2 * D * 4 + 64 : 0); }

int launch_shape(int D, bool fp8, int C, int ctas_per_sm, LaunchShape* ls, bool pro = false, int q_len = 1) {
  const int elt = fp8 ? 1 : 2;
  const int planes = D * elt / 128;
  const int plane_bytes = C * 128;
  const int stage_bytes = 2 * planes * plane_bytes;
  const int q_pad = q_pad_of(q_len);
  const int bpc = C / 16, nb = blocks_per_warp(bpc, fp8, q_pad), groups = kConsumerWarps / ((bpc / nb) * q_pad);
  const int red = kConsumerWarps * 8 * D * 4 + 2 * kConsumerWarps * 8 * 4;
  const int budget = kSmemLimit / (ctas_per_sm < 1 ? 1 : ctas_per_sm) - static_smem_bytes(D, pro);
  int stages = kMaxStages;
  // reduce buffers, full[stages][groups] + empty[stages] barriers, 1 KB alignment slack
  auto need = [&](int st) { return st * stage_bytes + red + (st * groups + st) * 8 + 1024; };
  while (stages > 2 && need(stages) > budget) --stages;
  if (need(stages) > budget) return fail(HPC_ERR_SHAPE, "page chunk of %d tokens does not fit two pipeline stages", C);
  ls->stages = stages;
  ls->plane_bytes = plane_bytes;
  ls->stage_bytes = stage_bytes;
  ls->smem = need(stages);
  return HPC_OK;
}

// Tokens per pipeline stage: one TMA box per tensor plane. A box never crosses a page and is
// at most 64 tokens, so a stage is at most 32 KB and the ring keeps several stages in flight.
inline int chunk_tokens(int tile_len, int page_size) {
  int C = tile_len < page_size ? tile_len : page_size;
  return C > 64 ? 64 : C;
}

template <int D, bool FP8, bool FUSED, bool PRO = false, bool MULTI = false>
int launch(const CUtensorMap& mk, const CUtensorMap& mv, const AttnParams& prm, int grid, int smem,
           cudaStream_t stream) {
  auto kern = decode_attention_kernel<D, FP8, FUSED, PRO, MULTI>;
  static int configured[64] = {0};  // per device: largest dynamic smem already allowed
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && configured[dev] < smem) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
      return check_launch("cudaFuncSetAttribute(decode_attention_kernel)");
    configured[dev] = smem;
  }
  const cudaError_t e = launch_pdl(kern, dim3(grid), dim3(kThreads), static_cast<size_t>(smem), stream, mk, mv, prm);
  if (e != cudaSuccess) return fail(HPC_ERR_CUDA, "decode_attention_kernel: %s", cudaGetErrorString(e));
  return check_launch("decode_attention_kernel");
}

}  // namespace
}  // namespace hpc

using namespace hpc;

extern "C" size_t hpc_partial_o_bytes(const hpc_plan* plan, int32_t num_heads, int32_t head_dim) {
  if (!plan || plan->kv_heads < 1) return 0;
  return static_cast<size_t>(plan->max_items) * (num_heads / plan->kv_heads) * head_dim * sizeof(float);
}

extern "C" size_t hpc_partial_ml_bytes(const hpc_plan* plan, int32_t num_heads) {
  if (!plan || plan->kv_heads < 1) return 0;
  return static_cast<size_t>(plan->max_items) * (num_heads / plan->kv_heads) * 2 * sizeof(float);
}

extern "C" int hpc_attention_launch_info(int32_t head_dim, hpc_dtype kv_dtype, int32_t page_size, int32_t tile_len,
                                         int32_t ctas_per_sm, int32_t e4m3_kernel, int32_t* stages,
                                         int32_t* smem_bytes, int32_t* threads) {
  if (tile_len <= 0 || page_size <= 0) return fail(HPC_ERR_ARG, "bad tile/page size");
  LaunchShape ls;
  const int C = chunk_tokens(tile_len, page_size);
  if (kv_dtype == HPC_E4M3 && e4m3_kernel == HPC_E4M3_TCGEN05 && tc_supported(head_dim, true, 8, 1, false)) {
    const int sm = tc_smem_bytes(ctas_per_sm);
    if (!sm) return fail(HPC_ERR_SHAPE, "tensor-core E4M3 attention does not fit shared memory");
    if (stages) *stages = (sm - 12288 - 1024) / (2 * 128 * 128);
    if (smem_bytes) *smem_bytes = sm;
    if (threads) *threads = tc_threads();
    return HPC_OK;
  }
  int rc = launch_shape(head_dim, kv_dtype == HPC_E4M3, C, ctas_per_sm, &ls);
  if (rc) return rc;
  if (stages) *stages = ls.stages;
  if (smem_bytes) *smem_bytes = ls.smem;
  if (threads) *threads = kThreads;
  return HPC_OK;
}

extern "C" size_t hpc_step_record_bytes(int32_t num_ctas, int32_t record_items) {
  if (num_ctas < 1 || record_items < 0) return 0;
  return static_cast<size_t>(num_ctas) * record_stride(record_items);
}

extern "C" uint32_t hpc_build_flags(void) {
#ifdef HPC_TRACE
  return HPC_BUILD_TRACE;
#else
  return 0u;
#endif
}

namespace hpc {
namespace {

// Per-call options, checked. single_launch: the call is one of the hpc_decode_step entry points,
// where the item cost and the record apply.
struct Options {
  int32_t item_cost = HPC_ITEM_COST_DEFAULT;
  bool tc = false;
  int32_t multi_kernel = HPC_MULTI_DEFAULT;  // several new tokens: which kernel
  uint8_t* record = nullptr;
  int32_t record_items = 0;
  uint64_t* trace = nullptr;
  int32_t seq_lens_ready = 0;  // single launch: plan before waiting for the previous kernel
};

int read_options(const hpc_step_options* o, bool single_launch, Options* out) {
  *out = Options{};
  if (!o) return HPC_OK;
  if (o->item_cost != HPC_ITEM_COST_DEFAULT && (o->item_cost < 0 || o->item_cost > HPC_ITEM_COST_MAX))
    return fail(HPC_ERR_ARG, "item_cost must be HPC_ITEM_COST_DEFAULT or 0 .. %d", HPC_ITEM_COST_MAX);
  if (o->e4m3_kernel != HPC_E4M3_MMA && o->e4m3_kernel != HPC_E4M3_TCGEN05)
    return fail(HPC_ERR_ARG, "e4m3_kernel must be HPC_E4M3_MMA or HPC_E4M3_TCGEN05");
  if (o->multi_kernel != HPC_MULTI_DEFAULT && o->multi_kernel != HPC_MULTI_MMA && o->multi_kernel != HPC_MULTI_TCGEN05)
    return fail(HPC_ERR_ARG, "multi_kernel must be HPC_MULTI_DEFAULT, HPC_MULTI_MMA or HPC_MULTI_TCGEN05");
  if (o->seq_lens_ready != 0 && o->seq_lens_ready != 1) return fail(HPC_ERR_ARG, "seq_lens_ready must be 0 or 1");
  if (!single_launch && (o->item_cost != HPC_ITEM_COST_DEFAULT || o->record || o->seq_lens_ready))
    return fail(HPC_ERR_ARG, "item_cost, record and seq_lens_ready apply to the single-launch steps only");
  if (o->record && (o->record_items < 0 || (reinterpret_cast<uintptr_t>(o->record) & 15)))
    return fail(HPC_ERR_ARG, "record needs record_items >= 0 and 16-byte alignment");
#ifndef HPC_TRACE
  if (o->trace) return fail(HPC_ERR_ARG, "a trace buffer needs a library built with HPC_TRACE");
#endif
  if (o->trace && (reinterpret_cast<uintptr_t>(o->trace) & 7)) return fail(HPC_ERR_ALIGN, "trace must be 8-byte aligned");
  out->item_cost = o->item_cost;
  out->tc = o->e4m3_kernel == HPC_E4M3_TCGEN05;
  out->multi_kernel = o->multi_kernel;
  out->record = static_cast<uint8_t*>(o->record);
  out->record_items = o->record ? o->record_items : 0;
  out->trace = o->trace;
  out->seq_lens_ready = o->seq_lens_ready;
  return HPC_OK;
}

// Checks shared by the attention entry points; fills the tensor maps, launch shape and the
// common kernel parameters.
int prepare(const void* q, const void* k_pages, const void* v_pages, hpc_dtype kv_dtype, hpc_kv_layout kv_layout,
            const float* k_scale,
            const float* v_scale, int32_t num_pages, int32_t page_size, int32_t num_heads, int32_t kv_heads,
            int32_t head_dim, const int32_t* block_table, int32_t max_pages_per_req, const int32_t* seq_lens,
            int32_t tile_len, int32_t grid, bool persistent, float sm_scale, void* out, hpc_dtype out_dtype,
            uint32_t* status, CUtensorMap* mk, CUtensorMap* mv, LaunchShape* ls, AttnParams* prm,
            bool pro = false, int q_len = 1) {
  if (!q || !k_pages || !v_pages || !block_table || !seq_lens || !out || !status)
    return fail(HPC_ERR_ARG, "null pointer argument");
  if (kv_dtype != HPC_BF16 && kv_dtype != HPC_E4M3) return fail(HPC_ERR_DTYPE, "kv_dtype must be BF16 or E4M3");
  if (out_dtype != HPC_FP32 && out_dtype != HPC_BF16) return fail(HPC_ERR_DTYPE, "out_dtype must be FP32 or BF16");
  if (kv_layout != HPC_HND && kv_layout != HPC_NHD) return fail(HPC_ERR_ARG, "kv_layout must be HND or NHD");
  const bool fp8 = kv_dtype == HPC_E4M3;
  const bool nhd = kv_layout == HPC_NHD;
  if (fp8 && (!k_scale || !v_scale)) return fail(HPC_ERR_ARG, "E4M3 cache needs k_scale and v_scale");
  if (num_pages < 1 || max_pages_per_req < 1 || num_heads < 1 || kv_heads < 1 || grid < 1)
    return fail(HPC_ERR_ARG, "sizes must be >= 1");
  if (num_heads % kv_heads) return fail(HPC_ERR_SHAPE, "num_heads %% kv_heads != 0");
  const int group = num_heads / kv_heads;
  if (group != 1 && group != 2 && group != 4 && group != 8) return fail(HPC_ERR_SHAPE, "group size must be 1, 2, 4 or 8");
  if (!(head_dim == 128 || (head_dim == 64 && !fp8)))
    return fail(HPC_ERR_SHAPE, "head_dim must be 128 (or 64 with a bf16 cache)");
  if (page_size != 16 && page_size != 32 && page_size != 64 && page_size != 128)
    return fail(HPC_ERR_SHAPE, "page_size must be 16, 32, 64 or 128");
  const int tl = tile_len;
  if (tl < 16 || tl % 16 || !(tl % page_size == 0 || page_size % tl == 0))
    return fail(HPC_ERR_SHAPE, "tile_len %d must be a multiple of 16 and of page_size %d, or divide it", tl, page_size);
  if (static_cast<int64_t>(max_pages_per_req) * page_size > INT32_MAX)
    return fail(HPC_ERR_SHAPE, "max_pages_per_req * page_size must fit in int32");
  if (!aligned16(q) || !aligned16(k_pages) || !aligned16(v_pages) || !aligned16(out))
    return fail(HPC_ERR_ALIGN, "q, caches and out must be 16-byte aligned");

  const int C = chunk_tokens(tl, page_size);
  const int sms = device_sm_count();
  int ctas_per_sm = (persistent && sms > 0) ? (grid + sms - 1) / sms : 1;
  if (ctas_per_sm < 1) ctas_per_sm = 1;
  if (ctas_per_sm > 4) ctas_per_sm = 4;
  int rc = launch_shape(head_dim, fp8, C, ctas_per_sm, ls, pro, q_len);
  if (rc) return rc;
  if ((rc = make_pool_map(mk, k_pages, fp8, nhd, head_dim, page_size, kv_heads, num_pages, C))) return rc;
  if ((rc = make_pool_map(mv, v_pages, fp8, nhd, head_dim, page_size, kv_heads, num_pages, C))) return rc;

  *prm = AttnParams{};
  prm->q = static_cast<const __nv_bfloat16*>(q);
  prm->block_table = block_table;
  prm->seq_lens = seq_lens;
  prm->k_scale = k_scale;
  prm->v_scale = v_scale;
  prm->out = out;
  prm->status = status;
  prm->max_pages = max_pages_per_req;
  prm->num_pages = num_pages;
  prm->page_size = page_size;
  prm->tile_len = tl;
  prm->chunk_tokens = C;
  prm->num_heads = num_heads;
  prm->group = group;
  prm->stages = ls->stages;
  prm->out_bf16 = out_dtype == HPC_BF16;
  prm->plane_bytes = ls->plane_bytes;
  prm->stage_bytes = ls->stage_bytes;
  prm->score_scale = sm_scale * kLog2e;
  prm->kv_heads = kv_heads;
  prm->max_seq_len = max_pages_per_req * page_size;  // checked above to fit int32
  prm->nhd = nhd ? 1 : 0;
  prm->q_len = q_len;
  return HPC_OK;
}

template <bool FUSED, bool PRO = false, bool MULTI = false>
int dispatch(int head_dim, bool fp8, bool tc, const CUtensorMap& mk, const CUtensorMap& mv, const AttnParams& prm,
             int grid, int smem, cudaStream_t st, bool tcm = false) {
  if (fp8 && !PRO && !MULTI && tc && tc_supported(head_dim, fp8, prm.group, prm.q_len, PRO)) {
    if (prm.trace) return fail(HPC_ERR_ARG, "the tcgen05 kernel writes no trace");
    return launch_attention_tc(FUSED, mk, mv, prm, grid, st);
  }
  if (FUSED && MULTI && tcm && tcm_supported(head_dim, fp8, prm.group, prm.q_len, PRO))
    return launch_attention_tcm(mk, mv, prm, grid, st);  // stamps the trace in 128-token stages
  if (fp8) return launch<128, true, FUSED, PRO, MULTI>(mk, mv, prm, grid, smem, st);
  if (head_dim == 128) return launch<128, false, FUSED, PRO, MULTI>(mk, mv, prm, grid, smem, st);
  return launch<64, false, FUSED, PRO, MULTI>(mk, mv, prm, grid, smem, st);
}

struct StepLayout {
  size_t tickets, partial_o, partial_ml, total;
};

// Rows of a partial slot: group heads for each of the q_len query tokens.
StepLayout step_layout(int32_t batch, int32_t group, int32_t kv_heads, int32_t head_dim, int32_t num_ctas,
                       int32_t q_len = 1) {
  auto up = [](size_t x) { return (x + 255) & ~size_t(255); };
  const size_t rows = static_cast<size_t>(group) * q_len;
  StepLayout L;
  L.tickets = 0;
  L.partial_o = up(static_cast<size_t>(batch) * kv_heads * sizeof(int32_t));
  L.partial_ml = L.partial_o + up(2 * static_cast<size_t>(num_ctas) * rows * head_dim * sizeof(float));
  L.total = L.partial_ml + up(2 * static_cast<size_t>(num_ctas) * rows * 2 * sizeof(float));
  return L;
}

}  // namespace
}  // namespace hpc

extern "C" int hpc_decode_attention(const void* q, const void* k_pages, const void* v_pages, hpc_dtype kv_dtype,
                                    hpc_kv_layout kv_layout, const float* k_scale, const float* v_scale, int32_t num_pages,
                                    int32_t page_size, int32_t num_heads, int32_t kv_heads, int32_t head_dim,
                                    const int32_t* block_table, int32_t max_pages_per_req, const int32_t* seq_lens,
                                    const hpc_plan* plan, float sm_scale, float* partial_o, float* partial_ml,
                                    void* out, hpc_dtype out_dtype, const hpc_step_options* options,
                                    uint32_t* status, void* stream) {
  if (!plan || !partial_o || !partial_ml) return fail(HPC_ERR_ARG, "null pointer argument");
  Options opt;
  if (int rc = read_options(options, false, &opt)) return rc;
  if (plan->kv_heads != kv_heads || plan->num_ctas < 1) return fail(HPC_ERR_ARG, "plan does not match kv_heads");
  if (!aligned16(partial_o)) return fail(HPC_ERR_ALIGN, "partial_o must be 16-byte aligned");
  CUtensorMap mk, mv;
  LaunchShape ls;
  AttnParams prm;
  int rc = prepare(q, k_pages, v_pages, kv_dtype, kv_layout, k_scale, v_scale, num_pages, page_size, num_heads,
                   kv_heads,
                   head_dim, block_table, max_pages_per_req, seq_lens, plan->tile_len, plan->num_ctas,
                   !plan->is_static, sm_scale, out, out_dtype, status, &mk, &mv, &ls, &prm);
  if (rc) return rc;
  prm.items = plan->items;
  prm.cta_indptr = plan->cta_indptr;
  prm.partial_o = partial_o;
  prm.partial_ml = partial_ml;
  prm.batch = plan->batch;
  prm.trace = opt.trace;
  return dispatch<false>(head_dim, kv_dtype == HPC_E4M3, opt.tc, mk, mv, prm, plan->num_ctas, ls.smem,
                         static_cast<cudaStream_t>(stream));
}

namespace hpc {

int step_three_launch(const void* q, const void* k_pages, const void* v_pages, hpc_dtype kv_dtype,
                      const float* k_scale, const float* v_scale, int32_t num_pages, int32_t page_size,
                      int32_t num_heads, int32_t kv_heads, int32_t head_dim, const int32_t* block_table,
                      int32_t max_pages_per_req, const int32_t* seq_lens, int32_t batch, int32_t tile_len,
                      int32_t num_ctas, float sm_scale, void* out, hpc_dtype out_dtype, uint32_t* status,
                      void* plan_workspace, size_t plan_bytes, float* partial_o, size_t partial_o_bytes,
                      float* partial_ml, size_t partial_ml_bytes, void* stream) {
  // every check first: the attention's (shapes, dtypes, alignment, the int32 token bound, the
  // tensor maps and launch shape), then the planner's, then the scratch sizes
  CUtensorMap mk, mv;
  LaunchShape ls;
  AttnParams prm;
  int rc = prepare(q, k_pages, v_pages, kv_dtype, HPC_HND, k_scale, v_scale, num_pages, page_size, num_heads,
                   kv_heads, head_dim, block_table, max_pages_per_req, seq_lens, tile_len, num_ctas, true, sm_scale,
                   out, out_dtype, status, &mk, &mv, &ls, &prm);
  if (rc) return rc;
  hpc_plan plan;
  rc = check_plan_args(seq_lens, batch, num_heads, kv_heads, tile_len, num_ctas, plan_workspace, &plan, status);
  if (rc) return rc;
  const size_t need_plan = hpc_plan_workspace_bytes(batch, kv_heads, num_ctas);
  const int64_t max_items = static_cast<int64_t>(num_ctas) + static_cast<int64_t>(batch) * kv_heads;
  const size_t rows = static_cast<size_t>(max_items) * (num_heads / kv_heads);
  if (!partial_o || !partial_ml) return fail(HPC_ERR_ARG, "null pointer argument");
  if (!aligned16(partial_o)) return fail(HPC_ERR_ALIGN, "partial_o must be 16-byte aligned");
  if (need_plan == 0 || plan_bytes < need_plan || partial_o_bytes < rows * head_dim * sizeof(float) ||
      partial_ml_bytes < rows * 2 * sizeof(float))
    return fail(HPC_ERR_CAPACITY, "scratch too small for the plan or the partial states");
  // max_pages_per_req * page_size fits int32 (checked by prepare)
  rc = hpc_decode_plan(seq_lens, batch, num_heads, kv_heads, tile_len, num_ctas, prm.max_seq_len, plan_workspace,
                       plan_bytes, &plan, status, stream);
  if (rc) return rc;
  prm.items = plan.items;
  prm.cta_indptr = plan.cta_indptr;
  prm.partial_o = partial_o;
  prm.partial_ml = partial_ml;
  prm.batch = batch;
  rc = dispatch<false>(head_dim, kv_dtype == HPC_E4M3, false, mk, mv, prm, num_ctas, ls.smem,
                       static_cast<cudaStream_t>(stream));
  if (rc) return rc;
  return hpc_merge_states(partial_o, partial_ml, &plan, num_heads, head_dim, out, out_dtype, status, stream);
}

}  // namespace hpc

extern "C" size_t hpc_decode_step_workspace_bytes(int32_t batch, int32_t num_heads, int32_t kv_heads,
                                                  int32_t head_dim, int32_t num_ctas) {
  if (batch < 1 || num_heads < 1 || kv_heads < 1 || head_dim < 1 || num_ctas < 1 || num_heads % kv_heads) return 0;
  return step_layout(batch, num_heads / kv_heads, kv_heads, head_dim, num_ctas).total;
}

namespace hpc {
namespace {

struct PrologueArgs {
  const void* qkv;
  const float* q_norm_w;
  const float* k_norm_w;
  float eps, rope_theta;
};

// Single-launch step; with `pro`, q is formed from qkv in the kernel and the new token's K/V
// are written into the cache first.
// Fixed cost of starting an item in the single-launch step's split, in 1/kCostPerTile of a
// tile. At an item end the consumers combine their states, write the output or a partial
// state, take the merge ticket (and merge), and load the next item's q; the ring keeps
// streaming, but only a few stages beyond what covers the memory latency. Per-CTA
// %globaltimer stamps on B200 put that cost near the time a CTA takes to stream 152 KB of KV
// at its share of HBM (one new token). With several new tokens a sweep of the cost put it at
// 320 KB on the mma.sync consumers and 224 KB on the tcgen05 kernel. A CTA that starts many
// items (many short requests) therefore gets fewer tiles. A caller's options->item_cost
// (1/16 tile) replaces it; 0 splits by tiles alone, the pages' rule.
int item_cost_units(int head_dim, bool fp8, int tile_len, int q_len, int32_t requested, bool tcm) {
  constexpr int64_t kMax = HPC_ITEM_COST_MAX;
  if (requested != HPC_ITEM_COST_DEFAULT) return requested;  // checked to lie in 0 .. kMax
  const int64_t tile_bytes = static_cast<int64_t>(tile_len) * head_dim * 2 * (fp8 ? 1 : 2);
  const int64_t item_bytes = (q_len == 1 ? 152 : (tcm ? 224 : 320)) * 1024;
  const int64_t c = (kCostPerTile * item_bytes + tile_bytes / 2) / tile_bytes;
  return static_cast<int>(c > kMax ? kMax : c);
}

int step_impl(const void* q, const void* k_pages, const void* v_pages, hpc_dtype kv_dtype, hpc_kv_layout kv_layout,
              const float* k_scale, const float* v_scale, int32_t num_pages, int32_t page_size, int32_t num_heads,
              int32_t kv_heads, int32_t head_dim, const int32_t* block_table, int32_t max_pages_per_req,
              const int32_t* seq_lens, int32_t batch, int32_t tile_len, int32_t num_ctas, float sm_scale,
              void* workspace, size_t workspace_bytes, void* out, hpc_dtype out_dtype,
              const hpc_step_options* options, uint32_t* status, void* stream, const PrologueArgs* pro,
              int32_t q_len = 1, float* lse = nullptr) {
  if (!workspace) return fail(HPC_ERR_ARG, "null pointer argument");
  Options opt;
  if (int rc = read_options(options, true, &opt)) return rc;
  if (lse && (q_len != 1 || pro)) return fail(HPC_ERR_ARG, "the log-sum-exp output is for the one-token step");
  if (q_len < 1 || q_len > 4) return fail(HPC_ERR_SHAPE, "q_len must be 1 to 4");
  if (pro && q_len != 1) return fail(HPC_ERR_SHAPE, "the folded prologue takes one new token per request");
  if (batch < 1) return fail(HPC_ERR_ARG, "batch must be >= 1");
  if ((reinterpret_cast<uintptr_t>(workspace) & 255) != 0) return fail(HPC_ERR_ALIGN, "workspace must be 256-byte aligned");
  if (kv_heads > 32767 || static_cast<int64_t>(batch) * kv_heads > (1ll << 30))
    return fail(HPC_ERR_SHAPE, "batch * kv_heads too large");
  CUtensorMap mk, mv;
  LaunchShape ls;
  AttnParams prm;
  int rc = prepare(q, k_pages, v_pages, kv_dtype, kv_layout, k_scale, v_scale, num_pages, page_size, num_heads,
                   kv_heads,
                   head_dim, block_table, max_pages_per_req, seq_lens, tile_len, num_ctas, true, sm_scale, out,
                   out_dtype, status, &mk, &mv, &ls, &prm, pro != nullptr, q_len);
  if (rc) return rc;
  // the per-request tile prefix lives in the reduce buffer while the CTA plans
  const size_t red_bytes = static_cast<size_t>(kConsumerWarps) * 8 * head_dim * sizeof(float);
  if ((static_cast<size_t>(batch) + 1) * sizeof(int64_t) > red_bytes)
    return fail(HPC_ERR_SHAPE, "batch %d is above the single-launch limit %zu; plan with hpc_decode_plan", batch,
                red_bytes / sizeof(int64_t) - 1);
  const StepLayout L = step_layout(batch, num_heads / kv_heads, kv_heads, head_dim, num_ctas, q_len);
  if (workspace_bytes < L.total) return fail(HPC_ERR_CAPACITY, "step workspace %zu < %zu bytes", workspace_bytes, L.total);
  char* ws = static_cast<char*>(workspace);
  prm.tickets = reinterpret_cast<int32_t*>(ws + L.tickets);
  prm.partial_o = reinterpret_cast<float*>(ws + L.partial_o);
  prm.partial_ml = reinterpret_cast<float*>(ws + L.partial_ml);
  prm.batch = batch;
  prm.lse = lse;
  const bool fp8 = kv_dtype == HPC_E4M3;
  // by default three or four new tokens go to the tcgen05 kernel (one product per stage for all
  // of them), two to the mma.sync consumers, where they are faster
  const bool tcm = !pro && q_len > 1 && tcm_supported(head_dim, fp8, prm.group, q_len, false) &&
                   (opt.multi_kernel == HPC_MULTI_TCGEN05 || (opt.multi_kernel == HPC_MULTI_DEFAULT && q_len >= 3));
  prm.item_cost = item_cost_units(head_dim, fp8, tile_len, q_len, opt.item_cost, tcm);
  prm.record = opt.record;
  prm.record_items = opt.record_items;
  prm.trace = opt.trace;
  prm.plan_early = opt.seq_lens_ready;
  if (!pro && q_len > 1)
    return dispatch<true, false, true>(head_dim, fp8, opt.tc, mk, mv, prm, num_ctas, ls.smem,
                                       static_cast<cudaStream_t>(stream), tcm);
  if (!pro)
    return dispatch<true>(head_dim, fp8, opt.tc, mk, mv, prm, num_ctas, ls.smem, static_cast<cudaStream_t>(stream));
  prm.qkv = static_cast<const __nv_bfloat16*>(pro->qkv);
  prm.q_norm_w = pro->q_norm_w;
  prm.k_norm_w = pro->k_norm_w;
  prm.eps = pro->eps;
  prm.rope_theta = static_cast<double>(pro->rope_theta);
  prm.k_pages_w = const_cast<void*>(k_pages);
  prm.v_pages_w = const_cast<void*>(v_pages);
  return dispatch<true, true>(head_dim, fp8, opt.tc, mk, mv, prm, num_ctas, ls.smem,
                              static_cast<cudaStream_t>(stream));
}

}  // namespace
}  // namespace hpc

extern "C" int hpc_decode_step(const void* q, const void* k_pages, const void* v_pages, hpc_dtype kv_dtype,
                               hpc_kv_layout kv_layout, const float* k_scale, const float* v_scale, int32_t num_pages, int32_t page_size,
                               int32_t num_heads, int32_t kv_heads, int32_t head_dim, const int32_t* block_table,
                               int32_t max_pages_per_req, const int32_t* seq_lens, int32_t batch, int32_t tile_len,
                               int32_t num_ctas, float sm_scale, void* workspace, size_t workspace_bytes, void* out,
                               hpc_dtype out_dtype, const hpc_step_options* options, uint32_t* status,
                               void* stream) {
  return step_impl(q, k_pages, v_pages, kv_dtype, kv_layout, k_scale, v_scale, num_pages, page_size, num_heads,
                   kv_heads, head_dim, block_table, max_pages_per_req, seq_lens, batch, tile_len, num_ctas, sm_scale,
                   workspace, workspace_bytes, out, out_dtype, options, status, stream, nullptr);
}

extern "C" int hpc_decode_step_lse(const void* q, const void* k_pages, const void* v_pages, hpc_dtype kv_dtype,
                                   hpc_kv_layout kv_layout, const float* k_scale, const float* v_scale,
                                   int32_t num_pages, int32_t page_size, int32_t num_heads, int32_t kv_heads,
                                   int32_t head_dim, const int32_t* block_table, int32_t max_pages_per_req,
                                   const int32_t* seq_lens, int32_t batch, int32_t tile_len, int32_t num_ctas,
                                   float sm_scale, void* workspace, size_t workspace_bytes, void* out,
                                   hpc_dtype out_dtype, float* lse, const hpc_step_options* options,
                                   uint32_t* status, void* stream) {
  if (!lse) return fail(HPC_ERR_ARG, "null pointer argument");
  return step_impl(q, k_pages, v_pages, kv_dtype, kv_layout, k_scale, v_scale, num_pages, page_size, num_heads,
                   kv_heads, head_dim, block_table, max_pages_per_req, seq_lens, batch, tile_len, num_ctas, sm_scale,
                   workspace, workspace_bytes, out, out_dtype, options, status, stream, nullptr, 1, lse);
}

extern "C" size_t hpc_decode_step_multi_workspace_bytes(int32_t batch, int32_t q_len, int32_t num_heads,
                                                        int32_t kv_heads, int32_t head_dim, int32_t num_ctas) {
  if (batch < 1 || q_len < 1 || num_heads < 1 || kv_heads < 1 || head_dim < 1 || num_ctas < 1 || num_heads % kv_heads)
    return 0;
  return step_layout(batch, num_heads / kv_heads, kv_heads, head_dim, num_ctas, q_len).total;
}

extern "C" int hpc_decode_step_multi(const void* q, int32_t q_len, const void* k_pages, const void* v_pages,
                                     hpc_dtype kv_dtype, hpc_kv_layout kv_layout, const float* k_scale,
                                     const float* v_scale, int32_t num_pages, int32_t page_size, int32_t num_heads,
                                     int32_t kv_heads, int32_t head_dim, const int32_t* block_table,
                                     int32_t max_pages_per_req, const int32_t* seq_lens, int32_t batch,
                                     int32_t tile_len, int32_t num_ctas, float sm_scale, void* workspace,
                                     size_t workspace_bytes, void* out, hpc_dtype out_dtype,
                                     const hpc_step_options* options, uint32_t* status, void* stream) {
  return step_impl(q, k_pages, v_pages, kv_dtype, kv_layout, k_scale, v_scale, num_pages, page_size, num_heads,
                   kv_heads, head_dim, block_table, max_pages_per_req, seq_lens, batch, tile_len, num_ctas, sm_scale,
                   workspace, workspace_bytes, out, out_dtype, options, status, stream, nullptr, q_len);
}

extern "C" int hpc_decode_step_prologue(const void* qkv, const float* q_norm_w, const float* k_norm_w, float eps,
                                        float rope_theta, void* k_pages, void* v_pages, hpc_dtype kv_dtype,
                                        hpc_kv_layout kv_layout, const float* k_scale, const float* v_scale,
                                        int32_t num_pages, int32_t page_size, int32_t num_heads, int32_t kv_heads,
                                        int32_t head_dim, const int32_t* block_table, int32_t max_pages_per_req,
                                        const int32_t* seq_lens, int32_t batch, int32_t tile_len, int32_t num_ctas,
                                        float sm_scale, void* workspace, size_t workspace_bytes, void* out,
                                        hpc_dtype out_dtype, const hpc_step_options* options, uint32_t* status,
                                        void* stream) {
  if (!qkv || !q_norm_w || !k_norm_w) return fail(HPC_ERR_ARG, "null pointer argument");
  if (!(rope_theta > 0.f) || !(eps >= 0.f)) return fail(HPC_ERR_ARG, "rope_theta must be > 0 and eps >= 0");
  const PrologueArgs pro{qkv, q_norm_w, k_norm_w, eps, rope_theta};
  return step_impl(qkv, k_pages, v_pages, kv_dtype, kv_layout, k_scale, v_scale, num_pages, page_size, num_heads,
                   kv_heads, head_dim, block_table, max_pages_per_req, seq_lens, batch, tile_len, num_ctas, sm_scale,
                   workspace, workspace_bytes, out, out_dtype, options, status, stream, &pro);
}
