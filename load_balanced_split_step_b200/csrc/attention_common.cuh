// Device code shared by the attention kernels of libhpcdecode: kernel parameters, the work
// cursors (a materialised plan, or the planner's closed form walked in the kernel), the
// in-kernel plan prefix, the zero rows of empty requests and the ticket merge of split
// (request, kv head) segments. The mma.sync kernel (attention.cu) and the tcgen05 kernel for
// E4M3 caches (attention_tc.cu) both include it.
#pragma once

#include <math.h>
#include <stdlib.h>

#include "hpc_common.cuh"

namespace hpc {
namespace attn {

constexpr int kConsumerWarps = 8;
constexpr int kThreads = (kConsumerWarps + 1) * 32;
constexpr int kMaxStages = 16;
constexpr int kSmemLimit = 232448;  // 227 KB per block on sm_100
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
// Single-launch step: cost units per tile in the planner's split (item_cost is in the same units)
constexpr int64_t kCostPerTile = 16;
// The request prefix packs two sums: valid requests (nt > 0) above bit 44, tiles below it.
constexpr int kPreShift = 44;
constexpr int64_t kPreTiles = (int64_t(1) << kPreShift) - 1;

struct AttnParams {
  const __nv_bfloat16* q;
  const int32_t* block_table;
  const int32_t* seq_lens;
  const hpc_work_item* items;
  const int32_t* cta_indptr;
  const float* k_scale;
  const float* v_scale;
  float* partial_o;
  float* partial_ml;
  void* out;
  uint32_t* status;
  int64_t max_pages;
  int32_t num_pages, page_size, tile_len, chunk_tokens, num_heads, group;
  int32_t stages, out_bf16;
  uint32_t plane_bytes, stage_bytes;
  float score_scale;  // sm_scale * log2(e)
  int32_t q_len;      // new tokens per request (single-launch step); 1 elsewhere
  float* lse;         // optional [batch][num_heads]: natural log of sum_j exp(score_j) (one-token step)
  int32_t nhd;        // cache layout: token stride Hkv*D (NHD) or D (HND); only the TMA coordinates differ
  // single-launch step only: the plan is derived in the kernel from seq_lens
  int32_t batch, kv_heads, max_seq_len;
  int32_t* tickets;  // [batch * kv_heads], zero between steps
  int32_t item_cost;  // cost of starting an item, in 1/kCostPerTile of a tile (0: split by tiles alone)
  int32_t plan_early;  // seq_lens are not the previous kernel's output: plan before waiting for it
  // single-launch step with the prologue folded in: q comes from qkv through RMSNorm and RoPE,
  // and the new token's K/V are written into the cache
  const __nv_bfloat16* qkv;  // [batch][num_heads + 2 kv_heads][D]
  const float* q_norm_w;
  const float* k_norm_w;
  void* k_pages_w;  // the caches, for the new token's write
  void* v_pages_w;
  float eps;
  double rope_theta;
  // single-launch step, on request: each CTA's record of its split (hpc_cta_record + items)
  uint8_t* record;
  int32_t record_items;
  uint64_t* trace;  // HPC_TRACE builds: [grid][HPC_TRACE_WORDS] timestamps and counts
};

// Byte stride of one CTA's record: the header, then record_items work items.
__host__ __device__ __forceinline__ size_t record_stride(int record_items) {
  return sizeof(hpc_cta_record) + static_cast<size_t>(record_items) * sizeof(hpc_work_item);
}

// One work item as the producer and the consumers see it.
struct ItemInfo {
  int32_t req, kvh;
  int64_t tok0, tok1;  // tokens to stream
  bool direct;         // covers its whole (request, kv head): writes the output itself
  int64_t slot;        // partial-state slot of a split item
  int64_t U;           // single-launch step: first unit of the (request, kv head) segment,
  int32_t nt;          // its tile count
  int64_t S;           // and its 1-based index among the segments that have tiles
};

// 16-token blocks that one consumer warp takes from a stage of `bpc` blocks. Two blocks give
// two independent MMA chains. An E4M3 stage carries half the bytes per token, so the fixed
// per-call softmax work (row max across lanes, rescale factors) and the stage handshake weigh
// twice as much per byte: there a warp takes up to four blocks, a whole 64-token stage. With
// several new tokens on a bf16 cache a warp also takes four: the stage then needs q_pad warps
// instead of 2 q_pad, so two stages are consumed at once instead of one, and each warp has four
// independent chains (on the heavy-tailed batch with four new tokens: 1055 -> 590 us).
__host__ __device__ __forceinline__ int blocks_per_warp(int bpc, bool fp8, int q_pad = 1) {
  if (bpc >= 4 && (fp8 ? q_pad == 1 : q_pad > 1)) return 4;
  return bpc >= 2 ? 2 : 1;
}

// Several new tokens per request: q_len query tokens take q_pad = 1, 2 or 4 warp slots of each
// stage (q_len 3 leaves one slot idle). Each warp computes one query token's rows over its
// blocks, so a stage is read by (blocks per stage / blocks per warp) * q_pad warps.
__host__ __device__ __forceinline__ int q_pad_of(int q_len) { return q_len <= 1 ? 1 : (q_len <= 2 ? 2 : 4); }

__device__ __forceinline__ int32_t tiles_of(int32_t L, int32_t tl) {
  return L > 0 ? static_cast<int32_t>(static_cast<uint32_t>(L - 1) / static_cast<uint32_t>(tl) + 1) : 0;
}

// A length is valid when it is 0 (no tiles, zero output) or holds the step's q_len new tokens
// and fits the block table.
__device__ __forceinline__ bool len_ok(int32_t L, int32_t max_seq_len, int32_t q_len = 1) {
  return L >= 0 && (L == 0 || L >= q_len) && (max_seq_len <= 0 || L <= max_seq_len);
}

template <int D, bool FP8>
struct Shape {
  static constexpr int kElt = FP8 ? 1 : 2;
  static constexpr int kPlanes = D * kElt / 128;  // 128-byte swizzle planes per token row
  static constexpr int kRedStride = D;  // floats per (warp, head) row; columns XOR 4h against bank conflicts
};

// Output row index of accumulator register `half` (0: c0/c1, 1: c2/c3) for lane row g
// inside a 16-row block. bf16 V comes from ldmatrix.trans in natural order (rows g, g+8).
// E4M3 V comes from ldmatrix.trans on byte pairs, so rows g and g+8 hold d = 2g and 2g+1.
template <bool FP8>
__device__ __forceinline__ int out_row(int g, int half) {
  if (FP8) return 2 * g + half;
  return g + 8 * half;
}

// One past the last token of an item: its last tile, clipped to the request length and to
// what the block table can address (a plan built for other lengths cannot read past it).
__device__ __forceinline__ int64_t item_end(const hpc_work_item& w, int32_t L, int tl, int64_t capacity) {
  int64_t e = static_cast<int64_t>(w.tile_end) * tl;
  if (e > L) e = L;
  if (e > capacity) e = capacity;
  return e;
}

// Items of one CTA, read from a device plan (hpc_decode_plan / hpc_decode_plan_static).
struct PlanCursor {
  int it, it_end;
  __device__ bool next(const AttnParams& p, ItemInfo& x) {
    if (it >= it_end) return false;
    const hpc_work_item w = p.items[it];
    x.req = w.req;
    x.kvh = w.kv_head;
    x.tok0 = static_cast<int64_t>(w.tile_begin) * p.tile_len;
    x.tok1 = item_end(w, p.seq_lens[w.req], p.tile_len, p.max_pages * p.page_size);
    x.direct = (w.flags & HPC_ITEM_DIRECT) != 0;
    x.slot = it;
    x.U = 0;
    x.nt = 0;
    x.S = 0;
    ++it;
    return true;
  }
};

// Items of one CTA, derived in the kernel by the planner's closed form: the CTA owns units
// [u, u_end) of the request -> kv head -> tile enumeration and cuts them at (request, kv head)
// boundaries. A split (request, kv head) is always this CTA's first or last item, so two
// partial slots per CTA suffice: 2g for a piece that starts at the CTA's first unit, 2g + 1
// otherwise. V counts the requests with tiles before r, which numbers the segments.
struct WalkCursor {
  int64_t u, u_end, u_first, U_r, V;
  int32_t r, kvh, nt, tb, g;
  __device__ bool next(const AttnParams& p, ItemInfo& x) {
    if (u >= u_end) return false;
    const int32_t te = static_cast<int32_t>(min(static_cast<int64_t>(nt), tb + (u_end - u)));
    const int32_t L = p.seq_lens[r];
    x.req = r;
    x.kvh = kvh;
    x.tok0 = static_cast<int64_t>(tb) * p.tile_len;
    int64_t e = static_cast<int64_t>(te) * p.tile_len;
    if (e > L) e = L;
    x.tok1 = e;
    x.direct = tb == 0 && te == nt;
    x.slot = 2 * static_cast<int64_t>(g) + (u == u_first ? 0 : 1);
    x.U = U_r + static_cast<int64_t>(kvh) * nt;
    x.nt = nt;
    x.S = V * p.kv_heads + kvh + 1;
    u += te - tb;
    tb = 0;
    if (u < u_end) {  // step to the next (request, kv head) with tiles
      if (++kvh == p.kv_heads) {
        kvh = 0;
        ++V;
        U_r += static_cast<int64_t>(p.kv_heads) * nt;
        do {
          ++r;
          const int32_t Ln = p.seq_lens[r];
          nt = len_ok(Ln, p.max_seq_len, p.q_len) ? tiles_of(Ln, p.tile_len) : 0;
        } while (nt == 0);
      }
    }
    return true;
  }
};

template <bool FUSED>
struct CursorOf {
  using type = PlanCursor;
};
template <>
struct CursorOf<true> {
  using type = WalkCursor;
};

// The k-th item of CTA g's record (single-launch step, when a record buffer is given): the item
// as the planner would list it, with HPC_ITEM_SECOND_SLOT for a split item in slot 2g + 1.
__device__ __forceinline__ void record_item(const AttnParams& p, int64_t k, const ItemInfo& x) {
  if (k >= p.record_items) return;
  hpc_work_item w;
  w.req = x.req;
  w.kv_head = static_cast<int16_t>(x.kvh);
  w.flags = static_cast<int16_t>(x.direct ? HPC_ITEM_DIRECT : ((x.slot & 1) ? HPC_ITEM_SECOND_SLOT : 0));
  w.tile_begin = static_cast<int32_t>(x.tok0 / p.tile_len);
  // tok1 = min(te * tile_len, L), and only the segment's last tile is clipped: te = ceil(tok1 / tile_len)
  w.tile_end = static_cast<int32_t>((x.tok1 + p.tile_len - 1) / p.tile_len);
  uint8_t* rec = p.record + static_cast<size_t>(blockIdx.x) * record_stride(p.record_items);
  reinterpret_cast<hpc_work_item*>(rec + sizeof(hpc_cta_record))[k] = w;
}

// CTA g's record header: its unit run, the chunk and cost of the split, and its item count.
__device__ __forceinline__ void record_header(const AttnParams& p, int64_t u0, int64_t u1, int64_t chunk,
                                              int64_t n_items) {
  hpc_cta_record h;
  h.unit_begin = u0;
  h.unit_end = u1;
  h.chunk = chunk;
  h.item_cost = p.item_cost;
  h.n_items = static_cast<int32_t>(n_items);
  *reinterpret_cast<hpc_cta_record*>(p.record + static_cast<size_t>(blockIdx.x) * record_stride(p.record_items)) = h;
}

// Where the single-launch step's split puts a unit. Unit u (tile t of segment S, the S-th
// (request, kv head) with tiles, 1-based) sits at cost position W*u + c*S: every tile costs
// W = kCostPerTile and every segment start adds c = item_cost, the fixed cost of an item
// (its combine, partial write, ticket and merge, and the next item's first loads). CTA g owns
// the units whose positions fall in [g*chunk, (g+1)*chunk), chunk = W * ceil(total / (W*G)).
// With c = 0 this is the pages' rule: chunk / W = ceil(T / G) units per CTA.
__device__ __forceinline__ int64_t unit_pos(int64_t u, int64_t S, int64_t c) { return kCostPerTile * u + c * S; }

// CTAs that own the first and the last tile of an item's segment, and the partial slot of the
// segment's first piece (2 g1 when the segment starts CTA g1's range, 2 g1 + 1 otherwise).
// Every CTA between g1 and g2 owns at least one tile of the segment (chunk >= W), so the
// segment has g2 - g1 + 1 pieces, and the piece in CTA g1 + i (i >= 1) is in slot 2 (g1 + i).
__device__ __forceinline__ void segment_ctas(const ItemInfo& x, int64_t c, int64_t chunk, int64_t& g1, int64_t& g2,
                                             int64_t& first_slot) {
  const int64_t p_first = unit_pos(x.U, x.S, c);
  g1 = p_first / chunk;
  g2 = (p_first + kCostPerTile * (x.nt - 1)) / chunk;
  // the unit before the segment is the last tile of segment S - 1
  const bool starts_cta = x.U == 0 || unit_pos(x.U - 1, x.S - 1, c) / chunk != g1;
  first_slot = starts_cta ? 2 * g1 : 2 * g1 + 1;
}

// Single-launch step: each CTA finds its unit range. It forms the exclusive prefix sums of
// per-request tile counts and of requests with tiles (packed in one int64, kPreShift) in
// shared memory (the reduce buffer, unused until the first item ends) and binary-searches
// them. Requests with no valid tiles get a zero output from CTA r % num_ctas. Returns the
// walk cursor (all threads get the same one) and the split's chunk in cost units.
template <int D>
__device__ void plan_in_kernel(const AttnParams& p, int64_t* s_pre, int64_t* s_scan, int64_t* s_walk,
                               WalkCursor& cur, int64_t& chunk) {
  const int tid = threadIdx.x, nthr = blockDim.x;
  const int B = p.batch, Hkv = p.kv_heads, G = gridDim.x, g = blockIdx.x;
  // per-thread contiguous run of requests, then a block scan of the run totals
  const int per = (B + nthr - 1) / nthr;
  const int r0 = min(B, tid * per), r1 = min(B, r0 + per);
  int64_t run = 0;
  uint32_t bad = 0;
  for (int r = r0; r < r1; ++r) {
    const int32_t L = p.seq_lens[r];
    const bool ok = len_ok(L, p.max_seq_len, p.q_len);
    if (!ok) bad |= HPC_DEV_BAD_SEQLEN;
    const int32_t nt = ok ? tiles_of(L, p.tile_len) : 0;
    run += nt > 0 ? (int64_t(1) << kPreShift) + nt : 0;
  }
  if (bad && (r0 % G) == g) atomicOr(p.status, bad);
  const int lane = tid & 31, warp = tid >> 5, nwarps = (nthr + 31) >> 5;
  int64_t x = run;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int64_t y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) s_scan[warp] = x;
  __syncthreads();
  if (tid == 0) {
    int64_t acc = 0;
    for (int w = 0; w < nwarps; ++w) {
      const int64_t t = s_scan[w];
      s_scan[w] = acc;
      acc += t;
    }
    s_scan[nwarps] = acc;
  }
  __syncthreads();
  int64_t pre = s_scan[warp] + x - run;
  for (int r = r0; r < r1; ++r) {
    s_pre[r] = pre;
    const int32_t L = p.seq_lens[r];
    const int32_t nt = len_ok(L, p.max_seq_len, p.q_len) ? tiles_of(L, p.tile_len) : 0;
    pre += nt > 0 ? (int64_t(1) << kPreShift) + nt : 0;
  }
  if (tid == 0) s_pre[B] = s_scan[nwarps];
  __syncthreads();
  if (tid == 0) {
    auto tiles = [&](int i) -> int64_t { return s_pre[i] & kPreTiles; };
    auto valid = [&](int i) -> int64_t { return s_pre[i] >> kPreShift; };
    const int64_t c = p.item_cost, W = kCostPerTile;
    const int64_t T = tiles(B) * Hkv;
    const int64_t total = W * T + c * valid(B) * Hkv;
    const int64_t ch = T > 0 ? W * ((total + W * G - 1) / (W * G)) : 0;
    // first unit whose cost position is >= P (T if none)
    auto first_unit_at = [&](int64_t P) -> int64_t {
      if (T == 0 || P <= 0) return 0;
      if (P > unit_pos(T - 1, valid(B) * Hkv, c)) return T;
      // largest r whose cost prefix is <= P: the request whose segments hold position P
      auto cost_pre = [&](int i) -> int64_t { return (W * tiles(i) + c * valid(i)) * Hkv; };
      int lo = 0, hi = B - 1;
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (cost_pre(mid) <= P) lo = mid;
        else hi = mid - 1;
      }
      const int64_t nt = tiles(lo + 1) - tiles(lo), seg = c + W * nt;
      const int64_t off = P - cost_pre(lo), kv = off / seg, o = off - kv * seg;
      const int64_t t = o <= c ? 0 : min(nt, (o - c + W - 1) / W);  // nt: the next segment's first unit
      return tiles(lo) * Hkv + kv * nt + t;
    };
    const int64_t u0 = first_unit_at(static_cast<int64_t>(g) * ch);
    const int64_t u1 = max(u0, first_unit_at(static_cast<int64_t>(g + 1) * ch));
    int64_t r = 0, kvh = 0, tb = 0, nt = 0, U_r = 0;
    if (u0 < T) {
      // largest r with Hkv * tiles(r) <= u0: the request that holds unit u0
      int lo = 0, hi = B - 1;
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (tiles(mid) * Hkv <= u0) lo = mid;
        else hi = mid - 1;
      }
      r = lo;
      nt = tiles(r + 1) - tiles(r);
      U_r = tiles(r) * Hkv;
      kvh = (u0 - U_r) / nt;
      tb = u0 - U_r - kvh * nt;
    }
    s_walk[0] = u0;
    s_walk[1] = u1;
    s_walk[2] = U_r;
    s_walk[3] = r;
    s_walk[4] = kvh;
    s_walk[5] = nt;
    s_walk[6] = tb;
    s_walk[7] = ch;
    s_walk[8] = u0 < T ? valid(static_cast<int>(r)) : 0;
  }
  __syncthreads();
  cur.u = s_walk[0];
  cur.u_first = s_walk[0];
  cur.u_end = s_walk[1];
  cur.U_r = s_walk[2];
  cur.r = static_cast<int32_t>(s_walk[3]);
  cur.kvh = static_cast<int32_t>(s_walk[4]);
  cur.nt = static_cast<int32_t>(s_walk[5]);
  cur.tb = static_cast<int32_t>(s_walk[6]);
  cur.V = s_walk[8];
  cur.g = g;
  chunk = s_walk[7];
}

// Zero output rows of requests that own no tiles (L = 0 or an invalid length).
template <int D>
__device__ void zero_empty_requests(const AttnParams& p, int tid, int nthr) {
  for (int r = blockIdx.x; r < p.batch; r += gridDim.x) {
    const int32_t L = p.seq_lens[r];
    if (len_ok(L, p.max_seq_len, p.q_len) && L > 0) continue;
    const int64_t rows = static_cast<int64_t>(p.q_len) * p.num_heads * D;
    const int64_t base = static_cast<int64_t>(r) * rows;
    if (p.lse)
      for (int h = tid; h < p.num_heads; h += nthr) p.lse[static_cast<int64_t>(r) * p.num_heads + h] = -INFINITY;
    for (int64_t i = tid; i < rows; i += nthr) {
      if (p.out_bf16) reinterpret_cast<__nv_bfloat16*>(p.out)[base + i] = __float2bfloat16_rn(0.f);
      else reinterpret_cast<float*>(p.out)[base + i] = 0.f;
    }
  }
}

// Log-sum-exp merge of a split (request, kv head) by the CTA that finished its last piece.
// Piece slots follow the walk cursor's rule: the piece in CTA gg is slot 2gg, except the first
// piece when it starts inside CTA g1's range (slot 2 g1 + 1). All (piece, head) states are
// loaded at once into shared memory (the reduce buffer, free at this point) and turned into
// weights exp(m_i - M) / L. The output is then a weighted sum over independent loads. The
// other CTAs' partial states are read through L2 (ld.global.cg) after the ticket's fence.
template <int D>
__device__ void merge_segment(const AttnParams& p, const ItemInfo& x, int64_t chunk, int tid, int nthr,
                              float* s_buf, int buf_floats) {
  int64_t g1, g2, first_slot;
  segment_ctas(x, p.item_cost, chunk, g1, g2, first_slot);
  // rows of a piece: query token t, head h -> row t * group + h
  const int grp = p.group * p.q_len;
  const int n = static_cast<int>(g2 - g1 + 1);
  auto slot_of = [&](int i) -> int64_t { return i == 0 ? first_slot : 2 * (g1 + i); };
  auto out_at = [&](int idx) -> int64_t {  // idx = row * D + d
    const int row = idx / D, t = row / p.group, h = row - t * p.group;
    return ((static_cast<int64_t>(x.req) * p.q_len + t) * p.num_heads + x.kvh * p.group + h) * D + (idx - row * D);
  };
  float* s_m = s_buf;
  float* s_w = s_buf + n * grp;
  float* s_M = s_w + n * grp;
  float* s_iL = s_M + grp;
  if (2 * n * grp + 2 * grp <= buf_floats) {
    for (int k = tid; k < n * grp; k += nthr) {
      const int i = k / grp, h = k - i * grp;
      const float* ml = p.partial_ml + 2 * (slot_of(i) * grp + h);
      s_m[k] = __ldcg(ml);
      s_w[k] = __ldcg(ml + 1);
    }
    named_barrier_sync(1, nthr);
    if (tid < grp) {
      float M = -INFINITY;
      for (int i = 0; i < n; ++i) M = fmaxf(M, s_m[i * grp + tid]);
      float L = 0.f;
      for (int i = 0; i < n && M != -INFINITY; ++i) L += expf(s_m[i * grp + tid] - M) * s_w[i * grp + tid];
      s_M[tid] = M;
      s_iL[tid] = L > 0.f ? 1.f / L : 0.f;
      if (p.lse) {  // one new token per request: row tid is head kvh * group + tid
        p.lse[static_cast<int64_t>(x.req) * p.num_heads + x.kvh * p.group + tid] = L > 0.f ? M + logf(L) : -INFINITY;
      }
    }
    named_barrier_sync(1, nthr);
    for (int k = tid; k < n * grp; k += nthr) {
      const int h = k % grp;
      s_w[k] = s_iL[h] > 0.f ? expf(s_m[k] - s_M[h]) * s_iL[h] : 0.f;  // no live piece: zeros
    }
    named_barrier_sync(1, nthr);
    for (int idx = tid; idx < grp * D; idx += nthr) {
      const int h = idx / D;
      float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
      int i = 0;
      for (; i + 4 <= n; i += 4) {
        a0 += s_w[(i + 0) * grp + h] * __ldcg(p.partial_o + slot_of(i + 0) * grp * D + idx);
        a1 += s_w[(i + 1) * grp + h] * __ldcg(p.partial_o + slot_of(i + 1) * grp * D + idx);
        a2 += s_w[(i + 2) * grp + h] * __ldcg(p.partial_o + slot_of(i + 2) * grp * D + idx);
        a3 += s_w[(i + 3) * grp + h] * __ldcg(p.partial_o + slot_of(i + 3) * grp * D + idx);
      }
      for (; i < n; ++i) a0 += s_w[i * grp + h] * __ldcg(p.partial_o + slot_of(i) * grp * D + idx);
      const float val = (a0 + a1) + (a2 + a3);
      if (p.out_bf16) reinterpret_cast<__nv_bfloat16*>(p.out)[out_at(idx)] = __float2bfloat16_rn(val);
      else reinterpret_cast<float*>(p.out)[out_at(idx)] = val;
    }
    return;
  }
  // more pieces than the buffer holds: two passes over the partial states per output
  for (int idx = tid; idx < grp * D; idx += nthr) {
    const int h = idx / D;
    float M = -INFINITY;
    for (int i = 0; i < n; ++i) M = fmaxf(M, __ldcg(p.partial_ml + 2 * (slot_of(i) * grp + h)));
    float Ls = 0.f, acc = 0.f;
    for (int i = 0; i < n && M != -INFINITY; ++i) {
      const int64_t pi = slot_of(i) * grp + h;
      const float e = expf(__ldcg(p.partial_ml + 2 * pi) - M);
      Ls += e * __ldcg(p.partial_ml + 2 * pi + 1);
      acc += e * __ldcg(p.partial_o + pi * D + (idx - h * D));
    }
    const float val = Ls > 0.f ? acc / Ls : 0.f;
    if (p.out_bf16) reinterpret_cast<__nv_bfloat16*>(p.out)[out_at(idx)] = __float2bfloat16_rn(val);
    else reinterpret_cast<float*>(p.out)[out_at(idx)] = val;
    if (p.lse && idx - h * D == 0)
      p.lse[static_cast<int64_t>(x.req) * p.num_heads + x.kvh * p.group + h] = Ls > 0.f ? M + logf(Ls) : -INFINITY;
  }
}

// The tcgen05 kernel for E4M3 caches (attention_tc.cu). It serves the one-token single-launch
// step and the three-launch attention when the cache is E4M3, head_dim is 128 and the group is
// at most 8 heads. Returns an hpc_status.
bool tc_supported(int head_dim, bool fp8, int group, int q_len, bool pro);
int tc_smem_bytes(int ctas_per_sm);
int tc_threads();
int launch_attention_tc(bool fused, const CUtensorMap& mk, const CUtensorMap& mv, const AttnParams& prm, int grid,
                        cudaStream_t stream);

// The tcgen05 kernel for several new tokens per request on a bf16 cache (attention_tcm.cu): the
// single-launch step only, head_dim 128, q_len * group <= 32.
bool tcm_supported(int head_dim, bool fp8, int group, int q_len, bool pro);
int launch_attention_tcm(const CUtensorMap& mk, const CUtensorMap& mv, const AttnParams& prm, int grid,
                         cudaStream_t stream);

}  // namespace attn
}  // namespace hpc
