/*
 * hpc_decode.h: C ABI of libhpcdecode.so, load-balanced split-KV decode attention for
 * B200 (sm_100a).
 *
 * One decode step runs four stages, all asynchronous on the caller's stream:
 *
 *   hpc_decode_prologue   (optional) RMSNorm + RoPE on the new token's q and k, and the
 *                         K/V page write of the new token;
 *   hpc_decode_plan       the per-step tile planner (a device kernel; no host sync);
 *   hpc_decode_attention  the persistent attention kernel; it consumes the plan;
 *   hpc_merge_states      the log-sum-exp merge of split (request, kv head) pairs.
 *
 * Sources: "Tencent HPC llega a SGLang y desafía a los kernels de inferencia
 * predeterminados" (remio.ai), section "Por qué Tencent HPC importa para el serving de
 * modelos en línea": uniform KV tiles spread over CTAs by current load, and a mapping
 * rebuilt as lengths change. "腾讯混元三算子杀入 SGLang" (AREX), Dynamic Attention
 * paragraph under "Router GEMM：精度不丢，速度翻三倍": a persistent kernel that assigns
 * tiles every decode step by actual KV length. "vLLM × HPC-Ops: High-Performance
 * Attention and MoE Backends from Tencent Hunyuan" (8sync News summary): a fused
 * RoPE + QK-Norm + KV-write prologue, and a dynamic scheduler that replaces fixed
 * split-KV.
 *
 * Conventions, for every entry point:
 *  - Ownership: the caller owns every buffer. Device pointers must point to memory of
 *    the current CUDA device. The library allocates no device memory and never
 *    synchronises the stream.
 *  - stream: a cudaStream_t passed as void* (NULL = legacy default stream).
 *  - Return value: hpc_status. A non-zero return means nothing was launched. Host-
 *    checkable problems are reported this way: null pointers, unsupported shapes or
 *    dtypes, misaligned pointers, too-small workspaces, launch failures.
 *    hpc_last_error() gives a message for the calling thread.
 *  - Device-detected problems are OR-ed into the caller's device word *status (uint32,
 *    HPC_DEV_* bits). These depend on data the host does not read: seq_lens, page
 *    ids, and wait timeouts. The kernels never trap. After a non-zero status the
 *    outputs of the affected requests are unspecified (but no out-of-bounds access
 *    happens). Clear *status before the step.
 *  - Cache layout: k_pages / v_pages are [num_pages][kv_heads][page_size][head_dim] (HPC_HND)
 *    or [num_pages][page_size][kv_heads][head_dim] (HPC_NHD), row-major, with elements bf16 or
 *    E4M3 codes. block_table is int32
 *    [batch][max_pages_per_req]. block_table[r][j] is the page that holds tokens
 *    [j*page_size, (j+1)*page_size) of request r. seq_lens is int32 [batch]: the number
 *    of valid tokens, including the one being decoded.
 *  - Query head h reads kv head h / (num_heads / kv_heads) (contiguous GQA groups).
 */
#ifndef HPC_DECODE_H_
#define HPC_DECODE_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define HPC_DECODE_ABI_VERSION 9

/* Symbols of the library are hidden by default; the entry points below are exported. */
#if defined(__GNUC__)
#define HPC_API __attribute__((visibility("default")))
#else
#define HPC_API
#endif

typedef enum {
  HPC_OK = 0,
  HPC_ERR_ARG = 1,      /* null pointer or out-of-range scalar argument */
  HPC_ERR_SHAPE = 2,    /* unsupported head_dim / page_size / tile_len / group size */
  HPC_ERR_DTYPE = 3,    /* unsupported dtype combination */
  HPC_ERR_ALIGN = 4,    /* a pointer is not 16-byte aligned */
  HPC_ERR_CUDA = 5,     /* a CUDA runtime/driver call failed */
  HPC_ERR_CAPACITY = 6  /* a caller buffer is smaller than required */
} hpc_status;

typedef enum { HPC_BF16 = 0, HPC_FP32 = 1, HPC_E4M3 = 2 } hpc_dtype;

/* Page layout of the KV cache.
 *   HPC_HND: [num_pages][kv_heads][page_size][head_dim]. One (page, kv head) block is contiguous.
 *   HPC_NHD: [num_pages][page_size][kv_heads][head_dim]. The vLLM paged-cache layout: the
 *            kv heads of one token are contiguous.
 * Both stream through the same TMA boxes: a box holds up to 64 tokens x 128 bytes of one kv
 * head, with the token stride given by the layout. */
typedef enum { HPC_HND = 0, HPC_NHD = 1 } hpc_kv_layout;

/* Bits the kernels OR into the caller's device status word. */
#define HPC_DEV_BAD_SEQLEN 0x1u /* seq_len < 0 or > max tokens; the request gets no tiles and a zero output */
#define HPC_DEV_BAD_PAGE 0x2u   /* a block_table entry outside [0, num_pages); no load is issued for that page
                                   and its tokens are left out of the request's softmax */
#define HPC_DEV_CAPACITY 0x4u   /* more work items than the plan can hold (cannot happen for a valid plan) */
#define HPC_DEV_TIMEOUT 0x8u    /* a bounded pipeline wait expired; the kernel gave up and returned */
#define HPC_DEV_BAD_INDEX 0x10u /* a row index outside its table (hpc_gather_rows, hpc_merge_lse_gather) */

/* One unit of a CTA's work: tiles [tile_begin, tile_end) of one (request, kv head). */
typedef struct {
  int32_t req;
  int16_t kv_head;
  int16_t flags; /* HPC_ITEM_DIRECT: the item covers its whole (req, kv_head); the attention
                    kernel writes the final output for it, with no partial state or merge */
  int32_t tile_begin;
  int32_t tile_end;
} hpc_work_item;

#define HPC_ITEM_DIRECT 1
/* Set only in hpc_cta_record items: the item's partial state goes to slot 2g + 1 of its CTA g
 * (without it, a non-DIRECT item uses slot 2g). */
#define HPC_ITEM_SECOND_SLOT 2

/* A plan is a host struct of device pointers into one caller-owned workspace. Layout:
 *   counts       int64[4]             n_items, n_merge, n_units, chunk (written on the device)
 *   items        hpc_work_item[max_items]
 *   cta_indptr   int32[num_ctas + 1]  CTA g owns items [cta_indptr[g], cta_indptr[g+1])
 *   merge_indptr int32[batch*kv_heads + 1]  items of segment s = r*kv_heads + kvh are
 *                                      [merge_indptr[s], merge_indptr[s+1]) (contiguous)
 *   merge_list   int32[batch*kv_heads] segments whose item count != 1 (first n_merge valid)
 * Item k writes partial slot k. */
typedef struct {
  int32_t batch, kv_heads, tile_len, num_ctas, max_items, merge_capacity, is_static, reserved;
  int64_t* counts;
  hpc_work_item* items;
  int32_t* cta_indptr;
  int32_t* merge_indptr;
  int32_t* merge_list;
} hpc_plan;

/* ---- per-call options (ABI 9) ----------------------------------------------------------- */

/* Record of one CTA's share of a single-launch step, written when a caller asks for it (tests,
 * debugging). CTA g writes the record at byte offset g * hpc_step_record_bytes(1, record_items):
 * this header, then min(n_items, record_items) hpc_work_item entries in the order the CTA ran
 * them. An entry's flags hold HPC_ITEM_DIRECT, or HPC_ITEM_SECOND_SLOT for a split item whose
 * partial state went to slot 2g + 1 (slot 2g without it). */
typedef struct {
  int64_t unit_begin, unit_end; /* the CTA's run [begin, end) of the request -> kv head -> tile units */
  int64_t chunk;                /* cost units per CTA of the split */
  int32_t item_cost;            /* cost of an item start used by the split, in 1/16 tile */
  int32_t n_items;              /* items the CTA ran */
} hpc_cta_record;

#define HPC_ITEM_COST_DEFAULT (-1)
#define HPC_ITEM_COST_MAX 1024
#define HPC_E4M3_MMA 0     /* E4M3 caches on the mma.sync consumers (the default) */
#define HPC_E4M3_TCGEN05 1 /* E4M3 caches on the tcgen05 kernel, where it applies */
#define HPC_MULTI_DEFAULT 0 /* several new tokens: the library's choice (see multi_kernel below) */
#define HPC_MULTI_MMA 1     /* several new tokens on the mma.sync consumers */
#define HPC_MULTI_TCGEN05 2 /* several new tokens on the tcgen05 kernel, where it applies */
#define HPC_TRACE_WORDS 8  /* uint64 words per CTA in a trace buffer */
#define HPC_BUILD_TRACE 1u /* hpc_build_flags(): the library was built with HPC_TRACE */

/* Options of one call. A NULL options pointer selects the defaults, as does a struct set from
 * HPC_STEP_OPTIONS_INIT (note that item_cost 0 is not the default). The library reads no
 * environment variables.
 *   item_cost:    single-launch steps only. The fixed cost of starting an item in the split of
 *                 units over CTAs, in 1/16 of a tile, 0 .. HPC_ITEM_COST_MAX. 0 splits by tiles
 *                 alone (exactly hpc_decode_plan's CTA ranges). HPC_ITEM_COST_DEFAULT: the time
 *                 one item start takes, as KV bytes a CTA streams meanwhile: 152 KB with one new
 *                 token; with several, 320 KB on the mma.sync consumers and 224 KB on the tcgen05
 *                 kernel; converted to tiles of the call's shape (rounded).
 *   e4m3_kernel:  HPC_E4M3_MMA or HPC_E4M3_TCGEN05. The tcgen05 kernel serves E4M3 caches with
 *                 head_dim 128 in hpc_decode_attention, hpc_decode_step and hpc_decode_step_lse;
 *                 elsewhere the choice is ignored.
 *   multi_kernel: HPC_MULTI_DEFAULT, HPC_MULTI_MMA or HPC_MULTI_TCGEN05: the kernel for
 *                 hpc_decode_step_multi with q_len > 1. The tcgen05 kernel serves bf16 caches with
 *                 head_dim 128 and q_len * (num_heads / kv_heads) <= 32; elsewhere the choice is
 *                 ignored. The default takes the tcgen05 kernel for q_len >= 3 where it applies
 *                 and the mma.sync consumers otherwise.
 *   record:       single-launch steps only: device buffer of hpc_step_record_bytes(num_ctas,
 *                 record_items) bytes that receives every CTA's hpc_cta_record, or NULL.
 *   trace:        device uint64 [num_ctas][HPC_TRACE_WORDS], or NULL. Only a library built with
 *                 HPC_TRACE (hpc_build_flags() & HPC_BUILD_TRACE) accepts it; the default build
 *                 returns HPC_ERR_ARG, and its kernels carry no trace code. Per CTA, from
 *                 %globaltimer (ns): [0] entry, [1] plan ready and the previous kernel on the
 *                 stream finished, [2] first stage consumed, [3] last item finished by the consumers,
 *                 [4] producer done; then [5] items, [6] pipeline stages, [7] SM id. Words [2]
 *                 and [3] stay 0 for a CTA without work. The mma.sync kernels and the
 *                 several-token tcgen05 kernel write it (the latter counts 128-token stages in
 *                 [6], filled by its K producer); with the E4M3 tcgen05 kernel a trace buffer
 *                 returns HPC_ERR_ARG.
 *   seq_lens_ready: single-launch steps only, 0 or 1. 1 promises that the kernel launched just
 *                 before this call on the stream does not write seq_lens (they were copied from
 *                 the host, or written earlier). The kernel then reads them and plans its split
 *                 while that kernel finishes (programmatic dependent launch), before it waits
 *                 for it; everything else (q, the cache, the block table, the outputs) is still
 *                 touched only after the wait. With 0 (the default) the plan follows the wait.
 *                 A step whose previous kernel writes seq_lens must pass 0: with 1 its split
 *                 would be planned on lengths being written, and its results are undefined. */
typedef struct {
  int32_t item_cost;
  int32_t e4m3_kernel;
  void* record;
  int32_t record_items;
  int32_t multi_kernel;
  uint64_t* trace;
  int32_t seq_lens_ready;
} hpc_step_options;

#define HPC_STEP_OPTIONS_INIT {HPC_ITEM_COST_DEFAULT, HPC_E4M3_MMA, NULL, 0, HPC_MULTI_DEFAULT, NULL, 0}

/* Bytes of a record buffer for num_ctas CTAs with record_items entries each. */
HPC_API size_t hpc_step_record_bytes(int32_t num_ctas, int32_t record_items);

/* Bit set of build options: HPC_BUILD_TRACE. */
HPC_API uint32_t hpc_build_flags(void);

/* ---- planning ------------------------------------------------------------------------ */

/* Bytes of workspace a dynamic plan needs (max_items = num_ctas + batch*kv_heads). */
HPC_API size_t hpc_plan_workspace_bytes(int32_t batch, int32_t kv_heads, int32_t num_ctas);

/* Bytes of workspace a static split-k plan needs (num_ctas = batch*kv_heads*splits). */
HPC_API size_t hpc_plan_static_workspace_bytes(int32_t batch, int32_t kv_heads, int32_t splits);

/* The load-balanced per-step planner (remio "Por qué …"; AREX Dynamic Attention paragraph).
 * It runs as one device kernel on `stream` and reads seq_lens from device memory.
 * For request r, nt_r = ceil(L_r / tile_len) tiles per kv head. Units are enumerated
 * request-major, then kv head, then tile: T units in total. With chunk = ceil(T / num_ctas),
 * CTA g owns units [g*chunk, min((g+1)*chunk, T)), cut into items at (request, kv head)
 * boundaries.
 *   seq_lens:    device int32 [batch].
 *   num_heads:   query heads; must be a multiple of kv_heads (checked only).
 *   tile_len:    tokens per tile, a multiple of 16.
 *   num_ctas:    persistent CTAs, normally (#SMs x resident CTAs per SM).
 *   max_seq_len: L_r above this (or below 0) sets HPC_DEV_BAD_SEQLEN and plans no tiles
 *                for r (<= 0: no upper check).
 *   workspace:   device buffer of >= hpc_plan_workspace_bytes(), 256-byte aligned.
 *   plan:        host struct filled with pointers into workspace. The attention and merge
 *                calls read it.
 *   status:      device uint32 status word. */
HPC_API int hpc_decode_plan(const int32_t* seq_lens, int32_t batch, int32_t num_heads, int32_t kv_heads,
                    int32_t tile_len, int32_t num_ctas, int32_t max_seq_len, void* workspace,
                    size_t workspace_bytes, hpc_plan* plan, uint32_t* status, void* stream);

/* Static split-k plan: the fixed split that remio ("Por qué …") describes as leaving units
 * idle or launching empty chunks for short requests. CTA (r*kv_heads + kvh)*splits + j takes
 * tiles [j*ceil(nt/splits), min((j+1)*ceil(nt/splits), nt)) of (r, kvh), possibly none.
 * num_ctas of the plan = batch*kv_heads*splits. The attention kernel runs it unchanged,
 * one launch wave per CTA group. Arguments as hpc_decode_plan. */
HPC_API int hpc_decode_plan_static(const int32_t* seq_lens, int32_t batch, int32_t num_heads, int32_t kv_heads,
                           int32_t tile_len, int32_t splits, int32_t max_seq_len, void* workspace,
                           size_t workspace_bytes, hpc_plan* plan, uint32_t* status, void* stream);

/* Host twin of hpc_decode_plan. It reads seq_lens from host memory and writes the same
 * bytes into a host buffer of hpc_plan_workspace_bytes(). *status is a host word.
 * plan receives host pointers. */
HPC_API int hpc_plan_cpu(const int32_t* seq_lens, int32_t batch, int32_t num_heads, int32_t kv_heads,
                 int32_t tile_len, int32_t num_ctas, int32_t max_seq_len, void* workspace,
                 size_t workspace_bytes, hpc_plan* plan, uint32_t* status);

/* ---- attention ----------------------------------------------------------------------- */

/* Bytes of partial state a plan needs: partial_o is float[max_items][group][head_dim],
 * partial_ml is float[max_items][group][2] (m, l). group = num_heads / kv_heads. */
HPC_API size_t hpc_partial_o_bytes(const hpc_plan* plan, int32_t num_heads, int32_t head_dim);
HPC_API size_t hpc_partial_ml_bytes(const hpc_plan* plan, int32_t num_heads);

/* Persistent split-KV decode attention (AREX Dynamic Attention paragraph).
 * grid = plan->num_ctas CTAs. Each CTA streams its items' KV pages through a shared-memory
 * ring filled by TMA, with tensor-core QK^T and PV on the GQA group.
 *   q:        device bf16 [batch][num_heads][head_dim].
 *   k_pages, v_pages: device cache, see the layouts above. kv_dtype is HPC_BF16 or HPC_E4M3,
 *             kv_layout HPC_HND or HPC_NHD. Base addresses must be 16-byte aligned.
 *   k_scale, v_scale: device float [kv_heads], required for HPC_E4M3 (value = code * scale),
 *             ignored for HPC_BF16.
 *   page_size: 16, 32, 64 or 128.  head_dim: 64 or 128 for bf16, 128 for E4M3.
 *   num_heads / kv_heads in {1, 2, 4, 8}.
 *   plan:     from hpc_decode_plan(_static) for the same seq_lens; its tile_len must be a
 *             multiple of page_size or divide it.
 *   sm_scale: score scale, normally 1/sqrt(head_dim).
 *   partial_o, partial_ml: device scratch of hpc_partial_*_bytes(). Non-DIRECT item k
 *             writes slot k with natural-log state m = max score, l = sum exp(s - m),
 *             o = sum exp(s - m) v.
 *   out:      device [batch][num_heads][head_dim], out_dtype HPC_FP32 or HPC_BF16. DIRECT
 *             items write it here; hpc_merge_states writes the rest.
 *   options:  NULL, or hpc_step_options: e4m3_kernel and trace apply here; item_cost must be
 *             HPC_ITEM_COST_DEFAULT and record NULL (they belong to the single-launch steps). */
HPC_API int hpc_decode_attention(const void* q, const void* k_pages, const void* v_pages, hpc_dtype kv_dtype,
                         hpc_kv_layout kv_layout, const float* k_scale, const float* v_scale, int32_t num_pages, int32_t page_size,
                         int32_t num_heads, int32_t kv_heads, int32_t head_dim, const int32_t* block_table,
                         int32_t max_pages_per_req, const int32_t* seq_lens, const hpc_plan* plan,
                         float sm_scale, float* partial_o, float* partial_ml, void* out,
                         hpc_dtype out_dtype, const hpc_step_options* options,
                                 uint32_t* status, void* stream);

/* ---- single-launch step ---------------------------------------------------------------- */

/* Bytes of workspace hpc_decode_step needs: batch*kv_heads int32 merge tickets, then
 * 2*num_ctas partial states (group*(head_dim+2) floats each), each part rounded up to 256. */
HPC_API size_t hpc_decode_step_workspace_bytes(int32_t batch, int32_t num_heads, int32_t kv_heads,
                                               int32_t head_dim, int32_t num_ctas);

/* One decode step in a single launch: the planner, the attention and the merge together.
 * This is the fewer-launches direction of the pages' own roadmap: "Tencent HPC llega a
 * SGLang …" (remio.ai), section "Tres señales …", lists megakernels; "vLLM × HPC-Ops"
 * describes PDL-chained stages.
 *  - Planning: each of the num_ctas persistent CTAs reads seq_lens and derives its own items
 *    with a closed form over the same tiles and unit order as hpc_decode_plan. The CTAs take
 *    contiguous unit runs of equal cost, where a tile costs 16 and each (request, kv head)
 *    segment start adds the fixed cost of an item: 152 KB worth of KV streaming with one new
 *    token (2.4 tiles of bf16 KV at tile_len 128, head_dim 128); with several, 320 KB on the
 *    mma.sync consumers and 224 KB on the tcgen05 kernel.
 *    options->item_cost (1/16 of a tile, 0 .. HPC_ITEM_COST_MAX) sets it per call; 0 assigns
 *    exactly hpc_decode_plan's ranges (ceil(T / num_ctas) units per CTA).
 *  - options: NULL for the defaults, or see hpc_step_options (item cost, E4M3 kernel, per-CTA
 *    record of the split, trace).
 *  - Merge: a split (request, kv head) is merged by the CTA that finishes its last piece. It
 *    finds out via an atomic ticket; there is no wait.
 *  - Requests with no tiles (L = 0, or an invalid length with HPC_DEV_BAD_SEQLEN) get a
 *    zero output.
 *  - Arguments as hpc_decode_attention, plus batch, tile_len and num_ctas. max_seq_len is
 *    max_pages_per_req * page_size.
 *  - workspace: device, 256-byte aligned, >= hpc_decode_step_workspace_bytes(). Its ticket
 *    part must be zero before the first call (e.g. cudaMemset the whole workspace once).
 *    Each call leaves it zero again. After a call that reported HPC_DEV_TIMEOUT, zero it
 *    again. Calls that overlap on the GPU must not share a workspace.
 *  - batch <= 4095 for head_dim 128 and <= 2047 for head_dim 64 (the per-request prefix is
 *    held in shared memory). Beyond that, HPC_ERR_SHAPE: use hpc_decode_plan. */
HPC_API int hpc_decode_step(const void* q, const void* k_pages, const void* v_pages, hpc_dtype kv_dtype,
                            hpc_kv_layout kv_layout, const float* k_scale, const float* v_scale, int32_t num_pages, int32_t page_size,
                            int32_t num_heads, int32_t kv_heads, int32_t head_dim, const int32_t* block_table,
                            int32_t max_pages_per_req, const int32_t* seq_lens, int32_t batch, int32_t tile_len,
                            int32_t num_ctas, float sm_scale, void* workspace, size_t workspace_bytes, void* out,
                            hpc_dtype out_dtype, const hpc_step_options* options,
                            uint32_t* status, void* stream);

/* hpc_decode_step with the decode prologue folded in ("vLLM × HPC-Ops" summary: "RoPE +
 * QK-Norm + KV-write" in front of attention). One launch does what hpc_decode_prologue followed
 * by hpc_decode_step does, without the q_out round trip through memory:
 *  - For each (request r, kv head) the CTA that owns its last tile writes request r's new token
 *    (position pos = seq_lens[r] - 1) into the cache for that kv head, with the arithmetic of
 *    hpc_decode_prologue: k through RMSNorm (k_norm_w, eps) and NeoX RoPE at pos, v as is, both
 *    as bf16 or E4M3 codes of x / scale. That CTA then reads the token back through its TMA
 *    stream; no other CTA reads it.
 *  - The attention query of every item is formed in registers from qkv: RMSNorm (q_norm_w),
 *    RoPE at pos (angles pos * theta^(-2i/D) evaluated in fp64), rounded to bf16.
 *  - qkv: device bf16 [batch][num_heads + 2*kv_heads][head_dim], 16-byte aligned.
 *    q_norm_w, k_norm_w: device float [head_dim]. eps >= 0, rope_theta > 0.
 *  - k_pages / v_pages are written (one token slot per request and kv head) and read.
 *  - seq_lens[r] must count the new token. seq_lens[r] = 0 sets HPC_DEV_BAD_SEQLEN (there is no
 *    token to decode) and gives a zero output row; a page id out of range sets
 *    HPC_DEV_BAD_PAGE and skips that write.
 *  - Everything else (workspace, batch limit, tickets) as hpc_decode_step. The rotated q is not
 *    written out. */
HPC_API int hpc_decode_step_prologue(const void* qkv, const float* q_norm_w, const float* k_norm_w, float eps,
                                     float rope_theta, void* k_pages, void* v_pages, hpc_dtype kv_dtype,
                                     hpc_kv_layout kv_layout, const float* k_scale, const float* v_scale,
                                     int32_t num_pages, int32_t page_size, int32_t num_heads, int32_t kv_heads,
                                     int32_t head_dim, const int32_t* block_table, int32_t max_pages_per_req,
                                     const int32_t* seq_lens, int32_t batch, int32_t tile_len, int32_t num_ctas,
                                     float sm_scale, void* workspace, size_t workspace_bytes, void* out,
                                     hpc_dtype out_dtype, const hpc_step_options* options,
                                     uint32_t* status, void* stream);

/* hpc_decode_step that also writes the log-sum-exp of every output row:
 *   lse[r][h] = log sum_j exp(sm_scale * q[r,h] . k_j)   (natural log; -inf when L_r = 0),
 * the quantity that combines outputs over disjoint parts of one request's keys (see
 * hpc_merge_lse). lse: device float [batch][num_heads]. Everything else as hpc_decode_step. */
HPC_API int hpc_decode_step_lse(const void* q, const void* k_pages, const void* v_pages, hpc_dtype kv_dtype,
                                hpc_kv_layout kv_layout, const float* k_scale, const float* v_scale, int32_t num_pages,
                                int32_t page_size, int32_t num_heads, int32_t kv_heads, int32_t head_dim,
                                const int32_t* block_table, int32_t max_pages_per_req, const int32_t* seq_lens,
                                int32_t batch, int32_t tile_len, int32_t num_ctas, float sm_scale, void* workspace,
                                size_t workspace_bytes, void* out, hpc_dtype out_dtype, float* lse, const hpc_step_options* options,
                                uint32_t* status,
                                void* stream);

/* Log-sum-exp merge of outputs computed over disjoint parts of the same keys (a request split
 * across GPUs in request-sharded placement; the pages describe the split of a request's tiles
 * across processing units but no merge step, so this extends the in-GPU merge to parts made
 * elsewhere). For each row r:
 *   LSE = log sum_i exp(lses[i][r]),   out[r] = sum_i exp(lses[i][r] - LSE) outs[i][r].
 * A row whose parts are all -inf gets zeros and -inf.
 *   outs: device float [parts][rows][head_dim]; lses: device float [parts][rows].
 *   out:  device float [rows][head_dim]; lse_out: device float [rows], or NULL. */
HPC_API int hpc_merge_lse(const float* outs, const float* lses, int32_t parts, int64_t rows, int32_t head_dim,
                          float* out, float* lse_out, void* stream);

/* The log-sum-exp merge with its parts found through an index, for a request-sharded batch:
 * the all-gathered parts of every rank are rows of outs / lses, and each request lists its
 * rows. For request r and head h, with p_k = part_index[r][k] over the k < max_parts where
 * p_k >= 0:
 *   LSE = log sum_k exp(lses[p_k][h]),  out[r][h][:] = sum_k exp(lses[p_k][h] - LSE) outs[p_k][h][:].
 * A request with one part gets that part's row exactly (weight exp(0) = 1); a request with
 * none gets zeros and LSE = -inf. An index >= part_rows is skipped and sets HPC_DEV_BAD_INDEX.
 *   outs:       device fp32 [part_rows][num_heads][head_dim]; lses: fp32 [part_rows][num_heads].
 *   part_index: device int32 [batch][max_parts], -1 for unused entries.
 *   out:        fp32 [batch][num_heads][head_dim]; lse_out: fp32 [batch][num_heads] or NULL.
 *   status:     device uint32 word or NULL.
 * One warp per (request, head); lanes split head_dim. */
HPC_API int hpc_merge_lse_gather(const float* outs, const float* lses, int64_t part_rows, const int32_t* part_index,
                                 int32_t max_parts, int32_t batch, int32_t num_heads, int32_t head_dim, float* out,
                                 float* lse_out, uint32_t* status, void* stream);

/* Row gather: dst[j] = src[index[j]] for j < n, rows of row_bytes bytes (a multiple of 16;
 * src and dst 16-byte aligned). A request-sharded rank uses it to collect the q rows of its
 * parts. An index outside [0, src_rows) gives a zero row and sets HPC_DEV_BAD_INDEX in
 * *status (device uint32, or NULL). */
HPC_API int hpc_gather_rows(const void* src, int64_t src_rows, int64_t row_bytes, const int32_t* index, int64_t n,
                            void* dst, uint32_t* status, void* stream);

/* Block-table view of the parts a request-sharded rank runs (each part is a page-aligned token
 * range of one request; see hpc_merge_lse_gather): row i of the view lists the pages of request
 * req[i] from column col0[i] on,
 *   dst[i][j] = src[req[i]][col0[i] + j]  for j < width and col0[i] + j < src_cols, else -1,
 * so that the rank's parts run as a batch of their own. Rebuilt every step on the device, it
 * follows pages the caller appends to the table as requests grow. A req[i] outside
 * [0, src_rows) or a negative col0[i] gives a row of -1 and sets HPC_DEV_BAD_INDEX.
 *   src: device int32 [src_rows][src_cols]; req, col0: device int32 [n];
 *   dst: device int32 [n][width]; status: device uint32 word or NULL. */
HPC_API int hpc_gather_pages(const int32_t* src, int32_t src_rows, int32_t src_cols, const int32_t* req,
                             const int32_t* col0, int32_t n, int32_t width, int32_t* dst, uint32_t* status,
                             void* stream);

/* ---- several new tokens per request ----------------------------------------------------- */

/* Bytes of workspace hpc_decode_step_multi needs: as hpc_decode_step_workspace_bytes, with
 * q_len * num_heads / kv_heads rows in each partial state. 0 for a bad shape. */
HPC_API size_t hpc_decode_step_multi_workspace_bytes(int32_t batch, int32_t q_len, int32_t num_heads,
                                                     int32_t kv_heads, int32_t head_dim, int32_t num_ctas);

/* hpc_decode_step for q_len new tokens per request, attending causally: speculative-decode
 * verification, or a chunked extend. The pages report the attention backend's effect on time
 * to first token ("vLLM × HPC-Ops" summary; remio.ai, "Por qué Tencent HPC importa …") but
 * do not describe a multi-token kernel; this entry point is the plainest extension of the
 * split-KV decode step to it. The planner is unchanged: KV tiles of a request do not depend
 * on how many queries read them.
 *  - q:   device bf16 [batch][q_len][num_heads][head_dim]. The q_len query tokens of request r
 *         are the last q_len of its seq_lens[r] cached tokens: query token t sits at position
 *         seq_lens[r] - q_len + t and attends to positions 0 .. seq_lens[r] - q_len + t.
 *  - out: device [batch][q_len][num_heads][head_dim], HPC_FP32 or HPC_BF16.
 *  - q_len: 1 to 4. Each consumer warp computes one query token's rows over its blocks of a
 *         stage; q_len 3 leaves one warp slot of four idle.
 *  - seq_lens[r] = 0 gives a zero output; 0 < seq_lens[r] < q_len sets HPC_DEV_BAD_SEQLEN and
 *         also gives zeros.
 *  - workspace: >= hpc_decode_step_multi_workspace_bytes(), zeroed once, as for
 *         hpc_decode_step. Everything else as hpc_decode_step. q_len = 1 is hpc_decode_step. */
HPC_API int hpc_decode_step_multi(const void* q, int32_t q_len, const void* k_pages, const void* v_pages,
                                  hpc_dtype kv_dtype, hpc_kv_layout kv_layout, const float* k_scale,
                                  const float* v_scale, int32_t num_pages, int32_t page_size, int32_t num_heads,
                                  int32_t kv_heads, int32_t head_dim, const int32_t* block_table,
                                  int32_t max_pages_per_req, const int32_t* seq_lens, int32_t batch,
                                  int32_t tile_len, int32_t num_ctas, float sm_scale, void* workspace,
                                  size_t workspace_bytes, void* out, hpc_dtype out_dtype, const hpc_step_options* options,
                                  uint32_t* status,
                                  void* stream);

/* ---- merge --------------------------------------------------------------------------- */

/* Log-sum-exp merge of the partial states of every (request, kv head) that the plan split
 * across items: M = max m_i, L = sum exp(m_i - M) l_i, out = sum exp(m_i - M) o_i / L.
 * A (request, kv head) with no items (L_r = 0) gets a zero output. Arguments as in
 * hpc_decode_attention. */
HPC_API int hpc_merge_states(const float* partial_o, const float* partial_ml, const hpc_plan* plan,
                     int32_t num_heads, int32_t head_dim, void* out, hpc_dtype out_dtype,
                     uint32_t* status, void* stream);

/* ---- prologue ------------------------------------------------------------------------ */

/* Fused decode prologue (vllm summary: "RoPE + QK-Norm + KV-write"). For each request r
 * with pos = seq_lens[r] - 1:
 *   q heads:  RMSNorm (q_norm_w, eps), then NeoX RoPE at pos (pairs (i, i+D/2),
 *             angle pos * theta^(-2i/D), computed in fp64), written as bf16 to q_out.
 *   k heads:  RMSNorm (k_norm_w), RoPE, then stored to page block_table[r][pos/page_size],
 *             slot pos % page_size (in kv_layout), as bf16 or as E4M3 code of x / k_scale[g]
 *             (RNE, saturating to +-448).
 *   v heads:  stored as is (bf16) or as E4M3 of v / v_scale[g].
 *   qkv:      device bf16 [batch][num_heads + 2*kv_heads][head_dim] (q heads, then k, then v).
 *   q_norm_w, k_norm_w: device float [head_dim].
 *   q_out:    device bf16 [batch][num_heads][head_dim].
 * seq_lens[r] < 1 or beyond the block table sets HPC_DEV_BAD_SEQLEN, and request r's
 * q_out row is zeroed. */
HPC_API int hpc_decode_prologue(const void* qkv, const float* q_norm_w, const float* k_norm_w, float eps,
                        float rope_theta, void* q_out, void* k_pages, void* v_pages, hpc_dtype kv_dtype,
                        hpc_kv_layout kv_layout,
                        const float* k_scale, const float* v_scale, int32_t num_pages, int32_t page_size,
                        const int32_t* block_table, int32_t max_pages_per_req, const int32_t* seq_lens,
                        int32_t batch, int32_t num_heads, int32_t kv_heads, int32_t head_dim,
                        uint32_t* status, void* stream);

/* ---- decode step without caller scratch ------------------------------------------------ */

/* Scratch held by the library for hpc_decode_step_noalloc: one static device array of this
 * many bytes. Every GPU that loads the library holds it until the process exits. */
#define HPC_NOALLOC_SCRATCH_BYTES (16u << 20)

/* The pages have no counterpart to this entry point. It is for callers that cannot call
 * cudaMalloc: code that runs inside a CUDA graph capture, serving loops that reserve all
 * device memory up front and must not stall (cudaMalloc can synchronise the device and can
 * fail under memory pressure), and plugins hosted by a framework whose allocator owns the
 * device memory.
 * It runs hpc_decode_plan, hpc_decode_attention and hpc_merge_states for one decode step.
 * The plan workspace and the partial states live in the library's static array of
 * HPC_NOALLOC_SCRATCH_BYTES; the caller passes only inputs (as in hpc_decode_attention, with
 * an HPC_HND cache, plus batch, tile_len and num_ctas) and outputs (out, status). It
 * allocates nothing.
 *  - Needed scratch = plan workspace + max_items*group*(head_dim+2)*4 bytes (each part
 *    rounded up to 256), with max_items = num_ctas + batch*kv_heads. A shape that needs
 *    more than HPC_NOALLOC_SCRATCH_BYTES returns HPC_ERR_CAPACITY and launches nothing.
 *  - All calls share the one array and leave its contents behind. Nothing in it has to
 *    start at zero. Calls that overlap on the GPU race: issue them on one stream, or
 *    order them.
 *  - The first call on a device (with that device current) looks up the array's device
 *    address and caches it. Make that first call before any stream capture begins. */
HPC_API int hpc_decode_step_noalloc(const void* q, const void* k_pages, const void* v_pages, hpc_dtype kv_dtype,
                                    const float* k_scale, const float* v_scale, int32_t num_pages, int32_t page_size,
                                    int32_t num_heads, int32_t kv_heads, int32_t head_dim, const int32_t* block_table,
                                    int32_t max_pages_per_req, const int32_t* seq_lens, int32_t batch,
                                    int32_t tile_len, int32_t num_ctas, float sm_scale, void* out,
                                    hpc_dtype out_dtype, uint32_t* status, void* stream);

/* ---- misc ---------------------------------------------------------------------------- */

/* Launch shape the attention kernel would use: pipeline stages, dynamic shared memory
 * bytes and threads per CTA. e4m3_kernel as in hpc_step_options. For introspection and
 * benchmarking. */
HPC_API int hpc_attention_launch_info(int32_t head_dim, hpc_dtype kv_dtype, int32_t page_size, int32_t tile_len,
                              int32_t ctas_per_sm, int32_t e4m3_kernel, int32_t* stages, int32_t* smem_bytes,
                              int32_t* threads);

/* Diagnostic of the bounded pipeline waits. Every wait in the library's kernels (stage
 * barriers, the new-token barrier, the final drain) gives up after a time limit, ORs
 * HPC_DEV_TIMEOUT into the status word and lets the kernel return; the library never
 * traps. This call runs that same wait in a one-warp kernel on a shared-memory barrier
 * phase:
 *   arrive != 0  the phase completes before the wait, which returns at once;
 *   arrive == 0  nothing completes it; the wait gives up after limit_ns and
 *                HPC_DEV_TIMEOUT is OR-ed into *status.
 * limit_ns: 1 .. 2e9 (the kernels' own limit is 2 s), else HPC_ERR_ARG.
 * status: device uint32 word (required). waited_ns: device uint64 (8-byte aligned) that
 * receives the wait's duration from %globaltimer, or NULL. Asynchronous on stream. */
HPC_API int hpc_wait_selftest(uint64_t limit_ns, int32_t arrive, uint32_t* status, uint64_t* waited_ns,
                              void* stream);

HPC_API const char* hpc_status_string(int status);
HPC_API const char* hpc_last_error(void); /* message of the calling thread's last failure ("" if none) */
HPC_API int hpc_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* HPC_DECODE_H_ */
