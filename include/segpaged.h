/*
 * segpaged.h — C ABI of libsegpaged.so, head-aware paged KV attention
 * (SegPagedAttention) for NVIDIA B200 (sm_100a).
 *
 * The KV cache is paged per (sequence, kv-head, segment).  Every kv-head
 * follows its own policy: a GLOBAL head stores and reads its whole causal
 * context; a LOCAL head stores and reads only the first `sink` tokens of the
 * sequence plus its `window` most recent tokens.  Attention evaluates every
 * (query-head, kv-head) pair over exactly the tokens that head stores, with no
 * mask over tokens it cannot see ("SegPagedAttention runtime design", §1 why
 * heads see different contexts, §3 per-head page tables, §4 mask-free fused
 * kernel; "RedKnot head classification", four head kinds).
 *
 * Conventions shared by every call:
 *  - Device memory (K/V pools, the table blob, workspace, Q/K/V/O tensors) is
 *    owned by the caller.  Pointers are borrowed for the duration of the call.
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *    stream).  Device calls only enqueue work and return; nothing synchronises
 *    except segpaged_read_device_status.
 *  - Every argument and layout error is detected on the host before any launch
 *    and leaves every output untouched.  No C++ exception crosses the ABI.
 *    segpaged_last_error() returns a message for the calling thread's last
 *    failure.
 *  - Positions are 0-based absolute positions in a sequence.  Query q-head h
 *    uses kv-head h / (num_q_heads / num_kv_heads).
 *  - Supported: head_dim 64 or 128; dtype fp32 with page size 16 or 64; dtype
 *    bf16 with page size 64 (pages bf16, or FP8 E4M3 for decode plans);
 *    num_q_heads / num_kv_heads <= 16.  Anything else returns
 *    SP_ERR_UNSUPPORTED.  bf16 pages are 64 tokens only: the kernels stage a
 *    page as one 128-byte-swizzled tensor-core operand of 64 rows (the pages'
 *    own runtime uses page size 64, "SegPagedAttention runtime design", §6).
 */
#ifndef SEGPAGED_H_
#define SEGPAGED_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define SP_API __attribute__((visibility("default")))
#else
#define SP_API
#endif

#define SEGPAGED_ABI_VERSION 2

/* stride_seq value selecting sequences packed back to back (varlen). */
#define SP_VARLEN (-1)

typedef enum {
  SP_OK = 0,
  SP_ERR_INVALID_ARG = 1,  /* malformed sizes, positions, policies, pointers or strides */
  SP_ERR_UNSUPPORTED = 2,  /* valid request outside the supported shapes / kinds / dtypes */
  SP_ERR_WORKSPACE = 3,    /* table or workspace buffer smaller than the plan needs */
  SP_ERR_CUDA = 4,         /* a CUDA runtime call or launch failed */
  SP_ERR_DEVICE_CHECK = 5  /* a kernel recorded an error in the workspace status word */
} sp_status;

/* Head kinds ("RedKnot head classification", four-kind table).  DENSE reads
 * the full causal context like GLOBAL (its RoPE re-alignment belongs to KV
 * reuse, outside attention).  RETRIEVAL has the whole context as candidates
 * but keeps only its top-p important tokens, fetched page by page (same
 * table; "SegPagedAttention runtime design", closing summary: retrieval heads
 * fetch pages on demand).  The pages give no scoring rule; this library's
 * reading: the caller gives an importance per block of page_size positions
 * (sp_problem.block_mass, e.g. the head's attention mass per page); the head
 * keeps its first `sink` tokens and its `window` most recent tokens, like a
 * LOCAL head, plus the fewest blocks that, taken in decreasing importance
 * (ties: the lower block first), reach the fraction top_p of the total
 * importance of the candidate blocks (those holding a position >= sink); sums
 * run in fp64 in that order.  top_p >= 1 keeps every block (the head is then
 * GLOBAL), top_p <= 0 none (LOCAL).  A query at position p sees the kept
 * blocks' positions up to p, the sink and its window. */
typedef enum { SP_GLOBAL = 0, SP_LOCAL = 1, SP_DENSE = 2, SP_RETRIEVAL = 3 } sp_kind;

/* SP_E4M3 is a page type only (sp_problem.kv_dtype): FP8 E4M3 codes, 1 byte. */
typedef enum { SP_F32 = 0, SP_BF16 = 1, SP_E4M3 = 2 } sp_dtype;

/* Problem flags. */
enum {
  /* Dense-plus-mask baseline: every head stores its whole context [0, L) and
   * the kernels visit every causal tile, masking LOCAL heads per element
   * ("SegPagedAttention runtime design", §4 verify_against_dense and §5: the
   * dense baseline the speedups are quoted against). */
  SP_FLAG_DENSE_MASKED = 1u,
  /* Ring plan (decode plans only): every page holds positions aligned to
   * multiples of page_size; a LOCAL head's recent window lives in a ring of
   * ceil(window / page_size) + 1 pages (position a in ring slot
   * a mod (ring pages * page_size)), and GLOBAL heads reserve pages for
   * append_capacity more tokens.  segpaged_decode_append then adds one token
   * per sequence and evicts the token that leaves each LOCAL window, in
   * place, with no new plan ("SegPagedAttention runtime design", §3: local
   * occupancy independent of context length; "RedKnot overview (aipuzi)",
   * §3.2: per-head pools that reclaim free pages). */
  SP_FLAG_RING = 2u
};

/* Policy of one (sequence, kv-head).  `sink` >= 0 and `window` are read for
 * SP_LOCAL and SP_RETRIEVAL.  window >= 1 is a fixed window; window <= -1 is
 * an adaptive window of max(1, ctx_len / -window) tokens for that sequence
 * ("RedKnot head classification", adaptive window: e.g. -2 gives ctx_len // 2).
 * window == 0 is invalid.  `top_p` (finite) is read for SP_RETRIEVAL only. */
typedef struct {
  int32_t kind;
  int32_t sink;
  int32_t window;
  float top_p;
} sp_head_policy;

/* One attention layer's batch.  All arrays are host memory, copied by
 * segpaged_plan_create.
 *   ctx_len[b]  L_b >= 1, tokens of sequence b in the cache (queries included)
 *   q_start[b]  q0_b in [0, L_b): the call's queries sit at q0_b .. L_b - 1, so
 *               C_b = L_b - q0_b queries; every C_b == 1 makes a decode plan.
 *   policy      [batch * num_kv_heads], (b, kv) order
 *   first_page  physical page id of the plan's first page, so that several
 *               layers' plans can share one pool
 *   page_ids    NULL, or [num_pages] distinct non-negative ids (logical page i
 *               goes to physical page first_page + page_ids[i]); num_pages is
 *               reported by segpaged_plan_sizes of a plan made with NULL
 *   target_ctas decode work is split into this many CTAs (at most one per
 *               page): contiguous ranges of the heads' concatenated page
 *               lists, balanced on pages plus a cost of 3.5 pages for each
 *               head a range starts; 0 picks 2 x 148 (two CTAs on each B200 SM).
 *               A CTA whose share is below one head start's cost can be left
 *               without work; it exits at once
 *   append_capacity  SP_FLAG_RING plans: extra tokens per sequence that
 *               segpaged_decode_append may add (GLOBAL heads reserve pages for
 *               them); must be 0 otherwise
 *   kv_dtype, k_scale, v_scale  SP_E4M3: pages hold FP8 E4M3 codes of
 *               fp32(x * (1 / scale)) (round to nearest even, saturating at
 *               +-448), one scale per layer for K and one for V; attention uses
 *               code * scale.  Supported for bf16 decode plans (page size 64);
 *               halves the bytes decode reads.  The pages say the system works
 *               with FP8 quantisation ("RedKnot overview (aipuzi)", FAQ Q5); the
 *               per-layer scale is this library's reading.
 *   block_mass  NULL when no head is SP_RETRIEVAL; else [batch * num_kv_heads]
 *               host pointers, (b, kv) order: the entry of a retrieval head
 *               points to ceil(ctx_len[b] / page_size) finite, non-negative
 *               floats, the importance of positions [i * page_size,
 *               (i + 1) * page_size); other entries are ignored.  Copied (as
 *               the kept-block choice) by segpaged_plan_create.  Retrieval
 *               heads are not supported in ring plans (SP_ERR_UNSUPPORTED).
 *   spare_pages SP_FLAG_RING plans: a pool of this many pages shared by the
 *               plan's GLOBAL heads ("RedKnot overview (aipuzi)", §3.2: per-head
 *               pools that hand out pages as heads grow).  With spare_pages > 0
 *               the pages a GLOBAL head reserves for append_capacity are page
 *               records only, with no physical page: an append that reaches
 *               such a record takes a page from the shared pool, so the pool is
 *               sized for the growth of all heads together rather than each
 *               head's worst case.  build_segpaged_cache zero-fills the spare
 *               pages.  0 keeps one physical page per reserved record.
 */
typedef struct {
  int32_t batch;
  int32_t num_q_heads;
  int32_t num_kv_heads;
  int32_t head_dim;
  int32_t page_size;
  int32_t dtype; /* sp_dtype */
  const int32_t* ctx_len;
  const int32_t* q_start;
  const sp_head_policy* policy;
  int64_t first_page;
  const int32_t* page_ids;
  int32_t target_ctas;
  uint32_t flags;
  int32_t append_capacity; /* ring plans: tokens every sequence may still gain */
  int32_t kv_dtype;        /* page type: 0 = dtype, or SP_E4M3 (bf16 decode plans) */
  float k_scale, v_scale;  /* SP_E4M3 pages: stored code = E4M3(x * (1 / scale)) */
  const float* const* block_mass; /* SP_RETRIEVAL heads: importance per page-size block */
  int32_t spare_pages;            /* ring plans: size of the shared spare pool (0: none) */
} sp_problem;

typedef struct {
  int64_t num_pages;          /* pages the plan owns in each of the K and V pools (spare pool included) */
  int64_t pool_pages;         /* pages each pool must hold: first_page + max id + 1 */
  int64_t page_bytes;         /* bytes of one page = page_size * head_dim * element size */
  int64_t table_bytes;        /* size of the device table blob */
  int64_t workspace_bytes;    /* workspace segpaged_attention needs (>= 256) */
  int64_t stored_token_heads; /* (position, kv-head) rows held in the cache */
  int64_t dense_token_heads;  /* sum over (b, kv) of L_b: rows a dense cache holds */
  int64_t visible_pairs;      /* sum over (b, q-head, query p) of |visible set of p| */
  int64_t num_queries;        /* sum_b C_b */
  int32_t is_decode;          /* 1 if every C_b == 1 */
  int32_t num_decode_ctas;    /* decode grid size (0 for prefill plans) */
  int32_t num_prefill_items;  /* prefill grid size (0 for decode plans) */
  int32_t num_combine;        /* decode heads split across CTAs */
  int32_t launches_per_call;  /* kernels one segpaged_attention call launches */
} sp_sizes;

/* One contiguous run of stored positions of a head; it starts on a fresh page. */
typedef struct {
  int32_t abs_start; /* first absolute position */
  int32_t length;    /* number of positions */
  int32_t first_page_index; /* index into the head's page list */
  int32_t num_pages;
} sp_segment;

typedef struct sp_plan sp_plan;

/* Build the SegmentPageTable of a batch ("SegPagedAttention runtime design",
 * §3 SegmentPageTable: page ids per head segment plus per-head policy).  Host
 * only, no CUDA call.  For each (b, kv): GLOBAL/DENSE keep one segment
 * [0, L); LOCAL keeps [0, min(sink, L)) and [max(sink, q0 - window + 1), L),
 * the union of what the call's queries see (merged when they touch);
 * RETRIEVAL keeps the LOCAL runs plus its kept blocks (in prefill plans a
 * run that every query sees causally, sink or kept blocks, is a segment of
 * its own, apart from the window's runs).  Each segment starts on a fresh
 * page.  The plan also holds the decode split list
 * and the prefill tile list, so that no layout work happens per attention
 * call (same page, §5: layout computed on every call cost a 0.70x slowdown).
 * The plan is immutable and may be shared by several streams. */
SP_API sp_status segpaged_plan_create(const sp_problem* problem, sp_plan** out);
SP_API void segpaged_plan_destroy(sp_plan* plan);

/* Sizes of a plan's buffers and its ledger ("SegPagedAttention runtime
 * design", §3: the per-head page table decides how many pages each head owns;
 * §5 and the closing summary: KV savings = 1 - stored / dense).  Host only;
 * fills *out with the fields of sp_sizes: pages each pool must hold, table and
 * workspace bytes, stored and dense token-heads, visible (query, key) pairs
 * (the prefill FLOP ledger is 4 * head_dim * visible_pairs) and the launch
 * shape.  SP_ERR_INVALID_ARG if plan or out is NULL. */
SP_API sp_status segpaged_plan_sizes(const sp_plan* plan, sp_sizes* out);

/* Inspect the segments / physical page ids of (b, kv) ("SegPagedAttention
 * runtime design", §3: (layer, head, segment) -> contiguous virtual pages ->
 * physical pages).  Host only.  *count receives the number available; at most
 * `max` are written (segs / page_ids may be NULL when max is 0).
 * SP_ERR_INVALID_ARG for a NULL plan or count, or (b, kv) out of range. */
SP_API sp_status segpaged_plan_head_segments(const sp_plan* plan, int32_t b, int32_t kv,
                                      sp_segment* segs, int32_t max, int32_t* count);
SP_API sp_status segpaged_plan_head_pages(const sp_plan* plan, int32_t b, int32_t kv, int64_t* page_ids,
                                   int32_t max, int32_t* count);

/* Inspect the decode work split of a plan (host only; prefill plans have no
 * decode items).  The pages have no counterpart: this is the bookkeeping of
 * this library's split-KV decode, exposed for tuning target_ctas and for
 * tests.  One record of SP_DECODE_ITEM_WORDS int32 per work item, in launch
 * order:
 *   [0] CTA   [1] b   [2] kv
 *   [3] first page, [4] one past the last page (indices into the head's page
 *       list, as segpaged_plan_head_pages orders it)
 *   [5] the item's partial slot in the workspace, or -1 when the item covers
 *       the whole head (no merge)
 *   [6] items of the head   [7] the head's first slot
 *   [8] merge group size: 0 for a one-level merge, else the head's slots form
 *       groups of this many, each merged into a group slot first
 *   [9] the head's first group slot
 *   [10] the head's arrival counter (-1 when the head is not split)
 *   [11] the arrival counter of the item's merge group (-1 when none)
 * *count receives the number of items; at most `max` records are written. */
#define SP_DECODE_ITEM_WORDS 12
SP_API sp_status segpaged_plan_decode_items(const sp_plan* plan, int32_t* records, int32_t max, int32_t* count);

/* Inspect the prefill work list of a plan (host only; decode plans have no
 * prefill items).  Each item is one CTA of the prefill kernel: one or two
 * query tiles of the same (b, kv) and the KV tiles it visits
 * ("SegPagedAttention runtime design", §4: only KV a head can see is
 * visited).  One record of SP_PREFILL_ITEM_WORDS int32 per item, in launch
 * order:
 *   [0] b   [1] kv   [2] KV tile size in tokens (128 bf16, 64 fp32)
 *   [3], [4] q-head of query tile 0 / 1 (-1: no second tile)
 *   [5], [6] first query row (index into q) of tile 0 / 1
 *   [7], [8] number of rows of tile 0 / 1
 *   [9], [10] position of the first row of tile 0 / 1
 *   [11]..[14] visited KV tiles [t0, t1) then [t2, t3), counted in tiles of
 *       the head's page list (tile i = pages [i * tile / page_size,
 *       (i + 1) * tile / page_size) in segpaged_plan_head_pages order)
 *   [15] visited KV tiles
 * *count receives the number of items; at most `max` records are written. */
#define SP_PREFILL_ITEM_WORDS 16
SP_API sp_status segpaged_plan_prefill_items(const sp_plan* plan, int32_t* records, int32_t max, int32_t* count);

/* Upload the SegmentPageTable ("SegPagedAttention runtime design", §3: page
 * ids per head segment plus per-head policy, built once when KV is written;
 * §5: never rebuilt per attention call).  Copies the plan's table blob to
 * `d_table` (device, caller-owned, >= table_bytes, 16-byte aligned) with one
 * asynchronous host-to-device copy on `stream`; the host plan stays valid and
 * unchanged.  The blob holds the heads' descriptors, their page records and
 * the decode / prefill work lists.  SP_ERR_WORKSPACE if `bytes` is smaller
 * than table_bytes, SP_ERR_INVALID_ARG for a NULL or misaligned pointer,
 * SP_ERR_CUDA if the copy cannot be enqueued.  Writing it again restores a
 * table that segpaged_decode_append has advanced. */
SP_API sp_status segpaged_table_write(const sp_plan* plan, void* d_table, size_t bytes, void* stream);

/* build_segpaged_cache ("SegPagedAttention runtime design", §3: build the
 * per-head store from dense KV, keeping only the tokens each head can see).
 * Copies, bit for bit, every stored (b, kv, position) row of the dense K and
 * V into the pools; unused slots of a segment's last page are zeroed.
 *   k_dense, v_dense  device, element (b, kv, t, i) at
 *                     base + seq_off(b) + kv*stride_head + t*stride_tok + i
 *                     (elements), with seq_off(b) = b*stride_seq, or, when
 *                     stride_seq == SP_VARLEN, (L_0 + ... + L_{b-1})*stride_tok
 *                     (sequences packed back to back in token order).
 *                     Covers [B,Hkv,Lmax,d] (stride_tok = d) and varlen
 *                     [sum L, Hkv, d] (stride_tok = Hkv*d, SP_VARLEN) layouts.
 *   k_pool, v_pool    device, pool_pages * page_bytes each, 16-byte aligned.
 * Base pointers and strides must give 16-byte aligned rows.  With SP_E4M3
 * pages the dense input is bf16 and is quantised here. */
SP_API sp_status build_segpaged_cache(const sp_plan* plan, const void* d_table, const void* k_dense,
                               const void* v_dense, int64_t stride_seq, int64_t stride_head,
                               int64_t stride_tok, void* k_pool, void* v_pool, void* stream);

/* build_segpaged_cache for several layers in one launch.  Every (layer,
 * kv-head) pair has its own policy ("SegPagedAttention runtime design", §2:
 * e.g. 80 layers x 8 kv-heads for a 70B model), so a model's cache is one
 * table per layer; this call packs several of them with a single launch (the
 * pages have no counterpart: it only saves launches).  Layer i uses
 * plans[i] / d_tables[i] and its dense K/V k_dense[i] / v_dense[i]; all
 * layers share dtype, head_dim, page_size, page type, the dense strides and
 * the pools (give each layer's plan its own first_page so that their pages do
 * not overlap; the pools must hold every layer's pool_pages).  The result is
 * bit for bit that of n_layers separate build_segpaged_cache calls.
 * 1 <= n_layers <= 128.  Arguments are checked as in build_segpaged_cache,
 * for every layer, before the launch. */
SP_API sp_status build_segpaged_cache_layers(int32_t n_layers, const sp_plan* const* plans,
                                             const void* const* d_tables, const void* const* k_dense,
                                             const void* const* v_dense, int64_t stride_seq, int64_t stride_head,
                                             int64_t stride_tok, void* k_pool, void* v_pool, void* stream);

/* Inverse of build_segpaged_cache, for checking the packing bit for bit
 * ("SegPagedAttention runtime design", §3: each head's store holds exactly
 * the tokens it can see; §4: the result is verified against a dense
 * baseline).  Writes each stored (b, kv, position) row of the pools back into
 * dense-shaped k_out / v_out (device, caller-owned; same addressing rules and
 * alignment checks as build_segpaged_cache); rows that are not stored are left
 * untouched.  With SP_E4M3 pages it writes the 1-byte codes (strides then
 * count bytes).  Errors as build_segpaged_cache. */
SP_API sp_status segpaged_gather(const sp_plan* plan, const void* d_table, const void* k_pool,
                          const void* v_pool, void* k_out, void* v_out, int64_t stride_seq,
                          int64_t stride_head, int64_t stride_tok, void* stream);

/* segpaged_attention ("SegPagedAttention runtime design", §4, the paper's
 * Algorithm 2: read each head's true KV length from the page table, evaluate
 * all (query-head, kv-head) pairs in one launch at their own lengths, no
 * mask over invisible KV).
 *   q    device [sum_b C_b, num_q_heads, head_dim], rows in sequence order,
 *        row i of sequence b at position q0_b + i; dtype of the plan
 *   out  device, same shape and dtype as q
 *   lse  device [sum_b C_b, num_q_heads] fp32 natural-log sum-exp, or NULL
 *   softmax_scale  <= 0 selects 1/sqrt(head_dim)
 *   workspace      device, >= workspace_bytes, 256-byte aligned, zero-filled
 *                  before its first use; it holds the device status word (first
 *                  256 bytes), arrival counters of split decode heads and of
 *                  their merge groups (the kernels return them to zero) and
 *                  the split partial results.
 *                  After a non-zero device status, zero it again before reuse.
 *                  Calls that overlap on the GPU need separate workspaces.
 * Decode plans run a split-KV kernel over each head's own pages plus a
 * combine pass; prefill plans run one tile kernel (tcgen05 for bf16). */
SP_API sp_status segpaged_attention(const sp_plan* plan, const void* d_table, const void* k_pool,
                             const void* v_pool, const void* q, void* out, float* lse,
                             float softmax_scale, void* workspace, size_t workspace_bytes,
                             void* stream);

/* segpaged_attention_decode_noalloc: decode attention that allocates nothing.
 * (The paper has no counterpart; this is a deployment variant of the decode
 * call above.)  Some callers cannot hand this library a workspace: engines
 * whose device memory is divided into a fixed arena before serving starts,
 * and latency-critical loops that must not call cudaMalloc because it can
 * synchronise the device.  This call runs the same split-KV decode kernels as
 * segpaged_attention on a decode plan, but takes their scratch (split heads'
 * arrival counters + partial results) from a 4 MiB array built into the
 * library's device image, one per GPU, held until the process exits.  It
 * calls no cudaMalloc, cudaFree or allocating library routine.  For the same
 * plan and inputs its output is bit for bit that of segpaged_attention.
 *   - Decode plans only (SP_ERR_UNSUPPORTED otherwise).  A plan whose
 *     workspace_bytes exceed 4 MiB is rejected with SP_ERR_WORKSPACE before
 *     any launch (lower target_ctas, or use segpaged_attention).
 *   - It runs on the current CUDA device.  The first call on a device looks
 *     up the array's device address (cudaGetSymbolAddress) with that device
 *     current; make that first call before any stream capture.  A lookup
 *     that fails is reported (SP_ERR_CUDA) and tried again by the next call.
 *   - All calls on one GPU share the array and leave their contents in it.
 *     Each call clears the split heads' arrival counters; the partial results
 *     need no clearing.  Calls whose kernels overlap on the GPU race on the
 *     array: serialise them.
 *   - d_status: required, a 4-byte aligned device int32 the caller owns (a
 *     word of its arena) that receives the device status code (the codes of
 *     segpaged_read_device_status; the first error sticks).  The call does not
 *     clear it: the caller zeroes it once and again after reading an error.
 *     NULL returns SP_ERR_INVALID_ARG.
 * Other arguments as segpaged_attention, checked the same way. */
SP_API sp_status segpaged_attention_decode_noalloc(const sp_plan* plan, const void* d_table, const void* k_pool,
                                                   const void* v_pool, const void* q, void* out, float* lse,
                                                   float softmax_scale, int32_t* d_status, void* stream);

/* segpaged_decode_append: the next decode step of a ring plan (SP_FLAG_RING),
 * in place.  For every sequence b, the token at position L_b (its current
 * context length, as held by the device table) is written into the cache:
 *   k_new, v_new  device [batch, num_kv_heads, head_dim]: element (b, kv, i) at
 *                 base + b*stride_seq + kv*stride_head + i (16-byte aligned rows)
 * and the device table d_table is updated: L_b grows by one, the new token
 * joins its page, and the token at L_b - window leaves each LOCAL head's
 * window (its page slot is released; a ring page whose tokens have all left
 * is reused when the ring wraps onto it).  GLOBAL heads use the pages
 * reserved by append_capacity; when none is left the append of that head is
 * skipped and the device status word records the error.  Subsequent
 * segpaged_attention calls on the same table see the longer context; the
 * host plan (and segpaged_plan_sizes) keep describing the state at plan
 * creation, and segpaged_table_write restores that state. */
SP_API sp_status segpaged_decode_append(const sp_plan* plan, void* d_table, const void* k_new, const void* v_new,
                                        int64_t stride_seq, int64_t stride_head, void* k_pool, void* v_pool,
                                        void* workspace, void* stream);

/* segpaged_decode_step: one serving decode step of a ring plan, the same as
 * segpaged_decode_append followed by segpaged_attention on the same table,
 * with bit for bit the same outputs, pool and table ("SegPagedAttention
 * runtime design", §3: a LOCAL head's window moves without moving tokens; §5:
 * no layout work per call).  On bf16 and E4M3 pages it is one launch: the
 * decode CTA whose page range holds a head's target page changes that page's
 * record as it streams the page, and the warp whose tokens hold the new slot
 * writes the new token into the staged copy of the page and into the pool
 * page, so no page copy waits for the append; the CTA whose range holds the
 * page of the token that leaves a LOCAL window changes that record the same
 * way; the CTA that finishes a head advances its context length.  fp32 pages
 * run the two calls.
 *   k_new, v_new, stride_seq, stride_head  as segpaged_decode_append
 *   q    device [batch, num_q_heads, head_dim]: the queries at the new
 *        positions (each sequence's current context length before the call)
 *   out, lse, softmax_scale, workspace, workspace_bytes  as segpaged_attention
 * Errors: as the two calls (a ring without room records device code 6 and
 * attends over the unchanged context; SP_ERR_INVALID_ARG for a plan that is
 * not a ring plan). */
SP_API sp_status segpaged_decode_step(const sp_plan* plan, void* d_table, const void* k_new, const void* v_new,
                                      int64_t stride_seq, int64_t stride_head, void* k_pool, void* v_pool,
                                      const void* q, void* out, float* lse, float softmax_scale, void* workspace,
                                      size_t workspace_bytes, void* stream);

/* Device status word.  The pages have no counterpart: this is the failure
 * detection of this library's kernels.  Kernels never trap; a failed
 * device-side check or a bounded wait that ran out records a non-zero code in
 * the first int32 of the workspace (the first one sticks):
 *   1, 2  a wait on a page copy (full / empty stage) ran out
 *   3     a wait on the tensor cores ran out      4  a wait on the softmax ran out
 *   5     a page id in the device table lies outside [0, pool_pages): the
 *         kernel read or wrote nothing there (a corrupted table)
 *   6     a ring append found no reserved page left (the append was skipped)
 *   7     a ring append found the shared spare pool empty (the append was skipped)
 * read synchronises `stream`, copies the word to *code (host) and returns
 * SP_OK for 0, SP_ERR_DEVICE_CHECK for a recorded code (SP_ERR_CUDA if the
 * synchronisation or the copy fails); clear zeroes the word's 256-byte block
 * asynchronously on `stream`.  `workspace` is the one given to the kernels. */
SP_API sp_status segpaged_read_device_status(const void* workspace, int32_t* code, void* stream);
SP_API sp_status segpaged_clear_device_status(void* workspace, void* stream);

/* segpaged_block_mass: the importance a RETRIEVAL head's top-p selection
 * reads, computed on the device from the dense cache: the head's own
 * attention mass per page-size block.  The pages leave the scoring rule open
 * ("RedKnot head classification", four-kind table, retrieval row: the head
 * fetches only the important tokens, page by page); the reading taken: for
 * sequence b and kv-head kv, each q-head h of the GQA group attends with its
 * query at the last position L_b - 1 over the whole context [0, L_b), and
 *   mass[b * num_kv_heads + kv][i] = (1 / g) sum_h sum_{j in block i} softmax_j(scale q_h . k_j)
 * for blocks i of page_size positions [i P, (i + 1) P), the last one ragged;
 * every row sums to 1.  Its rows are the block_mass entries a plan takes.
 *   problem   host; only batch, num_q_heads, num_kv_heads, head_dim,
 *             page_size, dtype and ctx_len are read.  bf16 only, page_size 64,
 *             head_dim 64 or 128, g = num_q_heads / num_kv_heads <= 16,
 *             batch <= 2048, batch * num_kv_heads <= 65535 (else
 *             SP_ERR_UNSUPPORTED); ctx_len[b] >= 1.
 *   k_dense   device bf16 keys, element strides stride_seq, stride_head,
 *             stride_tok (multiples of 8, head_dim contiguous), 16-byte aligned
 *             (the layout build_segpaged_cache reads)
 *   q         device bf16 [batch, num_q_heads, head_dim], 16-byte aligned:
 *             each sequence's queries at its last position
 *   softmax_scale  <= 0 selects 1 / sqrt(head_dim)
 *   mass      device fp32 [batch * num_kv_heads][mass_stride], mass_stride >=
 *             ceil(max ctx_len / page_size); entries i < ceil(ctx_len[b] /
 *             page_size) of each row are written, the rest left as they are
 *   workspace device, 256-byte aligned, at least the bytes
 *             segpaged_block_mass_workspace gives (SP_ERR_WORKSPACE if smaller);
 *             fully overwritten, no zeroing needed
 * Two launches on `stream` (a pass over the keys, one warp per block, then a
 * per (sequence, kv-head) normalisation, launched as a programmatic dependent
 * of the pass: it is placed while the pass ends and waits for it on the
 * device); fixed summation orders, so the result is bitwise reproducible.  Argument errors are reported before any
 * launch.  Calls from several host threads are serialised on the host. */
SP_API sp_status segpaged_block_mass_workspace(const sp_problem* problem, size_t* bytes);
SP_API sp_status segpaged_block_mass(const sp_problem* problem, const void* k_dense, int64_t stride_seq,
                                     int64_t stride_head, int64_t stride_tok, const void* q, float softmax_scale,
                                     float* mass, int64_t mass_stride, void* workspace, size_t workspace_bytes,
                                     void* stream);

/* segpaged_eval_exp2_fma: y[i] = 2^x[i] as the bf16 prefill kernel computes
 * it on the FMA pipe for one exponent pair in sixteen (the pages have no
 * counterpart: it is this library's own 2^x, a cubic on [-1/2, 1/2] fitted by
 * relative-error least squares, maximum relative error 7.8e-5 in fp32 for
 * x in [-125, 8], below the 2^-8 rounding of P to bf16; x below -126,
 * including -inf, gives a value in [0, 2^-125]).  Exposed so that the bound
 * can be tested on the device that runs the kernel.  d_x, d_y: device,
 * caller-owned, n floats each, 4-byte aligned; enqueued on `stream`.
 * SP_ERR_INVALID_ARG for n < 0 or bad pointers. */
SP_API sp_status segpaged_eval_exp2_fma(const float* d_x, float* d_y, int64_t n, void* stream);

SP_API const char* segpaged_status_string(sp_status status);
SP_API const char* segpaged_last_error(void);
SP_API int32_t segpaged_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* SEGPAGED_H_ */
