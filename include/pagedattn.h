/*
 * pagedattn.h — C ABI of libpagedattn.so: batched decode attention over a
 * paged KV cache on B200 (sm_100a).
 *
 * Where each call comes from (the FlashInfer pages):
 *   - README, core feature 1: single/batch attention over a sparse (paged)
 *     KV store; page_size 1 is the "vector-sparse" case.
 *   - README, core feature 2: the plan/run split.  pa_plan_create is the
 *     plan stage (host, cuts variable-length requests into equal shares
 *     per CTA, stream-K style, which the README lists among FlashInfer's
 *     inspirations); pa_run is the run stage.
 *   - README, core feature 3: cascade attention for a shared prefix
 *     (pa_cascade_plan_create / pa_cascade_run) and head-query fusion for
 *     grouped-query attention (every q head of one kv head is computed by
 *     the same CTA from one load of each K/V row).
 *   - README, core feature 1 and its usage example of append (causal mask)
 *     and prefill attention: pa_prefill_plan_create / pa_prefill_run (new
 *     query tokens of each request against its paged keys, on the tensor
 *     cores).
 *   - README, core feature 5: CUDA-graph capture.  pa_run, pa_cascade_run,
 *     pa_prefill_run and pa_merge_state only enqueue work on the given
 *     stream: no host synchronisation, no allocation.
 *   - flashinfer-cubin registry page, quickstart: the paged-table names
 *     kv_indptr, kv_indices, last_page_len and kv_layout (NHD here).
 *   - hysenlabs project review, "Installing FlashInfer and running a first
 *     decode": the decode example's query has shape [num_qo_heads, head_dim],
 *     its keys and values [kv_len, num_kv_heads, head_dim] (NHD).
 * The merge of partial states by log-sum-exp (pa_merge_state) is not named
 * on the pages; split-KV and cascade both need it.
 *
 * Math (per request b, q head hq, kv head h = hq / (Hq / Hkv)):
 *   L_b  = 0 if n_b = 0 else (n_b - 1) * P + last_page_len[b]
 *   row  = kv_indices[kv_indptr[b] + t / P] * P + t % P   for token t < L_b
 *   s_t  = sm_scale * <q[b,hq,:], k_pool[row,h,:]>
 *   lse  = ln sum_t exp(s_t)                 (natural log, fp32)
 *   o    = sum_t exp(s_t - lse) * v_pool[row,h,:]   (rounded once to q's dtype)
 *   An empty request gives o = 0 and lse = -inf.
 *
 * Layouts (all row-major, contiguous, device memory unless marked host):
 *   q, o        [batch, num_qo_heads, head_dim]          fp16 or bf16
 *   lse         [batch, num_qo_heads]                    fp32 (may be NULL)
 *   k/v pool    [num_pages, page_size, num_kv_heads, head_dim]   (NHD)
 *   kv_indptr   [batch + 1] int32, kv_indices [kv_indptr[batch]] int32,
 *   last_page_len [batch] int32.
 *
 * Ownership: the caller owns every device buffer, the workspace included;
 * the library never allocates device memory.  A plan owns its host arrays
 * until pa_plan_destroy.  Functions return a pa_status; nothing throws
 * across the ABI.  Launch failures return PA_ERR_CUDA.
 *
 * Supported: head_dim 128; num_qo_heads / num_kv_heads in {1, 2, 4, 8};
 * page_size a power of two in [1, 1024]; fp16 and bf16 q (and pools), and for
 * decode also 8-bit FP8 pools (E4M3 / E5M2 with a K and a V scale) and rotary
 * positions applied on the fly (pa_problem.kv_dtype, rope_theta).
 */
#ifndef PAGEDATTN_H_
#define PAGEDATTN_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define PA_ABI_VERSION 6

typedef enum {
  PA_OK = 0,
  PA_ERR_INVALID_ARG = 1,          /* malformed tables, null pointers, bad sizes */
  PA_ERR_UNSUPPORTED = 2,          /* valid but not built (head_dim, group size, page size) */
  PA_ERR_WORKSPACE_TOO_SMALL = 3,  /* workspace shorter than pa_plan_workspace_bytes */
  PA_ERR_CUDA = 4,                 /* a CUDA runtime call or launch failed */
  PA_ERR_DEVICE_CHECK = 5,         /* a checked run found an out-of-range page index */
  PA_ERR_NO_MEMORY = 6,            /* host allocation failed */
  PA_ERR_DEVICE_TIMEOUT = 7        /* a kernel gave up on a bounded wait (see pa_plan_check) */
} pa_status;

typedef enum {
  PA_F16 = 0,
  PA_BF16 = 1,
  PA_F32 = 2,   /* pa_merge_state only */
  PA_E4M3 = 3,  /* 8-bit KV cache (pa_problem.kv_dtype): OCP FP8 E4M3, no infinities, max 448 */
  PA_E5M2 = 4   /* 8-bit KV cache (pa_problem.kv_dtype): OCP FP8 E5M2 */
} pa_dtype;

/* Flags for pa_problem.flags. */
#define PA_FLAG_CHECK_INDICES 1u /* kernels bounds-check every page index against
                                    num_pages; a bad index is skipped (its tokens
                                    read as zero) and recorded for pa_plan_check */
/* Decode kernel choice.  By default GQA group 8 runs on the tensor-core kernel
 * and groups 1, 2 and 4 on the CUDA-core kernel (the faster of the two at
 * those shapes on B200); the work list is the same either way, only the
 * schedule defaults differ (pa_default_schedule). */
#define PA_FLAG_CUDA_CORES 2u    /* CUDA-core decode kernel for every group */
#define PA_FLAG_TENSOR_CORES 4u  /* tensor-core decode kernel for every group (fp16/bf16);
                                    PA_FLAG_CUDA_CORES wins if both are set */

typedef struct {
  int32_t batch;            /* requests B >= 0 */
  int32_t num_qo_heads;     /* Hq */
  int32_t num_kv_heads;     /* Hkv; Hq % Hkv == 0 */
  int32_t head_dim;         /* D (128) */
  int32_t page_size;        /* P, tokens per page */
  pa_dtype dtype;           /* of q, o, k_pool, v_pool */
  float sm_scale;           /* softmax scale, always given by the caller (1/sqrt(D) usually) */
  int32_t num_sms;          /* CTA budget W = num_sms * ctas_per_sm; explicit so that  */
  int32_t ctas_per_sm;      /*   the plan is a pure function of its inputs              */
  int32_t min_chunk_tokens; /* smallest per-CTA quota, in tokens; 0 means 256 */
  int64_t num_pages;        /* pages in the pool; num_pages * page_size < 2^32 (pool rows
                               are 32-bit indices); bounds for PA_FLAG_CHECK_INDICES */
  uint32_t flags;           /* PA_FLAG_* */
  int32_t piece_cost_tokens; /* plan budget charged for each further piece of a CTA
                                (see pa_plan_create): 0 = the default of the decode
                                kernel the problem runs (300 CUDA cores, 128 tensor
                                cores), > 0 that many tokens, < 0 none */
  /* Compressed KV cache (README core feature 3: low-precision attention for a
   * compressed KV-Cache).  kv_dtype PA_E4M3 or PA_E5M2: the pools hold 8-bit
   * codes, [num_pages, page_size, num_kv_heads, head_dim] bytes, and the cached
   * key is k_scale * code, the value v_scale * code (one scale per tensor;
   * both finite and > 0).  q and o stay in `dtype`.  Any other kv_dtype
   * (PA_F16 / PA_BF16) means the pools hold `dtype` and the scales are unused.
   * 8-bit caches run on the CUDA-core decode kernel (pa_run,
   * pa_run_static_workspace); cascade plans with a prefix, prefill plans and
   * PA_FLAG_TENSOR_CORES refuse them with PA_ERR_UNSUPPORTED. */
  pa_dtype kv_dtype;
  float k_scale, v_scale;
  /* Rotary positions on the fly (README usage example: decode with
   * pos_encoding_mode="ROPE_LLAMA"), when rope_theta > 0: before the dot
   * product, q is rotated to position L_b - 1 (the new token is the last one
   * in the cache) and the key of token t to position t; element pairs
   * (d, d + 64) turn by the angle pos * rope_theta^(-2d/128) (rotate-half
   * pairing; values are not rotated).  0 = no rotation.  Decode only, on the
   * CUDA-core kernel, as for 8-bit caches. */
  float rope_theta;
} pa_problem;

/* One piece of run-stage work: tokens [token_begin, token_end) of kv head
 * `kv_head` of request `request`.  Token t of the request lives on page
 * kv_indices[page_begin + t / P] at row t % P (page_begin = kv_indptr[request],
 * so the run stage needs no kv_indptr).  partial_slot is -1 when the piece is
 * the whole (request, kv head) segment (the piece writes o and lse itself),
 * else the row of the fp32 partial-state buffer it fills. */
typedef struct {
  int32_t request, kv_head, page_begin, token_begin, token_end, partial_slot;
} pa_work_item;

typedef struct pa_plan_s* pa_plan_t;

/* Plan stage (host only, no CUDA call).  Specification of the work list
 * (a stream-K style split of the whole decode step over tokens, each piece
 * boundary charged a cost c = piece_cost_tokens in token time):
 *   L_b = 0 if n_b = 0 else (n_b - 1) * P + last_page_len[b]; T = sum_b L_b;
 *   N = number of requests with L_b > 0;
 *   W = num_sms * ctas_per_sm (CTAs resident at once);
 *   groups = max(1, floor(W / Hkv)) groups of Hkv CTAs, one CTA per kv head.
 *   Walk for a budget q: the requests' tokens, laid end to end, fill groups
 *   in order.  A group takes pieces (request, [t0, t1)) in request order; a
 *   piece after the group's first one costs c + (t1 - t0) of its budget q,
 *   the first one t1 - t0.  A group is full when the next token would not
 *   fit (it holds a piece and used + c >= q); the next token then opens the
 *   next group, and a request cut there continues as the first piece of that
 *   group.  An empty request is a zero-length piece of the group the next
 *   token goes to (the last group at the very end) and costs nothing.
 *   q = 32 * ceil(max(min_chunk_tokens, ceil((T + c * max(N - 1, 0)) / groups)) / 32);
 *   n_groups is the number of groups the walk fills, never more than groups
 *   (0 for an empty batch, 1 when every request is empty); n_cta = n_groups * Hkv.
 *   With c = 0 group g holds exactly the token positions [g q, (g + 1) q).
 *   CTA g * Hkv + h runs the pieces of group g for kv head h, so the Hkv CTAs
 *   of a group read the same pages at the same time.
 *   A (request, kv head) segment cut into k > 1 pieces owns partial slots
 *   merge_indptr[b * Hkv + h] + 0 .. k - 1, in token order; merge_indptr is
 *   the running sum of those k.
 * Every CTA is resident from the start and no CTA waits for another; the
 * costs make a CTA with more pieces take fewer tokens, so all finish together.
 * Validates: kv_indptr[0] == 0 and non-decreasing, 1 <= last_page_len[b] <= P
 * whenever request b has pages, Hq % Hkv == 0, positive sizes.
 * Returns PA_ERR_INVALID_ARG / PA_ERR_UNSUPPORTED otherwise.  The host arrays
 * are copied; the caller may free them after the call. */
pa_status pa_plan_create(const pa_problem* problem, const int32_t* kv_indptr_host,
                         const int32_t* last_page_len_host, pa_plan_t* out);

/* Plan for a two-level cascade: a shared prefix of prefix_len tokens (whole
 * pages, prefix_len % P == 0) that every request attends to first, plus each
 * request's own pages described by kv_indptr_host / last_page_len_host.  The
 * work list is the one pa_plan_create gives for the per-request pages; the
 * prefix level is scheduled as (kv head, 128-query-row tile, prefix chunk)
 * tiles on the tensor cores. */
pa_status pa_cascade_plan_create(const pa_problem* problem, int32_t prefix_len,
                                 const int32_t* kv_indptr_host,
                                 const int32_t* last_page_len_host, pa_plan_t* out);

/* One query tile of a prefill plan: query tokens [q_begin, q_begin + n_q)
 * (rows of q and o) of request `request`; token q_begin + j sees keys
 * [0, min(kv_base + j + 1, kv_end)) of the request, page_begin =
 * kv_indptr[request].  Causal plans have kv_end = kv_base + n_q, plans
 * without the mask kv_base = kv_end - 1 = L_b - 1. */
typedef struct {
  int32_t request, q_begin, n_q, page_begin, kv_base, kv_end;
} pa_prefill_tile;
/* Plan for prefill / append attention (host only, no CUDA call).  Request b
 * has Q_b = qo_indptr[b + 1] - qo_indptr[b] new query tokens, rows
 * qo_indptr[b] .. qo_indptr[b + 1] - 1 of q and o, and L_b keys in its pages
 * (kv_indptr / last_page_len as for pa_plan_create).  With causal != 0 the
 * last Q_b keys are the new tokens' own and new token i (0-based within the
 * request) attends to keys t < L_b - Q_b + i + 1 (Q_b = L_b is prefill,
 * Q_b < L_b append); with causal == 0 every token attends to all L_b keys.
 *   s_t = sm_scale <q[qo_indptr[b] + i, hq, :], k_pool[row(b, t), h, :]>,
 *   lse = ln sum_t exp(s_t) (fp32), o = sum_t exp(s_t - lse) v_pool[row(b, t), h, :]
 *   rounded once to the input type; a token that sees no key gets o = 0,
 *   lse = -inf.
 * Layouts: q and o are [total_q, num_qo_heads, head_dim] with total_q =
 * qo_indptr[batch]; lse is [total_q, num_qo_heads]; the pools as above.
 * Work: the query tokens of each request are cut into tiles of 256 / G
 * consecutive tokens (G = Hq / Hkv; the last tile of a request may be
 * shorter).  Tile order: the
 * tiles of one request together, requests in decreasing order of their
 * longest tile's ceil(kv_end / 128) (ties by request index), and within a
 * request decreasing ceil(kv_end / 128), ties in token order.  Item
 * w = tile * num_kv_heads + kv head is the work of one (tile, kv head).
 * The run launches min(num_sms, items) persistent CTAs (one per SM; pass the
 * device's SM count), each running its own list of items in order: the items
 * are dealt in order w = 0, 1, ... to the CTA with the least estimated load
 * so far (ties to the lower CTA), an item's load being the 128-key tiles of
 * its two 128-row halves (ceil(min(kv_base + n0, kv_end) / 128) and, if the
 * tile has more than n0 = 128 / G tokens, ceil(kv_end / 128)) plus 2.
 * pa_plan_cta_indptr and pa_plan_prefill_schedule return the lists.
 * ctas_per_sm, min_chunk_tokens and piece_cost_tokens are not used.
 * Validates as pa_plan_create, plus: qo_indptr[0] == 0 and non-decreasing,
 * total_q < 2^31, and Q_b <= L_b when causal.  page_size must be >= 8
 * (pages move as tensor-memory-access boxes of >= 8 rows) and num_pages *
 * page_size < 2^31 - 1: PA_ERR_UNSUPPORTED otherwise. */
pa_status pa_prefill_plan_create(const pa_problem* problem, int32_t causal,
                                 const int32_t* qo_indptr_host, const int32_t* kv_indptr_host,
                                 const int32_t* last_page_len_host, pa_plan_t* out);
/* Read-only views of the plan (borrowed; valid until pa_plan_destroy). */
pa_status pa_plan_quota_tokens(pa_plan_t plan, int32_t* quota);
pa_status pa_plan_work_items(pa_plan_t plan, const pa_work_item** items, int64_t* n_items);
pa_status pa_plan_cta_indptr(pa_plan_t plan, const int32_t** cta_indptr /* [n_cta+1] */,
                             int64_t* n_cta);
/* Prefill plans: the items of CTA c are items[cta_indptr[c] .. cta_indptr[c + 1]),
 * each w = tile * num_kv_heads + kv head; n_items = tiles * num_kv_heads
 * (decode and cascade plans: none). */
pa_status pa_plan_prefill_schedule(pa_plan_t plan, const int32_t** items, int64_t* n_items);
pa_status pa_plan_merge_indptr(pa_plan_t plan,
                               const int32_t** merge_indptr /* [B*Hkv+1] */);
pa_status pa_plan_num_partials(pa_plan_t plan, int64_t* n_partials);
pa_status pa_plan_prefix_chunks(pa_plan_t plan, int32_t* n_chunks, int32_t* chunk_tokens);
/* The tiles of a prefill plan in launch order (0 tiles for other plans). */
pa_status pa_plan_prefill_tiles(pa_plan_t plan, const pa_prefill_tile** tiles, int64_t* n_tiles);

/* Device workspace the run stage needs: work list, CTA and merge offsets,
 * arrival counters and fp32 partial states.  Caller-allocated, 256-byte
 * aligned. */
pa_status pa_plan_workspace_bytes(pa_plan_t plan, size_t* bytes);

/* Byte offset, within the workspace, of the two 64-bit status words that
 * pa_plan_check reads: word 0 holds the first out-of-range kv_indices
 * position a PA_FLAG_CHECK_INDICES run met (all ones: none), word 1 is
 * nonzero once a kernel abandoned a bounded wait.  pa_plan_upload writes
 * both as "nothing seen"; 8-byte aligned. */
pa_status pa_plan_status_offset(pa_plan_t plan, size_t* offset);

/* Copy the work list into the workspace and zero its counters (enqueued on
 * `stream`, a cudaStream_t or NULL for the legacy default stream).  Once per
 * plan and workspace; any number of runs may follow.  The counters return to
 * zero at the end of every run, so captured graphs can be replayed. */
pa_status pa_plan_upload(pa_plan_t plan, void* d_workspace, size_t workspace_bytes,
                         void* stream);

/* Run stage: decode attention for every request of the plan.  kv_indices is
 * the device copy of the table the plan was made from.  One launch of n_cta
 * CTAs; the pieces of a split (request, kv head) are merged inside it by the
 * last CTA to finish one of them (no second kernel).  lse may be NULL. */
pa_status pa_run(pa_plan_t plan, const void* q, const void* k_pool, const void* v_pool,
                 const int32_t* d_kv_indices, void* o, float* lse, void* d_workspace,
                 size_t workspace_bytes, void* stream);

/* Cascade run: level 1 attends all B * Hq query rows to the shared prefix
 * (pages d_prefix_indices[0 .. prefix_len / P)) on the tensor cores; level 2
 * is the paged decode over each request's own pages; both are merged by
 * log-sum-exp into o and lse.  Two launches: level 1 leaves one state per
 * prefix chunk and row in the workspace, and level 2 (a programmatic
 * dependent of level 1, which may start while level 1 finishes) merges all
 * of a row's chunk states with its own in its epilogue.  The plan must come
 * from pa_cascade_plan_create. */
pa_status pa_cascade_run(pa_plan_t plan, const void* q, const void* k_pool,
                         const void* v_pool, const int32_t* d_prefix_indices,
                         const int32_t* d_kv_indices, void* o, float* lse, void* d_workspace,
                         size_t workspace_bytes, void* stream);

/* Prefill / append run: attention of every new query token of the plan
 * (pa_prefill_plan_create) to its request's keys, written to o and
 * lse (lse may be NULL).  One launch; the plan's tiles must have been
 * uploaded (pa_plan_upload) into d_workspace.  PA_FLAG_CHECK_INDICES
 * bounds-checks page indices as for pa_run.  Other plans are rejected with
 * PA_ERR_INVALID_ARG, as prefill plans are by pa_run and pa_cascade_run. */
pa_status pa_prefill_run(pa_plan_t plan, const void* q, const void* k_pool, const void* v_pool,
                         const int32_t* d_kv_indices, void* o, float* lse, void* d_workspace,
                         size_t workspace_bytes, void* stream);
/* Combine two attention states over disjoint token sets, row by row:
 *   M = max(lse_a, lse_b), w_x = exp(lse_x - M),
 *   o = (w_a o_a + w_b o_b) / (w_a + w_b),   lse = M + ln(w_a + w_b).
 * Both lse = -inf gives o = 0, lse = -inf.  o_* are [rows, head_dim] in
 * `dtype` (fp16, bf16 or fp32), lse_* are [rows] fp32 natural-log.  The
 * outputs may alias either input. */
pa_status pa_merge_state(const void* o_a, const float* lse_a, const void* o_b,
                         const float* lse_b, void* o, float* lse, int64_t rows,
                         int32_t head_dim, pa_dtype dtype, void* stream);

/* pa_run without a caller-provided workspace, for callers that cannot
 * allocate device memory (an engine whose pool already holds all free GPU
 * memory, a host program that does not own the process's allocator, a path
 * that must not take cudaMalloc's implicit synchronisation).  The source
 * pages have no counterpart: this is a convenience of this library.
 * The workspace is a fixed 8 MiB array inside libpagedattn.so on every GPU
 * that loads it, held until the process exits; a plan needing more
 * (pa_plan_workspace_bytes > 8 MiB) is rejected with
 * PA_ERR_WORKSPACE_TOO_SMALL before anything is enqueued, and cascade and
 * prefill plans with PA_ERR_INVALID_ARG.  Nothing is allocated: each call uploads the plan
 * into the array (as pa_plan_upload) and runs it (as pa_run).  The first call
 * on a device looks the array up (cudaGetSymbolAddress); the looked-up address
 * is kept for the life of the process: after a cudaDeviceReset on that device this entry point must not
 * be used again.  All calls share the array: calls that overlap on the GPU
 * (different streams or threads) race. */
pa_status pa_run_static_workspace(pa_plan_t plan, const void* q, const void* k_pool,
                                  const void* v_pool, const int32_t* d_kv_indices, void* o,
                                  float* lse, void* stream);

/* pa_plan_check for the library's fixed workspace: synchronously reads and
 * clears the status words that the last pa_run_static_workspace call on this
 * device left in it, with the same results as pa_plan_check (PA_ERR_DEVICE_TIMEOUT,
 * PA_ERR_DEVICE_CHECK with *bad_position, or PA_OK).  Call it after that run
 * and before the next one, which clears the words again.  `plan` must be the
 * plan of that run (its layout locates the words); plans that
 * pa_run_static_workspace refuses are refused here with the same status. */
pa_status pa_static_workspace_check(pa_plan_t plan, int64_t* bad_position, void* stream);

/* Synchronously read and clear the device status words of a workspace.
 * Returns PA_ERR_DEVICE_TIMEOUT if a kernel abandoned one of its bounded
 * pipeline waits (its outputs are then undefined), else PA_ERR_DEVICE_CHECK
 * with the first bad kv_indices position in *bad_position if a run with
 * PA_FLAG_CHECK_INDICES met an out-of-range page index, else PA_OK
 * (*bad_position = -1). */
pa_status pa_plan_check(pa_plan_t plan, void* d_workspace, int64_t* bad_position, void* stream);

/* Scheduling defaults for `device`: its SM count and how many CTAs of the
 * decode kernel that a problem with this shape, dtype and `flags` (PA_FLAG_*)
 * runs fit on one SM.  The tensor-core kernel holds one CTA per SM. */
pa_status pa_default_schedule(int32_t device, int32_t num_qo_heads, int32_t num_kv_heads,
                              pa_dtype dtype, uint32_t flags, int32_t* num_sms,
                              int32_t* ctas_per_sm);

/* pa_default_schedule for a whole problem: the SM count of `device` and how
 * many CTAs of the decode kernel that `problem` runs fit on one SM, its
 * 8-bit cache and rotary positions included (only the shape, dtype, flags,
 * kv_dtype and rope_theta fields are read). */
pa_status pa_problem_schedule(const pa_problem* problem, int32_t device, int32_t* num_sms,
                              int32_t* ctas_per_sm);

/* 1 if the plan's decode level runs on the tensor-core kernel, 0 if on the
 * CUDA-core kernel, -1 for a null plan.  Prefill plans always run on the
 * tensor cores (1). */
int32_t pa_plan_uses_tensor_cores(pa_plan_t plan);

void pa_plan_destroy(pa_plan_t plan);
const char* pa_status_string(pa_status status);
int32_t pa_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* PAGEDATTN_H_ */
