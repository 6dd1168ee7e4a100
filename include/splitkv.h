/*
 * splitkv.h -- C ABI of libsplitkv: batched attention over a paged KV cache with split-KV
 * partials and an exact log-sum-exp merge, for NVIDIA B200 (sm_100a).
 *
 * Operations and where they are defined
 *   skv_paged_attn_fwd  GQA attention over a paged KV cache whose K and V may have equal or
 *                       independent strides (FlashInfer PR #4736 page, section 1
 *                       "batch_pod.cu: flexible stride handling" and section 2 "SAME_KV_STRIDES
 *                       template specialisation"); one KV sequence may be listed by many query
 *                       batches (PyTorch MPS FlexAttention page, "KV batch broadcast").  The
 *                       cache may be bf16 or fp8 e4m3 with a per-tensor scale (FP8 KV decode,
 *                       FlashInfer PR #3309 page, introduction).
 *   skv_mla_decode_fwd  Multi-head latent attention decode: every head reads one 512+64-d latent
 *                       row per token, V is the 512-d latent; seqlen_q is folded into heads to
 *                       fill the MMA M tile (FlashInfer PR #3309 page, sections 1-2 and "why it
 *                       is good": M tile 128, 2D/3D LSE layouts).
 *   skv_merge_states    Exact merge of partial (O, LSE) states of KV splits (route primitive:
 *                       partial attention at the KV holder merged "via online softmax",
 *                       "Move the Query, Not the Cache", Methodology; in-CTA split with
 *                       shared-memory merge, FlashInfer PR #5597 page, section 3).
 *   skv_plan_paged_subset  Planner for part of a batch: a mixed prefill + decode batch is planned
 *                       as two subsets, each on the kernel that suits its requests.
 *   skv_pod_attn_fwd    Such a batch in one attention launch (FlashInfer PR #4736 page, section 1,
 *                       batch_pod.cu: prefill and decode work fused in one kernel).
 *   skv_causal_tables   Host planner that turns causal / multi-token attention into a prefix
 *                       call, a diagonal call over token rows and an exact merge.
 *   skv_mla_splice      The fetch primitive's local compute: move a chunk's latent rows between
 *                       page lists and re-rotate their RoPE part to the new positions ("Move
 *                       the Query, Not the Cache", problem statement and Methodology: fetch
 *                       adapts cached position encodings to new offsets, the "splice").
 *
 * Semantics shared by all calls (natural-log LSE of the scaled logits):
 *   s_t = sm_scale * q . k_t ;  O = sum_t softmax(s)_t v_t ;  LSE = ln sum_t exp(s_t).
 *   A request with no KV tokens gives O = 0, LSE = -inf.  The attention calls take no mask:
 *   every query token of a request attends to all of the request's KV tokens; causal attention
 *   is planned by skv_causal_tables on top of them.
 *
 * Page table (device int32 arrays): request r owns pages kv_indices[kv_indptr[r] ..
 *   kv_indptr[r+1]); its length is L_r = (n_r - 1) * page_size + kv_last_page_len[r] with
 *   kv_last_page_len[r] in [1, page_size] (L_r = 0 when n_r = 0).  Token t of request r is
 *   slot t % page_size of physical page kv_indices[kv_indptr[r] + t / page_size].
 *
 * Conventions
 *   - Pure C.  Every pointer argument is a DEVICE pointer unless its name ends in _h (host).
 *   - The caller owns every buffer; the library never allocates, never synchronises, never
 *     prints.  Work is enqueued on `stream` (a cudaStream_t; NULL = legacy default stream).
 *   - Host-detectable errors return a status before anything is launched.
 *   - Device-detected errors (a page id >= num_pages, a barrier wait that timed out) are
 *     written to the optional device int32 word `status` (first error wins; 0 = ok) and the
 *     affected outputs are unspecified.  Kernels never trap.
 *   - Calls are asynchronous: buffers must stay valid until the stream reaches the work.
 */
#ifndef SPLITKV_H_
#define SPLITKV_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define SKV_API __attribute__((visibility("default")))
#else
#define SKV_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* skv_stream_t; /* same handle type as cudaStream_t */

typedef enum {
  SKV_OK = 0,
  SKV_ERR_INVALID = 1,     /* bad argument: null pointer, negative size, inconsistent table   */
  SKV_ERR_UNSUPPORTED = 2, /* valid but not implemented: head_dim, group size, dtype          */
  SKV_ERR_ALIGNMENT = 3,   /* base pointer / stride not 16-byte aligned (TMA requirement)     */
  SKV_ERR_WORKSPACE = 4,   /* plan or partial buffers too small for the plan                  */
  SKV_ERR_CUDA = 5         /* a CUDA runtime call (attribute set, launch) failed              */
} skv_status;

/* codes written to the device status word */
#define SKV_DEV_OK 0
#define SKV_DEV_TIMEOUT 16   /* an mbarrier wait exceeded its iteration cap                  */
#define SKV_DEV_PAGE_OOB 17  /* a page id outside [0, num_pages)                              */
#define SKV_DEV_PLAN_BAD 18  /* a work item outside the request's pages / query rows          */

typedef enum { SKV_BF16 = 0, SKV_F32 = 1, SKV_E4M3 = 2 } skv_dtype;

/* split policies for the planners */
typedef enum {
  SKV_SPLIT_NONE = 0,     /* one split per request                                           */
  SKV_SPLIT_FIXED = 1,    /* `param` splits per request (earlier splits take the extra page)  */
  SKV_SPLIT_BALANCED = 2, /* splits chosen so all SMs stay busy; `param` = SM count (0 = query */
                          /* the current device).  For the persistent tensor-core kernels the  */
                          /* KV of all requests is cut into `param` equal slices, one per CTA. */
  SKV_SPLIT_EXPLICIT = 3  /* boundaries given in split_indptr_h / split_bounds_h               */
} skv_split_policy;

/* Summary of a plan.  The plan itself is an int32 array the caller copies to the device. */
typedef struct {
  int32_t num_work;         /* work items (CTAs per KV head for GQA, per split for MLA)       */
  int32_t num_partial_rows; /* rows the o_part / lse_part buffers must hold (0: no split)     */
  int32_t num_merge_rows;   /* output rows combined from >1 split by the merge pass           */
  int32_t kernel;           /* kernel variant the dispatcher picked (informational): 1 GQA on  */
                            /*   CUDA cores, 2 GQA tensor-core decode per KV head, 3 GQA      */
                            /*   tensor-core decode over all KV heads, 4 GQA tensor-core      */
                            /*   prefill (128 query rows), 11 MLA on CUDA cores, 12 / 13 / 14 */
                            /*   MLA tensor cores with 16 / 32 / 64 query rows per tile       */
  int32_t q_tile;           /* query tokens per work item (MLA: the fold ratio F)             */
  int32_t plan_words;       /* int32 words of the plan actually used                          */
  int32_t max_splits;       /* largest split count of any request                             */
  int32_t total_splits;     /* sum over requests of their split counts                        */
  int32_t num_ctas;         /* persistent kernels: CTAs the plan was balanced for (else 0);  */
                            /*   CTA c runs work items cta_indptr[c] .. cta_indptr[c+1]; for  */
                            /*   kernel 14 a group of R CTAs shares each KV slice s (CTA c    */
                            /*   runs slice c / R), R = (q_len / q_tile) * head groups        */
                            /*   (num_heads / 64 when num_heads > 64, else 1)                 */
  int32_t cta_offset;       /* int32 word offset of cta_indptr [num_ctas+1] in the plan       */
} skv_plan_info;

/* -------------------------------------------------------------------------------------------
 * skv_plan_paged -- host-side planner for skv_paged_attn_fwd.
 *   qo_indptr_h [batch+1]      query tokens of request r are rows qo_indptr_h[r] ..
 *   kv_indptr_h [batch+1], kv_last_page_len_h [batch]   host copies of the page-table shape
 *   page_size, num_qo_heads, num_kv_heads (divides num_qo_heads), head_dim in {64, 128}
 *   policy / param              see skv_split_policy
 *   split_indptr_h [batch+1], split_bounds_h   only for SKV_SPLIT_EXPLICIT: request r has
 *       S_r = split_indptr_h[r+1] - split_indptr_h[r] splits whose S_r + 1 request-relative
 *       page boundaries are split_bounds_h[split_indptr_h[r] + r ...] (non-decreasing, first 0,
 *       last n_r; empty splits allowed).  Pass NULL otherwise.
 *   plan_h / plan_capacity      output int32 buffer (host); SKV_ERR_WORKSPACE if too small,
 *                               with info->plan_words set to the size needed.
 *   info                        output summary.
 * With S_r > 1 the split partials of query token i, split j of request r are row
 *   part_base_r + i * S_r + j of o_part / lse_part; requests with S_r = 1 write O directly.
 * ----------------------------------------------------------------------------------------- */
SKV_API skv_status skv_plan_paged(int32_t batch, const int32_t* qo_indptr_h, const int32_t* kv_indptr_h,
                          const int32_t* kv_last_page_len_h, int32_t page_size,
                          int32_t num_qo_heads, int32_t num_kv_heads, int32_t head_dim,
                          int32_t policy, int32_t param, const int32_t* split_indptr_h,
                          const int32_t* split_bounds_h, int32_t* plan_h,
                          int64_t plan_capacity, skv_plan_info* info);

/* Arguments of skv_paged_attn_fwd.  All pointers are device pointers. */
typedef struct {
  const void* q;            /* bf16 [total_q, Hq, D], contiguous                              */
  const void* k_cache;      /* bf16: K(page, slot, head, d) = k_cache[page*k_stride[0] +       */
  const void* v_cache;      /*   slot*k_stride[1] + head*k_stride[2] + d]; V likewise with      */
  int64_t k_stride[3];      /*   v_stride.  Strides in elements, each a multiple of 8 (16 B);  */
  int64_t v_stride[3];      /*   when all three are equal the SAME_KV_STRIDES kernel runs.     */
  const int32_t* kv_indptr;         /* [batch+1]                                              */
  const int32_t* kv_indices;        /* [kv_indptr[batch]] physical page ids                   */
  const int32_t* kv_last_page_len;  /* [batch]                                                */
  int32_t batch;
  int32_t total_q;          /* rows of q / o                                                  */
  int32_t num_pages;        /* physical pages in the cache (device bound check)               */
  int32_t page_size;
  int32_t num_qo_heads;
  int32_t num_kv_heads;
  int32_t head_dim;         /* 64 or 128                                                       */
  float sm_scale;
  void* o;                  /* [total_q, Hq, D] of o_dtype                                     */
  int32_t o_dtype;          /* SKV_F32 or SKV_BF16                                             */
  float* lse;               /* [total_q, Hq] fp32 (may be NULL)                                */
  float* o_part;            /* [num_partial_rows, Hq, D] fp32, needed when the plan splits     */
  float* lse_part;          /* [num_partial_rows, Hq] fp32                                     */
  int32_t* status;          /* device status word (may be NULL)                                */
  int32_t kv_dtype;         /* SKV_BF16 (0, the default) or SKV_E4M3: K and V hold OCP e4m3fn   */
                            /*   codes (one byte per element; strides then multiples of 16),    */
                            /*   k = kv_scale * code(k), v = kv_scale * code(v).  e4m3 runs on  */
                            /*   plans whose kernel is 3 (all KV heads on the tensor cores);    */
                            /*   other plans return SKV_ERR_UNSUPPORTED                          */
  float kv_scale;           /* per-tensor dequantisation scale for SKV_E4M3 (finite, > 0)      */
} skv_paged_params;

/* -------------------------------------------------------------------------------------------
 * skv_paged_attn_fwd -- O, LSE (and split partials) of GQA attention over the paged cache.
 *   plan_d: device copy of the plan from skv_plan_paged for the same shapes; info: its summary.
 *   Query head h reads KV head h / (Hq / Hk).  Split partials are written to o_part/lse_part
 *   and merged into o/lse on the same stream.
 * ----------------------------------------------------------------------------------------- */
SKV_API skv_status skv_paged_attn_fwd(const skv_paged_params* p, const int32_t* plan_d,
                              const skv_plan_info* info, skv_stream_t stream);

/* The two phases of skv_paged_attn_fwd, for callers that schedule (or time) them separately:
 *   skv_paged_attn_partial  the attention kernel only: writes o / lse of requests with one
 *                           split and o_part / lse_part of split requests;
 *   skv_merge_plan          the plan's merge pass: combines o_part / lse_part into o / lse
 *                           (num_heads, head_dim: 512 for MLA).  A no-op for plans without
 *                           merge rows.  Calling both in order equals skv_paged_attn_fwd. */
SKV_API skv_status skv_paged_attn_partial(const skv_paged_params* p, const int32_t* plan_d,
                                          const skv_plan_info* info, skv_stream_t stream);
SKV_API skv_status skv_merge_plan(const float* o_part, const float* lse_part, const int32_t* plan_d,
                                  const skv_plan_info* info, int32_t num_heads, int32_t head_dim,
                                  void* o, int32_t o_dtype, float* lse, skv_stream_t stream);

/* -------------------------------------------------------------------------------------------
 * skv_paged_attn_fwd_static_scratch -- skv_paged_attn_fwd without caller-provided split partials.
 *   No counterpart on the pages this library follows: it exists for callers that cannot
 *   allocate device memory -- a serving engine that gives nearly all device memory to its KV
 *   cache at start-up and keeps no allocator on the decode path, or a plain-C / foreign-runtime
 *   caller with no device allocator of its own (cudaMalloc would also synchronize the device).
 *   Same arguments and results as skv_paged_attn_fwd; p->o_part / p->lse_part are ignored.  The
 *   partials go to one file-scope device array of 32 MiB that every GPU loading this library
 *   holds until the process exits; plans whose partials (num_partial_rows * Hq * (D + 1) floats,
 *   each part rounded up to 256 B) exceed it return SKV_ERR_WORKSPACE with nothing launched.
 *   The first call on a device looks up the array's device address (cudaGetSymbolAddress, with
 *   that device current); make that first call before any stream capture.  Allocates nothing.
 *   All calls share the array and it keeps the last call's contents (every partial is written
 *   before it is read, so nothing needs clearing); calls that overlap on the GPU race.
 *   `info` must be the summary returned together with `plan_d`: the size check reads
 *   info->num_partial_rows while the kernels write the partial rows plan_d names, so a summary
 *   from another plan would let them write past the array (the regular entry point would
 *   write past the caller's own buffers instead).
 * ----------------------------------------------------------------------------------------- */
SKV_API skv_status skv_paged_attn_fwd_static_scratch(const skv_paged_params* p, const int32_t* plan_d,
                                                     const skv_plan_info* info, skv_stream_t stream);

/* -------------------------------------------------------------------------------------------
 * skv_plan_mla -- host-side planner for skv_mla_decode_fwd (same split policies); kv_dtype is
 *   the cache type (SKV_BF16 or SKV_E4M3) the plan will run on.  The fold ratio F (seqlen_q
 *   tokens folded into the query-row dimension of a work item) is reported in info->q_tile:
 *   F = skv_mla_fold_ratio(H, q_len, R) with R the rows the chosen kernel puts on one tile
 *   (16 or 32 for the tensor-core kernels, and 64 for the bf16 cache when H * q_len > 32 and the
 *   page size is not 1; they split H > R heads into groups of R; 128 for the CUDA-core kernel).
 *   With R = 64 the (query tile, head group) units of a KV slice run on a group of co-resident
 *   CTAs at once, so each slice is read from HBM about once.  The tensor-core kernels take page
 *   sizes >= 8 that divide or are multiples of 64, and (bf16 cache only) page size 1, where every
 *   page id is a token row; other page sizes run on the CUDA-core kernel.  Run a plan on the
 *   kv_dtype it was made for.
 * ----------------------------------------------------------------------------------------- */
SKV_API skv_status skv_plan_mla(int32_t batch, int32_t q_len, const int32_t* kv_indptr_h,
                        const int32_t* kv_last_page_len_h, int32_t page_size, int32_t num_heads,
                        int32_t kv_dtype, int32_t policy, int32_t param, const int32_t* split_indptr_h,
                        const int32_t* split_bounds_h, int32_t* plan_h, int64_t plan_capacity,
                        skv_plan_info* info);

/* Arguments of skv_mla_decode_fwd.  All pointers are device pointers. */
typedef struct {
  const void* q_nope;       /* bf16 [B, q_len, H, 512], contiguous                            */
  const void* q_pe;         /* bf16 [B, q_len, H, 64], contiguous                             */
  const void* ckv;          /* latent: ckv(page, slot, d) = ckv[page*ckv_stride[0] +           */
  const void* kpe;          /*   slot*ckv_stride[1] + d], d < 512; kpe likewise, d < 64        */
  int64_t ckv_stride[2];    /* elements; multiples of 16 bytes                                 */
  int64_t kpe_stride[2];
  int32_t kv_dtype;         /* SKV_BF16 or SKV_E4M3 (OCP e4m3fn codes)                          */
  float kv_scale;           /* per-tensor dequantisation scale (1 for bf16)                    */
  const int32_t* kv_indptr;
  const int32_t* kv_indices;
  const int32_t* kv_last_page_len;
  int32_t batch;
  int32_t q_len;
  int32_t num_heads;
  int32_t num_pages;
  int32_t page_size;
  float sm_scale;
  void* o;                  /* [B, q_len, H, 512] of o_dtype                                   */
  int32_t o_dtype;          /* SKV_F32 or SKV_BF16                                             */
  float* lse;               /* [B, q_len, H] fp32 (== 2D [B*q_len, H]); may be NULL            */
  float* o_part;            /* [num_partial_rows, H, 512] fp32 when the plan splits            */
  float* lse_part;          /* [num_partial_rows, H]                                           */
  int32_t* status;
} skv_mla_params;

/* skv_mla_decode_fwd -- MLA decode: s = sm_scale (q_nope . ckv + q_pe . kpe), V = ckv (times
 *   kv_scale for e4m3).  Partial rows follow the skv_plan_paged layout with query "token" =
 *   (decode position i) of the request. */
SKV_API skv_status skv_mla_decode_fwd(const skv_mla_params* p, const int32_t* plan_d,
                              const skv_plan_info* info, skv_stream_t stream);
/* First phase of skv_mla_decode_fwd (attention kernel only); finish with skv_merge_plan. */
SKV_API skv_status skv_mla_decode_partial(const skv_mla_params* p, const int32_t* plan_d,
                                          const skv_plan_info* info, skv_stream_t stream);

/* -------------------------------------------------------------------------------------------
 * skv_merge_states -- exact merge of partial states.
 *   For each output row r and head h, over its states j:
 *     M = max_j LSE_j, LSE = M + ln sum_j exp(LSE_j - M), O = sum_j exp(LSE_j - LSE) O_j;
 *     no state, or all LSE_j = -inf: O = 0, LSE = -inf.
 *   State layout: with state_indptr (device [num_rows+1]) the states of row r are rows
 *   state_indptr[r] .. state_indptr[r+1] of o_states [*, H, D] / lse_states [*, H]; with
 *   state_indptr == NULL there are `num_states` states per row stored state-major:
 *   o_states [num_states, num_rows, H, D], lse_states [num_states, num_rows, H] (for example
 *   one buffer per KV chunk holder).  head_dim a multiple of 4; o_out of o_dtype
 *   [num_rows, H, D]; lse_out [num_rows, H] (may be NULL).
 * ----------------------------------------------------------------------------------------- */
SKV_API skv_status skv_merge_states(const float* o_states, const float* lse_states,
                            const int32_t* state_indptr, int32_t num_states, int64_t num_rows,
                            int32_t num_heads, int32_t head_dim, void* o_out, int32_t o_dtype,
                            float* lse_out, skv_stream_t stream);

/* -------------------------------------------------------------------------------------------
 * skv_plan_paged_subset -- skv_plan_paged for the requests listed in requests_h only (distinct
 *   indices in [0, batch)); the others get no work, so a launch with this plan writes only the
 *   listed requests' query rows and partial rows.  One batch that mixes prefill and decode
 *   requests (a POD batch: prefill on decode, FlashInfer PR #4736 page, batch_pod.cu) is planned
 *   as two subsets, each choosing its own kernel, and launched with the batch's own q, page table
 *   and outputs -- no copy of any of them -- in one launch by skv_pod_attn_fwd, or one launch per
 *   plan.  Every plan needs its own o_part / lse_part.  Explicit splits are not accepted here
 *   (SKV_ERR_INVALID).
 * ----------------------------------------------------------------------------------------- */
SKV_API skv_status skv_plan_paged_subset(int32_t batch, const int32_t* qo_indptr_h, const int32_t* kv_indptr_h,
                                         const int32_t* kv_last_page_len_h, int32_t page_size,
                                         int32_t num_qo_heads, int32_t num_kv_heads, int32_t head_dim,
                                         int32_t policy, int32_t param, const int32_t* requests_h,
                                         int32_t num_requests, int32_t* plan_h, int64_t plan_capacity,
                                         skv_plan_info* info);

/* -------------------------------------------------------------------------------------------
 * skv_pod_attn_fwd -- one batch mixing decode and prefill requests in ONE attention launch (POD,
 *   FlashInfer PR #4736 page, section 1: batch_pod.cu fuses prefill and decode work in one kernel).
 *   decode_plan_d / decode_info: skv_plan_paged_subset over the batch's decode requests; it must
 *     pick kernel 3 (all KV heads on the tensor cores; 8 query rows per KV head) and, with
 *     SKV_SPLIT_BALANCED, its `param` is the number of SMs (persistent CTAs) given to decode.
 *   prefill_plan_d / prefill_info: skv_plan_paged_subset over the prefill requests; it must pick
 *     kernel 4 (128-row prefill tiles).  Either plan may be empty (then only the other runs).
 *   p: the batch's q, K/V caches (bf16), page table and outputs o / lse; p->o_part / p->lse_part
 *     hold the decode plan's split partials and prefill_o_part / prefill_lse_part the prefill
 *     plan's (each sized by its plan's num_partial_rows).
 *   The launch has decode_info->num_ctas + prefill units CTAs: the first num_ctas stream the decode
 *   slices (HBM-bound) for the whole launch while the rest take the prefill units (tensor-bound) on
 *   the other SMs.  Results equal skv_paged_attn_fwd on each plan.  The two plans' merge passes
 *   follow on the same stream.  Errors: as skv_paged_attn_fwd; SKV_ERR_UNSUPPORTED for another
 *   kernel choice or an e4m3 cache.
 * ----------------------------------------------------------------------------------------- */
SKV_API skv_status skv_pod_attn_fwd(const skv_paged_params* p, const int32_t* decode_plan_d,
                                    const skv_plan_info* decode_info, const int32_t* prefill_plan_d,
                                    const skv_plan_info* prefill_info, float* prefill_o_part,
                                    float* prefill_lse_part, skv_stream_t stream);

/* -------------------------------------------------------------------------------------------
 * skv_causal_tables -- host planner for causal / multi-token attention.  The n_q query tokens of
 *   request r (rows qo_indptr[r] .. qo_indptr[r+1]) are its last n_q positions; query token i
 *   sees keys t <= L_r - n_q + i (multi-token prediction decode, mentioned on the FlashInfer PR
 *   #3309 page; causal prefill).  The call splits this into two unmasked problems whose exact
 *   merge (skv_merge_states, two states per query row) is the causal result:
 *     prefix -- request r keeps its first ceil(Lp_r / P) pages, Lp_r = min(L_r, max(0, L_r - n_q + 1)):
 *               the keys every query token of r sees (same query rows, same page size);
 *     diag   -- one request per query row j = qo_indptr[r] + i, page size 1, whose "pages" are the
 *               token rows page * P + slot of keys [Lp_r, L_r - n_q + 1 + i): the keys token i sees
 *               beyond the prefix (none for i = 0).  Run it on a [num_pages * P, 1, ...] view of the
 *               cache (pages back to back) with num_pages * P rows.
 *   Outputs are host arrays the caller allocates: prefix_indptr [batch+1], prefix_indices
 *   [kv_indptr_h[batch]], prefix_last [batch]; diag_indptr [total_q+1], diag_last [total_q] (all 1),
 *   diag_rows [diag_capacity].  *diag_rows_needed receives the number of diagonal rows; if it
 *   exceeds diag_capacity nothing else is written and SKV_ERR_WORKSPACE is returned (size the
 *   buffer with a first call of capacity 0).  Token rows must fit int32 (SKV_ERR_UNSUPPORTED).
 * ----------------------------------------------------------------------------------------- */
SKV_API skv_status skv_causal_tables(int32_t batch, const int32_t* qo_indptr_h, const int32_t* kv_indptr_h,
                                     const int32_t* kv_indices_h, const int32_t* kv_last_page_len_h,
                                     int32_t page_size, int32_t* prefix_indptr_h, int32_t* prefix_indices_h,
                                     int32_t* prefix_last_h, int32_t* diag_indptr_h, int32_t* diag_rows_h,
                                     int32_t* diag_last_h, int64_t diag_capacity, int64_t* diag_rows_needed);

/* -------------------------------------------------------------------------------------------
 * skv_mla_splice -- the fetch primitive's local compute.  "Move the Query, Not the Cache"
 *   (Methodology, primitive comparison): fetch brings a whole KV chunk to the requester, adapts
 *   its positions ("splice") and attends locally; the problem statement describes the
 *   adaptation as re-rotating cached position encodings to new offsets.
 *
 *   For each chunk c and token t in [0, chunks_h[c].n_tokens): the latent row at logical
 *   position chunks_h[c].src_start + t of the source page list (page
 *   src_pages[pos / src_page_size], slot pos % src_page_size) is written at logical position
 *   chunks_h[c].dst_start + t of the destination page list (same rule with the dst_ fields).
 *   The 512-d latent (ckv) is copied bit for bit.  The 64-d rope part (kpe) holds keys rotated
 *   to their old positions; each of its 32 pairs (a, b) turns by delta_pos * theta_i, with the
 *   chunk's delta_pos (new position - old position):  a' = a cos - b sin, b' = a sin + b cos;
 *   theta_i = inv_freq[i] when inv_freq (device, 32 floats) is given, else
 *   rope_theta^(-2i/64).  Pairs are (2i, 2i+1) for SKV_ROPE_INTERLEAVED and (i, i+32) for
 *   SKV_ROPE_HALVES.  Angles are formed in fp64, the rotation in fp32, results rounded to bf16
 *   (nearest even).  All chunks of one call run in one launch (up to 64 chunks per launch).
 *
 *   Caches: bf16 only (kv_dtype SKV_BF16; anything else is SKV_ERR_UNSUPPORTED).  Layout as in
 *   skv_mla_params: ckv(page, slot, d) = ckv[page*stride[0] + slot*stride[1] + d], strides in
 *   elements and multiples of 8 (16 bytes), base pointers 16-byte aligned (SKV_ERR_ALIGNMENT).
 *   The page lists must cover every position a chunk names.  A row may be read and written by
 *   the same token (an in-place re-rotation, source = destination); otherwise no row written by
 *   the call may be read or written by any other token of the call.  A page id outside
 *   [0, *_num_pages) reports SKV_DEV_PAGE_OOB in *status and that token is skipped.  Chunks
 *   with no tokens are allowed; a call with none launches nothing.  chunks_h is a host array
 *   that the call reads before it returns.
 * ----------------------------------------------------------------------------------------- */
#define SKV_ROPE_INTERLEAVED 0
#define SKV_ROPE_HALVES 1

typedef struct {
  const void* src_ckv;        /* bf16 latent rows of the source pages                          */
  const void* src_kpe;        /* bf16 rope rows of the source pages                            */
  int64_t src_ckv_stride[2];  /* (page, slot) strides in elements                              */
  int64_t src_kpe_stride[2];
  const int32_t* src_pages;   /* source page list                                              */
  int32_t src_num_pages;      /* page ids must lie in [0, src_num_pages)                      */
  int32_t src_page_size;
  void* dst_ckv;
  void* dst_kpe;
  int64_t dst_ckv_stride[2];
  int64_t dst_kpe_stride[2];
  const int32_t* dst_pages;
  int32_t dst_num_pages;
  int32_t dst_page_size;
  float rope_theta;           /* frequency base when inv_freq is NULL (> 0)                    */
  int32_t rope_layout;        /* SKV_ROPE_INTERLEAVED or SKV_ROPE_HALVES                       */
  const float* inv_freq;      /* optional device [32] per-pair frequencies                     */
  int32_t kv_dtype;           /* SKV_BF16                                                      */
  int32_t* status;            /* optional device status word                                   */
} skv_splice_params;

typedef struct {
  int64_t src_start;          /* logical position of the chunk's first token, source list     */
  int64_t dst_start;          /* logical position of its first token, destination list        */
  int64_t n_tokens;
  int64_t delta_pos;          /* new position - old position of every token of the chunk      */
} skv_splice_chunk;

SKV_API skv_status skv_mla_splice(const skv_splice_params* p, const skv_splice_chunk* chunks_h,
                                  int32_t num_chunks, skv_stream_t stream);

/* -------------------------------------------------------------------------------------------
 * skv_paged_kv_gather -- test hook for the page-table walk: copies the logical K and V of every
 *   request, through the same address generation the attention kernels use, into dense
 *   k_out / v_out [sum_r L_r, Hk, D] bf16 (request r's tokens start at row token_indptr[r],
 *   token_indptr device [batch+1] = prefix sums of L_r).  Bit-exact by construction.
 * ----------------------------------------------------------------------------------------- */
SKV_API skv_status skv_paged_kv_gather(const skv_paged_params* p, const int32_t* token_indptr,
                               int64_t total_tokens, void* k_out, void* v_out,
                               skv_stream_t stream);

/* -------------------------------------------------------------------------------------------
 * skv_test_wait_timeout -- test hook for device-side failure detection: one CTA waits on an
 *   mbarrier that is never arrived on, with the bounded wait every tensor-core kernel uses, and
 *   gives up after limit_ns (<= 10 s) writing SKV_DEV_TIMEOUT to the device status word.  The
 *   context stays usable (nothing traps or hangs).
 * ----------------------------------------------------------------------------------------- */
SKV_API skv_status skv_test_wait_timeout(int32_t* status, int64_t limit_ns, skv_stream_t stream);

/* Fold ratio used by the MLA kernels: the largest divisor F of q_len with num_heads * F <=
 * tile_m (F >= 1).  Rows per work item = num_heads * F; work items per request = q_len / F. */
SKV_API int32_t skv_mla_fold_ratio(int32_t num_heads, int32_t q_len, int32_t tile_m);

SKV_API const char* skv_status_str(int32_t status);
SKV_API int32_t skv_version(void);

#ifdef __cplusplus
}
#endif
#endif /* SPLITKV_H_ */
