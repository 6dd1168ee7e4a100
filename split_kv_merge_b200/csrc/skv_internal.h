// Internal layout of plans and the launcher interface between the C ABI (api.cu) and the
// kernel translation units.  Not part of the public ABI.
#pragma once
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>

#include "../../include/splitkv.h"

namespace skv {

// One work item = one CTA (per KV head for GQA): request r, query tokens
// [q_start, q_start + q_count) (global rows of q), logical pages [page_begin, page_end) of the
// request.  part_row < 0: write O/LSE directly; otherwise the partial of query token i (0-based
// within the item) goes to row part_row + i * part_stride of o_part / lse_part.
struct WorkItem {
  int32_t r, q_start, q_count, page_begin, page_end, part_row, part_stride, split;
};
static_assert(sizeof(WorkItem) == 32, "work item is 8 int32 words");

// One merge item = one output row combined from state_count consecutive partial rows.
struct MergeItem {
  int32_t out_row, state_begin, state_count, pad;
};
static_assert(sizeof(MergeItem) == 16, "merge item is 4 int32 words");

enum KernelId : int32_t {
  KERNEL_GQA_SIMT = 1,
  KERNEL_GQA_TC_DECODE = 2,
  KERNEL_GQA_TC_WIDE = 3,
  KERNEL_GQA_TC_PREFILL = 4,  // tensor-core, 128 query rows (tokens x group heads) per unit
  KERNEL_MLA_SIMT = 11,
  KERNEL_MLA_TC16 = 12,  // tensor-core MLA, 16 query rows per unit (bf16 or e4m3 cache)
  KERNEL_MLA_TC32 = 13,  // tensor-core MLA, 32 query rows per unit (bf16 or e4m3 cache)
  KERNEL_MLA_TC64 = 14,  // tensor-core MLA, 64 query rows per unit, CTA groups per KV slice (bf16)
};

// Host caches of per-device state.  cudaFuncSetAttribute and device attributes belong to the
// device current at the call, so each cache is indexed by that device's ordinal: a launch on a
// second GPU raises the kernel's shared-memory limit there too.
constexpr int kMaxCachedDevices = 64;

inline int current_device() {
  int d = 0;
  return cudaGetDevice(&d) == cudaSuccess ? d : -1;
}

// One per kernel instantiation: raises the kernel's dynamic shared-memory limit to `bytes` on
// the current device, once per device (devices beyond the table set it on every launch).
class DeviceSmemAttr {
 public:
  int ensure(const void* func, int bytes) {
    const int dev = current_device();
    if (dev < 0) return (int)cudaErrorNoDevice;
    const bool cached = dev < kMaxCachedDevices;
    if (cached && done_[dev].load(std::memory_order_acquire) == bytes) return 0;
    const cudaError_t e = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e != cudaSuccess) return (int)e;
    if (cached) done_[dev].store(bytes, std::memory_order_release);
    return 0;
  }

 private:
  std::atomic<int> done_[kMaxCachedDevices] = {};
};

// SM count of the current device (cached per device; 148 if the query fails).
inline int device_sm_count() {
  static std::atomic<int> cache[kMaxCachedDevices];
  const int dev = current_device();
  if (dev >= 0 && dev < kMaxCachedDevices) {
    const int n = cache[dev].load(std::memory_order_relaxed);
    if (n > 0) return n;
  }
  int n = 0;
  if (dev < 0 || cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) {
    cudaGetLastError();
    return 148;
  }
  if (dev < kMaxCachedDevices) cache[dev].store(n, std::memory_order_relaxed);
  return n;
}

// Plan words: [work items (8 words each)] [merge items (4 words each)].
inline int64_t plan_words(int32_t num_work, int32_t num_merge) {
  return 8LL * num_work + 4LL * num_merge;
}

// Launchers (host functions defined next to their kernels).  Return cudaError_t as int.
int launch_gqa_simt(const skv_paged_params& p, const WorkItem* work, int num_work, int q_tile,
                    bool same_kv, cudaStream_t s);
bool gqa_tc_decode_supported(int head_dim, int page_size, int group, int q_tile);
int launch_gqa_tc_decode(const skv_paged_params& p, const WorkItem* work, int num_work, int q_tile,
                         cudaStream_t s);
bool gqa_tc_wide_supported(int head_dim, int page_size, int num_kv_heads, int group, int q_tile);
int launch_gqa_tc_wide(const skv_paged_params& p, const WorkItem* work, const int32_t* cta_indptr, int num_ctas,
                       int q_tile, cudaStream_t s);
int launch_gqa_tc_wide_fp8(const skv_paged_params& p, const WorkItem* work, const int32_t* cta_indptr, int num_ctas,
                           int q_tile, cudaStream_t s);
int launch_gqa_pod(const skv_paged_params& dp, const WorkItem* dwork, const int32_t* cta_indptr, int num_ctas,
                   int dq_tile, const skv_paged_params& pp, const WorkItem* pwork, int pnum_work, int pq_tile,
                   cudaStream_t s);
bool gqa_tc_prefill_supported(int head_dim, int page_size, int group);
int launch_gqa_tc_prefill(const skv_paged_params& p, const WorkItem* work, int num_work, int q_tile,
                          cudaStream_t s);
int launch_mla_simt(const skv_mla_params& p, const WorkItem* work, int num_work, int q_tile,
                    cudaStream_t s);
bool mla_tc_supported(int kv_dtype, int page_size, int num_heads, int rows_per_unit);
int mla_tc_tile_tokens();
bool mla_tc64_supported(int kv_dtype, int page_size, int num_heads);
int launch_mla_tc64(const skv_mla_params& p, const WorkItem* work, const int32_t* cta_indptr, int num_ctas,
                    int q_tile, cudaStream_t s);
int launch_mla_tc(const skv_mla_params& p, const WorkItem* work, const int32_t* cta_indptr, int num_ctas,
                  int q_tile, int rows_per_unit, cudaStream_t s);
bool mla_tc_fp8_supported(int page_size, int num_heads, int rows_per_unit);
int launch_mla_tc_fp8(const skv_mla_params& p, const WorkItem* work, const int32_t* cta_indptr, int num_ctas,
                      int q_tile, int rows_per_unit, cudaStream_t s);
int launch_wait_timeout(int32_t* status, uint64_t limit_ns, cudaStream_t s);
int launch_merge(const float* o_states, const float* lse_states, const int32_t* state_indptr,
                 int32_t num_states, const MergeItem* items, int64_t num_rows, int32_t num_heads,
                 int32_t head_dim, void* o_out, int32_t o_dtype, float* lse_out, cudaStream_t s);
int launch_splice(const skv_splice_params& p, const skv_splice_chunk* chunks, int num_chunks, cudaStream_t s);
int launch_gather(const skv_paged_params& p, const int32_t* token_indptr, int64_t total_tokens,
                  void* k_out, void* v_out, bool same_kv, cudaStream_t s);

}  // namespace skv
