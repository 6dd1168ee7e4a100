// skv_paged_attn_fwd_static_scratch: skv_paged_attn_fwd for callers that cannot allocate device
// memory.  The split partials (o_part / lse_part), which the regular entry point takes from the
// caller, live here in one file-scope device array instead.
//
// Who needs it: a serving engine that hands nearly all device memory to its KV cache at start-up
// and keeps no allocator on the decode path, or a plain-C / foreign-runtime caller that has no
// device allocator of its own.  (cudaMalloc would also synchronize the device, which a decode step
// measured in microseconds cannot afford.)  Such a caller passes only inputs and outputs.
//
// Contract:
//  - The array is kStaticScratchBytes (32 MiB) per GPU, reserved on every GPU that loads this
//    library until the process exits.  A plan whose partials need more is rejected with
//    SKV_ERR_WORKSPACE before anything is launched.
//  - The first call on a device resolves the array's device address with
//    cudaGetSymbolAddress (device current at that time) and caches it; make that first call
//    before any stream capture.  Nothing here allocates (no cudaMalloc / cudaFree / library
//    allocation).
//  - Every call shares the one array and it keeps the last call's contents.  The attention
//    kernel writes every partial row before the merge reads it, so nothing needs clearing;
//    calls that overlap on the GPU (different streams) race on the array.
//  - `info` must be the summary the planner returned with `plan_d`: the size check uses
//    info->num_partial_rows, the kernels the partial rows stored in plan_d.
#include <mutex>

#include "skv_internal.h"

namespace {

constexpr size_t kStaticScratchBytes = size_t(32) << 20;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_split_scratch[kStaticScratchBytes];

void* g_scratch_dev[kMaxDevices];
cudaError_t g_scratch_err[kMaxDevices];
std::once_flag g_scratch_once[kMaxDevices];

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

}  // namespace

extern "C" {

SKV_API skv_status skv_paged_attn_fwd_static_scratch(const skv_paged_params* p, const int32_t* plan_d,
                                                     const skv_plan_info* info, skv_stream_t stream) {
  if (p == nullptr || info == nullptr) return SKV_ERR_INVALID;
  if (info->num_partial_rows < 0 || p->num_qo_heads < 1 || p->head_dim < 1) return SKV_ERR_INVALID;
  const size_t rows = (size_t)info->num_partial_rows;
  const size_t o_bytes = align256(rows * (size_t)p->num_qo_heads * (size_t)p->head_dim * sizeof(float));
  const size_t lse_bytes = align256(rows * (size_t)p->num_qo_heads * sizeof(float));
  if (o_bytes + lse_bytes > kStaticScratchBytes) return SKV_ERR_WORKSPACE;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return SKV_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return SKV_ERR_UNSUPPORTED;
  // host code may not use g_split_scratch as a pointer: resolve its device address once per device
  std::call_once(g_scratch_once[dev], [dev] {
    g_scratch_err[dev] = cudaGetSymbolAddress(&g_scratch_dev[dev], g_split_scratch);
  });
  if (g_scratch_err[dev] != cudaSuccess || g_scratch_dev[dev] == nullptr) return SKV_ERR_CUDA;
  skv_paged_params q = *p;
  unsigned char* base = static_cast<unsigned char*>(g_scratch_dev[dev]);
  q.o_part = rows ? reinterpret_cast<float*>(base) : nullptr;
  q.lse_part = rows ? reinterpret_cast<float*>(base + o_bytes) : nullptr;
  return skv_paged_attn_fwd(&q, plan_d, info, stream);
}

}  // extern "C"
