// Paged GQA attention for many query rows per KV head on the tensor cores: the kernel (its body,
// with the design notes, is in gqa_tc_prefill_body.cuh) and its host launcher.
#include <cudaTypedefs.h>

#include <algorithm>
#include <mutex>

#include "gqa_tc_prefill_body.cuh"

namespace skv {

using namespace prefill;

namespace {

template <typename OutT>
__global__ void __launch_bounds__(kThreads, 1)
gqa_tc_prefill_kernel(const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap vmap,
                      const __grid_constant__ CUtensorMap qmap, PArgs a, const WorkItem* __restrict__ work) {
  prefill_body<OutT>(kmap, vmap, qmap, a, work, blockIdx.x);
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn_p() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

bool make_map_p(CUtensorMap* m, const void* base, int rank, const cuuint64_t* dims, const cuuint64_t* strides_bytes,
                const cuuint32_t* box) {
  auto fn = encode_fn_p();
  if (fn == nullptr) return false;
  cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, const_cast<void*>(base), dims, strides_bytes, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <typename OutT>
int launch_p(const CUtensorMap& km, const CUtensorMap& vm, const CUtensorMap& qm, const PArgs& a,
             const WorkItem* work, cudaStream_t s) {
  const int smem = Smem::total + 1024;
  static DeviceSmemAttr attr;  // per device: the attribute belongs to the current device
  if (const int e = attr.ensure(reinterpret_cast<const void*>(gqa_tc_prefill_kernel<OutT>), smem)) return e;
  gqa_tc_prefill_kernel<OutT><<<a.num_units, kThreads, smem, s>>>(km, vm, qm, a, work);
  return (int)cudaGetLastError();
}

}  // namespace

bool gqa_tc_prefill_supported(int head_dim, int page_size, int group) {
  const bool page_ok = page_size >= 8 && (page_size <= kTile ? kTile % page_size == 0 : page_size % kTile == 0);
  return head_dim == kD && page_ok && group >= 1 && group <= kRows && kRows % group == 0;
}

int prefill::prepare(const skv_paged_params& p, int num_work, int q_tile, CUtensorMap* maps, PArgs* a) {
  const int g = p.num_qo_heads / p.num_kv_heads;
  if (!gqa_tc_prefill_supported(p.head_dim, p.page_size, g) || q_tile * g != kRows) return (int)cudaErrorInvalidValue;
  const int box_rows = std::min(p.page_size, kTile);
  {
    const cuuint64_t dims[4] = {(cuuint64_t)kD, (cuuint64_t)p.num_kv_heads, (cuuint64_t)p.page_size,
                                (cuuint64_t)std::max(1, p.num_pages)};
    const cuuint32_t box[4] = {64, 1, (cuuint32_t)box_rows, 1};
    const cuuint64_t ks[3] = {(cuuint64_t)p.k_stride[2] * 2, (cuuint64_t)p.k_stride[1] * 2,
                              (cuuint64_t)p.k_stride[0] * 2};
    const cuuint64_t vs[3] = {(cuuint64_t)p.v_stride[2] * 2, (cuuint64_t)p.v_stride[1] * 2,
                              (cuuint64_t)p.v_stride[0] * 2};
    if (!make_map_p(&maps[0], p.k_cache, 4, dims, ks, box)) return (int)cudaErrorInvalidValue;
    if (!make_map_p(&maps[1], p.v_cache, 4, dims, vs, box)) return (int)cudaErrorInvalidValue;
  }
  {
    const cuuint64_t dims[3] = {(cuuint64_t)kD, (cuuint64_t)p.num_qo_heads, (cuuint64_t)std::max(1, p.total_q)};
    const cuuint64_t st[2] = {(cuuint64_t)kD * 2, (cuuint64_t)p.num_qo_heads * kD * 2};
    const cuuint32_t box[3] = {64, (cuuint32_t)g, (cuuint32_t)q_tile};
    if (!make_map_p(&maps[2], p.q, 3, dims, st, box)) return (int)cudaErrorInvalidValue;
  }
  a->kv_indptr = p.kv_indptr;
  a->kv_indices = p.kv_indices;
  a->last = p.kv_last_page_len;
  a->num_pages = p.num_pages;
  a->page_size = p.page_size;
  a->hq = p.num_qo_heads;
  a->hk = p.num_kv_heads;
  a->g = g;
  a->q_tile = q_tile;
  a->num_units = num_work * p.num_kv_heads;
  a->scale_log2 = p.sm_scale * kLog2e;
  a->o = p.o;
  a->lse = p.lse;
  a->o_part = p.o_part;
  a->lse_part = p.lse_part;
  a->status = p.status;
  return 0;
}

int launch_gqa_tc_prefill(const skv_paged_params& p, const WorkItem* work, int num_work, int q_tile, cudaStream_t s) {
  if (num_work == 0) return 0;
  CUtensorMap maps[3];
  PArgs a;
  if (const int e = prefill::prepare(p, num_work, q_tile, maps, &a)) return e;
  return p.o_dtype == SKV_BF16 ? launch_p<__nv_bfloat16>(maps[0], maps[1], maps[2], a, work, s)
                               : launch_p<float>(maps[0], maps[1], maps[2], a, work, s);
}

}  // namespace skv
