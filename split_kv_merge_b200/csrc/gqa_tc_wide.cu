// Paged GQA decode, all KV heads of a work item in one CTA (tcgen05 + TMEM, TMA page staging):
// the kernel (its body, with the design notes, is in gqa_tc_wide_body.cuh) and its host launcher.
#include <cudaTypedefs.h>

#include <mutex>

#include "gqa_tc_wide_body.cuh"

namespace skv {

using namespace wide;

namespace {

template <int G, typename OutT>
__global__ void __launch_bounds__(kThreads, 1)
gqa_tc_wide_kernel(const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap vmap,
                   const __grid_constant__ CUtensorMap qmap, WArgs a, const WorkItem* __restrict__ work) {
  wide_body<G, OutT>(kmap, vmap, qmap, a, work, blockIdx.x);
}

// ------------------------------------------------------------------------------ host side
PFN_cuTensorMapEncodeTiled_v12000 encode_fn_w() {
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

bool make_map_w(CUtensorMap* m, const void* base, int rank, const cuuint64_t* dims, const cuuint64_t* strides_bytes,
                const cuuint32_t* box) {
  auto fn = encode_fn_w();
  if (fn == nullptr) return false;
  cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, const_cast<void*>(base), dims, strides_bytes, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int G, typename OutT>
int launch_w(const CUtensorMap& km, const CUtensorMap& vm, const CUtensorMap& qm, const WArgs& a,
             const WorkItem* work, cudaStream_t s) {
  const int smem = Smem::total + 1024;
  static DeviceSmemAttr attr;  // per device: the attribute belongs to the current device
  if (const int e = attr.ensure(reinterpret_cast<const void*>(gqa_tc_wide_kernel<G, OutT>), smem)) return e;
  gqa_tc_wide_kernel<G, OutT><<<a.num_ctas, kThreads, smem, s>>>(km, vm, qm, a, work);
  return (int)cudaGetLastError();
}

template <typename OutT>
int launch_w_g(int g, const CUtensorMap& km, const CUtensorMap& vm, const CUtensorMap& qm, const WArgs& a,
               const WorkItem* work, cudaStream_t s) {
  switch (g) {
    case 8: return launch_w<8, OutT>(km, vm, qm, a, work, s);
    case 4: return launch_w<4, OutT>(km, vm, qm, a, work, s);
    case 2: return launch_w<2, OutT>(km, vm, qm, a, work, s);
    case 1: return launch_w<1, OutT>(km, vm, qm, a, work, s);
    default: return (int)cudaErrorInvalidValue;
  }
}

}  // namespace

bool gqa_tc_wide_supported(int head_dim, int page_size, int num_kv_heads, int group, int q_tile) {
  return head_dim == kD && num_kv_heads == kHk && group * q_tile == 8 && page_size >= kTok &&
         page_size <= 256 && page_size % kTok == 0;
}

int wide::prepare(const skv_paged_params& p, const int32_t* cta_indptr, int num_ctas, int q_tile, CUtensorMap* maps,
                  WArgs* a) {
  const int g = p.num_qo_heads / p.num_kv_heads;
  if (!gqa_tc_wide_supported(p.head_dim, p.page_size, p.num_kv_heads, g, q_tile)) return (int)cudaErrorInvalidValue;
  {
    // dimension order (d, slot, head, page): a box of 16 slots x 8 heads lands head-major
    const cuuint64_t dims[4] = {(cuuint64_t)kD, (cuuint64_t)p.page_size, (cuuint64_t)kHk,
                                (cuuint64_t)std::max(1, p.num_pages)};
    const cuuint32_t box[4] = {64, (cuuint32_t)kTok, (cuuint32_t)kHk, 1};
    const cuuint64_t ks[3] = {(cuuint64_t)p.k_stride[1] * 2, (cuuint64_t)p.k_stride[2] * 2,
                              (cuuint64_t)p.k_stride[0] * 2};
    const cuuint64_t vs[3] = {(cuuint64_t)p.v_stride[1] * 2, (cuuint64_t)p.v_stride[2] * 2,
                              (cuuint64_t)p.v_stride[0] * 2};
    if (!make_map_w(&maps[0], p.k_cache, 4, dims, ks, box)) return (int)cudaErrorInvalidValue;
    if (!make_map_w(&maps[1], p.v_cache, 4, dims, vs, box)) return (int)cudaErrorInvalidValue;
  }
  {
    // q viewed as (d, j < g, token, kv head): a box (64, g, q_tile, 8) lands as rows
    // kv_head * (q_tile * g) + token * g + j, the column order of S^T
    const cuuint64_t dims[4] = {(cuuint64_t)kD, (cuuint64_t)g, (cuuint64_t)std::max(1, p.total_q), (cuuint64_t)kHk};
    const cuuint64_t st[3] = {(cuuint64_t)kD * 2, (cuuint64_t)p.num_qo_heads * kD * 2, (cuuint64_t)g * kD * 2};
    const cuuint32_t box[4] = {64, (cuuint32_t)g, (cuuint32_t)q_tile, (cuuint32_t)kHk};
    if (!make_map_w(&maps[2], p.q, 4, dims, st, box)) return (int)cudaErrorInvalidValue;
  }
  a->kv_indptr = p.kv_indptr;
  a->kv_indices = p.kv_indices;
  a->last = p.kv_last_page_len;
  a->num_pages = p.num_pages;
  a->page_size = p.page_size;
  a->hq = p.num_qo_heads;
  a->q_tile = q_tile;
  a->num_ctas = num_ctas;
  a->cta_indptr = cta_indptr;
  a->scale_log2 = p.sm_scale * kLog2e;
  a->o = p.o;
  a->lse = p.lse;
  a->o_part = p.o_part;
  a->lse_part = p.lse_part;
  a->status = p.status;
  return 0;
}

int launch_gqa_tc_wide(const skv_paged_params& p, const WorkItem* work, const int32_t* cta_indptr, int num_ctas,
                       int q_tile, cudaStream_t s) {
  if (num_ctas == 0) return 0;
  CUtensorMap maps[3];
  WArgs a;
  if (const int e = wide::prepare(p, cta_indptr, num_ctas, q_tile, maps, &a)) return e;
  const int g = p.num_qo_heads / p.num_kv_heads;
  return p.o_dtype == SKV_BF16 ? launch_w_g<__nv_bfloat16>(g, maps[0], maps[1], maps[2], a, work, s)
                               : launch_w_g<float>(g, maps[0], maps[1], maps[2], a, work, s);
}

}  // namespace skv
