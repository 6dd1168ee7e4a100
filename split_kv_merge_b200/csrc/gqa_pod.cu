// POD: one batch that mixes decode and prefill requests in ONE attention launch (FlashInfer PR
// #4736 page, section 1: batch_pod.cu fuses prefill and decode work in one kernel).
//
// The batch is planned as two subsets of its requests (skv_plan_paged_subset): decode requests on
// the all-KV-heads decode plan, whose slices were balanced over `num_ctas` persistent CTAs, and
// prefill requests on 128-row prefill units.  The launch has num_ctas + prefill units CTAs:
// CTA c < num_ctas runs the decode body over its slice (gqa_tc_wide_body.cuh) and every later CTA
// runs one prefill unit (gqa_tc_prefill_body.cuh).  CTAs start in index order, so the decode
// slices occupy num_ctas SMs for the whole launch and stream the KV cache from HBM, while the
// prefill units fill the other SMs wave after wave on the tensor cores: the HBM-bound and the
// tensor-bound halves of the batch overlap instead of running one after the other.  Each body is
// the same code its own kernel runs, so the results are the same as the two separate launches.
//
// Block shape: the prefill body's 352 threads (11 warps); the decode body uses warps 0-5 and the
// other warps only join its block-wide barriers.  Dynamic shared memory: the larger of the two
// layouts (one CTA per SM either way).
#include <cudaTypedefs.h>

#include <algorithm>

#include "gqa_tc_prefill_body.cuh"
#include "gqa_tc_wide_body.cuh"

namespace skv {

namespace {

static_assert(prefill::kThreads >= wide::kThreads, "the decode body runs inside the prefill block shape");
constexpr int kPodSmem = (wide::Smem::total > prefill::Smem::total ? wide::Smem::total : prefill::Smem::total) + 1024;

template <int G, typename OutT>
__global__ void __launch_bounds__(prefill::kThreads, 1)
gqa_pod_kernel(const __grid_constant__ CUtensorMap dk, const __grid_constant__ CUtensorMap dv,
               const __grid_constant__ CUtensorMap dq, const __grid_constant__ CUtensorMap pk,
               const __grid_constant__ CUtensorMap pv, const __grid_constant__ CUtensorMap pq, wide::WArgs wa,
               const WorkItem* __restrict__ dwork, prefill::PArgs pa, const WorkItem* __restrict__ pwork) {
  if ((int)blockIdx.x < wa.num_ctas)
    wide::wide_body<G, OutT>(dk, dv, dq, wa, dwork, (int)blockIdx.x);
  else
    prefill::prefill_body<OutT>(pk, pv, pq, pa, pwork, (int)blockIdx.x - wa.num_ctas);
}

template <int G, typename OutT>
int launch_pod_t(const CUtensorMap* dm, const CUtensorMap* pm, const wide::WArgs& wa, const WorkItem* dwork,
                 const prefill::PArgs& pa, const WorkItem* pwork, cudaStream_t s) {
  static DeviceSmemAttr attr;  // per device: the attribute belongs to the current device
  if (const int e = attr.ensure(reinterpret_cast<const void*>(gqa_pod_kernel<G, OutT>), kPodSmem)) return e;
  gqa_pod_kernel<G, OutT><<<wa.num_ctas + pa.num_units, prefill::kThreads, kPodSmem, s>>>(
      dm[0], dm[1], dm[2], pm[0], pm[1], pm[2], wa, dwork, pa, pwork);
  return (int)cudaGetLastError();
}

template <typename OutT>
int launch_pod_g(int g, const CUtensorMap* dm, const CUtensorMap* pm, const wide::WArgs& wa, const WorkItem* dwork,
                 const prefill::PArgs& pa, const WorkItem* pwork, cudaStream_t s) {
  switch (g) {
    case 8: return launch_pod_t<8, OutT>(dm, pm, wa, dwork, pa, pwork, s);
    case 4: return launch_pod_t<4, OutT>(dm, pm, wa, dwork, pa, pwork, s);
    case 2: return launch_pod_t<2, OutT>(dm, pm, wa, dwork, pa, pwork, s);
    case 1: return launch_pod_t<1, OutT>(dm, pm, wa, dwork, pa, pwork, s);
    default: return (int)cudaErrorInvalidValue;
  }
}

}  // namespace

int launch_gqa_pod(const skv_paged_params& dp, const WorkItem* dwork, const int32_t* cta_indptr, int num_ctas,
                   int dq_tile, const skv_paged_params& pp, const WorkItem* pwork, int pnum_work, int pq_tile,
                   cudaStream_t s) {
  CUtensorMap dm[3], pm[3];
  wide::WArgs wa;
  prefill::PArgs pa;
  if (const int e = wide::prepare(dp, cta_indptr, num_ctas, dq_tile, dm, &wa)) return e;
  if (const int e = prefill::prepare(pp, pnum_work, pq_tile, pm, &pa)) return e;
  const int g = dq_tile > 0 ? 8 / dq_tile : 0;  // the decode plan's GQA group (g * q_tile = 8)
  return dp.o_dtype == SKV_BF16 ? launch_pod_g<__nv_bfloat16>(g, dm, pm, wa, dwork, pa, pwork, s)
                                : launch_pod_g<float>(g, dm, pm, wa, dwork, pa, pwork, s);
}

}  // namespace skv
