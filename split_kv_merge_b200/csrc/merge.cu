// merge_states: exact combination of split partials (O_j, LSE_j) into (O, LSE).
//   M = max_j LSE_j,  LSE = M + ln sum_j exp(LSE_j - M),  O = sum_j exp(LSE_j - LSE) O_j
// (the merge "via online softmax" of the route primitive, "Move the Query, Not the Cache",
// Methodology; the in-CTA partial + row-statistics merge of the FlashInfer PR #5597 page,
// section 3).  HBM-bound: a CTA per output row and group of heads streams its S x H x D partial
// floats with 16-byte loads.
#include <algorithm>

#include "tc_ptx.cuh"

namespace skv {

namespace {

constexpr int kMergeThreads = 128;
constexpr int kStateChunk = 8;
constexpr int kMaxHeadsPerBlock = 8;

// One CTA per (output row, group of hg heads): hg * D = 512 floats, one float4 per thread.  A
// thread issues the LSE and the O float4 of up to kStateChunk states at once (one memory round
// trip for the usual few splits) and combines them with a running maximum:
//   M' = max(M, max_j LSE_j),  l' = l e^(M - M') + sum_j e^(LSE_j - M'),  acc likewise with O_j,
// so after the last chunk LSE = M + ln l and O = acc / l -- the same sums as the two-pass form.
template <typename OutT>
__global__ void __launch_bounds__(kMergeThreads)
merge_kernel(const float* __restrict__ o_states, const float* __restrict__ lse_states,
             const int32_t* __restrict__ state_indptr, int num_states, const MergeItem* __restrict__ items,
             int64_t num_rows, int H, int D, int hg, OutT* __restrict__ o_out, float* __restrict__ lse_out) {
  const int64_t row = blockIdx.x;
  const int h0 = blockIdx.y * hg;
  const int nh = min(hg, H - h0);
  // a plan's merge items are written by the host before the attention launch, never by the
  // preceding grid: read them before waiting on it, so only the partials' loads follow the wait
  int64_t out_row = row, base = row, jstride = num_rows;
  int S = num_states;
  if (items != nullptr) {
    const MergeItem it = items[row];
    out_row = it.out_row; base = it.state_begin; S = it.state_count; jstride = 1;
  }
  tc::grid_dependency_wait();  // the partials of the preceding attention grid are complete
  if (items == nullptr && state_indptr != nullptr) {
    base = state_indptr[row]; S = state_indptr[row + 1] - state_indptr[row]; jstride = 1;
  }
  const int n4 = nh * D / 4;  // float4 of this block
  for (int e = threadIdx.x; e < n4; e += kMergeThreads) {
    const int h = h0 + (e * 4) / D;
    float M = -INFINITY, l = 0.f;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int j0 = 0; j0 < S; j0 += kStateChunk) {
      const int nj = min(kStateChunk, S - j0);
      float lj[kStateChunk];
      float4 x[kStateChunk];
#pragma unroll
      for (int j = 0; j < kStateChunk; ++j) {  // all loads of the chunk in flight together
        if (j < nj) {
          const int64_t st = base + (int64_t)(j0 + j) * jstride;
          lj[j] = __ldg(lse_states + st * H + h);
          x[j] = __ldg(reinterpret_cast<const float4*>(o_states + (st * H + h0) * (int64_t)D) + e);
        } else {
          lj[j] = -INFINITY;
          x[j] = make_float4(0.f, 0.f, 0.f, 0.f);
        }
      }
      float mc = M;
#pragma unroll
      for (int j = 0; j < kStateChunk; ++j) mc = fmaxf(mc, lj[j]);
      if (mc == -INFINITY) continue;  // every state so far is empty
      const float sc = M == -INFINITY ? 0.f : exp2f((M - mc) * kLog2e);
      l *= sc;
      acc.x *= sc;
      acc.y *= sc;
      acc.z *= sc;
      acc.w *= sc;
#pragma unroll
      for (int j = 0; j < kStateChunk; ++j) {
        const float wt = lj[j] == -INFINITY ? 0.f : exp2f((lj[j] - mc) * kLog2e);
        l += wt;
        acc.x = fmaf(wt, x[j].x, acc.x);
        acc.y = fmaf(wt, x[j].y, acc.y);
        acc.z = fmaf(wt, x[j].z, acc.z);
        acc.w = fmaf(wt, x[j].w, acc.w);
      }
      M = mc;
    }
    const float inv = l > 0.f ? 1.f / l : 0.f;
    OutT* dst = o_out + (out_row * (int64_t)H + h0) * D + (int64_t)e * 4;
    store_out(dst + 0, acc.x * inv);
    store_out(dst + 1, acc.y * inv);
    store_out(dst + 2, acc.z * inv);
    store_out(dst + 3, acc.w * inv);
    if (lse_out != nullptr && (e * 4) % D == 0)
      lse_out[out_row * H + h] = l > 0.f ? M + log2f(l) * kLn2 : -INFINITY;
  }
}

// Test hook for failure detection: waits on an mbarrier that nothing ever arrives on, with the
// same bounded wait the tensor-core kernels use (limit `limit_ns`), and must come back with
// SKV_DEV_TIMEOUT in the status word instead of hanging.
__global__ void wait_timeout_kernel(int32_t* status, uint64_t limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  const uint32_t b = tc::smem_u32(&bar);
  if (threadIdx.x == 0) {
    tc::mbar_init(b, 1);
    abort_flag = 0;
    tc::fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const uint64_t t0 = tc::globaltimer_ns();
    while (!tc::mbar_try_wait(b, 0)) {
      if (tc::globaltimer_ns() - t0 > limit_ns) {
        report(status, SKV_DEV_TIMEOUT);
        break;
      }
    }
  }
}

}  // namespace

int launch_wait_timeout(int32_t* status, uint64_t limit_ns, cudaStream_t s) {
  wait_timeout_kernel<<<1, 32, 0, s>>>(status, limit_ns);
  return (int)cudaGetLastError();
}

int launch_merge(const float* o_states, const float* lse_states, const int32_t* state_indptr,
                 int32_t num_states, const MergeItem* items, int64_t num_rows, int32_t num_heads,
                 int32_t head_dim, void* o_out, int32_t o_dtype, float* lse_out, cudaStream_t s) {
  if (num_rows == 0) return 0;
  if (head_dim % 4 != 0) return (int)cudaErrorInvalidValue;
  const int hg = std::max(1, std::min(kMaxHeadsPerBlock, 512 / head_dim));
  // programmatic stream serialization: the merge may launch while the attention grid that wrote
  // the partials is finishing; merge_kernel waits for that grid before its first read
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)num_rows, (unsigned)((num_heads + hg - 1) / hg));
  cfg.blockDim = dim3(kMergeThreads);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e;
  if (o_dtype == SKV_BF16)
    e = cudaLaunchKernelEx(&cfg, merge_kernel<__nv_bfloat16>, o_states, lse_states, state_indptr, num_states, items,
                           num_rows, num_heads, head_dim, hg, static_cast<__nv_bfloat16*>(o_out), lse_out);
  else
    e = cudaLaunchKernelEx(&cfg, merge_kernel<float>, o_states, lse_states, state_indptr, num_states, items, num_rows,
                           num_heads, head_dim, hg, static_cast<float*>(o_out), lse_out);
  return (int)e;
}

}  // namespace skv
