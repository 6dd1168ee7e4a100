// merge_states: exact combination of split partials (O_j, LSE_j) into (O, LSE).
//   M = max_j LSE_j,  LSE = M + ln sum_j exp(LSE_j - M),  O = sum_j exp(LSE_j - LSE) O_j
// (the merge "via online softmax" of the route primitive, "Move the Query, Not the Cache",
// Methodology; the in-CTA partial + row-statistics merge of the FlashInfer PR #5597 page,
// section 3).  HBM-bound: one CTA per output row streams its S x H x D partial floats with
// 16-byte loads; per-(state, head) weights are computed once into shared memory.
#include <algorithm>

#include "tc_ptx.cuh"

namespace skv {

namespace {

constexpr int kMergeThreads = 128;
constexpr int kStateChunk = 32;
constexpr int kMaxHeadsPerBlock = 8;

// One CTA per (output row, group of hg heads): hg * D = 512 floats, one float4 per thread per
// state.  Pass 1 (one warp per head): M and LSE over the row's states.  Pass 2: per state chunk,
// the weights exp(LSE_j - LSE) go to shared memory and every thread accumulates its float4.
template <typename OutT>
__global__ void __launch_bounds__(kMergeThreads)
merge_kernel(const float* __restrict__ o_states, const float* __restrict__ lse_states,
             const int32_t* __restrict__ state_indptr, int num_states, const MergeItem* __restrict__ items,
             int64_t num_rows, int H, int D, int hg, OutT* __restrict__ o_out, float* __restrict__ lse_out) {
  __shared__ float lse_s[kMaxHeadsPerBlock];
  __shared__ float w_s[kStateChunk][kMaxHeadsPerBlock];
  const int64_t row = blockIdx.x;
  const int h0 = blockIdx.y * hg;
  const int nh = min(hg, H - h0);
  int64_t out_row, base, jstride;
  int S;
  if (items != nullptr) {
    const MergeItem it = items[row];
    out_row = it.out_row; base = it.state_begin; S = it.state_count; jstride = 1;
  } else if (state_indptr != nullptr) {
    out_row = row; base = state_indptr[row]; S = state_indptr[row + 1] - state_indptr[row]; jstride = 1;
  } else {
    out_row = row; base = row; S = num_states; jstride = num_rows;
  }
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int hh = warp; hh < nh; hh += kMergeThreads / 32) {
    const int h = h0 + hh;
    float M = -INFINITY;
    for (int j = lane; j < S; j += 32) M = fmaxf(M, lse_states[(base + j * jstride) * H + h]);
    M = warp_max(M);
    float tot = 0.f;
    if (M != -INFINITY)
      for (int j = lane; j < S; j += 32) {
        const float lj = lse_states[(base + j * jstride) * H + h];
        tot += (lj == -INFINITY) ? 0.f : exp2f((lj - M) * kLog2e);
      }
    tot = warp_sum(tot);
    const float lse = (M == -INFINITY) ? -INFINITY : M + log2f(tot) * kLn2;
    if (lane == 0) {
      lse_s[hh] = lse;
      if (lse_out != nullptr) lse_out[out_row * H + h] = lse;
    }
  }
  __syncthreads();
  const int n4 = nh * D / 4;  // float4 of this block
  for (int e0 = 0; e0 < n4; e0 += kMergeThreads) {
    const int e = e0 + threadIdx.x;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    const int hh = (e * 4) / D;
    for (int j0 = 0; j0 < S; j0 += kStateChunk) {
      const int nj = min(kStateChunk, S - j0);
      __syncthreads();
      for (int idx = threadIdx.x; idx < nj * nh; idx += kMergeThreads) {
        const int j = idx / nh, k = idx % nh;
        const float lj = lse_states[(base + (j0 + j) * jstride) * H + h0 + k];
        const float L = lse_s[k];
        w_s[j][k] = (lj == -INFINITY || L == -INFINITY) ? 0.f : exp2f((lj - L) * kLog2e);
      }
      __syncthreads();
      if (e < n4) {
        for (int j = 0; j < nj; ++j) {
          const float4* src = reinterpret_cast<const float4*>(
              o_states + ((base + (j0 + j) * jstride) * (int64_t)H + h0) * D);
          const float wt = w_s[j][hh];
          const float4 x = __ldg(src + e);
          acc.x = fmaf(wt, x.x, acc.x);
          acc.y = fmaf(wt, x.y, acc.y);
          acc.z = fmaf(wt, x.z, acc.z);
          acc.w = fmaf(wt, x.w, acc.w);
        }
      }
    }
    if (e < n4) {
      OutT* dst = o_out + (out_row * (int64_t)H + h0) * D + (int64_t)e * 4;
      store_out(dst + 0, acc.x);
      store_out(dst + 1, acc.y);
      store_out(dst + 2, acc.z);
      store_out(dst + 3, acc.w);
    }
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
  dim3 grid((unsigned)num_rows, (unsigned)((num_heads + hg - 1) / hg));
  if (o_dtype == SKV_BF16)
    merge_kernel<__nv_bfloat16><<<grid, kMergeThreads, 0, s>>>(o_states, lse_states, state_indptr, num_states, items,
                                                              num_rows, num_heads, head_dim, hg,
                                                              static_cast<__nv_bfloat16*>(o_out), lse_out);
  else
    merge_kernel<float><<<grid, kMergeThreads, 0, s>>>(o_states, lse_states, state_indptr, num_states, items,
                                                      num_rows, num_heads, head_dim, hg, static_cast<float*>(o_out),
                                                      lse_out);
  return (int)cudaGetLastError();
}

}  // namespace skv
