// merge_states: exact combination of split partials (O_j, LSE_j) into (O, LSE).
//   M = max_j LSE_j,  LSE = M + ln sum_j exp(LSE_j - M),  O = sum_j exp(LSE_j - LSE) O_j
// (the merge "via online softmax" of the route primitive, "Move the Query, Not the Cache",
// Methodology; the in-CTA partial + row-statistics merge of the FlashInfer PR #5597 page,
// section 3).  HBM-bound: one CTA per output row streams its S x H x D partial floats with
// 16-byte loads; per-(state, head) weights are computed once into shared memory.
#include "skv_common.cuh"

namespace skv {

namespace {

constexpr int kMergeThreads = 256;
constexpr int kMaxHeads = 256;
constexpr int kStateChunk = 16;

template <typename OutT>
__global__ void __launch_bounds__(kMergeThreads)
merge_kernel(const float* __restrict__ o_states, const float* __restrict__ lse_states,
             const int32_t* __restrict__ state_indptr, int num_states, const MergeItem* __restrict__ items,
             int64_t num_rows, int H, int D, OutT* __restrict__ o_out, float* __restrict__ lse_out) {
  __shared__ float lse_s[kMaxHeads];
  __shared__ float w_s[kStateChunk][kMaxHeads];
  const int64_t row = blockIdx.x;
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
  // pass 1: per head, M and LSE (log2 domain internally)
  for (int h = threadIdx.x; h < H; h += kMergeThreads) {
    float M = -INFINITY;
    for (int j = 0; j < S; ++j) M = fmaxf(M, lse_states[(base + j * jstride) * H + h]);
    float lse = -INFINITY;
    if (M != -INFINITY) {
      float tot = 0.f;
      for (int j = 0; j < S; ++j) {
        const float lj = lse_states[(base + j * jstride) * H + h];
        tot += (lj == -INFINITY) ? 0.f : exp2f((lj - M) * kLog2e);
      }
      lse = M + log2f(tot) * kLn2;
    }
    lse_s[h] = lse;
    if (lse_out != nullptr) lse_out[out_row * H + h] = lse;
  }
  __syncthreads();
  // pass 2: O = sum_j w_j O_j over state chunks
  const int n4 = H * D / 4;
  constexpr int kPer = 8;  // float4 per thread kept in registers per sweep
  for (int e0 = 0; e0 < n4; e0 += kMergeThreads * kPer) {
    float4 acc[kPer];
#pragma unroll
    for (int u = 0; u < kPer; ++u) acc[u] = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int j0 = 0; j0 < S; j0 += kStateChunk) {
      const int nj = min(kStateChunk, S - j0);
      __syncthreads();
      for (int idx = threadIdx.x; idx < nj * H; idx += kMergeThreads) {
        const int j = idx / H, h = idx % H;
        const float lj = lse_states[(base + (j0 + j) * jstride) * H + h];
        const float L = lse_s[h];
        w_s[j][h] = (lj == -INFINITY || L == -INFINITY) ? 0.f : exp2f((lj - L) * kLog2e);
      }
      __syncthreads();
      for (int j = 0; j < nj; ++j) {
        const float4* src = reinterpret_cast<const float4*>(o_states + (base + (j0 + j) * jstride) * (int64_t)H * D);
#pragma unroll
        for (int u = 0; u < kPer; ++u) {
          const int e = e0 + u * kMergeThreads + threadIdx.x;
          if (e < n4) {
            const float wt = w_s[j][(e * 4) / D];
            const float4 x = __ldg(src + e);
            acc[u].x = fmaf(wt, x.x, acc[u].x);
            acc[u].y = fmaf(wt, x.y, acc[u].y);
            acc[u].z = fmaf(wt, x.z, acc[u].z);
            acc[u].w = fmaf(wt, x.w, acc[u].w);
          }
        }
      }
    }
#pragma unroll
    for (int u = 0; u < kPer; ++u) {
      const int e = e0 + u * kMergeThreads + threadIdx.x;
      if (e < n4) {
        OutT* dst = o_out + out_row * (int64_t)H * D + (int64_t)e * 4;
        store_out(dst + 0, acc[u].x);
        store_out(dst + 1, acc[u].y);
        store_out(dst + 2, acc[u].z);
        store_out(dst + 3, acc[u].w);
      }
    }
  }
}

}  // namespace

int launch_merge(const float* o_states, const float* lse_states, const int32_t* state_indptr,
                 int32_t num_states, const MergeItem* items, int64_t num_rows, int32_t num_heads,
                 int32_t head_dim, void* o_out, int32_t o_dtype, float* lse_out, cudaStream_t s) {
  if (num_rows == 0) return 0;
  if (num_heads > kMaxHeads || head_dim % 4 != 0) return (int)cudaErrorInvalidValue;
  if (o_dtype == SKV_BF16)
    merge_kernel<__nv_bfloat16><<<(unsigned)num_rows, kMergeThreads, 0, s>>>(
        o_states, lse_states, state_indptr, num_states, items, num_rows, num_heads, head_dim,
        static_cast<__nv_bfloat16*>(o_out), lse_out);
  else
    merge_kernel<float><<<(unsigned)num_rows, kMergeThreads, 0, s>>>(
        o_states, lse_states, state_indptr, num_states, items, num_rows, num_heads, head_dim,
        static_cast<float*>(o_out), lse_out);
  return (int)cudaGetLastError();
}

}  // namespace skv
