// Test hook: copy each request's logical K and V rows (through the page-table walk and the
// SAME_KV_STRIDES / independent-stride address generation the attention kernels use) into
// dense [sum_r L_r, Hk, D] buffers, so the indexing can be checked bit for bit.
#include "skv_common.cuh"

namespace skv {

namespace {

template <bool SAME_KV>
__global__ void gather_kernel(skv_paged_params p, const int32_t* __restrict__ token_indptr,
                              int64_t total_tokens, uint16_t* __restrict__ k_out,
                              uint16_t* __restrict__ v_out) {
  const int64_t row = blockIdx.x;  // dense token row
  if (row >= total_tokens) return;
  // request owning this row: binary search over token_indptr
  int lo = 0, hi = p.batch;
  while (hi - lo > 1) {
    const int mid = (lo + hi) / 2;
    if (token_indptr[mid] <= row) lo = mid; else hi = mid;
  }
  const int r = lo;
  const int t = (int)(row - token_indptr[r]);
  const int page_base = p.kv_indptr[r];
  const uint16_t* k = static_cast<const uint16_t*>(p.k_cache);
  const uint16_t* v = static_cast<const uint16_t*>(p.v_cache);
  for (int kh = threadIdx.y; kh < p.num_kv_heads; kh += blockDim.y) {
    const int64_t koff = token_offset(p.kv_indices, page_base, t, p.page_size, p.num_pages, p.k_stride[0],
                                      p.k_stride[1], p.k_stride[2], kh, p.status);
    if (koff < 0) continue;
    const int page = p.kv_indices[page_base + t / p.page_size];
    const int64_t voff = v_offset_from<SAME_KV>(koff, page, t % p.page_size, kh, p.v_stride[0],
                                                p.v_stride[1], p.v_stride[2]);
    const int64_t dst = (row * p.num_kv_heads + kh) * p.head_dim;
    for (int d = threadIdx.x; d < p.head_dim; d += blockDim.x) {
      k_out[dst + d] = k[koff + d];
      v_out[dst + d] = v[voff + d];
    }
  }
}

}  // namespace

int launch_gather(const skv_paged_params& p, const int32_t* token_indptr, int64_t total_tokens,
                  void* k_out, void* v_out, bool same_kv, cudaStream_t s) {
  if (total_tokens == 0) return 0;
  dim3 block(32, 4);
  if (same_kv)
    gather_kernel<true><<<(unsigned)total_tokens, block, 0, s>>>(p, token_indptr, total_tokens,
                                                                 static_cast<uint16_t*>(k_out),
                                                                 static_cast<uint16_t*>(v_out));
  else
    gather_kernel<false><<<(unsigned)total_tokens, block, 0, s>>>(p, token_indptr, total_tokens,
                                                                  static_cast<uint16_t*>(k_out),
                                                                  static_cast<uint16_t*>(v_out));
  return (int)cudaGetLastError();
}

}  // namespace skv
