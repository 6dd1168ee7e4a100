// Device helpers shared by the libsplitkv kernels: page-table walk, storage-format decoding,
// the device status word, and mbarrier / TMA / tcgen05 wrappers in inline PTX (sm_100a).
#pragma once
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "skv_internal.h"

namespace skv {

// ------------------------------------------------------------------------------ status word
__device__ __forceinline__ void report(int32_t* status, int32_t code) {
  if (status != nullptr) atomicCAS(status, 0, code);
}

// ------------------------------------------------------------------------------ formats
__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// OCP e4m3fn code -> float, exact (sign, 4-bit exponent with bias 7, 3-bit mantissa;
// exponent 0 subnormal; S.1111.111 NaN).
__device__ __forceinline__ float e4m3_to_float(uint32_t c) {
  const uint32_t e = (c >> 3) & 15u, m = c & 7u;
  float v;
  if ((c & 0x7Fu) == 0x7Fu) {
    v = __uint_as_float(0x7FC00000u);
  } else if (e == 0) {
    v = (float)m * 0.001953125f;  // m * 2^-9
  } else {
    v = __uint_as_float(((e + 120u) << 23) | (m << 20));
  }
  return (c & 0x80u) ? -v : v;
}

// ------------------------------------------------------------------------------ page walk
// Request r: n_r pages at kv_indices[kv_indptr[r]..]; L_r = (n_r - 1) P + last_page_len.
__device__ __forceinline__ int request_len(const int32_t* kv_indptr, const int32_t* last, int r,
                                           int page_size) {
  const int n = kv_indptr[r + 1] - kv_indptr[r];
  return n == 0 ? 0 : (n - 1) * page_size + last[r];
}

// Element offset of (token t of request r, head kh) in a cache with strides s[3]
// (page, slot, head).  Returns -1 (and reports) for an out-of-range page id.
__device__ __forceinline__ int64_t token_offset(const int32_t* kv_indices, int page_base, int t,
                                                int page_size, int num_pages, int64_t s0,
                                                int64_t s1, int64_t s2, int kh,
                                                int32_t* status) {
  const int page = kv_indices[page_base + t / page_size];
  if ((unsigned)page >= (unsigned)num_pages) {
    report(status, SKV_DEV_PAGE_OOB);
    return -1;
  }
  return (int64_t)page * s0 + (int64_t)(t % page_size) * s1 + (int64_t)kh * s2;
}

// V offset from the K offset.  SAME_KV_STRIDES: K's address math is reused as is (one
// computation for both tensors, no extra registers); otherwise V's strides are applied.
template <bool SAME_KV_STRIDES>
__device__ __forceinline__ int64_t v_offset_from(int64_t k_off, int page, int slot, int kh,
                                                 int64_t v0, int64_t v1, int64_t v2) {
  if constexpr (SAME_KV_STRIDES) {
    return k_off;
  } else {
    return (int64_t)page * v0 + (int64_t)slot * v1 + (int64_t)kh * v2;
  }
}

// ------------------------------------------------------------------------------ warp reductions
__device__ __forceinline__ float warp_max(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
  return x;
}
__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

// ------------------------------------------------------------------------------ output stores
__device__ __forceinline__ void store_out(float* p, float v) { *p = v; }
__device__ __forceinline__ void store_out(__nv_bfloat16* p, float v) { *p = __float2bfloat16_rn(v); }

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

}  // namespace skv
