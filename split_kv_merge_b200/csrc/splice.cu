// Fetch primitive, local compute ("Move the Query, Not the Cache", problem statement and
// Methodology: fetch brings a whole KV chunk to the requester, adapts its positions -- the
// "splice" -- and attends locally).  A latent row is 512 position-free values plus a 64-d rope
// part whose 32 pairs are turned by delta * theta_i when the row moves by delta positions.
//
// One launch moves up to 64 chunks.  The chunks' tokens are laid end to end and cut into one
// contiguous range per CTA, with one wave of CTAs (resident CTAs per SM x SMs), so there is no
// tail wave and no launch per chunk.  A CTA walks the chunk segments of its range; on entering a
// segment it forms that chunk's 32 (cos, sin) pairs in fp64 -- delta * theta reaches 1e5
// radians, far beyond what an fp32 argument resolves -- and rounds them to fp32.
//
// One warp moves one row: the 1024-byte latent as two coalesced 16-byte accesses per lane, the
// 128-byte rope part by lanes 0-7 (interleaved pairs: 16 bytes hold four whole pairs) or lanes
// 0-3 (pairs (i, i+32): 16 bytes from each half).  Each warp loads two rows before it stores
// either, so two rows per warp are in flight.  HBM-bound: 2 x 1152 bytes per token; streaming
// (evict-first) loads and stores keep the moved rows from displacing L2.
#include <cuda_bf16.h>
#include <string.h>

#include <algorithm>

#include "skv_common.cuh"

namespace skv {

namespace {

constexpr int kWarps = 8;  // 256 threads per CTA
constexpr int kPairs = 32;
constexpr int kMaxChunks = 64;
constexpr int kRows = 4;   // rows each warp has in flight

struct SpliceArgs {
  const uint16_t* sc;
  const uint16_t* sk;
  int64_t sc0, sc1, sk0, sk1;
  const int32_t* sp;
  int32_t snp, sps;
  uint16_t* dc;
  uint16_t* dk;
  int64_t dc0, dc1, dk0, dk1;
  const int32_t* dp;
  int32_t dnp, dps;
  double theta;
  int32_t halves;
  const float* inv_freq;
  int32_t* status;
  int32_t num_chunks;
  int64_t total;                       // tokens of all chunks
  int64_t prefix[kMaxChunks + 1];      // first flattened token of each chunk
  int64_t src_start[kMaxChunks];
  int64_t dst_start[kMaxChunks];
  int64_t delta[kMaxChunks];
};

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  uint32_t u;
  memcpy(&u, &h, 4);
  return u;
}

// (a, b) -> (a c - b s, a s + b c)
__device__ __forceinline__ void turn(float a, float b, float2 cs, float& ra, float& rb) {
  ra = a * cs.x - b * cs.y;
  rb = a * cs.y + b * cs.x;
}

__device__ __forceinline__ uint32_t word(const uint4& v, int j) {
  return j == 0 ? v.x : j == 1 ? v.y : j == 2 ? v.z : v.w;
}
__device__ __forceinline__ void set_word(uint4& v, int j, uint32_t w) {
  if (j == 0) v.x = w; else if (j == 1) v.y = w; else if (j == 2) v.z = w; else v.w = w;
}

// One row in flight: its page ids and slots (pointers are formed where they are used, so a row
// costs few registers beyond its data) and the loaded data.
struct Row {
  int32_t sp, ss, dp, ds;
  uint4 c0, c1, k0, k1;
  bool ok;
};

__device__ __forceinline__ void row_locate(const SpliceArgs& a, int64_t ls, int64_t ld, int lane, Row& r) {
  const int64_t sq = ls / a.sps, dq = ld / a.dps;
  r.sp = __ldg(a.sp + sq);
  r.dp = __ldg(a.dp + dq);
  r.ss = (int32_t)(ls - sq * a.sps);
  r.ds = (int32_t)(ld - dq * a.dps);
  r.ok = (uint32_t)r.sp < (uint32_t)a.snp && (uint32_t)r.dp < (uint32_t)a.dnp;
  if (!r.ok && lane == 0) report(a.status, SKV_DEV_PAGE_OOB);
}

__device__ __forceinline__ void row_load(const SpliceArgs& a, Row& r, int lane, bool rope_lane, bool halves) {
  if (!r.ok) return;
  const uint4* sc = reinterpret_cast<const uint4*>(a.sc + (int64_t)r.sp * a.sc0 + (int64_t)r.ss * a.sc1);
  r.c0 = __ldcs(sc + lane);
  r.c1 = __ldcs(sc + 32 + lane);
  if (rope_lane) {
    const uint4* sk = reinterpret_cast<const uint4*>(a.sk + (int64_t)r.sp * a.sk0 + (int64_t)r.ss * a.sk1);
    r.k0 = __ldcs(sk + lane);                 // interleaved: elements 8*lane ..; halves: first entries
    if (halves) r.k1 = __ldcs(sk + 4 + lane);  // halves: second entries at 32 + 8*lane
  }
}

__device__ __forceinline__ void row_store(const SpliceArgs& a, Row& r, int lane, bool rope_lane, bool halves,
                                          const float2* cs) {
  if (!r.ok) return;
  uint4* dc = reinterpret_cast<uint4*>(a.dc + (int64_t)r.dp * a.dc0 + (int64_t)r.ds * a.dc1);
  __stcs(dc + lane, r.c0);
  __stcs(dc + 32 + lane, r.c1);
  if (!rope_lane) return;
  uint4* dk = reinterpret_cast<uint4*>(a.dk + (int64_t)r.dp * a.dk0 + (int64_t)r.ds * a.dk1);
  if (!halves) {
#pragma unroll
    for (int j = 0; j < 4; ++j) {  // word j = pair 4*lane + j
      const uint32_t w = word(r.k0, j);
      float ra, rb;
      turn(bf16_lo(w), bf16_hi(w), cs[4 * lane + j], ra, rb);
      set_word(r.k0, j, pack_bf16(ra, rb));
    }
    __stcs(dk + lane, r.k0);
  } else {
#pragma unroll
    for (int j = 0; j < 4; ++j) {  // word j = pairs 8*lane + 2j and 8*lane + 2j + 1
      const uint32_t wa = word(r.k0, j), wb = word(r.k1, j);
      float ra0, rb0, ra1, rb1;
      turn(bf16_lo(wa), bf16_lo(wb), cs[8 * lane + 2 * j], ra0, rb0);
      turn(bf16_hi(wa), bf16_hi(wb), cs[8 * lane + 2 * j + 1], ra1, rb1);
      set_word(r.k0, j, pack_bf16(ra0, ra1));
      set_word(r.k1, j, pack_bf16(rb0, rb1));
    }
    __stcs(dk + lane, r.k0);
    __stcs(dk + 4 + lane, r.k1);
  }
}

__global__ void __launch_bounds__(kWarps * 32) splice_kernel(const __grid_constant__ SpliceArgs a) {
  __shared__ float2 rot[kPairs];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const bool halves = a.halves != 0;
  const bool rope_lane = halves ? lane < 4 : lane < 8;
  const int64_t lo = (int64_t)blockIdx.x * a.total / gridDim.x;
  const int64_t hi = ((int64_t)blockIdx.x + 1) * a.total / gridDim.x;
  int c = 0;
  for (int64_t seg = lo; seg < hi;) {
    while (a.prefix[c + 1] <= seg) ++c;  // skips empty chunks; prefix[num_chunks] = total > seg
    const int64_t seg_end = min(hi, a.prefix[c + 1]);
    __syncthreads();  // the previous segment's rows no longer read rot
    if (tid < kPairs) {
      const double th = a.inv_freq != nullptr ? (double)a.inv_freq[tid] : pow(a.theta, -2.0 * tid / 64.0);
      double s, co;
      sincos((double)a.delta[c] * th, &s, &co);
      rot[tid] = make_float2((float)co, (float)s);
    }
    __syncthreads();
    const int64_t off_s = a.src_start[c] - a.prefix[c], off_d = a.dst_start[c] - a.prefix[c];
    for (int64_t i = seg + warp; i < seg_end; i += kRows * kWarps) {
      Row r[kRows];
#pragma unroll
      for (int j = 0; j < kRows; ++j) {
        const int64_t t = i + j * kWarps;
        if (t < seg_end) row_locate(a, t + off_s, t + off_d, lane, r[j]);
        else r[j].ok = false;
      }
#pragma unroll
      for (int j = 0; j < kRows; ++j) row_load(a, r[j], lane, rope_lane, halves);
#pragma unroll
      for (int j = 0; j < kRows; ++j) row_store(a, r[j], lane, rope_lane, halves, rot);
    }
    seg = seg_end;
  }
}

int resident_grid(int64_t total) {
  // resident CTAs per SM depend only on the kernel (same on every B200); SMs come per device
  static std::atomic<int> per_sm_cache{0};
  int per_sm = per_sm_cache.load(std::memory_order_relaxed);
  if (per_sm == 0) {
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, splice_kernel, kWarps * 32, 0) != cudaSuccess ||
        per_sm <= 0)
      per_sm = 4;
    cudaGetLastError();
    per_sm_cache.store(per_sm, std::memory_order_relaxed);
  }
  const int64_t full = (int64_t)device_sm_count() * per_sm;
  const int64_t want = (total + kRows * kWarps - 1) / (kRows * kWarps);  // a full row group per warp
  return (int)std::max<int64_t>(1, std::min<int64_t>(want, full));
}

}  // namespace

int launch_splice(const skv_splice_params& p, const skv_splice_chunk* chunks, int num_chunks, cudaStream_t s) {
  SpliceArgs a;
  memset(&a, 0, sizeof(a));
  a.sc = static_cast<const uint16_t*>(p.src_ckv);
  a.sk = static_cast<const uint16_t*>(p.src_kpe);
  a.sc0 = p.src_ckv_stride[0];
  a.sc1 = p.src_ckv_stride[1];
  a.sk0 = p.src_kpe_stride[0];
  a.sk1 = p.src_kpe_stride[1];
  a.sp = p.src_pages;
  a.snp = p.src_num_pages;
  a.sps = p.src_page_size;
  a.dc = static_cast<uint16_t*>(p.dst_ckv);
  a.dk = static_cast<uint16_t*>(p.dst_kpe);
  a.dc0 = p.dst_ckv_stride[0];
  a.dc1 = p.dst_ckv_stride[1];
  a.dk0 = p.dst_kpe_stride[0];
  a.dk1 = p.dst_kpe_stride[1];
  a.dp = p.dst_pages;
  a.dnp = p.dst_num_pages;
  a.dps = p.dst_page_size;
  a.theta = (double)p.rope_theta;
  a.halves = p.rope_layout == SKV_ROPE_HALVES;
  a.inv_freq = p.inv_freq;
  a.status = p.status;
  for (int base = 0; base < num_chunks; base += kMaxChunks) {
    const int n = std::min(kMaxChunks, num_chunks - base);
    a.num_chunks = n;
    a.prefix[0] = 0;
    for (int c = 0; c < n; ++c) {
      const skv_splice_chunk& ch = chunks[base + c];
      a.prefix[c + 1] = a.prefix[c] + ch.n_tokens;
      a.src_start[c] = ch.src_start;
      a.dst_start[c] = ch.dst_start;
      a.delta[c] = ch.delta_pos;
    }
    for (int c = n + 1; c <= kMaxChunks; ++c) a.prefix[c] = a.prefix[n];
    a.total = a.prefix[n];
    if (a.total == 0) continue;
    splice_kernel<<<resident_grid(a.total), kWarps * 32, 0, s>>>(a);
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return (int)e;
  }
  return 0;
}

}  // namespace skv
