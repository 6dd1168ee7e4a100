// Generic MLA latent decode on CUDA cores: one warp per folded (query token, head) row.
// Each cache row holds a 512-d compressed KV (ckv) and a 64-d rope key part (kpe) shared by all
// heads; s = scale * (q_nope . ckv + q_pe . kpe), V = ckv (FlashInfer PR #3309 page, MLA decode).
// The e4m3 cache is decoded exactly and scaled by the per-tensor kv_scale.
#include "skv_common.cuh"

namespace skv {

namespace {

struct MlaArgs {
  const __nv_bfloat16* q_nope;
  const __nv_bfloat16* q_pe;
  const uint8_t* ckv;   // byte pointers; element size from KV_E4M3
  const uint8_t* kpe;
  int64_t cs0, cs1, ps0, ps1;  // element strides
  const int32_t* kv_indptr;
  const int32_t* kv_indices;
  const int32_t* last;
  int num_pages, page_size, heads, row_blocks;
  float scale_log2;   // sm_scale * kv_scale * log2(e)
  float kv_scale;
  void* o;
  float* lse;
  float* o_part;
  float* lse_part;
  int32_t* status;
};

template <bool E4M3>
__device__ __forceinline__ float load_kv(const uint8_t* base, int64_t elem) {
  if constexpr (E4M3) {
    return e4m3_to_float(__ldg(base + elem));
  } else {
    const uint16_t b = __ldg(reinterpret_cast<const unsigned short*>(base) + elem);
    return __uint_as_float((uint32_t)b << 16);
  }
}

template <bool E4M3>
__device__ __forceinline__ float dot_span(const float* qs, const uint8_t* base, int64_t off, int n) {
  float acc = 0.f;
  if constexpr (E4M3) {
    const uint32_t* p4 = reinterpret_cast<const uint32_t*>(base + off);
    for (int i = 0; i < n / 4; ++i) {
      const uint32_t w = __ldg(p4 + i);
      acc = fmaf(qs[4 * i + 0], e4m3_to_float(w & 0xFF), acc);
      acc = fmaf(qs[4 * i + 1], e4m3_to_float((w >> 8) & 0xFF), acc);
      acc = fmaf(qs[4 * i + 2], e4m3_to_float((w >> 16) & 0xFF), acc);
      acc = fmaf(qs[4 * i + 3], e4m3_to_float(w >> 24), acc);
    }
  } else {
    const uint4* p4 = reinterpret_cast<const uint4*>(reinterpret_cast<const __nv_bfloat16*>(base) + off);
    for (int i = 0; i < n / 8; ++i) {
      const uint4 w = __ldg(p4 + i);
      const float* qq = qs + 8 * i;
      acc = fmaf(qq[0], bf16_lo(w.x), acc);
      acc = fmaf(qq[1], bf16_hi(w.x), acc);
      acc = fmaf(qq[2], bf16_lo(w.y), acc);
      acc = fmaf(qq[3], bf16_hi(w.y), acc);
      acc = fmaf(qq[4], bf16_lo(w.z), acc);
      acc = fmaf(qq[5], bf16_hi(w.z), acc);
      acc = fmaf(qq[6], bf16_lo(w.w), acc);
      acc = fmaf(qq[7], bf16_hi(w.w), acc);
    }
  }
  return acc;
}

template <bool E4M3, typename OutT>
__global__ void __launch_bounds__(128) mla_simt_kernel(MlaArgs a, const WorkItem* __restrict__ work) {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");  // the merge pass may be scheduled
  constexpr int DV = 512, DR = 64, PER_LANE = DV / 32;
  __shared__ __align__(16) float q_s[4][DV + DR];
  const WorkItem w = work[blockIdx.x];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rr = blockIdx.y * 4 + warp;
  if (rr >= w.q_count * a.heads) return;
  const int qi = rr / a.heads, h = rr % a.heads;
  const int qrow = w.q_start + qi;  // row of the [B*q_len, H] view

  const int r = w.r;
  const int L = request_len(a.kv_indptr, a.last, r, a.page_size);
  const int t0 = w.page_begin * a.page_size;
  const int t1 = min(w.page_end * a.page_size, L);
  const int page_base = a.kv_indptr[r];

  const __nv_bfloat16* qn = a.q_nope + ((int64_t)qrow * a.heads + h) * DV;
  const __nv_bfloat16* qp = a.q_pe + ((int64_t)qrow * a.heads + h) * DR;
  for (int d = lane; d < DV; d += 32) q_s[warp][d] = __bfloat162float(qn[d]);
  for (int d = lane; d < DR; d += 32) q_s[warp][DV + d] = __bfloat162float(qp[d]);
  __syncwarp();

  float m = -INFINITY, l = 0.f;
  float o[PER_LANE];
#pragma unroll
  for (int i = 0; i < PER_LANE; ++i) o[i] = 0.f;

  for (int tb = t0; tb < t1; tb += 32) {
    const int t = tb + lane;
    float s = -INFINITY;
    int64_t coff = -1;
    if (t < t1) {
      const int page = a.kv_indices[page_base + t / a.page_size];
      if ((unsigned)page >= (unsigned)a.num_pages) {
        report(a.status, SKV_DEV_PAGE_OOB);
      } else {
        const int slot = t % a.page_size;
        coff = (int64_t)page * a.cs0 + (int64_t)slot * a.cs1;
        const int64_t poff = (int64_t)page * a.ps0 + (int64_t)slot * a.ps1;
        s = (dot_span<E4M3>(q_s[warp], a.ckv, coff, DV) + dot_span<E4M3>(q_s[warp] + DV, a.kpe, poff, DR)) *
            a.scale_log2;
      }
    }
    const float m_new = fmaxf(m, warp_max(s));
    if (m_new == -INFINITY) continue;
    const float p = (s == -INFINITY) ? 0.f : exp2f(s - m_new);
    const float alpha = (m == -INFINITY) ? 0.f : exp2f(m - m_new);
    l = l * alpha + warp_sum(p);
#pragma unroll
    for (int i = 0; i < PER_LANE; ++i) o[i] *= alpha;
    const int nt = min(32, t1 - tb);
    for (int j = 0; j < nt; ++j) {
      const float pj = __shfl_sync(0xffffffffu, p, j);
      const int64_t cj = __shfl_sync(0xffffffffu, coff, j);
      if (cj < 0) continue;
#pragma unroll
      for (int i = 0; i < PER_LANE; ++i) o[i] = fmaf(pj, load_kv<E4M3>(a.ckv, cj + lane * PER_LANE + i), o[i]);
    }
    m = m_new;
  }

  const bool empty = (l == 0.f);
  const float inv = empty ? 0.f : a.kv_scale / l;
  const float lse = empty ? -INFINITY : (m + log2f(l)) * kLn2;
  if (w.part_row < 0) {
    OutT* op = reinterpret_cast<OutT*>(a.o) + ((int64_t)qrow * a.heads + h) * DV + lane * PER_LANE;
#pragma unroll
    for (int i = 0; i < PER_LANE; ++i) store_out(op + i, o[i] * inv);
    if (a.lse != nullptr && lane == 0) a.lse[(int64_t)qrow * a.heads + h] = lse;
  } else {
    const int64_t prow = (int64_t)w.part_row + (int64_t)qi * w.part_stride;
    float* op = a.o_part + (prow * a.heads + h) * DV + lane * PER_LANE;
#pragma unroll
    for (int i = 0; i < PER_LANE; ++i) op[i] = o[i] * inv;
    if (lane == 0) a.lse_part[prow * a.heads + h] = lse;
  }
}

template <bool E4M3, typename OutT>
int launch_t(const MlaArgs& a, const WorkItem* work, int num_work, cudaStream_t s) {
  dim3 grid(num_work, a.row_blocks);
  mla_simt_kernel<E4M3, OutT><<<grid, 128, 0, s>>>(a, work);
  return (int)cudaGetLastError();
}

}  // namespace

int launch_mla_simt(const skv_mla_params& p, const WorkItem* work, int num_work, int q_tile,
                    cudaStream_t s) {
  if (num_work == 0) return 0;
  MlaArgs a;
  a.q_nope = static_cast<const __nv_bfloat16*>(p.q_nope);
  a.q_pe = static_cast<const __nv_bfloat16*>(p.q_pe);
  a.ckv = static_cast<const uint8_t*>(p.ckv);
  a.kpe = static_cast<const uint8_t*>(p.kpe);
  a.cs0 = p.ckv_stride[0]; a.cs1 = p.ckv_stride[1]; a.ps0 = p.kpe_stride[0]; a.ps1 = p.kpe_stride[1];
  a.kv_indptr = p.kv_indptr; a.kv_indices = p.kv_indices; a.last = p.kv_last_page_len;
  a.num_pages = p.num_pages; a.page_size = p.page_size; a.heads = p.num_heads;
  a.row_blocks = (q_tile * p.num_heads + 3) / 4;
  a.kv_scale = p.kv_dtype == SKV_E4M3 ? p.kv_scale : 1.f;
  a.scale_log2 = p.sm_scale * a.kv_scale * kLog2e;
  a.o = p.o; a.lse = p.lse; a.o_part = p.o_part; a.lse_part = p.lse_part; a.status = p.status;
  const bool bf = p.o_dtype == SKV_BF16;
  if (p.kv_dtype == SKV_E4M3)
    return bf ? launch_t<true, __nv_bfloat16>(a, work, num_work, s) : launch_t<true, float>(a, work, num_work, s);
  return bf ? launch_t<false, __nv_bfloat16>(a, work, num_work, s) : launch_t<false, float>(a, work, num_work, s);
}

}  // namespace skv
