// Generic paged GQA attention on CUDA cores: one warp per (query token, query head) row of a
// work item, lane-per-token scores, online softmax, lane-per-dimension PV.  This is the
// general path (any page size, any group size, head_dim 64/128, short query tiles); the
// tensor-core decode kernel (gqa_tc_decode.cu) takes the decode shapes.
//
// The K and V addresses follow the paged_kv_t description of the FlashInfer PR #4736 page
// (section 1): page id from the table, then page / slot / head strides; V reuses K's offset when
// the strides are the same (section 2, SAME_KV_STRIDES), else applies its own strides.
#include "skv_common.cuh"

namespace skv {

namespace {

struct GqaArgs {
  const __nv_bfloat16* q;
  const __nv_bfloat16* k;
  const __nv_bfloat16* v;
  int64_t ks0, ks1, ks2, vs0, vs1, vs2;
  const int32_t* kv_indptr;
  const int32_t* kv_indices;
  const int32_t* last;
  int num_pages, page_size, hq, hk, row_blocks;
  float scale_log2;  // sm_scale * log2(e)
  void* o;
  float* lse;
  float* o_part;
  float* lse_part;
  int32_t* status;
};

template <int D>
__device__ __forceinline__ float dot_row(const float* qs, const __nv_bfloat16* kp) {
  const uint4* k4 = reinterpret_cast<const uint4*>(kp);
  float acc = 0.f;
#pragma unroll 4
  for (int i = 0; i < D / 8; ++i) {
    const uint4 w = __ldg(k4 + i);
    const float* qq = qs + i * 8;
    acc = fmaf(qq[0], bf16_lo(w.x), acc);
    acc = fmaf(qq[1], bf16_hi(w.x), acc);
    acc = fmaf(qq[2], bf16_lo(w.y), acc);
    acc = fmaf(qq[3], bf16_hi(w.y), acc);
    acc = fmaf(qq[4], bf16_lo(w.z), acc);
    acc = fmaf(qq[5], bf16_hi(w.z), acc);
    acc = fmaf(qq[6], bf16_lo(w.w), acc);
    acc = fmaf(qq[7], bf16_hi(w.w), acc);
  }
  return acc;
}

template <int D, bool SAME_KV, typename OutT>
__global__ void __launch_bounds__(128) gqa_simt_kernel(GqaArgs a, const WorkItem* __restrict__ work) {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");  // the merge pass may be scheduled
  constexpr int PER_LANE = D / 32;  // V dims per lane
  __shared__ __align__(16) float q_s[4][D];
  const WorkItem w = work[blockIdx.x];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = a.hq / a.hk;
  const int kh = blockIdx.y / a.row_blocks;
  const int rr = (blockIdx.y % a.row_blocks) * 4 + warp;  // row within (item, kv head)
  if (rr >= w.q_count * g) return;
  const int qi = rr / g;              // query token within the item
  const int h = kh * g + rr % g;      // query head
  const int qrow = w.q_start + qi;

  const int r = w.r;
  const int L = request_len(a.kv_indptr, a.last, r, a.page_size);
  const int t0 = w.page_begin * a.page_size;
  const int t1 = min(w.page_end * a.page_size, L);
  const int page_base = a.kv_indptr[r];

  const __nv_bfloat16* qp = a.q + ((int64_t)qrow * a.hq + h) * D;
  for (int d = lane; d < D; d += 32) q_s[warp][d] = __bfloat162float(qp[d]);
  __syncwarp();

  float m = -INFINITY, l = 0.f;
  float o[PER_LANE];
#pragma unroll
  for (int i = 0; i < PER_LANE; ++i) o[i] = 0.f;

  for (int tb = t0; tb < t1; tb += 32) {
    const int t = tb + lane;
    float s = -INFINITY;
    int64_t koff = -1, voff = -1;
    if (t < t1) {
      koff = token_offset(a.kv_indices, page_base, t, a.page_size, a.num_pages, a.ks0, a.ks1, a.ks2,
                          kh, a.status);
      if (koff >= 0) {
        const int page = a.kv_indices[page_base + t / a.page_size];
        voff = v_offset_from<SAME_KV>(koff, page, t % a.page_size, kh, a.vs0, a.vs1, a.vs2);
        s = dot_row<D>(q_s[warp], a.k + koff) * a.scale_log2;
      }
    }
    const float m_new = fmaxf(m, warp_max(s));
    if (m_new == -INFINITY) continue;  // nothing valid yet
    const float p = (s == -INFINITY) ? 0.f : exp2f(s - m_new);
    const float alpha = (m == -INFINITY) ? 0.f : exp2f(m - m_new);
    l = l * alpha + warp_sum(p);
#pragma unroll
    for (int i = 0; i < PER_LANE; ++i) o[i] *= alpha;
    const int nt = min(32, t1 - tb);
    for (int j = 0; j < nt; ++j) {
      const float pj = __shfl_sync(0xffffffffu, p, j);
      const int64_t vj = __shfl_sync(0xffffffffu, voff, j);
      if (vj < 0) continue;
      const __nv_bfloat16* vp = a.v + vj + lane * PER_LANE;
      if constexpr (PER_LANE == 4) {
        const uint2 w2 = __ldg(reinterpret_cast<const uint2*>(vp));
        o[0] = fmaf(pj, bf16_lo(w2.x), o[0]);
        o[1] = fmaf(pj, bf16_hi(w2.x), o[1]);
        o[2] = fmaf(pj, bf16_lo(w2.y), o[2]);
        o[3] = fmaf(pj, bf16_hi(w2.y), o[3]);
      } else {
        const uint32_t w1 = __ldg(reinterpret_cast<const uint32_t*>(vp));
        o[0] = fmaf(pj, bf16_lo(w1), o[0]);
        o[1] = fmaf(pj, bf16_hi(w1), o[1]);
      }
    }
    m = m_new;
  }

  const bool empty = (l == 0.f);
  const float inv = empty ? 0.f : 1.f / l;
  const float lse = empty ? -INFINITY : (m + log2f(l)) * kLn2;
  if (w.part_row < 0) {
    OutT* op = reinterpret_cast<OutT*>(a.o) + ((int64_t)qrow * a.hq + h) * D + lane * PER_LANE;
#pragma unroll
    for (int i = 0; i < PER_LANE; ++i) store_out(op + i, o[i] * inv);
    if (a.lse != nullptr && lane == 0) a.lse[(int64_t)qrow * a.hq + h] = lse;
  } else {
    const int64_t prow = (int64_t)w.part_row + (int64_t)qi * w.part_stride;
    float* op = a.o_part + (prow * a.hq + h) * D + lane * PER_LANE;
#pragma unroll
    for (int i = 0; i < PER_LANE; ++i) op[i] = o[i] * inv;
    if (lane == 0) a.lse_part[prow * a.hq + h] = lse;
  }
}

template <int D, bool SAME_KV, typename OutT>
int launch_t(const GqaArgs& a, const WorkItem* work, int num_work, cudaStream_t s) {
  dim3 grid(num_work, a.hk * a.row_blocks);
  gqa_simt_kernel<D, SAME_KV, OutT><<<grid, 128, 0, s>>>(a, work);
  return (int)cudaGetLastError();
}

}  // namespace

int launch_gqa_simt(const skv_paged_params& p, const WorkItem* work, int num_work, int q_tile,
                    bool same_kv, cudaStream_t s) {
  if (num_work == 0) return 0;
  GqaArgs a;
  a.q = static_cast<const __nv_bfloat16*>(p.q);
  a.k = static_cast<const __nv_bfloat16*>(p.k_cache);
  a.v = static_cast<const __nv_bfloat16*>(p.v_cache);
  a.ks0 = p.k_stride[0]; a.ks1 = p.k_stride[1]; a.ks2 = p.k_stride[2];
  a.vs0 = p.v_stride[0]; a.vs1 = p.v_stride[1]; a.vs2 = p.v_stride[2];
  a.kv_indptr = p.kv_indptr; a.kv_indices = p.kv_indices; a.last = p.kv_last_page_len;
  a.num_pages = p.num_pages; a.page_size = p.page_size; a.hq = p.num_qo_heads; a.hk = p.num_kv_heads;
  const int g = p.num_qo_heads / p.num_kv_heads;
  a.row_blocks = (q_tile * g + 3) / 4;
  a.scale_log2 = p.sm_scale * kLog2e;
  a.o = p.o; a.lse = p.lse; a.o_part = p.o_part; a.lse_part = p.lse_part; a.status = p.status;
  const bool bf = p.o_dtype == SKV_BF16;
#define SKV_GQA_CASE(D_)                                                                       \
  if (p.head_dim == D_) {                                                                      \
    if (same_kv) return bf ? launch_t<D_, true, __nv_bfloat16>(a, work, num_work, s)           \
                           : launch_t<D_, true, float>(a, work, num_work, s);                  \
    return bf ? launch_t<D_, false, __nv_bfloat16>(a, work, num_work, s)                       \
              : launch_t<D_, false, float>(a, work, num_work, s);                              \
  }
  SKV_GQA_CASE(64)
  SKV_GQA_CASE(128)
#undef SKV_GQA_CASE
  return (int)cudaErrorInvalidValue;
}

}  // namespace skv
