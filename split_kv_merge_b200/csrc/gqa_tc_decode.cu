// Paged GQA decode on the 5th-generation tensor cores (tcgen05 + TMEM) with TMA page staging.
//
// What it computes: for one work item (request r, query tokens [q_start, q_start+q_count),
// logical pages [page_begin, page_end)) and one KV head kh, the attention of the g*q_count query
// rows of that KV head over the item's tokens -- the output directly, or the split partial
// (O_j, LSE_j) that merge_states later combines (split-KV: FlashInfer PR #5597 page, section 3;
// route primitive, "Move the Query, Not the Cache").
//
// B200 design (the FlashInfer FA2 kernel of the PR #4736 page is prior art only):
//  * The GQA group (8 rows) is far too small for an M=128 tile, so both products are swapped:
//      S^T[128 tokens, 16]  = K_tile[128, D]   . Q^T[D, 16]      (M = tokens)
//      O^T[D = 128, 16]    += V_tile^T[D, 128] . P^T[128, 16]     (M = head dims, V MN-major)
//    with fp32 accumulators in TMEM (2 x 16 columns for S, 2 x 16 for O, double buffered).
//  * Pages are staged by TMA (one 64-column box per page and half of D, page id from the table;
//    TMA generates every K and V address, so the SAME_KV_STRIDES address reuse of the PR #4736
//    page costs nothing here either way) into a 3-stage ring of 128-token K and V tiles with the
//    128-byte swizzle the MMA descriptors expect.  Out-of-range page ids are reported and read as
//    zeros by the TMA bounds check.
//  * Warp roles: warp 4 issues TMA, warp 5 allocates TMEM and issues the MMAs, warps 0-3 run the
//    online softmax (thread = token lane of S^T: tile row-max by warp shuffles + a 4-warp
//    exchange, per-thread partial row sums reduced once per work item) and accumulate O^T from
//    TMEM in registers (thread = head-dim lane), rescaling by exp2(m_old - m_new).
//  * Persistent: one CTA per SM walks its share of (work item, KV head) units; the TMA ring runs
//    across unit boundaries so HBM stays busy.
//  * Masked tokens (past the request's length or the split) get s = -inf by selection and their V
//    rows are zeroed in shared memory, so stale or non-finite tail slots cannot leak into O.
//  * Every mbarrier wait is bounded; on timeout the kernel records SKV_DEV_TIMEOUT, all roles
//    leave their loops together, and TMEM is released.
#include <cudaTypedefs.h>

#include <mutex>

#include "tc_ptx.cuh"

namespace skv {

namespace {

constexpr int kTile = 128;       // tokens per KV tile (the M of S^T)
constexpr int kD = 128;          // head dim handled here
constexpr int kRegions = kD / 64;
constexpr int kStages = 3;
constexpr int kKBytes = kTile * kD * 2;          // 32 KB
constexpr int kStageBytes = 2 * kKBytes;         // K + V
constexpr int kQBytes = 16 * kD * 2;             // 16 query rows
constexpr int kPBytes = 16 * kTile * 2;          // 16 x 128 bf16
constexpr int kThreads = 192;
constexpr int kSoftmaxThreads = 128;
constexpr int kTmemCols = 64;                    // S0 S1 O0 O1, 16 columns each

struct Smem {
  // offsets (bytes) from the 1024-aligned dynamic shared memory base
  static constexpr int kv = 0;
  static constexpr int q = kv + kStages * kStageBytes;
  static constexpr int p = q + 2 * kQBytes;
  static constexpr int red = p + 2 * kPBytes;                 // [2][4][16] float
  static constexpr int lred = red + 2 * 4 * 16 * 4;           // [4][16] float
  static constexpr int bars = lred + 4 * 16 * 4;              // mbarriers
  static constexpr int nbars = 2 * kStages + 2 * 6;
  static constexpr int misc = bars + nbars * 8;               // tmem base, abort flag
  static constexpr int total = misc + 16;
};

struct TcArgs {
  const int32_t* kv_indptr;
  const int32_t* kv_indices;
  const int32_t* last;
  int num_pages, page_size, hq, hk, g, q_tile, num_units;
  float scale_log2;
  void* o;
  float* lse;
  float* o_part;
  float* lse_part;
  int32_t* status;
};

struct Unit {
  int r, kh, q_start, q_count, page_begin, page_end, part_row, part_stride;
  int t0, t1, ntiles;
};

__device__ __forceinline__ Unit load_unit(const TcArgs& a, const WorkItem* work, int u) {
  Unit x;
  const WorkItem w = work[u / a.hk];
  x.kh = u % a.hk;
  x.r = w.r;
  x.q_start = w.q_start;
  x.q_count = w.q_count;
  x.page_begin = w.page_begin;
  x.page_end = w.page_end;
  x.part_row = w.part_row;
  x.part_stride = w.part_stride;
  const int L = request_len(a.kv_indptr, a.last, w.r, a.page_size);
  x.t0 = w.page_begin * a.page_size;
  x.t1 = min(w.page_end * a.page_size, L);
  x.ntiles = x.t1 > x.t0 ? (x.t1 - x.t0 + kTile - 1) / kTile : 0;
  return x;
}

__device__ __forceinline__ bool bar_and(int id, int n, bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred pi, po;\n\t"
      "setp.ne.u32 pi, %1, 0;\n\t"
      "barrier.cta.red.and.pred po, %2, %3, pi;\n\t"
      "selp.u32 %0, 1, 0, po;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)v), "r"(id), "r"(n)
      : "memory");
  return r != 0;
}

template <int NC, typename OutT>
__global__ void __launch_bounds__(kThreads, 1)
gqa_tc_decode_kernel(const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap vmap,
                     const __grid_constant__ CUtensorMap qmap, TcArgs a, const WorkItem* __restrict__ work) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = tc::smem_u32(smem);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  tc::grid_launch_dependents();  // the merge pass may be scheduled; it waits for this grid

  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + Smem::misc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Smem::misc + 4);
  const uint32_t bar0 = sbase + Smem::bars;
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (kStages + s); };
  auto qfull_bar = [&](int b) { return bar0 + 8u * (2 * kStages + b); };
  auto qempty_bar = [&](int b) { return bar0 + 8u * (2 * kStages + 2 + b); };
  auto sfull_bar = [&](int b) { return bar0 + 8u * (2 * kStages + 4 + b); };
  auto sempty_bar = [&](int b) { return bar0 + 8u * (2 * kStages + 6 + b); };
  auto pfull_bar = [&](int b) { return bar0 + 8u * (2 * kStages + 8 + b); };
  auto ofull_bar = [&](int b) { return bar0 + 8u * (2 * kStages + 10 + b); };
  auto oempty_bar = [&](int b) { return bar0 + 8u * (2 * kStages + 12 + b); };
  static_assert(Smem::nbars == 2 * kStages + 12, "barrier count");

  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      tc::mbar_init(full_bar(s), 1);
      tc::mbar_init(empty_bar(s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      tc::mbar_init(qfull_bar(b), 1);
      tc::mbar_init(qempty_bar(b), 1);
      tc::mbar_init(sfull_bar(b), 1);
      tc::mbar_init(sempty_bar(b), 4);
      tc::mbar_init(pfull_bar(b), 4);
      tc::mbar_init(ofull_bar(b), 1);
      tc::mbar_init(oempty_bar(b), 4);
    }
    *abort_flag = 0;
    tc::fence_mbar_init();
    tc::fence_proxy_async_smem();
  }
  if (warp == 4 && lane == 0) {
    tc::prefetch_tmap(&kmap);
    tc::prefetch_tmap(&vmap);
    tc::prefetch_tmap(&qmap);
  }
  // zero the V stages once so never-loaded rows of a partial tile are finite
  for (int i = tid; i < kStages * kKBytes / 16; i += kThreads) {
    const int s = i / (kKBytes / 16), o = i % (kKBytes / 16);
    reinterpret_cast<uint4*>(smem + Smem::kv + s * kStageBytes + kKBytes)[o] = make_uint4(0, 0, 0, 0);
  }
  tc::fence_proxy_async_smem();
  if (warp == 5) tc::tmem_alloc(tc::smem_u32(tmem_holder), kTmemCols);
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  const int G = gridDim.x;
  if (warp == 4) {
    // ======================================================================= TMA producer
    // The whole warp walks the units: lanes fetch the next tile's page ids (one per lane), the
    // whole warp waits for a free stage, lane 0 issues the copies.
    const uint64_t pol = tc::policy_evict_first();
    const int ppt = kTile / a.page_size;  // pages per tile (<= 16)
    int n_tile = 0, n_unit = 0;
    bool ok = true;
    for (int u = blockIdx.x; u < a.num_units && ok; u += G) {
      const Unit x = load_unit(a, work, u);
      if (x.ntiles == 0) continue;
      const int* ids = a.kv_indices + a.kv_indptr[x.r] + x.page_begin;
      const int npages = x.page_end - x.page_begin;
      int pid = lane < min(ppt, npages) ? __ldg(ids + lane) : 0;
      const int qb = n_unit & 1;
      if (lane == 0) {
        if (n_unit >= 2) ok = tc::mbar_wait(qempty_bar(qb), ((n_unit >> 1) + 1) & 1, abort_flag, a.status);
        if (ok) {
          const uint32_t qdst = sbase + Smem::q + qb * kQBytes;
          tc::mbar_arrive_expect_tx(qfull_bar(qb), (uint32_t)(kD * 2 * a.g * a.q_tile));
          for (int rgn = 0; rgn < kRegions; ++rgn)
            tc::tma_load_3d(qdst + rgn * (16 * 128), &qmap, qfull_bar(qb), rgn * 64, x.kh * a.g, x.q_start);
        }
      }
      ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
      for (int j = 0; j < x.ntiles && ok; ++j) {
        const int t = n_tile + j, st = t % kStages;
        const int npg = min(ppt, npages - j * ppt);
        const int nxt = (j + 1) * ppt;
        const int pid_next = (j + 1 < x.ntiles && lane < min(ppt, npages - nxt)) ? __ldg(ids + nxt + lane) : 0;
        // no lane waits alone while the others stand at a convergence point
        if (t >= kStages) ok = tc::mbar_wait(empty_bar(st), ((t / kStages) + 1) & 1, abort_flag, a.status);
        ok = __all_sync(0xffffffffu, ok);
        if (ok && lane == 0) tc::mbar_arrive_expect_tx(full_bar(st), (uint32_t)(npg * a.page_size * kD * 2 * 2));
        if (!ok) break;
        const uint32_t kdst = sbase + Smem::kv + st * kStageBytes;
        const uint32_t vdst = kdst + kKBytes;
        for (int i = 0; i < npg; ++i) {
          const int page = __shfl_sync(0xffffffffu, pid, i);
          if (lane == 0) {
            if ((unsigned)page >= (unsigned)a.num_pages) report(a.status, SKV_DEV_PAGE_OOB);
            const uint32_t row_off = (uint32_t)(i * a.page_size * 128);
#pragma unroll
            for (int rgn = 0; rgn < kRegions; ++rgn) {
              tc::tma_load_4d(kdst + rgn * (kTile * 128) + row_off, &kmap, full_bar(st), rgn * 64, x.kh, 0, page, pol);
              tc::tma_load_4d(vdst + rgn * (kTile * 128) + row_off, &vmap, full_bar(st), rgn * 64, x.kh, 0, page, pol);
            }
          }
        }
        pid = pid_next;
      }
      n_tile += x.ntiles;
      ++n_unit;
    }
    if (!ok && lane == 0) {  // drain the copies already issued (bounded) before the CTA can exit
      for (int t = max(0, n_tile - kStages); t < n_tile; ++t) {
        const uint64_t t_start = tc::globaltimer_ns();
        while (!tc::mbar_try_wait(full_bar(t % kStages), (t / kStages) & 1) &&
               tc::globaltimer_ns() - t_start < 50000000ull) {
        }
      }
    }
  } else if (warp == 5) {
    // ======================================================================= MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_s = tc::idesc_bf16_f32(128, 16, false, false);
      constexpr uint32_t idesc_o = tc::idesc_bf16_f32(128, 16, true, false);
      int n_tile = 0, n_unit = 0;
      bool ok = true;
      auto issue_pv = [&](int t) -> bool {
        const int st = t % kStages, pb = t & 1, ob = t & 1;
        if (!tc::mbar_wait(pfull_bar(pb), (t >> 1) & 1, abort_flag, a.status)) return false;
        if (t >= 2 && !tc::mbar_wait(oempty_bar(ob), ((t >> 1) + 1) & 1, abort_flag, a.status)) return false;
        tc::tc_fence_after();
        const uint32_t vs = sbase + Smem::kv + st * kStageBytes + kKBytes;
        const uint32_t ps = sbase + Smem::p + pb * kPBytes;
#pragma unroll
        for (int k = 0; k < kTile / 16; ++k) {
          const uint64_t ad = tc::sdesc_sw128(vs + k * 2048, kTile * 128, 1024);
          const uint64_t bd = tc::sdesc_sw128(ps + (k >> 2) * 2048 + (k & 3) * 32, 16, 1024);
          tc::mma_bf16(tmem + 32 + ob * 16, ad, bd, idesc_o, k > 0 ? 1u : 0u);
        }
        tc::mma_commit(ofull_bar(ob));
        tc::mma_commit(empty_bar(st));
        return true;
      };
      for (int u = blockIdx.x; u < a.num_units && ok; u += G) {
        const Unit x = load_unit(a, work, u);
        if (x.ntiles == 0) continue;
        const int qb = n_unit & 1;
        ok = tc::mbar_wait(qfull_bar(qb), (n_unit >> 1) & 1, abort_flag, a.status);
        if (!ok) break;
        tc::tc_fence_after();
        const uint32_t qs = sbase + Smem::q + qb * kQBytes;
        for (int j = 0; j < x.ntiles && ok; ++j) {
          const int t = n_tile + j, st = t % kStages, sb = t & 1;
          ok = tc::mbar_wait(full_bar(st), (t / kStages) & 1, abort_flag, a.status);
          if (ok && t >= 2) ok = tc::mbar_wait(sempty_bar(sb), ((t >> 1) + 1) & 1, abort_flag, a.status);
          if (!ok) break;
          tc::tc_fence_after();
          const uint32_t ks = sbase + Smem::kv + st * kStageBytes;
#pragma unroll
          for (int k = 0; k < kD / 16; ++k) {
            const uint64_t ad = tc::sdesc_sw128(ks + (k >> 2) * (kTile * 128) + (k & 3) * 32, 16, 1024);
            const uint64_t bd = tc::sdesc_sw128(qs + (k >> 2) * (16 * 128) + (k & 3) * 32, 16, 1024);
            tc::mma_bf16(tmem + sb * 16, ad, bd, idesc_s, k > 0 ? 1u : 0u);
          }
          tc::mma_commit(sfull_bar(sb));
          if (j >= 1) ok = issue_pv(t - 1);
        }
        if (ok) ok = issue_pv(n_tile + x.ntiles - 1);
        if (ok) tc::mma_commit(qempty_bar(qb));
        n_tile += x.ntiles;
        ++n_unit;
      }
    }
  } else {
    // ======================================================================= softmax / accumulate
    float* red = reinterpret_cast<float*>(smem + Smem::red);
    float* lred = reinterpret_cast<float*>(smem + Smem::lred);
    const uint32_t tm_lane = tmem + ((uint32_t)(warp * 32) << 16);
    int n_tile = 0;
    bool ok = true;
    for (int u = blockIdx.x; u < a.num_units && ok; u += G) {
      const Unit x = load_unit(a, work, u);
      const int rows = x.q_count * a.g;
      if (x.ntiles == 0) {
        // no tokens: O = 0, LSE = -inf
        for (int c = 0; c < rows; ++c) {
          const int qi = c / a.g, h = x.kh * a.g + c % a.g;
          if (x.part_row < 0) {
            store_out(reinterpret_cast<OutT*>(a.o) + ((int64_t)(x.q_start + qi) * a.hq + h) * kD + tid, 0.f);
            if (a.lse != nullptr && tid == 0) a.lse[(int64_t)(x.q_start + qi) * a.hq + h] = -INFINITY;
          } else {
            const int64_t prow = (int64_t)x.part_row + (int64_t)qi * x.part_stride;
            a.o_part[(prow * a.hq + h) * kD + tid] = 0.f;
            if (tid == 0) a.lse_part[prow * a.hq + h] = -INFINITY;
          }
        }
        continue;
      }
      float m[NC], l[NC], acc[NC], alpha[NC], alpha_prev[NC];
#pragma unroll
      for (int c = 0; c < NC; ++c) {
        m[c] = -INFINITY;
        l[c] = 0.f;
        acc[c] = 0.f;
        alpha_prev[c] = 1.f;
      }
      auto accumulate = [&](int t, const float (&al)[NC]) {
        const int ob = t & 1;
        ok = tc::mbar_wait(ofull_bar(ob), (t >> 1) & 1, abort_flag, a.status) && ok;
        tc::tc_fence_after();
        float o[NC];
        tc::tmem_ld<NC>(tm_lane + 32 + ob * 16, o);
        tc::tmem_wait_ld();
        tc::tc_fence_before();
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(oempty_bar(ob));
#pragma unroll
        for (int c = 0; c < NC; ++c) acc[c] = fmaf(acc[c], al[c], o[c]);
      };
      bool failed = false;
      for (int j = 0; j < x.ntiles; ++j) {
        const int t = n_tile + j, sb = t & 1, st = t % kStages;
        ok = tc::mbar_wait(sfull_bar(sb), (t >> 1) & 1, abort_flag, a.status) && ok;
        tc::tc_fence_after();
        float s[NC];
        tc::tmem_ld<NC>(tm_lane + sb * 16, s);
        tc::tmem_wait_ld();
        tc::tc_fence_before();
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(sempty_bar(sb));
        const bool valid = x.t0 + j * kTile + tid < x.t1;
        float* rr = red + (t & 1) * 64;
#pragma unroll
        for (int c = 0; c < NC; ++c) {
          s[c] = (valid && c < rows) ? s[c] * a.scale_log2 : -INFINITY;
          const float v = warp_max(s[c]);
          if (lane == 0) rr[warp * 16 + c] = v;
        }
        if (!valid) {  // zero this token's V row (both 64-column halves) before the PV MMA reads it
          uint8_t* vrow = smem + Smem::kv + st * kStageBytes + kKBytes + tid * 128;
#pragma unroll
          for (int rgn = 0; rgn < kRegions; ++rgn)
#pragma unroll
            for (int i = 0; i < 8; ++i)
              reinterpret_cast<uint4*>(vrow + rgn * (kTile * 128))[i] = make_uint4(0, 0, 0, 0);
        }
        if (!bar_and(1, kSoftmaxThreads, ok)) {
          ok = false;
          failed = true;
          break;
        }
        uint8_t* pbuf = smem + Smem::p + (t & 1) * kPBytes + (tid >> 6) * 2048;
#pragma unroll
        for (int c = 0; c < NC; ++c) {
          const float tmax = fmaxf(fmaxf(rr[c], rr[16 + c]), fmaxf(rr[32 + c], rr[48 + c]));
          const float mn = fmaxf(m[c], tmax);
          alpha[c] = (mn == -INFINITY) ? 1.f : exp2f(m[c] - mn);
          const float p = (s[c] == -INFINITY) ? 0.f : exp2f(s[c] - mn);
          l[c] = fmaf(l[c], alpha[c], p);
          m[c] = mn;
          if (c < rows)
            *reinterpret_cast<__nv_bfloat16*>(pbuf + tc::sw128_offset(c, tid & 63)) = __float2bfloat16_rn(p);
        }
        tc::fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(pfull_bar(t & 1));
        if (j >= 1) accumulate(t - 1, alpha_prev);
#pragma unroll
        for (int c = 0; c < NC; ++c) alpha_prev[c] = alpha[c];
      }
      if (failed) break;  // uniform: set only from a bar_and result
      accumulate(n_tile + x.ntiles - 1, alpha_prev);
      n_tile += x.ntiles;
      // row sums: per-thread partials -> per column totals
#pragma unroll
      for (int c = 0; c < NC; ++c) {
        const float v = warp_sum(l[c]);
        if (lane == 0) lred[warp * 16 + c] = v;
      }
      if (!bar_and(1, kSoftmaxThreads, ok)) {
        ok = false;
        break;
      }
#pragma unroll
      for (int c = 0; c < NC; ++c) {
        if (c >= rows) break;
        const float lt = lred[c] + lred[16 + c] + lred[32 + c] + lred[48 + c];
        const float inv = lt > 0.f ? 1.f / lt : 0.f;
        const float lse = lt > 0.f ? (m[c] + log2f(lt)) * kLn2 : -INFINITY;
        const int qi = c / a.g, h = x.kh * a.g + c % a.g;
        if (x.part_row < 0) {
          store_out(reinterpret_cast<OutT*>(a.o) + ((int64_t)(x.q_start + qi) * a.hq + h) * kD + tid, acc[c] * inv);
          if (a.lse != nullptr && tid == c) a.lse[(int64_t)(x.q_start + qi) * a.hq + h] = lse;
        } else {
          const int64_t prow = (int64_t)x.part_row + (int64_t)qi * x.part_stride;
          a.o_part[(prow * a.hq + h) * kD + tid] = acc[c] * inv;
          if (tid == c) a.lse_part[prow * a.hq + h] = lse;
        }
      }
    }
  }

  tc::tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, kTmemCols);
  }
}

// ------------------------------------------------------------------------------ host side
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
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

bool make_map(CUtensorMap* m, const void* base, int rank, const cuuint64_t* dims, const cuuint64_t* strides_bytes,
              const cuuint32_t* box) {
  auto fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, const_cast<void*>(base), dims, strides_bytes, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

int num_sms() { return device_sm_count(); }

template <int NC, typename OutT>
int launch_t(const CUtensorMap& km, const CUtensorMap& vm, const CUtensorMap& qm, const TcArgs& a,
             const WorkItem* work, cudaStream_t s) {
  const int smem = Smem::total + 1024;
  static DeviceSmemAttr attr;  // per device: the attribute belongs to the current device
  if (const int e = attr.ensure(reinterpret_cast<const void*>(gqa_tc_decode_kernel<NC, OutT>), smem)) return e;
  const int grid = std::min(a.num_units, num_sms());
  gqa_tc_decode_kernel<NC, OutT><<<grid, kThreads, smem, s>>>(km, vm, qm, a, work);
  return (int)cudaGetLastError();
}

}  // namespace

bool gqa_tc_decode_supported(int head_dim, int page_size, int group, int q_tile) {
  return head_dim == kD && page_size >= 8 && page_size <= kTile && (kTile % page_size) == 0 && group >= 1 &&
         q_tile >= 1 && group * q_tile <= 16;
}

int launch_gqa_tc_decode(const skv_paged_params& p, const WorkItem* work, int num_work, int q_tile,
                         cudaStream_t s) {
  if (num_work == 0) return 0;
  const int g = p.num_qo_heads / p.num_kv_heads;
  if (!gqa_tc_decode_supported(p.head_dim, p.page_size, g, q_tile)) return (int)cudaErrorInvalidValue;
  CUtensorMap km, vm, qm;
  {
    const cuuint64_t dims[4] = {(cuuint64_t)kD, (cuuint64_t)p.num_kv_heads, (cuuint64_t)p.page_size,
                                (cuuint64_t)std::max(1, p.num_pages)};
    const cuuint32_t box[4] = {64, 1, (cuuint32_t)p.page_size, 1};
    const cuuint64_t ks[3] = {(cuuint64_t)p.k_stride[2] * 2, (cuuint64_t)p.k_stride[1] * 2,
                              (cuuint64_t)p.k_stride[0] * 2};
    const cuuint64_t vs[3] = {(cuuint64_t)p.v_stride[2] * 2, (cuuint64_t)p.v_stride[1] * 2,
                              (cuuint64_t)p.v_stride[0] * 2};
    if (!make_map(&km, p.k_cache, 4, dims, ks, box)) return (int)cudaErrorInvalidValue;
    if (!make_map(&vm, p.v_cache, 4, dims, vs, box)) return (int)cudaErrorInvalidValue;
  }
  {
    const cuuint64_t dims[3] = {(cuuint64_t)kD, (cuuint64_t)p.num_qo_heads, (cuuint64_t)std::max(1, p.total_q)};
    const cuuint64_t st[2] = {(cuuint64_t)kD * 2, (cuuint64_t)p.num_qo_heads * kD * 2};
    const cuuint32_t box[3] = {64, (cuuint32_t)g, (cuuint32_t)q_tile};
    if (!make_map(&qm, p.q, 3, dims, st, box)) return (int)cudaErrorInvalidValue;
  }
  TcArgs a;
  a.kv_indptr = p.kv_indptr;
  a.kv_indices = p.kv_indices;
  a.last = p.kv_last_page_len;
  a.num_pages = p.num_pages;
  a.page_size = p.page_size;
  a.hq = p.num_qo_heads;
  a.hk = p.num_kv_heads;
  a.g = g;
  a.q_tile = q_tile;
  a.num_units = num_work * p.num_kv_heads;
  a.scale_log2 = p.sm_scale * kLog2e;
  a.o = p.o;
  a.lse = p.lse;
  a.o_part = p.o_part;
  a.lse_part = p.lse_part;
  a.status = p.status;
  const bool bf = p.o_dtype == SKV_BF16;
  if (g * q_tile <= 8)
    return bf ? launch_t<8, __nv_bfloat16>(km, vm, qm, a, work, s) : launch_t<8, float>(km, vm, qm, a, work, s);
  return bf ? launch_t<16, __nv_bfloat16>(km, vm, qm, a, work, s) : launch_t<16, float>(km, vm, qm, a, work, s);
}

}  // namespace skv
