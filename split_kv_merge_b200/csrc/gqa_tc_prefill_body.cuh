#pragma once
// Device body of paged GQA attention for many query rows per KV head (prefill, shared-KV
// broadcast) on the tensor cores (tcgen05 + TMEM), TMA page staging.
//
// What it computes: for a work item (request r, query tokens [q_start, q_start + q_count),
// logical pages [page_begin, page_end)) and KV head kh, the attention of its q_count * g query
// rows over the item's tokens, no mask (every query token sees all of the request's KV) -- the
// output, or the split partial (O_j, LSE_j) that merge_states combines.  Query batches that list
// the same pages share one KV with no copy (KV batch broadcast, PyTorch MPS FlexAttention page);
// each row's arithmetic depends only on logical positions, so a shared and a replicated KV give
// bit-identical results.
//
// B200 design: the standard (non-swapped) flash-attention tile with 128 query rows as M:
//   S[128 rows, 128 keys] = Q[128, 128] . K^T      (rows = (query token, head of the group))
//   O[128 rows, 128]     += P[128, 128 keys] . V  (V read MN-major from the same TMA tile)
// S (double buffered), O and P (double buffered, bf16 pairs) all live in TMEM: the softmax writes
// P with tcgen05.st and the PV MMA reads it as its A operand straight from TMEM, so P never
// touches shared memory, which holds three 64 KB K+V stages instead.  A row is owned by two
// threads of two warps on the same TMEM lane quarter (keys [64 hf, 64 hf + 64) of every tile and
// head dims [64 hf, 64 hf + 64) of O each), exchanging row maxima and sums through shared memory;
// the running max is raised lazily (only when a score passes it by more than 2^8) and O is
// rescaled in TMEM (warp-uniform decision, since TMEM access is warp-collective).  Roles: warp 4
// TMA (3-stage ring of 128-key K and V tiles, 3-D Q box), warp 5 TMEM + QK MMA issue, warp 6 PV
// MMA issue, warps 0-3 and 7-10 softmax / epilogue.  Keys past the end of the item get s = -inf by
// selection and their V rows are zeroed before the PV that reads them.  All waits are bounded.
#include <algorithm>

#include "tc_ptx.cuh"

namespace skv {
namespace prefill {

constexpr int kTile = 128;                      // keys per tile
constexpr int kRows = 128;                      // query rows per CTA
constexpr int kD = 128;
constexpr int kStages = 3;
constexpr int kRegion = kTile * 128;            // 16 KB: one 64-column half of a 128 x 128 tile
constexpr int kKBytes = 2 * kRegion;            // 32 KB
constexpr int kStageBytes = 2 * kKBytes;        // K + V
constexpr int kThreads = 352;  // softmax warps 0-3 and 7-10, TMA warp 4, QK warp 5, PV warp 6
constexpr float kRaise = 8.f;

struct Smem {
  static constexpr int kv = 0;
  static constexpr int q = kv + kStages * kStageBytes;    // 196608
  static constexpr int bars = q + kKBytes;                // 229376 (P lives in TMEM)
  static constexpr int nbars = 2 * kStages + 1 + 2 * 4;
  static constexpr int xch = bars + nbars * 8;            // [2][128] float: per-row exchange between halves
  static constexpr int misc = xch + 2 * 128 * 4;
  static constexpr int total = misc + 16;
};
static_assert(Smem::total + 1024 <= 232448, "fits the 227 KB opt-in shared memory");

// D[tmem] (+)= A[tmem] . B[smem], kind::f16: A rows in TMEM lanes, two bf16 per 32-bit column
// (the even k in the low half)
__device__ __forceinline__ void mma_bf16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                            uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// packed f32 pairs (sm_100 f32x2 arithmetic), 3-input max, hardware exp2
__device__ __forceinline__ uint64_t pk2(float a, float b) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
  return r;
}
__device__ __forceinline__ void upk2(uint64_t v, float& a, float& b) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(v));
}
__device__ __forceinline__ uint64_t fma2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
  return r;
}
__device__ __forceinline__ uint64_t add2(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}
__device__ __forceinline__ float ex2(float x) {
  float r;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
  return r;
}

struct PArgs {
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

// The kernel body, run by a CTA of kThreads threads for unit `unit` (work item unit / Hk, KV head
// unit % Hk).
template <typename OutT>
__device__ __forceinline__ void prefill_body(const CUtensorMap& kmap, const CUtensorMap& vmap,
                                             const CUtensorMap& qmap, const PArgs& a,
                                             const WorkItem* __restrict__ work, int unit) {
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
  auto qfull_bar = [&]() { return bar0 + 8u * (2 * kStages); };
  auto sfull_bar = [&](int b) { return bar0 + 8u * (2 * kStages + 1 + b); };
  auto sempty_bar = [&](int b) { return bar0 + 8u * (2 * kStages + 3 + b); };
  auto pfull_bar = [&](int b) { return bar0 + 8u * (2 * kStages + 5 + b); };
  auto ofull_bar = [&](int b) { return bar0 + 8u * (2 * kStages + 7 + b); };

  // ---- the unit: work item u / Hk, KV head u % Hk
  const int u = unit;
  const WorkItem w = work[u / a.hk];
  const int kh = u % a.hk;
  const int L = request_len(a.kv_indptr, a.last, w.r, a.page_size);
  const int t0 = w.page_begin * a.page_size;
  const int t1 = min(w.page_end * a.page_size, L);
  const int T = t1 > t0 ? (t1 - t0 + kTile - 1) / kTile : 0;
  const int rows = w.q_count * a.g;

  if (T == 0) {  // no keys: O = 0, LSE = -inf (rows only; no TMEM, no barriers)
    if (tid < 128 && tid < rows) {
      const int qi = tid / a.g, h = kh * a.g + tid % a.g;
      if (w.part_row < 0) {
        OutT* dst = reinterpret_cast<OutT*>(a.o) + ((int64_t)(w.q_start + qi) * a.hq + h) * kD;
        for (int d = 0; d < kD; ++d) store_out(dst + d, 0.f);
        if (a.lse != nullptr) a.lse[(int64_t)(w.q_start + qi) * a.hq + h] = -INFINITY;
      } else {
        const int64_t prow = (int64_t)w.part_row + (int64_t)qi * w.part_stride;
        for (int d = 0; d < kD; ++d) a.o_part[(prow * a.hq + h) * kD + d] = 0.f;
        a.lse_part[prow * a.hq + h] = -INFINITY;
      }
    }
    return;
  }

  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      tc::mbar_init(full_bar(s), 1);
      tc::mbar_init(empty_bar(s), 1);
    }
    tc::mbar_init(qfull_bar(), 1);
    for (int b = 0; b < 2; ++b) {
      tc::mbar_init(sfull_bar(b), 1);
      tc::mbar_init(sempty_bar(b), 8);
      tc::mbar_init(pfull_bar(b), 8);
      tc::mbar_init(ofull_bar(b), 1);
    }
    *abort_flag = 0;
    tc::fence_mbar_init();
  }
  if (warp == 5) tc::tmem_alloc(tc::smem_u32(tmem_holder), 512);
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  // TMEM: S0, S1 (128 fp32 columns each), O (128), P0, P1 (64 columns each: 128 bf16 keys per row)
  const uint32_t tm_s = tmem, tm_o = tmem + 2 * kTile, tm_p = tmem + 3 * kTile;

  if (warp == 4) {
    // ======================================================================= TMA producer
    // The whole warp streams the tiles: lanes hold the ids of the next 32 pages of the item (one
    // per lane), the whole warp waits for the stage, and lane i issues the K and V boxes of page i
    // of the tile (a 128-key tile of 16-token pages is eight pages: their boxes go out at once
    // instead of one after another behind eight dependent page-id loads).
    bool ok = true;
    int issued = 0;
    if (lane == 0) {
      tc::prefetch_tmap(&kmap);
      tc::prefetch_tmap(&vmap);
      tc::mbar_arrive_expect_tx(qfull_bar(), (uint32_t)(kRows * kD * 2));
      for (int rgn = 0; rgn < 2; ++rgn)
        tc::tma_load_3d(sbase + Smem::q + rgn * kRegion, &qmap, qfull_bar(), rgn * 64, kh * a.g, w.q_start);
    }
    const int* ids = a.kv_indices + a.kv_indptr[w.r] + w.page_begin;
    const int npages = w.page_end - w.page_begin;
    const int P = a.page_size, box_rows = min(P, kTile);
    const uint64_t pol = tc::policy_evict_first();
    int win = -1000000, pid = 0;  // lanes hold the ids of pages [win, win + 32) of the item
    for (int t = 0; t < T && ok; ++t) {
      const int st = t % kStages;
      // the whole warp waits for the stage (no lane waits alone while the others stand at a
      // convergence point)
      if (t >= kStages) ok = tc::mbar_wait(empty_bar(st), ((t / kStages) + 1) & 1, abort_flag, a.status);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      const int pi0 = (t * kTile) / P;
      const int npg = P >= kTile ? 1 : min(kTile / P, npages - pi0);
      const int slot0 = P >= kTile ? (t * kTile) % P : 0;
      if (pi0 < win || pi0 + npg > win + 32) {
        win = pi0;
        pid = (win + lane < npages) ? __ldg(ids + win + lane) : 0;
      }
      const int page = __shfl_sync(0xffffffffu, pid, (pi0 - win + lane) & 31);
      if (lane == 0) tc::mbar_arrive_expect_tx(full_bar(st), (uint32_t)(2 * 2 * npg * box_rows * 128));
      __syncwarp();
      if (lane < npg) {
        if ((unsigned)page >= (unsigned)a.num_pages) report(a.status, SKV_DEV_PAGE_OOB);
        const uint32_t kdst = sbase + Smem::kv + st * kStageBytes + (uint32_t)(lane * box_rows * 128);
        for (int rgn = 0; rgn < 2; ++rgn) {
          tc::tma_load_4d(kdst + rgn * kRegion, &kmap, full_bar(st), rgn * 64, kh, slot0, page, pol);
          tc::tma_load_4d(kdst + kKBytes + rgn * kRegion, &vmap, full_bar(st), rgn * 64, kh, slot0, page, pol);
        }
      }
      issued = t + 1;
    }
    if (!ok && lane == 0) {  // the copies of the last tile in each stage may still be landing: wait (bounded)
      for (int t = max(0, issued - kStages); t < issued; ++t) {
        const uint64_t t_start = tc::globaltimer_ns();
        while (!tc::mbar_try_wait(full_bar(t % kStages), (t / kStages) & 1) &&
               tc::globaltimer_ns() - t_start < 20000000ull) {
        }
      }
    }
  } else if (warp == 5) {
    // ======================================================================= QK MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_s = tc::idesc_bf16_f32(128, kTile, false, false);
      bool ok = tc::mbar_wait(qfull_bar(), 0, abort_flag, a.status);
      tc::tc_fence_after();
      const uint32_t qs = sbase + Smem::q;
      for (int t = 0; t < T && ok; ++t) {
        const int st = t % kStages, sb = t & 1;
        ok = tc::mbar_wait(full_bar(st), (t / kStages) & 1, abort_flag, a.status);
        if (ok && t >= 2) ok = tc::mbar_wait(sempty_bar(sb), ((t >> 1) + 1) & 1, abort_flag, a.status);
        if (!ok) break;
        tc::tc_fence_after();
        const uint32_t ks = sbase + Smem::kv + st * kStageBytes;
#pragma unroll
        for (int k = 0; k < kD / 16; ++k) {
          const uint64_t ad = tc::sdesc_sw128(qs + (k >> 2) * kRegion + (k & 3) * 32, 16, 1024);
          const uint64_t bd = tc::sdesc_sw128(ks + (k >> 2) * kRegion + (k & 3) * 32, 16, 1024);
          tc::mma_bf16(tm_s + sb * kTile, ad, bd, idesc_s, k > 0 ? 1u : 0u);
        }
        tc::mma_commit(sfull_bar(sb));
      }
    }
  } else if (warp == 6) {
    // ======================================================================= PV MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_o = tc::idesc_bf16_f32(128, kD, false, true);
      bool ok = true;
      for (int t = 0; t < T && ok; ++t) {
        const int st = t % kStages, pb = t & 1;
        ok = tc::mbar_wait(pfull_bar(pb), (t >> 1) & 1, abort_flag, a.status);
        if (!ok) break;
        tc::tc_fence_after();
        const uint32_t vs = sbase + Smem::kv + st * kStageBytes + kKBytes;
#pragma unroll
        for (int k = 0; k < kTile / 16; ++k) {  // A = P from TMEM: 16 keys = 8 packed columns
          const uint64_t bd = tc::sdesc_sw128(vs + k * 2048, kRegion, 1024);
          mma_bf16_ts(tm_o, tm_p + pb * (kTile / 2) + k * 8, bd, idesc_o, (t > 0 || k > 0) ? 1u : 0u);
        }
        tc::mma_commit(ofull_bar(pb));
        tc::mma_commit(empty_bar(st));
      }
    }
  } else if (warp < 4 || warp >= 7) {
    // ======================================================================= softmax / epilogue
    // Each row is split over two warps on the same TMEM lane quarter (warp w and warp w + 8, or
    // 3 and 7): half hf takes keys [64 hf, 64 hf + 64) of every tile and head dims [64 hf,
    // 64 hf + 64) of O; the two threads of a row exchange row maxima and sums through shared
    // memory with a 64-thread named barrier per pair.
    const int quarter = warp & 3, hf = warp < 4 ? 0 : 1;
    const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
    const int r = quarter * 32 + lane;       // this thread's query row
    float* xch = reinterpret_cast<float*>(smem + Smem::xch);
    auto pair_sync = [&]() { tc::named_bar_sync(1 + quarter, 64); };
    // l: sum of the exact weights (for the LSE); lr: of the bf16-rounded weights PV multiplies (the
    // divisor of O, so that a row dominated by one key reproduces that key's V)
    float m = -INFINITY, l = 0.f, lr = 0.f;
    int pv_seen = 0;
    bool ok = true;
    auto consume_pv = [&](int upto) {
      for (; pv_seen <= upto; ++pv_seen)
        ok = tc::mbar_wait(ofull_bar(pv_seen & 1), (pv_seen >> 1) & 1, abort_flag, a.status) && ok;
      tc::tc_fence_after();
    };
    for (int t = 0; t < T; ++t) {
      const int sb = t & 1, st = t % kStages;
      ok = tc::mbar_wait(sfull_bar(sb), (t >> 1) & 1, abort_flag, a.status) && ok;
      tc::tc_fence_after();
      constexpr int kH = kTile / 2;           // keys of this half
      float s[kH];
#pragma unroll
      for (int c = 0; c < kH; c += 16) {  // all loads in flight, one wait
        float v16[16];
        tc::tmem_ld_x16(tm_s + lane_base + sb * kTile + hf * kH + c, v16);
#pragma unroll
        for (int i = 0; i < 16; ++i) s[c + i] = v16[i];
      }
      tc::tmem_wait_ld();
      tc::tc_fence_before();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(sempty_bar(sb));
      const int nvalid = t1 - (t0 + t * kTile) - hf * kH;  // keys of this half that exist (may be <= 0)
      if (nvalid < kH) {                                    // the item's last tile only
#pragma unroll
        for (int c = 0; c < kH; ++c) s[c] = c < nvalid ? s[c] : -INFINITY;
      }
      float mx;
      {  // raw row maximum in 4 independent chains (the scale is positive: scale after), then the
         // other half's through shared memory
        float q[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          float v = fmax3(s[16 * j], s[16 * j + 1], s[16 * j + 2]);
#pragma unroll
          for (int i = 3; i < 15; i += 2) v = fmax3(v, s[16 * j + i], s[16 * j + i + 1]);
          q[j] = fmaxf(v, s[16 * j + 15]);
        }
        mx = fmaxf(fmaxf(q[0], q[1]), fmaxf(q[2], q[3])) * a.scale_log2;
        xch[hf * 128 + r] = mx;
        pair_sync();
        mx = fmaxf(mx, xch[(1 - hf) * 128 + r]);
        pair_sync();  // both reads done before the next tile's writes
      }
      const bool raise = mx > m + kRaise;
      if (__any_sync(0xffffffffu, raise)) {  // warp-uniform: TMEM access below is warp-collective
        const float mn = raise ? mx : m;
        const float al = (mn == -INFINITY || m == mn) ? 1.f : exp2f(m - mn);
        l *= al;
        lr *= al;
        m = mn;
        if (t > 0) {  // rescale this row of O once the previous PV is done
          consume_pv(t - 1);
#pragma unroll
          for (int c = 0; c < kD / 2; c += 16) {  // this half's head dims of the row
            float ov[16];
            tc::tmem_ld_x16(tm_o + lane_base + hf * (kD / 2) + c, ov);
            tc::tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 16; ++i) ov[i] *= al;
            tc::tmem_st_x16(tm_o + lane_base + hf * (kD / 2) + c, ov);
          }
          tc::tmem_wait_st();
          tc::tc_fence_before();
        }
      }
      const int nvalid_tile = t1 - (t0 + t * kTile);
      if (nvalid_tile < kTile) {  // zero V rows of missing keys (each thread its share of the rows)
        // the tile's copies have landed (the QK that read them is done); make that visible here
        ok = tc::mbar_wait(full_bar(st), (t / kStages) & 1, abort_flag, a.status) && ok;
        uint8_t* vb = smem + Smem::kv + st * kStageBytes + kKBytes;
        for (int row = nvalid_tile + hf * 128 + r; row < kTile; row += 256)
#pragma unroll
          for (int rgn = 0; rgn < 2; ++rgn)
#pragma unroll
            for (int i = 0; i < 8; ++i)
              reinterpret_cast<uint4*>(vb + rgn * kRegion + row * 128)[i] = make_uint4(0, 0, 0, 0);
      }
      if (t >= 2 && pv_seen <= t - 2) consume_pv(t - 2);  // P(t) reuses the buffer PV(t-2) read
      // p = 2^(s * scale - m) (ex2 of -inf is +0), bf16 pairs into this row's P columns in TMEM; sums
      // of the exact and of the rounded weights in packed pairs, two chains each
      const uint64_t sc2 = pk2(a.scale_log2, a.scale_log2), nm2 = pk2(-m, -m);
      uint64_t la[2] = {pk2(0.f, 0.f), pk2(0.f, 0.f)}, lb[2] = {pk2(0.f, 0.f), pk2(0.f, 0.f)};
      float pw[kH / 2];  // packed bf16 pairs (bit patterns)
#pragma unroll
      for (int c = 0; c < kH; c += 2) {
        float x0, x1;
        upk2(fma2(pk2(s[c], s[c + 1]), sc2, nm2), x0, x1);
        const float p0 = ex2(x0), p1 = ex2(x1);
        __nv_bfloat162 h2 = __floats2bfloat162_rn(p0, p1);
        const uint32_t u = *reinterpret_cast<uint32_t*>(&h2);
        pw[c >> 1] = __uint_as_float(u);
        la[(c >> 1) & 1] = add2(la[(c >> 1) & 1], pk2(p0, p1));
        lb[(c >> 1) & 1] = add2(lb[(c >> 1) & 1], pk2(__uint_as_float(u << 16), __uint_as_float(u & 0xffff0000u)));
      }
      {
        float a0, a1, b0, b1;
        upk2(add2(la[0], la[1]), a0, a1);
        upk2(add2(lb[0], lb[1]), b0, b1);
        l += a0 + a1;
        lr += b0 + b1;
      }
      const uint32_t pcol = tm_p + (t & 1) * (kTile / 2) + hf * (kH / 2);
#pragma unroll
      for (int c = 0; c < kH / 2; c += 16) {
        float w16[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) w16[i] = pw[c + i];
        tc::tmem_st_x16(pcol + lane_base + c, w16);
      }
      tc::tmem_wait_st();
      tc::fence_proxy_async_smem();  // V rows zeroed above are read by the PV MMA
      tc::tc_fence_before();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(pfull_bar(t & 1));
    }
    consume_pv(T - 1);
    xch[hf * 128 + r] = l;  // row sums: exact weights, then rounded weights, over both halves
    pair_sync();
    l += xch[(1 - hf) * 128 + r];
    pair_sync();
    xch[hf * 128 + r] = lr;
    pair_sync();
    lr += xch[(1 - hf) * 128 + r];
    const bool live = r < rows;
    const int qi = r / a.g, h = kh * a.g + r % a.g;
    const float inv = lr > 0.f ? 1.f / lr : 0.f;
    float* op = nullptr;
    OutT* oo = nullptr;
    if (live) {
      const float lse = l > 0.f ? (m + log2f(l)) * kLn2 : -INFINITY;
      if (w.part_row < 0) {
        oo = reinterpret_cast<OutT*>(a.o) + ((int64_t)(w.q_start + qi) * a.hq + h) * kD + hf * (kD / 2);
        if (a.lse != nullptr && hf == 0) a.lse[(int64_t)(w.q_start + qi) * a.hq + h] = lse;
      } else {
        const int64_t prow = (int64_t)w.part_row + (int64_t)qi * w.part_stride;
        op = a.o_part + (prow * a.hq + h) * kD + hf * (kD / 2);
        if (hf == 0) a.lse_part[prow * a.hq + h] = lse;
      }
    }
#pragma unroll
    for (int c = 0; c < kD / 2; c += 16) {  // every lane loads (warp-collective); live rows store
      float ov[16];
      tc::tmem_ld_x16(tm_o + lane_base + hf * (kD / 2) + c, ov);
      tc::tmem_wait_ld();
      if (op != nullptr) {
#pragma unroll
        for (int i = 0; i < 16; i += 4)
          *reinterpret_cast<float4*>(op + c + i) =
              make_float4(ov[i] * inv, ov[i + 1] * inv, ov[i + 2] * inv, ov[i + 3] * inv);
      } else if (oo != nullptr) {
#pragma unroll
        for (int i = 0; i < 16; ++i) store_out(oo + c + i, ov[i] * inv);
      }
    }
  }

  tc::tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, 512);
  }
}

// Tensor maps and arguments of a launch (host; gqa_tc_prefill.cu): 0 on success, else a CUDA error code.
int prepare(const skv_paged_params& p, int num_work, int q_tile, CUtensorMap* maps, PArgs* a);

}  // namespace prefill
}  // namespace skv
