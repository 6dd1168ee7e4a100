#pragma once
// Device body of the paged GQA decode kernel, all KV heads of a work item in one CTA
// (tcgen05 + TMEM, TMA page staging).
//
// Same result as gqa_tc_decode.cu (attention or split partial of a work item: request r, query
// token(s), logical pages [page_begin, page_end); split-KV + merge per the FlashInfer PR #5597
// page, section 3, and the route primitive of "Move the Query, Not the Cache"), for the shape
// Hk = 8 KV heads, g * q_tile = 8 query rows per KV head, head_dim 128, page_size 16..256.
//
// Why this layout: in the NHD page [slot][head][dim] one KV head's rows are 256 B pieces 2 KB
// apart.  Per-head CTAs read those pieces at different times and HBM then delivers about 3 TB/s;
// reading each 16-token window of a page for all heads at once (two 16 KB TMA boxes per tensor,
// one per half of D) streams the page contiguously at ~6.8 TB/s.  A tile is 16 tokens x 8 heads =
// 128 rows (head-major in shared memory, via the tensor map's dimension order slot-then-head):
//   S^T[128 rows, 64] = K_tile[128, 128] . Q^T[128, 64]          (N = all 64 query rows)
// is block diagonal in meaning: row (h, tok) only uses the 8 columns of its own GQA group.
// PV is done per pair of heads so the probability tile stays small:
//   O^T[:, 16p..16p+16) += V_rows(pair p)^T[128, 32] . P_p^T[32, 16]
// where P_p (16 x 32, K-major) is zero outside its two 8x16 diagonal blocks (zeroed once, only the
// diagonal blocks are ever written).  O^T accumulates in TMEM across the tiles of a work item
// (one 64-column buffer per work item parity).
//
// Online softmax with a lazily raised maximum: each column keeps the maximum m it currently
// exponentiates against, p = exp2(s - m).  The maximum is raised (and l and O^T rescaled by
// exp2(m_old - m_new)) only when some score of a tile exceeds m by more than kRaise = 8, i.e.
// only when p could exceed 2^8; otherwise a tile costs no row-max reduction and no O^T access.
// This is the same exact softmax (every p, l and O term uses one consistent m), computed with
// fewer rescales.  A rescale happens in TMEM by all four softmax warps (each owns 32 head-dim
// lanes) after the previous PV has completed and before the next PV is issued.
//
// Roles: warp 4 TMA producer (3-stage ring of 64 KB K+V tiles, page ids prefetched one per lane,
// Q staged once per work item), warp 5 TMEM allocation + MMA issue, warps 0-3 softmax (thread = one
// (head, token) row of S^T; masked rows get s = -inf by selection and their V rows are zeroed).
// All waits are bounded (SKV_DEV_TIMEOUT); the roles leave together and TMEM is always released.
#include "tc_ptx.cuh"

namespace skv {
namespace wide {

constexpr int kHk = 8;              // KV heads per CTA
constexpr int kTok = 16;            // tokens per tile
constexpr int kRows = kHk * kTok;   // 128 = M of S^T
constexpr int kD = 128;
constexpr int kN = 64;              // query rows (columns of S^T): kHk * 8
constexpr int kStages = 3;
constexpr int kKBytes = kRows * kD * 2;       // 32 KB
constexpr int kStageBytes = 2 * kKBytes;      // K + V
constexpr int kRegion = kRows * 128;          // 16 KB: one 64-column half of D
constexpr int kQBytes = kN * kD * 2;          // 16 KB
constexpr int kQRegion = kN * 128;            // 8 KB
constexpr int kPairBytes = 16 * 128;          // 16 rows x 128 B (32 K columns used)
constexpr int kPBytes = 4 * kPairBytes;       // 8 KB per buffer
constexpr int kThreads = 192;
constexpr int kTmemCols = 256;                // S0 S1 (64 each), O0 O1 (64 each)
constexpr float kRaise = 8.f;                 // raise the running max only past m + 8 (log2 units)

struct Smem {
  static constexpr int kv = 0;
  static constexpr int q = kv + kStages * kStageBytes;     // 196608
  static constexpr int p = q + kQBytes;                     // 212992
  static constexpr int alpha = p + 2 * kPBytes;             // [64] float
  static constexpr int inv = alpha + kN * 4;                // [64] float: 1/l per column
  static constexpr int lse = inv + kN * 4;                  // [64] float
  static constexpr int lsum = lse + kN * 4;                 // [64] float
  static constexpr int msum = lsum + kN * 4;                // [64] float
  static constexpr int bars = msum + kN * 4;
  static constexpr int nbars = 2 * kStages + 2 + 2 * 5;  // ring, Q, S, P, O full / free
  static constexpr int misc = bars + nbars * 8;
  static constexpr int total = misc + 16;
};
static_assert(Smem::total + 1024 <= 232448, "fits the 227 KB opt-in shared memory");

struct WArgs {
  const int32_t* kv_indptr;
  const int32_t* kv_indices;
  const int32_t* last;
  int num_pages, page_size, hq, q_tile, num_ctas;
  const int32_t* cta_indptr;  // CTA c runs work items cta_indptr[c] .. cta_indptr[c+1]
  float scale_log2;
  void* o;
  float* lse;
  float* o_part;
  float* lse_part;
  int32_t* status;
};

struct WUnit {
  int r, q_start, q_count, page_begin, page_end, part_row, part_stride;
  int t0, t1, ntiles;
};

__device__ __forceinline__ WUnit load_wunit(const WArgs& a, const WorkItem* work, int u) {
  WUnit x;
  const WorkItem w = work[u];
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
  x.ntiles = x.t1 > x.t0 ? (x.t1 - x.t0 + kTok - 1) / kTok : 0;
  return x;
}

__device__ __forceinline__ void tma_load_4d_nohint(uint32_t dst, const CUtensorMap* map, uint32_t bar, int c0, int c1,
                                                   int c2, int c3) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5, %6}], "
      "[%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
      : "memory");
}

// column n of S^T / O^T -> (query token offset, query head), G = GQA group size (8 / q_tile)
template <int G>
__device__ __forceinline__ void column_row(int n, int& qi, int& hq) {
  const int e = n & 7;
  qi = e / G;
  hq = (n >> 3) * G + e % G;
}

// The kernel body, run by CTA `cta` of the persistent grid (blockDim >= 192: warps 0-5 take the
// roles below; any further warps only join the block-wide barriers at entry and exit).
template <int G, typename OutT>
__device__ __forceinline__ void wide_body(const CUtensorMap& kmap, const CUtensorMap& vmap, const CUtensorMap& qmap,
                                          const WArgs& a, const WorkItem* __restrict__ work, int cta) {
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
  auto qempty_bar = [&]() { return bar0 + 8u * (2 * kStages + 1); };
  auto sfull_bar = [&](int b) { return bar0 + 8u * (2 * kStages + 2 + b); };
  auto sempty_bar = [&](int b) { return bar0 + 8u * (2 * kStages + 4 + b); };
  auto pfull_bar = [&](int b) { return bar0 + 8u * (2 * kStages + 6 + b); };
  auto ofull_bar = [&](int b) { return bar0 + 8u * (2 * kStages + 8 + b); };
  auto ofree_bar = [&](int b) { return bar0 + 8u * (2 * kStages + 10 + b); };
  static_assert(Smem::nbars == 2 * kStages + 12, "barrier count");

  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      tc::mbar_init(full_bar(s), 1);
      tc::mbar_init(empty_bar(s), 1);
    }
    tc::mbar_init(qfull_bar(), 1);
    tc::mbar_init(qempty_bar(), 1);
    for (int b = 0; b < 2; ++b) {
      tc::mbar_init(sfull_bar(b), 1);
      tc::mbar_init(sempty_bar(b), 4);
      tc::mbar_init(pfull_bar(b), 4);
      tc::mbar_init(ofull_bar(b), 1);
      tc::mbar_init(ofree_bar(b), 4);
    }
    *abort_flag = 0;
    tc::fence_mbar_init();
  }
  if (warp == 4 && lane == 0) {
    tc::prefetch_tmap(&kmap);
    tc::prefetch_tmap(&vmap);
    tc::prefetch_tmap(&qmap);
  }
  // zero the V stages (rows of a partial tile that no page fills must be finite) and both
  // probability buffers (their off-diagonal blocks stay zero for the whole kernel)
  for (int i = tid; i < kStages * kKBytes / 16; i += blockDim.x) {
    const int s = i / (kKBytes / 16), o = i % (kKBytes / 16);
    reinterpret_cast<uint4*>(smem + Smem::kv + s * kStageBytes + kKBytes)[o] = make_uint4(0, 0, 0, 0);
  }
  for (int i = tid; i < 2 * kPBytes / 16; i += blockDim.x)
    reinterpret_cast<uint4*>(smem + Smem::p)[i] = make_uint4(0, 0, 0, 0);
  tc::fence_proxy_async_smem();
  if (warp == 5) tc::tmem_alloc(tc::smem_u32(tmem_holder), kTmemCols);
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  const uint32_t tm_s = tmem, tm_o = tmem + 2 * kN;

  const int u_begin = a.cta_indptr[cta], u_end = a.cta_indptr[cta + 1];
  if (warp == 4) {
    // ======================================================================= TMA producer
    // The whole warp walks the units: lanes hold the page ids of the next 32 tiles (one per lane)
    // while lane 0 waits for ring slots and issues the copies.  The single Q buffer is refilled
    // for unit n once unit n-1's last S MMA is done; until then the unit's KV tiles keep
    // streaming and the Q slot is polled (it must be loaded before a ring slot holding one of
    // this unit's own tiles is waited for, since those slots are released only after Q arrives).
    int n_tile = 0, n_unit = 0;
    bool ok = true;
    bool q_pending = false;
    int q_pending_start = 0;
    auto issue_q = [&](int q_start) {
      tc::mbar_arrive_expect_tx(qfull_bar(), (uint32_t)(kD * 2 * kN));
      for (int rgn = 0; rgn < 2; ++rgn)
        tma_load_4d_nohint(sbase + Smem::q + rgn * kQRegion, &qmap, qfull_bar(), rgn * 64, 0, q_start, 0);
    };
    auto flush_q = [&]() -> bool {  // lane 0: block until Q can be issued
      if (!q_pending) return true;
      if (!tc::mbar_wait(qempty_bar(), (n_unit + 1) & 1, abort_flag, a.status)) return false;
      issue_q(q_pending_start);
      q_pending = false;
      return true;
    };
    for (int u = u_begin; u < u_end && ok; ++u) {
      const WUnit x = load_wunit(a, work, u);
      if (x.ntiles == 0) continue;
      const int* ids = a.kv_indices + a.kv_indptr[x.r] + x.page_begin;
      // tile j covers tokens t0 + 16 j .. +16: page (16 j) / P of the unit, slot (16 j) % P
      const int tiles_per_page = a.page_size / kTok;
      int pid = (lane < x.ntiles) ? __ldg(ids + lane * kTok / a.page_size) : 0;
      if (lane == 0) {
        if (n_unit == 0 || tc::mbar_try_wait(qempty_bar(), (n_unit + 1) & 1)) {
          issue_q(x.q_start);
        } else {
          q_pending = true;
          q_pending_start = x.q_start;
        }
      }
      for (int j0 = 0; j0 < x.ntiles && ok; j0 += 32) {
        const int jn = j0 + 32 + lane;
        const int pid_next = (jn < x.ntiles) ? __ldg(ids + jn * kTok / a.page_size) : 0;
        const int nj = min(32, x.ntiles - j0);
        for (int jj = 0; jj < nj; ++jj) {
          const int j = j0 + jj, t = n_tile + j, st = t % kStages;
          const int page = __shfl_sync(0xffffffffu, pid, jj);
          bool plain_wait = false;  // the slot wait without a pending Q copy: done by the whole warp
          if (lane == 0) {
            if (t >= kStages) {
              if (t - kStages >= n_tile) ok = flush_q();  // the slot holds a tile of this unit
              if (ok && q_pending) {
                const uint64_t t_start = tc::globaltimer_ns();  // poll the ring slot and the Q slot
                while (true) {
                  if (q_pending && tc::mbar_try_wait(qempty_bar(), (n_unit + 1) & 1)) {
                    issue_q(q_pending_start);
                    q_pending = false;
                  }
                  if (tc::mbar_try_wait(empty_bar(st), ((t / kStages) + 1) & 1)) break;
                  if (*abort_flag || tc::globaltimer_ns() - t_start > tc::kWaitLimitNs) {
                    *abort_flag = 1;
                    report(a.status, SKV_DEV_TIMEOUT);
                    ok = false;
                    break;
                  }
                }
              } else if (ok) {
                plain_wait = true;
              }
            }
          }
          ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
          if (__shfl_sync(0xffffffffu, plain_wait ? 1 : 0, 0)) {
            // no lane waits alone while the others stand at a convergence point
            ok = tc::mbar_wait(empty_bar(st), ((t / kStages) + 1) & 1, abort_flag, a.status);
            ok = __all_sync(0xffffffffu, ok);
          }
          if (lane == 0) {
            if (ok) {
              if ((unsigned)page >= (unsigned)a.num_pages) report(a.status, SKV_DEV_PAGE_OOB);
              const int slot0 = (j % tiles_per_page) * kTok;
              tc::mbar_arrive_expect_tx(full_bar(st), (uint32_t)kStageBytes);
              const uint32_t kdst = sbase + Smem::kv + st * kStageBytes;
              for (int rgn = 0; rgn < 2; ++rgn) {
                tma_load_4d_nohint(kdst + rgn * kRegion, &kmap, full_bar(st), rgn * 64, slot0, 0, page);
                tma_load_4d_nohint(kdst + kKBytes + rgn * kRegion, &vmap, full_bar(st), rgn * 64, slot0, 0, page);
              }
            }
          }
          ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
          if (!ok) break;
        }
        pid = pid_next;
      }
      if (lane == 0 && ok) ok = flush_q();  // this unit's Q goes out before the next unit's
      ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
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
      constexpr uint32_t idesc_s = tc::idesc_bf16_f32(128, kN, false, false);
      constexpr uint32_t idesc_o = tc::idesc_bf16_f32(128, 16, true, false);
      int n_tile = 0, n_unit = 0;
      bool ok = true;
      auto issue_pv = [&](int t, int j, uint32_t o_cols) -> bool {
        const int st = t % kStages, pb = t & 1;
        if (!tc::mbar_wait(pfull_bar(pb), (t >> 1) & 1, abort_flag, a.status)) return false;
        tc::tc_fence_after();
        const uint32_t vs = sbase + Smem::kv + st * kStageBytes + kKBytes;
        const uint32_t ps = sbase + Smem::p + pb * kPBytes;
#pragma unroll
        for (int pr = 0; pr < 4; ++pr) {
#pragma unroll
          for (int k = 0; k < 2; ++k) {
            const uint64_t ad = tc::sdesc_sw128(vs + (32 * pr + 16 * k) * 128, kRegion, 1024);
            const uint64_t bd = tc::sdesc_sw128(ps + pr * kPairBytes + k * 32, 16, 1024);
            tc::mma_bf16(o_cols + 16 * pr, ad, bd, idesc_o, (j > 0 || k > 0) ? 1u : 0u);
          }
        }
        tc::mma_commit(ofull_bar(t & 1));
        tc::mma_commit(empty_bar(st));
        return true;
      };
      for (int u = u_begin; u < u_end && ok; ++u) {
        const WUnit x = load_wunit(a, work, u);
        if (x.ntiles == 0) continue;
        const int ob = n_unit & 1;
        const uint32_t o_cols = tm_o + ob * kN;
        ok = tc::mbar_wait(qfull_bar(), n_unit & 1, abort_flag, a.status);
        // this unit's O^T buffer was last read by the finalize of unit n_unit - 2
        if (ok && n_unit >= 2) ok = tc::mbar_wait(ofree_bar(ob), ((n_unit >> 1) + 1) & 1, abort_flag, a.status);
        if (!ok) break;
        tc::tc_fence_after();
        const uint32_t qs = sbase + Smem::q;
        for (int j = 0; j < x.ntiles && ok; ++j) {
          const int t = n_tile + j, st = t % kStages, sb = t & 1;
          ok = tc::mbar_wait(full_bar(st), (t / kStages) & 1, abort_flag, a.status);
          if (ok && t >= 2) ok = tc::mbar_wait(sempty_bar(sb), ((t >> 1) + 1) & 1, abort_flag, a.status);
          if (!ok) break;
          tc::tc_fence_after();
          const uint32_t ks = sbase + Smem::kv + st * kStageBytes;
#pragma unroll
          for (int k = 0; k < kD / 16; ++k) {
            const uint64_t ad = tc::sdesc_sw128(ks + (k >> 2) * kRegion + (k & 3) * 32, 16, 1024);
            const uint64_t bd = tc::sdesc_sw128(qs + (k >> 2) * kQRegion + (k & 3) * 32, 16, 1024);
            tc::mma_bf16(tm_s + sb * kN, ad, bd, idesc_s, k > 0 ? 1u : 0u);
          }
          tc::mma_commit(sfull_bar(sb));
          if (j == x.ntiles - 1) tc::mma_commit(qempty_bar());  // Q free once the last S is done
          if (j >= 1) ok = issue_pv(t - 1, j - 1, o_cols);
        }
        if (ok) ok = issue_pv(n_tile + x.ntiles - 1, x.ntiles - 1, o_cols);
        n_tile += x.ntiles;
        ++n_unit;
      }
    }
  } else if (warp < 4) {
    // ======================================================================= softmax
    float* alpha_s = reinterpret_cast<float*>(smem + Smem::alpha);
    float* inv_s = reinterpret_cast<float*>(smem + Smem::inv);
    float* lse_s = reinterpret_cast<float*>(smem + Smem::lse);
    float* lsum_s = reinterpret_cast<float*>(smem + Smem::lsum);
    float* msum_s = reinterpret_cast<float*>(smem + Smem::msum);
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
    const int hh = lane >> 4;              // which head of the warp's pair
    const int head = 2 * warp + hh;        // this thread's (head, token) row
    const int tok = lane & 15;
    int n_tile = 0, n_unit = 0, pv_seen = 0;  // PV completions consumed, in order
    bool ok = true;
    // consume PV completions up to and including tile `upto` (in order, one phase each)
    auto consume_pv = [&](int upto) {
      for (; pv_seen <= upto; ++pv_seen)
        ok = tc::mbar_wait(ofull_bar(pv_seen & 1), (pv_seen >> 1) & 1, abort_flag, a.status) && ok;
      tc::tc_fence_after();
    };
    for (int u = u_begin; u < u_end && ok; ++u) {
      const WUnit x = load_wunit(a, work, u);
      const int rows = x.q_count * G;      // valid columns per KV head
      if (x.ntiles == 0) {
        for (int n = 0; n < kN; ++n) {
          if ((n & 7) >= rows) continue;
          int qi, hq;
          column_row<G>(n, qi, hq);
          if (x.part_row < 0) {
            store_out(reinterpret_cast<OutT*>(a.o) + ((int64_t)(x.q_start + qi) * a.hq + hq) * kD + tid, 0.f);
            if (a.lse != nullptr && tid == 0) a.lse[(int64_t)(x.q_start + qi) * a.hq + hq] = -INFINITY;
          } else {
            const int64_t prow = (int64_t)x.part_row + (int64_t)qi * x.part_stride;
            a.o_part[(prow * a.hq + hq) * kD + tid] = 0.f;
            if (tid == 0) a.lse_part[prow * a.hq + hq] = -INFINITY;
          }
        }
        continue;
      }
      const int ob = n_unit & 1;
      const uint32_t o_cols = tm_o + ob * kN;
      float m[8], l[8];
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        m[c] = -INFINITY;
        l[c] = 0.f;
      }
      bool failed = false;
      for (int j = 0; j < x.ntiles; ++j) {
        const int t = n_tile + j, sb = t & 1, st = t % kStages;
        ok = tc::mbar_wait(sfull_bar(sb), (t >> 1) & 1, abort_flag, a.status) && ok;
        tc::tc_fence_after();
        float s16[16];
        tc::tmem_ld_x16(tm_s + lane_base + sb * kN + 16 * warp, s16);
        tc::tmem_wait_ld();
        tc::tc_fence_before();
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(sempty_bar(sb));
        const bool valid = x.t0 + j * kTok + tok < x.t1;
        float s[8];
        bool raise = false;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const float v = hh ? s16[8 + c] : s16[c];
          s[c] = (valid && c < rows) ? v * a.scale_log2 : -INFINITY;
          raise |= s[c] > m[c] + kRaise;
        }
        // first tile of the unit, a score past the threshold anywhere, or a failed wait: slow path
        if (tc::bar_or(1, 128, raise || !ok || j == 0)) {
          if (!tc::bar_and(1, 128, ok)) {
            failed = true;
            break;
          }
          float al[8];
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            float mx = s[c];
#pragma unroll
            for (int o = 8; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
            const float mn = fmaxf(m[c], mx);
            al[c] = (mn == -INFINITY || m[c] == mn) ? 1.f : exp2f(m[c] - mn);
            l[c] *= al[c];
            m[c] = mn;
          }
          if (j > 0) {
            // rescale O^T in TMEM: publish alpha, wait for the last PV, each thread scales its lane
            if (tok == 0) {
#pragma unroll
              for (int c = 0; c < 8; ++c) alpha_s[head * 8 + c] = al[c];
            }
            tc::named_bar_sync(1, 128);
            consume_pv(t - 1);
#pragma unroll
            for (int q4 = 0; q4 < kN / 16; ++q4) {
              float ov[16];
              tc::tmem_ld_x16(o_cols + lane_base + 16 * q4, ov);
              tc::tmem_wait_ld();
#pragma unroll
              for (int i = 0; i < 16; ++i) ov[i] *= alpha_s[16 * q4 + i];
              tc::tmem_st_x16(o_cols + lane_base + 16 * q4, ov);
            }
            tc::tmem_wait_st();
            tc::tc_fence_before();
          }
        }
        // P(t) overwrites the buffer PV(t-2) read: consume that completion first
        if (t >= 2 && pv_seen <= t - 2) consume_pv(t - 2);
        // probabilities: pair `warp`, row hh*8 + c, column lane (= hh*16 + tok)
        uint8_t* pb = smem + Smem::p + (t & 1) * kPBytes + warp * kPairBytes;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const float p = (s[c] == -INFINITY) ? 0.f : exp2f(s[c] - m[c]);
          l[c] += p;
          *reinterpret_cast<__nv_bfloat16*>(pb + tc::sw128_offset(hh * 8 + c, lane)) = __float2bfloat16_rn(p);
        }
        if (!valid) {  // zero this row's V (both 64-column halves) before the PV MMA reads it
          uint8_t* vrow = smem + Smem::kv + st * kStageBytes + kKBytes + tid * 128;
#pragma unroll
          for (int rgn = 0; rgn < 2; ++rgn)
#pragma unroll
            for (int i = 0; i < 8; ++i)
              reinterpret_cast<uint4*>(vrow + rgn * kRegion)[i] = make_uint4(0, 0, 0, 0);
        }
        tc::fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(pfull_bar(t & 1));
      }
      if (failed) {
        ok = false;
        break;  // uniform: decided by bar_and
      }
      const int t_last = n_tile + x.ntiles - 1;
      n_tile += x.ntiles;
      ++n_unit;
      consume_pv(t_last);
      // per-column sums over the 16 token rows of each head
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        float v = l[c];
#pragma unroll
        for (int o = 8; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        if (tok == 0) {
          lsum_s[head * 8 + c] = v;
          msum_s[head * 8 + c] = m[c];
        }
      }
      if (!tc::bar_and(1, 128, ok)) {
        ok = false;
        break;
      }
      if (tid < kN) {
        const float lt = lsum_s[tid];
        inv_s[tid] = lt > 0.f ? 1.f / lt : 0.f;
        lse_s[tid] = lt > 0.f ? (msum_s[tid] + log2f(lt)) * kLn2 : -INFINITY;
      }
      float ov[kN];
#pragma unroll
      for (int q4 = 0; q4 < kN / 16; ++q4) {
        float v16[16];
        tc::tmem_ld_x16(o_cols + lane_base + 16 * q4, v16);
        tc::tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 16; ++i) ov[16 * q4 + i] = v16[i];
      }
      tc::tc_fence_before();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(ofree_bar(ob));
      tc::named_bar_sync(1, 128);
#pragma unroll
      for (int n = 0; n < kN; ++n) {
        if ((n & 7) >= rows) continue;
        int qi, hq;
        column_row<G>(n, qi, hq);
        if (x.part_row < 0) {
          store_out(reinterpret_cast<OutT*>(a.o) + ((int64_t)(x.q_start + qi) * a.hq + hq) * kD + tid, ov[n] * inv_s[n]);
        } else {
          const int64_t prow = (int64_t)x.part_row + (int64_t)qi * x.part_stride;
          a.o_part[(prow * a.hq + hq) * kD + tid] = ov[n] * inv_s[n];
        }
      }
      if (tid < kN && (tid & 7) < rows) {
        int qi, hq;
        column_row<G>(tid, qi, hq);
        if (x.part_row < 0) {
          if (a.lse != nullptr) a.lse[(int64_t)(x.q_start + qi) * a.hq + hq] = lse_s[tid];
        } else {
          a.lse_part[((int64_t)x.part_row + (int64_t)qi * x.part_stride) * a.hq + hq] = lse_s[tid];
        }
      }
      // alpha / inv / lse / lsum / msum are rewritten only after a later barrier of this group
    }
  }

  tc::tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, kTmemCols);
  }
}

// Tensor maps and arguments of a launch (host; gqa_tc_wide.cu): 0 on success, else a CUDA error code.
int prepare(const skv_paged_params& p, const int32_t* cta_indptr, int num_ctas, int q_tile, CUtensorMap* maps,
            WArgs* a);

}  // namespace wide
}  // namespace skv
