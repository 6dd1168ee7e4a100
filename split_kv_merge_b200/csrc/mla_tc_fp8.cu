// MLA latent decode on the tensor cores for an fp8 (e4m3) latent cache, in native fp8 MMAs.
//
// What it computes (FlashInfer PR #3309 page, MLA decode; the e4m3 cache of the same page):
// every head reads one latent row per token, a 512-d compressed KV (ckv) and a 64-d rope key
// (kpe), both stored as e4m3 with one per-tensor scale; s = sm_scale * kv_scale *
// (q_nope . ckv + q_pe . kpe), V = kv_scale * ckv.  seqlen_q is folded into the row dimension as
// in the bf16 kernel: rows n = qi * Hc + h of a unit, Hc = min(H, NR), F = q_tile tokens with
// F * Hc <= NR.  The (query tile, head group) units of a request -- q_len / F tiles times H / Hc
// groups -- run on a group of that many co-resident CTAs that stream the same KV slice together
// (as the 64-row bf16 kernel does), so the slice is read from HBM about once, not once per unit.
//
// B200 design: tcgen05.mma kind::f8f6f4 straight on the e4m3 cache tiles, so the cache is never
// converted and a 64-token tile is 36 KB of shared memory (four or three of them in flight).
//   * Both other operands are split into two e4m3 terms, hi = rn(x) and lo = rn(x - hi), stacked
//     as 2 NR columns of N: queries (bf16, 8 significant bits) after a power-of-two scaling that
//     puts the unit's largest |q| in [128, 256) -- exact for every |q| of at least 2^-9 of that
//     maximum, within 2^-17 of it below -- and the softmax weights, shifted up by 2^4 to
//     p' in [0, 2^8] (2^-8 relative precision from 2^-6 of the running maximum's weight up, 2^-14
//     absolute below).  The query scaling goes back into the softmax scale, the weight shift into
//     the LSE; S and O sum their hi and lo columns.
//   * S^T[64 tokens, 2 NR] = C . [Q_hi; Q_lo]^T, K = 32 per MMA: 16 ckv k-steps (128-byte
//     swizzled rows) + 2 rope k-steps (64-byte swizzled rows); M = 64, so TMEM rows sit in lanes
//     0-15 of each warp quarter.  The k-steps are split over two issuers into two partial
//     accumulators that the softmax adds.
//   * O^T[512, 2 NR] += V^T . [P_hi; P_lo]^T in four M = 128 blocks (V read MN-major from the same
//     tile), one block per issuer.
//   * Online softmax with a lazily raised maximum (only when a score passes it by more than 2^4),
//     O^T rescaled in TMEM on a raise; tokens past the end of the unit get s = -inf by selection
//     and their V rows are zeroed in the tile before the PV that reads them.
// Roles: warps 0-3 softmax / query split / epilogue, warp 4 TMA, warps 5-8 MMA issue (one per SM
// sub-partition; each polls for whichever of PV(t) and QK(t') is ready).  All waits are bounded.
#include <cudaTypedefs.h>

#include <algorithm>
#include <mutex>

#include "tc_ptx.cuh"

namespace skv {

namespace {

constexpr int kTile = 64;                        // tokens per tile
constexpr int kCRegion = kTile * 128;            // 128 ckv dims (bytes) x 64 tokens: 8 KB
constexpr int kKRegion = kTile * 64;             // 64 rope dims x 64 tokens: 4 KB (64-byte rows)
constexpr int kTileBytes = 4 * kCRegion + kKRegion;
constexpr int kBlocks = 4;
constexpr int kIssuers = 4;
constexpr int kThreads = (5 + kIssuers) * 32;
// The running maximum is raised only when a score passes it by more than 2^4 (log2 units), and
// every weight is formed as p' = 2^(s - m + 4) <= 2^8 (e4m3 holds up to 448): the shift moves the
// small weights of a row up into the range where the hi + lo split is relative (2^-8 from
// p' = 2^-2 up, 2^-10 absolute below -- 2^-14 of the unshifted weight).  O / l is unchanged by
// the shift; the LSE subtracts it.
constexpr float kRaise = 4.f;
constexpr float kPShift = 4.f;

template <int NR>
struct Cfg8 {
  static constexpr int kQParts = 2;                     // QK partial accumulators (issuers 0, 1)
  static constexpr int kStages = NR == 16 ? 4 : 3;     // tiles in flight
  static constexpr int kQStage = NR * 128;             // one 64-column bf16 region of the query copy
  static constexpr int kQOps = 2 * NR * 128;           // one 128-dim region of [Q_hi; Q_lo] (e4m3)
  static constexpr int kPBytes = kTile * 128;          // P^T MN-major: token rows of [P_hi | P_lo] bytes
  static constexpr int tiles = 0;
  static constexpr int qstage = tiles + kStages * kTileBytes;
  static constexpr int qops = qstage + 9 * kQStage;
  static constexpr int p = qops + 5 * kQOps;
  static constexpr int kPBufs = 3;                      // P(t) reuses the buffer of PV(t - 3)
  static constexpr int red = p + kPBufs * kPBytes;      // [4][NR] float
  static constexpr int alpha = red + 4 * NR * 4;
  static constexpr int inv = alpha + NR * 4;
  static constexpr int lse = inv + NR * 4;
  static constexpr int mrow = lse + NR * 4;             // [NR] running maxima
  static constexpr int qmax = mrow + NR * 4;            // [4] float
  static constexpr int bars = qmax + 16;
  static constexpr int nbars = 2 * kStages + 14;
  static constexpr int misc = bars + nbars * 8;
  static constexpr int total = misc + 16;
  static constexpr int s_cols = 2 * kQParts * 2 * NR;  // 2 buffers x parts x [hi | lo]
  static constexpr int tmem_cols = 512;                 // S + O^T (4 blocks x 2 NR) <= 512
  static_assert(s_cols + 4 * 2 * NR <= 512, "TMEM");
};

struct M8Args {
  const int32_t* kv_indptr;
  const int32_t* kv_indices;
  const int32_t* last;
  const int32_t* cta_indptr;  // per KV slice
  int num_pages, page_size, heads, hc, hg, q_tile;
  int group;                  // CTAs per KV slice: (q_len / q_tile) query tiles x hg head groups
  float scale_log2;                             // sm_scale * kv_scale * log2(e)
  float kv_scale;
  void* o;
  float* lse;
  float* o_part;
  float* lse_part;
  int32_t* status;
};

struct MUnit8 {
  int r, q_start, q_count, page_begin, page_end, part_row, part_stride;
  int t0, t1, ntiles;
};

// work item u as seen by the CTA of query tile qt of its group (the plan holds tile 0's item)
__device__ __forceinline__ MUnit8 load_unit8(const M8Args& a, const WorkItem* work, int u, int qt) {
  MUnit8 x;
  const WorkItem w = work[u];
  x.r = w.r;
  x.q_start = w.q_start + qt * a.q_tile;
  x.q_count = w.q_count;
  x.page_begin = w.page_begin;
  x.page_end = w.page_end;
  x.part_row = w.part_row < 0 ? w.part_row : w.part_row + qt * a.q_tile * w.part_stride;
  x.part_stride = w.part_stride;
  const int L = request_len(a.kv_indptr, a.last, w.r, a.page_size);
  x.t0 = w.page_begin * a.page_size;
  x.t1 = min(w.page_end * a.page_size, L);
  x.ntiles = x.t1 > x.t0 ? (x.t1 - x.t0 + kTile - 1) / kTile : 0;
  return x;
}

// shared-memory matrix descriptor (sm_100): layout 2 = 128-byte swizzle, 4 = 64-byte swizzle
__device__ __forceinline__ uint64_t sdesc(uint32_t saddr, uint32_t lbo, uint32_t sbo, uint32_t layout) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
  d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
  d |= (uint64_t)1 << 46;
  d |= (uint64_t)layout << 61;
  return d;
}
__device__ __forceinline__ uint64_t sw128(uint32_t saddr) { return sdesc(saddr, 16, 1024, 2); }

// D[tmem] (+)= A . B, kind::f8f6f4 (the e4m3 formats come from the instruction descriptor)
__device__ __forceinline__ void mma_f8(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a), "l"(b), "r"(idesc), "r"(acc)
      : "memory");
}
// instruction descriptor: e4m3 A and B (format code 0), f32 D
__host__ __device__ constexpr uint32_t idesc_e4m3(int M, int N, bool a_mn) {
  return (1u << 4) | ((a_mn ? 1u : 0u) << 15) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// two floats -> two e4m3 bytes (round to nearest even, saturating), low byte = a
__device__ __forceinline__ uint32_t e4m3x2(float a, float b) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(b), "f"(a));
  return r;
}
// two e4m3 bytes (low byte first) -> the two floats (exact)
__device__ __forceinline__ float2 e4m3x2_val(uint32_t two) {
  uint32_t h;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h) : "h"((uint16_t)two));
  return __half22float2(*reinterpret_cast<__half2*>(&h));
}
// [hi | lo] e4m3 split of two floats: hi = rn(x), lo = rn(x - hi), as two packed byte pairs
__device__ __forceinline__ void split2(float x0, float x1, uint32_t& hi, uint32_t& lo) {
  hi = e4m3x2(x0, x1);
  const float2 hv = e4m3x2_val(hi);
  lo = e4m3x2(x0 - hv.x, x1 - hv.y);
}
__device__ __forceinline__ float ex2(float x) {
  float r;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
  return r;
}

__device__ __forceinline__ float redux_max(float v) {
  float r;
  asm volatile("redux.sync.max.f32 %0, %1, 0xffffffff;" : "=f"(r) : "f"(v));
  return r;
}

template <int NR, typename OutT>
__global__ void __launch_bounds__(kThreads, 1)
mla_tc_fp8_kernel(const __grid_constant__ CUtensorMap ckv_map, const __grid_constant__ CUtensorMap kpe_map,
                  const __grid_constant__ CUtensorMap qn_map, const __grid_constant__ CUtensorMap qp_map, M8Args a,
                  const WorkItem* __restrict__ work) {
  using C = Cfg8<NR>;
  constexpr int NS = C::kStages, NQ = C::kQParts;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = tc::smem_u32(smem);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  tc::grid_launch_dependents();  // the merge pass may be scheduled; it waits for this grid

  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + C::misc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::misc + 4);
  const uint32_t bar0 = sbase + C::bars;
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (NS + s); };
  const uint32_t bar1 = bar0 + 8u * (2 * NS);
  auto qfull_bar = [&]() { return bar1; };
  auto qready_bar = [&]() { return bar1 + 8u; };
  auto sfull_bar = [&](int b) { return bar1 + 8u * (2 + b); };
  auto sempty_bar = [&](int b) { return bar1 + 8u * (4 + b); };
  auto pfull_bar = [&](int b) { return bar1 + 8u * (6 + b); };   // one per P buffer
  auto ofull_bar = [&](int b) { return bar1 + 8u * (9 + b); };   // four: PV(t) on t & 3
  auto ofree_bar = [&]() { return bar1 + 8u * 13; };
  static_assert(C::total + 1024 <= 232448, "fits the 227 KB opt-in shared memory");

  if (tid == 0) {
    for (int s = 0; s < NS; ++s) {
      tc::mbar_init(full_bar(s), 1);
      tc::mbar_init(empty_bar(s), kIssuers);
    }
    tc::mbar_init(qfull_bar(), 1);
    tc::mbar_init(qready_bar(), 4);
    for (int b = 0; b < 2; ++b) {
      tc::mbar_init(sfull_bar(b), NQ);
      tc::mbar_init(sempty_bar(b), 4);
    }
    for (int b = 0; b < C::kPBufs; ++b) tc::mbar_init(pfull_bar(b), 4);
    for (int b = 0; b < 4; ++b) tc::mbar_init(ofull_bar(b), kIssuers);
    tc::mbar_init(ofree_bar(), 4);
    *abort_flag = 0;
    tc::fence_mbar_init();
  }
  if (warp == 4 && lane == 0) {
    tc::prefetch_tmap(&ckv_map);
    tc::prefetch_tmap(&kpe_map);
    tc::prefetch_tmap(&qn_map);
    tc::prefetch_tmap(&qp_map);
  }
  if (warp == 5) tc::tmem_alloc(tc::smem_u32(tmem_holder), C::tmem_cols);
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  const uint32_t tm_s = tmem, tm_o = tmem + C::s_cols;

  // CTA c runs KV slice c / group for one (query tile, head group) unit, c % group: the group's
  // CTAs stream the same pages at the same time, so each page comes from HBM about once
  const int slice = (int)blockIdx.x / a.group, gsel = (int)blockIdx.x % a.group;
  const int my_qt = gsel / a.hg, my_hg = gsel % a.hg;
  const int u_begin = a.cta_indptr[slice], u_end = a.cta_indptr[slice + 1];
  const int P = a.page_size;
  const int box_rows = min(P, kTile);

  if (warp == 4) {
    // ======================================================================= TMA producer
    int g = 0, n_unit = 0;
    bool ok = true;
    for (int u = u_begin; u < u_end && ok; ++u) {
      const MUnit8 x = load_unit8(a, work, u, my_qt);
      if (x.ntiles == 0) continue;
      const int* ids = a.kv_indices + a.kv_indptr[x.r] + x.page_begin;
      const int npages = x.page_end - x.page_begin;
      for (int hgi = my_hg; hgi == my_hg && ok; ++hgi) {
        if (lane == 0) {  // queries of this unit once the previous unit's copy has been split
          if (n_unit >= 1) ok = tc::mbar_wait_sleep(qready_bar(), (n_unit - 1) & 1, abort_flag, a.status);
          if (ok) {
            const int rows = a.hc * a.q_tile;
            tc::mbar_arrive_expect_tx(qfull_bar(), (uint32_t)(9 * rows * 128));
            for (int rg = 0; rg < 8; ++rg)
              tc::tma_load_3d(sbase + C::qstage + rg * C::kQStage, &qn_map, qfull_bar(), rg * 64, hgi * a.hc,
                              x.q_start);
            tc::tma_load_3d(sbase + C::qstage + 8 * C::kQStage, &qp_map, qfull_bar(), 0, hgi * a.hc, x.q_start);
          }
        }
        ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
        int win = -1000000, pid = 0;  // lanes hold the ids of pages [win, win + 32) of the unit
        for (int t = 0; t < x.ntiles && ok; ++t, ++g) {
          const int pi0 = (t * kTile) / P;
          const int npg = P >= kTile ? 1 : min(kTile / P, npages - pi0);
          const int slot0 = P >= kTile ? (t * kTile) % P : 0;
          if (pi0 < win || pi0 + npg > win + 32) {
            win = pi0;
            pid = (win + lane < npages) ? __ldg(ids + win + lane) : 0;
          }
          const int st = g % NS;
          // the whole warp waits for the slot (no lane waits alone while the others stand at a
          // convergence point); lane 0 posts the expected bytes
          if (g >= NS) ok = tc::mbar_wait_sleep(empty_bar(st), ((g / NS) + 1) & 1, abort_flag, a.status);
          ok = __all_sync(0xffffffffu, ok);
          if (ok && lane == 0) tc::mbar_arrive_expect_tx(full_bar(st), (uint32_t)(npg * box_rows * (4 * 128 + 64)));
          if (!ok) break;
          const uint32_t tb = sbase + C::tiles + st * kTileBytes;
          for (int i = 0; i < npg; ++i) {  // five boxes per page, issued by five lanes at once
            const int page = __shfl_sync(0xffffffffu, pid, pi0 + i - win);
            if (lane == 0 && (unsigned)page >= (unsigned)a.num_pages) report(a.status, SKV_DEV_PAGE_OOB);
            if (lane < 4)
              tc::tma_load_3d(tb + lane * kCRegion + i * box_rows * 128, &ckv_map, full_bar(st), lane * 128, slot0,
                              page);
            else if (lane == 4)
              tc::tma_load_3d(tb + 4 * kCRegion + i * box_rows * 64, &kpe_map, full_bar(st), 0, slot0, page);
          }
        }
        ++n_unit;
      }
    }
    if (!ok && lane == 0) {  // drain issued copies (bounded) before the CTA can exit
      for (int q = max(0, g - NS); q < g; ++q) {
        const uint64_t t_start = tc::globaltimer_ns();
        while (!tc::mbar_try_wait(full_bar(q % NS), (q / NS) & 1) && tc::globaltimer_ns() - t_start < 50000000ull) {
        }
      }
      if (n_unit >= 1) {
        const uint64_t t_start = tc::globaltimer_ns();
        while (!tc::mbar_try_wait(qfull_bar(), (n_unit - 1) & 1) && tc::globaltimer_ns() - t_start < 50000000ull) {
        }
      }
    }
  } else if (warp >= 5) {
    // ======================================================================= MMA issuers
    // Issuer w: PV block w (two k-steps of 32 tokens) and, for w < NQ, QK part w (its share of the
    // 16 ckv k-steps; parts 0 and 1 also take rope k-steps 0 and 1).  PV first when both are ready.
    if (lane == 0) {
      const int w = warp - 5;
      constexpr uint32_t idesc_s = idesc_e4m3(64, 2 * NR, false);
      constexpr uint32_t idesc_o = idesc_e4m3(128, 2 * NR, true) | (1u << 16);  // P^T MN-major too
      constexpr int kRegionsPerPart = 4 / NQ;
      int g = 0, n_unit = 0, n_tile = 0;
      bool ok = true;
      const uint32_t qo = sbase + C::qops;
      for (int u = u_begin; u < u_end && ok; ++u) {
        const MUnit8 x = load_unit8(a, work, u, my_qt);
        if (x.ntiles == 0) continue;
        for (int hgi = my_hg; hgi == my_hg && ok; ++hgi) {
          const int T = x.ntiles;
          ok = tc::mbar_wait_sleep(qready_bar(), n_unit & 1, abort_flag, a.status);
          if (ok) tc::tc_fence_after();
          int qk = w < NQ ? 0 : T, pv = 0;  // issuers without a QK part only run PV
          tc::PollClock clk;
          while (ok && pv < T) {
            bool did = false;
            {  // ---- PV(pv), block w: needs P(pv), which implies every QK part of the tile is done
              const int tp = n_tile + pv, pb = tp % C::kPBufs, gg = g + pv, st = gg % NS;
              if (pv < T && tc::mbar_test_wait(pfull_bar(pb), (tp / C::kPBufs) & 1) &&
                  (pv > 0 || n_unit == 0 || tc::mbar_test_wait(ofree_bar(), (n_unit + 1) & 1))) {
                tc::tc_fence_after();
                const uint32_t vs = sbase + C::tiles + st * kTileBytes + w * kCRegion;
                const uint32_t ps = sbase + C::p + pb * C::kPBytes;
#pragma unroll
                for (int k = 0; k < 2; ++k)
                  mma_f8(tm_o + w * 2 * NR, sdesc(vs + k * 4096, 8192, 1024, 2), sdesc(ps + k * 4096, 8192, 1024, 2),
                         idesc_o, (pv > 0 || k > 0) ? 1u : 0u);
                tc::mma_commit(empty_bar(st));
                tc::mma_commit(ofull_bar(tp & 3));
                ++pv;
                did = true;
              }
            }
            if (!did && qk < T) {  // ---- QK(qk), part w
              const int tt = n_tile + qk, sb = tt & 1, gg = g + qk, st = gg % NS;
              if ((tt < 2 || tc::mbar_test_wait(sempty_bar(sb), ((tt >> 1) + 1) & 1)) &&
                  tc::mbar_test_wait(full_bar(st), (gg / NS) & 1)) {
                tc::tc_fence_after();
                const uint32_t tb = sbase + C::tiles + st * kTileBytes;
                const uint32_t d = tm_s + (sb * NQ + w) * 2 * NR;
#pragma unroll
                for (int rr = 0; rr < kRegionsPerPart; ++rr) {
                  const int r = w * kRegionsPerPart + rr;
#pragma unroll
                  for (int k = 0; k < 4; ++k)
                    mma_f8(d, sw128(tb + r * kCRegion + k * 32), sw128(qo + r * C::kQOps + k * 32), idesc_s,
                           (rr > 0 || k > 0) ? 1u : 0u);
                }
                if (w < 2)  // rope k-step w (64-byte swizzled rows)
                  mma_f8(d, sdesc(tb + 4 * kCRegion + w * 32, 16, 512, 4), sw128(qo + 4 * C::kQOps + w * 32),
                         idesc_s, 1u);
                tc::mma_commit(sfull_bar(sb));
                ++qk;
                did = true;
              }
            }
            ok = clk.step(did, abort_flag, a.status);
          }
          g += T;
          n_tile += T;
          ++n_unit;
        }
      }
    }
  } else {
    // ======================================================================= softmax / epilogue
    float* red = reinterpret_cast<float*>(smem + C::red);
    float* alpha_s = reinterpret_cast<float*>(smem + C::alpha);
    float* inv_s = reinterpret_cast<float*>(smem + C::inv);
    float* lse_s = reinterpret_cast<float*>(smem + C::lse);
    float* m_s = reinterpret_cast<float*>(smem + C::mrow);  // the same in every thread
    float* qmax_s = reinterpret_cast<float*>(smem + C::qmax);
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
    const bool srow = lane < 16;              // this lane holds an S^T row (M = 64 layout)
    const int tok_in_tile = 16 * warp + (lane & 15);
    int g = 0, n_unit = 0, n_tile = 0, pv_seen = 0;
    bool ok = true;
    auto consume_pv = [&](int upto) {
      for (; pv_seen <= upto; ++pv_seen)
        ok = tc::mbar_wait_sleep(ofull_bar(pv_seen & 3), (pv_seen >> 2) & 1, abort_flag, a.status) && ok;
      tc::tc_fence_after();
    };
    for (int u = u_begin; u < u_end && ok; ++u) {
      const MUnit8 x = load_unit8(a, work, u, my_qt);
      const int rows = x.q_count * a.hc;
      for (int hgi = my_hg; hgi == my_hg && ok; ++hgi) {
        const int h0 = hgi * a.hc;
        if (x.ntiles == 0) {  // no tokens: O = 0, LSE = -inf
          for (int n = 0; n < rows; ++n) {
            const int qi = n / a.hc, h = h0 + n % a.hc;
            for (int d = tid; d < 512; d += 128) {
              if (x.part_row < 0)
                store_out(reinterpret_cast<OutT*>(a.o) + ((int64_t)(x.q_start + qi) * a.heads + h) * 512 + d, 0.f);
              else
                a.o_part[(((int64_t)x.part_row + (int64_t)qi * x.part_stride) * a.heads + h) * 512 + d] = 0.f;
            }
            if (tid == 0) {
              if (x.part_row < 0) {
                if (a.lse != nullptr) a.lse[(int64_t)(x.q_start + qi) * a.heads + h] = -INFINITY;
              } else {
                a.lse_part[((int64_t)x.part_row + (int64_t)qi * x.part_stride) * a.heads + h] = -INFINITY;
              }
            }
          }
          continue;
        }
        // ---- queries: bf16 copy -> [Q_hi; Q_lo] e4m3 terms of q * 2^e, 2^e putting max |q| in [128, 256)
        ok = tc::mbar_wait_sleep(qfull_bar(), n_unit & 1, abort_flag, a.status) && ok;
        const int qrows = a.hc * a.q_tile;     // rows the query copy filled
        float qm = 0.f;
        for (int ci = tid; ci < 9 * NR * 8; ci += 128) {
          if ((ci % (NR * 8)) / 8 >= qrows) continue;
          const uint4 v = *reinterpret_cast<const uint4*>(smem + C::qstage + ci * 16);
          const uint32_t wv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
          for (int i = 0; i < 4; ++i)
            qm = fmaxf(qm, fmaxf(fabsf(__uint_as_float(wv[i] << 16)), fabsf(__uint_as_float(wv[i] & 0xffff0000u))));
        }
        qm = warp_max(qm);
        if (lane == 0) qmax_s[warp] = qm;
        if (tid < NR) m_s[tid] = -INFINITY;
        tc::named_bar_sync(1, 128);
        qm = fmaxf(fmaxf(qmax_s[0], qmax_s[1]), fmaxf(qmax_s[2], qmax_s[3]));
        const int e = (qm > 0.f && qm < INFINITY) ? 7 - ilogbf(qm) : 0;
        const float qmul = ldexpf(1.f, e);
        // staging chunk ci: region rg (64 dims), row n, 16-byte chunk c (8 dims); it becomes 8
        // bytes of Q_hi (row n) and of Q_lo (row NR + n); rows past the copy are zeros
        for (int ci = tid; ci < 9 * NR * 8; ci += 128) {
          const int rg = ci / (NR * 8), n = (ci % (NR * 8)) / 8, c = ci % 8;
          uint32_t hi[2] = {0u, 0u}, lo[2] = {0u, 0u};
          if (n < qrows) {
            const int cs = (c ^ (n & 7)) & 7;  // the copy is 128-byte swizzled
            const uint4 v = *reinterpret_cast<const uint4*>(smem + C::qstage + rg * C::kQStage + n * 128 + cs * 16);
            const uint32_t wv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const float x0 = __uint_as_float(wv[i] << 16) * qmul;
              const float x1 = __uint_as_float(wv[i] & 0xffff0000u) * qmul;
              uint32_t h2, l2;
              split2(x0, x1, h2, l2);
              hi[i >> 1] |= h2 << (16 * (i & 1));
              lo[i >> 1] |= l2 << (16 * (i & 1));
            }
          }
          // dims d0 .. d0 + 7: region d0 / 128 (region 4 = rope), byte b0 within the 128-byte row
          const int d0 = rg < 8 ? rg * 64 + c * 8 : 512 + c * 8;
          const int r = d0 >> 7, b0 = d0 & 127;
          const int rh = n, rl = NR + n;
          uint8_t* base = smem + C::qops + r * C::kQOps;
          *reinterpret_cast<uint2*>(base + rh * 128 + ((((b0 >> 4) ^ (rh & 7)) & 7) << 4) + (b0 & 15)) =
              make_uint2(hi[0], hi[1]);
          *reinterpret_cast<uint2*>(base + rl * 128 + ((((b0 >> 4) ^ (rl & 7)) & 7) << 4) + (b0 & 15)) =
              make_uint2(lo[0], lo[1]);
        }
        tc::fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(qready_bar());
        const float sl2 = ldexpf(a.scale_log2, -e);

        const int T = x.ntiles;
        // P phase: lanes 0-15 take rows [0, NR/2) of their token, lanes 16-31 rows [NR/2, NR) of the
        // token of lane - 16; l[j] is the partial sum of row half * NR/2 + j
        constexpr int NH = NR / 2;
        const int half = lane >> 4;
        float l[NH];
#pragma unroll
        for (int j = 0; j < NH; ++j) l[j] = 0.f;
        bool failed = false;
        for (int t = 0; t < T; ++t) {
          const int tt = n_tile + t, sb = tt & 1, gg = g + t, st = gg % NS;
          ok = tc::mbar_wait_sleep(sfull_bar(sb), (tt >> 1) & 1, abort_flag, a.status) && ok;
          tc::tc_fence_after();
          float s[NR];
          constexpr int kGrp = NR == 16 ? 2 : 1;  // partial accumulators loaded per TMEM wait (one wait at 16 rows)
#pragma unroll
          for (int pp = 0; pp < NQ; pp += kGrp) {  // partial accumulators, hi + lo columns
            float v[kGrp][2 * NR];
#pragma unroll
            for (int q = 0; q < kGrp; ++q)
#pragma unroll
              for (int c = 0; c < 2 * NR; c += 16) {
                float v16[16];
                tc::tmem_ld_x16(tm_s + lane_base + (sb * NQ + pp + q) * 2 * NR + c, v16);
#pragma unroll
                for (int i = 0; i < 16; ++i) v[q][c + i] = v16[i];
              }
            tc::tmem_wait_ld();  // registers of a TMEM load are read only after the wait
#pragma unroll
            for (int q = 0; q < kGrp; ++q)
#pragma unroll
              for (int n = 0; n < NR; ++n)
                s[n] = (pp == 0 && q == 0) ? v[q][n] + v[q][NR + n] : s[n] + (v[q][n] + v[q][NR + n]);
          }
          tc::tc_fence_before();
          __syncwarp();
          if (lane == 0) tc::mbar_arrive(sempty_bar(sb));
          const bool valid = srow && x.t0 + t * kTile + tok_in_tile < x.t1;
          bool raise = false;
#pragma unroll
          for (int n = 0; n < NR; ++n) {
            s[n] = (valid && n < rows) ? s[n] * sl2 : -INFINITY;
            raise |= s[n] > m_s[n] + kRaise;
          }
          if (tc::bar_or(1, 128, raise || !ok || t == 0)) {
            if (!tc::bar_and(1, 128, ok)) {
              failed = true;
              break;
            }
#pragma unroll
            for (int n = 0; n < NR; ++n) {  // column max over the warp's 16 token lanes (others -inf)
              const float v = redux_max(s[n]);
              if (lane == 0) red[warp * NR + n] = v;
            }
            tc::named_bar_sync(1, 128);
            if (tid < NR) {  // one thread per row: new maximum and the factor for l and O
              const int n = tid;
              const float mx = fmaxf(fmaxf(red[n], red[NR + n]), fmaxf(red[2 * NR + n], red[3 * NR + n]));
              const float mo = m_s[n], mn = fmaxf(mo, mx);
              alpha_s[n] = (mn == -INFINITY || mo == mn) ? 1.f : exp2f(mo - mn);
              m_s[n] = mn;
            }
            tc::named_bar_sync(1, 128);
#pragma unroll
            for (int j = 0; j < NH; ++j) l[j] *= alpha_s[half * NH + j];
            if (t > 0) {  // rescale O^T (hi and lo columns) in TMEM; thread tid owns lane tid of each block
              consume_pv(tt - 1);
#pragma unroll 1
              for (int c = 0; c < 2 * NR; c += 16) {
                float al[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) al[i] = alpha_s[(c + i) % NR];
#pragma unroll 1
                for (int b = 0; b < kBlocks; ++b) {
                  float ov[16];
                  tc::tmem_ld_x16(tm_o + lane_base + b * 2 * NR + c, ov);
                  tc::tmem_wait_ld();
#pragma unroll
                  for (int i = 0; i < 16; ++i) ov[i] *= al[i];
                  tc::tmem_st_x16(tm_o + lane_base + b * 2 * NR + c, ov);
                }
              }
              tc::tmem_wait_st();
              tc::tc_fence_before();
            }
            tc::named_bar_sync(1, 128);  // red / alpha_s reads done before any later rewrite
          }
          if (srow && !valid) {  // zero this token's V row in the tile (the copy landed before QK)
            ok = tc::mbar_wait_sleep(full_bar(st), (gg / NS) & 1, abort_flag, a.status) && ok;
            uint8_t* row = smem + C::tiles + st * kTileBytes + tok_in_tile * 128;
#pragma unroll
            for (int b = 0; b < kBlocks; ++b)
#pragma unroll
              for (int i = 0; i < 8; ++i) reinterpret_cast<uint4*>(row + b * kCRegion)[i] = make_uint4(0, 0, 0, 0);
          }
          if (tt >= C::kPBufs && pv_seen <= tt - C::kPBufs) consume_pv(tt - C::kPBufs);  // P(t)'s buffer was PV's
          {
            float sv[NH], mloc[NH];
#pragma unroll
            for (int jj = 0; jj < NH; ++jj) {  // upper rows move from lane l to lane l + 16
              const float up = __shfl_sync(0xffffffffu, s[NH + jj], lane & 15);
              sv[jj] = half ? up : s[jj];
              mloc[jj] = m_s[half * NH + jj];
            }
            // token row of P^T (MN-major, 128-byte swizzle): bytes [0, NR) = P_hi, [NR, 2 NR) = P_lo
            uint8_t* prow = smem + C::p + (tt % C::kPBufs) * C::kPBytes + tok_in_tile * 128;
            uint32_t hw[NH / 4], lw[NH / 4];
#pragma unroll
            for (int jj = 0; jj < NH; jj += 2) {
              // masked scores give 0 (rows past the unit's rows have no finite maximum)
              const float p0 = sv[jj] == -INFINITY ? 0.f : ex2(sv[jj] - mloc[jj] + kPShift);
              const float p1 = sv[jj + 1] == -INFINITY ? 0.f : ex2(sv[jj + 1] - mloc[jj + 1] + kPShift);
              l[jj] += p0;
              l[jj + 1] += p1;
              uint32_t h2, l2;
              split2(p0, p1, h2, l2);
              if ((jj & 2) == 0) {
                hw[jj >> 2] = h2;
                lw[jj >> 2] = l2;
              } else {
                hw[jj >> 2] |= h2 << 16;
                lw[jj >> 2] |= l2 << 16;
              }
            }
            const int x7 = tok_in_tile & 7;
            const int bh = half * NH, bl = NR + half * NH;  // first byte of this lane's hi / lo rows
            if constexpr (NH == 8) {
              *reinterpret_cast<uint2*>(prow + ((((bh >> 4) ^ x7) & 7) << 4) + (bh & 15)) = make_uint2(hw[0], hw[1]);
              *reinterpret_cast<uint2*>(prow + ((((bl >> 4) ^ x7) & 7) << 4) + (bl & 15)) = make_uint2(lw[0], lw[1]);
            } else {
              *reinterpret_cast<uint4*>(prow + ((((bh >> 4) ^ x7) & 7) << 4)) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
              *reinterpret_cast<uint4*>(prow + ((((bl >> 4) ^ x7) & 7) << 4)) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
            }
          }
          tc::fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) tc::mbar_arrive(pfull_bar(tt % C::kPBufs));
        }
        if (failed) {
          ok = false;
          break;
        }
        g += T;
        n_tile += T;
        ++n_unit;
        consume_pv(n_tile - 1);
        // row sums over the 64 tokens: each 16-lane half of a warp holds half of the rows
#pragma unroll
        for (int j = 0; j < NH; ++j) {
          float v = l[j];
#pragma unroll
          for (int o = 8; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
          if ((lane & 15) == 0) red[warp * NR + half * NH + j] = v;
        }
        if (!tc::bar_and(1, 128, ok)) {
          ok = false;
          break;
        }
        if (tid < NR) {
          const int n = tid;
          const float lt = red[n] + red[NR + n] + red[2 * NR + n] + red[3 * NR + n];
          inv_s[n] = lt > 0.f ? a.kv_scale / lt : 0.f;
          lse_s[n] = lt > 0.f ? (m_s[n] - kPShift + log2f(lt)) * kLn2 : -INFINITY;
        }
        tc::named_bar_sync(1, 128);
        // O^T block by block: thread tid holds head dim b * 128 + tid of every row (hi + lo)
#pragma unroll 1
        for (int b = 0; b < kBlocks; ++b) {
          float ov[NR];
#pragma unroll
          for (int hl = 0; hl < 2; ++hl) {
            float vv[NR];
#pragma unroll
            for (int c = 0; c < NR; c += 16) {
              float v16[16];
              tc::tmem_ld_x16(tm_o + lane_base + b * 2 * NR + hl * NR + c, v16);
#pragma unroll
              for (int i = 0; i < 16; ++i) vv[c + i] = v16[i];
            }
            tc::tmem_wait_ld();
#pragma unroll
            for (int n = 0; n < NR; ++n) ov[n] = hl == 0 ? vv[n] : ov[n] + vv[n];
          }
#pragma unroll
          for (int n = 0; n < NR; ++n) {
            if (n >= rows) break;
            const int qi = n / a.hc, h = h0 + n % a.hc;
            const float v = ov[n] * inv_s[n];
            if (x.part_row < 0)
              store_out(reinterpret_cast<OutT*>(a.o) + ((int64_t)(x.q_start + qi) * a.heads + h) * 512 + b * 128 + tid,
                        v);
            else
              a.o_part[(((int64_t)x.part_row + (int64_t)qi * x.part_stride) * a.heads + h) * 512 + b * 128 + tid] = v;
          }
        }
        tc::tc_fence_before();
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(ofree_bar());
        if (tid < rows) {
          const int qi = tid / a.hc, h = h0 + tid % a.hc;
          if (x.part_row < 0) {
            if (a.lse != nullptr) a.lse[(int64_t)(x.q_start + qi) * a.heads + h] = lse_s[tid];
          } else {
            a.lse_part[((int64_t)x.part_row + (int64_t)qi * x.part_stride) * a.heads + h] = lse_s[tid];
          }
        }
        tc::named_bar_sync(1, 128);  // inv_s / lse_s / red reads done before the next unit
      }
    }
  }

  tc::tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, Cfg8<NR>::tmem_cols);
  }
}

// ------------------------------------------------------------------------------ host side
PFN_cuTensorMapEncodeTiled_v12000 encode_fn_m8() {
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

bool make_map8(CUtensorMap* m, CUtensorMapDataType type, CUtensorMapSwizzle swz, const void* base,
               const cuuint64_t* dims, const cuuint64_t* strides_bytes, const cuuint32_t* box) {
  auto fn = encode_fn_m8();
  if (fn == nullptr) return false;
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, type, 3, const_cast<void*>(base), dims, strides_bytes, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int NR, typename OutT>
int launch_m8(const CUtensorMap* maps, const M8Args& a, int num_ctas, const WorkItem* work, cudaStream_t s) {
  const int smem = Cfg8<NR>::total + 1024;
  static DeviceSmemAttr attr;  // per device: the attribute belongs to the current device
  if (const int e = attr.ensure(reinterpret_cast<const void*>(mla_tc_fp8_kernel<NR, OutT>), smem)) return e;
  mla_tc_fp8_kernel<NR, OutT><<<num_ctas, kThreads, smem, s>>>(maps[0], maps[1], maps[2], maps[3], a, work);
  return (int)cudaGetLastError();
}

}  // namespace

bool mla_tc_fp8_supported(int page_size, int num_heads, int rows_per_unit) {
  const bool page_ok = page_size >= 8 && (page_size <= kTile ? kTile % page_size == 0 : page_size % kTile == 0);
  return page_ok && (rows_per_unit == 16 || rows_per_unit == 32) &&
         (num_heads <= rows_per_unit || num_heads % rows_per_unit == 0);
}

int launch_mla_tc_fp8(const skv_mla_params& p, const WorkItem* work, const int32_t* cta_indptr, int num_ctas,
                      int q_tile, int rows_per_unit, cudaStream_t s) {
  if (num_ctas == 0) return 0;
  const int NR = rows_per_unit;
  if (p.kv_dtype != SKV_E4M3 || !mla_tc_fp8_supported(p.page_size, p.num_heads, NR))
    return (int)cudaErrorInvalidValue;
  const int hc = std::min(p.num_heads, NR);
  if (hc * q_tile > NR) return (int)cudaErrorInvalidValue;
  const int total_q = p.batch * p.q_len;
  const int box_rows = std::min(p.page_size, kTile);
  CUtensorMap maps[4];
  {
    const cuuint64_t dims[3] = {512, (cuuint64_t)p.page_size, (cuuint64_t)std::max(1, p.num_pages)};
    const cuuint64_t st[2] = {(cuuint64_t)p.ckv_stride[1], (cuuint64_t)p.ckv_stride[0]};
    const cuuint32_t box[3] = {128, (cuuint32_t)box_rows, 1};
    if (!make_map8(&maps[0], CU_TENSOR_MAP_DATA_TYPE_UINT8, CU_TENSOR_MAP_SWIZZLE_128B, p.ckv, dims, st, box))
      return (int)cudaErrorInvalidValue;
  }
  {
    const cuuint64_t dims[3] = {64, (cuuint64_t)p.page_size, (cuuint64_t)std::max(1, p.num_pages)};
    const cuuint64_t st[2] = {(cuuint64_t)p.kpe_stride[1], (cuuint64_t)p.kpe_stride[0]};
    const cuuint32_t box[3] = {64, (cuuint32_t)box_rows, 1};
    if (!make_map8(&maps[1], CU_TENSOR_MAP_DATA_TYPE_UINT8, CU_TENSOR_MAP_SWIZZLE_64B, p.kpe, dims, st, box))
      return (int)cudaErrorInvalidValue;
  }
  {
    const cuuint64_t dims[3] = {512, (cuuint64_t)p.num_heads, (cuuint64_t)std::max(1, total_q)};
    const cuuint64_t st[2] = {512 * 2, (cuuint64_t)p.num_heads * 512 * 2};
    const cuuint32_t box[3] = {64, (cuuint32_t)hc, (cuuint32_t)q_tile};
    if (!make_map8(&maps[2], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, CU_TENSOR_MAP_SWIZZLE_128B, p.q_nope, dims, st, box))
      return (int)cudaErrorInvalidValue;
  }
  {
    const cuuint64_t dims[3] = {64, (cuuint64_t)p.num_heads, (cuuint64_t)std::max(1, total_q)};
    const cuuint64_t st[2] = {64 * 2, (cuuint64_t)p.num_heads * 64 * 2};
    const cuuint32_t box[3] = {64, (cuuint32_t)hc, (cuuint32_t)q_tile};
    if (!make_map8(&maps[3], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, CU_TENSOR_MAP_SWIZZLE_128B, p.q_pe, dims, st, box))
      return (int)cudaErrorInvalidValue;
  }
  M8Args a;
  a.kv_indptr = p.kv_indptr;
  a.kv_indices = p.kv_indices;
  a.last = p.kv_last_page_len;
  a.cta_indptr = cta_indptr;
  a.num_pages = p.num_pages;
  a.page_size = p.page_size;
  a.heads = p.num_heads;
  a.hc = hc;
  a.hg = p.num_heads / hc;
  a.q_tile = q_tile;
  a.group = (p.q_len / q_tile) * a.hg;  // CTAs per KV slice, grid = slices x group
  if (p.q_len % q_tile != 0 || num_ctas % a.group != 0) return (int)cudaErrorInvalidValue;
  a.kv_scale = p.kv_scale;
  a.scale_log2 = p.sm_scale * p.kv_scale * kLog2e;
  a.o = p.o;
  a.lse = p.lse;
  a.o_part = p.o_part;
  a.lse_part = p.lse_part;
  a.status = p.status;
  const bool bf = p.o_dtype == SKV_BF16;
  if (NR == 16)
    return bf ? launch_m8<16, __nv_bfloat16>(maps, a, num_ctas, work, s)
              : launch_m8<16, float>(maps, a, num_ctas, work, s);
  return bf ? launch_m8<32, __nv_bfloat16>(maps, a, num_ctas, work, s)
            : launch_m8<32, float>(maps, a, num_ctas, work, s);
}

}  // namespace skv
