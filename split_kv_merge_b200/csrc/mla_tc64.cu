// MLA latent decode on the tensor cores for 64 query rows per tile (bf16 latent cache, TMA page
// staging): requests whose rows do not fit 32 -- num_heads * q_len > 32 -- such as H = 16 with
// q_len = 4 (folded into 64 rows) and H = 128 (two 64-head groups).
//
// What it computes is the bf16 MLA kernel's (mla_tc.cu; FlashInfer PR #3309 page, MLA decode):
// s = scale (q_nope . ckv + q_pe . kpe), V = ckv, rows n = qi * Hc + h of a unit (Hc = min(H, 64)
// heads, fold F = q_tile tokens with F * Hc <= 64).
//
// B200 design.
//   * CTA groups.  A request's units -- (query tile, head group) pairs -- would each stream the
//     whole KV.  The planner instead cuts the KV into slices and gives every slice a group of R
//     co-resident CTAs, R = query tiles x head groups; CTA c runs unit c % R of every work item of
//     slice c / R.  The R CTAs stream the same pages at the same time, so each page comes from
//     HBM about once and from L2 for the others.
//   * Tiles of 64 tokens (72 KB of latent rows) stay in shared memory from QK to PV:
//       S^T[64 tokens, 64] = C[64, 576] . Q^T[576, 64]  (M = 64: rows in lanes 0-15 of each TMEM
//       lane quarter), as two partial accumulators (ckv blocks 0-1 + rope k-steps 0-1, blocks
//       2-3 + rope 2-3), double buffered;
//       O^T[512, 64] += V^T[512, 64] . P^T[64, 64] in four M = 128 blocks, V read MN-major from
//       the held ckv blocks.  S (2 x 2 x 64 columns) and O^T (4 x 64) fill the 512 TMEM columns.
//   * The query copy is 72 KB, so the ring holds two whole tiles of ckv (8 slots of 16 KB, each
//     freed after that block's PV) with one kpe slot (freed after QK) and one P buffer; the
//     producer issues a tile's ckv blocks before it waits for the kpe slot.
//   * Issue: a tcgen05.mma streaming its operands from shared memory holds its issuing thread
//     ~80 cycles, so QK and PV have their own issuers and never queue behind each other: warps 5
//     and 6 issue the two QK partials (18 MMAs each per tile), warps 7 and 8 the PV blocks 0-1
//     and 2-3 (8 MMAs each).
//   * Softmax: eight warps in two groups, group g owning columns [32 g, 32 g + 32) of S^T (warps
//     0-3 and 9-12; warp w reads TMEM lane quarter w % 4, i.e. tokens 16 (w % 4) + 0..15).  Each
//     group keeps its own lazily raised running maxima (raised only when a score passes them by
//     more than 2^8), decides raises with its own named barrier and rescales its columns of O^T
//     in TMEM.  A token's scores sit in lanes 0-15; lanes 16-31 take the upper half of the
//     group's columns by shuffle, so each thread exponentiates 16 weights per tile.
//   * Tokens past the end of the unit get s = -inf by selection and their V rows are zeroed in
//     the held tile before the PV that reads them.
// Roles: warp 4 producer; warps 5-8 MMA issue (warp 5 also allocates TMEM); warps 0-3, 9-12
// softmax / epilogue.  All waits are bounded (SKV_DEV_TIMEOUT); roles leave together; TMEM is
// always released.
#include <cudaTypedefs.h>

#include <algorithm>
#include <mutex>

#include "tc_ptx.cuh"

namespace skv {

namespace {

constexpr int NR = 64;                  // query rows per tile
constexpr int kTile = 64;               // tokens per tile
constexpr int kHalf = kTile * 128;      // one 64-column swizzled region of a tile: 8 KB
constexpr int kCSlot = 2 * kHalf;       // ckv slot: one 128-dim block (16 KB)
constexpr int kKSlot = kHalf;           // kpe slot (8 KB)
constexpr int kBlocks = 4;              // 512 ckv dims = 4 blocks of 128
constexpr int kCStages = 8;
constexpr int kThreads = 13 * 32;       // softmax 0-3, producer 4, issuers 5-8, softmax 9-12
constexpr int kGroupCols = 32;          // S^T columns per softmax group
constexpr float kRaise = 8.f;

struct Cfg {
  static constexpr int kQRegion = NR * 128;             // one 64-column region of Q: 8 KB
  static constexpr int cring = 0;
  static constexpr int kring = cring + kCStages * kCSlot;
  static constexpr int q = kring + kKSlot;
  static constexpr int p = q + 9 * kQRegion;            // P^T MN-major: one 128-byte row per token
  static constexpr int red = p + kTile * 128;           // [2 groups][4 warps][32] float
  static constexpr int alpha = red + 2 * 4 * kGroupCols * 4;  // [64]
  static constexpr int inv = alpha + NR * 4;            // [64]
  static constexpr int lse = inv + NR * 4;              // [64]
  static constexpr int mrow = lse + NR * 4;             // [64] running maximum of every column
  static constexpr int bars = mrow + NR * 4;
  static constexpr int nbars = 2 * kCStages + 2 + 14;
  static constexpr int misc = bars + nbars * 8;
  static constexpr int total = misc + 16;
  static constexpr int s_cols = 2 * 2 * NR;             // 2 buffers x 2 partials
  static constexpr int tmem_cols = 512;                 // S (256) + O^T (4 blocks x 64)
};
static_assert(Cfg::total + 1024 <= 232448, "fits the 227 KB opt-in shared memory");
static_assert(Cfg::s_cols + kBlocks * NR <= Cfg::tmem_cols, "TMEM");

struct M64Args {
  const int32_t* kv_indptr;
  const int32_t* kv_indices;
  const int32_t* last;
  const int32_t* cta_indptr;  // per slice
  int num_pages, page_size, heads, hc, hg, q_tile, group;
  int block_box;  // page size a multiple of 64: one 4-D box moves a whole 128-dim ckv block
  float scale_log2;
  void* o;
  float* lse;
  float* o_part;
  float* lse_part;
  int32_t* status;
};

struct Unit64 {
  int r, q_start, q_count, page_begin, page_end, part_row, part_stride;
  int t0, t1, ntiles;
};

// The work item stands for query tile 0 of its request; this CTA's query tile qt shifts its rows
// by qt * q_tile and its partial rows by qt * q_tile * part_stride.
__device__ __forceinline__ Unit64 load_unit64(const M64Args& a, const WorkItem* work, int u, int qt) {
  Unit64 x;
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

__device__ __forceinline__ float ex2f_approx(float x) {
  float r;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
  return r;
}
__device__ __forceinline__ float redux_max(float v) {
  float r;
  asm volatile("redux.sync.max.f32 %0, %1, 0xffffffff;" : "=f"(r) : "f"(v));
  return r;
}

__device__ __forceinline__ void tma4(uint32_t dst, const CUtensorMap* map, uint32_t bar, int c0, int c1, int c2,
                                     int c3) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5, %6}], "
      "[%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
      : "memory");
}

template <typename OutT>
__device__ __forceinline__ void write_row_out(const M64Args& a, const Unit64& x, int n, int h0, int d, float v) {
  const int qi = n / a.hc, h = h0 + n % a.hc;
  if (x.part_row < 0)
    store_out(reinterpret_cast<OutT*>(a.o) + ((int64_t)(x.q_start + qi) * a.heads + h) * 512 + d, v);
  else
    a.o_part[(((int64_t)x.part_row + (int64_t)qi * x.part_stride) * a.heads + h) * 512 + d] = v;
}
__device__ __forceinline__ void write_row_lse(const M64Args& a, const Unit64& x, int n, int h0, float v) {
  const int qi = n / a.hc, h = h0 + n % a.hc;
  if (x.part_row < 0) {
    if (a.lse != nullptr) a.lse[(int64_t)(x.q_start + qi) * a.heads + h] = v;
  } else {
    a.lse_part[((int64_t)x.part_row + (int64_t)qi * x.part_stride) * a.heads + h] = v;
  }
}

template <typename OutT>
__global__ void __launch_bounds__(kThreads, 1)
mla_tc64_kernel(const __grid_constant__ CUtensorMap ckv_map, const __grid_constant__ CUtensorMap kpe_map,
                const __grid_constant__ CUtensorMap qn_map, const __grid_constant__ CUtensorMap qp_map, M64Args a,
                const WorkItem* __restrict__ work) {
  using C = Cfg;
  constexpr int NC = kCStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = tc::smem_u32(smem);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  tc::grid_launch_dependents();  // the merge pass may be scheduled; it waits for this grid

  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + C::misc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::misc + 4);
  const uint32_t bar0 = sbase + C::bars;
  auto cfull_bar = [&](int s) { return bar0 + 8u * s; };
  auto cempty_bar = [&](int s) { return bar0 + 8u * (NC + s); };
  const uint32_t bar1 = bar0 + 8u * (2 * NC);
  auto kfull_bar = [&]() { return bar1; };
  auto kempty_bar = [&]() { return bar1 + 8u; };
  auto qfull_bar = [&]() { return bar1 + 16u; };
  auto qempty_bar = [&]() { return bar1 + 24u; };
  auto sfull_bar = [&](int b) { return bar1 + 8u * (4 + b); };
  auto sempty_bar = [&](int b) { return bar1 + 8u * (6 + b); };
  auto pfull_bar = [&]() { return bar1 + 8u * 8; };
  auto ofull_bar = [&](int b) { return bar1 + 8u * (9 + b); };   // four: PV(t) on t & 3
  auto ofree_bar = [&]() { return bar1 + 8u * 13; };
  static_assert(Cfg::nbars >= 2 * kCStages + 14, "barrier count");

  if (tid == 0) {
    for (int s = 0; s < NC; ++s) {
      tc::mbar_init(cfull_bar(s), 1);
      tc::mbar_init(cempty_bar(s), 1);
    }
    tc::mbar_init(kfull_bar(), 1);
    tc::mbar_init(kempty_bar(), 2);    // the two QK issuers
    tc::mbar_init(qfull_bar(), 1);
    tc::mbar_init(qempty_bar(), 2);
    for (int b = 0; b < 2; ++b) {
      tc::mbar_init(sfull_bar(b), 2);
      tc::mbar_init(sempty_bar(b), 8);  // the eight softmax warps
    }
    tc::mbar_init(pfull_bar(), 8);
    for (int b = 0; b < 4; ++b) tc::mbar_init(ofull_bar(b), 2);  // the two PV issuers
    tc::mbar_init(ofree_bar(), 8);
    *abort_flag = 0;
    tc::fence_mbar_init();
  }
  if (warp == 4 && lane == 0) {
    tc::prefetch_tmap(&ckv_map);
    tc::prefetch_tmap(&kpe_map);
    tc::prefetch_tmap(&qn_map);
    tc::prefetch_tmap(&qp_map);
  }
  // ckv slots start as zeros: rows of a partial tile that no page fills must be finite
  for (int i = tid; i < NC * kCSlot / 16; i += blockDim.x)
    reinterpret_cast<uint4*>(smem + C::cring)[i] = make_uint4(0, 0, 0, 0);
  tc::fence_proxy_async_smem();
  if (warp == 5) tc::tmem_alloc(tc::smem_u32(tmem_holder), C::tmem_cols);
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  const uint32_t tm_s = tmem, tm_o = tmem + C::s_cols;

  // CTA c runs slice c / group: query tile and head group from c % group
  const int slice = (int)blockIdx.x / a.group, gsel = (int)blockIdx.x % a.group;
  const int my_qt = gsel / a.hg, hgi = gsel % a.hg, h0 = hgi * a.hc;
  const int u_begin = a.cta_indptr[slice], u_end = a.cta_indptr[slice + 1];
  const int P = a.page_size;
  const int box_rows = min(P, kTile);

  if (warp == 4) {
    // ======================================================================= TMA producer
    int gc = 0, gk = 0, n_unit = 0;
    bool ok = true;
    for (int u = u_begin; u < u_end && ok; ++u) {
      const Unit64 x = load_unit64(a, work, u, my_qt);
      if (x.ntiles == 0) continue;
      const int* ids = a.kv_indices + a.kv_indptr[x.r] + x.page_begin;
      const int npages = x.page_end - x.page_begin;
      if (lane == 0) {  // Q of this unit once the previous unit's last S MMA is done
        if (n_unit >= 1) ok = tc::mbar_wait_sleep(qempty_bar(), (n_unit + 1) & 1, abort_flag, a.status);
        if (ok) {
          const int rows = a.hc * a.q_tile;
          tc::mbar_arrive_expect_tx(qfull_bar(), (uint32_t)(9 * rows * 128));
          for (int rg = 0; rg < 8; ++rg)
            tc::tma_load_3d(sbase + C::q + rg * C::kQRegion, &qn_map, qfull_bar(), rg * 64, h0, x.q_start);
          tc::tma_load_3d(sbase + C::q + 8 * C::kQRegion, &qp_map, qfull_bar(), 0, h0, x.q_start);
        }
      }
      ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
      int win = -1000000, pid = 0;  // lanes hold the ids of pages [win, win + 32) of the unit
      for (int t = 0; t < x.ntiles && ok; ++t) {
        const int pi0 = (t * kTile) / P;
        const int npg = P >= kTile ? 1 : min(kTile / P, npages - pi0);
        const int slot0 = P >= kTile ? (t * kTile) % P : 0;
        if (pi0 < win || pi0 + npg > win + 32) {
          win = pi0;
          pid = (win + lane < npages) ? __ldg(ids + win + lane) : 0;
        }
        // the four ckv slots first (the whole warp waits, lane 0 posts the bytes, up to eight lanes
        // issue one box each per page), then the kpe slot, which frees only when the previous
        // tile's QK is done
        int sc[kBlocks];
#pragma unroll
        for (int b = 0; b < kBlocks; ++b) sc[b] = (gc + b) % NC;
        // the whole warp waits for the slots (no lane waits alone while the others stand at a
        // convergence point); lane 0 posts the expected bytes
        for (int b = 0; b < kBlocks && ok; ++b) {
          const int g = gc + b;
          if (g >= NC) ok = tc::mbar_wait_sleep(cempty_bar(sc[b]), ((g / NC) + 1) & 1, abort_flag, a.status);
        }
        ok = __all_sync(0xffffffffu, ok);
        if (ok && lane == 0)
          for (int b = 0; b < kBlocks; ++b) tc::mbar_arrive_expect_tx(cfull_bar(sc[b]), (uint32_t)(2 * npg * box_rows * 128));
        if (!ok) break;
        for (int i = 0; i < npg; ++i) {
          const int page = __shfl_sync(0xffffffffu, pid, pi0 + i - win);
          if (lane == 0 && (unsigned)page >= (unsigned)a.num_pages) report(a.status, SKV_DEV_PAGE_OOB);
          if (a.block_box) {  // one box per 128-dim block: both 64-column halves (fewer TMA issues)
            if (lane < 4) tma4(sbase + C::cring + sc[lane] * kCSlot, &ckv_map, cfull_bar(sc[lane]), 0, slot0, 2 * lane, page);
          } else if (lane < 8) {
            const int b = lane >> 1, hf = lane & 1;
            tc::tma_load_3d(sbase + C::cring + sc[b] * kCSlot + hf * kHalf + (uint32_t)(i * box_rows * 128), &ckv_map,
                            cfull_bar(sc[b]), b * 128 + hf * 64, slot0, page);
          }
        }
        gc += kBlocks;
        if (gk >= 1) ok = tc::mbar_wait_sleep(kempty_bar(), (gk + 1) & 1, abort_flag, a.status);
        ok = __all_sync(0xffffffffu, ok);
        if (ok && lane == 0) tc::mbar_arrive_expect_tx(kfull_bar(), (uint32_t)(npg * box_rows * 128));
        if (!ok) break;
        for (int i = 0; i < npg; ++i) {
          const int page = __shfl_sync(0xffffffffu, pid, pi0 + i - win);
          if (lane == 8)
            tc::tma_load_3d(sbase + C::kring + (uint32_t)(i * box_rows * 128), &kpe_map, kfull_bar(), 0, slot0, page);
        }
        ++gk;
      }
      ++n_unit;
    }
    if (!ok && lane == 0) {  // drain issued TMA copies (bounded) before the CTA can exit
      for (int q = max(0, gc - NC); q < gc; ++q) {
        const uint64_t t_start = tc::globaltimer_ns();
        while (!tc::mbar_try_wait(cfull_bar(q % NC), (q / NC) & 1) && tc::globaltimer_ns() - t_start < 50000000ull) {
        }
      }
      if (gk >= 1) {
        const uint64_t t_start = tc::globaltimer_ns();
        while (!tc::mbar_try_wait(kfull_bar(), (gk - 1) & 1) && tc::globaltimer_ns() - t_start < 50000000ull) {
        }
      }
      if (n_unit >= 1) {
        const uint64_t t_start = tc::globaltimer_ns();
        while (!tc::mbar_try_wait(qfull_bar(), (n_unit - 1) & 1) && tc::globaltimer_ns() - t_start < 50000000ull) {
        }
      }
    }
  } else if (warp == 5 || warp == 6) {
    // ======================================================================= QK issuers
    // Issuer w: partial accumulator w of S^T(t) = rope k-steps 2w, 2w+1 (then the kpe slot can
    // be reused) + ckv blocks 2w, 2w+1 (16 MMAs).
    if (lane == 0) {
      const int w = warp - 5;
      constexpr uint32_t idesc_s = tc::idesc_bf16_f32(64, NR, false, false);
      int g = 0, n_unit = 0, n_tile = 0;
      bool ok = true;
      const uint32_t qs = sbase + C::q;
      for (int u = u_begin; u < u_end && ok; ++u) {
        const Unit64 x = load_unit64(a, work, u, my_qt);
        if (x.ntiles == 0) continue;
        ok = tc::mbar_wait_sleep(qfull_bar(), n_unit & 1, abort_flag, a.status);
        for (int t = 0; t < x.ntiles && ok; ++t) {
          const int tt = n_tile + t, sb = tt & 1, gk = g + t;
          if (tt >= 2) ok = tc::mbar_wait_sleep(sempty_bar(sb), ((tt >> 1) + 1) & 1, abort_flag, a.status);
          if (ok) ok = tc::mbar_wait_sleep(kfull_bar(), gk & 1, abort_flag, a.status);
#pragma unroll
          for (int qq = 0; qq < 2 && ok; ++qq) {
            const int cb = kBlocks * gk + 2 * w + qq;
            ok = tc::mbar_wait_sleep(cfull_bar(cb % NC), (cb / NC) & 1, abort_flag, a.status);
          }
          if (!ok) break;
          tc::tc_fence_after();
          const uint32_t d = tm_s + (sb * 2 + w) * NR;
#pragma unroll
          for (int qq = 0; qq < 2; ++qq) {
            const int qw = 2 * w + qq;
            tc::mma_bf16(d, tc::sdesc_sw128(sbase + C::kring + qw * 32, 16, 1024),
                         tc::sdesc_sw128(qs + 8 * C::kQRegion + qw * 32, 16, 1024), idesc_s, qq > 0 ? 1u : 0u);
          }
          tc::mma_commit(kempty_bar());
#pragma unroll
          for (int qq = 0; qq < 2; ++qq) {
            const int qw = 2 * w + qq;
            const uint32_t cbase = sbase + C::cring + ((kBlocks * gk + qw) % NC) * kCSlot;
#pragma unroll
            for (int k = 0; k < 8; ++k) {
              const uint64_t ad = tc::sdesc_sw128(cbase + (k >> 2) * kHalf + (k & 3) * 32, 16, 1024);
              const uint64_t bd = tc::sdesc_sw128(qs + (2 * qw + (k >> 2)) * C::kQRegion + (k & 3) * 32, 16, 1024);
              tc::mma_bf16(d, ad, bd, idesc_s, 1u);
            }
          }
          tc::mma_commit(sfull_bar(sb));
          if (t + 1 == x.ntiles) tc::mma_commit(qempty_bar());  // Q free after the unit's last QK
        }
        g += x.ntiles;
        n_tile += x.ntiles;
        ++n_unit;
      }
    }
  } else if (warp == 7 || warp == 8) {
    // ======================================================================= PV issuers
    // Issuer v: O^T blocks 2v, 2v+1 (4 MMAs each over the tile's 64 tokens); each block's ckv slot
    // is released after its PV.
    if (lane == 0) {
      const int v = warp - 7;
      constexpr uint32_t idesc_o = tc::idesc_bf16_f32(128, NR, true, true);  // V^T and P^T MN-major
      int g = 0, n_unit = 0, n_tile = 0;
      bool ok = true;
      const uint32_t ps = sbase + C::p;
      for (int u = u_begin; u < u_end && ok; ++u) {
        const Unit64 x = load_unit64(a, work, u, my_qt);
        if (x.ntiles == 0) continue;
        // the single O^T buffer was read by the previous unit's epilogue
        if (n_unit >= 1) ok = tc::mbar_wait_sleep(ofree_bar(), (n_unit + 1) & 1, abort_flag, a.status);
        for (int t = 0; t < x.ntiles && ok; ++t) {
          const int tt = n_tile + t;
          ok = tc::mbar_wait_sleep(pfull_bar(), tt & 1, abort_flag, a.status);
          if (!ok) break;
          tc::tc_fence_after();
#pragma unroll
          for (int bb = 0; bb < 2; ++bb) {
            const int b = 2 * v + bb;
            const int cb = kBlocks * (g + t) + b, st = cb % NC;
            const uint32_t vs = sbase + C::cring + st * kCSlot;
#pragma unroll
            for (int k = 0; k < kTile / 16; ++k) {
              const uint64_t ad = tc::sdesc_sw128(vs + k * 2048, kHalf, 1024);
              const uint64_t bd = tc::sdesc_sw128(ps + k * 2048, 8192, 1024);
              tc::mma_bf16(tm_o + b * NR, ad, bd, idesc_o, (t > 0 || k > 0) ? 1u : 0u);
            }
            tc::mma_commit(cempty_bar(st));
          }
          tc::mma_commit(ofull_bar(tt & 3));
        }
        g += x.ntiles;
        n_tile += x.ntiles;
        ++n_unit;
      }
    }
  } else {
    // ======================================================================= softmax / epilogue
    // group gw: columns [cb0, cb0 + 32); warp quarter wq: tokens 16 wq .. +16 of a tile (lanes
    // 0-15 hold S^T rows), TMEM lanes 32 wq .. +32 (= head dims 32 wq + lane of each O^T block)
    const int gw = warp < 4 ? 0 : 1;
    const int wq = warp & 3;
    const int gtid = wq * 32 + lane;                 // 0 .. 127 within the group
    const int cb0 = gw * kGroupCols;
    const int bar_id = 1 + gw;
    float* red = reinterpret_cast<float*>(smem + C::red) + gw * 4 * kGroupCols;
    float* alpha_s = reinterpret_cast<float*>(smem + C::alpha);
    float* inv_s = reinterpret_cast<float*>(smem + C::inv);
    float* lse_s = reinterpret_cast<float*>(smem + C::lse);
    float* m_s = reinterpret_cast<float*>(smem + C::mrow);
    const uint32_t lane_base = (uint32_t)(wq * 32) << 16;
    const bool srow = lane < 16;
    const int tok_in_tile = 16 * wq + (lane & 15);
    const int half = lane >> 4;
    constexpr int NH = kGroupCols / 2;               // weights per thread per tile
    int gc = 0, n_unit = 0, n_tile = 0, pv_seen = 0;
    bool ok = true;
    auto consume_pv = [&](int upto) {
      for (; pv_seen <= upto; ++pv_seen)
        ok = tc::mbar_wait_sleep(ofull_bar(pv_seen & 3), (pv_seen >> 2) & 1, abort_flag, a.status) && ok;
      tc::tc_fence_after();
    };
    for (int u = u_begin; u < u_end && ok; ++u) {
      const Unit64 x = load_unit64(a, work, u, my_qt);
      const int rows = x.q_count * a.hc;
      if (x.ntiles == 0) {  // no tokens: O = 0, LSE = -inf for this group's rows
        for (int n = cb0; n < min(rows, cb0 + kGroupCols); ++n) {
          for (int d = gtid; d < 512; d += 128) write_row_out<OutT>(a, x, n, h0, d, 0.f);
          if (gtid == 0) write_row_lse(a, x, n, h0, -INFINITY);
        }
        continue;
      }
      const int T = x.ntiles;
      const int gc0 = gc;
      float l[NH];
#pragma unroll
      for (int j = 0; j < NH; ++j) l[j] = 0.f;
      if (gtid < kGroupCols) m_s[cb0 + gtid] = -INFINITY;
      tc::named_bar_sync(bar_id, 128);
      bool failed = false;
      for (int t = 0; t < T; ++t) {
        const int tt = n_tile + t, sb = tt & 1;
        ok = tc::mbar_wait_sleep(sfull_bar(sb), (tt >> 1) & 1, abort_flag, a.status) && ok;
        tc::tc_fence_after();
        float s[kGroupCols];
        {
          float v0[16], v1[16], w0[16], w1[16];  // both partials, both 16-column halves, one wait
          tc::tmem_ld_x16(tm_s + lane_base + (sb * 2 + 0) * NR + cb0, v0);
          tc::tmem_ld_x16(tm_s + lane_base + (sb * 2 + 0) * NR + cb0 + 16, v1);
          tc::tmem_ld_x16(tm_s + lane_base + (sb * 2 + 1) * NR + cb0, w0);
          tc::tmem_ld_x16(tm_s + lane_base + (sb * 2 + 1) * NR + cb0 + 16, w1);
          tc::tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            s[i] = v0[i] + w0[i];
            s[16 + i] = v1[i] + w1[i];
          }
        }
        tc::tc_fence_before();
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(sempty_bar(sb));
        const bool valid = srow && x.t0 + t * kTile + tok_in_tile < x.t1;
        bool raise = false;
#pragma unroll
        for (int n4 = 0; n4 < kGroupCols; n4 += 4) {
          const float4 mv = *reinterpret_cast<const float4*>(m_s + cb0 + n4);
          const float mm[4] = {mv.x, mv.y, mv.z, mv.w};
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int n = n4 + i;
            s[n] = (valid && cb0 + n < rows) ? s[n] * a.scale_log2 : -INFINITY;
            raise |= s[n] > mm[i] + kRaise;
          }
        }
        if (tc::bar_or(bar_id, 128, raise || !ok || t == 0)) {
          if (!tc::bar_and(bar_id, 128, ok)) {
            failed = true;
            break;
          }
#pragma unroll
          for (int n = 0; n < kGroupCols; ++n) {  // column max over the warp's 16 token lanes (others -inf)
            const float v = redux_max(s[n]);
            if (lane == 0) red[wq * kGroupCols + n] = v;
          }
          tc::named_bar_sync(bar_id, 128);
          if (gtid < kGroupCols) {  // one thread per column: new maximum and the factor for l and O
            const int n = gtid;
            const float mx = fmaxf(fmaxf(red[n], red[kGroupCols + n]), fmaxf(red[2 * kGroupCols + n], red[3 * kGroupCols + n]));
            const float mo = m_s[cb0 + n], mn = fmaxf(mo, mx);
            alpha_s[cb0 + n] = (mn == -INFINITY || mo == mn) ? 1.f : exp2f(mo - mn);
            m_s[cb0 + n] = mn;
          }
          tc::named_bar_sync(bar_id, 128);
#pragma unroll
          for (int j = 0; j < NH; ++j) l[j] *= alpha_s[cb0 + half * NH + j];
          if (t > 0) {  // rescale this group's columns of O^T (every thread owns TMEM lane 32 wq + lane)
            consume_pv(tt - 1);
#pragma unroll 1
            for (int c = 0; c < kGroupCols; c += 16) {
              float al[16];
#pragma unroll
              for (int i = 0; i < 16; ++i) al[i] = alpha_s[cb0 + c + i];
#pragma unroll 1
              for (int b = 0; b < kBlocks; ++b) {
                float ov[16];
                tc::tmem_ld_x16(tm_o + lane_base + b * NR + cb0 + c, ov);
                tc::tmem_wait_ld();
#pragma unroll
                for (int i = 0; i < 16; ++i) ov[i] *= al[i];
                tc::tmem_st_x16(tm_o + lane_base + b * NR + cb0 + c, ov);
              }
            }
            tc::tmem_wait_st();
            tc::tc_fence_before();
          }
          tc::named_bar_sync(bar_id, 128);  // red / alpha_s reads done before any later rewrite
        }
        if (gw == 0 && srow && !valid) {  // zero this token's V row in the tile's four held ckv blocks
#pragma unroll 1
          for (int b = 0; b < kBlocks; ++b) {
            const int st = (gc0 + kBlocks * t + b) % NC;
            uint8_t* row = smem + C::cring + st * kCSlot + tok_in_tile * 128;
#pragma unroll
            for (int hf = 0; hf < 2; ++hf)
#pragma unroll
              for (int i = 0; i < 8; ++i) reinterpret_cast<uint4*>(row + hf * kHalf)[i] = make_uint4(0, 0, 0, 0);
          }
        }
        if (tt >= 1 && pv_seen <= tt - 1) consume_pv(tt - 1);  // the single P buffer was PV(t - 1)'s
        {
          float sv[NH], mloc[NH];
#pragma unroll
          for (int jj = 0; jj < NH; ++jj) {  // upper columns move from lane l to lane l + 16
            const float up = __shfl_sync(0xffffffffu, s[NH + jj], lane & 15);
            sv[jj] = half ? up : s[jj];
            mloc[jj] = m_s[cb0 + half * NH + jj];
          }
          // token row of P^T (MN-major, 128-byte swizzle): bf16 of columns cb0 + half * NH + 0..NH
          uint8_t* prow = smem + C::p + tok_in_tile * 128;
          uint32_t pw[NH / 2];
#pragma unroll
          for (int jj = 0; jj < NH; jj += 2) {
            const float p0 = sv[jj] == -INFINITY ? 0.f : ex2f_approx(sv[jj] - mloc[jj]);
            const float p1 = sv[jj + 1] == -INFINITY ? 0.f : ex2f_approx(sv[jj + 1] - mloc[jj + 1]);
            l[jj] += p0;
            l[jj + 1] += p1;
            __nv_bfloat162 h2 = __floats2bfloat162_rn(p0, p1);
            pw[jj >> 1] = *reinterpret_cast<uint32_t*>(&h2);
          }
          const int x7 = tok_in_tile & 7;
#pragma unroll
          for (int c = 0; c < NH / 8; ++c) {  // 16-byte chunk of the row: columns (cb0 + half NH) / 8 + c
            const int ch = (cb0 + half * NH) / 8 + c;
            *reinterpret_cast<uint4*>(prow + (((ch ^ x7) & 7) << 4)) =
                make_uint4(pw[4 * c], pw[4 * c + 1], pw[4 * c + 2], pw[4 * c + 3]);
          }
        }
        tc::fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(pfull_bar());
      }
      if (failed) {
        ok = false;
        break;
      }
      gc = gc0 + kBlocks * T;
      n_tile += T;
      ++n_unit;
      consume_pv(n_tile - 1);
      // row sums over the 64 tokens: each 16-lane half of a warp holds half of the group's columns
#pragma unroll
      for (int j = 0; j < NH; ++j) {
        float v = l[j];
#pragma unroll
        for (int o = 8; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        if ((lane & 15) == 0) red[wq * kGroupCols + half * NH + j] = v;
      }
      if (!tc::bar_and(bar_id, 128, ok)) {
        ok = false;
        break;
      }
      if (gtid < kGroupCols) {
        const int n = gtid;
        const float lt = red[n] + red[kGroupCols + n] + red[2 * kGroupCols + n] + red[3 * kGroupCols + n];
        inv_s[cb0 + n] = lt > 0.f ? 1.f / lt : 0.f;
        lse_s[cb0 + n] = lt > 0.f ? (m_s[cb0 + n] + log2f(lt)) * kLn2 : -INFINITY;
      }
      tc::named_bar_sync(bar_id, 128);
      // O^T of this group's columns, 16 at a time per block: thread = head dim b * 128 + 32 wq + lane
#pragma unroll 1
      for (int b = 0; b < kBlocks; ++b) {
#pragma unroll 1
        for (int c = 0; c < kGroupCols; c += 16) {
          float v16[16];
          tc::tmem_ld_x16(tm_o + lane_base + b * NR + cb0 + c, v16);
          tc::tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const int n = cb0 + c + i;
            if (n < rows) write_row_out<OutT>(a, x, n, h0, b * 128 + gtid, v16[i] * inv_s[n]);
          }
        }
      }
      tc::tc_fence_before();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(ofree_bar());
      if (gtid < kGroupCols && cb0 + gtid < rows) write_row_lse(a, x, cb0 + gtid, h0, lse_s[cb0 + gtid]);
      tc::named_bar_sync(bar_id, 128);  // inv_s / lse_s / red reads done before the next unit
    }
  }

  tc::tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, Cfg::tmem_cols);
  }
}

// ------------------------------------------------------------------------------ host side
PFN_cuTensorMapEncodeTiled_v12000 encode_fn_m64() {
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

bool make_map_m64(CUtensorMap* m, const void* base, const cuuint64_t* dims, const cuuint64_t* strides_bytes,
                  const cuuint32_t* box, int rank = 3) {
  auto fn = encode_fn_m64();
  if (fn == nullptr) return false;
  cuuint32_t estr[4] = {1, 1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, const_cast<void*>(base), dims, strides_bytes, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <typename OutT>
int launch_m64(const CUtensorMap* maps, const M64Args& a, int num_ctas, const WorkItem* work, cudaStream_t s) {
  const int smem = Cfg::total + 1024;
  static DeviceSmemAttr attr;  // per device: the attribute belongs to the current device
  if (const int e = attr.ensure(reinterpret_cast<const void*>(mla_tc64_kernel<OutT>), smem)) return e;
  mla_tc64_kernel<OutT><<<num_ctas, kThreads, smem, s>>>(maps[0], maps[1], maps[2], maps[3], a, work);
  return (int)cudaGetLastError();
}

}  // namespace

bool mla_tc64_supported(int kv_dtype, int page_size, int num_heads) {
  const bool paged = page_size >= 8 && (page_size <= kTile ? kTile % page_size == 0 : page_size % kTile == 0);
  return kv_dtype == SKV_BF16 && paged && (num_heads <= NR || num_heads % NR == 0);
}

int launch_mla_tc64(const skv_mla_params& p, const WorkItem* work, const int32_t* cta_indptr, int num_ctas,
                    int q_tile, cudaStream_t s) {
  if (num_ctas == 0) return 0;
  if (!mla_tc64_supported(p.kv_dtype, p.page_size, p.num_heads)) return (int)cudaErrorInvalidValue;
  const int hc = std::min(p.num_heads, NR);
  if (q_tile < 1 || hc * q_tile > NR || p.q_len % q_tile != 0) return (int)cudaErrorInvalidValue;
  M64Args a;
  a.hc = hc;
  a.hg = p.num_heads / hc;
  a.group = (p.q_len / q_tile) * a.hg;  // CTAs per KV slice, grid = slices x group
  if (num_ctas % a.group != 0) return (int)cudaErrorInvalidValue;
  const int box_rows = std::min(p.page_size, kTile);
  const int total_q = p.batch * p.q_len;
  CUtensorMap maps[4];
  a.block_box = p.page_size % kTile == 0 ? 1 : 0;
  if (a.block_box) {
    // (64 dims, slot, 64-dim chunk, page): a box of 64 slots x 2 chunks is one 128-dim block, landing
    // as its two 64-column swizzled halves one after the other
    const cuuint64_t dims[4] = {64, (cuuint64_t)p.page_size, 8, (cuuint64_t)std::max(1, p.num_pages)};
    const cuuint64_t st[3] = {(cuuint64_t)p.ckv_stride[1] * 2, 128, (cuuint64_t)p.ckv_stride[0] * 2};
    const cuuint32_t box[4] = {64, (cuuint32_t)kTile, 2, 1};
    if (!make_map_m64(&maps[0], p.ckv, dims, st, box, 4)) return (int)cudaErrorInvalidValue;
  } else {
    const cuuint64_t dims[3] = {512, (cuuint64_t)p.page_size, (cuuint64_t)std::max(1, p.num_pages)};
    const cuuint64_t st[2] = {(cuuint64_t)p.ckv_stride[1] * 2, (cuuint64_t)p.ckv_stride[0] * 2};
    const cuuint32_t box[3] = {64, (cuuint32_t)box_rows, 1};
    if (!make_map_m64(&maps[0], p.ckv, dims, st, box)) return (int)cudaErrorInvalidValue;
  }
  {
    const cuuint64_t dims[3] = {64, (cuuint64_t)p.page_size, (cuuint64_t)std::max(1, p.num_pages)};
    const cuuint64_t st[2] = {(cuuint64_t)p.kpe_stride[1] * 2, (cuuint64_t)p.kpe_stride[0] * 2};
    const cuuint32_t box[3] = {64, (cuuint32_t)box_rows, 1};
    if (!make_map_m64(&maps[1], p.kpe, dims, st, box)) return (int)cudaErrorInvalidValue;
  }
  {
    const cuuint64_t dims[3] = {512, (cuuint64_t)p.num_heads, (cuuint64_t)std::max(1, total_q)};
    const cuuint64_t st[2] = {512 * 2, (cuuint64_t)p.num_heads * 512 * 2};
    const cuuint32_t box[3] = {64, (cuuint32_t)hc, (cuuint32_t)q_tile};
    if (!make_map_m64(&maps[2], p.q_nope, dims, st, box)) return (int)cudaErrorInvalidValue;
  }
  {
    const cuuint64_t dims[3] = {64, (cuuint64_t)p.num_heads, (cuuint64_t)std::max(1, total_q)};
    const cuuint64_t st[2] = {64 * 2, (cuuint64_t)p.num_heads * 64 * 2};
    const cuuint32_t box[3] = {64, (cuuint32_t)hc, (cuuint32_t)q_tile};
    if (!make_map_m64(&maps[3], p.q_pe, dims, st, box)) return (int)cudaErrorInvalidValue;
  }
  a.kv_indptr = p.kv_indptr;
  a.kv_indices = p.kv_indices;
  a.last = p.kv_last_page_len;
  a.cta_indptr = cta_indptr;
  a.num_pages = p.num_pages;
  a.page_size = p.page_size;
  a.heads = p.num_heads;
  a.q_tile = q_tile;
  a.scale_log2 = p.sm_scale * kLog2e;
  a.o = p.o;
  a.lse = p.lse;
  a.o_part = p.o_part;
  a.lse_part = p.lse_part;
  a.status = p.status;
  return p.o_dtype == SKV_BF16 ? launch_m64<__nv_bfloat16>(maps, a, num_ctas, work, s)
                               : launch_m64<float>(maps, a, num_ctas, work, s);
}

}  // namespace skv
