// MLA latent decode on the tensor cores (tcgen05 + TMEM), bf16 latent cache: TMA page staging, or
// for page size 1 (route: every page id is a token row) a cp.async row gather.
//
// What it computes (FlashInfer PR #3309 page, MLA decode): every head reads one latent row per
// token -- a 512-d compressed KV (ckv) and a 64-d rope key (kpe); s = scale (q_nope . ckv +
// q_pe . kpe), V = ckv.  seqlen_q is folded into the row dimension: a work item's rows are
// (query token, head) pairs, n = qi * Hc + h, with Hc = min(H, NR) heads per unit and the fold
// ratio F = q_tile tokens chosen by the planner so rows = F * Hc <= NR.  When H > NR the heads
// are split into H / NR unit groups that run one after another on the same CTA and slice of KV.
//
// B200 design.  A latent row is 1152 B, so a tile is 64 tokens (72 KB) and is held in shared
// memory from QK to PV while the next tiles stream in:
//   * S^T[64 tokens, NR] = C[64, 576] . Q^T[576, NR]  (M = 64 tokens: TMEM rows land in lanes
//     0-15 of each warp quarter; the 16-32 query rows are far too few for M);
//   * O^T[512, NR] += V^T[512, 64] . P^T[64, NR]  in four M = 128 blocks of head dims, V read
//     MN-major from the same shared tiles, O^T accumulated in TMEM across the tiles of a unit.
//   * Two rings: ckv in 16 KB slots, each one 128-dim V block of a tile (two 64-column swizzled
//     halves), released after that block's PV; kpe in 8 KB slots released after QK.  Paged
//     caches fill them with TMA boxes (page windows, issued from nine lanes); page size 1 fills
//     them with 16-byte cp.async from four warps, eight lanes per 128-byte row segment.
//   * Online softmax with a lazily raised maximum (only when a score passes the running max by
//     more than 2^8): the column max is a warp redux + 4-warp exchange paid only on a raise; O^T
//     is rescaled in TMEM by all four softmax warps then.  P^T goes to shared memory MN-major,
//     the two 16-lane halves of a warp writing the two halves of each token's rows.
//   * Tokens past the end of the unit get s = -inf by selection and their V rows are zeroed in
//     the held tile before the PV that reads them.
// Roles: warp 4 producer (with warps 9-11 in row-gather mode); warps 5-8 MMA issue, one per SM
// sub-partition (an MMA whose operands stream from shared memory holds its issuing thread for ~80
// cycles, and issuers on different sub-partitions overlap): issuer w computes QK quarter w into its
// own partial S^T accumulator and PV block w; warp 5 also allocates TMEM; warps 0-3 softmax /
// epilogue.
// All waits are bounded (SKV_DEV_TIMEOUT); roles leave together; TMEM is always released.
#include <cudaTypedefs.h>

#include <mutex>

#include "tc_ptx.cuh"

namespace skv {

namespace {

constexpr int kTile = 64;              // tokens per tile
constexpr int kHalf = kTile * 128;     // one 64-column swizzled region of a tile: 8 KB
constexpr int kCSlot = 2 * kHalf;      // ckv slot: one 128-dim block (16 KB)
constexpr int kKSlot = kHalf;          // kpe slot (8 KB)
constexpr int kIssuers = 4;          // MMA issuing warps 5-8, one per SM sub-partition
constexpr int kGatherWarps = 4;      // page size 1: warp 4 and warps 9-11 fetch rows with cp.async
constexpr int kThreads = (5 + kIssuers + kGatherWarps - 1) * 32;  // softmax, TMA, MMA, gather warps
constexpr int kBlocks = 4;             // 512 ckv dims = 4 blocks of 128
constexpr float kRaise = 8.f;

template <int NR>
struct MlaCfg {
  static constexpr int kCStages = NR == 16 ? 9 : 8;
  static constexpr int kKStages = 4;
  static constexpr int kQRegion = NR * 128;             // one 64-column region of Q
  static constexpr int kQBytes = 9 * kQRegion;          // q_nope (8 regions) + q_pe
  static constexpr int kPBytes = kTile * 128;           // P^T MN-major: one 128-byte row per token
  static constexpr int kPBufs = 3;                      // P(t) reuses the buffer of PV(t - 3)
  static constexpr int cring = 0;
  static constexpr int kring = cring + kCStages * kCSlot;
  static constexpr int q = kring + kKStages * kKSlot;
  static constexpr int p = q + kQBytes;
  static constexpr int red = p + kPBufs * kPBytes;      // [4][NR] float
  static constexpr int alpha = red + 4 * NR * 4;        // [NR]
  static constexpr int inv = alpha + NR * 4;            // [NR]
  static constexpr int lse = inv + NR * 4;              // [NR]
  static constexpr int mrow = lse + NR * 4;             // [NR] running maximum of every row
  static constexpr int bars = mrow + NR * 4;
  static constexpr int nbars = 2 * kCStages + 2 * kKStages + 14;
  static constexpr int misc = bars + nbars * 8;
  static constexpr int total = misc + 16;
  // S: 2 buffers x 4 partial accumulators (one per issuer) x NR (M=64 lanes); O^T: 4 blocks x NR
  static constexpr int s_cols = 2 * kIssuers * NR;
  static constexpr int tmem_cols = s_cols + 4 * NR <= 256 ? 256 : 512;
};

struct MArgs {
  const int32_t* kv_indptr;
  const int32_t* kv_indices;
  const int32_t* last;
  const int32_t* cta_indptr;
  int num_pages, page_size, heads, hc, hg, q_tile;
  int gather;  // page size 1: token rows fetched with 16-byte cp.async by four warps
  int block_box;  // page size a multiple of 64: one 4-D box moves a whole 128-dim ckv block
  const uint8_t* ckv_rows;  // page size 1: row id i starts at ckv_rows + i * ckv_row_bytes
  const uint8_t* kpe_rows;
  int64_t ckv_row_bytes, kpe_row_bytes;
  float scale_log2;
  void* o;
  float* lse;
  float* o_part;
  float* lse_part;
  int32_t* status;
};

struct MUnit {
  int r, q_start, q_count, page_begin, page_end, part_row, part_stride;
  int t0, t1, ntiles;
};

__device__ __forceinline__ MUnit load_munit(const MArgs& a, const WorkItem* work, int u) {
  MUnit x;
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
  x.ntiles = x.t1 > x.t0 ? (x.t1 - x.t0 + kTile - 1) / kTile : 0;
  return x;
}

__device__ __forceinline__ float ex2(float x) {
  float r;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
  return r;
}

// maximum over the warp (sm_100 redux on f32)
__device__ __forceinline__ float redux_max(float v) {
  float r;
  asm volatile("redux.sync.max.f32 %0, %1, 0xffffffff;" : "=f"(r) : "f"(v));
  return r;
}

__device__ __forceinline__ void tma3(uint32_t dst, const CUtensorMap* map, uint32_t bar, int c0, int c1, int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5}], "
      "[%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}

__device__ __forceinline__ void tma4(uint32_t dst, const CUtensorMap* map, uint32_t bar, int c0, int c1, int c2,
                                     int c3) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5, %6}], "
      "[%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
      : "memory");
}

template <int NR, typename OutT>
__global__ void __launch_bounds__(kThreads, 1)
mla_tc_kernel(const __grid_constant__ CUtensorMap ckv_map, const __grid_constant__ CUtensorMap kpe_map,
              const __grid_constant__ CUtensorMap qn_map, const __grid_constant__ CUtensorMap qp_map, MArgs a,
              const WorkItem* __restrict__ work) {
  using C = MlaCfg<NR>;
  constexpr int NC = C::kCStages, NK = C::kKStages;
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
  auto kfull_bar = [&](int s) { return bar0 + 8u * (2 * NC + s); };
  auto kempty_bar = [&](int s) { return bar0 + 8u * (2 * NC + NK + s); };
  const uint32_t bar1 = bar0 + 8u * (2 * NC + 2 * NK);
  auto qfull_bar = [&]() { return bar1; };
  auto qempty_bar = [&]() { return bar1 + 8u; };
  auto sfull_bar = [&](int b) { return bar1 + 8u * (2 + b); };
  auto sempty_bar = [&](int b) { return bar1 + 8u * (4 + b); };
  auto pfull_bar = [&](int b) { return bar1 + 8u * (6 + b); };   // one per P buffer
  auto ofull_bar = [&](int b) { return bar1 + 8u * (9 + b); };   // four: PV(t) on t & 3
  auto ofree_bar = [&]() { return bar1 + 8u * 13; };
  static_assert(C::total + 1024 <= 232448, "fits the 227 KB opt-in shared memory");

  if (tid == 0) {
    for (int s = 0; s < NC; ++s) {
      tc::mbar_init(cfull_bar(s), a.gather ? kGatherWarps * 32 : 1);
      tc::mbar_init(cempty_bar(s), 1);
    }
    for (int s = 0; s < NK; ++s) {
      tc::mbar_init(kfull_bar(s), a.gather ? kGatherWarps * 32 : 1);
      tc::mbar_init(kempty_bar(s), kIssuers);
    }
    tc::mbar_init(qfull_bar(), 1);
    tc::mbar_init(qempty_bar(), kIssuers);
    for (int b = 0; b < 2; ++b) {
      tc::mbar_init(sfull_bar(b), kIssuers);
      tc::mbar_init(sempty_bar(b), 4);
    }
    for (int b = 0; b < C::kPBufs; ++b) tc::mbar_init(pfull_bar(b), 4);
    for (int b = 0; b < 4; ++b) tc::mbar_init(ofull_bar(b), kIssuers);
    tc::mbar_init(ofree_bar(), 4);
    *abort_flag = 0;
    tc::fence_mbar_init();
  }
  if (warp == 4 && lane == 0) {
    if (!a.gather) {
      tc::prefetch_tmap(&ckv_map);
      tc::prefetch_tmap(&kpe_map);
    }
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

  const int u_begin = a.cta_indptr[blockIdx.x], u_end = a.cta_indptr[blockIdx.x + 1];
  const int P = a.page_size;
  const int box_rows = min(P, kTile);

  if (warp == 4 || (warp >= 5 + kIssuers && a.gather)) {
    // ======================================================================= TMA producer
    int gc = 0, gk = 0, n_unit = 0;
    bool ok = true;
    for (int u = u_begin; u < u_end && ok; ++u) {
      const MUnit x = load_munit(a, work, u);
      if (x.ntiles == 0) continue;
      const int* ids = a.kv_indices + a.kv_indptr[x.r] + x.page_begin;
      const int npages = x.page_end - x.page_begin;
      for (int hgi = 0; hgi < a.hg && ok; ++hgi) {
        if (warp == 4 && lane == 0) {  // Q of this unit once the previous unit's last S MMA is done
          if (n_unit >= 1) ok = tc::mbar_wait_sleep(qempty_bar(), (n_unit + 1) & 1, abort_flag, a.status);
          if (ok) {
            const int rows = a.hc * a.q_tile;
            tc::mbar_arrive_expect_tx(qfull_bar(), (uint32_t)(9 * rows * 128));
            for (int rg = 0; rg < 8; ++rg)
              tma3(sbase + C::q + rg * C::kQRegion, &qn_map, qfull_bar(), rg * 64, hgi * a.hc, x.q_start);
            tma3(sbase + C::q + 8 * C::kQRegion, &qp_map, qfull_bar(), 0, hgi * a.hc, x.q_start);
          }
        }
        ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
        if (a.gather) {
          // page size 1 (a page id is a token row): 128 threads of four warps fetch the tile's 64
          // rows with 16-byte cp.async, thread p taking half (p & 1) of row p >> 1 (36 chunks),
          // straight into the swizzled slots; its row id is loaded a tile ahead.  Rows past the
          // unit repeat the unit's first row (masked, and their V rows zeroed, downstream); an
          // out-of-range id reads zeros.  A tile's barriers get one arrival per thread once its
          // copies have landed (cp.async group wait + proxy fence), with the next tile in flight.
          const int pidx = (warp == 4 ? 0 : warp - (5 + kIssuers) + 1) * 32 + lane;
          // lane group of 8 per 128-byte row segment: thread (rg = pidx / 8, sub = pidx % 8) copies
          // chunk sub of segment seg (0-7: ckv block seg / 2, half seg % 2; 8: rope) of rows
          // pass * 16 + rg, so one warp instruction moves four rows x 128 contiguous bytes
          const int rg = pidx >> 3, sub = pidx & 7;
          const int gk0 = gk, gc0 = gc, T = x.ntiles;
          auto row_ids = [&](int t, int (&v)[4]) {
#pragma unroll
            for (int ps = 0; ps < 4; ++ps) {
              const int k = t * kTile + ps * 16 + rg;
              v[ps] = (t < T && k < npages) ? __ldg(ids + k) : (t < T ? __ldg(ids) : 0);
            }
          };
          // slots of tile t are free (blocking wait, or a non-blocking test); warp-uniform result
          auto claim = [&](int t, bool blocking) -> bool {
            bool free = true;
            if (lane == 0) {
              const int g = gk0 + t;
              if (g >= NK) {
                const uint32_t par = ((g / NK) + 1) & 1;
                free = blocking ? tc::mbar_wait_sleep(kempty_bar(g % NK), par, abort_flag, a.status)
                                : tc::mbar_test_wait(kempty_bar(g % NK), par);
              }
              for (int b = 0; b < kBlocks && free; ++b) {
                const int gb = gc0 + kBlocks * t + b;
                if (gb >= NC) {
                  const uint32_t par = ((gb / NC) + 1) & 1;
                  free = blocking ? tc::mbar_wait_sleep(cempty_bar(gb % NC), par, abort_flag, a.status)
                                  : tc::mbar_test_wait(cempty_bar(gb % NC), par);
                }
              }
            }
            return __shfl_sync(0xffffffffu, free ? 1 : 0, 0) != 0;
          };
          int id_next[4];
          row_ids(0, id_next);
          auto issue = [&](int t) {  // this thread's 36 chunks of tile t, one commit group
            int idv[4];
#pragma unroll
            for (int ps = 0; ps < 4; ++ps) idv[ps] = id_next[ps];
            row_ids(t + 1, id_next);
            uint32_t seg_base[9];
#pragma unroll
            for (int sg = 0; sg < 8; ++sg)
              seg_base[sg] = sbase + C::cring + ((gc0 + kBlocks * t + (sg >> 1)) % NC) * kCSlot + (sg & 1) * kHalf;
            seg_base[8] = sbase + C::kring + ((gk0 + t) % NK) * kKSlot;
#pragma unroll
            for (int ps = 0; ps < 4; ++ps) {
              const int row = ps * 16 + rg;
              const bool in_range = (unsigned)idv[ps] < (unsigned)a.num_pages;
              if (!in_range) report(a.status, SKV_DEV_PAGE_OOB);
              const uint8_t* crow = a.ckv_rows + (int64_t)(in_range ? idv[ps] : 0) * a.ckv_row_bytes + sub * 16;
              const uint8_t* krow = a.kpe_rows + (int64_t)(in_range ? idv[ps] : 0) * a.kpe_row_bytes + sub * 16;
              const uint32_t nbytes = in_range ? 16u : 0u;
              const uint32_t off = (uint32_t)row * 128u + ((((uint32_t)sub) ^ ((uint32_t)row & 7u)) << 4);
#pragma unroll
              for (int sg = 0; sg < 9; ++sg) {
                const uint8_t* src = sg < 8 ? crow + sg * 128 : krow;
                asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(seg_base[sg] + off), "l"(src),
                             "r"(nbytes)
                             : "memory");
              }
            }
            asm volatile("cp.async.commit_group;" ::: "memory");
          };
          auto release = [&](int t) {  // this thread's copies of tile t have landed
            tc::fence_proxy_async_smem();
            tc::mbar_arrive(kfull_bar((gk0 + t) % NK));
#pragma unroll
            for (int b = 0; b < kBlocks; ++b) tc::mbar_arrive(cfull_bar((gc0 + kBlocks * t + b) % NC));
          };
          if (T > 0) {
            ok = claim(0, true);
            if (ok) issue(0);
          }
          // keep the next tile in flight when its slots are already free; never hold tile t's
          // release behind a wait for tile t + 1's slots
          for (int t = 0; t < T && ok; ++t) {
            const bool ahead = t + 1 < T && claim(t + 1, false);
            if (ahead) {
              issue(t + 1);
              asm volatile("cp.async.wait_group 1;" ::: "memory");
            } else {
              asm volatile("cp.async.wait_group 0;" ::: "memory");
            }
            release(t);
            if (t + 1 < T && !ahead) {
              ok = claim(t + 1, true);
              if (ok) issue(t + 1);
            }
          }
          asm volatile("cp.async.wait_group 0;" ::: "memory");
          gk = gk0 + T;
          gc = gc0 + kBlocks * T;
          ++n_unit;
          continue;
        }
        int win = -1000000, pid = 0;  // lanes hold the ids of pages [win, win + 32) of the unit
        for (int t = 0; t < x.ntiles && ok; ++t) {
          const int pi0 = (t * kTile) / P;
          const int npg = P >= kTile ? 1 : min(kTile / P, npages - pi0);
          const int slot0 = P >= kTile ? (t * kTile) % P : 0;
          if (pi0 < win || pi0 + npg > win + 32) {
            win = pi0;
            pid = (win + lane < npages) ? __ldg(ids + win + lane) : 0;
          }
          // the whole warp waits for the tile's kpe slot and its four ckv slots (no lane waits
          // alone while the others stand at a convergence point), lane 0 posts the expected bytes;
          // then up to nine lanes issue the TMA boxes at once (a single issuing thread serialises them)
          const int sk = gk % NK;
          int sc[kBlocks];
#pragma unroll
          for (int b = 0; b < kBlocks; ++b) sc[b] = (gc + b) % NC;
          if (gk >= NK) ok = tc::mbar_wait_sleep(kempty_bar(sk), ((gk / NK) + 1) & 1, abort_flag, a.status);
          for (int b = 0; b < kBlocks && ok; ++b) {
            const int g = gc + b;
            if (g >= NC) ok = tc::mbar_wait_sleep(cempty_bar(sc[b]), ((g / NC) + 1) & 1, abort_flag, a.status);
          }
          ok = __all_sync(0xffffffffu, ok);
          if (ok && lane == 0) {
            tc::mbar_arrive_expect_tx(kfull_bar(sk), (uint32_t)(npg * box_rows * 128));
            for (int b = 0; b < kBlocks; ++b)
              tc::mbar_arrive_expect_tx(cfull_bar(sc[b]), (uint32_t)(2 * npg * box_rows * 128));
          }
          if (!ok) break;
          for (int i = 0; i < npg; ++i) {
            const int page = __shfl_sync(0xffffffffu, pid, pi0 + i - win);
            if (lane == 0 && (unsigned)page >= (unsigned)a.num_pages) report(a.status, SKV_DEV_PAGE_OOB);
            const uint32_t row_off = (uint32_t)(i * box_rows * 128);
            if (lane == 8) {
              tma3(sbase + C::kring + sk * kKSlot + row_off, &kpe_map, kfull_bar(sk), 0, slot0, page);
            } else if (a.block_box) {  // one box per 128-dim block: both 64-column halves (fewer TMA issues)
              if (lane < 4)
                tma4(sbase + C::cring + sc[lane] * kCSlot, &ckv_map, cfull_bar(sc[lane]), 0, slot0, 2 * lane, page);
            } else if (lane < 8) {
              const int b = lane >> 1, hf = lane & 1;
              tma3(sbase + C::cring + sc[b] * kCSlot + hf * kHalf + row_off, &ckv_map, cfull_bar(sc[b]),
                   b * 128 + hf * 64, slot0, page);
            }
          }
          ++gk;
          gc += kBlocks;
        }
        ++n_unit;
      }
    }
    if (!ok && lane == 0 && !a.gather) {  // drain issued TMA copies (bounded) before the CTA can exit
      for (int q = max(0, gc - NC); q < gc; ++q) {
        const uint64_t t_start = tc::globaltimer_ns();
        while (!tc::mbar_try_wait(cfull_bar(q % NC), (q / NC) & 1) && tc::globaltimer_ns() - t_start < 50000000ull) {
        }
      }
      for (int q = max(0, gk - NK); q < gk; ++q) {
        const uint64_t t_start = tc::globaltimer_ns();
        while (!tc::mbar_try_wait(kfull_bar(q % NK), (q / NK) & 1) && tc::globaltimer_ns() - t_start < 50000000ull) {
        }
      }
    }
  } else if (warp >= 5 && warp < 5 + kIssuers) {
    // ======================================================================= MMA issuers
    // Issuer w: QK quarter w of every tile (rope k-step w + ckv block w: 9 MMAs) into its own
    // partial S^T accumulator, and PV block w (4 MMAs) into O^T block w: four issuing threads on
    // four sub-partitions keep several MMAs' operand fetches in flight.  Per tile the order is
    // QK(t) then PV(t - 1).  Only issuer w reads ckv block w of a tile, so it alone frees it.
    if (lane == 0) {
      const int w = warp - 5;
      constexpr uint32_t idesc_s = tc::idesc_bf16_f32(64, NR, false, false);
      constexpr uint32_t idesc_o = tc::idesc_bf16_f32(128, NR, true, true);  // V^T and P^T MN-major
      int g = 0, n_unit = 0, n_tile = 0;
      bool ok = true;
      const uint32_t qs = sbase + C::q;
      for (int u = u_begin; u < u_end && ok; ++u) {
        const MUnit x = load_munit(a, work, u);
        if (x.ntiles == 0) continue;
        for (int hgi = 0; hgi < a.hg && ok; ++hgi) {
          const int T = x.ntiles;
          ok = tc::mbar_wait_sleep(qfull_bar(), n_unit & 1, abort_flag, a.status);
          if (ok) tc::tc_fence_after();
          // issue whichever is ready: PV(pv) (frees the tile's ckv blocks: first) or QK(qk)
          int qk = 0, pv = 0;
          tc::PollClock clk;
          while (ok && pv < T) {
            bool did = false;
            if (pv < qk) {  // ---- PV(pv), block w
              const int tp = n_tile + pv, pb = tp % C::kPBufs;
              const int cb = kBlocks * (g + pv) + w, st = cb % NC;
              // the single O^T buffer was read by the previous unit's epilogue
              if (tc::mbar_test_wait(pfull_bar(pb), (tp / C::kPBufs) & 1) &&
                  (pv > 0 || n_unit == 0 || tc::mbar_test_wait(ofree_bar(), (n_unit + 1) & 1))) {
                tc::tc_fence_after();
                const uint32_t ps = sbase + C::p + pb * C::kPBytes;
                const uint32_t vs = sbase + C::cring + st * kCSlot;
#pragma unroll
                for (int k = 0; k < kTile / 16; ++k) {
                  const uint64_t ad = tc::sdesc_sw128(vs + k * 2048, kHalf, 1024);
                  const uint64_t bd = tc::sdesc_sw128(ps + k * 2048, 8192, 1024);
                  tc::mma_bf16(tm_o + w * NR, ad, bd, idesc_o, (pv > 0 || k > 0) ? 1u : 0u);
                }
                tc::mma_commit(cempty_bar(st));
                tc::mma_commit(ofull_bar(tp & 3));
                ++pv;
                did = true;
              }
            }
            if (!did && qk < T) {  // ---- QK(qk), quarter w
              const int tt = n_tile + qk, sb = tt & 1, gk = g + qk, sk = gk % NK;
              const int cb = kBlocks * (g + qk) + w, st = cb % NC;
              if ((tt < 2 || tc::mbar_test_wait(sempty_bar(sb), ((tt >> 1) + 1) & 1)) &&
                  tc::mbar_test_wait(kfull_bar(sk), (gk / NK) & 1) && tc::mbar_test_wait(cfull_bar(st), (cb / NC) & 1)) {
                tc::tc_fence_after();
                const uint32_t d = tm_s + (sb * kIssuers + w) * NR;
                tc::mma_bf16(d, tc::sdesc_sw128(sbase + C::kring + sk * kKSlot + w * 32, 16, 1024),
                             tc::sdesc_sw128(qs + 8 * C::kQRegion + w * 32, 16, 1024), idesc_s, 0u);
                tc::mma_commit(kempty_bar(sk));
                const uint32_t cbase = sbase + C::cring + st * kCSlot;
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                  const uint64_t ad = tc::sdesc_sw128(cbase + (k >> 2) * kHalf + (k & 3) * 32, 16, 1024);
                  const uint64_t bd =
                      tc::sdesc_sw128(qs + (2 * w + (k >> 2)) * C::kQRegion + (k & 3) * 32, 16, 1024);
                  tc::mma_bf16(d, ad, bd, idesc_s, 1u);
                }
                tc::mma_commit(sfull_bar(sb));
                if (qk + 1 == T) tc::mma_commit(qempty_bar());  // Q free after the unit's last QK
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
  } else if (warp < 4) {
    // ======================================================================= softmax / epilogue
    float* red = reinterpret_cast<float*>(smem + C::red);
    float* alpha_s = reinterpret_cast<float*>(smem + C::alpha);
    float* inv_s = reinterpret_cast<float*>(smem + C::inv);
    float* lse_s = reinterpret_cast<float*>(smem + C::lse);
    // the running maxima are the same in every thread: they live in shared memory
    float* m_s = reinterpret_cast<float*>(smem + C::mrow);
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
    const bool srow = lane < 16;              // this lane holds an S^T row (M = 64 layout)
    const int tok_in_tile = 16 * warp + (lane & 15);
    int gc = 0, n_unit = 0, n_tile = 0, pv_seen = 0;
    bool ok = true;
    auto consume_pv = [&](int upto) {
      for (; pv_seen <= upto; ++pv_seen)
        ok = tc::mbar_wait_sleep(ofull_bar(pv_seen & 3), (pv_seen >> 2) & 1, abort_flag, a.status) && ok;
      tc::tc_fence_after();
    };
    for (int u = u_begin; u < u_end && ok; ++u) {
      const MUnit x = load_munit(a, work, u);
      const int rows = x.q_count * a.hc;
      for (int hgi = 0; hgi < a.hg && ok; ++hgi) {
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
        const int T = x.ntiles;
        const int gc0 = gc;
        // P phase: lanes 0-15 take rows [0, NR/2) of their token, lanes 16-31 rows [NR/2, NR) of the
        // token of lane - 16; l[j] is the partial sum of row half * NR/2 + j
        constexpr int NH = NR / 2;
        const int half = lane >> 4;
        float l[NH];
#pragma unroll
        for (int j = 0; j < NH; ++j) l[j] = 0.f;
        if (tid < NR) m_s[tid] = -INFINITY;
        tc::named_bar_sync(1, 128);
        bool failed = false;
        for (int t = 0; t < T; ++t) {
          const int tt = n_tile + t, sb = tt & 1;
          ok = tc::mbar_wait_sleep(sfull_bar(sb), (tt >> 1) & 1, abort_flag, a.status) && ok;
          tc::tc_fence_after();
          float s[NR];
#pragma unroll
          for (int w = 0; w < kIssuers; ++w) {  // sum of the four partial accumulators
            float v[NR];
#pragma unroll
            for (int c = 0; c < NR; c += 16) {
              float v16[16];
              tc::tmem_ld_x16(tm_s + lane_base + (sb * kIssuers + w) * NR + c, v16);
#pragma unroll
              for (int i = 0; i < 16; ++i) v[c + i] = v16[i];
            }
            tc::tmem_wait_ld();  // registers of a TMEM load are read only after the wait
#pragma unroll
            for (int n = 0; n < NR; ++n) s[n] = w == 0 ? v[n] : s[n] + v[n];
          }
          tc::tc_fence_before();
          __syncwarp();
          if (lane == 0) tc::mbar_arrive(sempty_bar(sb));
          const bool valid = srow && x.t0 + t * kTile + tok_in_tile < x.t1;
          bool raise = false;
#pragma unroll
          for (int n = 0; n < NR; ++n) {
            s[n] = (valid && n < rows) ? s[n] * a.scale_log2 : -INFINITY;
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
            if (t > 0) {  // rescale O^T in TMEM (every thread owns lane `tid` of the 4 blocks)
              consume_pv(tt - 1);
#pragma unroll 1
              for (int c = 0; c < NR; c += 16) {  // 16 columns at a time: few registers held
                float al[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) al[i] = alpha_s[c + i];
#pragma unroll 1
                for (int b = 0; b < kBlocks; ++b) {
                  float ov[16];
                  tc::tmem_ld_x16(tm_o + lane_base + b * NR + c, ov);
                  tc::tmem_wait_ld();
#pragma unroll
                  for (int i = 0; i < 16; ++i) ov[i] *= al[i];
                  tc::tmem_st_x16(tm_o + lane_base + b * NR + c, ov);
                }
              }
              tc::tmem_wait_st();
              tc::tc_fence_before();
            }
            tc::named_bar_sync(1, 128);  // red / alpha_s reads done before any later rewrite
          }
          if (srow && !valid) {  // zero this token's V row in the tile's four held ckv blocks
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
          if (tt >= C::kPBufs && pv_seen <= tt - C::kPBufs) consume_pv(tt - C::kPBufs);  // P(t)'s buffer was PV's
          {
            float sv[NH], mloc[NH];
#pragma unroll
            for (int jj = 0; jj < NH; ++jj) {  // upper rows move from lane l to lane l + 16
              const float up = __shfl_sync(0xffffffffu, s[NH + jj], lane & 15);
              sv[jj] = half ? up : s[jj];
              mloc[jj] = m_s[half * NH + jj];
            }
            // token row of P^T (MN-major, 128-byte swizzle): bf16 of rows 0 .. NR-1
            uint8_t* prow = smem + C::p + (tt % C::kPBufs) * C::kPBytes + tok_in_tile * 128;
            uint32_t pw[NH / 2];
#pragma unroll
            for (int jj = 0; jj < NH; jj += 2) {
              // masked scores give 0 (rows past the unit's rows have no finite maximum)
              const float p0 = sv[jj] == -INFINITY ? 0.f : ex2(sv[jj] - mloc[jj]);
              const float p1 = sv[jj + 1] == -INFINITY ? 0.f : ex2(sv[jj + 1] - mloc[jj + 1]);
              l[jj] += p0;
              l[jj + 1] += p1;
              __nv_bfloat162 h2 = __floats2bfloat162_rn(p0, p1);
              pw[jj >> 1] = *reinterpret_cast<uint32_t*>(&h2);
            }
            const int x7 = tok_in_tile & 7;
#pragma unroll
            for (int c = 0; c < NH / 8; ++c) {  // 16-byte chunk (half * NH / 8 + c) of the row
              const int ch = half * (NH / 8) + c;
              *reinterpret_cast<uint4*>(prow + (((ch ^ x7) & 7) << 4)) =
                  make_uint4(pw[4 * c], pw[4 * c + 1], pw[4 * c + 2], pw[4 * c + 3]);
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
        gc = gc0 + kBlocks * T;
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
        if (tid == 0) {
#pragma unroll
          for (int n = 0; n < NR; ++n) {
            const float lt = red[n] + red[NR + n] + red[2 * NR + n] + red[3 * NR + n];
            inv_s[n] = lt > 0.f ? 1.f / lt : 0.f;
            lse_s[n] = lt > 0.f ? (m_s[n] + log2f(lt)) * kLn2 : -INFINITY;
          }
        }
        float ov[kBlocks][NR];
#pragma unroll
        for (int b = 0; b < kBlocks; ++b)
#pragma unroll
          for (int c = 0; c < NR; c += 16) {
            float v16[16];
            tc::tmem_ld_x16(tm_o + lane_base + b * NR + c, v16);
            tc::tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 16; ++i) ov[b][c + i] = v16[i];
          }
        tc::tc_fence_before();
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(ofree_bar());
        tc::named_bar_sync(1, 128);
#pragma unroll
        for (int n = 0; n < NR; ++n) {
          if (n >= rows) break;
          const int qi = n / a.hc, h = h0 + n % a.hc;
          const float iv = inv_s[n];
          if (x.part_row < 0) {
            OutT* dst = reinterpret_cast<OutT*>(a.o) + ((int64_t)(x.q_start + qi) * a.heads + h) * 512 + tid;
#pragma unroll
            for (int b = 0; b < kBlocks; ++b) store_out(dst + b * 128, ov[b][n] * iv);
          } else {
            float* dst = a.o_part + (((int64_t)x.part_row + (int64_t)qi * x.part_stride) * a.heads + h) * 512 + tid;
#pragma unroll
            for (int b = 0; b < kBlocks; ++b) dst[b * 128] = ov[b][n] * iv;
          }
        }
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
    tc::tmem_dealloc(tmem, MlaCfg<NR>::tmem_cols);
  }
}

// ------------------------------------------------------------------------------ host side
PFN_cuTensorMapEncodeTiled_v12000 encode_fn_m() {
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

bool make_map_m(CUtensorMap* m, const void* base, const cuuint64_t* dims, const cuuint64_t* strides_bytes,
                const cuuint32_t* box, int rank = 3) {
  // rank 4 is the ckv block view (64 dims, slot, 64-dim chunk, page)
  auto fn = encode_fn_m();
  if (fn == nullptr) return false;
  cuuint32_t estr[4] = {1, 1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, const_cast<void*>(base), dims, strides_bytes, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int NR, typename OutT>
int launch_m(const CUtensorMap* maps, const MArgs& a, int num_ctas, const WorkItem* work, cudaStream_t s) {
  const int smem = MlaCfg<NR>::total + 1024;
  static DeviceSmemAttr attr;  // per device: the attribute belongs to the current device
  if (const int e = attr.ensure(reinterpret_cast<const void*>(mla_tc_kernel<NR, OutT>), smem)) return e;
  // the three extra gather warps exist only in row-gather mode
  const int threads = a.gather ? kThreads : kThreads - (kGatherWarps - 1) * 32;
  mla_tc_kernel<NR, OutT><<<num_ctas, threads, smem, s>>>(maps[0], maps[1], maps[2], maps[3], a, work);
  return (int)cudaGetLastError();
}

}  // namespace

bool mla_tc_supported(int kv_dtype, int page_size, int num_heads, int rows_per_unit) {
  const bool page_ok = page_size == 1 ||
                       (page_size >= 8 && (page_size <= kTile ? kTile % page_size == 0 : page_size % kTile == 0));
  return kv_dtype == SKV_BF16 && page_ok && (rows_per_unit == 16 || rows_per_unit == 32) &&
         (num_heads <= rows_per_unit || num_heads % rows_per_unit == 0);
}

int mla_tc_tile_tokens() { return kTile; }

int launch_mla_tc(const skv_mla_params& p, const WorkItem* work, const int32_t* cta_indptr, int num_ctas,
                  int q_tile, int rows_per_unit, cudaStream_t s) {
  if (num_ctas == 0) return 0;
  const int NR = rows_per_unit;
  if (!mla_tc_supported(p.kv_dtype, p.page_size, p.num_heads, NR)) return (int)cudaErrorInvalidValue;
  const int hc = std::min(p.num_heads, NR);
  if (hc * q_tile > NR) return (int)cudaErrorInvalidValue;
  const int box_rows = std::min(p.page_size, kTile);
  const int total_q = p.batch * p.q_len;
  CUtensorMap maps[4];
  const bool gather = p.page_size == 1;
  if (gather) {  // rows are fetched by cp.async; the maps are unused but must be valid objects
    maps[0] = CUtensorMap{};
    maps[1] = CUtensorMap{};
  }
  const bool block_box = !gather && p.page_size % kTile == 0;
  if (block_box) {
    // (64 dims, slot, 64-dim chunk, page): a box of 64 slots x 2 chunks is one 128-dim block, landing
    // as its two 64-column swizzled halves one after the other
    const cuuint64_t dims[4] = {64, (cuuint64_t)p.page_size, 8, (cuuint64_t)std::max(1, p.num_pages)};
    const cuuint64_t st[3] = {(cuuint64_t)p.ckv_stride[1] * 2, 128, (cuuint64_t)p.ckv_stride[0] * 2};
    const cuuint32_t box[4] = {64, (cuuint32_t)kTile, 2, 1};
    if (!make_map_m(&maps[0], p.ckv, dims, st, box, 4)) return (int)cudaErrorInvalidValue;
  } else if (!gather) {
    const cuuint64_t dims[3] = {512, (cuuint64_t)p.page_size, (cuuint64_t)std::max(1, p.num_pages)};
    const cuuint64_t st[2] = {(cuuint64_t)p.ckv_stride[1] * 2, (cuuint64_t)p.ckv_stride[0] * 2};
    const cuuint32_t box[3] = {64, (cuuint32_t)box_rows, 1};
    if (!make_map_m(&maps[0], p.ckv, dims, st, box)) return (int)cudaErrorInvalidValue;
  }
  if (!gather) {
    const cuuint64_t dims[3] = {64, (cuuint64_t)p.page_size, (cuuint64_t)std::max(1, p.num_pages)};
    const cuuint64_t st[2] = {(cuuint64_t)p.kpe_stride[1] * 2, (cuuint64_t)p.kpe_stride[0] * 2};
    const cuuint32_t box[3] = {64, (cuuint32_t)box_rows, 1};
    if (!make_map_m(&maps[1], p.kpe, dims, st, box)) return (int)cudaErrorInvalidValue;
  }
  {
    const cuuint64_t dims[3] = {512, (cuuint64_t)p.num_heads, (cuuint64_t)std::max(1, total_q)};
    const cuuint64_t st[2] = {512 * 2, (cuuint64_t)p.num_heads * 512 * 2};
    const cuuint32_t box[3] = {64, (cuuint32_t)hc, (cuuint32_t)q_tile};
    if (!make_map_m(&maps[2], p.q_nope, dims, st, box)) return (int)cudaErrorInvalidValue;
  }
  {
    const cuuint64_t dims[3] = {64, (cuuint64_t)p.num_heads, (cuuint64_t)std::max(1, total_q)};
    const cuuint64_t st[2] = {64 * 2, (cuuint64_t)p.num_heads * 64 * 2};
    const cuuint32_t box[3] = {64, (cuuint32_t)hc, (cuuint32_t)q_tile};
    if (!make_map_m(&maps[3], p.q_pe, dims, st, box)) return (int)cudaErrorInvalidValue;
  }
  MArgs a;
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
  a.gather = gather ? 1 : 0;
  a.block_box = block_box ? 1 : 0;
  a.ckv_rows = static_cast<const uint8_t*>(p.ckv);
  a.kpe_rows = static_cast<const uint8_t*>(p.kpe);
  a.ckv_row_bytes = p.ckv_stride[0] * 2;
  a.kpe_row_bytes = p.kpe_stride[0] * 2;
  a.scale_log2 = p.sm_scale * kLog2e;
  a.o = p.o;
  a.lse = p.lse;
  a.o_part = p.o_part;
  a.lse_part = p.lse_part;
  a.status = p.status;
  const bool bf = p.o_dtype == SKV_BF16;
  if (NR == 16)
    return bf ? launch_m<16, __nv_bfloat16>(maps, a, num_ctas, work, s) : launch_m<16, float>(maps, a, num_ctas, work, s);
  return bf ? launch_m<32, __nv_bfloat16>(maps, a, num_ctas, work, s) : launch_m<32, float>(maps, a, num_ctas, work, s);
}

}  // namespace skv
