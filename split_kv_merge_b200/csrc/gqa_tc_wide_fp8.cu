// Paged GQA decode over an fp8 (e4m3) K/V cache, all KV heads of a work item in one CTA, in
// native fp8 tensor-core MMAs (tcgen05 kind::f8f6f4 + TMEM, TMA page staging).
//
// What it computes: the same attention / split partial as gqa_tc_wide.cu (request r, query
// token(s), logical pages [page_begin, page_end); split-KV + merge per the FlashInfer PR #5597
// page, section 3) for a K/V cache stored as OCP e4m3 codes with one per-tensor scale:
// k = kv_scale * code(k), v = kv_scale * code(v) (the FP8 KV decode the FlashInfer PR #3309 page
// stresses; the GQA e4m3 cache of its native-fp8 item).  s = sm_scale * kv_scale * q . code(k),
// O = kv_scale * sum_t p_t code(v_t) / l.  Shape: Hk = 8 KV heads, g * q_tile = 8 query rows per
// KV head, head_dim 128, page_size 16..256 (multiple of 16).
//
// B200 design.  A tile is 16 tokens x 8 heads = 128 rows of 128 e4m3 bytes per tensor: one 16 KB
// TMA box (slot-then-head dimension order, 128-byte swizzle), so a K+V stage is 32 KB and five
// stages are in flight.  The cache tiles feed the MMAs as they are (never converted):
//   S^T[128 rows, 64] = K[128, 128] . Q_hi^T + K . Q_lo^T        (K = 32 per MMA: 8 MMAs)
//   O^T[:, 16p..16p+16) += V_pair(p)^T[128, 32] . P_hi,p^T + V_pair(p)^T . P_lo,p^T
// The other operand of each product is split into two exact e4m3 terms, hi = rn(x) and
// lo = rn(x - hi), and the two products accumulate into the same TMEM columns (the split is
// stacked along K, so S^T and O^T keep the bf16 kernel's 64 + 64 columns):
//   * queries: each query row is scaled by the power of two that puts its largest |q| in
//     [128, 256) -- then hi + lo reproduces every bf16 q of at least 2^-9 of the row maximum
//     exactly -- and the scale goes back into that column's softmax scale;
//   * softmax weights, shifted up by 2^4 to p' in [0, 2^8] (the maximum is raised past m + 4):
//     hi + lo keeps 2^-8 relative precision from 2^-6 of the running maximum's weight up and
//     2^-14 absolute below (the bf16 paths' precision); the shift comes out of the LSE.
// P_p (pair p = two heads, 16 columns) is a [16 x 64] e4m3 K-major block: bytes 0-31 hold the
// hi terms of the pair's 32 token rows, bytes 32-63 the lo terms; two such blocks share each
// 128-byte row (bytes 0-63 and 64-127), so four P buffers fit in 16 KB.  V^T is read MN-major
// straight from the V tile (128 dims = one 128-byte swizzle row).
//
// Online softmax with a lazily raised maximum as in gqa_tc_wide.cu (raise only past m + 4 in
// log2 units here; O^T rescaled in TMEM on a raise).  Masked rows get s = -inf by selection and
// their V rows are zeroed before the PV that reads them.  The softmax of one tile is a chain of
// dependent steps (TMEM load, scale and raise test, exponentials, the split, byte stores) that
// one warp per SM sub-partition cannot hide, so two groups of four warps take alternate tiles:
// group g owns the tiles of parity g of a work item with its own running maximum m_g, row sums
// l_g and O^T_g accumulator in TMEM (the split-KV decomposition of the pages' section 3, applied
// inside the CTA over interleaved tiles), and the epilogue merges the two states exactly:
// O = (2^(m_0 - m) O_0 + 2^(m_1 - m) O_1) / (2^(m_0 - m) l_0 + 2^(m_1 - m) l_1), m = max(m_0, m_1).
//
// Roles: warps 0-7 query split (at the start of each work item), softmax (groups 0-3 and 4-7)
// and epilogue; warp 8 TMA producer (query staging copy + the K/V ring), warp 9 TMEM allocation
// + QK issue, warp 10 PV issue.  All waits are bounded (SKV_DEV_TIMEOUT); the roles leave
// together and TMEM is always released.
#include <cuda_fp16.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "tc_ptx.cuh"

namespace skv {

namespace {

constexpr int kHk = 8;              // KV heads per CTA
constexpr int kTok = 16;            // tokens per tile
constexpr int kRows = kHk * kTok;   // 128 = M of S^T
constexpr int kD = 128;             // head dim = bytes per e4m3 row
constexpr int kN = 64;              // query rows (columns of S^T): kHk * 8
constexpr int kStages = 5;
// work items of a CTA whose descriptors are staged in shared memory at kernel start, so no role
// waits on dependent global loads (work item, then the request's page range) at a unit boundary
constexpr int kUnitTab = 32;
constexpr int kKBytes = kRows * kD;           // 16 KB per tensor per tile
constexpr int kStageBytes = 2 * kKBytes;      // K + V
constexpr int kQRegion = kN * 128;            // 8 KB: one 64-column bf16 half of the query copy
constexpr int kQStage = 2 * kQRegion;         // bf16 query copy (TMA)
constexpr int kQOps = 2 * kN * 128;           // [Q_hi; Q_lo] e4m3, 64 rows x 128 B each
constexpr int kPairBytes = 16 * 128;          // 16 rows x 128 B (64 bytes of K used)
constexpr int kPBytes = 4 * kPairBytes;       // 8 KB per buffer
constexpr int kWarpTma = 8, kWarpQK = 9, kWarpPV = 10;  // warps 0-7: two softmax groups of four
constexpr int kThreads = 32 * 11;
constexpr int kTmemCols = 512;                // S0 S1, then O^T per (unit parity, group): 6 x 64 used
// The running maximum is raised only when a score passes it by more than 2^4 (log2 units), and
// every weight is formed as p' = 2^(s - m + 4) <= 2^8 (e4m3 holds up to 448): the shift moves the
// small weights of a row up into the range where the hi + lo split is relative (2^-8 from
// p' = 2^-2 up, 2^-10 absolute below -- 2^-14 of the unshifted weight).  O / l is unchanged by
// the shift; the LSE subtracts it.
constexpr float kRaise = 4.f;
constexpr float kPShift = 4.f;

struct Smem {
  static constexpr int kv = 0;
  static constexpr int qstage = kv + kStages * kStageBytes;  // 163840
  static constexpr int qops = qstage + kQStage;                // 180224
  static constexpr int p = qops + kQOps;                       // 196608
  static constexpr int alpha = p + 2 * kPBytes;                // [2][64] float: rescale factors per group
  static constexpr int fac = alpha + 2 * kN * 4;               // [2][64] float: weight of each group's O^T
  static constexpr int lse = fac + 2 * kN * 4;
  static constexpr int lsum = lse + kN * 4;                    // [2][64]
  static constexpr int msum = lsum + 2 * kN * 4;               // [2][64]
  static constexpr int qscale = msum + 2 * kN * 4;             // [2][64] float: 2^-e per query row, by unit parity
  static constexpr int utab = qscale + 2 * kN * 4;             // [kUnitTab] work item descriptors
  static constexpr int bars = utab + kUnitTab * 48;
  // ring, Q full / ready / ops empty, S full / empty (2 each), P full and O full (4 each), O free (2)
  static constexpr int nbars = 2 * kStages + 3 + 4 + 8 + 2;
  static constexpr int misc = bars + nbars * 8;
  static constexpr int total = misc + 16;
};
static_assert(Smem::total + 1024 <= 232448, "fits the 227 KB opt-in shared memory");

struct W8Args {
  const int32_t* kv_indptr;
  const int32_t* kv_indices;
  const int32_t* last;
  int num_pages, page_size, hq, q_tile, num_ctas;
  const int32_t* cta_indptr;  // CTA c runs work items cta_indptr[c] .. cta_indptr[c+1]
  float scale_log2;           // sm_scale * kv_scale * log2(e)
  float kv_scale;
  void* o;
  float* lse;
  float* o_part;
  float* lse_part;
  int32_t* status;
};

struct WUnit8 {
  int r, q_start, q_count, page_begin, page_end, part_row, part_stride;
  int t0, t1, ntiles;
  int ids_off;  // kv_indptr[r] + page_begin: the unit's first page id in kv_indices
  int pad;
};

__device__ __forceinline__ WUnit8 load_wunit8(const W8Args& a, const WorkItem* work, int u) {
  WUnit8 x;
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
  x.ids_off = a.kv_indptr[w.r] + w.page_begin;
  x.pad = 0;
  return x;
}

__device__ __forceinline__ void tma4(uint32_t dst, const CUtensorMap* map, uint32_t bar, int c0, int c1, int c2,
                                     int c3) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5, %6}], "
      "[%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
      : "memory");
}

// shared-memory matrix descriptor (sm_100), 128-byte swizzle
__device__ __forceinline__ uint64_t sw128(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  return tc::sdesc_sw128(saddr, lbo, sbo);
}

// D[tmem] (+)= A . B, kind::f8f6f4 (e4m3 operands, from the instruction descriptor), one CTA
__device__ __forceinline__ void mma_f8(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a), "l"(b), "r"(idesc), "r"(acc)
      : "memory");
}
// instruction descriptor: e4m3 A and B (format code 0), f32 D; a_mn selects an MN-major A
__host__ __device__ constexpr uint32_t idesc_e4m3(int M, int N, bool a_mn) {
  return (1u << 4) | ((a_mn ? 1u : 0u) << 15) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// two floats -> two e4m3 bytes (round to nearest even, saturating), low byte = a
__device__ __forceinline__ uint32_t e4m3x2(float a, float b) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(b), "f"(a));
  return r;
}
// two e4m3 bytes (low byte first) -> their two values (exact)
__device__ __forceinline__ float2 e4m3x2_val(uint32_t two) {
  uint32_t h;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h) : "h"((uint16_t)two));
  return __half22float2(*reinterpret_cast<__half2*>(&h));
}
// hi = rn(x), lo = rn(x - hi) of two floats, each as a packed byte pair (low byte = x0)
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

// byte offset of byte `col` of row `row` in a tile of 128-byte rows with the 128-byte swizzle
__device__ __forceinline__ uint32_t sw128_byte(uint32_t row, uint32_t col) {
  return row * 128u + ((((col >> 4) ^ (row & 7u)) & 7u) << 4) + (col & 15u);
}

// column n of S^T / O^T -> (query token offset, query head), G = GQA group size (8 / q_tile)
template <int G>
__device__ __forceinline__ void column_row8(int n, int& qi, int& hq) {
  const int e = n & 7;
  qi = e / G;
  hq = (n >> 3) * G + e % G;
}

template <int G, typename OutT>
__global__ void __launch_bounds__(kThreads, 1)
gqa_tc_wide_fp8_kernel(const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap vmap,
                       const __grid_constant__ CUtensorMap qmap, W8Args a, const WorkItem* __restrict__ work) {
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
  const uint32_t bar1 = bar0 + 8u * (2 * kStages);
  auto qfull_bar = [&]() { return bar1; };             // query copy landed (TMA)
  auto qready_bar = [&]() { return bar1 + 8u; };       // [Q_hi; Q_lo] written, query copy read
  auto qempty_bar = [&]() { return bar1 + 16u; };      // last S MMA of the unit done (ops free)
  auto sfull_bar = [&](int g) { return bar1 + 8u * (3 + g); };   // S buffer g = tile parity
  auto sempty_bar = [&](int g) { return bar1 + 8u * (5 + g); };
  auto pfull_bar = [&](int b) { return bar1 + 8u * (7 + b); };   // P buffer b = tile & 3
  auto ofull_bar = [&](int b) { return bar1 + 8u * (11 + b); };  // PV of the tile that used P buffer b
  auto ofree_bar = [&](int b) { return bar1 + 8u * (15 + b); };  // O^T pair b read by the epilogue
  static_assert(Smem::nbars == 2 * kStages + 17, "barrier count");

  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      tc::mbar_init(full_bar(s), 1);
      tc::mbar_init(empty_bar(s), 1);
    }
    tc::mbar_init(qfull_bar(), 1);
    tc::mbar_init(qready_bar(), 8);
    tc::mbar_init(qempty_bar(), 1);
    for (int g = 0; g < 2; ++g) {
      tc::mbar_init(sfull_bar(g), 1);
      tc::mbar_init(sempty_bar(g), 4);
      tc::mbar_init(ofree_bar(g), 8);
    }
    for (int b = 0; b < 4; ++b) {
      tc::mbar_init(pfull_bar(b), 4);
      tc::mbar_init(ofull_bar(b), 1);
    }
    *abort_flag = 0;
    tc::fence_mbar_init();
  }
  if (warp == kWarpTma && lane == 0) {
    tc::prefetch_tmap(&kmap);
    tc::prefetch_tmap(&vmap);
    tc::prefetch_tmap(&qmap);
  }
  // zero the V stages (finite rows where nothing is loaded) and the probability buffers (their
  // off-diagonal blocks stay zero for the whole kernel)
  for (int i = tid; i < kStages * kKBytes / 16; i += kThreads) {
    const int s = i / (kKBytes / 16), o = i % (kKBytes / 16);
    reinterpret_cast<uint4*>(smem + Smem::kv + s * kStageBytes + kKBytes)[o] = make_uint4(0, 0, 0, 0);
  }
  for (int i = tid; i < 2 * kPBytes / 16; i += kThreads)
    reinterpret_cast<uint4*>(smem + Smem::p)[i] = make_uint4(0, 0, 0, 0);
  tc::fence_proxy_async_smem();
  const int u_begin = a.cta_indptr[blockIdx.x], u_end = a.cta_indptr[blockIdx.x + 1];
  WUnit8* utab = reinterpret_cast<WUnit8*>(smem + Smem::utab);
  if (tid < min(kUnitTab, u_end - u_begin)) utab[tid] = load_wunit8(a, work, u_begin + tid);
  if (warp == kWarpQK) tc::tmem_alloc(tc::smem_u32(tmem_holder), kTmemCols);
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  const uint32_t tm_s = tmem, tm_o = tmem + 2 * kN;  // O^T of (unit parity ob, group g): tm_o + (2 ob + g) kN
  auto unit = [&](int u) { return u - u_begin < kUnitTab ? utab[u - u_begin] : load_wunit8(a, work, u); };
  // the next unit at or after u that has tiles (u_end if none)
  auto next_with_tiles = [&](int u) {
    while (u < u_end && unit(u).ntiles == 0) ++u;
    return u;
  };
  if (warp == kWarpTma) {
    // ======================================================================= TMA producer
    // Per unit: the query copy (once the previous unit's copy has been split), then the unit's
    // K/V tiles; lanes hold the page ids of the next 32 tiles, the whole warp waits for a ring slot
    // and lane 0 issues.
    int n_tile = 0, n_unit = 0;
    bool ok = true;
    bool have_pid = false;  // pid already holds this unit's first 32 page ids (fetched a unit ahead)
    int pid = 0;
    for (int u = u_begin; u < u_end && ok; ++u) {
      const WUnit8 x = unit(u);
      if (x.ntiles == 0) continue;
      const int* ids = a.kv_indices + x.ids_off;
      const int tiles_per_page = a.page_size / kTok;
      if (!have_pid) pid = (lane < x.ntiles) ? __ldg(ids + lane * kTok / a.page_size) : 0;
      have_pid = false;
      if (lane == 0) {
        if (n_unit >= 1) ok = tc::mbar_wait_sleep(qready_bar(), (n_unit - 1) & 1, abort_flag, a.status);
        if (ok) {
          tc::mbar_arrive_expect_tx(qfull_bar(), (uint32_t)kQStage);
          for (int rgn = 0; rgn < 2; ++rgn)
            tma4(sbase + Smem::qstage + rgn * kQRegion, &qmap, qfull_bar(), rgn * 64, 0, x.q_start, 0);
        }
      }
      ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
      for (int j0 = 0; j0 < x.ntiles && ok; j0 += 32) {
        const int jn = j0 + 32 + lane;
        int pid_next = (jn < x.ntiles) ? __ldg(ids + jn * kTok / a.page_size) : 0;
        if (j0 + 32 >= x.ntiles) {  // last batch: fetch the next unit's first page ids meanwhile
          const int un = next_with_tiles(u + 1);
          if (un < u_end) {
            const WUnit8 xn = unit(un);
            pid_next = (lane < xn.ntiles) ? __ldg(a.kv_indices + xn.ids_off + lane * kTok / a.page_size) : 0;
            have_pid = true;
          }
        }
        const int nj = min(32, x.ntiles - j0);
        for (int jj = 0; jj < nj; ++jj) {
          const int j = j0 + jj, t = n_tile + j, st = t % kStages;
          const int page = __shfl_sync(0xffffffffu, pid, jj);
          // the whole warp waits for the slot (no lane waits alone while the others stand at a
          // convergence point); lane 0 posts the bytes and issues the two boxes
          if (t >= kStages) ok = tc::mbar_wait(empty_bar(st), ((t / kStages) + 1) & 1, abort_flag, a.status);
          ok = __all_sync(0xffffffffu, ok);
          if (ok && lane == 0) {
            if ((unsigned)page >= (unsigned)a.num_pages) report(a.status, SKV_DEV_PAGE_OOB);
            const int slot0 = (j % tiles_per_page) * kTok;
            tc::mbar_arrive_expect_tx(full_bar(st), (uint32_t)kStageBytes);
            const uint32_t kdst = sbase + Smem::kv + st * kStageBytes;
            tma4(kdst, &kmap, full_bar(st), 0, slot0, 0, page);
            tma4(kdst + kKBytes, &vmap, full_bar(st), 0, slot0, 0, page);
          }
          if (!ok) break;
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
      if (n_unit >= 1) {
        const uint64_t t_start = tc::globaltimer_ns();
        while (!tc::mbar_try_wait(qfull_bar(), (n_unit - 1) & 1) && tc::globaltimer_ns() - t_start < 50000000ull) {
        }
      }
    }
  } else if (warp == kWarpQK) {
    // ======================================================================= QK issuer
    // S^T(t) into S buffer t & 1 as soon as its K tile is in and softmax group t & 1 has read that
    // buffer's previous tile; PV has its own issuer, so a tile's QK never waits behind a PV (an MMA
    // streaming from shared memory holds its issuing thread for tens of cycles).
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_e4m3(128, kN, false);
      int n_tile = 0, n_unit = 0;
      bool ok = true;
      const uint32_t qo = sbase + Smem::qops;
      for (int u = u_begin; u < u_end && ok; ++u) {
        const WUnit8 x = unit(u);
        if (x.ntiles == 0) continue;
        ok = tc::mbar_wait(qready_bar(), n_unit & 1, abort_flag, a.status);
        if (!ok) break;
        tc::tc_fence_after();
        for (int j = 0; j < x.ntiles && ok; ++j) {
          const int t = n_tile + j, st = t % kStages, sb = t & 1;
          ok = tc::mbar_wait(full_bar(st), (t / kStages) & 1, abort_flag, a.status);
          if (ok && t >= 2) ok = tc::mbar_wait(sempty_bar(sb), ((t >> 1) + 1) & 1, abort_flag, a.status);
          if (!ok) break;
          tc::tc_fence_after();
          const uint32_t ks = sbase + Smem::kv + st * kStageBytes;
#pragma unroll
          for (int h = 0; h < 2; ++h)  // h = 0: Q_hi, h = 1: Q_lo
#pragma unroll
            for (int k = 0; k < kD / 32; ++k)
              mma_f8(tm_s + sb * kN, sw128(ks + k * 32, 16, 1024), sw128(qo + h * kN * 128 + k * 32, 16, 1024),
                     idesc_s, (h > 0 || k > 0) ? 1u : 0u);
          tc::mma_commit(sfull_bar(sb));
          if (j == x.ntiles - 1) tc::mma_commit(qempty_bar());  // query terms free once the last S is done
        }
        n_tile += x.ntiles;
        ++n_unit;
      }
    }
  } else if (warp == kWarpPV) {
    // ======================================================================= PV issuer
    // O^T(g) += V(t)^T . [P_hi; P_lo](t)^T into the O^T of tile t's group once P(t) is written;
    // then the K/V ring slot is free
    if (lane == 0) {
      constexpr uint32_t idesc_o = idesc_e4m3(128, 16, true);  // V^T MN-major, P K-major
      int n_tile = 0, n_unit = 0;
      bool ok = true;
      for (int u = u_begin; u < u_end && ok; ++u) {
        const WUnit8 x = unit(u);
        if (x.ntiles == 0) continue;
        const int ob = n_unit & 1;
        // this unit's O^T pair was last read by the epilogue of unit n_unit - 2
        if (n_unit >= 2) ok = tc::mbar_wait(ofree_bar(ob), ((n_unit >> 1) + 1) & 1, abort_flag, a.status);
        for (int j = 0; j < x.ntiles && ok; ++j) {
          const int t = n_tile + j, st = t % kStages, pb = t & 3, g = t & 1;
          ok = tc::mbar_wait(pfull_bar(pb), (t >> 2) & 1, abort_flag, a.status);
          if (!ok) break;
          tc::tc_fence_after();
          const uint32_t o_cols = tm_o + (2 * ob + g) * kN;
          const uint32_t vs = sbase + Smem::kv + st * kStageBytes + kKBytes;
          const uint32_t ps = sbase + Smem::p + g * kPBytes + (pb >> 1) * 64;
#pragma unroll
          for (int pr = 0; pr < 4; ++pr) {
#pragma unroll
            for (int k = 0; k < 2; ++k) {  // k = 0: hi terms, k = 1: lo terms (32 bytes further)
              const uint64_t ad = sw128(vs + pr * 32 * 128, 8192, 1024);
              const uint64_t bd = sw128(ps + pr * kPairBytes + k * 32, 16, 1024);
              // j < 2: the first tile of group g in this unit starts its O^T
              mma_f8(o_cols + 16 * pr, ad, bd, idesc_o, (j >= 2 || k > 0) ? 1u : 0u);
            }
          }
          tc::mma_commit(ofull_bar(pb));
          tc::mma_commit(empty_bar(st));
        }
        n_tile += x.ntiles;
        ++n_unit;
      }
    }
  } else if (warp < 8) {
    // ======================================================================= split / softmax
    // Two groups of four warps: group g takes the tiles of parity g with its own running maximum,
    // row sums and O^T; the unit's two partial states are merged in the epilogue.
    const int g = warp >> 2, w = warp & 3;
    const int gtid = tid & 127;            // TMEM lane = head dim of this thread
    const int gbar = 1 + g;                // the group's named barrier
    float* alpha_s = reinterpret_cast<float*>(smem + Smem::alpha) + g * kN;
    float* fac_s = reinterpret_cast<float*>(smem + Smem::fac);    // [2][64]
    float* lse_s = reinterpret_cast<float*>(smem + Smem::lse);
    float* lsum_s = reinterpret_cast<float*>(smem + Smem::lsum);  // [2][64]
    float* msum_s = reinterpret_cast<float*>(smem + Smem::msum);  // [2][64]
    float* qscale_s = reinterpret_cast<float*>(smem + Smem::qscale);
    const uint32_t lane_base = (uint32_t)(w * 32) << 16;
    const int hh = lane >> 4;              // which head of the warp's pair
    const int head = 2 * w + hh;           // this thread's (head, token) row
    const int tok = lane & 15;
    int n_tile = 0, n_unit = 0, pv_seen = g;  // next tile of this group whose PV completion is unseen
    bool ok = true;
    auto consume_pv = [&](int upto) {
      for (; pv_seen <= upto; pv_seen += 2)
        ok = tc::mbar_wait(ofull_bar(pv_seen & 3), (pv_seen >> 2) & 1, abort_flag, a.status) && ok;
      tc::tc_fence_after();
    };
    // ---- query split of the nu-th unit with tiles: threads 4 qr .. 4 qr + 3 take query row qr, 32
    // dims each; row scale 2^e puts the row's largest |q| in [128, 256).  Needs the unit's query
    // copy (qfull) and, after the first unit, the previous unit's last QK done (qempty); qscale
    // (one array per unit parity) is read after the next 256-thread barrier.
    auto split_query = [&](int nu) {
      ok = tc::mbar_wait(qfull_bar(), nu & 1, abort_flag, a.status) && ok;
      if (nu >= 1) ok = tc::mbar_wait(qempty_bar(), (nu - 1) & 1, abort_flag, a.status) && ok;
      const int qr = tid >> 2, qq = tid & 3, rgn = qq >> 1, c0 = (qq & 1) * 4;
      const uint8_t* src = smem + Smem::qstage + rgn * kQRegion + qr * 128;
      uint4 v[4];
      float mx = 0.f;
#pragma unroll
      for (int c = 0; c < 4; ++c) {  // logical 16-byte chunk c0 + c of the region row (8 bf16 dims)
        v[c] = *reinterpret_cast<const uint4*>(src + ((((c0 + c) ^ (qr & 7)) & 7) << 4));
        const uint32_t wv[4] = {v[c].x, v[c].y, v[c].z, v[c].w};
#pragma unroll
        for (int i = 0; i < 4; ++i)
          mx = fmaxf(mx, fmaxf(fabsf(__uint_as_float(wv[i] << 16)), fabsf(__uint_as_float(wv[i] & 0xffff0000u))));
      }
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
      // e with mx * 2^e in [128, 256), from the exponent field of mx; clamped so that 2^e and 2^-e
      // are normal floats (a row of bf16 subnormals keeps e = 126 and splits to zeros)
      const int ex = mx > 0.f ? max(-126, min(126, 134 - (int)((__float_as_uint(mx) >> 23) & 0xff))) : 0;
      const float sc = __uint_as_float((uint32_t)(127 + ex) << 23);  // 2^ex
      uint8_t* hi_row = smem + Smem::qops + qr * 128;
      uint8_t* lo_row = hi_row + kN * 128;
#pragma unroll
      for (int c = 0; c < 4; c += 2) {  // two chunks (16 dims) -> 16 hi bytes + 16 lo bytes
        uint32_t hw[4], lw[4];
        const uint32_t w0[8] = {v[c].x, v[c].y, v[c].z, v[c].w, v[c + 1].x, v[c + 1].y, v[c + 1].z, v[c + 1].w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          uint32_t h0, l0, h1, l1;
          split2(__uint_as_float(w0[2 * i] << 16) * sc, __uint_as_float(w0[2 * i] & 0xffff0000u) * sc, h0, l0);
          split2(__uint_as_float(w0[2 * i + 1] << 16) * sc, __uint_as_float(w0[2 * i + 1] & 0xffff0000u) * sc, h1,
                 l1);
          hw[i] = (h0 & 0xffffu) | (h1 << 16);
          lw[i] = (l0 & 0xffffu) | (l1 << 16);
        }
        const int ch = rgn * 4 + ((c0 + c) >> 1);  // 16-byte chunk of the 128-byte e4m3 row
        const uint32_t off = (uint32_t)(((ch ^ (qr & 7)) & 7) << 4);
        *reinterpret_cast<uint4*>(hi_row + off) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
        *reinterpret_cast<uint4*>(lo_row + off) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
      }
      if (qq == 0) qscale_s[(nu & 1) * kN + qr] = __uint_as_float((uint32_t)(127 - ex) << 23);  // 2^-ex
      tc::fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(qready_bar());
    };
    // the first unit's query is split up front; every later one at the end of the previous unit's
    // tile loop, so its QKs start while that unit's last PV and epilogue are still running
    if (next_with_tiles(u_begin) < u_end) split_query(0);
    tc::named_bar_sync(3, 256);
    for (int u = u_begin; u < u_end && ok; ++u) {
      const WUnit8 x = unit(u);
      const int rows = x.q_count * G;      // valid columns per KV head
      if (x.ntiles == 0) {
        if (g == 0) {
          for (int n = 0; n < kN; ++n) {
            if ((n & 7) >= rows) continue;
            int qi, hq;
            column_row8<G>(n, qi, hq);
            if (x.part_row < 0) {
              store_out(reinterpret_cast<OutT*>(a.o) + ((int64_t)(x.q_start + qi) * a.hq + hq) * kD + gtid, 0.f);
              if (a.lse != nullptr && gtid == 0) a.lse[(int64_t)(x.q_start + qi) * a.hq + hq] = -INFINITY;
            } else {
              const int64_t prow = (int64_t)x.part_row + (int64_t)qi * x.part_stride;
              a.o_part[(prow * a.hq + hq) * kD + gtid] = 0.f;
              if (gtid == 0) a.lse_part[prow * a.hq + hq] = -INFINITY;
            }
          }
        }
        continue;
      }
      float colscale[8];
#pragma unroll
      for (int c = 0; c < 8; ++c) colscale[c] = a.scale_log2 * qscale_s[(n_unit & 1) * kN + head * 8 + c];
      const int ob = n_unit & 1;
      const uint32_t o_cols = tm_o + (2 * ob + g) * kN;
      float m[8], l[8];
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        m[c] = -INFINITY;
        l[c] = 0.f;
      }
      bool failed = false;
      const int j_first = (n_tile & 1) ^ g;  // the unit's first tile of parity g
      int jg = 0;                            // tiles of this group done in the unit
      for (int j = j_first; j < x.ntiles; j += 2, ++jg) {
        const int t = n_tile + j, st = t % kStages;
        ok = tc::mbar_wait(sfull_bar(g), (t >> 1) & 1, abort_flag, a.status) && ok;
        tc::tc_fence_after();
        float s16[16];
        tc::tmem_ld_x16(tm_s + lane_base + g * kN + 16 * w, s16);
        tc::tmem_wait_ld();
        tc::tc_fence_before();
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(sempty_bar(g));
        const bool valid = x.t0 + j * kTok + tok < x.t1;
        float s[8];
        bool raise = false;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const float v = hh ? s16[8 + c] : s16[c];
          s[c] = (valid && c < rows) ? v * colscale[c] : -INFINITY;
          raise |= s[c] > m[c] + kRaise;
        }
        if (tc::bar_or(gbar, 128, raise || !ok || jg == 0)) {
          if (!tc::bar_and(gbar, 128, ok)) {
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
          if (jg > 0) {
            if (tok == 0) {
#pragma unroll
              for (int c = 0; c < 8; ++c) alpha_s[head * 8 + c] = al[c];
            }
            tc::named_bar_sync(gbar, 128);
            consume_pv(t - 2);  // the group's previous PV has landed in its O^T
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
        // P(t) overwrites the buffer PV(t-4) read: consume that completion first
        if (t >= 4 && pv_seen <= t - 4) consume_pv(t - 4);
        // P buffer t & 3 = bytes 64 ((t >> 1) & 1) .. + 64 of group g's rows; pair w, rows hh*8 + c,
        // token byte `lane` (hi) and 32 + lane (lo)
        uint8_t* pb = smem + Smem::p + g * kPBytes + w * kPairBytes;
        const int half = ((t >> 1) & 1) * 64;
#pragma unroll
        for (int c = 0; c < 8; c += 2) {
          const float p0 = (s[c] == -INFINITY) ? 0.f : ex2(s[c] - m[c] + kPShift);
          const float p1 = (s[c + 1] == -INFINITY) ? 0.f : ex2(s[c + 1] - m[c + 1] + kPShift);
          l[c] += p0;
          l[c + 1] += p1;
          uint32_t hi, lo;
          split2(p0, p1, hi, lo);
          const int r0 = hh * 8 + c;
          pb[sw128_byte(r0, half + lane)] = (uint8_t)(hi & 0xff);
          pb[sw128_byte(r0 + 1, half + lane)] = (uint8_t)((hi >> 8) & 0xff);
          pb[sw128_byte(r0, half + 32 + lane)] = (uint8_t)(lo & 0xff);
          pb[sw128_byte(r0 + 1, half + 32 + lane)] = (uint8_t)((lo >> 8) & 0xff);
        }
        if (!valid) {  // zero this row's V before the PV MMA reads it
          uint8_t* vrow = smem + Smem::kv + st * kStageBytes + kKBytes + gtid * 128;
#pragma unroll
          for (int i = 0; i < 8; ++i) reinterpret_cast<uint4*>(vrow)[i] = make_uint4(0, 0, 0, 0);
        }
        tc::fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(pfull_bar(t & 3));
      }
      if (!failed && next_with_tiles(u + 1) < u_end) split_query(n_unit + 1);
      // the group's last tile of the unit, if it had any
      const int n_own = (x.ntiles - j_first + 1) >> 1;
      if (!failed && n_own > 0) consume_pv(n_tile + j_first + 2 * (n_own - 1));
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        float v = l[c];
#pragma unroll
        for (int o = 8; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        if (tok == 0) {
          lsum_s[g * kN + head * 8 + c] = v;
          msum_s[g * kN + head * 8 + c] = m[c];
        }
      }
      n_tile += x.ntiles;
      ++n_unit;
      tc::tc_fence_before();
      if (!tc::bar_and(3, 256, ok && !failed)) {  // both groups leave together
        ok = false;
        break;
      }
      tc::tc_fence_after();  // the other group's last PV has landed in its O^T
      // ---- epilogue: group g writes columns 32 g .. 32 g + 31 of both groups' O^T, merged:
      // O = (2^(m0 - m) O_0 + 2^(m1 - m) O_1) * kv_scale / (2^(m0 - m) l_0 + 2^(m1 - m) l_1)
      if (tid < kN) {
        const float m0 = msum_s[tid], m1 = msum_s[kN + tid], mm = fmaxf(m0, m1);
        // a group with no tile (or only masked scores) has m = -inf: weight 0, its O^T never read
        const float f0 = m0 == -INFINITY ? 0.f : exp2f(m0 - mm);
        const float f1 = m1 == -INFINITY ? 0.f : exp2f(m1 - mm);
        const float lt = lsum_s[tid] * f0 + lsum_s[kN + tid] * f1;
        const float inv = lt > 0.f ? a.kv_scale / lt : 0.f;
        fac_s[tid] = f0 * inv;
        fac_s[kN + tid] = f1 * inv;
        lse_s[tid] = lt > 0.f ? (mm - kPShift + log2f(lt)) * kLn2 : -INFINITY;
      }
      tc::named_bar_sync(3, 256);
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        float o0[16], o1[16];
        tc::tmem_ld_x16(tm_o + (2 * ob) * kN + lane_base + 32 * g + 16 * h, o0);
        tc::tmem_ld_x16(tm_o + (2 * ob + 1) * kN + lane_base + 32 * g + 16 * h, o1);
        tc::tmem_wait_ld();
        if (h == 1) {
          tc::tc_fence_before();
          __syncwarp();
          if (lane == 0) tc::mbar_arrive(ofree_bar(ob));
        }
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const int n = 32 * g + 16 * h + i;
          if ((n & 7) >= rows) continue;
          const float F0 = fac_s[n], F1 = fac_s[kN + n];
          const float val = (F0 != 0.f ? o0[i] * F0 : 0.f) + (F1 != 0.f ? o1[i] * F1 : 0.f);
          int qi, hq;
          column_row8<G>(n, qi, hq);
          if (x.part_row < 0) {
            store_out(reinterpret_cast<OutT*>(a.o) + ((int64_t)(x.q_start + qi) * a.hq + hq) * kD + gtid, val);
          } else {
            const int64_t prow = (int64_t)x.part_row + (int64_t)qi * x.part_stride;
            a.o_part[(prow * a.hq + hq) * kD + gtid] = val;
          }
        }
      }
      if (tid < kN && (tid & 7) < rows) {
        int qi, hq;
        column_row8<G>(tid, qi, hq);
        if (x.part_row < 0) {
          if (a.lse != nullptr) a.lse[(int64_t)(x.q_start + qi) * a.hq + hq] = lse_s[tid];
        } else {
          a.lse_part[((int64_t)x.part_row + (int64_t)qi * x.part_stride) * a.hq + hq] = lse_s[tid];
        }
      }
      // fac / lse / lsum / msum / qscale are rewritten only after a later 256-thread barrier, alpha
      // after the group's next barrier
    }
  }

  tc::tc_fence_before();
  __syncthreads();
  if (warp == kWarpQK) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, kTmemCols);
  }
}

// ------------------------------------------------------------------------------ host side
PFN_cuTensorMapEncodeTiled_v12000 encode_fn_w8() {
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

bool make_map_w8(CUtensorMap* m, CUtensorMapDataType type, const void* base, const cuuint64_t* dims,
                 const cuuint64_t* strides_bytes, const cuuint32_t* box) {
  auto fn = encode_fn_w8();
  if (fn == nullptr) return false;
  cuuint32_t estr[4] = {1, 1, 1, 1};
  return fn(m, type, 4, const_cast<void*>(base), dims, strides_bytes, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int G, typename OutT>
int launch_w8(const CUtensorMap& km, const CUtensorMap& vm, const CUtensorMap& qm, const W8Args& a,
              const WorkItem* work, cudaStream_t s) {
  const int smem = Smem::total + 1024;
  static DeviceSmemAttr attr;  // per device: the attribute belongs to the current device
  if (const int e = attr.ensure(reinterpret_cast<const void*>(gqa_tc_wide_fp8_kernel<G, OutT>), smem)) return e;
  gqa_tc_wide_fp8_kernel<G, OutT><<<a.num_ctas, kThreads, smem, s>>>(km, vm, qm, a, work);
  return (int)cudaGetLastError();
}

template <typename OutT>
int launch_w8_g(int g, const CUtensorMap& km, const CUtensorMap& vm, const CUtensorMap& qm, const W8Args& a,
                const WorkItem* work, cudaStream_t s) {
  switch (g) {
    case 8: return launch_w8<8, OutT>(km, vm, qm, a, work, s);
    case 4: return launch_w8<4, OutT>(km, vm, qm, a, work, s);
    case 2: return launch_w8<2, OutT>(km, vm, qm, a, work, s);
    case 1: return launch_w8<1, OutT>(km, vm, qm, a, work, s);
    default: return (int)cudaErrorInvalidValue;
  }
}

}  // namespace

int launch_gqa_tc_wide_fp8(const skv_paged_params& p, const WorkItem* work, const int32_t* cta_indptr, int num_ctas,
                           int q_tile, cudaStream_t s) {
  if (num_ctas == 0) return 0;
  const int g = p.num_qo_heads / p.num_kv_heads;
  if (!gqa_tc_wide_supported(p.head_dim, p.page_size, p.num_kv_heads, g, q_tile)) return (int)cudaErrorInvalidValue;
  CUtensorMap km, vm, qm;
  {
    // e4m3 codes as bytes, dimension order (d, slot, head, page): a box of 16 slots x 8 heads
    // lands head-major, one 128-byte row per (head, slot)
    const cuuint64_t dims[4] = {(cuuint64_t)kD, (cuuint64_t)p.page_size, (cuuint64_t)kHk,
                                (cuuint64_t)std::max(1, p.num_pages)};
    const cuuint32_t box[4] = {(cuuint32_t)kD, (cuuint32_t)kTok, (cuuint32_t)kHk, 1};
    const cuuint64_t ks[3] = {(cuuint64_t)p.k_stride[1], (cuuint64_t)p.k_stride[2], (cuuint64_t)p.k_stride[0]};
    const cuuint64_t vs[3] = {(cuuint64_t)p.v_stride[1], (cuuint64_t)p.v_stride[2], (cuuint64_t)p.v_stride[0]};
    if (!make_map_w8(&km, CU_TENSOR_MAP_DATA_TYPE_UINT8, p.k_cache, dims, ks, box)) return (int)cudaErrorInvalidValue;
    if (!make_map_w8(&vm, CU_TENSOR_MAP_DATA_TYPE_UINT8, p.v_cache, dims, vs, box)) return (int)cudaErrorInvalidValue;
  }
  {
    // q (bf16) viewed as (d, j < g, token, kv head): a box (64, g, q_tile, 8) lands as rows
    // kv_head * (q_tile * g) + token * g + j, the column order of S^T
    const cuuint64_t dims[4] = {(cuuint64_t)kD, (cuuint64_t)g, (cuuint64_t)std::max(1, p.total_q), (cuuint64_t)kHk};
    const cuuint64_t st[3] = {(cuuint64_t)kD * 2, (cuuint64_t)p.num_qo_heads * kD * 2, (cuuint64_t)g * kD * 2};
    const cuuint32_t box[4] = {64, (cuuint32_t)g, (cuuint32_t)q_tile, (cuuint32_t)kHk};
    if (!make_map_w8(&qm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, p.q, dims, st, box)) return (int)cudaErrorInvalidValue;
  }
  W8Args a;
  a.kv_indptr = p.kv_indptr;
  a.kv_indices = p.kv_indices;
  a.last = p.kv_last_page_len;
  a.num_pages = p.num_pages;
  a.page_size = p.page_size;
  a.hq = p.num_qo_heads;
  a.q_tile = q_tile;
  a.num_ctas = num_ctas;
  a.cta_indptr = cta_indptr;
  a.scale_log2 = p.sm_scale * p.kv_scale * kLog2e;
  a.kv_scale = p.kv_scale;
  a.o = p.o;
  a.lse = p.lse;
  a.o_part = p.o_part;
  a.lse_part = p.lse_part;
  a.status = p.status;
  return p.o_dtype == SKV_BF16 ? launch_w8_g<__nv_bfloat16>(g, km, vm, qm, a, work, s)
                               : launch_w8_g<float>(g, km, vm, qm, a, work, s);
}

}  // namespace skv
