// MLA latent decode on the tensor cores for an fp8 (e4m3) latent cache.
//
// What it computes (FlashInfer PR #3309 page, MLA decode; the e4m3 cache of the same page):
// every head reads one latent row per token, a 512-d compressed KV (ckv) and a 64-d rope key
// (kpe), both stored as e4m3 with one per-tensor scale; s = sm_scale * kv_scale *
// (q_nope . ckv + q_pe . kpe), V = kv_scale * ckv.  The e4m3 values are decoded exactly.
// seqlen_q is folded into the row dimension as in the bf16 kernel: rows n = qi * Hc + h of a
// unit, Hc = min(H, NR), F = q_tile tokens with F * Hc <= NR; H > NR runs H / NR head groups.
//
// B200 design.  The MMAs run in kind::f16 with f16 operands: every e4m3 value is an f16
// normal (or zero), so cvt.rn.f16x2.e4m3x2 is exact and no scale touches the cache.  Queries
// are converted to f16 once per unit after a power-of-two shift 2^-k chosen from the unit's
// largest |q| (k = 0 unless |q| >= 2^15), and 2^k goes back into the softmax scale: exact for
// every query value of f16 normal magnitude.  P is written as f16.
//   * Converter warps (8) stream the cache with coalesced 16-byte loads (one 512-byte ckv row
//     per warp instruction), two tiles ahead in registers, convert and store f16 straight into
//     the swizzled K-major layout the MMAs read: no raw fp8 staging in shared memory, so the
//     per-tile shared-memory traffic stays at the converted tile plus the MMA operand reads.
//     Rows past the end of the unit are stored as zeros (finite V rows, masked scores).
//   * Converted tiles (64 tokens: four 16 KB ckv blocks + one 8 KB kpe block) sit in two slots,
//     held from QK to PV; PV's completion frees the slot.
//   * S^T[64 tokens, NR] = C . Q^T (M = 64: TMEM rows in lanes 0-15 of each warp quarter) and
//     O^T[512, NR] += V^T . P^T (four M = 128 blocks), online softmax with a lazily raised
//     maximum and O^T rescaled in TMEM on a raise -- as in the bf16 kernel.
// Roles: warps 0-3 softmax / query conversion / epilogue, warp 4 query TMA, warp 5 TMEM + QK
// MMA issue, warp 6 PV MMA issue, warps 7-14 cache conversion.  All waits are bounded.
#include <cudaTypedefs.h>
#include <cuda_fp16.h>

#include <algorithm>
#include <climits>
#include <mutex>

#include "tc_ptx.cuh"

namespace skv {

namespace {

constexpr int kTile = 64;                       // tokens per tile
constexpr int kHalf = kTile * 128;              // one 64-column swizzled region: 8 KB
constexpr int kCSlot = 2 * kHalf;               // one 128-dim ckv block of a tile: 16 KB
constexpr int kTileBytes = 4 * kCSlot + kHalf;  // ckv blocks + kpe block: 72 KB
constexpr int kSlots = 2;
constexpr int kBlocks = 4;
constexpr int kConvWarps = 8;
constexpr int kIssuers = 4;                     // MMA issuing warps 4-7, one per SM sub-partition
constexpr int kFirstConv = 4 + kIssuers;
constexpr int kThreads = (kFirstConv + kConvWarps) * 32;
constexpr float kRaise = 8.f;
constexpr int kNoRows = INT_MIN;                // page id placeholder: the warp has no rows in the tile

template <int NR>
struct Cfg8 {
  static constexpr int tiles = 0;
  static constexpr int kQRegion = NR * 128;
  static constexpr int kQBytes = 9 * kQRegion;
  static constexpr int kPBytes = NR * 128;
  static constexpr int q = tiles + kSlots * kTileBytes;
  static constexpr int p = q + kQBytes;
  static constexpr int red = p + 2 * kPBytes;   // [4][NR] float
  static constexpr int alpha = red + 4 * NR * 4;
  static constexpr int inv = alpha + NR * 4;
  static constexpr int lse = inv + NR * 4;
  static constexpr int qmax = lse + NR * 4;     // [4] float
  static constexpr int mrow = qmax + 16;        // [NR] float: running maximum of every row
  static constexpr int bars = mrow + NR * 4;
  static constexpr int nbars = 2 * kSlots + 11;
  static constexpr int misc = bars + nbars * 8;
  static constexpr int total = misc + 16;
  // S: 2 buffers x 4 partial accumulators (one per issuer) x NR; O^T: 4 blocks x NR
  static constexpr int s_cols = 2 * kIssuers * NR;
  static constexpr int tmem_cols = s_cols + 4 * NR <= 256 ? 256 : 512;
};

struct M8Args {
  const uint8_t* ckv;
  const uint8_t* kpe;
  int64_t cs0, cs1, ks0, ks1;                   // strides in bytes
  const int32_t* kv_indptr;
  const int32_t* kv_indices;
  const int32_t* last;
  const int32_t* cta_indptr;
  int num_pages, page_size, heads, hc, hg, q_tile;
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

__device__ __forceinline__ MUnit8 load_unit8(const M8Args& a, const WorkItem* work, int u) {
  MUnit8 x;
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

// Position in the CTA's sequence of tiles: unit u, head group hgi, tile t (units without
// tokens are skipped; every head group streams the unit's tiles again).
struct Cursor {
  int u, hgi, t, T, t0, t1;
  const int32_t* ids;
  bool done;
};

__device__ __forceinline__ void cursor_seek(Cursor& c, const M8Args& a, const WorkItem* work, int u_end) {
  for (; c.u < u_end; ++c.u) {
    const MUnit8 x = load_unit8(a, work, c.u);
    if (x.ntiles > 0) {
      c.T = x.ntiles;
      c.t0 = x.t0;
      c.t1 = x.t1;
      c.ids = a.kv_indices + a.kv_indptr[x.r];
      return;
    }
  }
  c.done = true;
}
__device__ __forceinline__ void cursor_next(Cursor& c, const M8Args& a, const WorkItem* work, int u_end) {
  if (c.done) return;
  if (++c.t < c.T) return;
  c.t = 0;
  if (++c.hgi < a.hg) return;
  c.hgi = 0;
  ++c.u;
  cursor_seek(c, a, work, u_end);
}

__device__ __forceinline__ uint4 ldg_stream(const uint8_t* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.L2::256B.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint32_t two_bytes) {
  uint32_t r;
  const uint16_t v = (uint16_t)two_bytes;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(r) : "h"(v));
  return r;
}

// 16 e4m3 values (bytes in memory order) -> 16 f16 in two 16-byte chunks (dims 0-7, 8-15)
__device__ __forceinline__ void cvt16(const uint4& v, uint4& lo, uint4& hi) {
  lo.x = e4m3x2_to_f16x2(v.x & 0xffffu);
  lo.y = e4m3x2_to_f16x2(v.x >> 16);
  lo.z = e4m3x2_to_f16x2(v.y & 0xffffu);
  lo.w = e4m3x2_to_f16x2(v.y >> 16);
  hi.x = e4m3x2_to_f16x2(v.z & 0xffffu);
  hi.y = e4m3x2_to_f16x2(v.z >> 16);
  hi.z = e4m3x2_to_f16x2(v.w & 0xffffu);
  hi.w = e4m3x2_to_f16x2(v.w >> 16);
}

// maximum over the warp (sm_100 redux on f32)
__device__ __forceinline__ float redux_max(float v) {
  float r;
  asm volatile("redux.sync.max.f32 %0, %1, 0xffffffff;" : "=f"(r) : "f"(v));
  return r;
}

// kind::f16 instruction descriptor with f16 A and B, f32 D
__host__ __device__ constexpr uint32_t idesc_f16_f32(int M, int N, bool a_mn, bool b_mn) {
  return (1u << 4) | ((a_mn ? 1u : 0u) << 15) | ((b_mn ? 1u : 0u) << 16) | ((uint32_t)(N >> 3) << 17) |
         ((uint32_t)(M >> 4) << 24);
}

template <int NR, typename OutT>
__global__ void __launch_bounds__(kThreads, 1)
mla_tc_fp8_kernel(const __grid_constant__ CUtensorMap qn_map, const __grid_constant__ CUtensorMap qp_map, M8Args a,
                  const WorkItem* __restrict__ work) {
  using C = Cfg8<NR>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = tc::smem_u32(smem);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + C::misc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::misc + 4);
  const uint32_t bar0 = sbase + C::bars;
  auto tfull_bar = [&](int s) { return bar0 + 8u * s; };
  auto tempty_bar = [&](int s) { return bar0 + 8u * (kSlots + s); };
  const uint32_t bar1 = bar0 + 8u * (2 * kSlots);
  auto qfull_bar = [&]() { return bar1; };
  auto qready_bar = [&]() { return bar1 + 8u; };
  auto sfull_bar = [&](int b) { return bar1 + 8u * (2 + b); };
  auto sempty_bar = [&](int b) { return bar1 + 8u * (4 + b); };
  auto pfull_bar = [&](int b) { return bar1 + 8u * (6 + b); };
  auto ofull_bar = [&](int b) { return bar1 + 8u * (8 + b); };
  auto ofree_bar = [&]() { return bar1 + 8u * 10; };
  static_assert(C::total + 1024 <= 232448, "fits the 227 KB opt-in shared memory");

  if (tid == 0) {
    for (int s = 0; s < kSlots; ++s) {
      tc::mbar_init(tfull_bar(s), kConvWarps);
      tc::mbar_init(tempty_bar(s), kIssuers);
    }
    tc::mbar_init(qfull_bar(), 1);
    tc::mbar_init(qready_bar(), 4);
    for (int b = 0; b < 2; ++b) {
      tc::mbar_init(sfull_bar(b), kIssuers);
      tc::mbar_init(sempty_bar(b), 4);
      tc::mbar_init(pfull_bar(b), 4);
      tc::mbar_init(ofull_bar(b), kIssuers);
    }
    tc::mbar_init(ofree_bar(), 4);
    *abort_flag = 0;
    tc::fence_mbar_init();
  }
  if (tid == 0) {
    tc::prefetch_tmap(&qn_map);
    tc::prefetch_tmap(&qp_map);
  }
  if (warp == 5) tc::tmem_alloc(tc::smem_u32(tmem_holder), C::tmem_cols);
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  const uint32_t tm_s = tmem, tm_o = tmem + C::s_cols;

  const int u_begin = a.cta_indptr[blockIdx.x], u_end = a.cta_indptr[blockIdx.x + 1];

  if (warp >= kFirstConv) {
    // ======================================================================= cache conversion
    const int cw = warp - kFirstConv;  // this warp's rows of every tile: tokens 8cw .. 8cw + 7
    const int P = a.page_size;
    bool ok = true;
    Cursor cf{u_begin, 0, 0, 0, 0, 0, nullptr, false};  // the next tile to fetch
    cursor_seek(cf, a, work, u_end);
    // page id of this warp's 8 rows of a tile (8 | P and tiles start on page starts: one page)
    auto load_id = [&](const Cursor& c) -> int {
      if (c.done) return kNoRows;
      const int tok = c.t0 + c.t * kTile + 8 * cw;
      return tok < c.t1 ? __ldg(c.ids + tok / P) : kNoRows;
    };
    // issue the loads of tile cf into D (zeros for rows past the unit's end), then advance cf
    // and start the page-id load of the tile after it
    int idf = load_id(cf);
    auto fetch = [&](uint4 (&D)[9]) -> bool {
      if (cf.done) return false;
      const int page = idf;
      const int tok = cf.t0 + cf.t * kTile + 8 * cw;
      const int n = page == kNoRows ? 0 : min(8, cf.t1 - tok);
      const bool oob = n > 0 && (unsigned)page >= (unsigned)a.num_pages;
      if (oob && lane == 0) report(a.status, SKV_DEV_PAGE_OOB);
      const int nv = oob ? 0 : n;
      const int slot = nv > 0 ? tok % P : 0;
      const uint8_t* cb = a.ckv + (int64_t)(nv > 0 ? page : 0) * a.cs0 + (int64_t)slot * a.cs1 + lane * 16;
#pragma unroll
      for (int j = 0; j < 8; ++j) D[j] = j < nv ? ldg_stream(cb + (int64_t)j * a.cs1) : make_uint4(0, 0, 0, 0);
      const int jk = lane >> 2;
      D[8] = jk < nv ? ldg_stream(a.kpe + (int64_t)page * a.ks0 + (int64_t)(slot + jk) * a.ks1 + (lane & 3) * 16)
                     : make_uint4(0, 0, 0, 0);
      cursor_next(cf, a, work, u_end);
      idf = load_id(cf);
      return true;
    };
    // store one tile's rows of this warp as f16 in the K-major 128-byte-swizzled layout
    auto convert = [&](const uint4 (&D)[9], uint8_t* tile) {
      const int b = lane >> 3, hf = (lane >> 2) & 1, ch = (lane & 3) * 2, sw = (lane >> 2) & 1;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int ti = 8 * cw + j, x = ti & 7;
        uint4 lo, hi;
        cvt16(D[j], lo, hi);
        uint8_t* row = tile + b * kCSlot + hf * kHalf + ti * 128;
        // alternate which chunk goes first between neighbouring lane quads: 4-way banks per store
        *reinterpret_cast<uint4*>(row + (((ch + sw) ^ x) << 4)) = sw ? hi : lo;
        *reinterpret_cast<uint4*>(row + (((ch + 1 - sw) ^ x) << 4)) = sw ? lo : hi;
      }
      {
        const int ti = 8 * cw + (lane >> 2), x = ti & 7, kc = (lane & 3) * 2;
        uint4 lo, hi;
        cvt16(D[8], lo, hi);
        uint8_t* row = tile + 4 * kCSlot + ti * 128;
        *reinterpret_cast<uint4*>(row + ((kc ^ x) << 4)) = lo;
        *reinterpret_cast<uint4*>(row + (((kc + 1) ^ x) << 4)) = hi;
      }
    };
    uint4 DA[9], DB[9];
    bool va = fetch(DA);
    bool vb = fetch(DB);
    int gt = 0;
    // one step: convert the oldest fetched tile (in D), refill D with the next tile
    auto step = [&](uint4 (&D)[9], bool& v) -> bool {
      if (!v || !ok) return false;
      const int slot = gt % kSlots;
      if (gt >= kSlots) {
        if (lane == 0) ok = tc::mbar_wait_sleep(tempty_bar(slot), ((gt / kSlots) + 1) & 1, abort_flag, a.status);
        ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
        if (!ok) return false;
      }
      convert(D, smem + C::tiles + slot * kTileBytes);
      tc::fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(tfull_bar(slot));
      ++gt;
      v = fetch(D);
      return true;
    };
    while (step(DA, va) && step(DB, vb)) {
    }
  } else if (warp >= 4) {
    // ======================================================================= MMA issuers
    // Issuer w: QK quarter w of every tile (rope k-step w + ckv block w: 9 MMAs) into its own
    // partial S^T accumulator, and PV block w (4 MMAs) into O^T block w.  Per tile the order is
    // QK(t) then PV(t - 1), so S(t) is in flight while the softmax finishes P(t - 1).
    if (lane == 0) {
      const int w = warp - 4;
      constexpr uint32_t idesc_s = idesc_f16_f32(64, NR, false, false);
      constexpr uint32_t idesc_o = idesc_f16_f32(128, NR, true, false);
      int gt = 0, n_unit = 0, n_tile = 0;
      bool ok = true;
      const uint32_t qs = sbase + C::q;
      for (int u = u_begin; u < u_end && ok; ++u) {
        const MUnit8 x = load_unit8(a, work, u);
        if (x.ntiles == 0) continue;
        for (int hgi = 0; hgi < a.hg && ok; ++hgi) {
          const int T = x.ntiles;
          ok = tc::mbar_wait_sleep(qready_bar(), n_unit & 1, abort_flag, a.status);
          if (ok) tc::tc_fence_after();
          // issue whichever is ready: PV(pv) (frees the tile slot: first) or QK(qk)
          int qk = 0, pv = 0;
          tc::PollClock clk;
          while (ok && pv < T) {
            bool did = false;
            if (pv < qk) {  // ---- PV(pv), block w
              const int tp = n_tile + pv, pb = tp & 1, g = gt + pv, slot = g % kSlots;
              // the single O^T buffer was read by the previous unit's epilogue
              if (tc::mbar_test_wait(pfull_bar(pb), (tp >> 1) & 1) &&
                  (pv > 0 || n_unit == 0 || tc::mbar_test_wait(ofree_bar(), (n_unit + 1) & 1))) {
                tc::tc_fence_after();
                const uint32_t ps = sbase + C::p + pb * C::kPBytes;
                const uint32_t vs = sbase + C::tiles + slot * kTileBytes + w * kCSlot;
#pragma unroll
                for (int k = 0; k < kTile / 16; ++k) {
                  const uint64_t ad = tc::sdesc_sw128(vs + k * 2048, kHalf, 1024);
                  const uint64_t bd = tc::sdesc_sw128(ps + k * 32, 16, 1024);
                  tc::mma_bf16(tm_o + w * NR, ad, bd, idesc_o, (pv > 0 || k > 0) ? 1u : 0u);
                }
                tc::mma_commit(tempty_bar(slot));
                tc::mma_commit(ofull_bar(pb));
                ++pv;
                did = true;
              }
            }
            if (!did && qk < T) {  // ---- QK(qk), quarter w
              const int tt = n_tile + qk, sb = tt & 1, g = gt + qk, slot = g % kSlots;
              if ((tt < 2 || tc::mbar_test_wait(sempty_bar(sb), ((tt >> 1) + 1) & 1)) &&
                  tc::mbar_test_wait(tfull_bar(slot), (g / kSlots) & 1)) {
                tc::tc_fence_after();
                const uint32_t tb = sbase + C::tiles + slot * kTileBytes;
                const uint32_t d = tm_s + (sb * kIssuers + w) * NR;
                tc::mma_bf16(d, tc::sdesc_sw128(tb + 4 * kCSlot + w * 32, 16, 1024),
                             tc::sdesc_sw128(qs + 8 * C::kQRegion + w * 32, 16, 1024), idesc_s, 0u);
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                  const uint64_t ad = tc::sdesc_sw128(tb + w * kCSlot + (k >> 2) * kHalf + (k & 3) * 32, 16, 1024);
                  const uint64_t bd =
                      tc::sdesc_sw128(qs + (2 * w + (k >> 2)) * C::kQRegion + (k & 3) * 32, 16, 1024);
                  tc::mma_bf16(d, ad, bd, idesc_s, 1u);
                }
                tc::mma_commit(sfull_bar(sb));
                ++qk;
                did = true;
              }
            }
            ok = clk.step(did, abort_flag, a.status);
          }
          gt += T;
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
    float* qmax_s = reinterpret_cast<float*>(smem + C::qmax);
    // the running maxima are the same in every thread: they live in shared memory (registers
    // are scarce with 480 threads)
    float* m_s = reinterpret_cast<float*>(smem + C::mrow);
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
    const bool srow = lane < 16;              // this lane holds an S^T row (M = 64 layout)
    const int tok_in_tile = 16 * warp + (lane & 15);
    int n_unit = 0, n_tile = 0, pv_seen = 0, q_issued = 0, q_landed = 0;
    bool ok = true;
    auto consume_pv = [&](int upto) {
      for (; pv_seen <= upto; ++pv_seen)
        ok = tc::mbar_wait_sleep(ofull_bar(pv_seen & 1), (pv_seen >> 1) & 1, abort_flag, a.status) && ok;
      tc::tc_fence_after();
    };
    for (int u = u_begin; u < u_end && ok; ++u) {
      const MUnit8 x = load_unit8(a, work, u);
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
        // ---- queries of this unit: bf16 (TMA) -> f16 in place, shifted by 2^-k.  The buffer is
        // free: every QK of the previous unit completed before its last S was consumed here.
        const int qrows = a.hc * a.q_tile;     // rows the query copy fills
        if (tid == 0) {
          tc::mbar_arrive_expect_tx(qfull_bar(), (uint32_t)(9 * qrows * 128));
          for (int rg = 0; rg < 8; ++rg)
            tc::tma_load_3d(sbase + C::q + rg * C::kQRegion, &qn_map, qfull_bar(), rg * 64, h0, x.q_start);
          tc::tma_load_3d(sbase + C::q + 8 * C::kQRegion, &qp_map, qfull_bar(), 0, h0, x.q_start);
        }
        q_issued = n_unit + 1;
        ok = tc::mbar_wait_sleep(qfull_bar(), n_unit & 1, abort_flag, a.status) && ok;
        if (ok) q_landed = n_unit + 1;
        constexpr int kChunks = 9 * NR * 8;     // 16-byte chunks of the query block
        float qm = 0.f;
        for (int ci = tid; ci < kChunks; ci += 128) {
          if ((ci % (NR * 8)) / 8 >= qrows) continue;
          const uint4 v = *reinterpret_cast<const uint4*>(smem + C::q + ci * 16);
          const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
          for (int i = 0; i < 4; ++i)
            qm = fmaxf(qm, fmaxf(fabsf(__uint_as_float(w[i] << 16)), fabsf(__uint_as_float(w[i] & 0xffff0000u))));
        }
        qm = warp_max(qm);
        if (lane == 0) qmax_s[warp] = qm;
        if (tid < NR) m_s[tid] = -INFINITY;
        tc::named_bar_sync(1, 128);
        qm = fmaxf(fmaxf(qmax_s[0], qmax_s[1]), fmaxf(qmax_s[2], qmax_s[3]));
        int k_shift = 0;
        if (qm >= 32768.f) k_shift = (qm == qm && qm < INFINITY) ? min(ilogbf(qm) - 14, 200) : 200;
        const float qs_mul = ldexpf(1.f, -k_shift);
        for (int ci = tid; ci < kChunks; ci += 128) {
          if ((ci % (NR * 8)) / 8 >= qrows) continue;
          uint4* pv = reinterpret_cast<uint4*>(smem + C::q + ci * 16);
          const uint4 v = *pv;
          const uint32_t w[4] = {v.x, v.y, v.z, v.w};
          uint32_t o4[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            __half2 h2 = __floats2half2_rn(__uint_as_float(w[i] << 16) * qs_mul,
                                           __uint_as_float(w[i] & 0xffff0000u) * qs_mul);
            o4[i] = *reinterpret_cast<uint32_t*>(&h2);
          }
          *pv = make_uint4(o4[0], o4[1], o4[2], o4[3]);
        }
        tc::fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(qready_bar());
        const float sl2 = ldexpf(a.scale_log2, k_shift);

        const int T = x.ntiles;
        float l[NR];
#pragma unroll
        for (int n = 0; n < NR; ++n) l[n] = 0.f;
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
            for (int n = 0; n < NR; ++n) l[n] *= alpha_s[n];
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
          if (tt >= 2 && pv_seen <= tt - 2) consume_pv(tt - 2);  // P(t) reuses PV(t-2)'s buffer
          if (srow) {
            uint8_t* pb = smem + C::p + (tt & 1) * C::kPBytes;
            float mloc[NR];  // read the maxima before the stores below (they may alias for the compiler)
#pragma unroll
            for (int n = 0; n < NR; ++n) mloc[n] = m_s[n];
#pragma unroll
            for (int n = 0; n < NR; ++n) {
              const float p = (s[n] == -INFINITY) ? 0.f : exp2f(s[n] - mloc[n]);
              l[n] += p;
              if (n < rows) *reinterpret_cast<__half*>(pb + tc::sw128_offset(n, tok_in_tile)) = __float2half_rn(p);
            }
          }
          tc::fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) tc::mbar_arrive(pfull_bar(tt & 1));
        }
        if (failed) {
          ok = false;
          break;
        }
        n_tile += T;
        ++n_unit;
        consume_pv(n_tile - 1);
        // column sums over the 64 token lanes (lanes 16-31 of each warp hold zeros)
#pragma unroll
        for (int n = 0; n < NR; ++n) {
          const float v = warp_sum(l[n]);
          if (lane == 0) red[warp * NR + n] = v;
        }
        if (!tc::bar_and(1, 128, ok)) {
          ok = false;
          break;
        }
        if (tid == 0) {
#pragma unroll
          for (int n = 0; n < NR; ++n) {
            const float lt = red[n] + red[NR + n] + red[2 * NR + n] + red[3 * NR + n];
            inv_s[n] = lt > 0.f ? a.kv_scale / lt : 0.f;
            lse_s[n] = lt > 0.f ? (m_s[n] + log2f(lt)) * kLn2 : -INFINITY;
          }
        }
        tc::named_bar_sync(1, 128);
        // O^T block by block: thread tid holds head dim b * 128 + tid of every row
#pragma unroll 1
        for (int b = 0; b < kBlocks; ++b) {
          float ov[NR];
#pragma unroll
          for (int c = 0; c < NR; c += 16) {
            float v16[16];
            tc::tmem_ld_x16(tm_o + lane_base + b * NR + c, v16);
#pragma unroll
            for (int i = 0; i < 16; ++i) ov[c + i] = v16[i];
          }
          tc::tmem_wait_ld();
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
    if (tid == 0 && q_issued > q_landed) {  // a query copy may still be landing (bounded wait)
      const uint64_t t_start = tc::globaltimer_ns();
      while (!tc::mbar_try_wait(qfull_bar(), (q_issued - 1) & 1) && tc::globaltimer_ns() - t_start < 50000000ull) {
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

bool make_qmap(CUtensorMap* m, const void* base, const cuuint64_t* dims, const cuuint64_t* strides_bytes,
               const cuuint32_t* box) {
  auto fn = encode_fn_m8();
  if (fn == nullptr) return false;
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides_bytes, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int NR, typename OutT>
int launch_m8(const CUtensorMap* maps, const M8Args& a, int num_ctas, const WorkItem* work, cudaStream_t s) {
  const int smem = Cfg8<NR>::total + 1024;
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e =
        cudaFuncSetAttribute(mla_tc_fp8_kernel<NR, OutT>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return (int)e;
    attr_set = true;
  }
  mla_tc_fp8_kernel<NR, OutT><<<num_ctas, kThreads, smem, s>>>(maps[0], maps[1], a, work);
  return (int)cudaGetLastError();
}

}  // namespace

bool mla_tc_fp8_supported(int page_size, int num_heads, int rows_per_unit) {
  return page_size >= 8 && page_size % 8 == 0 && (rows_per_unit == 16 || rows_per_unit == 32) &&
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
  CUtensorMap maps[2];
  {
    const cuuint64_t dims[3] = {512, (cuuint64_t)p.num_heads, (cuuint64_t)std::max(1, total_q)};
    const cuuint64_t st[2] = {512 * 2, (cuuint64_t)p.num_heads * 512 * 2};
    const cuuint32_t box[3] = {64, (cuuint32_t)hc, (cuuint32_t)q_tile};
    if (!make_qmap(&maps[0], p.q_nope, dims, st, box)) return (int)cudaErrorInvalidValue;
  }
  {
    const cuuint64_t dims[3] = {64, (cuuint64_t)p.num_heads, (cuuint64_t)std::max(1, total_q)};
    const cuuint64_t st[2] = {64 * 2, (cuuint64_t)p.num_heads * 64 * 2};
    const cuuint32_t box[3] = {64, (cuuint32_t)hc, (cuuint32_t)q_tile};
    if (!make_qmap(&maps[1], p.q_pe, dims, st, box)) return (int)cudaErrorInvalidValue;
  }
  M8Args a;
  a.ckv = static_cast<const uint8_t*>(p.ckv);
  a.kpe = static_cast<const uint8_t*>(p.kpe);
  a.cs0 = p.ckv_stride[0];
  a.cs1 = p.ckv_stride[1];
  a.ks0 = p.kpe_stride[0];
  a.ks1 = p.kpe_stride[1];
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
