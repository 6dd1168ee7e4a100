// C ABI of libsplitkv: argument validation, the split planner and kernel dispatch.
//
// Host-side dispatch picks the kernel variant (and the SAME_KV_STRIDES specialisation) before
// launch instead of branching inside the kernel (FlashInfer PR #4736 page, conclusion 1
// "host-side dispatch"; section 2 for the specialisation).  Split-KV planning turns each
// request's page list into chunks so every SM has work at small batch; the partials of a split
// request are merged exactly afterwards (route primitive, "Move the Query, Not the Cache").
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstring>
#include <vector>

#include "skv_internal.h"

using namespace skv;

namespace {

constexpr int32_t kVersion = 1;

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

struct ReqShape {
  int32_t q_start, q_len, n_pages;
};

int device_sms(int param) {
  int sms = param;
  if (sms <= 0) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      sms = 148;
    cudaGetLastError();
  }
  return sms;
}

// Persistent-kernel options of the planner: the CTA count the work is balanced over and the
// tokens one kernel tile covers.  flat_ctas == 0: not persistent (one CTA per work item).  For
// persistent kernels `units_per_page` counts how many times a CTA streams each page of a work
// item (MLA head groups), so the slices are balanced in streamed tiles.
struct PersistOpts {
  int32_t flat_ctas = 0;
  int32_t tile_tokens = 128;
  int32_t page_size = 1;
  int32_t piece_cost = 0;  // fixed cost of a work item (query load, pipeline refill, epilogue), in tiles
  // CTAs per KV slice.  With group > 1 the work items cover query tile 0 only and every slice is
  // run by `group` co-resident CTAs, each taking one (query tile, head group) of every item, so
  // the slice streams from HBM about once and the other CTAs read it from L2.  The plan's
  // num_ctas counts all CTAs (slices x group); cta_indptr has one entry per slice.
  int32_t group = 1;
};

// Tiles of logical pages [a, b) of a request of length L (pages of `page_size` tokens).
int64_t range_tiles(int64_t a, int64_t b, int64_t L, int32_t P, int32_t tile) {
  const int64_t t0 = a * P, t1 = std::min<int64_t>(b * P, L);
  return t1 > t0 ? (t1 - t0 + tile - 1) / tile : 0;
}

// Shared planner: work items over (request, query tile, split) and merge items for split rows.
// BALANCED with a persistent kernel cuts the concatenated KV of all requests into flat_ctas
// slices of equal tile count (cuts at page boundaries, no piece below a few tiles), so every CTA
// streams the same amount and requests are split only where a slice boundary falls; the other
// policies hand whole work items to the persistent CTAs longest-first (greedy least-loaded).
skv_status plan_common(int32_t batch, const std::vector<ReqShape>& req, const std::vector<int64_t>& kv_len,
                       int32_t q_tile, int64_t units_per_page, int32_t units_per_sm, int32_t policy, int32_t param,
                       const int32_t* split_indptr_h, const int32_t* split_bounds_h, int32_t kernel,
                       const PersistOpts& po, int32_t* plan_h, int64_t plan_capacity, skv_plan_info* info) {
  if (info == nullptr) return SKV_ERR_INVALID;
  std::memset(info, 0, sizeof(*info));
  if (q_tile < 1) return SKV_ERR_INVALID;
  if (policy == SKV_SPLIT_FIXED) {
    if (param < 1) return SKV_ERR_INVALID;
  } else if (policy == SKV_SPLIT_EXPLICIT) {
    if (split_indptr_h == nullptr || split_bounds_h == nullptr) return SKV_ERR_INVALID;
    if (split_indptr_h[0] != 0) return SKV_ERR_INVALID;
  } else if (policy != SKV_SPLIT_NONE && policy != SKV_SPLIT_BALANCED) {
    return SKV_ERR_INVALID;
  }
  const bool persistent = po.flat_ctas > 0;
  const bool flat = persistent && policy == SKV_SPLIT_BALANCED;
  const int P = po.page_size, T = po.tile_tokens;

  // ---- per-request split boundaries (and, for the flat cut, the CTA of every piece)
  std::vector<std::vector<int32_t>> bounds(batch);
  std::vector<std::vector<int32_t>> piece_cta(batch);
  int64_t chunk = 0;
  if (policy == SKV_SPLIT_BALANCED && !flat) {
    const int sms = device_sms(param);
    int64_t total_units = 0;
    for (const auto& q : req) {
      const int64_t tiles = (q.q_len + q_tile - 1) / q_tile;
      total_units += tiles * q.n_pages * units_per_page;
    }
    // pages per split so that about `units_per_sm` CTA-units land on every SM: a work item of p
    // pages becomes `units_per_page` CTA-units (one per KV head for GQA); never below 8 pages.
    const int64_t target = std::max<int64_t>(1, (int64_t)sms * units_per_sm);
    chunk = std::max<int64_t>(8, (total_units + target - 1) / target);
  }
  if (flat) {
    const int G = po.flat_ctas;
    std::vector<int64_t> w(batch, 0);
    double total = 0, piece_total = 0;
    int64_t nonempty = 0;
    for (int32_t r = 0; r < batch; ++r) {
      const int64_t qt = po.group > 1 ? (req[r].q_len > 0 ? 1 : 0)
                                      : (req[r].q_len + q_tile - 1) / q_tile * units_per_page;
      w[r] = qt * range_tiles(0, req[r].n_pages, kv_len[r], P, T);
      total += (double)w[r];
      if (w[r] > 0) {
        ++nonempty;
        piece_total += (double)po.piece_cost * (double)qt;
      }
    }
    // every piece of request r also costs po.piece_cost tiles per query unit of r: about one
    // piece per request plus one per CTA boundary (charged at the mean)
    if (nonempty > 0) total += piece_total + (double)(G - 1) * piece_total / (double)nonempty;
    const double target = total / G;
    const int64_t min_piece = std::max<int64_t>(1, std::min<int64_t>(4, (int64_t)target));
    int cta = 0;
    double cum = 0;
    for (int32_t r = 0; r < batch; ++r) {
      const int64_t qt = po.group > 1 ? (req[r].q_len > 0 ? 1 : 0)
                                      : (req[r].q_len + q_tile - 1) / q_tile * units_per_page;
      const int32_t n = req[r].n_pages;
      bounds[r].push_back(0);
      if (n == 0 || qt == 0) {  // nothing to stream: one (empty) piece on the current CTA
        bounds[r].push_back(n);
        piece_cta[r].push_back(cta);
        continue;
      }
      int32_t a = 0;
      const double pc = (double)po.piece_cost * (double)qt;
      while (a < n) {
        double room = (cta + 1) * target - cum - pc;
        if (room < (double)min_piece && cta < G - 1) {
          ++cta;
          room = (cta + 1) * target - cum - pc;
        }
        // largest b with work(a, b) <= room (at least one page), or the whole rest
        int32_t b = a + 1;
        if (cta == G - 1) {
          b = n;
        } else {
          // the work of [a, b) grows with b: binary search for the last b that still fits
          int32_t lo = a + 1, hi = n;
          while (lo < hi) {
            const int32_t mid = lo + (hi - lo + 1) / 2;
            if ((double)(qt * range_tiles(a, mid, kv_len[r], P, T)) <= room)
              lo = mid;
            else
              hi = mid - 1;
          }
          b = lo;
          if (qt * range_tiles(b, n, kv_len[r], P, T) < min_piece) b = n;  // no tiny remainder
        }
        const int64_t wt = qt * range_tiles(a, b, kv_len[r], P, T);
        bounds[r].push_back(b);
        piece_cta[r].push_back(cta);
        cum += (double)wt + pc;
        a = b;
        if (cum >= (cta + 1) * target - 0.5 && cta < G - 1) ++cta;
      }
    }
  } else {
    for (int32_t r = 0; r < batch; ++r) {
      const ReqShape& q = req[r];
      int32_t S = 1;
      if (policy == SKV_SPLIT_EXPLICIT) {
        S = split_indptr_h[r + 1] - split_indptr_h[r];
        if (S < 1) return SKV_ERR_INVALID;
        const int32_t* b = split_bounds_h + split_indptr_h[r] + r;
        if (b[0] != 0 || b[S] != q.n_pages) return SKV_ERR_INVALID;
        for (int j = 0; j <= S; ++j) {
          if (j > 0 && b[j] < b[j - 1]) return SKV_ERR_INVALID;
          bounds[r].push_back(b[j]);
        }
      } else {
        if (policy == SKV_SPLIT_FIXED) S = param;
        if (policy == SKV_SPLIT_BALANCED) {
          S = (int32_t)std::max<int64_t>(1, ((int64_t)q.n_pages + chunk - 1) / chunk);
          S = std::min<int32_t>(S, std::max<int32_t>(1, q.n_pages));
        }
        bounds[r].push_back(0);
        for (int j = 0; j < S; ++j) {
          const int32_t rem = q.n_pages - bounds[r].back();
          bounds[r].push_back(bounds[r].back() + (rem + (S - j) - 1) / (S - j));  // ceil first
        }
      }
    }
  }

  // ---- work items, merge items
  std::vector<WorkItem> work;
  std::vector<int32_t> work_cta;
  std::vector<MergeItem> merges;
  int32_t part_base = 0, max_splits = 0, total_splits = 0;
  for (int32_t r = 0; r < batch; ++r) {
    const ReqShape& q = req[r];
    const int32_t S = (int32_t)bounds[r].size() - 1;
    max_splits = std::max(max_splits, S);
    total_splits += S;
    if (q.q_len == 0) continue;
    const int32_t q_items = po.group > 1 ? 1 : q.q_len;  // grouped: query tile 0 stands for all tiles
    for (int32_t q0 = 0; q0 < q_items; q0 += q_tile) {
      const int32_t qc = std::min(q_tile, q.q_len - q0);
      for (int j = 0; j < S; ++j) {
        WorkItem w;
        w.r = r;
        w.q_start = q.q_start + q0;
        w.q_count = qc;
        w.page_begin = bounds[r][j];
        w.page_end = bounds[r][j + 1];
        w.part_row = S > 1 ? part_base + q0 * S + j : -1;
        w.part_stride = S;
        w.split = j;
        work.push_back(w);
        work_cta.push_back(flat ? piece_cta[r][j] : 0);
      }
    }
    if (S > 1) {
      for (int32_t i = 0; i < q.q_len; ++i) merges.push_back(MergeItem{q.q_start + i, part_base + i * S, S, 0});
      part_base += q.q_len * S;
    }
  }
  auto item_tiles = [&](const WorkItem& w) {
    return (int64_t)w.q_count * (1 + range_tiles(w.page_begin, w.page_end, kv_len[w.r], P, T));
  };
  std::vector<int32_t> cta_indptr;
  int32_t num_ctas = 0;
  if (persistent) {
    std::vector<int32_t> order(work.size());
    for (size_t i = 0; i < work.size(); ++i) order[i] = (int32_t)i;
    if (!flat) {
      // longest first onto the least-loaded CTA
      const int G = std::max<int32_t>(1, std::min<int32_t>(po.flat_ctas, (int32_t)work.size()));
      std::stable_sort(order.begin(), order.end(),
                       [&](int32_t x, int32_t y) { return item_tiles(work[x]) > item_tiles(work[y]); });
      std::vector<int64_t> load(G, 0);
      for (int32_t i : order) {
        const int c = (int)(std::min_element(load.begin(), load.end()) - load.begin());
        work_cta[i] = c;
        load[c] += item_tiles(work[i]);
      }
    }
    for (int32_t c : work_cta) num_ctas = std::max(num_ctas, c + 1);
    std::stable_sort(order.begin(), order.end(), [&](int32_t x, int32_t y) { return work_cta[x] < work_cta[y]; });
    std::vector<WorkItem> sorted;
    sorted.reserve(work.size());
    cta_indptr.assign(num_ctas + 1, 0);
    for (int32_t i : order) {
      sorted.push_back(work[i]);
      ++cta_indptr[work_cta[i] + 1];
    }
    for (int c = 0; c < num_ctas; ++c) cta_indptr[c + 1] += cta_indptr[c];
    work.swap(sorted);
  } else {
    // longest items first: the hardware hands out CTAs roughly in index order
    std::stable_sort(work.begin(), work.end(), [](const WorkItem& a, const WorkItem& b) {
      return (a.page_end - a.page_begin) * a.q_count > (b.page_end - b.page_begin) * b.q_count;
    });
  }
  info->num_work = (int32_t)work.size();
  info->num_partial_rows = part_base;
  info->num_merge_rows = (int32_t)merges.size();
  info->kernel = kernel;
  info->q_tile = q_tile;
  info->max_splits = max_splits;
  info->total_splits = total_splits;
  info->num_ctas = num_ctas * std::max<int32_t>(1, po.group);
  const int64_t base_words = plan_words(info->num_work, info->num_merge_rows);
  info->cta_offset = persistent ? (int32_t)base_words : 0;
  const int64_t words = base_words + (persistent ? num_ctas + 1 : 0);
  if (words > INT32_MAX) return SKV_ERR_INVALID;
  info->plan_words = (int32_t)words;
  if (plan_h == nullptr || plan_capacity < words) return SKV_ERR_WORKSPACE;
  if (!work.empty()) std::memcpy(plan_h, work.data(), work.size() * sizeof(WorkItem));
  if (!merges.empty())
    std::memcpy(plan_h + 8 * work.size(), merges.data(), merges.size() * sizeof(MergeItem));
  if (persistent) std::memcpy(plan_h + base_words, cta_indptr.data(), (num_ctas + 1) * sizeof(int32_t));
  return SKV_OK;
}

skv_status check_table_h(int32_t batch, const int32_t* kv_indptr_h, const int32_t* last_h,
                         int32_t page_size, std::vector<ReqShape>& req) {
  if (batch < 0 || page_size < 1 || kv_indptr_h == nullptr || last_h == nullptr) return SKV_ERR_INVALID;
  if (batch > 0 && kv_indptr_h[0] != 0) return SKV_ERR_INVALID;
  req.resize(batch);
  for (int32_t r = 0; r < batch; ++r) {
    const int32_t n = kv_indptr_h[r + 1] - kv_indptr_h[r];
    if (n < 0) return SKV_ERR_INVALID;
    if (n > 0 && (last_h[r] < 1 || last_h[r] > page_size)) return SKV_ERR_INVALID;
    if ((int64_t)n * page_size > INT32_MAX) return SKV_ERR_INVALID;
    req[r].n_pages = n;
  }
  return SKV_OK;
}

skv_status cuda_status(int e) { return e == 0 ? SKV_OK : SKV_ERR_CUDA; }

skv_status check_plan(const int32_t* plan_d, const skv_plan_info* info) {
  if (info == nullptr) return SKV_ERR_INVALID;
  if (info->num_work < 0 || info->num_merge_rows < 0 || info->num_partial_rows < 0) return SKV_ERR_INVALID;
  if (info->num_work > 0 && plan_d == nullptr) return SKV_ERR_INVALID;
  if (info->q_tile < 1) return SKV_ERR_INVALID;
  return SKV_OK;
}

// skv_plan_paged, optionally restricted to the requests marked in `include` (the others get no
// work: no query rows, no pages), so one batch can be planned as several kernel launches.
skv_status plan_paged_impl(int32_t batch, const int32_t* qo_indptr_h, const int32_t* kv_indptr_h,
                           const int32_t* kv_last_page_len_h, int32_t page_size, int32_t num_qo_heads,
                           int32_t num_kv_heads, int32_t head_dim, int32_t policy, int32_t param,
                           const int32_t* split_indptr_h, const int32_t* split_bounds_h,
                           const std::vector<char>* include, int32_t* plan_h, int64_t plan_capacity,
                           skv_plan_info* info) {
  if (info != nullptr) std::memset(info, 0, sizeof(*info));
  if (qo_indptr_h == nullptr || num_qo_heads < 1 || num_kv_heads < 1) return SKV_ERR_INVALID;
  if (num_qo_heads % num_kv_heads != 0) return SKV_ERR_INVALID;
  if (head_dim != 64 && head_dim != 128) return SKV_ERR_UNSUPPORTED;
  std::vector<ReqShape> req;
  skv_status st = check_table_h(batch, kv_indptr_h, kv_last_page_len_h, page_size, req);
  if (st != SKV_OK) return st;
  if (batch > 0 && qo_indptr_h[0] != 0) return SKV_ERR_INVALID;
  for (int32_t r = 0; r < batch; ++r) {
    req[r].q_start = qo_indptr_h[r];
    req[r].q_len = qo_indptr_h[r + 1] - qo_indptr_h[r];
    if (req[r].q_len < 0) return SKV_ERR_INVALID;
    if (include != nullptr && !(*include)[r]) {
      req[r].q_len = 0;
      req[r].n_pages = 0;
    }
  }
  const int32_t g = num_qo_heads / num_kv_heads;
  int32_t max_q = 1;
  for (const auto& q : req) max_q = std::max(max_q, q.q_len);
  // all-KV-heads tensor-core decode when every request's query rows per KV head fit its 8
  // columns (whole pages stream contiguously); else the per-KV-head tensor-core decode; else the
  // generic CUDA-core kernel
  const bool wide = g <= 8 && 8 % g == 0 && max_q * g <= 8 &&
                    gqa_tc_wide_supported(head_dim, page_size, num_kv_heads, g, 8 / g);
  // more query rows per KV head than one 16-column decode tile holds: 128-row prefill tiles
  const bool prefill = !wide && (int64_t)max_q * g > 16 && gqa_tc_prefill_supported(head_dim, page_size, g);
  const int32_t tc_q_tile = std::max<int32_t>(1, std::min<int32_t>(16 / std::max<int32_t>(g, 1), max_q));
  const bool tc = !wide && !prefill && g <= 16 && gqa_tc_decode_supported(head_dim, page_size, g, tc_q_tile);
  const int32_t kernel = wide      ? KERNEL_GQA_TC_WIDE
                         : prefill ? KERNEL_GQA_TC_PREFILL
                         : tc      ? KERNEL_GQA_TC_DECODE
                                   : KERNEL_GQA_SIMT;
  const int32_t q_tile = wide ? 8 / g : prefill ? 128 / g : tc ? tc_q_tile : std::max<int32_t>(1, 16 / g);
  std::vector<int64_t> kv_len(batch);
  for (int32_t r = 0; r < batch; ++r)
    kv_len[r] = req[r].n_pages == 0 ? 0
                                    : (int64_t)(req[r].n_pages - 1) * page_size + kv_last_page_len_h[r];
  PersistOpts po;
  po.page_size = page_size;
  if (wide) {  // persistent all-heads kernel: 16-token tiles, one CTA per SM
    po.flat_ctas = device_sms(policy == SKV_SPLIT_BALANCED ? param : 0);
    po.tile_tokens = 16;
    // measured: a work item's query load, pipeline refill and epilogue cost about three 16-token
    // tiles (a per-CTA trace of the e4m3 kernel put it at ~3 us per work item)
    po.piece_cost = 3;
  }
  // per-KV-head tensor-core kernel: a few large units per SM; CUDA-core kernel: many small CTAs
  return plan_common(batch, req, kv_len, q_tile, wide ? 1 : num_kv_heads, prefill ? 2 : tc ? 6 : 64, policy, param,
                     split_indptr_h, split_bounds_h, kernel, po, plan_h, plan_capacity, info);
}

}  // namespace

extern "C" {

int32_t skv_version(void) { return kVersion; }

const char* skv_status_str(int32_t s) {
  switch (s) {
    case SKV_OK: return "ok";
    case SKV_ERR_INVALID: return "invalid argument";
    case SKV_ERR_UNSUPPORTED: return "unsupported shape or dtype";
    case SKV_ERR_ALIGNMENT: return "pointer or stride not 16-byte aligned";
    case SKV_ERR_WORKSPACE: return "plan or partial buffer too small";
    case SKV_ERR_CUDA: return "CUDA launch failed";
    case SKV_DEV_TIMEOUT: return "device: barrier wait timed out";
    case SKV_DEV_PAGE_OOB: return "device: page id out of range";
    case SKV_DEV_PLAN_BAD: return "device: work item outside the request";
    default: return "unknown status";
  }
}

int32_t skv_mla_fold_ratio(int32_t num_heads, int32_t q_len, int32_t tile_m) {
  if (num_heads < 1 || q_len < 1 || tile_m < 1) return 1;
  int32_t best = 1;
  for (int32_t f = 1; f <= q_len; ++f)
    if (q_len % f == 0 && (int64_t)num_heads * f <= tile_m) best = f;
  return best;
}

skv_status skv_plan_paged(int32_t batch, const int32_t* qo_indptr_h, const int32_t* kv_indptr_h,
                          const int32_t* kv_last_page_len_h, int32_t page_size,
                          int32_t num_qo_heads, int32_t num_kv_heads, int32_t head_dim,
                          int32_t policy, int32_t param, const int32_t* split_indptr_h,
                          const int32_t* split_bounds_h, int32_t* plan_h,
                          int64_t plan_capacity, skv_plan_info* info) {
  return plan_paged_impl(batch, qo_indptr_h, kv_indptr_h, kv_last_page_len_h, page_size, num_qo_heads, num_kv_heads,
                         head_dim, policy, param, split_indptr_h, split_bounds_h, nullptr, plan_h, plan_capacity,
                         info);
}

skv_status skv_plan_paged_subset(int32_t batch, const int32_t* qo_indptr_h, const int32_t* kv_indptr_h,
                                 const int32_t* kv_last_page_len_h, int32_t page_size, int32_t num_qo_heads,
                                 int32_t num_kv_heads, int32_t head_dim, int32_t policy, int32_t param,
                                 const int32_t* requests_h, int32_t num_requests, int32_t* plan_h,
                                 int64_t plan_capacity, skv_plan_info* info) {
  if (info != nullptr) std::memset(info, 0, sizeof(*info));
  if (batch < 0 || num_requests < 0 || (num_requests > 0 && requests_h == nullptr)) return SKV_ERR_INVALID;
  if (policy == SKV_SPLIT_EXPLICIT) return SKV_ERR_INVALID;
  std::vector<char> include(batch, 0);
  for (int32_t i = 0; i < num_requests; ++i) {
    const int32_t r = requests_h[i];
    if (r < 0 || r >= batch || include[r]) return SKV_ERR_INVALID;  // out of range or listed twice
    include[r] = 1;
  }
  return plan_paged_impl(batch, qo_indptr_h, kv_indptr_h, kv_last_page_len_h, page_size, num_qo_heads, num_kv_heads,
                         head_dim, policy, param, nullptr, nullptr, &include, plan_h, plan_capacity, info);
}

skv_status skv_plan_mla(int32_t batch, int32_t q_len, const int32_t* kv_indptr_h,
                        const int32_t* kv_last_page_len_h, int32_t page_size, int32_t num_heads,
                        int32_t kv_dtype, int32_t policy, int32_t param, const int32_t* split_indptr_h,
                        const int32_t* split_bounds_h, int32_t* plan_h, int64_t plan_capacity,
                        skv_plan_info* info) {
  if (info != nullptr) std::memset(info, 0, sizeof(*info));
  if (q_len < 1 || num_heads < 1) return SKV_ERR_INVALID;
  if (kv_dtype != SKV_BF16 && kv_dtype != SKV_E4M3) return SKV_ERR_UNSUPPORTED;
  std::vector<ReqShape> req;
  skv_status st = check_table_h(batch, kv_indptr_h, kv_last_page_len_h, page_size, req);
  if (st != SKV_OK) return st;
  for (int32_t r = 0; r < batch; ++r) {
    req[r].q_start = r * q_len;
    req[r].q_len = q_len;
  }
  std::vector<int64_t> kv_len(batch);
  for (int32_t r = 0; r < batch; ++r)
    kv_len[r] = req[r].n_pages == 0 ? 0
                                    : (int64_t)(req[r].n_pages - 1) * page_size + kv_last_page_len_h[r];
  // tensor-core kernel: 16 query rows per tile when all of a request's rows fit, else 32; for the
  // bf16 cache 64 rows when a request has more (heads beyond 64 in groups of 64, their units spread
  // over a group of CTAs that share each KV slice); the fold puts as many query tokens as fit into
  // those rows
  const int64_t hq = (int64_t)num_heads * q_len;
  int32_t nr = hq <= 16 ? 16 : 32;
  if (kv_dtype == SKV_BF16 && hq > 32 && mla_tc64_supported(kv_dtype, page_size, num_heads)) nr = 64;
  const bool tc = kv_dtype == SKV_E4M3 ? mla_tc_fp8_supported(page_size, num_heads, nr)
                  : nr == 64           ? true
                                       : mla_tc_supported(kv_dtype, page_size, num_heads, nr);
  PersistOpts po;
  po.page_size = page_size;
  int32_t kernel = KERNEL_MLA_SIMT, fold = skv_mla_fold_ratio(num_heads, q_len, 128);
  int64_t head_groups = 1;
  if (tc) {
    kernel = nr == 16 ? KERNEL_MLA_TC16 : nr == 32 ? KERNEL_MLA_TC32 : KERNEL_MLA_TC64;
    fold = num_heads <= nr ? skv_mla_fold_ratio(num_heads, q_len, nr) : 1;
    head_groups = num_heads <= nr ? 1 : num_heads / nr;
    const int32_t sms = device_sms(policy == SKV_SPLIT_BALANCED ? param : 0);
    po.flat_ctas = sms;
    po.tile_tokens = mla_tc_tile_tokens();
    // measured (bench A/B of the charge): a work item's start and end cost about four 64-token
    // tiles on the e4m3 and 64-row kernels, about two on the bf16 16 / 32-row kernel
    po.piece_cost = (kv_dtype == SKV_BF16 && nr < 64) ? 2 : 4;
    if (nr == 64 || kv_dtype == SKV_E4M3) {  // CTA groups per KV slice (64-row and e4m3 kernels)
      po.group = (int32_t)(head_groups * (q_len / fold));
      po.flat_ctas = std::max<int32_t>(1, sms / po.group);
    }
  }
  return plan_common(batch, req, kv_len, fold, head_groups, 8, policy, param, split_indptr_h, split_bounds_h,
                     kernel, po, plan_h, plan_capacity, info);
}

}  // extern "C"

namespace {

// Host checks of a paged launch: the arguments, the plan summary and the kernel it names.
skv_status check_paged(const skv_paged_params* p, const int32_t* plan_d, const skv_plan_info* info) {
  if (p == nullptr) return SKV_ERR_INVALID;
  skv_status st = check_plan(plan_d, info);
  if (st != SKV_OK) return st;
  if (p->batch < 0 || p->total_q < 0 || p->page_size < 1 || p->num_pages < 0) return SKV_ERR_INVALID;
  if (p->num_qo_heads < 1 || p->num_kv_heads < 1 || p->num_qo_heads % p->num_kv_heads) return SKV_ERR_INVALID;
  if (p->head_dim != 64 && p->head_dim != 128) return SKV_ERR_UNSUPPORTED;
  if (p->o_dtype != SKV_F32 && p->o_dtype != SKV_BF16) return SKV_ERR_UNSUPPORTED;
  if (info->num_work > 0) {
    if (!p->q || !p->k_cache || !p->v_cache || !p->kv_indptr || !p->kv_indices || !p->kv_last_page_len || !p->o)
      return SKV_ERR_INVALID;
  }
  if (p->kv_dtype != SKV_BF16 && p->kv_dtype != SKV_E4M3) return SKV_ERR_UNSUPPORTED;
  const bool fp8 = p->kv_dtype == SKV_E4M3;
  if (fp8 && !(p->kv_scale > 0.f && std::isfinite(p->kv_scale))) return SKV_ERR_INVALID;
  const int64_t stride_unit = fp8 ? 16 : 8;  // elements per 16 bytes
  for (int i = 0; i < 3; ++i) {
    if (p->k_stride[i] < 0 || p->v_stride[i] < 0) return SKV_ERR_INVALID;
    if ((p->k_stride[i] % stride_unit) || (p->v_stride[i] % stride_unit)) return SKV_ERR_ALIGNMENT;
  }
  if (!aligned16(p->q) || !aligned16(p->k_cache) || !aligned16(p->v_cache) || !aligned16(p->o))
    return SKV_ERR_ALIGNMENT;
  if (info->num_partial_rows > 0 && (!p->o_part || !p->lse_part)) return SKV_ERR_WORKSPACE;
  if (info->kernel != KERNEL_GQA_SIMT && info->kernel != KERNEL_GQA_TC_DECODE && info->kernel != KERNEL_GQA_TC_WIDE &&
      info->kernel != KERNEL_GQA_TC_PREFILL)
    return SKV_ERR_INVALID;
  // the e4m3 cache runs on the all-KV-heads tensor-core kernel only
  if (fp8 && info->kernel != KERNEL_GQA_TC_WIDE) return SKV_ERR_UNSUPPORTED;
  if (info->num_work > 0 && info->kernel == KERNEL_GQA_TC_WIDE &&
      (info->num_ctas < 1 || info->cta_offset < 8LL * info->num_work + 4LL * info->num_merge_rows))
    return SKV_ERR_INVALID;
  return SKV_OK;
}

}  // namespace

extern "C" {

skv_status skv_paged_attn_partial(const skv_paged_params* p, const int32_t* plan_d,
                              const skv_plan_info* info, skv_stream_t stream) {
  skv_status st = check_paged(p, plan_d, info);
  if (st != SKV_OK) return st;
  const bool fp8 = p->kv_dtype == SKV_E4M3;
  if (info->num_work == 0) return SKV_OK;  // no query rows: nothing to launch
  const bool same_kv = p->k_stride[0] == p->v_stride[0] && p->k_stride[1] == p->v_stride[1] &&
                       p->k_stride[2] == p->v_stride[2];
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const WorkItem* work = reinterpret_cast<const WorkItem*>(plan_d);
  int e = info->kernel == KERNEL_GQA_TC_WIDE
              ? (fp8 ? launch_gqa_tc_wide_fp8(*p, work, plan_d + info->cta_offset, info->num_ctas, info->q_tile, s)
                     : launch_gqa_tc_wide(*p, work, plan_d + info->cta_offset, info->num_ctas, info->q_tile, s))
          : info->kernel == KERNEL_GQA_TC_PREFILL ? launch_gqa_tc_prefill(*p, work, info->num_work, info->q_tile, s)
          : info->kernel == KERNEL_GQA_TC_DECODE ? launch_gqa_tc_decode(*p, work, info->num_work, info->q_tile, s)
                                                 : launch_gqa_simt(*p, work, info->num_work, info->q_tile, same_kv, s);
  return cuda_status(e);
}

skv_status skv_merge_plan(const float* o_part, const float* lse_part, const int32_t* plan_d,
                          const skv_plan_info* info, int32_t num_heads, int32_t head_dim, void* o,
                          int32_t o_dtype, float* lse, skv_stream_t stream) {
  skv_status st = check_plan(plan_d, info);
  if (st != SKV_OK) return st;
  if (info->num_merge_rows == 0) return SKV_OK;
  if (plan_d == nullptr || o_part == nullptr || lse_part == nullptr || o == nullptr) return SKV_ERR_INVALID;
  if (num_heads < 1 || num_heads > 65535 || head_dim < 4 || head_dim % 4) return SKV_ERR_UNSUPPORTED;
  if (o_dtype != SKV_F32 && o_dtype != SKV_BF16) return SKV_ERR_UNSUPPORTED;
  const MergeItem* items = reinterpret_cast<const MergeItem*>(plan_d + 8LL * info->num_work);
  return cuda_status(launch_merge(o_part, lse_part, nullptr, 0, items, info->num_merge_rows, num_heads, head_dim, o,
                                  o_dtype, lse, reinterpret_cast<cudaStream_t>(stream)));
}

skv_status skv_paged_attn_fwd(const skv_paged_params* p, const int32_t* plan_d,
                              const skv_plan_info* info, skv_stream_t stream) {
  skv_status st = skv_paged_attn_partial(p, plan_d, info, stream);
  if (st != SKV_OK) return st;
  return skv_merge_plan(p->o_part, p->lse_part, plan_d, info, p->num_qo_heads, p->head_dim, p->o, p->o_dtype,
                        p->lse, stream);
}

skv_status skv_pod_attn_fwd(const skv_paged_params* p, const int32_t* decode_plan_d,
                            const skv_plan_info* decode_info, const int32_t* prefill_plan_d,
                            const skv_plan_info* prefill_info, float* prefill_o_part, float* prefill_lse_part,
                            skv_stream_t stream) {
  if (p == nullptr || decode_info == nullptr || prefill_info == nullptr) return SKV_ERR_INVALID;
  skv_paged_params pp = *p;  // the prefill plan's view: its own partial buffers
  pp.o_part = prefill_o_part;
  pp.lse_part = prefill_lse_part;
  skv_status st = check_paged(p, decode_plan_d, decode_info);
  if (st == SKV_OK) st = check_paged(&pp, prefill_plan_d, prefill_info);
  if (st != SKV_OK) return st;
  if (p->kv_dtype != SKV_BF16) return SKV_ERR_UNSUPPORTED;
  const bool has_dec = decode_info->num_work > 0, has_pre = prefill_info->num_work > 0;
  if ((has_dec && decode_info->kernel != KERNEL_GQA_TC_WIDE) || (has_pre && prefill_info->kernel != KERNEL_GQA_TC_PREFILL))
    return SKV_ERR_UNSUPPORTED;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (has_dec && has_pre) {
    st = cuda_status(launch_gqa_pod(*p, reinterpret_cast<const WorkItem*>(decode_plan_d),
                                    decode_plan_d + decode_info->cta_offset, decode_info->num_ctas,
                                    decode_info->q_tile, pp, reinterpret_cast<const WorkItem*>(prefill_plan_d),
                                    prefill_info->num_work, prefill_info->q_tile, s));
  } else if (has_dec) {
    st = skv_paged_attn_partial(p, decode_plan_d, decode_info, stream);
  } else if (has_pre) {
    st = skv_paged_attn_partial(&pp, prefill_plan_d, prefill_info, stream);
  }
  if (st != SKV_OK) return st;
  st = skv_merge_plan(p->o_part, p->lse_part, decode_plan_d, decode_info, p->num_qo_heads, p->head_dim, p->o,
                      p->o_dtype, p->lse, stream);
  if (st != SKV_OK) return st;
  return skv_merge_plan(pp.o_part, pp.lse_part, prefill_plan_d, prefill_info, p->num_qo_heads, p->head_dim, p->o,
                        p->o_dtype, p->lse, stream);
}

skv_status skv_mla_decode_partial(const skv_mla_params* p, const int32_t* plan_d,
                              const skv_plan_info* info, skv_stream_t stream) {
  if (p == nullptr) return SKV_ERR_INVALID;
  skv_status st = check_plan(plan_d, info);
  if (st != SKV_OK) return st;
  if (p->batch < 0 || p->q_len < 1 || p->num_heads < 1 || p->page_size < 1 || p->num_pages < 0)
    return SKV_ERR_INVALID;
  if (p->kv_dtype != SKV_BF16 && p->kv_dtype != SKV_E4M3) return SKV_ERR_UNSUPPORTED;
  if (p->o_dtype != SKV_F32 && p->o_dtype != SKV_BF16) return SKV_ERR_UNSUPPORTED;
  if (p->kv_dtype == SKV_E4M3 && !(p->kv_scale > 0.f && std::isfinite(p->kv_scale))) return SKV_ERR_INVALID;
  if (info->num_work > 0) {
    if (!p->q_nope || !p->q_pe || !p->ckv || !p->kpe || !p->kv_indptr || !p->kv_indices ||
        !p->kv_last_page_len || !p->o)
      return SKV_ERR_INVALID;
  }
  const int64_t esz = p->kv_dtype == SKV_E4M3 ? 1 : 2;
  for (int i = 0; i < 2; ++i) {
    if (p->ckv_stride[i] < 0 || p->kpe_stride[i] < 0) return SKV_ERR_INVALID;
    if ((p->ckv_stride[i] * esz) % 16 || (p->kpe_stride[i] * esz) % 16) return SKV_ERR_ALIGNMENT;
  }
  if (!aligned16(p->q_nope) || !aligned16(p->q_pe) || !aligned16(p->ckv) || !aligned16(p->kpe) ||
      !aligned16(p->o))
    return SKV_ERR_ALIGNMENT;
  if (info->num_partial_rows > 0 && (!p->o_part || !p->lse_part)) return SKV_ERR_WORKSPACE;
  const bool tc = info->kernel == KERNEL_MLA_TC16 || info->kernel == KERNEL_MLA_TC32 || info->kernel == KERNEL_MLA_TC64;
  if (info->kernel != KERNEL_MLA_SIMT && !tc) return SKV_ERR_INVALID;
  if (info->kernel == KERNEL_MLA_TC64 && p->kv_dtype != SKV_BF16) return SKV_ERR_INVALID;
  if (info->num_work == 0) return SKV_OK;  // no requests: nothing to launch
  if (tc && (info->num_ctas < 1 || info->cta_offset < 8LL * info->num_work + 4LL * info->num_merge_rows))
    return SKV_ERR_INVALID;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const WorkItem* work = reinterpret_cast<const WorkItem*>(plan_d);
  const int rows = info->kernel == KERNEL_MLA_TC16 ? 16 : 32;
  int e = !tc                                  ? launch_mla_simt(*p, work, info->num_work, info->q_tile, s)
          : info->kernel == KERNEL_MLA_TC64    ? launch_mla_tc64(*p, work, plan_d + info->cta_offset, info->num_ctas,
                                                                 info->q_tile, s)
          : p->kv_dtype == SKV_E4M3            ? launch_mla_tc_fp8(*p, work, plan_d + info->cta_offset, info->num_ctas,
                                                                   info->q_tile, rows, s)
                                               : launch_mla_tc(*p, work, plan_d + info->cta_offset, info->num_ctas,
                                                               info->q_tile, rows, s);
  return cuda_status(e);
}

skv_status skv_mla_decode_fwd(const skv_mla_params* p, const int32_t* plan_d,
                              const skv_plan_info* info, skv_stream_t stream) {
  skv_status st = skv_mla_decode_partial(p, plan_d, info, stream);
  if (st != SKV_OK) return st;
  return skv_merge_plan(p->o_part, p->lse_part, plan_d, info, p->num_heads, 512, p->o, p->o_dtype, p->lse,
                        stream);
}

skv_status skv_merge_states(const float* o_states, const float* lse_states,
                            const int32_t* state_indptr, int32_t num_states, int64_t num_rows,
                            int32_t num_heads, int32_t head_dim, void* o_out, int32_t o_dtype,
                            float* lse_out, skv_stream_t stream) {
  if (num_rows < 0 || num_heads < 1 || head_dim < 1) return SKV_ERR_INVALID;
  if (num_rows == 0) return SKV_OK;
  if (o_states == nullptr || lse_states == nullptr || o_out == nullptr) return SKV_ERR_INVALID;
  if (state_indptr == nullptr && num_states < 0) return SKV_ERR_INVALID;
  if (num_rows > INT32_MAX) return SKV_ERR_UNSUPPORTED;
  if (head_dim % 4 != 0 || num_heads > 65535) return SKV_ERR_UNSUPPORTED;
  if (o_dtype != SKV_F32 && o_dtype != SKV_BF16) return SKV_ERR_UNSUPPORTED;
  if (!aligned16(o_states) || !aligned16(o_out)) return SKV_ERR_ALIGNMENT;
  return cuda_status(launch_merge(o_states, lse_states, state_indptr, num_states, nullptr, num_rows, num_heads,
                                  head_dim, o_out, o_dtype, lse_out, reinterpret_cast<cudaStream_t>(stream)));
}

skv_status skv_test_wait_timeout(int32_t* status, int64_t limit_ns, skv_stream_t stream) {
  if (status == nullptr || limit_ns < 0 || limit_ns > 10000000000LL) return SKV_ERR_INVALID;
  return cuda_status(launch_wait_timeout(status, (uint64_t)limit_ns, reinterpret_cast<cudaStream_t>(stream)));
}

skv_status skv_causal_tables(int32_t batch, const int32_t* qo_indptr_h, const int32_t* kv_indptr_h,
                             const int32_t* kv_indices_h, const int32_t* kv_last_page_len_h, int32_t page_size,
                             int32_t* prefix_indptr_h, int32_t* prefix_indices_h, int32_t* prefix_last_h,
                             int32_t* diag_indptr_h, int32_t* diag_rows_h, int32_t* diag_last_h,
                             int64_t diag_capacity, int64_t* diag_rows_needed) {
  if (batch < 0 || page_size < 1 || diag_capacity < 0 || !qo_indptr_h || !kv_indptr_h || !kv_last_page_len_h ||
      !diag_rows_needed)
    return SKV_ERR_INVALID;
  if (qo_indptr_h[0] != 0 || kv_indptr_h[0] != 0) return SKV_ERR_INVALID;
  // validate the table and count the diagonal rows
  int64_t need = 0;
  for (int32_t r = 0; r < batch; ++r) {
    const int64_t nq = (int64_t)qo_indptr_h[r + 1] - qo_indptr_h[r];
    const int64_t n = (int64_t)kv_indptr_h[r + 1] - kv_indptr_h[r];
    if (nq < 0 || n < 0) return SKV_ERR_INVALID;
    if (n > 0 && (kv_last_page_len_h[r] < 1 || kv_last_page_len_h[r] > page_size)) return SKV_ERR_INVALID;
    const int64_t L = n == 0 ? 0 : (n - 1) * page_size + kv_last_page_len_h[r];
    const int64_t lp = std::min<int64_t>(L, std::max<int64_t>(0, L - nq + 1));  // nq = 0: no row sees more than L
    for (int64_t i = 0; i < nq; ++i) need += std::max<int64_t>(0, L - nq + 1 + i - lp);
  }
  *diag_rows_needed = need;
  if (need > diag_capacity) return SKV_ERR_WORKSPACE;
  if (need > INT32_MAX) return SKV_ERR_UNSUPPORTED;
  if (!prefix_indptr_h || !prefix_last_h || !diag_indptr_h || !diag_last_h || (need > 0 && !diag_rows_h) ||
      (kv_indptr_h[batch] > 0 && (!kv_indices_h || !prefix_indices_h)))
    return SKV_ERR_INVALID;
  prefix_indptr_h[0] = 0;
  diag_indptr_h[0] = 0;
  int64_t drow = 0;
  for (int32_t r = 0; r < batch; ++r) {
    const int64_t nq = (int64_t)qo_indptr_h[r + 1] - qo_indptr_h[r];
    const int64_t n = (int64_t)kv_indptr_h[r + 1] - kv_indptr_h[r];
    const int64_t L = n == 0 ? 0 : (n - 1) * page_size + kv_last_page_len_h[r];
    const int64_t lp = std::min<int64_t>(L, std::max<int64_t>(0, L - nq + 1));
    const int64_t np_ = (lp + page_size - 1) / page_size;  // <= n: the prefix stays inside the request
    const int32_t* pages = kv_indices_h + kv_indptr_h[r];
    for (int64_t j = 0; j < np_; ++j) prefix_indices_h[prefix_indptr_h[r] + j] = pages[j];
    prefix_indptr_h[r + 1] = prefix_indptr_h[r] + (int32_t)np_;
    prefix_last_h[r] = np_ > 0 ? (int32_t)(lp - (np_ - 1) * page_size) : 1;
    for (int64_t i = 0; i < nq; ++i) {
      const int64_t row = qo_indptr_h[r] + i;
      for (int64_t t = lp; t < L - nq + 1 + i; ++t) {
        const int64_t id = (int64_t)pages[t / page_size] * page_size + t % page_size;
        if (id < 0 || id > INT32_MAX) return SKV_ERR_UNSUPPORTED;
        diag_rows_h[drow++] = (int32_t)id;
      }
      diag_indptr_h[row + 1] = (int32_t)drow;
      diag_last_h[row] = 1;
    }
  }
  return SKV_OK;
}

skv_status skv_mla_splice(const skv_splice_params* p, const skv_splice_chunk* chunks_h, int32_t num_chunks,
                          skv_stream_t stream) {
  if (p == nullptr || num_chunks < 0 || (num_chunks > 0 && chunks_h == nullptr)) return SKV_ERR_INVALID;
  int64_t total = 0;
  for (int32_t c = 0; c < num_chunks; ++c) {
    const skv_splice_chunk& ch = chunks_h[c];
    if (ch.n_tokens < 0 || ch.src_start < 0 || ch.dst_start < 0) return SKV_ERR_INVALID;
    if (ch.src_start > INT64_MAX / 2 - ch.n_tokens || ch.dst_start > INT64_MAX / 2 - ch.n_tokens ||
        total > INT64_MAX / 4 - ch.n_tokens)
      return SKV_ERR_INVALID;
    total += ch.n_tokens;
  }
  if (total == 0) return SKV_OK;
  if (!p->src_ckv || !p->src_kpe || !p->dst_ckv || !p->dst_kpe || !p->src_pages || !p->dst_pages)
    return SKV_ERR_INVALID;
  if (p->src_page_size < 1 || p->dst_page_size < 1 || p->src_num_pages < 1 || p->dst_num_pages < 1)
    return SKV_ERR_INVALID;
  if (p->rope_layout != SKV_ROPE_INTERLEAVED && p->rope_layout != SKV_ROPE_HALVES) return SKV_ERR_INVALID;
  if (p->inv_freq == nullptr && !(p->rope_theta > 0.0f && p->rope_theta < INFINITY)) return SKV_ERR_INVALID;
  if (p->kv_dtype != SKV_BF16) return SKV_ERR_UNSUPPORTED;
  if (!aligned16(p->src_ckv) || !aligned16(p->src_kpe) || !aligned16(p->dst_ckv) || !aligned16(p->dst_kpe))
    return SKV_ERR_ALIGNMENT;
  const int64_t strides[8] = {p->src_ckv_stride[0], p->src_ckv_stride[1], p->src_kpe_stride[0],
                              p->src_kpe_stride[1], p->dst_ckv_stride[0], p->dst_ckv_stride[1],
                              p->dst_kpe_stride[0], p->dst_kpe_stride[1]};
  for (int64_t st : strides)
    if (st % 8 != 0) return SKV_ERR_ALIGNMENT;
  return cuda_status(launch_splice(*p, chunks_h, num_chunks, reinterpret_cast<cudaStream_t>(stream)));
}

skv_status skv_paged_kv_gather(const skv_paged_params* p, const int32_t* token_indptr,
                               int64_t total_tokens, void* k_out, void* v_out, skv_stream_t stream) {
  if (p == nullptr || total_tokens < 0) return SKV_ERR_INVALID;
  if (total_tokens == 0) return SKV_OK;
  if (!token_indptr || !k_out || !v_out || !p->k_cache || !p->v_cache || !p->kv_indptr || !p->kv_indices ||
      !p->kv_last_page_len)
    return SKV_ERR_INVALID;
  if (p->batch < 1 || p->page_size < 1 || p->num_kv_heads < 1 || p->head_dim < 1) return SKV_ERR_INVALID;
  if (total_tokens > INT32_MAX || p->kv_dtype != SKV_BF16) return SKV_ERR_UNSUPPORTED;
  const bool same_kv = p->k_stride[0] == p->v_stride[0] && p->k_stride[1] == p->v_stride[1] &&
                       p->k_stride[2] == p->v_stride[2];
  return cuda_status(launch_gather(*p, token_indptr, total_tokens, k_out, v_out, same_kv,
                                   reinterpret_cast<cudaStream_t>(stream)));
}

}  // extern "C"
