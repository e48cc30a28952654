// Host side of the C ABI: argument validation, the split-KV planner, the RoPE
// table, status handling, and the launch sequence of each entry point.
#include <math.h>
#include <stdarg.h>
#include <stdio.h>
#include <string.h>

#include <algorithm>
#include <mutex>
#include <queue>
#include <vector>

#include "internal.h"
#include "mla_debug.h"

namespace mla {

static thread_local char g_err[1024];

mla_status_t fail(mla_status_t st, const char *fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
  return st;
}

void clear_error() { g_err[0] = '\0'; }

mla_status_t device_info(int *num_sms, int *cc_major, int *cc_minor) {
  static std::mutex mu;
  static int cached[64][3];
  static bool have[64] = {};
  int dev = 0;
  MLA_CUDA_TRY(cudaGetDevice(&dev));
  std::lock_guard<std::mutex> lock(mu);
  if (dev < 0 || dev >= 64) return fail(MLA_ERR_UNSUPPORTED, "device index %d", dev);
  if (!have[dev]) {
    MLA_CUDA_TRY(cudaDeviceGetAttribute(&cached[dev][0], cudaDevAttrMultiProcessorCount, dev));
    MLA_CUDA_TRY(cudaDeviceGetAttribute(&cached[dev][1], cudaDevAttrComputeCapabilityMajor, dev));
    MLA_CUDA_TRY(cudaDeviceGetAttribute(&cached[dev][2], cudaDevAttrComputeCapabilityMinor, dev));
    have[dev] = true;
  }
  if (num_sms) *num_sms = cached[dev][0];
  if (cc_major) *cc_major = cached[dev][1];
  if (cc_minor) *cc_minor = cached[dev][2];
  return MLA_OK;
}

static mla_status_t require_sm100() {
  int major = 0, minor = 0;
  mla_status_t st = device_info(nullptr, &major, &minor);
  if (st != MLA_OK) return st;
  if (major != 10)
    return fail(MLA_ERR_UNSUPPORTED, "compute capability %d.%d: this library is built for sm_100a",
                major, minor);
  return MLA_OK;
}

static bool heads_supported(int n_h) { return n_h >= 16 && n_h <= 128 && n_h % 16 == 0; }

// ---------------------------------------------------------------- planner ---

static size_t align16(size_t x) { return (x + 15) & ~(size_t)15; }

static size_t plan_bytes_for(int batch, int q_len, int num_ctas) {
  const size_t units = (size_t)batch * q_len;
  const size_t max_items = units + (size_t)num_ctas;
  return sizeof(PlanHeader) + align16(sizeof(int32_t) * (num_ctas + 1)) +
         max_items * sizeof(WorkItem) + units * sizeof(CombineItem);
}

static mla_status_t resolve_ctas(int *num_ctas) {
  if (*num_ctas > 0) return MLA_OK;
  int sms = 0;
  mla_status_t st = device_info(&sms, nullptr, nullptr);
  if (st != MLA_OK) return st;
  *num_ctas = std::max(1, sms / 2);  // one CTA pair (cluster of 2) per work list
  return MLA_OK;
}

}  // namespace mla

using namespace mla;

extern "C" {

const char *mla_last_error(void) { return g_err; }

int mla_version(void) { return 2; }

mla_status_t mla_rope_table(float *table, int max_pos, double base) {
  clear_error();
  MLA_CHECK_ARG(table != nullptr, "rope table pointer is NULL");
  MLA_CHECK_ARG(max_pos > 0, "max_pos must be positive (got %d)", max_pos);
  MLA_CHECK_ARG(base > 1.0, "RoPE base must exceed 1 (got %g)", base);
  double denom[MLA_D_R / 2];
  for (int j = 0; j < MLA_D_R / 2; ++j) denom[j] = pow(base, 2.0 * j / MLA_D_R);
  for (int p = 0; p < max_pos; ++p) {
    for (int j = 0; j < MLA_D_R / 2; ++j) {
      const double th = (double)p / denom[j];
      table[(size_t)p * MLA_D_R + 2 * j] = (float)cos(th);
      table[(size_t)p * MLA_D_R + 2 * j + 1] = (float)sin(th);
    }
  }
  return MLA_OK;
}

mla_status_t mla_cache_append(mla_bf16_t *cache, int num_pages, const int32_t *block_table,
                              int batch, int max_pages, const int32_t *seq_idx,
                              const int32_t *pos, const mla_bf16_t *c_kv, int ld_c,
                              const mla_bf16_t *k_pe, int ld_k, const float *rope_table,
                              int max_pos, int n_tokens, uint32_t *status,
                              mla_stream_t stream) {
  clear_error();
  MLA_CHECK_ARG(n_tokens >= 0, "n_tokens < 0");
  if (n_tokens == 0) return MLA_OK;
  MLA_CHECK_ARG(cache && block_table && seq_idx && pos && c_kv && k_pe && rope_table,
                "NULL device pointer");
  MLA_CHECK_ARG(num_pages > 0 && batch > 0 && max_pages > 0 && max_pos > 0,
                "sizes must be positive");
  MLA_CHECK_ARG(aligned16(cache) && aligned16(c_kv) && aligned16(k_pe) && aligned16(rope_table),
                "cache, c_kv, k_pe and rope_table must be 16-byte aligned");
  MLA_CHECK_ARG(ld_c >= MLA_D_C && ld_c % 8 == 0, "ld_c must be >= 512 and a multiple of 8");
  MLA_CHECK_ARG(ld_k >= MLA_D_R && ld_k % 8 == 0, "ld_k must be >= 64 and a multiple of 8");
  mla_status_t st = require_sm100();
  if (st != MLA_OK) return st;
  return launch_cache_append(cache, num_pages, block_table, batch, max_pages, seq_idx, pos,
                             c_kv, ld_c, k_pe, ld_k, rope_table, max_pos, n_tokens, status,
                             (cudaStream_t)stream);
}

mla_status_t mla_absorb_q(const mla_bf16_t *q_nope, int ld_qn, const mla_bf16_t *q_pe,
                          int ld_qp, const mla_bf16_t *w_uk, const int32_t *pos,
                          const float *rope_table, int max_pos, int T, int n_h,
                          mla_bf16_t *q_full, uint32_t *status, mla_stream_t stream) {
  clear_error();
  MLA_CHECK_ARG(T >= 0, "T < 0");
  if (T == 0) return MLA_OK;
  if (!heads_supported(n_h))
    return fail(MLA_ERR_UNSUPPORTED, "n_h = %d (supported: 16..128, multiple of 16)", n_h);
  MLA_CHECK_ARG(q_nope && q_pe && w_uk && q_full, "NULL device pointer");
  MLA_CHECK_ARG(pos == nullptr || (rope_table != nullptr && max_pos > 0),
                "pos given without a RoPE table");
  MLA_CHECK_ARG(aligned16(q_nope) && aligned16(q_pe) && aligned16(w_uk) && aligned16(q_full) &&
                    (rope_table == nullptr || aligned16(rope_table)),
                "pointers must be 16-byte aligned");
  MLA_CHECK_ARG(ld_qn >= n_h * MLA_D_NOPE && ld_qn % 8 == 0, "ld_qn too small or unaligned");
  MLA_CHECK_ARG(ld_qp >= n_h * MLA_D_R && ld_qp % 8 == 0, "ld_qp too small or unaligned");
  mla_status_t st = require_sm100();
  if (st != MLA_OK) return st;
  return launch_absorb_q(q_nope, ld_qn, q_pe, ld_qp, pos, rope_table, max_pos, w_uk, T, n_h,
                         q_full, status, (cudaStream_t)stream);
}

mla_status_t mla_append_absorb_q(mla_bf16_t *cache, int num_pages, const int32_t *block_table,
                                 int batch, int max_pages, const int32_t *seq_idx,
                                 const int32_t *tok_pos, const mla_bf16_t *c_kv, int ld_c,
                                 const mla_bf16_t *k_pe, int ld_k, int n_tokens,
                                 const mla_bf16_t *q_nope, int ld_qn, const mla_bf16_t *q_pe,
                                 int ld_qp, const mla_bf16_t *w_uk, const int32_t *q_pos,
                                 const float *rope_table, int max_pos, int T, int n_h,
                                 mla_bf16_t *q_full, uint32_t *status, mla_stream_t stream) {
  clear_error();
  MLA_CHECK_ARG(n_tokens >= 0 && T >= 0, "negative size");
  if (T == 0)
    return mla_cache_append(cache, num_pages, block_table, batch, max_pages, seq_idx, tok_pos,
                            c_kv, ld_c, k_pe, ld_k, rope_table, max_pos, n_tokens, status, stream);
  if (n_tokens == 0)
    return mla_absorb_q(q_nope, ld_qn, q_pe, ld_qp, w_uk, q_pos, rope_table, max_pos, T, n_h,
                        q_full, status, stream);
  // the append's arguments, as mla_cache_append checks them
  MLA_CHECK_ARG(cache && block_table && seq_idx && tok_pos && c_kv && k_pe && rope_table,
                "NULL device pointer");
  MLA_CHECK_ARG(num_pages > 0 && batch > 0 && max_pages > 0 && max_pos > 0,
                "sizes must be positive");
  MLA_CHECK_ARG(aligned16(cache) && aligned16(c_kv) && aligned16(k_pe) && aligned16(rope_table),
                "cache, c_kv, k_pe and rope_table must be 16-byte aligned");
  MLA_CHECK_ARG(ld_c >= MLA_D_C && ld_c % 8 == 0, "ld_c must be >= 512 and a multiple of 8");
  MLA_CHECK_ARG(ld_k >= MLA_D_R && ld_k % 8 == 0, "ld_k must be >= 64 and a multiple of 8");
  // the absorption's, as mla_absorb_q checks them
  if (!heads_supported(n_h))
    return fail(MLA_ERR_UNSUPPORTED, "n_h = %d (supported: 16..128, multiple of 16)", n_h);
  MLA_CHECK_ARG(q_nope && q_pe && w_uk && q_full, "NULL device pointer");
  MLA_CHECK_ARG(aligned16(q_nope) && aligned16(q_pe) && aligned16(w_uk) && aligned16(q_full),
                "pointers must be 16-byte aligned");
  MLA_CHECK_ARG(ld_qn >= n_h * MLA_D_NOPE && ld_qn % 8 == 0, "ld_qn too small or unaligned");
  MLA_CHECK_ARG(ld_qp >= n_h * MLA_D_R && ld_qp % 8 == 0, "ld_qp too small or unaligned");
  mla_status_t st = require_sm100();
  if (st != MLA_OK) return st;
  AppendJob app;
  app.cache = cache;
  app.cache8 = nullptr;
  app.scales8 = nullptr;
  app.num_pages = num_pages;
  app.block_table = block_table;
  app.batch = batch;
  app.max_pages = max_pages;
  app.seq_idx = seq_idx;
  app.pos = tok_pos;
  app.c_kv = c_kv;
  app.ld_c = ld_c;
  app.k_pe = k_pe;
  app.ld_k = ld_k;
  app.n_tokens = n_tokens;
  return launch_absorb_q(q_nope, ld_qn, q_pe, ld_qp, q_pos, rope_table, max_pos, w_uk, T, n_h,
                         q_full, status, (cudaStream_t)stream, &app);
}

mla_status_t mla_append_fp8_absorb_q(uint8_t *cache, float *scales, int num_pages,
                                     const int32_t *block_table, int batch, int max_pages,
                                     const int32_t *seq_idx, const int32_t *tok_pos,
                                     const mla_bf16_t *c_kv, int ld_c, const mla_bf16_t *k_pe,
                                     int ld_k, int n_tokens, const mla_bf16_t *q_nope, int ld_qn,
                                     const mla_bf16_t *q_pe, int ld_qp, const mla_bf16_t *w_uk,
                                     const int32_t *q_pos, const float *rope_table, int max_pos,
                                     int T, int n_h, mla_bf16_t *q_full, uint32_t *status,
                                     mla_stream_t stream) {
  clear_error();
  MLA_CHECK_ARG(n_tokens >= 0 && T >= 0, "negative size");
  if (T == 0)
    return mla_cache_append_fp8(cache, scales, num_pages, block_table, batch, max_pages, seq_idx,
                                tok_pos, c_kv, ld_c, k_pe, ld_k, rope_table, max_pos, n_tokens,
                                status, stream);
  if (n_tokens == 0)
    return mla_absorb_q(q_nope, ld_qn, q_pe, ld_qp, w_uk, q_pos, rope_table, max_pos, T, n_h,
                        q_full, status, stream);
  // the append's arguments, as mla_cache_append_fp8 checks them
  MLA_CHECK_ARG(cache && scales && block_table && seq_idx && tok_pos && c_kv && k_pe &&
                    rope_table,
                "NULL device pointer");
  MLA_CHECK_ARG(num_pages > 0 && batch > 0 && max_pages > 0 && max_pos > 0,
                "sizes must be positive");
  MLA_CHECK_ARG(aligned16(cache) && aligned16(scales) && aligned16(c_kv) && aligned16(k_pe) &&
                    aligned16(rope_table),
                "cache, scales, c_kv, k_pe and rope_table must be 16-byte aligned");
  MLA_CHECK_ARG(ld_c >= MLA_D_C && ld_c % 8 == 0, "ld_c must be >= 512 and a multiple of 8");
  MLA_CHECK_ARG(ld_k >= MLA_D_R && ld_k % 8 == 0, "ld_k must be >= 64 and a multiple of 8");
  // the absorption's, as mla_absorb_q checks them
  if (!heads_supported(n_h))
    return fail(MLA_ERR_UNSUPPORTED, "n_h = %d (supported: 16..128, multiple of 16)", n_h);
  MLA_CHECK_ARG(q_nope && q_pe && w_uk && q_full, "NULL device pointer");
  MLA_CHECK_ARG(aligned16(q_nope) && aligned16(q_pe) && aligned16(w_uk) && aligned16(q_full),
                "pointers must be 16-byte aligned");
  MLA_CHECK_ARG(ld_qn >= n_h * MLA_D_NOPE && ld_qn % 8 == 0, "ld_qn too small or unaligned");
  MLA_CHECK_ARG(ld_qp >= n_h * MLA_D_R && ld_qp % 8 == 0, "ld_qp too small or unaligned");
  mla_status_t st = require_sm100();
  if (st != MLA_OK) return st;
  AppendJob app;
  app.cache = nullptr;
  app.cache8 = cache;
  app.scales8 = scales;
  app.num_pages = num_pages;
  app.block_table = block_table;
  app.batch = batch;
  app.max_pages = max_pages;
  app.seq_idx = seq_idx;
  app.pos = tok_pos;
  app.c_kv = c_kv;
  app.ld_c = ld_c;
  app.k_pe = k_pe;
  app.ld_k = ld_k;
  app.n_tokens = n_tokens;
  return launch_absorb_q(q_nope, ld_qn, q_pe, ld_qp, q_pos, rope_table, max_pos, w_uk, T, n_h,
                         q_full, status, (cudaStream_t)stream, &app);
}

size_t mla_plan_bytes(int batch, int q_len, int num_ctas) {
  if (batch < 0 || q_len < 0) return 0;
  if (resolve_ctas(&num_ctas) != MLA_OK) return 0;
  return plan_bytes_for(batch, q_len, num_ctas);
}

mla_status_t mla_decode_plan(const int32_t *seq_lens, int batch, int q_len, int n_h,
                             int num_ctas, int max_split, void *plan, size_t plan_bytes,
                             mla_plan_info_t *info) {
  clear_error();
  MLA_CHECK_ARG(batch >= 0, "batch < 0");
  MLA_CHECK_ARG(q_len >= 1, "q_len must be positive (got %d)", q_len);
  if (q_len > MLA_MAX_Q_LEN)
    return fail(MLA_ERR_UNSUPPORTED, "q_len = %d (supported: 1..%d)", q_len, MLA_MAX_Q_LEN);
  if (!heads_supported(n_h))
    return fail(MLA_ERR_UNSUPPORTED, "n_h = %d (supported: 16..128, multiple of 16)", n_h);
  MLA_CHECK_ARG(batch == 0 || seq_lens != nullptr, "seq_lens is NULL");
  MLA_CHECK_ARG(plan != nullptr, "plan is NULL");
  mla_status_t st = resolve_ctas(&num_ctas);
  if (st != MLA_OK) return st;
  const size_t need = plan_bytes_for(batch, q_len, num_ctas);
  if (plan_bytes < need)
    return fail(MLA_ERR_WORKSPACE_TOO_SMALL, "plan buffer %zu B < %zu B", plan_bytes, need);
  for (int b = 0; b < batch; ++b)
    MLA_CHECK_ARG(seq_lens[b] >= q_len, "seq_lens[%d] = %d < q_len = %d", b, seq_lens[b], q_len);

  // (b, j) units and their page counts: query j sees tokens 0..L-q_len+j.
  struct Unit { int b, j, pages, L, qpos; };
  std::vector<Unit> units;
  units.reserve((size_t)batch * q_len);
  long long total = 0;
  int max_unit = 0;
  for (int b = 0; b < batch; ++b)
    for (int j = 0; j < q_len; ++j) {
      const int L = seq_lens[b];
      const int qpos = L - q_len + j;
      const int pages = (qpos + 1 + MLA_PAGE - 1) / MLA_PAGE;
      units.push_back({b, j, pages, L, qpos});
      total += pages;
      max_unit = std::max(max_unit, pages);
    }
  // Work lists. The "whole" plan makes every (sequence, query) one item and
  // deals the items to lists in longest-processing-time order. The "cut" plan
  // lays the units' pages end to end and cuts them into num_ctas near-equal
  // ranges, so every list carries the same page count; a unit crossing a cut
  // becomes several items whose partial results the combine pass merges.
  // Adjacent units (the two queries of an MTP step) start on neighbouring
  // lists at the same time, so their shared pages are read once from HBM and
  // once from L2. max_split == 1 selects the whole plan, max_split >= 0 the
  // cut plan, max_split < 0 the one with the smaller estimated time.
  int max_pages_used = 0;
  for (const Unit &u : units) max_pages_used = std::max(max_pages_used, u.pages);
  typedef std::vector<std::vector<WorkItem>> Lists;
  auto plan_whole = [&](Lists &per) {
    std::vector<int> order(units.size());
    for (size_t i = 0; i < order.size(); ++i) order[i] = (int)i;
    std::stable_sort(order.begin(), order.end(),
                     [&](int x, int y) { return units[x].pages > units[y].pages; });
    const int lists = std::max(1, std::min<int>(num_ctas, (int)units.size()));
    typedef std::pair<long long, int> Load;
    std::priority_queue<Load, std::vector<Load>, std::greater<Load>> heap;
    for (int c = 0; c < lists; ++c) heap.push({0, c});
    per.assign(lists, {});
    for (int idx : order) {
      const Unit &u = units[idx];
      Load ld = heap.top();
      heap.pop();
      per[ld.second].push_back(WorkItem{u.b, u.j, 0, u.pages, -1, u.L, u.qpos, 0});
      ld.first += u.pages;
      heap.push(ld);
    }
  };
  auto plan_cut = [&](Lists &per, std::vector<CombineItem> &comb, int &slots) {
    // Cuts fall on 4-page boundaries of each unit (the kernels' tile), so a
    // split adds no partial tile. List c ends near the cumulative boundary
    // total * (c + 1) / lists: a tile joins the list unless it would overshoot
    // the boundary by more than half its size, so lists differ by about one
    // tile and the rounding does not drift onto the last list.
    const int lists = (int)std::max<long long>(1, std::min<long long>(num_ctas, total));
    auto boundary = [&](int c) { return (total * (c + 1) + lists / 2) / lists; };
    per.assign(lists, {});
    int c = 0;
    long long fill = 0, cum = 0;
    for (const Unit &u : units) {
      std::vector<std::pair<int, int>> where;  // (list, index in list)
      int begin = 0;
      while (begin < u.pages) {
        int end = begin;
        while (end < u.pages) {
          const int tile = std::min(4, u.pages - end);
          const bool over = c < lists - 1 && 2 * (cum + tile) > 2 * boundary(c) + tile;
          if (over && fill > 0) break;
          end += tile;
          cum += tile;
          fill += tile;
        }
        if (end > begin) {
          where.push_back({c, (int)per[c].size()});
          per[c].push_back(WorkItem{u.b, u.j, begin, end, -1, u.L, u.qpos, 0});
          begin = end;
        }
        if (begin < u.pages) {  // list c is full
          ++c;
          fill = 0;
        }
      }
      if (where.size() > 1) {
        comb.push_back(CombineItem{u.b, u.j, slots, (int)where.size()});
        for (size_t p = 0; p < where.size(); ++p)
          per[where[p].first][where[p].second].slot = slots + (int)p;
        slots += (int)where.size();
      }
    }
  };
  // Estimated time of a plan in units of one score/output tile (4 pages): the
  // busiest list's tiles plus a fixed cost per item (query load, pipeline
  // refill, epilogue) and, when parts must be merged, the combine pass.
  auto estimate = [&](const Lists &per, bool merged) {
    long long worst = 0;
    for (const auto &v : per) {
      long long t = 0;
      for (const WorkItem &it : v) t += (it.page_end - it.page_begin + 3) / 4 + 2;
      worst = std::max(worst, t);
    }
    return worst + (merged ? 2 : 0);
  };
  Lists per;
  std::vector<CombineItem> comb;
  int slots = 0;
  if (max_split == 1) {
    plan_whole(per);
  } else if (max_split >= 0) {
    plan_cut(per, comb, slots);
  } else {
    Lists whole;
    plan_whole(whole);
    plan_cut(per, comb, slots);
    if (estimate(whole, false) <= estimate(per, !comb.empty())) {
      per.swap(whole);
      comb.clear();
      slots = 0;
    }
  }
  size_t n_items = 0;
  for (auto &v : per) n_items += v.size();
  if (n_items > (size_t)batch * q_len + num_ctas)
    return fail(MLA_ERR_INVALID_ARGUMENT, "planner produced %zu items (bound %zu)", n_items,
                (size_t)batch * q_len + num_ctas);
  const int lists = batch == 0 ? 0 : (int)per.size();
  unsigned char *base = static_cast<unsigned char *>(plan);
  memset(base, 0, need);
  PlanHeader *h = reinterpret_cast<PlanHeader *>(base);
  h->magic = kPlanMagic;
  h->version = kPlanVersion;
  h->batch = batch;
  h->q_len = q_len;
  h->n_h = n_h;
  h->num_items = (int)n_items;
  h->num_ctas = lists;
  h->num_partials = slots;
  h->num_combine = (int)comb.size();
  h->cta_off = (int)sizeof(PlanHeader);
  h->items_off = h->cta_off + (int)align16(sizeof(int32_t) * (num_ctas + 1));
  h->combine_off = h->items_off + (int)((size_t)(batch * q_len + num_ctas) * sizeof(WorkItem));
  h->max_pages_used = max_pages_used;
  int32_t *cta_begin = reinterpret_cast<int32_t *>(base + h->cta_off);
  WorkItem *out_items = reinterpret_cast<WorkItem *>(base + h->items_off);
  int n = 0;
  for (int c = 0; c < lists; ++c) {
    cta_begin[c] = n;
    for (const WorkItem &it : per[c]) out_items[n++] = it;
  }
  cta_begin[lists] = n;
  CombineItem *out_comb = reinterpret_cast<CombineItem *>(base + h->combine_off);
  for (size_t i = 0; i < comb.size(); ++i) out_comb[i] = comb[i];
  if (info) {
    info->num_items = h->num_items;
    info->num_ctas = h->num_ctas;
    info->num_partials = slots;
    info->num_combine = h->num_combine;
    info->plan_bytes = (size_t)h->combine_off + comb.size() * sizeof(CombineItem);
    info->workspace_bytes = workspace_bytes(slots, n_h);
  }
  return MLA_OK;
}

}  // extern "C"

// Validation and launch shared by the decode entry points: the tensor-core
// kernel on the bf16 cache, the CUDA-core kernel (debug entry point), or the
// tensor-core kernel on the FP8 cache (`fp8_scales` != NULL).
enum DecodeKind { kTensorCore, kCudaCore, kTensorCoreFp8 };

static mla_status_t decode_entry(const mla_bf16_t *q_full, const void *cache,
                                 int num_pages, const int32_t *block_table, int max_pages,
                                 int batch, int q_len, int n_h, float scale,
                                 const void *plan_host, const void *plan_dev, void *workspace,
                                 size_t workspace_bytes_given, mla_bf16_t *o_latent, float *lse,
                                 uint32_t *status, mla_stream_t stream, DecodeKind kind,
                                 const float *fp8_scales = nullptr) {
  clear_error();
  MLA_CHECK_ARG(plan_host != nullptr && plan_dev != nullptr, "plan pointers are NULL");
  const PlanHeader *ph = static_cast<const PlanHeader *>(plan_host);
  MLA_CHECK_ARG(ph->magic == kPlanMagic && ph->version == kPlanVersion, "not a decode plan");
  MLA_CHECK_ARG(ph->batch == batch && ph->q_len == q_len && ph->n_h == n_h,
                "plan was built for batch %d, q_len %d, n_h %d", ph->batch, ph->q_len, ph->n_h);
  if (batch == 0 || ph->num_items == 0) return MLA_OK;
  MLA_CHECK_ARG(q_full && cache && block_table && o_latent, "NULL device pointer");
  MLA_CHECK_ARG(kind != kTensorCoreFp8 || (fp8_scales != nullptr && aligned16(fp8_scales)),
                "the FP8 cache needs a 16-byte aligned scale array");
  MLA_CHECK_ARG(aligned16(q_full) && aligned16(cache) && aligned16(o_latent) &&
                    aligned16(plan_dev) && (workspace == nullptr || aligned16(workspace)),
                "pointers must be 16-byte aligned");
  MLA_CHECK_ARG(num_pages > 0 && max_pages > 0, "num_pages and max_pages must be positive");
  MLA_CHECK_ARG(ph->max_pages_used <= max_pages,
                "a sequence needs %d pages but the block table has %d columns",
                ph->max_pages_used, max_pages);
  MLA_CHECK_ARG(isfinite(scale), "scale must be finite");
  const size_t ws_need = workspace_bytes(ph->num_partials, n_h);
  if (ph->num_partials > 0 && (workspace == nullptr || workspace_bytes_given < ws_need))
    return fail(MLA_ERR_WORKSPACE_TOO_SMALL, "workspace %zu B < %zu B", workspace_bytes_given,
                ws_need);
  mla_status_t st = require_sm100();
  if (st != MLA_OK) return st;
  DecodeArgs a;
  a.q_full = q_full;
  a.cache = static_cast<const uint16_t *>(cache);
  a.fp8_scales = fp8_scales;
  a.num_pages = num_pages;
  a.block_table = block_table;
  a.max_pages = max_pages;
  a.batch = batch;
  a.q_len = q_len;
  a.n_h = n_h;
  a.scale_log2 = scale * 1.4426950408889634f;
  a.plan_host = ph;
  a.plan_dev = static_cast<const unsigned char *>(plan_dev);
  a.ws_o = static_cast<float *>(workspace);
  a.ws_lse = workspace ? reinterpret_cast<float *>(static_cast<unsigned char *>(workspace) +
                                                   workspace_o_bytes(ph->num_partials, n_h))
                       : nullptr;
  a.o_latent = o_latent;
  a.lse = lse;
  a.status = status;
  st = kind == kCudaCore ? launch_decode_simt(a, (cudaStream_t)stream)
       : kind == kTensorCoreFp8 ? launch_decode_fp8(a, (cudaStream_t)stream)
                                : launch_decode(a, (cudaStream_t)stream);
  if (st != MLA_OK) return st;
  return launch_combine(a, (cudaStream_t)stream);
}

extern "C" {

mla_status_t mla_decode_attention(const mla_bf16_t *q_full, const mla_bf16_t *cache,
                                  int num_pages, const int32_t *block_table, int max_pages,
                                  int batch, int q_len, int n_h, float scale,
                                  const void *plan_host, const void *plan_dev, void *workspace,
                                  size_t workspace_bytes_given, mla_bf16_t *o_latent, float *lse,
                                  uint32_t *status, mla_stream_t stream) {
  return decode_entry(q_full, cache, num_pages, block_table, max_pages, batch, q_len, n_h, scale,
                      plan_host, plan_dev, workspace, workspace_bytes_given, o_latent, lse,
                      status, stream, kTensorCore);
}

mla_status_t mla_decode_attention_cudacore(const mla_bf16_t *q_full, const mla_bf16_t *cache,
                                           int num_pages, const int32_t *block_table,
                                           int max_pages, int batch, int q_len, int n_h,
                                           float scale, const void *plan_host,
                                           const void *plan_dev, void *workspace,
                                           size_t workspace_bytes_given, mla_bf16_t *o_latent,
                                           float *lse, uint32_t *status, mla_stream_t stream) {
  return decode_entry(q_full, cache, num_pages, block_table, max_pages, batch, q_len, n_h, scale,
                      plan_host, plan_dev, workspace, workspace_bytes_given, o_latent, lse,
                      status, stream, kCudaCore);
}

mla_status_t mla_decode_attention_fp8(const mla_bf16_t *q_full, const uint8_t *cache,
                                      const float *scales, int num_pages,
                                      const int32_t *block_table, int max_pages, int batch,
                                      int q_len, int n_h, float scale, const void *plan_host,
                                      const void *plan_dev, void *workspace,
                                      size_t workspace_bytes_given, mla_bf16_t *o_latent,
                                      float *lse, uint32_t *status, mla_stream_t stream) {
  return decode_entry(q_full, cache, num_pages, block_table, max_pages, batch, q_len, n_h, scale,
                      plan_host, plan_dev, workspace, workspace_bytes_given, o_latent, lse,
                      status, stream, kTensorCoreFp8, scales);
}

mla_status_t mla_cache_append_fp8(uint8_t *cache, float *scales, int num_pages,
                                  const int32_t *block_table, int batch, int max_pages,
                                  const int32_t *seq_idx, const int32_t *pos,
                                  const mla_bf16_t *c_kv, int ld_c, const mla_bf16_t *k_pe,
                                  int ld_k, const float *rope_table, int max_pos, int n_tokens,
                                  uint32_t *status, mla_stream_t stream) {
  clear_error();
  MLA_CHECK_ARG(n_tokens >= 0, "n_tokens < 0");
  if (n_tokens == 0) return MLA_OK;
  MLA_CHECK_ARG(cache && scales && block_table && seq_idx && pos && c_kv && k_pe && rope_table,
                "NULL device pointer");
  MLA_CHECK_ARG(num_pages > 0 && batch > 0 && max_pages > 0 && max_pos > 0,
                "sizes must be positive");
  MLA_CHECK_ARG(aligned16(cache) && aligned16(scales) && aligned16(c_kv) && aligned16(k_pe) &&
                    aligned16(rope_table),
                "cache, scales, c_kv, k_pe and rope_table must be 16-byte aligned");
  MLA_CHECK_ARG(ld_c >= MLA_D_C && ld_c % 8 == 0, "ld_c must be >= 512 and a multiple of 8");
  MLA_CHECK_ARG(ld_k >= MLA_D_R && ld_k % 8 == 0, "ld_k must be >= 64 and a multiple of 8");
  mla_status_t st = require_sm100();
  if (st != MLA_OK) return st;
  return launch_cache_append_fp8(cache, scales, num_pages, block_table, batch, max_pages, seq_idx,
                                 pos, c_kv, ld_c, k_pe, ld_k, rope_table, max_pos, n_tokens,
                                 status, (cudaStream_t)stream);
}

mla_status_t mla_debug_gemm_plan(int M, int N, int K, int batch, int a_mn, int c_fp32,
                                 int fp32_part, int atomic_split, int sms, int32_t *out) {
  clear_error();
  MLA_CHECK_ARG(out != nullptr, "NULL out");
  MLA_CHECK_ARG(M > 0 && N > 0 && K > 0 && batch > 0 && sms > 0, "non-positive size");
  const GemmPlan pl = plan_gemm(M, N, K, batch, a_mn != 0, c_fp32 != 0, fp32_part != 0,
                                atomic_split != 0, sms);
  out[0] = pl.BN;
  out[1] = pl.two_m ? 2 : 1;
  out[2] = pl.ntile;
  out[3] = pl.mtile;
  out[4] = pl.splits;
  out[5] = pl.k_chunks;
  out[6] = pl.part ? 1 : 0;
  out[7] = (int32_t)std::min<size_t>(pl.part_bytes, 0x7FFFFFFF);
  return MLA_OK;
}

mla_status_t mla_debug_decode_wait(double wait_cap_seconds, int suppress_arrive) {
  clear_error();
  return set_decode_wait(wait_cap_seconds, suppress_arrive);
}

mla_status_t mla_out_absorb(const mla_bf16_t *o_latent, const mla_bf16_t *w_uv, int T, int n_h,
                            mla_bf16_t *u, int ld_u, mla_stream_t stream) {
  clear_error();
  MLA_CHECK_ARG(T >= 0, "T < 0");
  if (T == 0) return MLA_OK;
  if (!heads_supported(n_h))
    return fail(MLA_ERR_UNSUPPORTED, "n_h = %d (supported: 16..128, multiple of 16)", n_h);
  MLA_CHECK_ARG(o_latent && w_uv && u, "NULL device pointer");
  MLA_CHECK_ARG(aligned16(o_latent) && aligned16(w_uv) && aligned16(u),
                "pointers must be 16-byte aligned");
  MLA_CHECK_ARG(ld_u >= n_h * MLA_D_V && ld_u % 8 == 0, "ld_u too small or unaligned");
  mla_status_t st = require_sm100();
  if (st != MLA_OK) return st;
  return launch_out_absorb(o_latent, w_uv, T, n_h, u, ld_u, (cudaStream_t)stream);
}

mla_status_t mla_gemm_bf16(const mla_bf16_t *X, int ld_x, const mla_bf16_t *W, int ld_w, void *C,
                           int ld_c, int c_fp32, int M, int N, int K, mla_stream_t stream) {
  return mla_gemm_bf16_ws(X, ld_x, W, ld_w, C, ld_c, c_fp32, M, N, K, nullptr, 0, stream);
}

size_t mla_gemm_bf16_workspace_bytes(int M, int N, int K) {
  if (M <= 0 || N <= 0 || K <= 0) return 0;
  // bf16 outputs accumulate a split in M*N floats; fp32 outputs keep one
  // partial tile per split (the projection GEMM: A = W with N rows, B = X)
  const size_t bf16_need = ((size_t)M * N * sizeof(float) + 255) & ~(size_t)255;
  int sms = 0;
  if (device_info(&sms, nullptr, nullptr) != MLA_OK) return bf16_need;
  return std::max(bf16_need, plan_gemm(N, M, K, 1, false, true, true, false, sms).part_bytes);
}

mla_status_t mla_gemm_bf16_ws(const mla_bf16_t *X, int ld_x, const mla_bf16_t *W, int ld_w,
                              void *C, int ld_c, int c_fp32, int M, int N, int K, void *workspace,
                              size_t workspace_bytes, mla_stream_t stream) {
  clear_error();
  MLA_CHECK_ARG(M >= 0 && N >= 0 && K >= 0, "negative size");
  if (M == 0 || N == 0) return MLA_OK;
  MLA_CHECK_ARG(X && W && C, "NULL device pointer");
  MLA_CHECK_ARG(K > 0, "K must be positive");
  if (K % 16 != 0) return fail(MLA_ERR_UNSUPPORTED, "K = %d (must be a multiple of 16)", K);
  MLA_CHECK_ARG(ld_x >= K && ld_w >= K && ld_c >= N, "leading dimension smaller than the row");
  MLA_CHECK_ARG(aligned16(X) && aligned16(W) && aligned16(C), "pointers must be 16-byte aligned");
  MLA_CHECK_ARG(ld_x % 8 == 0 && ld_w % 8 == 0 && ld_c % (c_fp32 ? 4 : 8) == 0,
                "leading dimensions must keep rows 16-byte aligned");
  MLA_CHECK_ARG(workspace == nullptr || aligned16(workspace), "workspace must be 16-byte aligned");
  mla_status_t st = require_sm100();
  if (st != MLA_OK) return st;
  const bool use_ws = workspace != nullptr &&
                      workspace_bytes >= mla_gemm_bf16_workspace_bytes(M, N, K);
  return launch_projection(X, ld_x, W, ld_w, C, ld_c, c_fp32, M, N, K,
                           use_ws ? static_cast<float *>(workspace) : nullptr,
                           use_ws ? workspace_bytes : 0, (cudaStream_t)stream);
}

size_t mla_plan_used_bytes(const void *plan_host) {
  if (plan_host == nullptr) return 0;
  const PlanHeader *ph = static_cast<const PlanHeader *>(plan_host);
  if (ph->magic != kPlanMagic || ph->version != kPlanVersion) return 0;
  return (size_t)ph->combine_off + (size_t)ph->num_combine * sizeof(CombineItem);
}

mla_status_t mla_plan_upload(const void *plan_host, void *plan_dev, size_t plan_dev_bytes,
                             mla_stream_t stream) {
  clear_error();
  MLA_CHECK_ARG(plan_host != nullptr && plan_dev != nullptr, "NULL plan pointer");
  MLA_CHECK_ARG(aligned16(plan_dev), "plan_dev must be 16-byte aligned");
  const size_t used = mla_plan_used_bytes(plan_host);
  MLA_CHECK_ARG(used > 0, "not a decode plan");
  if (plan_dev_bytes < used)
    return fail(MLA_ERR_WORKSPACE_TOO_SMALL, "device plan buffer %zu B < %zu B", plan_dev_bytes,
                used);
  MLA_CUDA_TRY(cudaMemcpyAsync(plan_dev, plan_host, used, cudaMemcpyHostToDevice,
                               (cudaStream_t)stream));
  return MLA_OK;
}

mla_status_t mla_check_status(uint32_t *status, uint32_t *bits, mla_stream_t stream) {
  return mla_read_status(status, bits, 0, stream);
}

mla_status_t mla_reset_status(uint32_t *status, mla_stream_t stream) {
  clear_error();
  MLA_CHECK_ARG(status != nullptr, "NULL status pointer");
  MLA_CUDA_TRY(cudaMemsetAsync(status, 0, sizeof(uint32_t), (cudaStream_t)stream));
  return MLA_OK;
}

mla_status_t mla_read_status(uint32_t *status, uint32_t *bits, int clear, mla_stream_t stream) {
  clear_error();
  MLA_CHECK_ARG(status != nullptr && bits != nullptr, "NULL pointer");
  cudaStream_t s = (cudaStream_t)stream;
  uint32_t v = 0;
  MLA_CUDA_TRY(cudaMemcpyAsync(&v, status, sizeof(v), cudaMemcpyDeviceToHost, s));
  MLA_CUDA_TRY(cudaStreamSynchronize(s));
  if (clear) {
    MLA_CUDA_TRY(cudaMemsetAsync(status, 0, sizeof(uint32_t), s));
    MLA_CUDA_TRY(cudaStreamSynchronize(s));
  }
  *bits = v;
  if (v != 0) return fail(MLA_ERR_DEVICE, "device status bits 0x%x", v);
  return MLA_OK;
}

}  // extern "C"
