// Plan stage: page tables and kv lengths -> load-balanced split-KV work list.
//
// FlashInfer README, core feature 2 ("Load-Balanced Scheduling"): the
// attention computation is split into a plan stage that schedules
// variable-length inputs and a run stage that computes; the same README
// names stream-K among the designs FlashInfer draws on.  The page gives no
// algorithm.  The specification implemented here (documented with
// pa_plan_create in pagedattn.h) is a stream-K style split: every group of
// Hkv CTAs gets an equal, contiguous share of the concatenated request
// tokens, one CTA per kv head.  Host code only: no CUDA call.
#include <algorithm>
#include <array>
#include <cmath>
#include <cstring>
#include <functional>
#include <new>
#include <queue>
#include <utility>

#include "pa_internal.h"

namespace {

bool is_pow2(int64_t x) { return x > 0 && (x & (x - 1)) == 0; }

int32_t ilog2(int64_t x) {
  int32_t r = 0;
  while ((int64_t(1) << r) < x) ++r;
  return r;
}

int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

pa_status validate_problem(const pa_problem* p) {
  if (!p) return PA_ERR_INVALID_ARG;
  if (p->batch < 0 || p->num_qo_heads <= 0 || p->num_kv_heads <= 0 || p->head_dim <= 0 ||
      p->page_size <= 0 || p->num_sms <= 0 || p->ctas_per_sm <= 0 || p->min_chunk_tokens < 0 ||
      p->num_pages < 0)
    return PA_ERR_INVALID_ARG;
  if (p->num_qo_heads % p->num_kv_heads) return PA_ERR_INVALID_ARG;
  if (!(p->sm_scale == p->sm_scale)) return PA_ERR_INVALID_ARG;  // NaN
  if (p->dtype != PA_F16 && p->dtype != PA_BF16) return PA_ERR_INVALID_ARG;
  if (p->kv_dtype != PA_F16 && p->kv_dtype != PA_BF16 && !pa::kv_is_8bit(*p))
    return PA_ERR_INVALID_ARG;
  if (pa::kv_is_8bit(*p) && !(std::isfinite(p->k_scale) && p->k_scale > 0.f &&
                              std::isfinite(p->v_scale) && p->v_scale > 0.f))
    return PA_ERR_INVALID_ARG;
  if (!(std::isfinite(p->rope_theta) && p->rope_theta >= 0.f)) return PA_ERR_INVALID_ARG;
  // rotary positions are built for the CUDA-core decode kernel only
  if (pa::decode_needs_cuda_cores(*p) && (p->flags & PA_FLAG_TENSOR_CORES) &&
      !(p->flags & PA_FLAG_CUDA_CORES))
    return PA_ERR_UNSUPPORTED;
  if (p->head_dim != pa::kHeadDim) return PA_ERR_UNSUPPORTED;
  if (!is_pow2(p->page_size) || p->page_size > 1024) return PA_ERR_UNSUPPORTED;
  if (!pa::decode_group_supported(p->num_qo_heads / p->num_kv_heads)) return PA_ERR_UNSUPPORTED;
  // pool rows (page * P + row) are 32-bit indices inside the kernels
  if (p->num_pages * int64_t(p->page_size) > int64_t(UINT32_MAX)) return PA_ERR_UNSUPPORTED;
  return PA_OK;
}

pa_status build(pa_plan_s* plan, const int32_t* indptr, const int32_t* last) {
  const pa_problem& p = plan->prob;
  const int64_t B = p.batch, P = p.page_size, Hkv = p.num_kv_heads;
  if (B > 0 && (!indptr || !last)) return PA_ERR_INVALID_ARG;
  if (indptr && indptr[0] != 0) return PA_ERR_INVALID_ARG;
  std::vector<int64_t> L(B);
  int64_t total = 0;
  for (int64_t b = 0; b < B; ++b) {
    if (indptr[b + 1] < indptr[b]) return PA_ERR_INVALID_ARG;
    const int64_t n = int64_t(indptr[b + 1]) - indptr[b];
    if (n > 0 && (last[b] < 1 || last[b] > P)) return PA_ERR_INVALID_ARG;
    L[b] = n > 0 ? (n - 1) * P + last[b] : 0;
    if (L[b] > INT32_MAX) return PA_ERR_UNSUPPORTED;
    // rotary positions are formed as exact fp32 integers in the kernel
    if (p.rope_theta > 0.f && L[b] > (int64_t(1) << 24)) return PA_ERR_UNSUPPORTED;
    total += L[b];
  }
  if (indptr) plan->kv_indptr.assign(indptr, indptr + B + 1);
  else plan->kv_indptr.assign(1, 0);
  plan->last_page_len.assign(last ? last : nullptr, last ? last + B : nullptr);

  // Token-level stream-K with a cost per piece: CTAs come in groups of Hkv
  // (one per kv head), so the Hkv CTAs of a group read the same pages at the
  // same time, each its own head.  Every group has the same budget q, filled
  // with the requests' tokens laid end to end; a piece that a group starts
  // after its first one (a new request) also charges c tokens, the measured
  // cost of a piece boundary (pipeline refill and epilogue) in token time.
  const int64_t W = int64_t(p.num_sms) * p.ctas_per_sm;
  const int64_t groups = std::max<int64_t>(1, W / Hkv);
  const int64_t min_tokens = p.min_chunk_tokens ? p.min_chunk_tokens : pa::kDefaultMinChunkTokens;
  const int64_t c = p.piece_cost_tokens > 0    ? p.piece_cost_tokens
                    : p.piece_cost_tokens == 0 ? pa::default_piece_cost_tokens(p)
                                               : 0;
  int64_t nonempty = 0;
  for (int64_t b = 0; b < B; ++b) nonempty += L[b] > 0;
  std::vector<std::vector<std::array<int64_t, 3>>> group_pieces;
  // The walk for budget q; returns the number of groups it fills.
  auto walk = [&](int64_t q) -> int64_t {
    group_pieces.assign(1, {});
    size_t g = 0;
    int64_t used = 0;
    bool has_piece = false;  // group g holds a non-empty piece
    for (int64_t b = 0; b < B; ++b) {
      if (L[b] == 0) {  // zero-length piece in the group the next token goes to
        const size_t target = has_piece && used + c >= q ? g + 1 : g;
        if (target == group_pieces.size()) group_pieces.emplace_back();
        group_pieces[target].push_back({b, 0, 0});
        continue;
      }
      int64_t t = 0;
      while (t < L[b]) {
        const int64_t cost = has_piece ? c : 0;
        if (has_piece && used + cost >= q) {  // the next token does not fit
          if (++g == group_pieces.size()) group_pieces.emplace_back();
          used = 0;
          has_piece = false;
          continue;
        }
        const int64_t take = std::min<int64_t>(L[b] - t, q - used - cost);
        group_pieces[g].push_back({b, t, t + take});
        used += cost + take;
        has_piece = true;
        t += take;
      }
    }
    // zero-length pieces past the last group with tokens join that group
    const size_t n = std::max<size_t>(1, g + 1);
    for (size_t k = n; k < group_pieces.size(); ++k)
      group_pieces[n - 1].insert(group_pieces[n - 1].end(), group_pieces[k].begin(),
                                 group_pieces[k].end());
    group_pieces.resize(n);
    return int64_t(n);
  };
  // q: the even share of the tokens plus one piece cost per further request.
  // The walk then always fits in `groups`: a group that closes with budget
  // left over (less than c) is followed by a group whose first piece starts
  // a request, a cost the share counted but the walk does not charge, so
  // (n_groups - 1) q < T + c (N - 1) <= groups q.
  const int64_t q = ceil_div(std::max<int64_t>(min_tokens,
                                               ceil_div(total + c * std::max<int64_t>(nonempty - 1, 0),
                                                        groups)),
                             32) * 32;
  if (q > INT32_MAX) return PA_ERR_UNSUPPORTED;
  int64_t n_groups = 0;
  if (B > 0) {
    n_groups = walk(q);
    if (n_groups > groups) return PA_ERR_UNSUPPORTED;  // cannot happen (see above)
  } else {
    group_pieces.clear();
  }
  plan->quota = int32_t(q);
  if (n_groups * Hkv > INT32_MAX) return PA_ERR_UNSUPPORTED;
  plan->items.clear();
  plan->cta_indptr.assign(size_t(n_groups * Hkv) + 1, 0);
  for (int64_t g = 0; g < n_groups; ++g)
    for (int64_t h = 0; h < Hkv; ++h) {
      for (const auto& pc : group_pieces[size_t(g)])
        plan->items.push_back(pa_work_item{int32_t(pc[0]), int32_t(h), indptr[pc[0]],
                                           int32_t(pc[1]), int32_t(pc[2]), -1});
      plan->cta_indptr[size_t(g * Hkv + h) + 1] = int32_t(plan->items.size());
    }

  // Partial slots: a segment (b, h) cut into k > 1 pieces owns k consecutive
  // slots, in token order (= work-list order, groups being in token order).
  std::vector<int32_t> count(size_t(B * Hkv), 0);
  for (const pa_work_item& it : plan->items) ++count[size_t(it.request * Hkv + it.kv_head)];
  plan->merge_indptr.assign(size_t(B * Hkv) + 1, 0);
  for (int64_t sgm = 0; sgm < B * Hkv; ++sgm)
    plan->merge_indptr[sgm + 1] =
        plan->merge_indptr[sgm] + (count[size_t(sgm)] > 1 ? count[size_t(sgm)] : 0);
  std::vector<int32_t> seen(size_t(B * Hkv), 0);
  for (pa_work_item& it : plan->items) {
    const int64_t sgm = int64_t(it.request) * Hkv + it.kv_head;
    if (count[size_t(sgm)] > 1) it.partial_slot = plan->merge_indptr[sgm] + seen[size_t(sgm)]++;
  }
  plan->n_partials = plan->merge_indptr.back();
  return PA_OK;
}

void layout_workspace(pa_plan_s* plan) {
  const pa_problem& p = plan->prob;
  pa::WorkspaceLayout& w = plan->ws;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    size_t at = off;
    off = pa::align_up(off + bytes);
    return at;
  };
  const size_t Hq = p.num_qo_heads, D = p.head_dim, B = p.batch;
  w.items = take(plan->items.size() * sizeof(pa_work_item));
  w.prefill_tiles = take(plan->prefill_tiles.size() * sizeof(pa_prefill_tile));
  w.prefill_sched = take(plan->prefill_sched.size() * sizeof(int32_t));
  w.cta_indptr = take(plan->cta_indptr.size() * sizeof(int32_t));
  w.merge_indptr = take(plan->merge_indptr.size() * sizeof(int32_t));
  w.kv_len = take(p.rope_theta > 0.f && !plan->prefill ? B * sizeof(int32_t) : 0);
  w.counters = take(plan->prefill ? 0 : B * p.num_kv_heads * pa::kCounterSlots * sizeof(int32_t));
  w.error = take(2 * sizeof(uint64_t));  // first bad index, timeout flag
  const size_t G = plan->group;
  w.partial_o = take(size_t(plan->n_partials) * G * D * sizeof(float));
  w.partial_lse = take(size_t(plan->n_partials) * G * sizeof(float));
  w.prefix_o = take(size_t(plan->prefix_chunks) * B * Hq * D * sizeof(float));
  w.prefix_lse = take(size_t(plan->prefix_chunks) * B * Hq * sizeof(float));
  w.total = off;
}

void build_upload_image(pa_plan_s* plan) {
  const pa::WorkspaceLayout& w = plan->ws;
  std::vector<uint8_t>& img = plan->upload_image;
  img.assign(w.partial_o, 0);  // counters stay zero
  if (!plan->items.empty())
    std::memcpy(img.data() + w.items, plan->items.data(), plan->items.size() * sizeof(pa_work_item));
  if (!plan->prefill_tiles.empty())
    std::memcpy(img.data() + w.prefill_tiles, plan->prefill_tiles.data(),
                plan->prefill_tiles.size() * sizeof(pa_prefill_tile));
  if (!plan->prefill_sched.empty())
    std::memcpy(img.data() + w.prefill_sched, plan->prefill_sched.data(),
                plan->prefill_sched.size() * sizeof(int32_t));
  std::memcpy(img.data() + w.cta_indptr, plan->cta_indptr.data(),
              plan->cta_indptr.size() * sizeof(int32_t));
  std::memcpy(img.data() + w.merge_indptr, plan->merge_indptr.data(),
              plan->merge_indptr.size() * sizeof(int32_t));
  if (plan->prob.rope_theta > 0.f && !plan->prefill) {
    const pa_problem& p = plan->prob;
    for (int32_t b = 0; b < p.batch; ++b) {
      const int64_t n = int64_t(plan->kv_indptr[b + 1]) - plan->kv_indptr[b];
      const int32_t L = n > 0 ? int32_t((n - 1) * p.page_size + plan->last_page_len[b]) : 0;
      std::memcpy(img.data() + w.kv_len + b * sizeof(int32_t), &L, sizeof L);
    }
  }
  std::memset(img.data() + w.error, 0xff, sizeof(uint64_t));  // first bad index: none
}

// Level-1 cascade schedule: (kv head, pair of 128-row query tiles, prefix
// chunk) CTAs, about one per SM; the prefix's 128-key tiles are split as
// evenly as possible over the chunks (the largest chunk has ceil(tiles /
// chunks) of them).
void schedule_prefix(pa_plan_s* plan) {
  const pa_problem& p = plan->prob;
  constexpr int64_t kTileKeys = 128, kRowsPerCta = 256;
  const int64_t rows = int64_t(p.batch) * plan->group;
  plan->q_tiles = int32_t(std::max<int64_t>(1, ceil_div(rows, kRowsPerCta)));
  const int64_t key_tiles = ceil_div(plan->prefix_len, kTileKeys);
  if (plan->prefix_len == 0 || p.batch == 0) {
    plan->prefix_chunks = 0;
    plan->prefix_chunk_tokens = 0;
    return;
  }
  const int64_t base = int64_t(p.num_kv_heads) * plan->q_tiles;
  const int64_t chunks = std::max<int64_t>(1, std::min<int64_t>(int64_t(p.num_sms) / base, key_tiles));
  plan->prefix_chunks = int32_t(chunks);
  plan->prefix_chunk_tokens = int32_t(ceil_div(key_tiles, chunks) * kTileKeys);
}

// Prefill CTAs are persistent: min(num_sms, items) CTAs, each running a list
// of (tile, kv head) items (item w = tile * Hkv + kv head).  The items are
// dealt in the plan's tile order by list scheduling: each goes to the CTA
// whose estimated load is least (ties to the lower CTA), the load of an item
// being the 128-key tiles its two 128-row halves compute plus a fixed
// per-item cost.  The CTAs running at a time thus work on neighbouring items
// of that order (a request's tiles share its K/V in L2), as a launch of one
// CTA per item would, and the per-CTA lists end within about one item of
// each other.
constexpr int64_t kPrefillItemCostTiles = 2;  // fill and drain of one item, in key tiles

int64_t prefill_item_tiles(const pa_prefill_tile& t, int32_t group) {
  constexpr int64_t kTileKeys = 128;
  const int64_t per_half = 128 / group;
  const int64_t nq0 = std::min<int64_t>(t.n_q, per_half), nq1 = t.n_q - nq0;
  const int64_t nt0 = ceil_div(std::min<int64_t>(int64_t(t.kv_base) + nq0, t.kv_end), kTileKeys);
  const int64_t nt1 = nq1 > 0 ? ceil_div(t.kv_end, kTileKeys) : 0;
  return nt0 + nt1;
}

void schedule_prefill(pa_plan_s* plan) {
  const int64_t H = plan->prob.num_kv_heads;
  const int64_t n_items = int64_t(plan->prefill_tiles.size()) * H;
  const int64_t n_cta = std::min<int64_t>(plan->prob.num_sms, n_items);
  std::vector<std::vector<int32_t>> lists(size_t(std::max<int64_t>(n_cta, 0)));
  using Load = std::pair<int64_t, int64_t>;  // (estimated load, CTA)
  std::priority_queue<Load, std::vector<Load>, std::greater<Load>> least;
  for (int64_t c = 0; c < n_cta; ++c) least.push({0, c});
  for (int64_t w = 0; w < n_items; ++w) {
    const pa_prefill_tile& t = plan->prefill_tiles[size_t(w / H)];
    const Load top = least.top();
    least.pop();
    lists[size_t(top.second)].push_back(int32_t(w));
    least.push({top.first + prefill_item_tiles(t, plan->group) + kPrefillItemCostTiles,
                top.second});
  }
  plan->prefill_sched.clear();
  plan->prefill_sched.reserve(size_t(n_items));
  plan->cta_indptr.assign(1, 0);
  for (const std::vector<int32_t>& l : lists) {
    plan->prefill_sched.insert(plan->prefill_sched.end(), l.begin(), l.end());
    plan->cta_indptr.push_back(int32_t(plan->prefill_sched.size()));
  }
}

// Prefill / append tiles: each request's new tokens cut into runs of 256 / G
// (two 128-row tensor-core tiles of (token, q head) rows per kv head, one CTA).
// A request's tiles are listed together (the CTAs running at a time then share
// its K/V in L2), requests in decreasing order of their longest tile, and the
// tiles of a request longest first; lengths count 128-key tiles.
pa_status build_prefill(pa_plan_s* plan, bool causal, const int32_t* qo, const int32_t* indptr,
                        const int32_t* last) {
  const pa_problem& p = plan->prob;
  const int64_t B = p.batch, P = p.page_size;
  if (B > 0 && (!qo || !indptr || !last)) return PA_ERR_INVALID_ARG;
  if ((qo && qo[0] != 0) || (indptr && indptr[0] != 0)) return PA_ERR_INVALID_ARG;
  const int64_t per_tile = 256 / plan->group;
  constexpr int64_t kTileKeys = 128;
  std::vector<pa_prefill_tile> tiles;
  for (int64_t b = 0; b < B; ++b) {
    if (indptr[b + 1] < indptr[b] || qo[b + 1] < qo[b]) return PA_ERR_INVALID_ARG;
    const int64_t n = int64_t(indptr[b + 1]) - indptr[b];
    if (n > 0 && (last[b] < 1 || last[b] > P)) return PA_ERR_INVALID_ARG;
    const int64_t L = n > 0 ? (n - 1) * P + last[b] : 0;
    if (L > INT32_MAX) return PA_ERR_UNSUPPORTED;
    const int64_t Q = int64_t(qo[b + 1]) - qo[b];
    if (causal && Q > L) return PA_ERR_INVALID_ARG;
    for (int64_t t0 = 0; t0 < Q; t0 += per_tile) {
      const int64_t nq = std::min(per_tile, Q - t0);
      const int64_t base = causal ? L - Q + t0 : L - 1;
      const int64_t end = causal ? base + nq : L;
      tiles.push_back(pa_prefill_tile{int32_t(b), int32_t(qo[b] + t0), int32_t(nq), indptr[b],
                                      int32_t(base), int32_t(end)});
    }
  }
  std::vector<int64_t> longest(size_t(B), 0);
  for (const pa_prefill_tile& t : tiles)
    longest[size_t(t.request)] = std::max(longest[size_t(t.request)], ceil_div(t.kv_end, kTileKeys));
  std::stable_sort(tiles.begin(), tiles.end(),
                   [&](const pa_prefill_tile& x, const pa_prefill_tile& y) {
                     const int64_t lx = longest[size_t(x.request)], ly = longest[size_t(y.request)];
                     if (lx != ly) return lx > ly;
                     if (x.request != y.request) return x.request < y.request;
                     return ceil_div(x.kv_end, kTileKeys) > ceil_div(y.kv_end, kTileKeys);
                   });
  plan->prefill_tiles = std::move(tiles);
  plan->total_q = B > 0 ? qo[B] : 0;
  if (B > 0) plan->kv_indptr.assign(indptr, indptr + B + 1);
  else plan->kv_indptr.assign(1, 0);
  plan->last_page_len.assign(last ? last : nullptr, last ? last + B : nullptr);
  if (B > 0) plan->qo_indptr.assign(qo, qo + B + 1);
  else plan->qo_indptr.assign(1, 0);
  plan->merge_indptr.assign(1, 0);
  if (plan->prefill_tiles.size() * size_t(p.num_kv_heads) > size_t(INT32_MAX))
    return PA_ERR_UNSUPPORTED;
  schedule_prefill(plan);
  return PA_OK;
}

enum class Mode { kDecode, kCascade, kPrefill };

pa_status create(const pa_problem* problem, int32_t prefix_len, Mode mode, bool causal,
                 const int32_t* qo, const int32_t* indptr, const int32_t* last, pa_plan_t* out) {
  const bool cascade = mode == Mode::kCascade;
  if (!out) return PA_ERR_INVALID_ARG;
  *out = nullptr;
  pa_status st = validate_problem(problem);
  if (st != PA_OK) return st;
  if (cascade && (prefix_len < 0 || prefix_len % problem->page_size)) return PA_ERR_INVALID_ARG;
  // the prefix level and prefill read 16-bit pools with TMA, without rotation
  if (((cascade && prefix_len > 0) || mode == Mode::kPrefill) && pa::decode_f32_path(*problem))
    return PA_ERR_UNSUPPORTED;
  // the prefix level moves whole pages (>= 8 rows) with TMA, whose row
  // coordinates are signed 32-bit
  if (((cascade && prefix_len > 0) || mode == Mode::kPrefill) &&
      (!pa::cascade_page_size_supported(problem->page_size) ||
       problem->num_pages * int64_t(problem->page_size) >= int64_t(INT32_MAX)))
    return PA_ERR_UNSUPPORTED;
  pa_plan_s* plan = new (std::nothrow) pa_plan_s;
  if (!plan) return PA_ERR_NO_MEMORY;
  try {
    plan->prob = *problem;
    if (plan->prob.min_chunk_tokens == 0) plan->prob.min_chunk_tokens = pa::kDefaultMinChunkTokens;
    plan->group = problem->num_qo_heads / problem->num_kv_heads;
    plan->log2_page = ilog2(problem->page_size);
    plan->cascade = cascade;
    plan->prefill = mode == Mode::kPrefill;
    plan->prefix_len = cascade ? prefix_len : 0;
    st = plan->prefill ? build_prefill(plan, causal, qo, indptr, last) : build(plan, indptr, last);
    if (st == PA_OK) {
      if (cascade) schedule_prefix(plan);
      layout_workspace(plan);
      build_upload_image(plan);
    }
  } catch (const std::bad_alloc&) {
    st = PA_ERR_NO_MEMORY;
  }
  if (st != PA_OK) {
    delete plan;
    return st;
  }
  *out = plan;
  return PA_OK;
}

}  // namespace

extern "C" {

pa_status pa_plan_create(const pa_problem* problem, const int32_t* kv_indptr_host,
                         const int32_t* last_page_len_host, pa_plan_t* out) {
  return create(problem, 0, Mode::kDecode, false, nullptr, kv_indptr_host, last_page_len_host,
                out);
}

pa_status pa_cascade_plan_create(const pa_problem* problem, int32_t prefix_len,
                                 const int32_t* kv_indptr_host,
                                 const int32_t* last_page_len_host, pa_plan_t* out) {
  return create(problem, prefix_len, Mode::kCascade, false, nullptr, kv_indptr_host,
                last_page_len_host, out);
}

pa_status pa_prefill_plan_create(const pa_problem* problem, int32_t causal,
                                 const int32_t* qo_indptr_host, const int32_t* kv_indptr_host,
                                 const int32_t* last_page_len_host, pa_plan_t* out) {
  return create(problem, 0, Mode::kPrefill, causal != 0, qo_indptr_host, kv_indptr_host,
                last_page_len_host, out);
}

pa_status pa_plan_prefill_tiles(pa_plan_t plan, const pa_prefill_tile** tiles, int64_t* n_tiles) {
  if (!plan || !tiles || !n_tiles) return PA_ERR_INVALID_ARG;
  *tiles = plan->prefill_tiles.data();
  *n_tiles = int64_t(plan->prefill_tiles.size());
  return PA_OK;
}

pa_status pa_plan_prefill_schedule(pa_plan_t plan, const int32_t** items, int64_t* n_items) {
  if (!plan || !items || !n_items) return PA_ERR_INVALID_ARG;
  *items = plan->prefill_sched.data();
  *n_items = int64_t(plan->prefill_sched.size());
  return PA_OK;
}

pa_status pa_plan_quota_tokens(pa_plan_t plan, int32_t* quota) {
  if (!plan || !quota) return PA_ERR_INVALID_ARG;
  *quota = plan->quota;
  return PA_OK;
}

pa_status pa_plan_cta_indptr(pa_plan_t plan, const int32_t** cta_indptr, int64_t* n_cta) {
  if (!plan || !cta_indptr || !n_cta) return PA_ERR_INVALID_ARG;
  *cta_indptr = plan->cta_indptr.data();
  *n_cta = int64_t(plan->cta_indptr.size()) - 1;
  return PA_OK;
}

pa_status pa_plan_work_items(pa_plan_t plan, const pa_work_item** items, int64_t* n_items) {
  if (!plan || !items || !n_items) return PA_ERR_INVALID_ARG;
  *items = plan->items.data();
  *n_items = int64_t(plan->items.size());
  return PA_OK;
}

pa_status pa_plan_merge_indptr(pa_plan_t plan, const int32_t** merge_indptr) {
  if (!plan || !merge_indptr) return PA_ERR_INVALID_ARG;
  *merge_indptr = plan->merge_indptr.data();
  return PA_OK;
}

pa_status pa_plan_num_partials(pa_plan_t plan, int64_t* n_partials) {
  if (!plan || !n_partials) return PA_ERR_INVALID_ARG;
  *n_partials = plan->n_partials;
  return PA_OK;
}

pa_status pa_plan_prefix_chunks(pa_plan_t plan, int32_t* n_chunks, int32_t* chunk_tokens) {
  if (!plan || !n_chunks || !chunk_tokens) return PA_ERR_INVALID_ARG;
  *n_chunks = plan->prefix_chunks;
  *chunk_tokens = plan->prefix_chunk_tokens;
  return PA_OK;
}

pa_status pa_plan_status_offset(pa_plan_t plan, size_t* offset) {
  if (!plan || !offset) return PA_ERR_INVALID_ARG;
  *offset = plan->ws.error;
  return PA_OK;
}

pa_status pa_plan_workspace_bytes(pa_plan_t plan, size_t* bytes) {
  if (!plan || !bytes) return PA_ERR_INVALID_ARG;
  *bytes = plan->ws.total;
  return PA_OK;
}

void pa_plan_destroy(pa_plan_t plan) { delete plan; }

const char* pa_status_string(pa_status s) {
  switch (s) {
    case PA_OK: return "ok";
    case PA_ERR_INVALID_ARG: return "invalid argument";
    case PA_ERR_UNSUPPORTED: return "unsupported shape or type";
    case PA_ERR_WORKSPACE_TOO_SMALL: return "workspace too small";
    case PA_ERR_CUDA: return "CUDA error";
    case PA_ERR_DEVICE_CHECK: return "device check failed: page index out of range";
    case PA_ERR_NO_MEMORY: return "host allocation failed";
    case PA_ERR_DEVICE_TIMEOUT: return "a kernel abandoned a bounded wait";
  }
  return "unknown status";
}

int32_t pa_plan_uses_tensor_cores(pa_plan_t plan) {
  if (!plan) return -1;
  return plan->prefill ? 1 : int32_t(pa::decode_uses_tensor_cores(plan->prob));
}

int32_t pa_abi_version(void) { return PA_ABI_VERSION; }

}  // extern "C"
