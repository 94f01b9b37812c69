// Host planner: descriptor validation, per-row key limits, tile classes, work list.
//
// The visibility rules follow the pages: HiDream-O1 ("hidream-o1-p100a" model card, "What
// this model is"; "HiDream-O1-Image" summary, "How it works") -- text and condition tokens
// causal, generation tokens see the whole sequence; HunyuanImage 3.0 Generalized Causal
// Attention (paper-graph-ui summary, section 3.4, "The core rule") -- image tokens see all
// previous tokens and their whole segment. Under each rule the keys a row sees form a
// prefix, so one exclusive limit per row describes the mask exactly:
//   causal: i + 1;  full_sequence: L;  full_in_segment and gen_image: end of i's segment.
// HunyuanImage 3.0 multi-Gen-Image training (section 3.4, "The multi-generation training
// complication", Figure 4(b)): the keys of a gen_image segment are hidden from every row of
// a later segment. Those "holes" lie inside the row's prefix; rows that have them get a
// bit mask of hidden keys per key block, and their work items an explicit key-block list.
#include "planner.h"

#include <algorithm>
#include <cmath>
#include <cstdio>
#include <functional>
#include <queue>

namespace hgx {

namespace {

std::string fmt(const char* f, long long a = 0, long long b = 0, long long c = 0) {
  char buf[256];
  std::snprintf(buf, sizeof(buf), f, a, b, c);
  return buf;
}

}  // namespace

hgx_status validate_descriptor(int32_t batch, const int32_t* cu_seqlens,
                               const hgx_segment* segs, const int32_t* cu_segs,
                               std::string* err, int32_t* total_tokens) {
  *total_tokens = 0;
  if (batch < 0) {
    *err = "batch must be >= 0";
    return HGX_ERR_INVALID_ARG;
  }
  if (batch == 0) return HGX_OK;
  if (!cu_seqlens || !cu_segs) {
    *err = "cu_seqlens and cu_segs must be non-null";
    return HGX_ERR_INVALID_ARG;
  }
  if (cu_seqlens[0] != 0 || cu_segs[0] != 0) {
    *err = "cu_seqlens[0] and cu_segs[0] must be 0";
    return HGX_ERR_INVALID_ARG;
  }
  for (int32_t b = 0; b < batch; ++b) {
    if (cu_seqlens[b + 1] < cu_seqlens[b]) {
      *err = fmt("cu_seqlens decreases at batch element %lld", b);
      return HGX_ERR_INVALID_ARG;
    }
    if (cu_seqlens[b + 1] > kMaxTokens) {
      *err = fmt("total tokens %lld exceed the maximum %lld", cu_seqlens[b + 1], kMaxTokens);
      return HGX_ERR_INVALID_ARG;
    }
    if (cu_segs[b + 1] < cu_segs[b]) {
      *err = fmt("cu_segs decreases at batch element %lld", b);
      return HGX_ERR_INVALID_ARG;
    }
  }
  if (cu_segs[batch] > 0 && !segs) {
    *err = "segs must be non-null";
    return HGX_ERR_INVALID_ARG;
  }
  for (int32_t b = 0; b < batch; ++b) {
    const int32_t L = cu_seqlens[b + 1] - cu_seqlens[b];
    int32_t at = 0;
    for (int32_t s = cu_segs[b]; s < cu_segs[b + 1]; ++s) {
      const hgx_segment& sg = segs[s];
      if (sg.kind < HGX_SEG_CAUSAL || sg.kind > HGX_SEG_GEN_IMAGE) {
        *err = fmt("segment %lld has invalid kind %lld", s, sg.kind);
        return HGX_ERR_INVALID_ARG;
      }
      if (sg.len < 1) {
        *err = fmt("segment %lld has length %lld (must be >= 1)", s, sg.len);
        return HGX_ERR_INVALID_ARG;
      }
      if (sg.start != at) {
        *err = fmt("segment %lld starts at %lld, expected %lld (segments must tile the "
                   "batch element in order)", s, sg.start, at);
        return HGX_ERR_INVALID_ARG;
      }
      if (sg.len > L - at) {
        *err = fmt("segment %lld runs past the end of batch element %lld", s, b);
        return HGX_ERR_INVALID_ARG;
      }
      at += sg.len;
    }
    if (at != L) {
      *err = fmt("segments of batch element %lld cover %lld of %lld tokens", b, at, L);
      return HGX_ERR_INVALID_ARG;
    }
  }
  *total_tokens = cu_seqlens[batch];
  return HGX_OK;
}

hgx_status row_limits(int32_t batch, const int32_t* cu_seqlens, const hgx_segment* segs,
                      const int32_t* cu_segs, std::vector<int32_t>* lim, std::string* err) {
  int32_t T = 0;
  hgx_status st = validate_descriptor(batch, cu_seqlens, segs, cu_segs, err, &T);
  if (st != HGX_OK) return st;
  lim->assign(static_cast<size_t>(T), 0);
  for (int32_t b = 0; b < batch; ++b) {
    const int32_t base = cu_seqlens[b];
    const int32_t L = cu_seqlens[b + 1] - base;
    for (int32_t s = cu_segs[b]; s < cu_segs[b + 1]; ++s) {
      const hgx_segment& sg = segs[s];
      for (int32_t i = sg.start; i < sg.start + sg.len; ++i) {
        int32_t l = 0;
        switch (sg.kind) {
          case HGX_SEG_CAUSAL: l = i + 1; break;
          case HGX_SEG_FULL_SEQUENCE: l = L; break;
          default: l = sg.start + sg.len; break;  // full_in_segment, gen_image
        }
        (*lim)[static_cast<size_t>(base + i)] = l;
      }
    }
  }
  return HGX_OK;
}

hgx_status check_first_rows(int32_t batch, const int32_t* cu_seqlens, const hgx_segment* segs,
                            const int32_t* cu_segs, const int32_t* first_rows, std::string* err) {
  if (batch > 0 && !first_rows) {
    *err = "first_rows must be non-null";
    return HGX_ERR_INVALID_ARG;
  }
  std::vector<int32_t> lim;
  hgx_status st = row_limits(batch, cu_seqlens, segs, cu_segs, &lim, err);
  if (st != HGX_OK) return st;
  for (int32_t b = 0; b < batch; ++b) {
    const int32_t L = cu_seqlens[b + 1] - cu_seqlens[b], f = first_rows[b];
    if (f < 0 || f > L) {
      *err = fmt("first row %lld of batch element %lld is outside [0, %lld]", f, b, L);
      return HGX_ERR_INVALID_ARG;
    }
    for (int32_t i = 0; i < f; ++i)
      if (lim[static_cast<size_t>(cu_seqlens[b] + i)] > f) {
        *err = fmt("row %lld of batch element %lld is reused but sees key %lld, which is "
                   "recomputed", i, b, f);
        return HGX_ERR_INVALID_ARG;
      }
  }
  return HGX_OK;
}

namespace {

int popcount4(const uint32_t* m) {
  return __builtin_popcount(m[0]) + __builtin_popcount(m[1]) + __builtin_popcount(m[2]) +
         __builtin_popcount(m[3]);
}

}  // namespace

hgx_status build_plan(int32_t batch, const int32_t* cu_seqlens, const hgx_segment* segs,
                      const int32_t* cu_segs, int32_t num_kv_heads, Plan* plan,
                      std::string* err, const int32_t* first_rows) {
  hgx_status st = row_limits(batch, cu_seqlens, segs, cu_segs, &plan->lim, err);
  if (st != HGX_OK) return st;
  if (first_rows && (st = check_first_rows(batch, cu_seqlens, segs, cu_segs, first_rows, err)) != HGX_OK)
    return st;
  plan->batch = batch;
  plan->total_tokens = batch ? cu_seqlens[batch] : 0;
  plan->items.clear();
  plan->kblocks.clear();
  plan->hole_base.clear();
  plan->hole_masks.clear();
  plan->has_holes = false;
  plan->visible_pairs = 0;
  for (int32_t b = 0; b < batch; ++b)
    for (int32_t i = first_rows ? first_rows[b] : 0; i < cu_seqlens[b + 1] - cu_seqlens[b]; ++i)
      plan->visible_pairs += static_cast<uint64_t>(plan->lim[static_cast<size_t>(cu_seqlens[b] + i)]);
  for (int32_t s = 0; batch > 0 && s < cu_segs[batch]; ++s)
    if (segs[s].kind == HGX_SEG_GEN_IMAGE) plan->has_holes = true;
  if (plan->has_holes) plan->hole_base.assign(static_cast<size_t>(plan->total_tokens), -1);

  std::vector<uint8_t> cls;  // classes of one query block, per key block
  for (int32_t b = 0; b < batch; ++b) {
    const int32_t base = cu_seqlens[b];
    const int32_t L = cu_seqlens[b + 1] - base;
    const int32_t nkb = (L + kBlockKeys - 1) / kBlockKeys;
    // hole masks: one 128-bit mask per key block for every segment preceded by a Gen Image
    if (plan->has_holes) {
      std::vector<std::pair<int32_t, int32_t>> gens;  // earlier gen_image segments
      for (int32_t s = cu_segs[b]; s < cu_segs[b + 1]; ++s) {
        const hgx_segment& sg = segs[s];
        if (!gens.empty()) {
          const int32_t mbase = static_cast<int32_t>(plan->hole_masks.size() / 4);
          plan->hole_masks.resize(plan->hole_masks.size() + 4 * static_cast<size_t>(nkb), 0u);
          uint32_t* m = plan->hole_masks.data() + 4 * static_cast<size_t>(mbase);
          int64_t hidden = 0;
          for (const auto& gsg : gens) {
            hidden += gsg.second - gsg.first;
            for (int32_t key = gsg.first; key < gsg.second; ++key)
              m[4 * (key / kBlockKeys) + (key % kBlockKeys) / 32] |= 1u << (key % 32);
          }
          for (int32_t i = sg.start; i < sg.start + sg.len; ++i) {
            plan->hole_base[static_cast<size_t>(base + i)] = mbase;
            if (!first_rows || i >= first_rows[b]) plan->visible_pairs -= static_cast<uint64_t>(hidden);
          }
        }
        if (sg.kind == HGX_SEG_GEN_IMAGE) gens.emplace_back(sg.start, sg.start + sg.len);
      }
    }
    const int32_t first = first_rows ? first_rows[b] : 0;
    for (int32_t r0 = first / kBlockTokens * kBlockTokens; r0 < L; r0 += kBlockTokens) {
      const int32_t r1 = std::min(L, r0 + kBlockTokens);
      int32_t lo = INT32_MAX, hi = 0;
      bool holes = false;
      for (int32_t i = r0; i < r1; ++i) {
        const int32_t l = plan->lim[static_cast<size_t>(base + i)];
        lo = std::min(lo, l);
        hi = std::max(hi, l);
        if (plan->has_holes && plan->hole_base[static_cast<size_t>(base + i)] >= 0) holes = true;
      }
      WorkItem it{};
      it.q0 = base + r0;
      it.kv0 = base;
      it.len = L;
      it.list_off = -1;
      it.first = first;
      if (!holes) {
        it.n_full = lo / kBlockKeys;
        it.n_total = (hi + kBlockKeys - 1) / kBlockKeys;
      } else {
        // classify every key block from each row's visible count
        cls.assign(static_cast<size_t>(nkb), HGX_TILE_SKIP);
        for (int32_t kb = 0; kb < nkb; ++kb) {
          bool all_full = true, all_empty = true;
          for (int32_t i = r0; i < r1; ++i) {
            const int32_t l = plan->lim[static_cast<size_t>(base + i)];
            int32_t vis = std::max(0, std::min(kBlockKeys, l - kb * kBlockKeys));
            const int32_t hb = plan->hole_base[static_cast<size_t>(base + i)];
            // hidden keys lie before the row's own segment, so inside [0, lim)
            if (hb >= 0) vis -= popcount4(plan->hole_masks.data() + 4 * static_cast<size_t>(hb + kb));
            all_full = all_full && vis == kBlockKeys;
            all_empty = all_empty && vis == 0;
          }
          cls[static_cast<size_t>(kb)] = all_full ? HGX_TILE_FULL : all_empty ? HGX_TILE_SKIP : HGX_TILE_PARTIAL;
        }
        it.n_full = -1;
        it.list_off = static_cast<int32_t>(plan->kblocks.size());
        for (int32_t kb = 0; kb < nkb; ++kb)
          if (cls[static_cast<size_t>(kb)] != HGX_TILE_SKIP)
            plan->kblocks.push_back(static_cast<uint32_t>(kb) |
                                    (static_cast<uint32_t>(cls[static_cast<size_t>(kb)]) << kListClassShift));
        it.n_total = static_cast<int32_t>(plan->kblocks.size()) - it.list_off;
      }
      for (int32_t g = 0; g < num_kv_heads; ++g) {
        it.g = g;
        plan->items.push_back(it);
      }
    }
  }
  std::stable_sort(plan->items.begin(), plan->items.end(),
                   [](const WorkItem& a, const WorkItem& b) { return a.n_total > b.n_total; });
  return HGX_OK;
}

namespace {

// Cost of a work item in the schedule, in tenths of a fully visible key block: the kernel's
// cycles per CTA fit a fully visible block at ~3060 cycles, a block that runs the per-score
// mask compare (PARTIAL) at ~3900 and an item's own overhead (Q load, pipeline fill,
// epilogue) at ~2100-3600 (B200, per-CTA clock64 counts on the edit step and the CFG pairs).
constexpr int64_t kFullCost = 10, kPartialCost = 13;
constexpr int64_t kPartOverhead = 30;  // an extra item's Q load, pipeline fill and epilogue, plus its share of the combine
constexpr int32_t kMinPartBlocks = 2;

// kblocks: the plan's key-block lists (entries of list-form items carry their class)
int64_t block_cost(const WorkItem& it, const uint32_t* kblocks) {
  int64_t nf = 0;
  if (it.list_off >= 0) {
    for (int32_t j = 0; j < it.n_total; ++j)
      nf += (kblocks[it.list_off + j] >> kListClassShift) == HGX_TILE_FULL;
  } else {
    nf = std::min<int64_t>(std::max<int64_t>(it.n_full - it.kb0, 0), it.n_total);
  }
  return nf * kFullCost + (it.n_total - nf) * kPartialCost;
}

int64_t item_cost(const WorkItem& it, const uint32_t* kblocks) {
  return block_cost(it, kblocks) + (it.part >= 0 ? kPartOverhead : kItemOverhead);
}

// Longest processing time first; items are sorted by decreasing cost. Returns the owner of
// every item and the makespan.
int64_t lpt(const std::vector<WorkItem>& items, int32_t g, std::vector<int32_t>* owner, const uint32_t* kblocks) {
  using Load = std::pair<int64_t, int32_t>;  // (load, cta)
  std::priority_queue<Load, std::vector<Load>, std::greater<Load>> heap;
  for (int32_t c = 0; c < g; ++c) heap.push({0, c});
  owner->assign(items.size(), 0);
  int64_t makespan = 0;
  for (size_t i = 0; i < items.size(); ++i) {
    Load l = heap.top();
    heap.pop();
    (*owner)[i] = l.second;
    l.first += item_cost(items[i], kblocks);
    makespan = std::max(makespan, l.first);
    heap.push(l);
  }
  return makespan;
}

// Tail split: start from the longest-first assignment; every CTA loaded above the target
// (the mean load plus one item overhead) gives back its last -- smallest -- items as long as
// they can be split (prefix form, two or more key blocks), and the key blocks of those items
// are handed out in parts, each part to the least-loaded CTA as much as fits under the
// target (at least kMinPartBlocks). An item that ends up in one part stays whole.
int64_t tail_split(const std::vector<WorkItem>& items, int32_t g, const std::vector<int32_t>& owner,
                   std::vector<std::vector<WorkItem>>* lists, std::vector<WorkItem>* splits,
                   const uint32_t* kblocks) {
  lists->assign(static_cast<size_t>(g), {});
  std::vector<int64_t> load(static_cast<size_t>(g), 0);
  int64_t total = 0;
  for (size_t i = 0; i < items.size(); ++i) {
    (*lists)[static_cast<size_t>(owner[i])].push_back(items[i]);
    load[static_cast<size_t>(owner[i])] += item_cost(items[i], kblocks);
    total += item_cost(items[i], kblocks);
  }
  const int64_t target = (total + g - 1) / g + kPartOverhead;
  std::vector<WorkItem> given;
  for (int32_t c = 0; c < g; ++c) {
    auto& l = (*lists)[static_cast<size_t>(c)];
    while (load[static_cast<size_t>(c)] > target && l.size() > 1) {
      const WorkItem& it = l.back();
      if (it.list_off >= 0 || it.part >= 0 || it.n_total < 2 * kMinPartBlocks) break;
      load[static_cast<size_t>(c)] -= item_cost(it, kblocks);
      given.push_back(it);
      l.pop_back();
    }
  }
  splits->clear();
  using Load = std::pair<int64_t, int32_t>;
  std::priority_queue<Load, std::vector<Load>, std::greater<Load>> heap;
  for (int32_t c = 0; c < g; ++c) heap.push({load[static_cast<size_t>(c)], c});
  int32_t slot = 0;
  for (const WorkItem& it : given) {
    int32_t remaining = it.n_total, kb = it.kb0;
    const int32_t first_slot = slot;
    std::vector<std::pair<int32_t, size_t>> placed;  // (cta, index in its list)
    while (remaining > 0) {
      Load l = heap.top();
      heap.pop();
      int64_t k = std::max<int64_t>(kMinPartBlocks, (target - l.first - kPartOverhead) / kFullCost);
      k = std::min<int64_t>(k, remaining);
      if (remaining - k > 0 && remaining - k < kMinPartBlocks) k = remaining;  // no tiny tail
      WorkItem part = it;
      part.kb0 = kb;
      part.n_total = static_cast<int32_t>(k);
      part.part = slot++;
      auto& dst = (*lists)[static_cast<size_t>(l.second)];
      placed.emplace_back(l.second, dst.size());
      dst.push_back(part);
      l.first += item_cost(part, kblocks);
      heap.push(l);
      remaining -= static_cast<int32_t>(k);
      kb += static_cast<int32_t>(k);
    }
    if (placed.size() == 1) {  // fitted whole: no partial results
      (*lists)[static_cast<size_t>(placed[0].first)][placed[0].second].part = -1;
      --slot;
      continue;
    }
    for (const auto& pl : placed) {  // every part knows its item's slots (merge in the kernel)
      WorkItem& part = (*lists)[static_cast<size_t>(pl.first)][pl.second];
      part.n_parts = static_cast<int32_t>(placed.size());
      part.pad = first_slot;
    }
    WorkItem whole = it;
    whole.part = first_slot;
    whole.n_parts = static_cast<int32_t>(placed.size());
    splits->push_back(whole);
  }
  int64_t makespan = 0;
  while (!heap.empty()) {
    makespan = std::max(makespan, heap.top().first);
    heap.pop();
  }
  return makespan;
}

}  // namespace

int64_t planned_cost(const WorkItem& it, const uint32_t* kblocks) { return item_cost(it, kblocks); }

void assign_ctas(Plan* plan, int32_t ctas, bool allow_split, bool force_split) {
  plan->splits.clear();
  if (force_split) {
    // test hook: every prefix-form item of two or more key blocks becomes two halves
    std::vector<WorkItem> halves;
    for (const WorkItem& it : plan->items) {
      if (it.list_off >= 0 || it.n_total < 2) {
        halves.push_back(it);
        continue;
      }
      const int32_t slot = 2 * static_cast<int32_t>(plan->splits.size());
      WorkItem whole = it;
      whole.part = slot;
      whole.n_parts = 2;
      plan->splits.push_back(whole);
      WorkItem head = it, tail = it;
      head.n_total = it.n_total / 2;
      head.part = slot;
      tail.kb0 = it.kb0 + head.n_total;
      tail.n_total = it.n_total - head.n_total;
      tail.part = slot + 1;
      head.n_parts = tail.n_parts = 2;
      head.pad = tail.pad = slot;
      halves.push_back(head);
      halves.push_back(tail);
    }
    std::stable_sort(halves.begin(), halves.end(),
                     [](const WorkItem& x, const WorkItem& y) { return x.n_total > y.n_total; });
    plan->items.swap(halves);
  }
  const uint32_t* kb = plan->kblocks.data();
  std::stable_sort(plan->items.begin(), plan->items.end(),
                   [kb](const WorkItem& x, const WorkItem& y) { return item_cost(x, kb) > item_cost(y, kb); });
  const int32_t n = static_cast<int32_t>(plan->items.size());
  const int32_t g = std::max(1, std::min(ctas, n));
  plan->grid = n ? g : 0;
  plan->cta_offsets.assign(static_cast<size_t>(g) + 1, 0);
  plan->makespan = 0;
  if (!n) return;
  std::vector<int32_t> owner;
  const int64_t lpt_span = lpt(plan->items, g, &owner, kb);
  std::vector<std::vector<WorkItem>> lists;
  std::vector<WorkItem> splits;
  int64_t span = lpt_span;
  bool use_split = false;
  if (allow_split && !force_split && g > 1) {
    span = tail_split(plan->items, g, owner, &lists, &splits, kb);
    use_split = !splits.empty() && span + kSplitPenalty < lpt_span;
  }
  if (!use_split) {  // the longest-first lists, each CTA keeping the longest-first order
    lists.assign(static_cast<size_t>(g), {});
    for (int32_t i = 0; i < n; ++i)
      lists[static_cast<size_t>(owner[static_cast<size_t>(i)])].push_back(plan->items[static_cast<size_t>(i)]);
    span = lpt_span;
  } else {
    plan->splits.swap(splits);
  }
  plan->makespan = span;
  std::vector<WorkItem> ordered;
  for (int32_t c = 0; c < g; ++c) {
    ordered.insert(ordered.end(), lists[static_cast<size_t>(c)].begin(), lists[static_cast<size_t>(c)].end());
    plan->cta_offsets[static_cast<size_t>(c) + 1] = static_cast<int32_t>(ordered.size());
  }
  plan->items.swap(ordered);
}

void tile_classes(const Plan& plan, int32_t batch, const int32_t* cu_seqlens,
                  std::vector<uint8_t>* out) {
  out->clear();
  std::vector<const WorkItem*> by_q0(static_cast<size_t>(plan.total_tokens), nullptr);
  for (const WorkItem& it : plan.items)
    if (it.g == 0) by_q0[static_cast<size_t>(it.q0)] = &it;
  for (int32_t b = 0; b < batch; ++b) {
    const int32_t base = cu_seqlens[b];
    const int32_t L = cu_seqlens[b + 1] - base;
    const int32_t nkb = (L + kBlockKeys - 1) / kBlockKeys;
    for (int32_t r0 = 0; r0 < L; r0 += kBlockTokens) {
      const WorkItem* it = by_q0[static_cast<size_t>(base + r0)];
      const size_t at = out->size();
      out->resize(at + static_cast<size_t>(nkb), HGX_TILE_SKIP);
      if (!it) continue;  // query block of a reused prefix: nothing is computed
      if (it->list_off < 0) {
        for (int32_t kb = 0; kb < nkb; ++kb)
          (*out)[at + kb] = kb < it->n_full ? HGX_TILE_FULL : kb < it->n_total ? HGX_TILE_PARTIAL : HGX_TILE_SKIP;
      } else {
        for (int32_t n = 0; n < it->n_total; ++n) {
          const uint32_t e = plan.kblocks[static_cast<size_t>(it->list_off + n)];
          (*out)[at + (e & kListBlockMask)] = static_cast<uint8_t>(e >> kListClassShift);
        }
      }
    }
  }
}

void mrope_tables(double theta, int32_t head_dim, const int32_t section[3], int32_t layout,
                  double* inv_freq, int32_t* axis) {
  const int32_t half = head_dim / 2;
  for (int32_t k = 0; k < half; ++k) {
    inv_freq[k] = std::pow(theta, -2.0 * static_cast<double>(k) / static_cast<double>(head_dim));
    int32_t a = 0;
    if (layout == HGX_ROPE_2D_ALTERNATING) {
      a = k % 2 == 0 ? 2 : 1;  // x (the w column) on even frequencies, y (h) on odd ones
    } else if (layout == HGX_ROPE_2D_HALVES) {
      a = k < half / 2 ? 2 : 1;  // x on the first half of the frequencies, y on the second
    } else {
      // interleaved: h and w take every third frequency (offsets 1 and 2) while they have
      // slots left; t takes offset 0 and everything after the interleaved run.
      if (k % 3 == 1 && k < 3 * section[1]) a = 1;
      else if (k % 3 == 2 && k < 3 * section[2]) a = 2;
    }
    axis[k] = a;
  }
}

}  // namespace hgx
