// Host planner: descriptor validation, per-row key limits, tile classes, work list.
//
// The visibility rules follow the pages: HiDream-O1 ("hidream-o1-p100a" model card, "What
// this model is"; "HiDream-O1-Image" summary, "How it works") -- text and condition tokens
// causal, generation tokens see the whole sequence; HunyuanImage 3.0 Generalized Causal
// Attention (paper-graph-ui summary, section 3.4, "The core rule") -- image tokens see all
// previous tokens and their whole segment. Under each rule the keys a row sees form a
// prefix, so one exclusive limit per row describes the mask exactly:
//   causal: i + 1;  full_sequence: L;  full_in_segment: end of i's segment.
#include "planner.h"

#include <algorithm>
#include <cmath>
#include <cstdio>

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
      if (sg.kind < HGX_SEG_CAUSAL || sg.kind > HGX_SEG_FULL_IN_SEGMENT) {
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
          default: l = sg.start + sg.len; break;  // full_in_segment
        }
        (*lim)[static_cast<size_t>(base + i)] = l;
      }
    }
  }
  return HGX_OK;
}

hgx_status build_plan(int32_t batch, const int32_t* cu_seqlens, const hgx_segment* segs,
                      const int32_t* cu_segs, int32_t num_kv_heads, Plan* plan,
                      std::string* err) {
  hgx_status st = row_limits(batch, cu_seqlens, segs, cu_segs, &plan->lim, err);
  if (st != HGX_OK) return st;
  plan->batch = batch;
  plan->total_tokens = batch ? cu_seqlens[batch] : 0;
  plan->items.clear();
  plan->visible_pairs = 0;
  for (int32_t x : plan->lim) plan->visible_pairs += static_cast<uint64_t>(x);
  for (int32_t b = 0; b < batch; ++b) {
    const int32_t base = cu_seqlens[b];
    const int32_t L = cu_seqlens[b + 1] - base;
    for (int32_t r0 = 0; r0 < L; r0 += kBlockTokens) {
      const int32_t r1 = std::min(L, r0 + kBlockTokens);
      int32_t lo = INT32_MAX, hi = 0;
      for (int32_t i = r0; i < r1; ++i) {
        const int32_t l = plan->lim[static_cast<size_t>(base + i)];
        lo = std::min(lo, l);
        hi = std::max(hi, l);
      }
      for (int32_t g = 0; g < num_kv_heads; ++g) {
        WorkItem it{};
        it.q0 = base + r0;
        it.kv0 = base;
        it.len = L;
        it.g = g;
        it.n_full = lo / kBlockKeys;
        it.n_total = (hi + kBlockKeys - 1) / kBlockKeys;
        plan->items.push_back(it);
      }
    }
  }
  std::stable_sort(plan->items.begin(), plan->items.end(),
                   [](const WorkItem& a, const WorkItem& b) { return a.n_total > b.n_total; });
  return HGX_OK;
}

void mrope_tables(double theta, int32_t head_dim, const int32_t section[3], double* inv_freq,
                  int32_t* axis) {
  const int32_t half = head_dim / 2;
  for (int32_t k = 0; k < half; ++k) {
    inv_freq[k] = std::pow(theta, -2.0 * static_cast<double>(k) / static_cast<double>(head_dim));
    // interleaved: h and w take every third frequency (offsets 1 and 2) while they have
    // slots left; t takes offset 0 and everything after the interleaved run.
    int32_t a = 0;
    if (k % 3 == 1 && k < 3 * section[1]) a = 1;
    else if (k % 3 == 2 && k < 3 * section[2]) a = 2;
    axis[k] = a;
  }
}

}  // namespace hgx
