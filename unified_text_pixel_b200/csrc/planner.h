// Host planner of the hybrid-masked attention: descriptor validation, per-row key limits,
// tile classes and the attention kernel's work list. Pure C++ (no CUDA calls), so every
// part of it runs and is tested on a machine without a GPU.
#pragma once

#include <cstdint>
#include <string>
#include <vector>

#include "../../include/hgx_attn.h"

namespace hgx {

// Tile of the attention kernel: kBlockTokens query tokens (x 4 query heads of one KV head,
// as two 128-row MMA tiles of 32 tokens each) against kBlockKeys keys.
constexpr int kTileTokens = 32;                 // tokens per 128-row MMA tile (4 heads each)
constexpr int kTilesPerBlock = 2;               // MMA tiles per work item (ping-pong)
constexpr int kBlockTokens = kTileTokens * kTilesPerBlock;
constexpr int kBlockKeys = 128;
// Largest packed token count: keeps every byte offset of q/out (T * 8192) below 2^32 and
// every TMA coordinate far inside int32.
constexpr int32_t kMaxTokens = (1 << 19) - 1;

// One unit of attention work: one KV head g and its 4 query heads over kBlockTokens
// consecutive query tokens of one batch element. Layout shared with the kernel.
//
// Prefix form (list_off < 0): the item processes key blocks kb0 .. kb0 + n_total - 1; blocks
// below n_full are visible to every row (no mask compare), the rest need the per-row
// compare. List form (list_off >= 0, items whose rows see a Gen Image hole): the item
// processes the n_total key blocks listed at kblocks[list_off ...], each entry
// kb | class << 24 with class an hgx_tile_class (FULL or PARTIAL; skipped blocks are not
// listed).
// Split items (part >= 0, prefix form only): the key blocks of one (query block, KV head)
// are divided between several work items that may run on different CTAs; each writes its
// unnormalised O, row maximum and row sum to partial-result slot `part`, and a combine
// kernel merges the item's slots into out.
struct WorkItem {
  int32_t q0;        // packed index of the first query token
  int32_t kv0;       // packed index of the batch element's first token
  int32_t len;       // tokens in the batch element
  int32_t g;         // KV head
  int32_t n_full;    // prefix form: key blocks [0, n_full) need no compare
  int32_t n_total;   // key blocks to process
  int32_t list_off;  // -1: prefix form; else offset into the key-block list
  int32_t first;     // rows before this local row are not written (cached prefix)
  int32_t kb0 = 0;   // prefix form: first key block processed
  int32_t part = -1; // -1: writes out; else its partial-result slot
  int32_t n_parts = 0;  // split items: number of parts of the whole item
  int32_t pad = 0;      // parts of split items: the whole item's first slot (Plan::splits: part)
};
static_assert(sizeof(WorkItem) == 48, "work item layout");

constexpr uint32_t kListClassShift = 24;
constexpr uint32_t kListBlockMask = (1u << kListClassShift) - 1;

struct Plan {
  int32_t batch = 0;
  int32_t total_tokens = 0;
  std::vector<int32_t> lim;        // [T] exclusive key limit per packed row, local
  std::vector<WorkItem> items;     // sorted by n_total, longest first
  uint64_t visible_pairs = 0;      // visible (query, key) pairs, holes excluded
  // Gen Image holes (empty when the descriptor has no gen_image segment):
  std::vector<uint32_t> kblocks;   // key-block lists of list-form items
  std::vector<int32_t> hole_base;  // [T] first mask index of the row's segment, or -1
  std::vector<uint32_t> hole_masks;  // 4 words per (segment, key block): keys hidden
  bool has_holes = false;
  // Assignment of the items to the persistent CTAs (assign_ctas): CTA c processes items
  // [cta_offsets[c], cta_offsets[c + 1]) of `items`, longest first.
  int32_t grid = 0;
  std::vector<int32_t> cta_offsets;
  // Split items (assign_ctas with splitting): splits[i] is the whole (query block, KV head)
  // item whose parts wrote the partial slots part .. part + n_parts - 1.
  std::vector<WorkItem> splits;
  int64_t makespan = 0;  // largest CTA load of the assignment, in key blocks + overheads
};

// Checks the packed-varlen descriptor. On failure returns INVALID_ARG with *err set.
hgx_status validate_descriptor(int32_t batch, const int32_t* cu_seqlens,
                               const hgx_segment* segs, const int32_t* cu_segs,
                               std::string* err, int32_t* total_tokens);

// Validates and fills lim (size T). Returns INVALID_ARG on a bad descriptor.
hgx_status row_limits(int32_t batch, const int32_t* cu_seqlens, const hgx_segment* segs,
                      const int32_t* cu_segs, std::vector<int32_t>* lim, std::string* err);

// Validates, computes limits and the sorted work list for num_kv_heads KV heads. With
// first_rows (host, [batch], may be NULL) only rows [first_rows[b], L_b) of element b are
// planned; every earlier row must see no key at or after first_rows[b] (a cached prefix).
hgx_status build_plan(int32_t batch, const int32_t* cu_seqlens, const hgx_segment* segs,
                      const int32_t* cu_segs, int32_t num_kv_heads, Plan* plan,
                      std::string* err, const int32_t* first_rows = nullptr);

// Checks first_rows (host, [batch]) against a valid descriptor: each within [0, L_b] and no
// row before it seeing a key at or after it. INVALID_ARG with *err otherwise.
hgx_status check_first_rows(int32_t batch, const int32_t* cu_seqlens, const hgx_segment* segs,
                            const int32_t* cu_segs, const int32_t* first_rows, std::string* err);

// Distributes plan->items over `ctas` persistent CTAs (longest-processing-time first: each
// item, in decreasing cost, goes to the least loaded CTA; cost = planned_cost: fully visible
// key blocks, the dearer blocks that run the mask compare and a per-item overhead), reorders
// the items so that every CTA's list is contiguous, and sets grid,
// cta_offsets and makespan. grid = min(ctas, number of items).
//
// With allow_split, a second schedule is tried: the CTAs loaded above the mean give back
// their last (smallest) items, whose key blocks are handed out in parts to the least-loaded
// CTAs (tail_split in planner.cpp). It replaces the first schedule when its makespan plus
// kSplitPenalty is smaller.
// Costs are in tenths of a fully visible key block (planner.cpp: a PARTIAL block costs 13).
constexpr int64_t kItemOverhead = 12;  // loading Q, filling the pipeline, writing O
constexpr int64_t kSplitPenalty = 30;  // the combine launch
// force_split (a test hook that exercises the split path on any input): every prefix-form
// item of two or more key blocks is split into two halves, then all items are assigned
// longest first.
void assign_ctas(Plan* plan, int32_t ctas, bool allow_split = false, bool force_split = false);

// Cost of a work item in the assignment (tenths of a fully visible key block): 10 per fully
// visible block, 13 per block that runs the mask compare, plus kItemOverhead (or the larger
// overhead of a part of a split item). kblocks: the plan's key-block lists, needed only for
// list-form items (may be NULL otherwise).
int64_t planned_cost(const WorkItem& it, const uint32_t* kblocks);
// The largest planned_cost of a prefix-form item of at most max_blocks key blocks.
constexpr int64_t planned_cost_bound(int64_t max_blocks) { return 13 * max_blocks + kItemOverhead; }

// Tile classes of every (query block, key block) of every batch element in order (after
// a successful build_plan with the same descriptor).
void tile_classes(const Plan& plan, int32_t batch, const int32_t* cu_seqlens,
                  std::vector<uint8_t>* out);

// Frequency table of the rotary embedding: inv_freq[k] = theta^(-2k/D) and the axis
// (0 t, 1 h, 2 w) that drives frequency k under the given hgx_rope_layout.
void mrope_tables(double theta, int32_t head_dim, const int32_t section[3], int32_t layout,
                  double* inv_freq, int32_t* axis);

}  // namespace hgx
