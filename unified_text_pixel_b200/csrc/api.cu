// C ABI of the hybrid-masked attention (declared in include/hgx_attn.h).
//
// Every argument is checked on the host before any device work, as the HiDream-O1 port
// does for contract errors ("hidream-o1-p100a" model card, "Serving (HTTP)": rejected
// without touching the card). The handle caches the plan (row limits, work list) of the
// last segment descriptor and re-uploads it only when the descriptor changes.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <string>
#include <vector>

#include "../../include/hgx_attn.h"
#include "kernels.h"
#include "planner.h"

struct hgx_attn_handle {
  hgx_attn_config cfg{};
  float scale = 0.f;
  hgx::RopeTables rope{};
  std::string last_error;
  uint32_t flags = 0;
  uint64_t wait_limit_ns = 2000000000ull;

  // cached descriptor and its plan
  int32_t key_batch = -1;
  std::vector<int32_t> key_cu, key_cu_segs;
  std::vector<hgx_segment> key_segs;
  std::vector<int32_t> key_first;  // first recomputed row per element; empty = all rows
  bool key_split_test = false;     // planned under HGX_DEBUG_SPLIT_TEST
  hgx::Plan plan;
  int plan_device = -1;

  // device scratch owned by the handle
  int device = -1;
  int num_sms = 0;
  int32_t* d_lim = nullptr;
  size_t lim_cap = 0;
  hgx::WorkItem* d_items = nullptr;
  size_t items_cap = 0;
  // Gen Image hole tables (allocated only for descriptors with gen_image segments)
  uint32_t* d_kblocks = nullptr;
  size_t kblocks_cap = 0;
  int32_t* d_hole_base = nullptr;
  size_t hole_base_cap = 0;
  uint32_t* d_hole_masks = nullptr;
  size_t hole_masks_cap = 0;
  int32_t* d_cta_offsets = nullptr;  // the persistent CTAs' item lists
  size_t cta_offsets_cap = 0;
  // split items: their list for the combine kernel and the partial results (fp32 O, then
  // (M, l) pairs), sized for the largest plan so far
  hgx::WorkItem* d_splits = nullptr;
  size_t splits_cap = 0;
  void* d_partial = nullptr;
  size_t partial_cap = 0;
  // (cos, sin) per (token, frequency) for the QKV projection's epilogue
  void* d_rope_cs = nullptr;
  size_t rope_cs_cap = 0;
  uint32_t* d_err = nullptr;
  // per-CTA clock64 / %globaltimer stamps of the last attention launch ([num_sms][4])
  uint64_t* d_stamps = nullptr;
  int stamps_grid = 0;
  // pinned staging for the plan upload, reused once the previous upload has completed
  uint8_t* h_stage = nullptr;
  size_t stage_cap = 0;
  cudaEvent_t stage_done = nullptr;
};

namespace {

#ifndef HGX_SPLIT_KV
#define HGX_SPLIT_KV 1
#endif
// 1: the planner may split items by key blocks when that balances the persistent CTAs
// better (hgx::assign_ctas); 0: longest-processing-time assignment only
constexpr bool kSplitKV = HGX_SPLIT_KV != 0;

using PFN_encodeTiled = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                     const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                     const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                     CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

hgx_status fail(hgx_attn_handle* h, hgx_status st, const std::string& msg) {
  if (h) h->last_error = msg;
  return st;
}

hgx_status cuda_fail(hgx_attn_handle* h, cudaError_t e, const char* what) {
  return fail(h, HGX_ERR_CUDA, std::string(what) + ": " + cudaGetErrorString(e));
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

PFN_encodeTiled encode_fn() {
  static PFN_encodeTiled fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_encodeTiled>(ptr);
  }
  return fn;
}

// 3-D bf16 tensor map over [T, heads, 128] with a box of (64 features, box_heads,
// box_tokens) and 128-byte swizzle; boxes past T read zeros.
bool make_map(CUtensorMap* map, const void* ptr, int heads, int T, int box_heads,
              int box_tokens) {
  PFN_encodeTiled enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[3] = {128, static_cast<cuuint64_t>(heads), static_cast<cuuint64_t>(T)};
  cuuint64_t strides[2] = {256, static_cast<cuuint64_t>(heads) * 256};
  cuuint32_t box[3] = {64, static_cast<cuuint32_t>(box_heads),
                       static_cast<cuuint32_t>(box_tokens)};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims,
                   strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// 2-D bf16 tensor map over a row-major [rows, cols] matrix with a (64, box_rows) box and
// 128-byte swizzle (the GEMM operands; rows past the end read zeros).
bool make_map_2d(CUtensorMap* map, const void* ptr, int64_t rows, int64_t cols, int box_rows) {
  PFN_encodeTiled enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols) * 2};
  cuuint32_t box[2] = {64, static_cast<cuuint32_t>(box_rows)};
  cuuint32_t estr[2] = {1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

hgx_status ensure_device(hgx_attn_handle* h) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(h, e, "cudaGetDevice");
  if (h->device == dev) return HGX_OK;
  if (h->device >= 0) return fail(h, HGX_ERR_INVALID_ARG, "handle is bound to another device");
  int major = 0, minor = 0;
  cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
  cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
  if (major != 10 || minor != 0)
    return fail(h, HGX_ERR_UNSUPPORTED, "this library is built for sm_100a (B200) only");
  e = cudaDeviceGetAttribute(&h->num_sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return cuda_fail(h, e, "cudaDeviceGetAttribute");
  // on failure, release what this call allocated, so that the handle stays unbound and
  // holds nothing of this device
  auto undo = [h]() {
    if (h->d_err) cudaFree(h->d_err);
    if (h->d_stamps) cudaFree(h->d_stamps);
    if (h->stage_done) cudaEventDestroy(h->stage_done);
    h->d_err = nullptr;
    h->d_stamps = nullptr;
    h->stage_done = nullptr;
  };
  e = cudaMalloc(&h->d_err, sizeof(uint32_t));
  if (e != cudaSuccess) {
    h->d_err = nullptr;
    return fail(h, HGX_ERR_OOM, "cudaMalloc of the error word failed");
  }
  e = cudaMemset(h->d_err, 0, sizeof(uint32_t));
  if (e != cudaSuccess) {
    undo();
    return cuda_fail(h, e, "cudaMemset");
  }
  e = cudaMalloc(&h->d_stamps, static_cast<size_t>(h->num_sms) * 4 * sizeof(uint64_t));
  if (e != cudaSuccess) {
    h->d_stamps = nullptr;
    undo();
    return fail(h, HGX_ERR_OOM, "cudaMalloc of the clock stamps failed");
  }
  e = cudaEventCreateWithFlags(&h->stage_done, cudaEventDisableTiming);
  if (e != cudaSuccess) {
    h->stage_done = nullptr;
    undo();
    return cuda_fail(h, e, "cudaEventCreate");
  }
  h->device = dev;
  return HGX_OK;
}

bool same_descriptor(const hgx_attn_handle* h, int32_t batch, const int32_t* cu,
                     const hgx_segment* segs, const int32_t* cu_segs, const int32_t* first) {
  if (h->key_batch != batch) return false;
  if (h->key_split_test != ((h->flags & HGX_DEBUG_SPLIT_TEST) != 0)) return false;
  if (first ? (h->key_first.size() != static_cast<size_t>(batch) ||
               std::memcmp(h->key_first.data(), first, sizeof(int32_t) * batch) != 0)
            : !h->key_first.empty())
    return false;
  if (std::memcmp(h->key_cu.data(), cu, sizeof(int32_t) * (batch + 1)) != 0) return false;
  if (std::memcmp(h->key_cu_segs.data(), cu_segs, sizeof(int32_t) * (batch + 1)) != 0)
    return false;
  const size_t ns = static_cast<size_t>(cu_segs[batch]);
  if (h->key_segs.size() != ns) return false;
  return ns == 0 || std::memcmp(h->key_segs.data(), segs, sizeof(hgx_segment) * ns) == 0;
}

// Builds (or reuses) the plan of this descriptor and makes sure it is on the device,
// uploaded in stream order.
hgx_status prepare_plan(hgx_attn_handle* h, cudaStream_t stream, int32_t batch,
                        const int32_t* cu, const hgx_segment* segs, const int32_t* cu_segs,
                        const int32_t* first = nullptr) {
  const bool same = same_descriptor(h, batch, cu, segs, cu_segs, first);
  if (!same) {
    hgx::Plan plan;
    std::string err;
    hgx_status st =
        hgx::build_plan(batch, cu, segs, cu_segs, h->cfg.num_kv_heads, &plan, &err, first);
    if (st != HGX_OK) return fail(h, st, err);
    const bool split_test = (h->flags & HGX_DEBUG_SPLIT_TEST) != 0;
    hgx::assign_ctas(&plan, h->num_sms, kSplitKV, split_test);
    h->plan = std::move(plan);
    h->key_batch = batch;
    h->key_split_test = split_test;
    h->key_cu.assign(cu, cu + batch + 1);
    h->key_cu_segs.assign(cu_segs, cu_segs + batch + 1);
    h->key_segs.assign(segs, segs + cu_segs[batch]);
    if (first)
      h->key_first.assign(first, first + batch);
    else
      h->key_first.clear();
    h->plan_device = -1;
  }
  if (h->plan_device == h->device) return HGX_OK;
  const hgx::Plan& pl = h->plan;
  // (device buffer, its capacity, host data, bytes) of every array the kernel reads
  struct Upload {
    void** dst;
    size_t* cap;
    const void* src;
    size_t bytes;
  } up[] = {
      {reinterpret_cast<void**>(&h->d_lim), &h->lim_cap, pl.lim.data(), pl.lim.size() * sizeof(int32_t)},
      {reinterpret_cast<void**>(&h->d_items), &h->items_cap, pl.items.data(),
       pl.items.size() * sizeof(hgx::WorkItem)},
      {reinterpret_cast<void**>(&h->d_kblocks), &h->kblocks_cap, pl.kblocks.data(),
       pl.kblocks.size() * sizeof(uint32_t)},
      {reinterpret_cast<void**>(&h->d_hole_base), &h->hole_base_cap, pl.hole_base.data(),
       pl.hole_base.size() * sizeof(int32_t)},
      {reinterpret_cast<void**>(&h->d_hole_masks), &h->hole_masks_cap, pl.hole_masks.data(),
       pl.hole_masks.size() * sizeof(uint32_t)},
      {reinterpret_cast<void**>(&h->d_cta_offsets), &h->cta_offsets_cap, pl.cta_offsets.data(),
       pl.cta_offsets.size() * sizeof(int32_t)},
      {reinterpret_cast<void**>(&h->d_splits), &h->splits_cap, pl.splits.data(),
       pl.splits.size() * sizeof(hgx::WorkItem)},
  };
  size_t need = 0;
  for (const Upload& u : up) {
    if (u.bytes > *u.cap) {
      if (h->flags & HGX_DEBUG_FAIL_ALLOC) {  // injected failure (test hook), one-shot
        h->flags &= ~HGX_DEBUG_FAIL_ALLOC;
        return fail(h, HGX_ERR_OOM, "cudaMalloc of the planner scratch failed (injected)");
      }
      if (*u.dst) cudaFree(*u.dst);
      *u.dst = nullptr;
      *u.cap = 0;
      if (cudaMalloc(u.dst, u.bytes) != cudaSuccess)
        return fail(h, HGX_ERR_OOM, "cudaMalloc of the planner scratch failed");
      *u.cap = u.bytes;
    }
    need += (u.bytes + 255) & ~size_t(255);
  }
  // partial results of split items (written and read on the device only)
  size_t slots = 0;
  for (const hgx::WorkItem& sp : pl.splits) slots += static_cast<size_t>(sp.n_parts);
  const size_t partial_bytes =
      slots * (hgx::kPartialSlotFloats * sizeof(float) + hgx::kPartialSlotRows * sizeof(float2));
  if (partial_bytes > h->partial_cap) {
    if (h->flags & HGX_DEBUG_FAIL_ALLOC) {
      h->flags &= ~HGX_DEBUG_FAIL_ALLOC;
      return fail(h, HGX_ERR_OOM, "cudaMalloc of the partial results failed (injected)");
    }
    if (h->d_partial) cudaFree(h->d_partial);
    h->d_partial = nullptr;
    h->partial_cap = 0;
    if (cudaMalloc(&h->d_partial, partial_bytes) != cudaSuccess)
      return fail(h, HGX_ERR_OOM, "cudaMalloc of the partial results failed");
    h->partial_cap = partial_bytes;
  }
  cudaError_t e;
  // the previous upload may still be reading the staging buffer
  e = cudaEventSynchronize(h->stage_done);
  if (e != cudaSuccess) return cuda_fail(h, e, "cudaEventSynchronize");
  if (need > h->stage_cap) {
    if (h->h_stage) cudaFreeHost(h->h_stage);
    h->h_stage = nullptr;
    h->stage_cap = 0;
    if (cudaMallocHost(&h->h_stage, need) != cudaSuccess)
      return fail(h, HGX_ERR_OOM, "cudaMallocHost of the plan staging buffer failed");
    h->stage_cap = need;
  }
  size_t off = 0;
  for (const Upload& u : up) {
    if (!u.bytes) continue;
    std::memcpy(h->h_stage + off, u.src, u.bytes);
    e = cudaMemcpyAsync(*u.dst, h->h_stage + off, u.bytes, cudaMemcpyHostToDevice, stream);
    if (e != cudaSuccess) return cuda_fail(h, e, "cudaMemcpyAsync (plan)");
    off += (u.bytes + 255) & ~size_t(255);
  }
  e = cudaEventRecord(h->stage_done, stream);
  if (e != cudaSuccess) return cuda_fail(h, e, "cudaEventRecord");
  h->plan_device = h->device;
  return HGX_OK;
}

hgx_status check_tensors(hgx_attn_handle* h, std::initializer_list<const void*> ptrs) {
  for (const void* p : ptrs) {
    if (!p) return fail(h, HGX_ERR_INVALID_ARG, "device pointer is NULL");
    if (!aligned16(p)) return fail(h, HGX_ERR_INVALID_ARG, "device pointer is not 16-byte aligned");
  }
  return HGX_OK;
}

bool overlaps(const void* a, size_t na, const void* b, size_t nb) {
  const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
  return x < y + nb && y < x + na;
}

hgx_status finish(hgx_attn_handle* h, cudaStream_t stream) {
  if (h->flags & HGX_DEBUG_CHECKED) return hgx_attn_sync_status(h, stream);
  return HGX_OK;
}

hgx_status run_attention(hgx_attn_handle* h, cudaStream_t stream, const void* q, const void* k,
                         const void* v, void* out) {
  const int32_t T = h->plan.total_tokens;
  CUtensorMap mq, mk, mv, mo;
  if (!make_map(&mq, q, 32, T, 4, hgx::kTileTokens) || !make_map(&mk, k, 8, T, 1, 128) ||
      !make_map(&mv, v, 8, T, 1, 128) || !make_map(&mo, out, 32, T, 4, 8))
    return fail(h, HGX_ERR_CUDA, "cuTensorMapEncodeTiled failed");
  hgx::AttnParams p{};
  p.items = h->d_items;
  p.n_items = static_cast<int32_t>(h->plan.items.size());
  p.cta_offsets = h->d_cta_offsets;
  p.total_tokens = T;
  p.lim = h->d_lim;
  p.kblocks = h->plan.has_holes ? h->d_kblocks : nullptr;
  p.hole_base = h->plan.has_holes ? h->d_hole_base : nullptr;
  p.hole_masks = h->plan.has_holes ? h->d_hole_masks : nullptr;
  p.out = out;
  p.out_tma = 1;
  size_t slots = 0;
  for (const hgx::WorkItem& sp : h->plan.splits) slots += static_cast<size_t>(sp.n_parts);
  p.partial_o = slots ? static_cast<float*>(h->d_partial) : nullptr;
  p.partial_ml = slots ? reinterpret_cast<float2*>(static_cast<float*>(h->d_partial) +
                                                   slots * hgx::kPartialSlotFloats)
                       : nullptr;

  p.scale_log2 = h->scale * 1.4426950408889634f;
  p.flags = h->flags;
  p.err = h->d_err;
  p.wait_limit_ns = h->wait_limit_ns;
  p.stamps = h->d_stamps;
  cudaError_t e = hgx::launch_attention(stream, mq, mk, mv, mo, p, h->plan.grid);
  if (e != cudaSuccess) return cuda_fail(h, e, "attention launch");
  h->stamps_grid = h->plan.grid;
  if (slots) {
    e = hgx::launch_combine(stream, h->d_splits, static_cast<int32_t>(h->plan.splits.size()), p.partial_o,
                            p.partial_ml, out);
    if (e != cudaSuccess) return cuda_fail(h, e, "combine launch");
  }
  return HGX_OK;
}

hgx_status run_gemm(hgx_attn_handle* h, cudaStream_t stream, const void* a, const void* b,
                    hgx::GemmParams p) {
  CUtensorMap ma, mb;
  if (!make_map_2d(&ma, a, p.M, p.K, 128) || !make_map_2d(&mb, b, p.N, p.K, 256))
    return fail(h, HGX_ERR_CUDA, "cuTensorMapEncodeTiled failed");
  p.err = h->d_err;
  p.wait_limit_ns = h->wait_limit_ns;
  const int tiles = ((p.M + 127) / 128) * (p.N / 256);
  const int grid = tiles < h->num_sms ? tiles : h->num_sms;
  cudaError_t e = hgx::launch_gemm(stream, ma, mb, p, grid);
  if (e != cudaSuccess) return cuda_fail(h, e, "gemm launch");
  return HGX_OK;
}

// QKV projection of total_tokens rows with q/k RMSNorm and rotation in the epilogue.
hgx_status run_qkv(hgx_attn_handle* h, cudaStream_t stream, const void* x, const void* w_qkv, void* q,
                   void* k, void* v, const int32_t* pos, const void* wq, const void* wk, int32_t T) {
  const size_t need = static_cast<size_t>(T) * 64 * sizeof(float2);
  if (need > h->rope_cs_cap) {
    if (h->d_rope_cs) cudaFree(h->d_rope_cs);
    h->d_rope_cs = nullptr;
    h->rope_cs_cap = 0;
    if (cudaMalloc(&h->d_rope_cs, need) != cudaSuccess)
      return fail(h, HGX_ERR_OOM, "cudaMalloc of the rotation table failed");
    h->rope_cs_cap = need;
  }
  cudaError_t e = hgx::launch_rope_table(stream, pos, T, h->rope, h->d_rope_cs);
  if (e != cudaSuccess) return cuda_fail(h, e, "rotation table launch");
  hgx::GemmParams p{};
  p.M = T;
  p.N = 6144;
  p.K = 4096;
  p.mode = 1;
  p.q = q;
  p.k = k;
  p.v = v;
  p.rope_cs = static_cast<const float2*>(h->d_rope_cs);
  p.wq = static_cast<const __nv_bfloat16*>(wq);
  p.wk = static_cast<const __nv_bfloat16*>(wk);
  p.eps = h->cfg.rms_eps;
  return run_gemm(h, stream, x, w_qkv, p);
}

hgx_status run_out_proj(hgx_attn_handle* h, cudaStream_t stream, const void* att, const void* w_o, void* y,
                        int32_t T) {
  hgx::GemmParams p{};
  p.M = T;
  p.N = 4096;
  p.K = 4096;
  p.mode = 0;
  p.c = y;
  return run_gemm(h, stream, att, w_o, p);
}

}  // namespace

extern "C" {

void hgx_attn_default_config(hgx_attn_config* cfg) {
  if (!cfg) return;
  cfg->num_q_heads = 32;
  cfg->num_kv_heads = 8;
  cfg->head_dim = 128;
  cfg->rope_theta = 5.0e6;
  cfg->mrope_section[0] = 24;
  cfg->mrope_section[1] = 20;
  cfg->mrope_section[2] = 20;
  cfg->rms_eps = 1e-6f;
  cfg->softmax_scale = 0.f;
  cfg->rope_layout = HGX_ROPE_MROPE_INTERLEAVED;
}

hgx_status hgx_attn_create(const hgx_attn_config* cfg, hgx_attn_handle** out) {
  if (!out) return HGX_ERR_INVALID_ARG;
  *out = nullptr;
  if (!cfg) return HGX_ERR_INVALID_ARG;
  if (!(cfg->rope_theta > 0.0) || !std::isfinite(cfg->rope_theta)) return HGX_ERR_INVALID_ARG;
  if (!(cfg->rms_eps >= 0.f) || !std::isfinite(cfg->rms_eps)) return HGX_ERR_INVALID_ARG;
  if (!(cfg->softmax_scale >= 0.f) || !std::isfinite(cfg->softmax_scale))
    return HGX_ERR_INVALID_ARG;
  for (int i = 0; i < 3; ++i)
    if (cfg->mrope_section[i] < 0) return HGX_ERR_INVALID_ARG;
  if (cfg->num_q_heads <= 0 || cfg->num_kv_heads <= 0 || cfg->head_dim <= 0)
    return HGX_ERR_INVALID_ARG;
  if (cfg->num_q_heads != 32 || cfg->num_kv_heads != 8 || cfg->head_dim != 128)
    return HGX_ERR_UNSUPPORTED;
  if (cfg->rope_layout < HGX_ROPE_MROPE_INTERLEAVED || cfg->rope_layout > HGX_ROPE_2D_HALVES)
    return HGX_ERR_INVALID_ARG;
  if (cfg->rope_layout == HGX_ROPE_MROPE_INTERLEAVED) {
    if (cfg->mrope_section[0] + cfg->mrope_section[1] + cfg->mrope_section[2] != cfg->head_dim / 2)
      return HGX_ERR_INVALID_ARG;
    // the interleaved assignment must give each axis exactly its section's count
    double inv[64];
    int32_t axis[64], count[3] = {0, 0, 0};
    hgx::mrope_tables(cfg->rope_theta, cfg->head_dim, cfg->mrope_section, cfg->rope_layout, inv, axis);
    for (int i = 0; i < 64; ++i) ++count[axis[i]];
    for (int i = 0; i < 3; ++i)
      if (count[i] != cfg->mrope_section[i]) return HGX_ERR_UNSUPPORTED;
  }
  hgx_attn_handle* h = new (std::nothrow) hgx_attn_handle();
  if (!h) return HGX_ERR_OOM;
  h->cfg = *cfg;
  h->scale = cfg->softmax_scale > 0.f ? cfg->softmax_scale
                                      : static_cast<float>(1.0 / std::sqrt(double(cfg->head_dim)));
  int32_t axis[64];
  hgx::mrope_tables(cfg->rope_theta, cfg->head_dim, cfg->mrope_section, cfg->rope_layout,
                    h->rope.inv_freq, axis);
  for (int i = 0; i < 64; ++i) h->rope.axis[i] = static_cast<uint8_t>(axis[i]);
  if (const char* env = std::getenv("HGX_DEBUG")) h->flags = static_cast<uint32_t>(std::atoi(env));
  *out = h;
  return HGX_OK;
}

void hgx_attn_destroy(hgx_attn_handle* h) {
  if (!h) return;
  if (h->d_lim) cudaFree(h->d_lim);
  if (h->d_items) cudaFree(h->d_items);
  if (h->d_kblocks) cudaFree(h->d_kblocks);
  if (h->d_hole_base) cudaFree(h->d_hole_base);
  if (h->d_hole_masks) cudaFree(h->d_hole_masks);
  if (h->d_cta_offsets) cudaFree(h->d_cta_offsets);
  if (h->d_splits) cudaFree(h->d_splits);
  if (h->d_partial) cudaFree(h->d_partial);
  if (h->d_rope_cs) cudaFree(h->d_rope_cs);
  if (h->d_err) cudaFree(h->d_err);
  if (h->d_stamps) cudaFree(h->d_stamps);
  if (h->h_stage) cudaFreeHost(h->h_stage);
  if (h->stage_done) cudaEventDestroy(h->stage_done);
  delete h;
}

const char* hgx_attn_last_error(const hgx_attn_handle* h) {
  return h ? h->last_error.c_str() : "null handle";
}

hgx_status hgx_attn_prologue(hgx_attn_handle* h, void* stream, void* q, void* k,
                             const int32_t* pos_thw, const void* q_norm_w, const void* k_norm_w,
                             int32_t total_tokens) {
  if (!h) return HGX_ERR_INVALID_ARG;
  h->last_error.clear();
  if (total_tokens < 0 || total_tokens > hgx::kMaxTokens)
    return fail(h, HGX_ERR_INVALID_ARG, "total_tokens out of range");
  if (total_tokens == 0) return HGX_OK;
  hgx_status st = check_tensors(h, {q, k, pos_thw, q_norm_w, k_norm_w});
  if (st != HGX_OK) return st;
  if ((st = ensure_device(h)) != HGX_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = hgx::launch_prologue(s, q, k, pos_thw, q_norm_w, k_norm_w, total_tokens,
                                       h->cfg.rms_eps, h->rope);
  if (e != cudaSuccess) return cuda_fail(h, e, "prologue launch");
  return finish(h, s);
}

hgx_status hgx_attn_attention(hgx_attn_handle* h, void* stream, const void* q, const void* k,
                              const void* v, void* out, int32_t batch,
                              const int32_t* cu_seqlens_host, const hgx_segment* segs_host,
                              const int32_t* cu_segs_host) {
  if (!h) return HGX_ERR_INVALID_ARG;
  h->last_error.clear();
  std::string err;
  int32_t T = 0;
  hgx_status st = hgx::validate_descriptor(batch, cu_seqlens_host, segs_host, cu_segs_host,
                                           &err, &T);
  if (st != HGX_OK) return fail(h, st, err);
  if (T == 0) return HGX_OK;
  if ((st = check_tensors(h, {q, k, v, out})) != HGX_OK) return st;
  const size_t qb = size_t(T) * 8192, kb = size_t(T) * 2048;
  if (overlaps(out, qb, q, qb) || overlaps(out, qb, k, kb) || overlaps(out, qb, v, kb))
    return fail(h, HGX_ERR_INVALID_ARG, "out overlaps q, k or v");
  if ((st = ensure_device(h)) != HGX_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if ((st = prepare_plan(h, s, batch, cu_seqlens_host, segs_host, cu_segs_host)) != HGX_OK)
    return st;
  if ((st = run_attention(h, s, q, k, v, out)) != HGX_OK) return st;
  return finish(h, s);
}

hgx_status hgx_attn_forward(hgx_attn_handle* h, void* stream, void* q, void* k, const void* v,
                            void* out, const int32_t* pos_thw, const void* q_norm_w,
                            const void* k_norm_w, int32_t batch, const int32_t* cu_seqlens_host,
                            const hgx_segment* segs_host, const int32_t* cu_segs_host) {
  if (!h) return HGX_ERR_INVALID_ARG;
  h->last_error.clear();
  std::string err;
  int32_t T = 0;
  hgx_status st = hgx::validate_descriptor(batch, cu_seqlens_host, segs_host, cu_segs_host,
                                           &err, &T);
  if (st != HGX_OK) return fail(h, st, err);
  if (T == 0) return HGX_OK;
  if ((st = check_tensors(h, {q, k, v, out, pos_thw, q_norm_w, k_norm_w})) != HGX_OK) return st;
  const size_t qb = size_t(T) * 8192, kb = size_t(T) * 2048;
  if (overlaps(out, qb, q, qb) || overlaps(out, qb, k, kb) || overlaps(out, qb, v, kb))
    return fail(h, HGX_ERR_INVALID_ARG, "out overlaps q, k or v");
  if ((st = ensure_device(h)) != HGX_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if ((st = prepare_plan(h, s, batch, cu_seqlens_host, segs_host, cu_segs_host)) != HGX_OK)
    return st;
  cudaError_t e =
      hgx::launch_prologue(s, q, k, pos_thw, q_norm_w, k_norm_w, T, h->cfg.rms_eps, h->rope);
  if (e != cudaSuccess) return cuda_fail(h, e, "prologue launch");
  if ((st = run_attention(h, s, q, k, v, out)) != HGX_OK) return st;
  return finish(h, s);
}

hgx_status hgx_attn_forward_from(hgx_attn_handle* h, void* stream, void* q, void* k,
                                 const void* v, void* out, const int32_t* pos_thw,
                                 const void* q_norm_w, const void* k_norm_w, int32_t batch,
                                 const int32_t* cu_seqlens_host, const hgx_segment* segs_host,
                                 const int32_t* cu_segs_host, const int32_t* first_rows_host) {
  if (!h) return HGX_ERR_INVALID_ARG;
  h->last_error.clear();
  std::string err;
  int32_t T = 0;
  hgx_status st = hgx::validate_descriptor(batch, cu_seqlens_host, segs_host, cu_segs_host,
                                           &err, &T);
  if (st != HGX_OK) return fail(h, st, err);
  if ((st = hgx::check_first_rows(batch, cu_seqlens_host, segs_host, cu_segs_host, first_rows_host,
                                  &err)) != HGX_OK)
    return fail(h, st, err);
  if (T == 0) return HGX_OK;
  if ((st = check_tensors(h, {q, k, v, out, pos_thw, q_norm_w, k_norm_w})) != HGX_OK) return st;
  const size_t qb = size_t(T) * 8192, kb = size_t(T) * 2048;
  if (overlaps(out, qb, q, qb) || overlaps(out, qb, k, kb) || overlaps(out, qb, v, kb))
    return fail(h, HGX_ERR_INVALID_ARG, "out overlaps q, k or v");
  if ((st = ensure_device(h)) != HGX_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if ((st = prepare_plan(h, s, batch, cu_seqlens_host, segs_host, cu_segs_host, first_rows_host)) !=
      HGX_OK)
    return st;
  for (int32_t b = 0; b < batch; ++b) {
    const int32_t t0 = cu_seqlens_host[b] + first_rows_host[b];
    const int32_t n = cu_seqlens_host[b + 1] - t0;
    if (n <= 0) continue;
    cudaError_t e = hgx::launch_prologue(
        s, static_cast<uint8_t*>(q) + size_t(t0) * 8192, static_cast<uint8_t*>(k) + size_t(t0) * 2048,
        pos_thw + 3 * size_t(t0), q_norm_w, k_norm_w, n, h->cfg.rms_eps, h->rope);
    if (e != cudaSuccess) return cuda_fail(h, e, "prologue launch");
  }
  if (!h->plan.items.empty() && (st = run_attention(h, s, q, k, v, out)) != HGX_OK) return st;
  return finish(h, s);
}

hgx_status hgx_attn_qkv_projection(hgx_attn_handle* h, void* stream, const void* x, const void* w_qkv,
                                   void* q, void* k, void* v, const int32_t* pos_thw,
                                   const void* q_norm_w, const void* k_norm_w, int32_t total_tokens) {
  if (!h) return HGX_ERR_INVALID_ARG;
  h->last_error.clear();
  if (total_tokens < 0 || total_tokens > hgx::kMaxTokens)
    return fail(h, HGX_ERR_INVALID_ARG, "total_tokens out of range");
  if (total_tokens == 0) return HGX_OK;
  hgx_status st = check_tensors(h, {x, w_qkv, q, k, v, pos_thw, q_norm_w, k_norm_w});
  if (st != HGX_OK) return st;
  if ((st = ensure_device(h)) != HGX_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if ((st = run_qkv(h, s, x, w_qkv, q, k, v, pos_thw, q_norm_w, k_norm_w, total_tokens)) != HGX_OK) return st;
  return finish(h, s);
}

hgx_status hgx_attn_out_projection(hgx_attn_handle* h, void* stream, const void* attn, const void* w_o,
                                   void* y, int32_t total_tokens) {
  if (!h) return HGX_ERR_INVALID_ARG;
  h->last_error.clear();
  if (total_tokens < 0 || total_tokens > hgx::kMaxTokens)
    return fail(h, HGX_ERR_INVALID_ARG, "total_tokens out of range");
  if (total_tokens == 0) return HGX_OK;
  hgx_status st = check_tensors(h, {attn, w_o, y});
  if (st != HGX_OK) return st;
  if ((st = ensure_device(h)) != HGX_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if ((st = run_out_proj(h, s, attn, w_o, y, total_tokens)) != HGX_OK) return st;
  return finish(h, s);
}

hgx_status hgx_attn_layer_forward(hgx_attn_handle* h, void* stream, const void* x, const void* w_qkv,
                                  const void* w_o, void* q, void* k, void* v, void* attn, void* y,
                                  const int32_t* pos_thw, const void* q_norm_w, const void* k_norm_w,
                                  int32_t batch, const int32_t* cu_seqlens_host,
                                  const hgx_segment* segs_host, const int32_t* cu_segs_host) {
  if (!h) return HGX_ERR_INVALID_ARG;
  h->last_error.clear();
  std::string err;
  int32_t T = 0;
  hgx_status st = hgx::validate_descriptor(batch, cu_seqlens_host, segs_host, cu_segs_host, &err, &T);
  if (st != HGX_OK) return fail(h, st, err);
  if (T == 0) return HGX_OK;
  if ((st = check_tensors(h, {x, w_qkv, w_o, q, k, v, attn, y, pos_thw, q_norm_w, k_norm_w})) != HGX_OK)
    return st;
  const size_t qb = size_t(T) * 8192, kb = size_t(T) * 2048;
  if (overlaps(attn, qb, q, qb) || overlaps(attn, qb, k, kb) || overlaps(attn, qb, v, kb))
    return fail(h, HGX_ERR_INVALID_ARG, "attn overlaps q, k or v");
  if ((st = ensure_device(h)) != HGX_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if ((st = prepare_plan(h, s, batch, cu_seqlens_host, segs_host, cu_segs_host)) != HGX_OK) return st;
  if ((st = run_qkv(h, s, x, w_qkv, q, k, v, pos_thw, q_norm_w, k_norm_w, T)) != HGX_OK) return st;
  if ((st = run_attention(h, s, q, k, v, attn)) != HGX_OK) return st;
  if ((st = run_out_proj(h, s, attn, w_o, y, T)) != HGX_OK) return st;
  return finish(h, s);
}

hgx_status hgx_attn_row_limits(int32_t batch, const int32_t* cu_seqlens_host,
                               const hgx_segment* segs_host, const int32_t* cu_segs_host,
                               int32_t* lim_out, size_t cap) {
  std::vector<int32_t> lim;
  std::string err;
  hgx_status st = hgx::row_limits(batch, cu_seqlens_host, segs_host, cu_segs_host, &lim, &err);
  if (st != HGX_OK) return st;
  if (lim.empty()) return HGX_OK;
  if (!lim_out || cap < lim.size()) return HGX_ERR_INVALID_ARG;
  std::memcpy(lim_out, lim.data(), lim.size() * sizeof(int32_t));
  return HGX_OK;
}

hgx_status hgx_attn_classify(int32_t batch, const int32_t* cu_seqlens_host,
                             const hgx_segment* segs_host, const int32_t* cu_segs_host,
                             int32_t* bm_tokens, int32_t* bn_keys, uint8_t* classes_out,
                             size_t cap, size_t* n_written) {
  if (bm_tokens) *bm_tokens = hgx::kBlockTokens;
  if (bn_keys) *bn_keys = hgx::kBlockKeys;
  hgx::Plan plan;
  std::string err;
  hgx_status st = hgx::build_plan(batch, cu_seqlens_host, segs_host, cu_segs_host, 1, &plan, &err);
  if (st != HGX_OK) return st;
  std::vector<uint8_t> classes;
  hgx::tile_classes(plan, batch, cu_seqlens_host, &classes);
  if (n_written) *n_written = classes.size();
  if (!classes_out) return HGX_OK;
  if (cap < classes.size()) return HGX_ERR_INVALID_ARG;
  if (!classes.empty()) std::memcpy(classes_out, classes.data(), classes.size());
  return HGX_OK;
}

hgx_status hgx_attn_schedule(int32_t batch, const int32_t* cu_seqlens_host,
                             const hgx_segment* segs_host, const int32_t* cu_segs_host, int32_t ctas,
                             int32_t mode, int32_t* out, size_t cap, size_t* n_items) {
  if (n_items) *n_items = 0;
  if (ctas < 1 || mode < 0 || mode > 2) return HGX_ERR_INVALID_ARG;
  hgx::Plan plan;
  std::string err;
  hgx_status st = hgx::build_plan(batch, cu_seqlens_host, segs_host, cu_segs_host, 8, &plan, &err);
  if (st != HGX_OK) return st;
  hgx::assign_ctas(&plan, ctas, mode == 0 ? kSplitKV : true, mode == 2);
  const size_t n = plan.items.size();
  if (n_items) *n_items = n;
  if (!out) return HGX_OK;
  if (cap < n) return HGX_ERR_INVALID_ARG;
  for (int32_t c = 0; c < plan.grid; ++c)
    for (int32_t i = plan.cta_offsets[static_cast<size_t>(c)]; i < plan.cta_offsets[static_cast<size_t>(c) + 1]; ++i) {
      const hgx::WorkItem& it = plan.items[static_cast<size_t>(i)];
      int32_t* r = out + 8 * static_cast<size_t>(i);
      r[0] = c;
      r[1] = it.q0;
      r[2] = it.g;
      r[3] = it.kb0;
      r[4] = it.n_total;
      r[5] = it.part;
      r[6] = it.n_full;
      r[7] = it.list_off;
    }
  return HGX_OK;
}

hgx_status hgx_attn_visible_pairs(int32_t batch, const int32_t* cu_seqlens_host,
                                  const hgx_segment* segs_host, const int32_t* cu_segs_host,
                                  uint64_t* pairs) {
  if (!pairs) return HGX_ERR_INVALID_ARG;
  *pairs = 0;
  hgx::Plan plan;
  std::string err;
  hgx_status st = hgx::build_plan(batch, cu_seqlens_host, segs_host, cu_segs_host, 1, &plan, &err);
  if (st != HGX_OK) return st;
  *pairs = plan.visible_pairs;
  return HGX_OK;
}

hgx_status hgx_attn_sync_status(hgx_attn_handle* h, void* stream) {
  if (!h) return HGX_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_fail(h, e, "cudaStreamSynchronize");
  if (!h->d_err) return HGX_OK;
  uint32_t word = 0;
  e = cudaMemcpy(&word, h->d_err, sizeof(word), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(h, e, "cudaMemcpy (error word)");
  if (word) {
    e = cudaMemset(h->d_err, 0, sizeof(uint32_t));
    if (e != cudaSuccess) return cuda_fail(h, e, "cudaMemset (error word)");
    char buf[128];
    std::snprintf(buf, sizeof(buf), "a bounded device wait ran out (error word 0x%08x)", word);
    return fail(h, HGX_ERR_TIMEOUT, buf);
  }
  return HGX_OK;
}

hgx_status hgx_attn_kernel_clock(hgx_attn_handle* h, void* stream, uint64_t* cycles, uint64_t* ns,
                                 double* sm_mhz) {
  if (!h || !cycles || !ns || !sm_mhz) return HGX_ERR_INVALID_ARG;
  if (h->stamps_grid <= 0) return fail(h, HGX_ERR_INVALID_ARG, "no attention launch on this handle yet");
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(h, e, "cudaStreamSynchronize");
  std::vector<uint64_t> st(static_cast<size_t>(h->stamps_grid) * 4);
  e = cudaMemcpy(st.data(), h->d_stamps, st.size() * sizeof(uint64_t), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(h, e, "cudaMemcpy (clock stamps)");
  uint64_t cmax = 0, nmax = 0;
  std::vector<double> mhz;
  for (int c = 0; c < h->stamps_grid; ++c) {
    const uint64_t* s = &st[4 * static_cast<size_t>(c)];
    if (s[2] < s[0] || s[3] <= s[1]) return fail(h, HGX_ERR_CUDA, "clock stamps out of order");
    const uint64_t dc = s[2] - s[0], dn = s[3] - s[1];
    cmax = std::max(cmax, dc);
    nmax = std::max(nmax, dn);
    mhz.push_back(1e3 * static_cast<double>(dc) / static_cast<double>(dn));
  }
  std::nth_element(mhz.begin(), mhz.begin() + mhz.size() / 2, mhz.end());
  *cycles = cmax;
  *ns = nmax;
  *sm_mhz = mhz[mhz.size() / 2];
  return HGX_OK;
}

hgx_status hgx_attn_set_debug(hgx_attn_handle* h, uint32_t flags, uint64_t wait_limit_ns) {
  if (!h) return HGX_ERR_INVALID_ARG;
  if (flags & ~(HGX_DEBUG_CHECKED | HGX_DEBUG_STALL_TEST | HGX_DEBUG_FAIL_ALLOC | HGX_DEBUG_SPLIT_TEST))
    return fail(h, HGX_ERR_INVALID_ARG, "unknown debug flag");
  h->flags = flags;
  h->wait_limit_ns = wait_limit_ns ? wait_limit_ns : 2000000000ull;
  return HGX_OK;
}

}  // extern "C"
