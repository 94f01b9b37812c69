// hgx_attn_forward_noalloc: the whole path (prologue + masked attention) for callers that
// cannot allocate memory.
//
// Who needs it: code that runs where cudaMalloc is off limits -- inside a framework that
// owns every byte of device memory through its own pool and forbids allocation behind its
// back, in a process that must not grow its device footprint after start-up, or in an
// embedding that cannot create the handle (the handle lazily allocates its planner scratch
// with cudaMalloc and pinned host memory with cudaMallocHost). This entry point takes no
// handle and allocates nothing: no cudaMalloc, no cudaFree, no cudaMallocHost, no heap.
//
// Where the scratch lives instead: the attention kernel needs, besides its inputs and
// outputs, the per-row key limits, the work list and a device error word. Here they sit
// in one file-scope __device__ array of fixed size (kScratchBytes, about 185 KB), which
// every GPU that loads this library holds until the process exits. The array's name in
// host code is only a host-side stand-in, so the device address is looked up once per
// device with cudaGetSymbolAddress (done by the first call on that device, with the device
// current) and passed to the kernels. The host side plans into file-scope static buffers
// of the same fixed size.
//
// Sharing: every call uses the same arrays, which keep the last call's contents. The error
// word is cleared at the start of each call; the limits, the work list and the CTA
// offsets are fully rewritten. Calls that overlap on the GPU (on different streams) race
// on the scratch, and calls from several host threads at once race on the host buffers:
// serialise them. The plan is uploaded with cudaMemcpyAsync from the static (pageable)
// host buffers; the driver stages such a copy before the call returns, so the next call
// may rewrite the buffers, but a replay of a recorded copy would read whatever they hold
// then -- which is why a call on a stream that is being captured is refused.
//
// Work assignment: as in the handle path, every persistent CTA gets a contiguous list of
// items, each item (largest planned cost first) going to the least-loaded CTA; the heap of CTA loads
// lives in a fixed static array.
//
// The paper has no counterpart to this entry point; it exists for the callers above.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstring>

#include "../../include/hgx_attn.h"
#include "kernels.h"
#include "planner.h"

namespace {

constexpr int32_t kMaxTokens = HGX_NOALLOC_MAX_TOKENS;
constexpr int32_t kMaxBatch = HGX_NOALLOC_MAX_BATCH;
constexpr int32_t kMaxKvHeads = 8;
// query blocks: sum over elements of ceil(L_b / 64) <= T / 64 + batch
constexpr int32_t kMaxItems = kMaxKvHeads * (kMaxTokens / hgx::kBlockTokens + kMaxBatch);
constexpr int32_t kMaxKeyBlocks = kMaxTokens / hgx::kBlockKeys;
constexpr int32_t kMaxCtas = 256;  // persistent CTAs (one per SM; B200 has 148)

constexpr size_t kErrOffset = 0;
constexpr size_t kLimOffset = 256;
constexpr size_t kItemsOffset = kLimOffset + sizeof(int32_t) * kMaxTokens;
constexpr size_t kCtaOffsetsOffset = kItemsOffset + sizeof(hgx::WorkItem) * kMaxItems;
constexpr size_t kScratchBytes = kCtaOffsetsOffset + sizeof(int32_t) * (kMaxCtas + 1);

// device scratch shared by every call (see the file comment)
static __device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

// host planning buffers, same fixed sizes
static int32_t s_lim[kMaxTokens];
static hgx::WorkItem s_unsorted[kMaxItems];
static hgx::WorkItem s_items[kMaxItems];
constexpr int64_t kMaxCost = hgx::planned_cost_bound(kMaxKeyBlocks);
static int32_t s_bucket[kMaxCost + 2];
static hgx::WorkItem s_assigned[kMaxItems];
static int32_t s_owner[kMaxItems];
static int32_t s_cta_offsets[kMaxCtas + 1];
static int64_t s_heap_load[kMaxCtas];
static int32_t s_heap_cta[kMaxCtas];

struct DeviceSetup {
  unsigned char* scratch = nullptr;  // device address of g_noalloc_scratch
  int num_sms = 0;
};
constexpr int kMaxDevices = 64;
static DeviceSetup s_dev[kMaxDevices];

using PFN_encodeTiled = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                     const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                     const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                     CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

bool encode(CUtensorMap* map, const void* ptr, int heads, int T, int box_heads, int box_tokens) {
  static PFN_encodeTiled fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return false;
    fn = reinterpret_cast<PFN_encodeTiled>(p);
  }
  cuuint64_t dims[3] = {128, static_cast<cuuint64_t>(heads), static_cast<cuuint64_t>(T)};
  cuuint64_t strides[2] = {256, static_cast<cuuint64_t>(heads) * 256};
  cuuint32_t box[3] = {64, static_cast<cuuint32_t>(box_heads), static_cast<cuuint32_t>(box_tokens)};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// One-time set-up per device, with that device current: the scratch array's device
// address and the SM count.
hgx_status setup_device(int dev) {
  if (dev < 0 || dev >= kMaxDevices) return HGX_ERR_UNSUPPORTED;
  DeviceSetup& d = s_dev[dev];
  if (d.scratch) return HGX_OK;
  int major = 0, minor = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
    return HGX_ERR_CUDA;
  if (major != 10 || minor != 0) return HGX_ERR_UNSUPPORTED;
  int sms = 0;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return HGX_ERR_CUDA;
  void* ptr = nullptr;
  if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || !ptr) return HGX_ERR_CUDA;
  d.num_sms = sms;
  d.scratch = static_cast<unsigned char*>(ptr);
  return HGX_OK;
}

bool aligned16(const void* p) { return p && (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool overlaps(const void* a, size_t na, const void* b, size_t nb) {
  const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
  return x < y + nb && y < x + na;
}

hgx_status check_config(const hgx_attn_config* cfg) {
  if (!cfg) return HGX_ERR_INVALID_ARG;
  if (!(cfg->rope_theta > 0.0) || !std::isfinite(cfg->rope_theta)) return HGX_ERR_INVALID_ARG;
  if (!(cfg->rms_eps >= 0.f) || !std::isfinite(cfg->rms_eps)) return HGX_ERR_INVALID_ARG;
  if (!(cfg->softmax_scale >= 0.f) || !std::isfinite(cfg->softmax_scale)) return HGX_ERR_INVALID_ARG;
  if (cfg->num_q_heads <= 0 || cfg->num_kv_heads <= 0 || cfg->head_dim <= 0) return HGX_ERR_INVALID_ARG;
  if (cfg->num_q_heads != 32 || cfg->num_kv_heads != 8 || cfg->head_dim != 128)
    return HGX_ERR_UNSUPPORTED;
  for (int i = 0; i < 3; ++i)
    if (cfg->mrope_section[i] < 0) return HGX_ERR_INVALID_ARG;
  if (cfg->rope_layout < HGX_ROPE_MROPE_INTERLEAVED || cfg->rope_layout > HGX_ROPE_2D_HALVES)
    return HGX_ERR_INVALID_ARG;
  if (cfg->rope_layout == HGX_ROPE_MROPE_INTERLEAVED) {
    if (cfg->mrope_section[0] + cfg->mrope_section[1] + cfg->mrope_section[2] != 64)
      return HGX_ERR_INVALID_ARG;
    // the interleaved assignment must give each axis exactly its section's count
    double inv[64];
    int32_t axis[64], count[3] = {0, 0, 0};
    hgx::mrope_tables(cfg->rope_theta, cfg->head_dim, cfg->mrope_section, cfg->rope_layout, inv, axis);
    for (int i = 0; i < 64; ++i) ++count[axis[i]];
    for (int i = 0; i < 3; ++i)
      if (count[i] != cfg->mrope_section[i]) return HGX_ERR_UNSUPPORTED;
  }
  return HGX_OK;
}

// Min-heap of (load, cta) pairs over the static arrays: the least-loaded CTA, ties to the
// lower index.
bool heap_less(int32_t a, int32_t b) {
  return s_heap_load[a] < s_heap_load[b] || (s_heap_load[a] == s_heap_load[b] && s_heap_cta[a] < s_heap_cta[b]);
}
void heap_swap(int32_t a, int32_t b) {
  const int64_t l = s_heap_load[a];
  s_heap_load[a] = s_heap_load[b];
  s_heap_load[b] = l;
  const int32_t c = s_heap_cta[a];
  s_heap_cta[a] = s_heap_cta[b];
  s_heap_cta[b] = c;
}
void heap_sift_down(int32_t n) {
  for (int32_t i = 0;;) {
    const int32_t l = 2 * i + 1, r = l + 1;
    int32_t m = i;
    if (l < n && heap_less(l, m)) m = l;
    if (r < n && heap_less(r, m)) m = r;
    if (m == i) return;
    heap_swap(i, m);
    i = m;
  }
}

// Longest-processing-time assignment of the n sorted items of s_items to `grid` CTAs
// (cost of an item: hgx::planned_cost, as in the handle path). Fills
// s_cta_offsets[0..grid] and reorders the items into s_assigned so that every CTA's list is
// contiguous and keeps the longest-first order.
void assign(int32_t n, int32_t grid) {
  for (int32_t c = 0; c < grid; ++c) {  // all loads 0: the index order is a valid heap
    s_heap_load[c] = 0;
    s_heap_cta[c] = c;
  }
  for (int32_t c = 0; c <= grid; ++c) s_cta_offsets[c] = 0;
  for (int32_t i = 0; i < n; ++i) {
    const int32_t c = s_heap_cta[0];
    s_owner[i] = c;
    ++s_cta_offsets[c + 1];
    s_heap_load[0] += hgx::planned_cost(s_items[i], nullptr);
    heap_sift_down(grid);
  }
  for (int32_t c = 0; c < grid; ++c) s_cta_offsets[c + 1] += s_cta_offsets[c];
  for (int32_t c = 0; c < grid; ++c) s_heap_cta[c] = s_cta_offsets[c];  // next free slot per CTA
  for (int32_t i = 0; i < n; ++i) s_assigned[s_heap_cta[s_owner[i]]++] = s_items[i];
}

// Validates the descriptor and plans into the static host buffers. Returns the number of
// work items through *n_items and the token count through *T.
hgx_status plan(int32_t batch, const int32_t* cu, const hgx_segment* segs, const int32_t* cu_segs,
                int32_t* T_out, int32_t* n_items) {
  *T_out = 0;
  *n_items = 0;
  if (batch < 0) return HGX_ERR_INVALID_ARG;
  if (batch == 0) return HGX_OK;
  if (batch > kMaxBatch) return HGX_ERR_UNSUPPORTED;
  if (!cu || !cu_segs || cu[0] != 0 || cu_segs[0] != 0) return HGX_ERR_INVALID_ARG;
  for (int32_t b = 0; b < batch; ++b) {
    if (cu[b + 1] < cu[b] || cu_segs[b + 1] < cu_segs[b]) return HGX_ERR_INVALID_ARG;
    if (cu[b + 1] > hgx::kMaxTokens) return HGX_ERR_INVALID_ARG;
  }
  const int32_t T = cu[batch];
  if (T > kMaxTokens) return HGX_ERR_UNSUPPORTED;
  if (cu_segs[batch] > 0 && !segs) return HGX_ERR_INVALID_ARG;
  for (int32_t b = 0; b < batch; ++b) {
    const int32_t base = cu[b], L = cu[b + 1] - cu[b];
    int32_t at = 0;
    for (int32_t s = cu_segs[b]; s < cu_segs[b + 1]; ++s) {
      const hgx_segment& sg = segs[s];
      if (sg.kind == HGX_SEG_GEN_IMAGE) return HGX_ERR_UNSUPPORTED;  // no hole tables here
      if (sg.kind < HGX_SEG_CAUSAL || sg.kind > HGX_SEG_FULL_IN_SEGMENT || sg.len < 1 ||
          sg.start != at || sg.len > L - at)
        return HGX_ERR_INVALID_ARG;
      for (int32_t i = sg.start; i < sg.start + sg.len; ++i)
        s_lim[base + i] = sg.kind == HGX_SEG_CAUSAL          ? i + 1
                          : sg.kind == HGX_SEG_FULL_SEQUENCE ? L
                                                             : sg.start + sg.len;
      at += sg.len;
    }
    if (at != L) return HGX_ERR_INVALID_ARG;
  }
  // work items, then a stable counting sort by planned cost, largest first
  int32_t n = 0;
  for (int32_t b = 0; b < batch; ++b) {
    const int32_t base = cu[b], L = cu[b + 1] - cu[b];
    for (int32_t r0 = 0; r0 < L; r0 += hgx::kBlockTokens) {
      const int32_t r1 = r0 + hgx::kBlockTokens < L ? r0 + hgx::kBlockTokens : L;
      int32_t lo = s_lim[base + r0], hi = lo;
      for (int32_t i = r0 + 1; i < r1; ++i) {
        lo = s_lim[base + i] < lo ? s_lim[base + i] : lo;
        hi = s_lim[base + i] > hi ? s_lim[base + i] : hi;
      }
      for (int32_t g = 0; g < kMaxKvHeads; ++g) {
        hgx::WorkItem& it = s_unsorted[n++];
        it = hgx::WorkItem{};
        it.q0 = base + r0;
        it.kv0 = base;
        it.len = L;
        it.g = g;
        it.n_full = lo / hgx::kBlockKeys;
        it.n_total = (hi + hgx::kBlockKeys - 1) / hgx::kBlockKeys;
        it.list_off = -1;  // prefix form
      }
    }
  }
  std::memset(s_bucket, 0, sizeof(s_bucket));
  for (int32_t i = 0; i < n; ++i) ++s_bucket[kMaxCost - hgx::planned_cost(s_unsorted[i], nullptr) + 1];
  for (int64_t k = 1; k < kMaxCost + 2; ++k) s_bucket[k] += s_bucket[k - 1];
  for (int32_t i = 0; i < n; ++i)
    s_items[s_bucket[kMaxCost - hgx::planned_cost(s_unsorted[i], nullptr)]++] = s_unsorted[i];
  *T_out = T;
  *n_items = n;
  return HGX_OK;
}

}  // namespace

extern "C" hgx_status hgx_attn_forward_noalloc(const hgx_attn_config* cfg, void* stream, void* q,
                                               void* k, const void* v, void* out,
                                               const int32_t* pos_thw, const void* q_norm_w,
                                               const void* k_norm_w, int32_t batch,
                                               const int32_t* cu_seqlens_host,
                                               const hgx_segment* segs_host,
                                               const int32_t* cu_segs_host, int32_t synchronize) {
  hgx_status st = check_config(cfg);
  if (st != HGX_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int32_t T = 0, n_items = 0;
  if ((st = plan(batch, cu_seqlens_host, segs_host, cu_segs_host, &T, &n_items)) != HGX_OK)
    return st;
  if (T == 0) return HGX_OK;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(pos_thw) ||
      !aligned16(q_norm_w) || !aligned16(k_norm_w))
    return HGX_ERR_INVALID_ARG;
  const size_t qb = size_t(T) * 8192, kb = size_t(T) * 2048;
  if (overlaps(out, qb, q, qb) || overlaps(out, qb, k, kb) || overlaps(out, qb, v, kb))
    return HGX_ERR_INVALID_ARG;
  {
    // refused while the stream is being captured (see the file comment); the legacy
    // stream under another stream's capture reports cudaErrorStreamCaptureImplicit
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    const cudaError_t e = cudaStreamIsCapturing(s, &cs);
    if (e == cudaErrorStreamCaptureImplicit || (e == cudaSuccess && cs != cudaStreamCaptureStatusNone))
      return HGX_ERR_UNSUPPORTED;
    if (e != cudaSuccess) return HGX_ERR_CUDA;
  }
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return HGX_ERR_CUDA;
  if ((st = setup_device(dev)) != HGX_OK) return st;
  const DeviceSetup& d = s_dev[dev];
  const int32_t grid = n_items < d.num_sms ? (n_items < kMaxCtas ? n_items : kMaxCtas)
                                            : (d.num_sms < kMaxCtas ? d.num_sms : kMaxCtas);
  assign(n_items, grid);

  uint32_t* d_err = reinterpret_cast<uint32_t*>(d.scratch + kErrOffset);
  int32_t* d_lim = reinterpret_cast<int32_t*>(d.scratch + kLimOffset);
  hgx::WorkItem* d_items = reinterpret_cast<hgx::WorkItem*>(d.scratch + kItemsOffset);
  int32_t* d_cta_offsets = reinterpret_cast<int32_t*>(d.scratch + kCtaOffsetsOffset);
  // the error word must start at zero; limits, work list and CTA offsets are rewritten in
  // full
  if (cudaMemsetAsync(d_err, 0, sizeof(uint32_t), s) != cudaSuccess ||
      cudaMemcpyAsync(d_lim, s_lim, sizeof(int32_t) * T, cudaMemcpyHostToDevice, s) != cudaSuccess ||
      cudaMemcpyAsync(d_items, s_assigned, sizeof(hgx::WorkItem) * n_items, cudaMemcpyHostToDevice, s) !=
          cudaSuccess ||
      cudaMemcpyAsync(d_cta_offsets, s_cta_offsets, sizeof(int32_t) * (grid + 1), cudaMemcpyHostToDevice, s) !=
          cudaSuccess)
    return HGX_ERR_CUDA;

  hgx::RopeTables rope{};
  int32_t axis[64];
  hgx::mrope_tables(cfg->rope_theta, cfg->head_dim, cfg->mrope_section, cfg->rope_layout,
                    rope.inv_freq, axis);
  for (int i = 0; i < 64; ++i) rope.axis[i] = static_cast<uint8_t>(axis[i]);
  if (hgx::launch_prologue(s, q, k, pos_thw, q_norm_w, k_norm_w, T, cfg->rms_eps, rope) != cudaSuccess)
    return HGX_ERR_CUDA;

  CUtensorMap mq, mk, mv, mo;
  if (!encode(&mq, q, 32, T, 4, hgx::kTileTokens) || !encode(&mk, k, 8, T, 1, 128) ||
      !encode(&mv, v, 8, T, 1, 128) || !encode(&mo, out, 32, T, 4, 8))
    return HGX_ERR_CUDA;
  const float scale = cfg->softmax_scale > 0.f ? cfg->softmax_scale
                                               : static_cast<float>(1.0 / std::sqrt(128.0));
  hgx::AttnParams p{};
  p.items = d_items;
  p.n_items = n_items;
  p.cta_offsets = d_cta_offsets;
  p.total_tokens = T;
  p.lim = d_lim;
  p.out = out;
  p.out_tma = 1;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.flags = 0;
  p.err = d_err;
  p.wait_limit_ns = 2000000000ull;
  if (hgx::launch_attention(s, mq, mk, mv, mo, p, grid) != cudaSuccess) return HGX_ERR_CUDA;
  if (!synchronize) return HGX_OK;
  if (cudaStreamSynchronize(s) != cudaSuccess) return HGX_ERR_CUDA;
  uint32_t word = 0;
  if (cudaMemcpy(&word, d_err, sizeof(word), cudaMemcpyDeviceToHost) != cudaSuccess)
    return HGX_ERR_CUDA;
  return word ? HGX_ERR_TIMEOUT : HGX_OK;
}
