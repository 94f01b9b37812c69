// Launch interfaces of the device kernels (internal to the library).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "planner.h"

namespace hgx {

// mRoPE tables passed by value to the prologue: inv_freq[k] = theta^(-2k/128) and the
// axis (0 t, 1 h, 2 w) that drives frequency k.
struct RopeTables {
  double inv_freq[64];
  uint8_t axis[64];
};

cudaError_t launch_prologue(cudaStream_t stream, void* q, void* k, const int32_t* pos,
                            const void* wq, const void* wk, int32_t T, float eps,
                            const RopeTables& tab);

struct AttnParams {
  const WorkItem* items;
  int32_t n_items;
  int32_t total_tokens;
  const int32_t* lim;      // [T] exclusive key limit per packed row, local
  const uint32_t* kblocks;     // key-block lists of list-form items (holes only)
  const int32_t* hole_base;    // [T] row's first hole-mask index, -1 = none (holes only)
  const uint32_t* hole_masks;  // 4 words per (segment, key block): hidden keys (holes only)
  void* out;               // bf16 [T, 32, 128]
  float scale_log2;        // softmax scale * log2(e)
  uint32_t flags;          // HGX_DEBUG_* bits
  uint32_t* err;           // device error word (sticky until read)
  uint64_t wait_limit_ns;  // bound of every wait
};

// Bytes of dynamic shared memory the attention kernel needs.
size_t attention_smem_bytes();

cudaError_t launch_attention(cudaStream_t stream, const CUtensorMap& tmap_q,
                             const CUtensorMap& tmap_k, const CUtensorMap& tmap_v,
                             const AttnParams& p, int grid);

// Device error word bits written by the attention kernel.
constexpr uint32_t kErrTimeout = 1u;

}  // namespace hgx
