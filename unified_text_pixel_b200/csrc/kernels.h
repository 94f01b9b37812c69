// Launch interfaces of the device kernels (internal to the library).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
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
  const int32_t* cta_offsets;  // CTA c takes items [cta_offsets[c], cta_offsets[c+1]);
                               // NULL: CTA c takes items c, c + gridDim.x, ...
  int32_t total_tokens;
  const int32_t* lim;      // [T] exclusive key limit per packed row, local
  const uint32_t* kblocks;     // key-block lists of list-form items (holes only)
  const int32_t* hole_base;    // [T] row's first hole-mask index, -1 = none (holes only)
  const uint32_t* hole_masks;  // 4 words per (segment, key block): hidden keys (holes only)
  void* out;               // bf16 [T, 32, 128]
  uint32_t out_tma;        // 1: tmap_out describes out (epilogue TMA stores)
  float* partial_o;        // split items: unnormalised O per slot, fp32 [slots][2][128][128]
  float2* partial_ml;      // split items: (row maximum x scale log2 e, row sum) [slots][2][128]
  float scale_log2;        // softmax scale * log2(e)
  uint32_t flags;          // HGX_DEBUG_* bits
  uint32_t* err;           // device error word (sticky until read)
  uint64_t wait_limit_ns;  // bound of every wait
  uint64_t* stamps;        // NULL, or [grid][4]: per CTA clock64 and %globaltimer at its start
                           // and at its end (the effective SM clock of the launch)
};

// Merges the partial results of every split item into out (bf16):
// out = sum_p O_p 2^(M_p - M) / sum_p l_p 2^(M_p - M), M = the largest M_p of the parts the
// row saw keys in.
cudaError_t launch_combine(cudaStream_t stream, const WorkItem* splits, int32_t n_splits,
                           const float* partial_o, const float2* partial_ml, void* out);
constexpr size_t kPartialSlotFloats = 2 * 128 * 128;  // fp32 O of one slot
constexpr size_t kPartialSlotRows = 2 * 128;          // rows (and (M, l) pairs) of one slot

// Bytes of dynamic shared memory the attention kernel needs.
size_t attention_smem_bytes();

// tmap_out: bf16 out [T, 32, 128] with a (64 features, 4 heads, 8 tokens) box and 128-byte
// swizzle, used when p.out_tma is set (the epilogue's TMA stores)
cudaError_t launch_attention(cudaStream_t stream, const CUtensorMap& tmap_q,
                             const CUtensorMap& tmap_k, const CUtensorMap& tmap_v,
                             const CUtensorMap& tmap_out, const AttnParams& p, int grid);

struct GemmParams {
  int32_t M, N, K;           // C[M, N] = A[M, K] * B[N, K]^T; N % 256 == 0, K % 64 == 0
  int32_t mode;              // 0: C bf16 [M, N]; 1: QKV split with q/k RMSNorm + rotation
  void* c;                   // mode 0 output
  void* q;                   // mode 1 outputs: q' [M,32,128], k' [M,8,128], v [M,8,128]
  void* k;
  void* v;
  const float2* rope_cs;     // mode 1: [M, 64] (cos, sin) of every (token, frequency)
  const __nv_bfloat16* wq;   // mode 1: RMSNorm weights [128]
  const __nv_bfloat16* wk;
  float eps;
  uint32_t* err;
  uint64_t wait_limit_ns;
};

cudaError_t launch_gemm(cudaStream_t stream, const CUtensorMap& tmap_a, const CUtensorMap& tmap_b,
                        const GemmParams& p, int grid);
cudaError_t launch_rope_table(cudaStream_t stream, const int32_t* pos, int32_t T,
                              const RopeTables& tab, void* cs);

// Device error word bits written by the attention kernel.
constexpr uint32_t kErrTimeout = 1u;

}  // namespace hgx
