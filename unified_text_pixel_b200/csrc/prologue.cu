// Prologue: q/k RMSNorm and interleaved 3-axis mRoPE, in place, bf16 in and out.
//
// "hidream-o1-p100a" model card, "What this model is": the language model applies "q/k
// RMSNorm" and "3-axis interleaved mRoPE [24,20,20] at theta 5e6" (32 query heads, 8 KV
// heads, head 128). Rotation pairs feature k with feature k + 64, the half-split layout of
// the 1D RoPE definition in "HunyuanImage 3.0 Technical Report" (paper-graph-ui summary),
// section 3.4, "Generalized 2D Rotary Position Embedding (RoPE)".
//
// Layout: one block handles kTok tokens and all 40 heads (32 q + 8 k) of each (1 token,
// 64 threads: many small blocks keep loads in flight while others compute). A head's
// 128 bf16 (256 B) is read by a half-warp as 16-byte loads, so a warp reads 512
// contiguous bytes; lanes j and j + 8 of a half-warp hold the partners (k, k + 64) of a
// rotation and swap values with one shuffle. Angles are computed once per (token, k) in
// fp64 (positions reach ~10^4 rad, far outside the range where a float angle keeps
// precision) and shared by all 40 heads through shared memory; they are computed while
// the thread's loads (all issued first, 160 bytes per thread) are in flight. HBM-bound:
// every byte of q and k is read once and written once.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "kernels.h"

namespace hgx {

namespace {

// Block shape, measured on B200 (edit step, 8449 tokens, read + write bytes / time):
// 1 token x 64 threads 4.96 TB/s, 1 x 128 4.75, 2 x 128 4.69, 2 x 64 3.99, 4 x 128 3.63,
// 2 x 256 3.32, 4 x 256 3.03, 4 x 512 2.07, 8 x 512 1.97.
#ifndef HGX_PRO_TOK
#define HGX_PRO_TOK 1
#endif
#ifndef HGX_PRO_THREADS
#define HGX_PRO_THREADS 64
#endif
constexpr int kTok = HGX_PRO_TOK;          // tokens per block
constexpr int kThreads = HGX_PRO_THREADS;  // kThreads / 16 heads in flight
constexpr int kHeads = 40;       // 32 query + 8 key heads per token
constexpr int kHalf = 64;        // rotation pairs per head

__device__ __forceinline__ void unpack8(const uint4& r, float (&x)[8]) {
  const uint32_t w[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    x[2 * i] = __uint_as_float(w[i] << 16);
    x[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

__device__ __forceinline__ uint4 pack8(const float (&y)[8]) {
  uint32_t w[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    __nv_bfloat162 b = __floats2bfloat162_rn(y[2 * i], y[2 * i + 1]);
    w[i] = *reinterpret_cast<uint32_t*>(&b);
  }
  return make_uint4(w[0], w[1], w[2], w[3]);
}

constexpr int kUnits = kTok * kHeads / (kThreads / 16);  // (token, head) pairs per half-warp
static_assert(kTok * kHeads % (kThreads / 16) == 0, "units must split evenly over half-warps");

#ifndef HGX_PRO_MIN_BLOCKS
#define HGX_PRO_MIN_BLOCKS 12
#endif
// resident blocks per SM the register allocation must allow: 12 caps the kernel at 80
// registers (96 unconstrained, i.e. 10 blocks), which measured 5 % faster on B200; 16 spills
constexpr int kProMinBlocks = HGX_PRO_MIN_BLOCKS;

__global__ void __launch_bounds__(kThreads, kProMinBlocks) prologue_kernel(
    __nv_bfloat16* __restrict__ q, __nv_bfloat16* __restrict__ k,
    const int32_t* __restrict__ pos, const __nv_bfloat16* __restrict__ wq,
    const __nv_bfloat16* __restrict__ wk, int32_t T, float eps, const RopeTables tab) {
  __shared__ float2 cs[kTok][kHalf];  // (cos, sin) per token and frequency
  const int t0 = blockIdx.x * kTok;
  const int j = threadIdx.x & 15;  // 16-byte chunk of the head: features 8j .. 8j+7
  const int u0 = threadIdx.x >> 4;

  // 1. every load of this thread first, so that kUnits x 16 bytes are in flight at once
  uint4 raw[kUnits];
#pragma unroll
  for (int n = 0; n < kUnits; ++n) {
    const int u = u0 + n * (kThreads / 16);
    const int tl = u / kHeads, hh = u % kHeads, t = t0 + tl;
    raw[n] = make_uint4(0, 0, 0, 0);
    if (t < T) {
      const __nv_bfloat16* base = hh < 32 ? q + (static_cast<size_t>(t) * 32 + hh) * 128
                                          : k + (static_cast<size_t>(t) * 8 + (hh - 32)) * 128;
      raw[n] = *reinterpret_cast<const uint4*>(base + 8 * j);
    }
  }
  // 2. angles while the loads are in flight: (token, frequency) pairs over the threads, fp64
  for (int idx = threadIdx.x; idx < kTok * kHalf; idx += kThreads) {
    const int tl = idx / kHalf;
    const int f = idx % kHalf;
    const int t = t0 + tl;
    float c = 1.f, sn = 0.f;
    if (t < T) {
      const double phi = static_cast<double>(pos[3 * t + tab.axis[f]]) * tab.inv_freq[f];
      double sd, cd;
      sincos(phi, &sd, &cd);
      c = static_cast<float>(cd);
      sn = static_cast<float>(sd);
    }
    cs[tl][f] = make_float2(c, sn);
  }
  float wqv[8], wkv[8];
  unpack8(*reinterpret_cast<const uint4*>(wq + 8 * j), wqv);
  unpack8(*reinterpret_cast<const uint4*>(wk + 8 * j), wkv);
  __syncthreads();

  // 3. normalise, rotate, store
  const bool low = j < 8;          // features < 64: first member of each pair
  const int f0 = (j & 7) * 8;      // frequency of this lane's first feature
#pragma unroll
  for (int n = 0; n < kUnits; ++n) {
    const int u = u0 + n * (kThreads / 16);
    const int tl = u / kHeads, hh = u % kHeads, t = t0 + tl;
    float x[8];
    unpack8(raw[n], x);
    float ss = 0.f;
#pragma unroll
    for (int e = 0; e < 8; ++e) ss = fmaf(x[e], x[e], ss);
#pragma unroll
    for (int off = 8; off >= 1; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
    const float r = rsqrtf(ss * (1.f / 128.f) + eps);
    const float* w = hh < 32 ? wqv : wkv;
    float y[8], yp[8], o[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) y[e] = x[e] * r * w[e];
#pragma unroll
    for (int e = 0; e < 8; ++e) yp[e] = __shfl_xor_sync(0xffffffffu, y[e], 8);
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const float2 c = cs[tl][f0 + e];
      o[e] = low ? fmaf(y[e], c.x, -yp[e] * c.y) : fmaf(y[e], c.x, yp[e] * c.y);
    }
    if (t < T) {
      __nv_bfloat16* base = hh < 32 ? q + (static_cast<size_t>(t) * 32 + hh) * 128
                                    : k + (static_cast<size_t>(t) * 8 + (hh - 32)) * 128;
      *reinterpret_cast<uint4*>(base + 8 * j) = pack8(o);
    }
  }
}

}  // namespace

cudaError_t launch_prologue(cudaStream_t stream, void* q, void* k, const int32_t* pos,
                            const void* wq, const void* wk, int32_t T, float eps,
                            const RopeTables& tab) {
  if (T <= 0) return cudaSuccess;
  const int grid = (T + kTok - 1) / kTok;
  prologue_kernel<<<grid, kThreads, 0, stream>>>(
      static_cast<__nv_bfloat16*>(q), static_cast<__nv_bfloat16*>(k), pos,
      static_cast<const __nv_bfloat16*>(wq), static_cast<const __nv_bfloat16*>(wk), T, eps, tab);
  return cudaGetLastError();
}

}  // namespace hgx
