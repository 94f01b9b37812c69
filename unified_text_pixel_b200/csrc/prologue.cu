// Prologue: q/k RMSNorm and interleaved 3-axis mRoPE, in place, bf16 in and out.
//
// "hidream-o1-p100a" model card, "What this model is": the language model applies "q/k
// RMSNorm" and "3-axis interleaved mRoPE [24,20,20] at theta 5e6" (32 query heads, 8 KV
// heads, head 128). Rotation pairs feature k with feature k + 64, the half-split layout of
// the 1D RoPE definition in "HunyuanImage 3.0 Technical Report" (paper-graph-ui summary),
// section 3.4, "Generalized 2D Rotary Position Embedding (RoPE)".
//
// HBM-bound: every byte of q and k is read once and written once. The default kernel
// (prologue_v2_kernel, described at its definition) gives each thread both members of its
// rotation pairs and reduces the angles exactly in fp32; the first layout (prologue_kernel,
// HGX_PRO_V2=0: a half-warp per head, partners exchanged by shuffles, fp64 angles) is kept
// for comparison.
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

// ----------------------------------------------------------------------------------------
// Second layout (HGX_PRO_V2, default): a thread holds both members of its rotation pairs --
// features 8j .. 8j+7 and 64+8j .. 64+8j+7 of a head (two 16-byte loads) -- so the rotation
// needs no shuffle; eight threads cover a head (the sum of squares is reduced over them with
// three shuffles) and the 64 threads of a block five heads each. The (cos, sin) table is
// stored transposed, entry (e, j) for frequency 8j + e, so that the eight threads of a head
// read 64 consecutive bytes (no bank conflicts). Angles are reduced in fp32 without loss:
// the position is an integer below 2^24, u = inv_freq / 2pi is split into u_hi + u_lo
// (floats), pos * u_hi is exact as hi + err (an FMA gives the rounding error), and the
// fraction of a turn r = (hi - rint(hi)) + (err + pos * u_lo) carries an error near 2^-25;
// sincospif(2r) gives cos and sin of 2 pi r. Positions of 2^24 or more take the fp64 sincos.
struct RopeTurns {
  float u_hi[64];
  float u_lo[64];
  double inv_freq[64];
  uint8_t axis[64];
};

#ifndef HGX_PRO_V2
#define HGX_PRO_V2 1
#endif
#ifndef HGX_PRO_V2_THREADS
#define HGX_PRO_V2_THREADS 160
#endif
constexpr int kV2Threads = HGX_PRO_V2_THREADS;  // 8 per head in flight
constexpr int kV2Units = kHeads * 8 / kV2Threads;  // heads per thread
static_assert(kV2Threads % 64 == 0 || kV2Threads == 160 || kV2Threads == 320, "block shape");
static_assert(kHeads * 8 % kV2Threads == 0, "heads must split evenly over the threads");
// resident blocks per SM the register allocation must allow (no spills at these shapes)
constexpr int kV2MinBlocks = kV2Threads == 320 ? 6 : kV2Threads == 160 ? 8 : 10;

__global__ void __launch_bounds__(kV2Threads, kV2MinBlocks) prologue_v2_kernel(
    __nv_bfloat16* __restrict__ q, __nv_bfloat16* __restrict__ k,
    const int32_t* __restrict__ pos, const __nv_bfloat16* __restrict__ wq,
    const __nv_bfloat16* __restrict__ wk, int32_t T, float eps, const __grid_constant__ RopeTurns tab) {
  __shared__ float2 cs[8][8];  // (cos, sin) of frequency 8j + e at [e][j]
  const int t = blockIdx.x;
  const int j = threadIdx.x & 7;   // pair chunk: features 8j.. and 64+8j..
  const int u0 = threadIdx.x >> 3; // first head of this thread (kV2Threads / 8 in flight)
  // 1. the loads: kV2Units heads x 2 chunks of 16 bytes, all in flight before any is used (and
  // before the angles, whose arithmetic then overlaps them)
  uint4 lo[kV2Units], hi[kV2Units];
#pragma unroll
  for (int n = 0; n < kV2Units; ++n) {
    const int hh = u0 + (kV2Threads / 8) * n;
    const __nv_bfloat16* base = hh < 32 ? q + (static_cast<size_t>(t) * 32 + hh) * 128
                                        : k + (static_cast<size_t>(t) * 8 + (hh - 32)) * 128;
    lo[n] = *reinterpret_cast<const uint4*>(base + 8 * j);
    hi[n] = *reinterpret_cast<const uint4*>(base + 64 + 8 * j);
  }
  // 2. the angle of frequency f = threadIdx.x (fp32 fast path: a few dozen instructions)
  if (threadIdx.x < 64) {
    const int f = threadIdx.x;
    const int32_t pv = pos[3 * t + tab.axis[f]];
    float c, sn;
    if (pv > -(1 << 24) && pv < (1 << 24)) {
      const float pf = static_cast<float>(pv);
      const float h = pf * tab.u_hi[f];
      const float err = fmaf(pf, tab.u_hi[f], -h);
      const float r = (h - rintf(h)) + fmaf(pf, tab.u_lo[f], err);
      sincospif(2.f * r, &sn, &c);
    } else {
      double sd, cd;
      sincos(static_cast<double>(pv) * tab.inv_freq[f], &sd, &cd);
      c = static_cast<float>(cd);
      sn = static_cast<float>(sd);
    }
    cs[f & 7][f >> 3] = make_float2(c, sn);
  }
  __syncthreads();
  float2 cj[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) cj[e] = cs[e][j];
  // 3. normalise, rotate, store
#pragma unroll
  for (int n = 0; n < kV2Units; ++n) {
    const int hh = u0 + (kV2Threads / 8) * n;
    float a[8], b[8];
    unpack8(lo[n], a);
    unpack8(hi[n], b);
    float ss = 0.f;
#pragma unroll
    for (int e = 0; e < 8; ++e) ss = fmaf(a[e], a[e], fmaf(b[e], b[e], ss));
#pragma unroll
    for (int off = 4; off >= 1; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
    const float r = rsqrtf(ss * (1.f / 128.f) + eps);
    // norm weights of this thread's 16 features (L1-resident after the first token)
    const __nv_bfloat16* wsrc = hh < 32 ? wq : wk;
    float wa[8], wb[8];
    unpack8(__ldg(reinterpret_cast<const uint4*>(wsrc + 8 * j)), wa);
    unpack8(__ldg(reinterpret_cast<const uint4*>(wsrc + 64 + 8 * j)), wb);
    float oa[8], ob[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const float ya = a[e] * r * wa[e], yb = b[e] * r * wb[e];
      oa[e] = fmaf(ya, cj[e].x, -yb * cj[e].y);
      ob[e] = fmaf(yb, cj[e].x, ya * cj[e].y);
    }
    __nv_bfloat16* base = hh < 32 ? q + (static_cast<size_t>(t) * 32 + hh) * 128
                                  : k + (static_cast<size_t>(t) * 8 + (hh - 32)) * 128;
    *reinterpret_cast<uint4*>(base + 8 * j) = pack8(oa);
    *reinterpret_cast<uint4*>(base + 64 + 8 * j) = pack8(ob);
  }
}

}  // namespace

cudaError_t launch_prologue(cudaStream_t stream, void* q, void* k, const int32_t* pos,
                            const void* wq, const void* wk, int32_t T, float eps,
                            const RopeTables& tab) {
  if (T <= 0) return cudaSuccess;
  if constexpr (HGX_PRO_V2 != 0) {
    RopeTurns turns{};
    for (int f = 0; f < 64; ++f) {
      const double u = tab.inv_freq[f] / (2.0 * 3.14159265358979323846);
      turns.u_hi[f] = static_cast<float>(u);
      turns.u_lo[f] = static_cast<float>(u - static_cast<double>(turns.u_hi[f]));
      turns.inv_freq[f] = tab.inv_freq[f];
      turns.axis[f] = tab.axis[f];
    }
    prologue_v2_kernel<<<T, kV2Threads, 0, stream>>>(
        static_cast<__nv_bfloat16*>(q), static_cast<__nv_bfloat16*>(k), pos,
        static_cast<const __nv_bfloat16*>(wq), static_cast<const __nv_bfloat16*>(wk), T, eps, turns);
    return cudaGetLastError();
  }
  const int grid = (T + kTok - 1) / kTok;
  prologue_kernel<<<grid, kThreads, 0, stream>>>(
      static_cast<__nv_bfloat16*>(q), static_cast<__nv_bfloat16*>(k), pos,
      static_cast<const __nv_bfloat16*>(wq), static_cast<const __nv_bfloat16*>(wk), T, eps, tab);
  return cudaGetLastError();
}

}  // namespace hgx
