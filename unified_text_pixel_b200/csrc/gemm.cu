// Projections of the attention layer as tcgen05 GEMMs: C[M, N] = A[M, K] * B[N, K]^T, bf16
// in, fp32 accumulation in tensor memory, bf16 out.
//
// The layer ("hidream-o1-p100a" model card, "What this model is": hidden 4096, 32 query
// heads over 8 KV heads of 128) projects x [T, 4096] to q | k | v (6144 columns) and the
// attention output [T, 4096] back to 4096. In the QKV epilogue every thread holds one token
// row of a whole 128-column head (tcgen05.ld 32x32b: one TMEM lane per thread), so the q/k
// RMSNorm over head_dim and the rotation of feature pairs (k, k + 64) are thread-local:
// q' and k' leave the GEMM already normalised and rotated, and the separate prologue pass
// over q and k in HBM disappears.
//
// CTA organisation (one CTA per SM, persistent): tiles of 128 x 256 (two heads) with K
// stepped by 64 (one 128-byte swizzle span), a 4-stage TMA ring of A and B tiles (48 KB per
// stage), two 256-column fp32 accumulators in tensor memory so that the epilogue of one
// tile overlaps the MMAs of the next.
//   warp 0      TMA producer         warp 1      TMEM allocator, single-thread MMA issuer
//   warps 2-5   epilogue (one accumulator row per thread)
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "kernels.h"
#include "sm100.cuh"
#include "waits.cuh"

namespace hgx {

namespace {

using namespace sm100;
using namespace waits;

#ifndef HGX_GEMM_L2_HINTS
#define HGX_GEMM_L2_HINTS 1
#endif
constexpr bool kL2Hints = HGX_GEMM_L2_HINTS != 0;  // L2 cache policies on the operand loads
#ifndef HGX_GEMM_A_FIRST
#define HGX_GEMM_A_FIRST 1
#endif
constexpr bool kAFirst = HGX_GEMM_A_FIRST != 0;
constexpr int kThreads = 192;
constexpr int BM = 128, BN = 256, BK = 64, kStages = 4;
constexpr uint32_t kABytes = BM * BK * 2;  // 16 KB
constexpr uint32_t kBBytes = BN * BK * 2;  // 32 KB
constexpr uint32_t kStageBytes = kABytes + kBBytes;
constexpr uint32_t kBarOffset = kStages * kStageBytes;
enum : uint32_t {
  G_FULL = 0,
  G_EMPTY = G_FULL + kStages,
  G_ACC_FULL = G_EMPTY + kStages,  // + accumulator buffer
  G_ACC_EMPTY = G_ACC_FULL + 2,
  G_DRAIN = G_ACC_EMPTY + 2,
  G_COUNT = G_DRAIN + 1
};
constexpr uint32_t kMiscOffset = kBarOffset + 8 * G_COUNT;  // tmem base, abort flag
constexpr uint32_t kWOffset = kMiscOffset + 16;             // RMSNorm weights (2 x 128 fp32)
constexpr uint32_t kSmemBytes = kWOffset + 2 * 128 * 4 + 1024;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kIdesc = idesc_bf16_f32(BM, BN, false);

enum : uint32_t { GSITE_PRODUCER = 11, GSITE_MMA = 12, GSITE_EPILOGUE = 13, GSITE_DRAIN = 14 };

// Normalise and rotate one 128-feature head row held in registers (QKV epilogue).
__device__ __forceinline__ void norm_rope_row(float (&x)[128], const float* w, const float2* cs,
                                              float eps) {
  float ss0 = 0.f, ss1 = 0.f, ss2 = 0.f, ss3 = 0.f;
#pragma unroll
  for (int e = 0; e < 128; e += 4) {
    ss0 = fmaf(x[e], x[e], ss0);
    ss1 = fmaf(x[e + 1], x[e + 1], ss1);
    ss2 = fmaf(x[e + 2], x[e + 2], ss2);
    ss3 = fmaf(x[e + 3], x[e + 3], ss3);
  }
  const float r = rsqrtf(((ss0 + ss1) + (ss2 + ss3)) * (1.f / 128.f) + eps);
#pragma unroll
  for (int e = 0; e < 128; ++e) x[e] *= r * w[e];
#pragma unroll
  for (int f = 0; f < 64; f += 2) {
    const float4 c2 = *reinterpret_cast<const float4*>(cs + f);  // (cos, sin) of f, f + 1
    const float a0 = x[f], b0 = x[f + 64], a1 = x[f + 1], b1 = x[f + 65];
    x[f] = fmaf(a0, c2.x, -b0 * c2.y);
    x[f + 64] = fmaf(b0, c2.x, a0 * c2.y);
    x[f + 1] = fmaf(a1, c2.z, -b1 * c2.w);
    x[f + 65] = fmaf(b1, c2.z, a1 * c2.w);
  }
}

#ifndef HGX_GEMM_STORE_FIRST
#define HGX_GEMM_STORE_FIRST 1
#endif
// 1: the epilogue's stores carry an L2 evict-first policy (the outputs are read by the next
// kernel, not by this one), so that they do not push the weights out of L2
constexpr bool kStoreFirst = HGX_GEMM_STORE_FIRST != 0;

__device__ __forceinline__ void store_row_bf16(__nv_bfloat16* dst, const float (&x)[128], uint64_t policy) {
  uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
  for (int e = 0; e < 16; ++e) {
    const uint4 v = make_uint4(pack_bf16x2(x[8 * e], x[8 * e + 1]), pack_bf16x2(x[8 * e + 2], x[8 * e + 3]),
                               pack_bf16x2(x[8 * e + 4], x[8 * e + 5]), pack_bf16x2(x[8 * e + 6], x[8 * e + 7]));
    if constexpr (kStoreFirst)
      asm volatile("st.global.L2::cache_hint.v4.b32 [%0], {%1, %2, %3, %4}, %5;" ::"l"(d4 + e), "r"(v.x),
                   "r"(v.y), "r"(v.z), "r"(v.w), "l"(policy)
                   : "memory");
    else
      d4[e] = v;
  }
}

__global__ void __launch_bounds__(kThreads, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ CUtensorMap tmap_b,
                const GemmParams p) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  volatile uint32_t* tmem_holder = reinterpret_cast<volatile uint32_t*>(gbase + kMiscOffset);
  volatile uint32_t* abort_flag = reinterpret_cast<volatile uint32_t*>(gbase + kMiscOffset + 4);
  float* s_w = reinterpret_cast<float*>(gbase + kWOffset);  // [0,128) q weights, [128,256) k
  Ctx c{base + kBarOffset, abort_flag, p.err, p.wait_limit_ns};

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(bar_addr(c, G_FULL + s), 1);
      mbar_init(bar_addr(c, G_EMPTY + s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar_addr(c, G_ACC_FULL + b), 1);
      mbar_init(bar_addr(c, G_ACC_EMPTY + b), 128);
    }
    mbar_init(bar_addr(c, G_DRAIN), 1);
    *abort_flag = 0u;
    fence_mbar_init();
    fence_proxy_async_smem();
  }
  if (p.mode == 1)
    for (int i = threadIdx.x; i < 256; i += kThreads)
      s_w[i] = __bfloat162float(i < 128 ? p.wq[i] : p.wk[i - 128]);
  if (warp == 1) {
    tmem_alloc(smem_u32(const_cast<uint32_t*>(tmem_holder)), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  const int m_tiles = (p.M + BM - 1) / BM;
  const int n_tiles = p.N / BN;
  const int n_tiles_total = m_tiles * n_tiles;
  const int k_blocks = p.K / BK;

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tmap_a);
      tma_prefetch_desc(&tmap_b);
      const uint64_t pol_a = l2_policy_evict_first(), pol_b = l2_policy_evict_last();
      uint32_t pos = 0, loaded = 0, last_par = 0;
      bool ok = true;
      for (int t = blockIdx.x; ok && t < n_tiles_total; t += gridDim.x) {
        const int m0 = (t / n_tiles) * BM, n0 = (t % n_tiles) * BN;
        for (int kb = 0; kb < k_blocks; ++kb) {
          const uint32_t slot = pos % kStages, round = pos / kStages;
          if (!(ok = wait_bounded(c, bar_addr(c, G_EMPTY + slot), (round & 1u) ^ 1u, GSITE_PRODUCER))) break;
          const uint32_t full = bar_addr(c, G_FULL + slot);
          mbar_arrive_expect_tx(full, kStageBytes);
          const uint32_t sa = base + slot * kStageBytes;
          if constexpr (kL2Hints) {
            // the weights (B) are read again by every row block: keep them in L2 (evict
            // last); the activations (A) are read by the column tiles of their row block at
            // about the same time (evict first when HGX_GEMM_A_FIRST, else the default)
            if constexpr (kAFirst)
              tma_load_2d_hint(sa, &tmap_a, full, kb * BK, m0, pol_a);
            else
              tma_load_2d(sa, &tmap_a, full, kb * BK, m0);
            tma_load_2d_hint(sa + kABytes, &tmap_b, full, kb * BK, n0, pol_b);
          } else {
            tma_load_2d(sa, &tmap_a, full, kb * BK, m0);
            tma_load_2d(sa + kABytes, &tmap_b, full, kb * BK, n0);
          }
          loaded |= 1u << slot;
          last_par = (last_par & ~(1u << slot)) | ((round & 1u) << slot);
          ++pos;
        }
      }
      for (int s = 0; s < kStages; ++s)
        if (loaded & (1u << s)) wait_drain(c, bar_addr(c, G_FULL + s), (last_par >> s) & 1u, GSITE_DRAIN);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      uint32_t pos = 0;
      int lt = 0;
      bool ok = true;
      for (int t = blockIdx.x; ok && t < n_tiles_total; t += gridDim.x, ++lt) {
        const int buf = lt & 1;
        if (!(ok = wait_bounded(c, bar_addr(c, G_ACC_EMPTY + buf), ((lt >> 1) & 1) ^ 1, GSITE_MMA))) break;
        tc_fence_after();
        const uint32_t acc = tmem + 256u * buf;
        for (int kb = 0; kb < k_blocks; ++kb) {
          const uint32_t slot = pos % kStages, round = pos / kStages;
          if (!(ok = wait_bounded(c, bar_addr(c, G_FULL + slot), round & 1u, GSITE_MMA))) break;
          tc_fence_after();
          const uint32_t sa = base + slot * kStageBytes, sb = sa + kABytes;
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk)
            mma_ss(acc, smem_desc_sw128(sa + kk * 32, 16, 1024), smem_desc_sw128(sb + kk * 32, 16, 1024),
                   kIdesc, (kb > 0 || kk > 0) ? 1u : 0u);
          mma_commit(bar_addr(c, G_EMPTY + slot));
          ++pos;
        }
        if (!ok) break;
        mma_commit(bar_addr(c, G_ACC_FULL + buf));
      }
      mma_commit(bar_addr(c, G_DRAIN));
      wait_drain(c, bar_addr(c, G_DRAIN), 0, GSITE_DRAIN);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------------ epilogue
    const int quarter = warp & 3;
    const uint64_t store_pol = l2_policy_evict_first();
    const int row = quarter * 32 + lane;
    const uint32_t lane_bits = static_cast<uint32_t>(quarter * 32) << 16;
    int lt = 0;
    for (int t = blockIdx.x; t < n_tiles_total; t += gridDim.x, ++lt) {
      const int buf = lt & 1;
      const bool ok = __all_sync(0xffffffffu, wait_bounded(c, bar_addr(c, G_ACC_FULL + buf), (lt >> 1) & 1,
                                                           GSITE_EPILOGUE));
      if (!ok) break;
      tc_fence_after();
      const int m0 = (t / n_tiles) * BM, n0 = (t % n_tiles) * BN;
      const int token = m0 + row;
      const bool valid = token < p.M;
#pragma unroll 1
      for (int h = 0; h < 2; ++h) {
        uint32_t r[4][32];
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) tmem_ld32(tmem + lane_bits + 256u * buf + 128u * h + 32u * ch, r[ch]);
        tmem_wait_ld();
        float x[128];
#pragma unroll
        for (int ch = 0; ch < 4; ++ch)
#pragma unroll
          for (int e = 0; e < 32; ++e) x[32 * ch + e] = __uint_as_float(r[ch][e]);
        if (!valid) continue;
        const int col = n0 + 128 * h;
        if (p.mode == 0) {
          store_row_bf16(static_cast<__nv_bfloat16*>(p.c) + static_cast<size_t>(token) * p.N + col, x, store_pol);
        } else {
          const int head = col / 128;  // 0..31 q, 32..39 k, 40..47 v
          __nv_bfloat16* dst;
          if (head < 32) {
            norm_rope_row(x, s_w, p.rope_cs + static_cast<size_t>(token) * 64, p.eps);
            dst = static_cast<__nv_bfloat16*>(p.q) + (static_cast<size_t>(token) * 32 + head) * 128;
          } else if (head < 40) {
            norm_rope_row(x, s_w + 128, p.rope_cs + static_cast<size_t>(token) * 64, p.eps);
            dst = static_cast<__nv_bfloat16*>(p.k) + (static_cast<size_t>(token) * 8 + (head - 32)) * 128;
          } else {
            dst = static_cast<__nv_bfloat16*>(p.v) + (static_cast<size_t>(token) * 8 + (head - 40)) * 128;
          }
          store_row_bf16(dst, x, store_pol);
        }
      }
      tc_fence_before();
      mbar_arrive(bar_addr(c, G_ACC_EMPTY + buf));
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// (cos, sin) of every (token, frequency): the angle pos[axis(f)] * inv_freq[f] in fp64.
__global__ void rope_table_kernel(const int32_t* __restrict__ pos, int32_t T, const RopeTables tab,
                                  float2* __restrict__ cs) {
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= static_cast<int64_t>(T) * 64) return;
  const int t = static_cast<int>(i / 64), f = static_cast<int>(i % 64);
  const double phi = static_cast<double>(pos[3 * t + tab.axis[f]]) * tab.inv_freq[f];
  double sd, cd;
  sincos(phi, &sd, &cd);
  cs[i] = make_float2(static_cast<float>(cd), static_cast<float>(sd));
}

}  // namespace

cudaError_t launch_gemm(cudaStream_t stream, const CUtensorMap& tmap_a, const CUtensorMap& tmap_b,
                        const GemmParams& p, int grid) {
  static uint64_t configured = 0;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev >= 64 || !(configured & (1ull << dev))) {
    e = cudaFuncSetAttribute(gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(kSmemBytes));
    if (e != cudaSuccess) return e;
    if (dev < 64) configured |= 1ull << dev;
  }
  gemm_kernel<<<grid, kThreads, kSmemBytes, stream>>>(tmap_a, tmap_b, p);
  return cudaGetLastError();
}

cudaError_t launch_rope_table(cudaStream_t stream, const int32_t* pos, int32_t T,
                              const RopeTables& tab, void* cs) {
  if (T <= 0) return cudaSuccess;
  const int64_t n = static_cast<int64_t>(T) * 64;
  rope_table_kernel<<<static_cast<unsigned>((n + 255) / 256), 256, 0, stream>>>(pos, T, tab,
                                                                                static_cast<float2*>(cs));
  return cudaGetLastError();
}

}  // namespace hgx
