// 2^x evaluated on the FMA pipe, to take part of the softmax's exponentials off the MUFU.
//
// Method (Cody-Waite style range reduction, then a polynomial): x = n + f with
// n = round(x) and f in [-0.5, 0.5]. Adding 1.5 * 2^23 to x rounds it to an integer and
// leaves n in the low mantissa bits of the sum t, so t - 1.5 * 2^23 is n exactly and
// f = x - n is exact. 2^f comes from a degree-3 polynomial whose coefficients are a
// minimax fit (Remez exchange on the relative error) of 2^f on [-0.5, 0.5] made for this
// library; its maximum relative error, float32 evaluation included, is 7.5e-5 -- far below
// the 2^-9 rounding of the bf16 probabilities the result feeds. 2^n is applied by adding n
// to the exponent field (the low bits of t shifted left by 23 are n << 23).
//
// Valid for x <= 8 (the online softmax never exponentiates above 2^8); inputs below -125
// are clamped to -125, giving 2^-125 (about 2.4e-38) instead of a smaller value. Callers
// that need exact zeros for -infinity use the MUFU instruction instead.
#pragma once

#include <cstdint>
#include <cstring>

#ifdef __CUDACC__
#define HGX_HD __host__ __device__ __forceinline__
#else
#define HGX_HD inline
#endif

namespace hgx {

HGX_HD uint32_t f2u(float x) {
#ifdef __CUDA_ARCH__
  return __float_as_uint(x);
#else
  uint32_t u;
  std::memcpy(&u, &x, 4);
  return u;
#endif
}

HGX_HD float u2f(uint32_t u) {
#ifdef __CUDA_ARCH__
  return __uint_as_float(u);
#else
  float x;
  std::memcpy(&x, &u, 4);
  return x;
#endif
}

HGX_HD float exp2_poly3(float x) {
  constexpr float kShift = 12582912.0f;  // 1.5 * 2^23
  x = fmaxf(x, -125.0f);
  const float t = x + kShift;
  const float f = x - (t - kShift);
  float p = fmaf(0.0551716685295105f, f, 0.2426111251115799f);
  p = fmaf(p, f, 0.6932609677314758f);
  p = fmaf(p, f, 0.9999280571937561f);
  return u2f(f2u(p) + (f2u(t) << 23));
}

#ifdef __CUDACC__
// The same evaluation for two arguments at once, with the floating-point steps as paired
// fp32 instructions (sm_100): about 10 instructions per pair instead of 2 MUFU operations.
__device__ __forceinline__ void exp2_poly3_pair(float x0, float x1, float& p0, float& p1) {
  constexpr float kShift = 12582912.0f;  // 1.5 * 2^23
  uint64_t x, t, r, f, p, c;
  asm("mov.b64 %0, {%1, %2};" : "=l"(x) : "f"(fmaxf(x0, -125.0f)), "f"(fmaxf(x1, -125.0f)));
  asm("mov.b64 %0, {%1, %1};" : "=l"(c) : "f"(kShift));
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(t) : "l"(x), "l"(c));
  asm("mov.b64 %0, {%1, %1};" : "=l"(c) : "f"(-kShift));
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(t), "l"(c));  // round(x), exact
  asm("mov.b64 %0, {%1, %1};" : "=l"(c) : "f"(-1.0f));
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(f) : "l"(r), "l"(c), "l"(x));  // x - round(x), exact
  uint64_t c3, c2, c1, c0;
  asm("mov.b64 %0, {%1, %1};" : "=l"(c3) : "f"(0.0551716685295105f));
  asm("mov.b64 %0, {%1, %1};" : "=l"(c2) : "f"(0.2426111251115799f));
  asm("mov.b64 %0, {%1, %1};" : "=l"(c1) : "f"(0.6932609677314758f));
  asm("mov.b64 %0, {%1, %1};" : "=l"(c0) : "f"(0.9999280571937561f));
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(p) : "l"(c3), "l"(f), "l"(c2));
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(p) : "l"(p), "l"(f), "l"(c1));
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(p) : "l"(p), "l"(f), "l"(c0));
  float pl, ph, tl, th;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(pl), "=f"(ph) : "l"(p));
  asm("mov.b64 {%0, %1}, %2;" : "=f"(tl), "=f"(th) : "l"(t));
  p0 = __uint_as_float(__float_as_uint(pl) + (__float_as_uint(tl) << 23));
  p1 = __uint_as_float(__float_as_uint(ph) + (__float_as_uint(th) << 23));
}
#endif

}  // namespace hgx
