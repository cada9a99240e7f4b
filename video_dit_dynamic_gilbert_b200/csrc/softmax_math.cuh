// Softmax arithmetic shared by the tcgen05 kernels (forward attention, estimator).
#pragma once

#include <stdint.h>

#include "common.cuh"

namespace asa {

// exp2 on the FMA pipe: 2^x = 2^n 2^f, n = round(x) (via the 1.5*2^23 rounding
// constant), f in [-1/2, 1/2], 2^f by a degree-3 minimax polynomial (relative error
// 7.5e-5; coefficients from csrc/gen_exp2_poly.py).  x is clamped at -125 so that the
// exponent add stays in the normal range.  Used for a share of the softmax
// exponentials so that MUFU and the FMA pipe split the work.
__device__ __forceinline__ float exp2_fma(float x) {
  x = fmaxf(x, -125.f);
  const float j = x + 12582912.f;
  const float f = x - (j - 12582912.f);
  const float p = fmaf(fmaf(fmaf(5.517166853e-02f, f, 2.426111251e-01f), f, 6.932609677e-01f), f,
                       9.999280572e-01f);
  return __int_as_float(__float_as_int(p) + (__float_as_int(j) << 23));
}

// Blackwell paired fp32 arithmetic: two lanes of work per instruction.
__device__ __forceinline__ uint64_t f2_pack(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void f2_unpack(uint64_t v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
  return r;
}
__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}

// exp2_fma on a pair of lanes, the adds and the polynomial in paired arithmetic
__device__ __forceinline__ void exp2_fma2(uint64_t x2, float& ea, float& eb) {
  float xa, xb;
  f2_unpack(x2, xa, xb);
  xa = fmaxf(xa, -125.f);
  xb = fmaxf(xb, -125.f);
  const uint64_t x = f2_pack(xa, xb);
  const uint64_t magic = f2_pack(12582912.f, 12582912.f);
  const uint64_t nmagic = f2_pack(-12582912.f, -12582912.f);
  const uint64_t j = f2_add(x, magic);
  const uint64_t n = f2_add(j, nmagic);
  float na, nb;
  f2_unpack(n, na, nb);
  const uint64_t f = f2_add(x, f2_pack(-na, -nb));
  uint64_t p = f2_fma(f2_pack(5.517166853e-02f, 5.517166853e-02f), f,
                      f2_pack(2.426111251e-01f, 2.426111251e-01f));
  p = f2_fma(p, f, f2_pack(6.932609677e-01f, 6.932609677e-01f));
  p = f2_fma(p, f, f2_pack(9.999280572e-01f, 9.999280572e-01f));
  float pa, pb, ja, jb;
  f2_unpack(p, pa, pb);
  f2_unpack(j, ja, jb);
  ea = __int_as_float(__float_as_int(pa) + (__float_as_int(ja) << 23));
  eb = __int_as_float(__float_as_int(pb) + (__float_as_int(jb) << 23));
}

__device__ __forceinline__ float max3f(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

}  // namespace asa
