// exp2.cuh - the base-2 exponentials of the softmax kernels: the SFU's ex2.approx and an
// FMA-pipe polynomial that takes part of the load off the SFU.  Shared by the attention kernels
// and by the self-test kernels that check the polynomial against its error bound.
#pragma once

#include <stdint.h>

#include "sm100.cuh"

namespace mla {

// 2^x on the SFU (ex2.approx, flush-to-zero).
__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// max(a, b, c) in one instruction (sm_100 three-input FMNMX).
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float y;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(y) : "f"(a), "f"(b), "f"(c));
  return y;
}

// 2^x on the FMA pipe, for a pair of arguments in packed form, so that part of the softmax's
// exponentials bypass the SFU (which otherwise sets the softmax's pace).  x = n + f with
// n = rint(x) and f in [-1/2, 1/2]; 2^f by the degree-3 polynomial interpolating 2^f at the four
// Chebyshev nodes of [-1/2, 1/2] (relative error below 1.0e-4, far under a bf16 half-ulp of P);
// 2^n is added to the exponent field.  Arguments are clamped to >= -125 (2^-125 is zero for
// the softmax's purposes and keeps the exponent field of the result positive); the softmax
// never passes more than +8 (the lazy-rescale bound).
constexpr float kExp2C0 = 0.9999245405197144f;
constexpr float kExp2C1 = 0.6931367516517639f;
constexpr float kExp2C2 = 0.2426394820213318f;
constexpr float kExp2C3 = 0.05583828315138817f;
constexpr float kRoundMagic = 12582912.0f;   // 1.5 * 2^23: x + this rounds x to an integer

__device__ __forceinline__ void exp2_poly_pair(float x0, float x1, float& y0, float& y1) {
  using namespace sm100;
  const uint64_t x = f2_pack(fmaxf(x0, -125.f), fmaxf(x1, -125.f));
  const uint64_t magic = f2_pack(kRoundMagic, kRoundMagic);
  const uint64_t t = f2_add(x, magic);                              // magic + n, exactly
  const uint64_t neg_n = f2_fma(t, f2_pack(-1.f, -1.f), magic);     // -n
  const uint64_t f = f2_add(x, neg_n);                              // x - n
  uint64_t q = f2_fma(f, f2_pack(kExp2C3, kExp2C3), f2_pack(kExp2C2, kExp2C2));
  q = f2_fma(q, f, f2_pack(kExp2C1, kExp2C1));
  q = f2_fma(q, f, f2_pack(kExp2C0, kExp2C0));
  float q0, q1, t0, t1;
  f2_unpack(q, q0, q1);
  f2_unpack(t, t0, t1);
  // the low bits of t hold n (bits(t) = bits(magic) + n); shifted into the exponent field the
  // bits of magic drop out, leaving n << 23
  y0 = __uint_as_float(__float_as_uint(q0) + (__float_as_uint(t0) << 23));
  y1 = __uint_as_float(__float_as_uint(q1) + (__float_as_uint(t1) << 23));
}

}  // namespace mla
