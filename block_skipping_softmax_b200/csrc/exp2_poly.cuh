// 2^x on the FMA pipes, for probabilities that are rounded to bf16 anyway.
//
// The exponential unit (MUFU, 16 results per clock per SM on B200) sets the
// pace of the softmax at d = 128: per 128 x 128 tile it needs as many cycles
// as the two MMAs.  Computing part of the exponentials with ordinary FMAs
// moves that work to pipes that are otherwise idle.  TurboAttention
// ("TurboAttention: Efficient Attention Approximation for High-Throughput LLM
// Serving", Technical Deep Dive: SAS) splits an exponential into an integer
// part and a polynomial for the fraction; this is the same idea, written for
// base 2 and bf16 outputs:
//
//   x  = max(x, -126)                 (so every result is a normal or zero-exponent bf16)
//   j  = rint(x)                      (adding 1.5 * 2^23 rounds to an integer)
//   f  = x - j                        (exact, f in [-1/2, 1/2])
//   p  = c0 + f (c1 + f (c2 + f c3))  (minimax fit of 2^f, relative error 7.5e-5)
//   2^x ~ p * 2^j                     (the j is added to the exponent field of bf16(p))
//
// The coefficients are a Remez (minimax, relative error) fit of degree 3 on
// [-1/2, 1/2], rounded to fp32; the fit's error is 25 times smaller than half
// a bf16 ulp, so the bf16 result is off by at most one ulp (and is the
// correctly rounded value in about 96 % of cases).  Scaling by 2^j commutes
// with the rounding to bf16, so the exponent is added to the packed bf16
// word: bf16(p0) + 128 j0 in the low half, bf16(p1) + 128 j1 in the high half.
#pragma once
#include <cuda_bf16.h>

#include <cstdint>

#include "ptx.cuh"

namespace bss {

constexpr float kExp2C0 = 0.9999280571937561f;
constexpr float kExp2C1 = 0.6932609677314758f;
constexpr float kExp2C2 = 0.2426111251115799f;
constexpr float kExp2C3 = 0.0551716685295105f;
constexpr float kExp2Round = 12582912.0f;  // 1.5 * 2^23
constexpr float kExp2Lo = -126.0f;

// bf16x2 word (low half = 2^x.x, high half = 2^x.y)
__device__ __forceinline__ uint32_t exp2_poly_bf16x2(float2 x) {
  x.x = fmaxf(x.x, kExp2Lo);
  x.y = fmaxf(x.y, kExp2Lo);
  const float2 t = __fadd2_rn(x, make_float2(kExp2Round, kExp2Round));
  const float2 j = __fadd2_rn(t, make_float2(-kExp2Round, -kExp2Round));
  const float2 f = __ffma2_rn(j, make_float2(-1.f, -1.f), x);
  float2 p = __ffma2_rn(f, make_float2(kExp2C3, kExp2C3), make_float2(kExp2C2, kExp2C2));
  p = __ffma2_rn(f, p, make_float2(kExp2C1, kExp2C1));
  p = __ffma2_rn(f, p, make_float2(kExp2C0, kExp2C0));
  const uint32_t w = pack_bf16x2(p.x, p.y);
  // the low 23 bits of t hold j + 2^22; (bits << 7) and (bits << 23) carry
  // 128 j and 2^23 j plus constants that sum to 0xA0000000 modulo 2^32
  const uint32_t tx = __float_as_uint(t.x), ty = __float_as_uint(t.y);
  return w + (tx << 7) + (ty << 23) + 0x60000000u;
}

}  // namespace bss
