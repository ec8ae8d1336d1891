// The symmetric 4-bit quantizer of TwinQuant §2, Eq. (1), with q_max = 7: code
// c = clamp(rint(v / s), -7, 7), where v / s is the correctly rounded fp32
// quotient and rint rounds half to even. Shared by the activation quantizer
// kernel and the decode kernel's in-kernel quantizer.
//
// A correctly rounded division per element is the slow part of the quantizer.
// The code only depends on which side of the nearest half-integer the quotient
// falls, so it is computed from the product q = v * rcp(s) instead:
//   rcp(s) = 1/s (1 + d1), q = (v / s)(1 + d1)(1 + d2), |d1|, |d2| <= 2^-24,
// and |v / s| <= 7 (1 + 2^-24) because s = fl(max|v| / 7). So q and the
// correctly rounded quotient both lie within 1.3e-6 of the exact v / s, and
// they round to the same integer unless a half-integer lies within 1.3e-6 of
// q. Where any of 8 elements has |q - rint(q)| >= 0.5 - 2^-16, the 8 take the
// exact division instead, as do groups whose scale (or its reciprocal) is not
// a normal number, where the bound above does not hold. The result is
// bit-identical to the plain definition.
#pragma once

#include <cstdint>

namespace twq {

struct Eq1Scale {
  float s;    // the group's scale max|v| / 7, correctly rounded
  float rs;   // its correctly rounded reciprocal (used only when fast)
  bool fast;  // s and 1/s are normal numbers: the product form is valid
};

__device__ __forceinline__ Eq1Scale eq1_scale(float absmax) {
  Eq1Scale k;
  k.s = __fdiv_rn(absmax, 7.0f);
  k.fast = k.s >= 0x1p-125f && k.s <= 0x1p125f;
  k.rs = k.fast ? __frcp_rn(k.s) : 0.0f;
  return k;
}

// Codes of 8 values of one group as integer-valued floats in [-7, 7]; needs
// k.s > 0. In the product form |q| <= 7 (1 + 4 * 2^-24), so rint(q) needs no
// clamp; the exact form clamps (it matters only for subnormal scales).
__device__ __forceinline__ void eq1_codes8(const float (&v)[8], const Eq1Scale& k, float (&t)[8]) {
  bool exact = !k.fast;
  if (k.fast) {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float q = __fmul_rn(v[i], k.rs);
      t[i] = rintf(q);
      exact |= fabsf(__fsub_rn(q, t[i])) >= 0.5f - 0x1p-16f;
    }
  }
  if (exact) {
#pragma unroll
    for (int i = 0; i < 8; ++i) t[i] = fminf(fmaxf(rintf(__fdiv_rn(v[i], k.s)), -7.0f), 7.0f);
  }
}

// Two's-complement nibble of an integer-valued float t in [-7, 7]: adding
// 1.5 * 2^23 puts t in the low mantissa bits.
__device__ __forceinline__ uint32_t eq1_nibble(float t) {
  return __float_as_uint(__fadd_rn(t, 12582912.0f)) & 0xFu;
}

}  // namespace twq
