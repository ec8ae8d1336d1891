// The symmetric 4-bit quantizer of TwinQuant §2, Eq. (1), with q_max = 7: code
// c = clamp(rint(v / s), -7, 7), where s = max|v| / 7 and v / s are correctly
// rounded fp32 values and rint rounds half to even. Shared by the activation
// quantizer, the weight packer and the decode kernel's in-kernel quantizer.
//
// A correctly rounded division per element would be the slow part. Both
// divisions are computed instead with Markstein's correction step, which
// yields the correctly rounded quotient from a correctly rounded reciprocal
// (P. Markstein, "Computation of elementary functions on the IBM RISC
// System/6000 processor", IBM J. Res. Dev. 34(1), 1990; see also Brisebarre,
// Muller and Raina, IEEE Trans. Computers 53(8), 2004, for a divisor known in
// advance):
//   y = RN(1/b), q0 = RN(a y), r = RN(a - b q0) (one fma), q = RN(q0 + r y).
// * Scale: b = 7, y = RN(1/7) a constant. For every non-negative finite BF16
//   value a (the quantizers only see BF16 inputs) q = RN(a / 7); checked
//   exhaustively in exact rational arithmetic.
// * Codes: b = s, y = RN(1/s) once per group. For every BF16 v with |v| <= a
//   and every BF16 a, q = RN(v / s); checked exhaustively over all significand
//   pairs and exponent offsets in exact rational arithmetic, which covers every
//   scale in [2^-100, 2^100] by scaling (no intermediate leaves the normal
//   range there). Groups with a scale outside that range (subnormal or huge
//   inputs) use the plain correctly rounded division.
// Then rint(q) = RN(q + 1.5 * 2^23) - 1.5 * 2^23 exactly (|q| < 2^22, ties to
// even), whose low four bits are the two's-complement nibble; |q| <= 7 (1 +
// 2^-23), so rint(q) needs no clamp. Tests run every BF16 absmax and rounding
// ties through the kernels against the plain definition.
#pragma once

#include <cstdint>

namespace twq {

struct Eq1Scale {
  float s;    // the group's scale RN(max|v| / 7)
  float rs;   // RN(1/s) (used only when fast)
  bool fast;  // 2^-100 <= s <= 2^100: the correction step is exact
};

// a: the group's absmax, a non-negative BF16 value.
__device__ __forceinline__ Eq1Scale eq1_scale(float a) {
  constexpr float kRcp7 = 0x1.24924ap-3f;  // RN(1/7)
  const float q0 = __fmul_rn(a, kRcp7);
  Eq1Scale k;
  k.s = __fmaf_rn(__fmaf_rn(-q0, 7.0f, a), kRcp7, q0);
  k.fast = k.s >= 0x1p-100f && k.s <= 0x1p100f;
  k.rs = k.fast ? __frcp_rn(k.s) : 0.0f;
  return k;
}

// The plain definition: clamp(rint(RN(v / s)), -7, 7).
static __device__ __noinline__ float eq1_code_exact(float v, float s) {
  return fminf(fmaxf(rintf(__fdiv_rn(v, s)), -7.0f), 7.0f);
}

// Two's-complement nibble of an integer-valued float t in [-7, 7]: adding
// 1.5 * 2^23 puts t in the low mantissa bits.
__device__ __forceinline__ uint32_t eq1_nibble(float t) {
  return __float_as_uint(__fadd_rn(t, 12582912.0f)) & 0xFu;
}

// Nibbles of N values of one group (needs k.s > 0); branch-free for fast scales.
template <int N>
__device__ __forceinline__ void eq1_nibbles(const float (&v)[N], const Eq1Scale& k,
                                            uint32_t (&nib)[N]) {
  if (k.fast) {
#pragma unroll
    for (int i = 0; i < N; ++i) {
      const float q0 = __fmul_rn(v[i], k.rs);
      const float q = __fmaf_rn(__fmaf_rn(-q0, k.s, v[i]), k.rs, q0);  // RN(v / s)
      nib[i] = __float_as_uint(__fadd_rn(q, 12582912.0f)) & 0xFu;
    }
  } else {
#pragma unroll
    for (int i = 0; i < N; ++i) nib[i] = eq1_nibble(eq1_code_exact(v[i], k.s));
  }
}

}  // namespace twq
