// The symmetric quantizer of TwinQuant §2, Eq. (1): code c = clamp(rint(v / s),
// -q_max, q_max), where s = max|v| / q_max and v / s are correctly rounded fp32
// values and rint rounds half to even. q_max = 7 for the 4-bit codes (weights and
// W4A4 activations), 127 for the 8-bit activations of the W4A8 setting (§5.1).
// Shared by the activation quantizers, the weight packer and the decode kernel's
// in-kernel quantizer.
//
// A correctly rounded division per element would be the slow part. Both
// divisions are computed instead with Markstein's correction step, which
// yields the correctly rounded quotient from a correctly rounded reciprocal
// (P. Markstein, "Computation of elementary functions on the IBM RISC
// System/6000 processor", IBM J. Res. Dev. 34(1), 1990; see also Brisebarre,
// Muller and Raina, IEEE Trans. Computers 53(8), 2004, for a divisor known in
// advance):
//   y = RN(1/b), q0 = RN(a y), r = RN(a - b q0) (one fma), q = RN(q0 + r y).
// * Scale: b = q_max, y = RN(1/q_max) a constant. For every non-negative finite
//   BF16 value a (the quantizers only see BF16 inputs) q = RN(a / q_max); checked
//   exhaustively in exact rational arithmetic for q_max = 7 and 127.
// * Codes: b = s, y = RN(1/s) once per group. For every BF16 v with |v| <= a
//   and every BF16 a, q = RN(v / s); checked exhaustively over all significand
//   pairs and exponent offsets in exact rational arithmetic, which covers every
//   scale in [2^-100, 2^100] by scaling (no intermediate leaves the normal
//   range there). Groups with a scale outside that range (subnormal or huge
//   inputs) use the plain correctly rounded division.
// Then rint(q) = RN(q + 1.5 * 2^23) - 1.5 * 2^23 exactly (|q| < 2^22, ties to
// even), whose low four (eight) bits are the two's-complement code; the absmax
// rounds to exactly q_max, so rint(q) needs no clamp. Tests run every BF16 absmax
// and rounding ties through the kernels against the plain definition.
#pragma once

#include <cstdint>

namespace twq {

template <int QMAX>
struct Eq1Rcp;
template <>
struct Eq1Rcp<7> {
  static constexpr float v = 0x1.24924ap-3f;  // RN(1/7)
};
template <>
struct Eq1Rcp<127> {
  static constexpr float v = 0x1.020408p-7f;  // RN(1/127)
};

struct Eq1Scale {
  float s;    // the group's scale RN(max|v| / q_max)
  float rs;   // RN(1/s) (used only when fast)
  bool fast;  // 2^-100 <= s <= 2^100: the correction step is exact
};

// a: the group's absmax, a non-negative BF16 value.
template <int QMAX = 7>
__device__ __forceinline__ Eq1Scale eq1_scale(float a) {
  constexpr float kRcp = Eq1Rcp<QMAX>::v;
  const float q0 = __fmul_rn(a, kRcp);
  Eq1Scale k;
  k.s = __fmaf_rn(__fmaf_rn(-q0, static_cast<float>(QMAX), a), kRcp, q0);
  k.fast = k.s >= 0x1p-100f && k.s <= 0x1p100f;
  k.rs = k.fast ? __frcp_rn(k.s) : 0.0f;
  return k;
}

// The plain definition: clamp(rint(RN(v / s)), -q_max, q_max).
template <int QMAX = 7>
static __device__ __noinline__ float eq1_code_exact(float v, float s) {
  return fminf(fmaxf(rintf(__fdiv_rn(v, s)), -static_cast<float>(QMAX)), static_cast<float>(QMAX));
}

// Two's-complement code bits of an integer-valued float t in [-q_max, q_max]:
// adding 1.5 * 2^23 puts t in the low mantissa bits.
template <uint32_t MASK>
__device__ __forceinline__ uint32_t eq1_bits(float t) {
  return __float_as_uint(__fadd_rn(t, 12582912.0f)) & MASK;
}
__device__ __forceinline__ uint32_t eq1_nibble(float t) { return eq1_bits<0xFu>(t); }

// Codes of N values of one group (needs k.s > 0), as two's-complement nibbles
// (q_max = 7) or bytes (q_max = 127, or kMask = 0xFF: the 4-bit codes sign-extended
// to int8, which the same low bits give); branch-free for fast scales.
template <int QMAX, int N, uint32_t kMask = (QMAX == 7 ? 0xFu : 0xFFu)>
__device__ __forceinline__ void eq1_codes(const float (&v)[N], const Eq1Scale& k,
                                          uint32_t (&code)[N]) {
  if (k.fast) {
#pragma unroll
    for (int i = 0; i < N; ++i) {
      const float q0 = __fmul_rn(v[i], k.rs);
      const float q = __fmaf_rn(__fmaf_rn(-q0, k.s, v[i]), k.rs, q0);  // RN(v / s)
      code[i] = eq1_bits<kMask>(q);
    }
  } else {
#pragma unroll
    for (int i = 0; i < N; ++i) code[i] = eq1_bits<kMask>(eq1_code_exact<QMAX>(v[i], k.s));
  }
}

// Sixteen 4-bit codes of one 16-element chunk (nb[0..7]: even elements 0, 2, .., 14;
// nb[8..15]: odd elements) as int8 bytes 16*q in the MMA operand order the 4-bit
// unpack produces: even elements 0..6, odd 1..7, even 8..14, odd 9..15.
__device__ __forceinline__ uint4 pack_codes16(const uint32_t (&nb)[16]) {
  uint4 o;
  o.x = (nb[0] << 4) | (nb[1] << 12) | (nb[2] << 20) | (nb[3] << 28);
  o.y = (nb[8] << 4) | (nb[9] << 12) | (nb[10] << 20) | (nb[11] << 28);
  o.z = (nb[4] << 4) | (nb[5] << 12) | (nb[6] << 20) | (nb[7] << 28);
  o.w = (nb[12] << 4) | (nb[13] << 12) | (nb[14] << 20) | (nb[15] << 28);
  return o;
}

template <int N>
__device__ __forceinline__ void eq1_nibbles(const float (&v)[N], const Eq1Scale& k,
                                            uint32_t (&nib)[N]) {
  eq1_codes<7, N>(v, k, nib);
}

}  // namespace twq
