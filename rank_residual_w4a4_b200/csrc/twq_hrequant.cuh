// The on-chip requantization of H for the INT4 stage 2 (TwinQuant §4.3, item 2: "s_H
// estimated from the accumulator", then Q_H · Q(V)): Eq. (1) with q_max = 7 on one
// token's 128 BF16 values of H, per group of 128 along r. Shared by the prefill kernels.
#pragma once

#include <cstdint>

#include "sm100_ptx.cuh"
#include "twq_eq1.cuh"

namespace twq {

// Offset of logical 16-byte chunk c of row `row` in a 128-byte-swizzled tile.
__device__ __forceinline__ uint32_t hq_sw128(int row, int c) {
  return static_cast<uint32_t>((row >> 3) * 1024 + (row & 7) * 128 + ((c ^ (row & 7)) << 4));
}

// Eq. (1) (q_max = 7) on one row of a group of 128 BF16 columns of H in the stage-2
// operand layout (two 16 KB chunks of 64 columns, 128-byte swizzle, starting at `grp`),
// written back as 16*q int8 codes in the 4-bit operand order over the first chunk.
// Piece p (columns [8p, 8p + 8)) sits at location p; output chunk c (columns
// [16c, 16c + 16)) reads pieces 2c and 2c + 1 and is written at location c, which
// holds piece c, already read by output chunk c / 2 <= c: in place, in one stream.
__device__ __forceinline__ const uint4* h_piece(const uint8_t* grp, int row, int p) {
  return reinterpret_cast<const uint4*>(grp + (p >> 3) * 16384 + hq_sw128(row, p & 7));
}

// push: also store the codes and the scale into CTA `peer` of the cluster (the same
// addresses there), completing bytes on its barrier `peer_bar` (a CTA pair).
static __device__ __noinline__ void requant_h_row(uint8_t* grp, int row, float* s_out, bool push,
                                                  uint32_t peer, uint32_t peer_bar) {
  float a = 0.0f;
#pragma unroll 4
  for (int p = 0; p < 16; ++p) {
    const uint4 w = *h_piece(grp, row, p);
    const uint32_t v[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int i = 0; i < 4; ++i)
      a = fmaxf(a, fmaxf(fabsf(__uint_as_float(v[i] << 16)),
                         fabsf(__uint_as_float(v[i] & 0xFFFF0000u))));
  }
  const Eq1Scale ks = eq1_scale<7>(a);
  *s_out = ks.s;
  if (push) st_async_peer_u32(map_peer(smem_u32(s_out), peer), __float_as_uint(ks.s), peer_bar);
#pragma unroll 1
  for (int c = 0; c < 8; ++c) {
    uint4 o = make_uint4(0, 0, 0, 0);
    if (ks.s != 0.0f) {
      const uint4 w0 = *h_piece(grp, row, 2 * c), w1 = *h_piece(grp, row, 2 * c + 1);
      const uint32_t u[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
      float f[16];  // f[0..7]: even columns 0, 2, .., 14 of the chunk; f[8..15]: odd
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        f[i] = __uint_as_float(u[i] << 16);
        f[8 + i] = __uint_as_float(u[i] & 0xFFFF0000u);
      }
      uint32_t nb[16];
      eq1_nibbles(f, ks, nb);
      o = pack_codes16(nb);
    }
    *reinterpret_cast<uint4*>(grp + hq_sw128(row, c)) = o;
    if (push) st_async_peer_v4u(map_peer(smem_u32(grp + hq_sw128(row, c)), peer), o, peer_bar);
  }
}

}  // namespace twq
