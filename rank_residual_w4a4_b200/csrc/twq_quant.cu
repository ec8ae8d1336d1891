// Quantization and packing kernels (TwinQuant §2, Eq. (1), groups of 128 along
// the reduction dimension per §5.1). HBM-bound: 128-bit loads, warp-shuffle
// absmax, a correctly rounded scale per group, and per element the code of the
// correctly rounded quotient, round half to even (twq_eq1.cuh).
#include <cuda_bf16.h>

#include "sm100_ptx.cuh"
#include "twq_eq1.cuh"
#include "twq_internal.h"

namespace twq {
namespace {

__device__ __forceinline__ float bf16_bits_to_f32(uint32_t h) { return __uint_as_float(h << 16); }


// One half-warp per (token, group): lane l of the half covers elements
// [8l, 8l + 8) of the group; a warp covers two consecutive groups of one row (a work
// item) and takes kItems consecutive items, whose loads it issues together so each
// thread keeps 64 bytes in flight on large inputs (one 16-byte load per thread does
// not cover HBM latency); small inputs take one item per warp, for more blocks.
// kQmax: 7 (4-bit codes) or 127 (W4A8's 8-bit codes). kBytes: one int8 code per
// element (element k of a row in byte k); else two's-complement nibbles, two per byte.
template <int kQmax, bool kBytes, int kItems>
__global__ void __launch_bounds__(256) quantize_act_kernel(const uint16_t* __restrict__ x,
                                                           int64_t b, int m, int64_t ldx,
                                                           uint8_t* __restrict__ xq,
                                                           float* __restrict__ sx) {
  // The layer kernel that follows may start its prologue and weight loads now;
  // it reads xq / sx only after this grid has completed.
  pdl_launch_dependents();
  const int G = m / 128;
  const int pairs = (G + 1) / 2;
  const int64_t items = b * pairs;
  const int64_t w0 = ((static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5) * kItems;
  const int lane = threadIdx.x & 31;
  const int l = lane & 15;
  // item w0 + u is pair p of row `row`: one division per warp, then increments
  int64_t row0 = w0 / pairs;
  const int p0 = static_cast<int>(w0 - row0 * pairs);
  int64_t rows[kItems];
  int gs[kItems];
  {
    int64_t rr = row0;
    int p = p0;
#pragma unroll
    for (int u = 0; u < kItems; ++u) {
      rows[u] = rr;
      gs[u] = p * 2 + (lane >> 4);
      if (++p == pairs) {
        p = 0;
        ++rr;
      }
    }
  }
  uint4 raw[kItems];
#pragma unroll
  for (int u = 0; u < kItems; ++u) {
    raw[u] = make_uint4(0, 0, 0, 0);
    if (w0 + u < items && gs[u] < G)
      raw[u] = __ldg(reinterpret_cast<const uint4*>(x + rows[u] * ldx + gs[u] * 128 + l * 8));
  }
#pragma unroll
  for (int u = 0; u < kItems; ++u) {
    if (w0 + u >= items) break;  // the same for the whole warp
    const int64_t row = rows[u];
    const int g = gs[u];
    const bool valid = g < G;
    // BF16 -> fp32: the 16 bits become the high half
    float f[8];
    f[0] = __uint_as_float(__byte_perm(raw[u].x, 0u, 0x1044));
    f[1] = __uint_as_float(raw[u].x & 0xFFFF0000u);
    f[2] = __uint_as_float(__byte_perm(raw[u].y, 0u, 0x1044));
    f[3] = __uint_as_float(raw[u].y & 0xFFFF0000u);
    f[4] = __uint_as_float(__byte_perm(raw[u].z, 0u, 0x1044));
    f[5] = __uint_as_float(raw[u].z & 0xFFFF0000u);
    f[6] = __uint_as_float(__byte_perm(raw[u].w, 0u, 0x1044));
    f[7] = __uint_as_float(raw[u].w & 0xFFFF0000u);
    float a = 0.0f;
#pragma unroll
    for (int k = 0; k < 8; ++k) a = fmaxf(a, fabsf(f[k]));
#pragma unroll
    for (int off = 8; off >= 1; off >>= 1) a = fmaxf(a, __shfl_xor_sync(0xFFFFFFFFu, a, off));
    const Eq1Scale ks = eq1_scale<kQmax>(a);
    const float s = ks.s;
    uint32_t code[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    if (valid) {
      if constexpr (kBytes) {  // element 8l + k in byte k, as a two's-complement int8
        if (s != 0.0f) eq1_codes<kQmax, 8, 0xFFu>(f, ks, code);
        const uint2 v = make_uint2(__byte_perm(__byte_perm(code[0], code[1], 0x0040),
                                               __byte_perm(code[2], code[3], 0x0040), 0x5410),
                                   __byte_perm(__byte_perm(code[4], code[5], 0x0040),
                                               __byte_perm(code[6], code[7], 0x0040), 0x5410));
        *reinterpret_cast<uint2*>(xq + row * m + g * 128 + l * 8) = v;
      } else {  // element 8l + k in nibble k (element 2p in the low nibble of byte p)
        if (s != 0.0f) eq1_codes<kQmax>(f, ks, code);
        uint32_t word = 0;
#pragma unroll
        for (int k = 0; k < 8; ++k) word |= code[k] << (4 * k);
        *reinterpret_cast<uint32_t*>(xq + row * (m / 2) + g * 64 + l * 4) = word;
      }
      if (l == 0) sx[row * G + g] = s;
    }
  }
}

// One thread per (group g, column j) of a row-major m x cols BF16 matrix:
// the group runs down column j (reads are coalesced across j).
__global__ void __launch_bounds__(128) pack_cols_kernel(const uint16_t* __restrict__ w, int m,
                                                        int cols, uint8_t* __restrict__ q,
                                                        float* __restrict__ s) {
  const int j = blockIdx.x * blockDim.x + threadIdx.x;
  const int g = blockIdx.y;
  if (j >= cols) return;
  const uint16_t* p = w + static_cast<int64_t>(g) * 128 * cols + j;
  float a = 0.0f;
  for (int k = 0; k < 128; ++k) a = fmaxf(a, fabsf(bf16_bits_to_f32(__ldg(p + static_cast<int64_t>(k) * cols))));
  const Eq1Scale ks = eq1_scale(a);
  const float sc = ks.s;
  s[static_cast<int64_t>(g) * cols + j] = sc;
  uint4* dst = reinterpret_cast<uint4*>(q + static_cast<int64_t>(j) * (m / 2) + g * 64);
#pragma unroll 1
  for (int c = 0; c < 4; ++c) {
    uint32_t words[4];
#pragma unroll
    for (int wi = 0; wi < 4; ++wi) {
      uint32_t word = 0;
      if (sc != 0.0f) {
        float v[8];
        uint32_t nib[8];
#pragma unroll
        for (int k = 0; k < 8; ++k)
          v[k] = bf16_bits_to_f32(__ldg(p + static_cast<int64_t>(c * 32 + wi * 8 + k) * cols));
        eq1_nibbles(v, ks, nib);
#pragma unroll
        for (int k = 0; k < 8; ++k) word |= nib[k] << (4 * k);
      }
      words[wi] = word;
    }
    dst[c] = make_uint4(words[0], words[1], words[2], words[3]);
  }
}

// out (cols x rows) = in (rows x cols)^T, 16-bit elements, 32 x 32 tiles.
__global__ void transpose16_kernel(const uint16_t* __restrict__ in, int rows, int cols,
                                   uint16_t* __restrict__ out) {
  __shared__ uint16_t tile[32][33];
  const int c0 = blockIdx.x * 32, r0 = blockIdx.y * 32;
  for (int i = threadIdx.y; i < 32; i += blockDim.y) {
    const int r = r0 + i, c = c0 + threadIdx.x;
    if (r < rows && c < cols) tile[i][threadIdx.x] = in[static_cast<int64_t>(r) * cols + c];
  }
  __syncthreads();
  for (int i = threadIdx.y; i < 32; i += blockDim.y) {
    const int c = c0 + i, r = r0 + threadIdx.x;
    if (r < rows && c < cols) out[static_cast<int64_t>(c) * rows + r] = tile[threadIdx.x][i];
  }
}

// y = bf16(a + b), elementwise (the unfused comparator's last step).
__global__ void add_cast_kernel(const float4* __restrict__ a, const float4* __restrict__ b,
                                int64_t n4, uint2* __restrict__ y) {
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n4;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const float4 u = __ldg(a + i), v = __ldg(b + i);
    __nv_bfloat162 lo = __floats2bfloat162_rn(u.x + v.x, u.y + v.y);
    __nv_bfloat162 hi = __floats2bfloat162_rn(u.z + v.z, u.w + v.w);
    y[i] = make_uint2(*reinterpret_cast<uint32_t*>(&lo), *reinterpret_cast<uint32_t*>(&hi));
  }
}

}  // namespace

template <int kItems>
void launch_quantize_items(const uint16_t* x, int64_t b, int m, int64_t ldx, uint8_t* xq, float* sx,
                           cudaStream_t st, bool a8, bool bytes4) {
  const int64_t items = b * ((m / 128 + 1) / 2);
  const int64_t warps = (items + kItems - 1) / kItems;
  const unsigned blocks = static_cast<unsigned>((warps + 7) / 8);
  if (a8)
    quantize_act_kernel<127, true, kItems><<<blocks, 256, 0, st>>>(x, b, m, ldx, xq, sx);
  else if (bytes4)
    quantize_act_kernel<7, true, kItems><<<blocks, 256, 0, st>>>(x, b, m, ldx, xq, sx);
  else
    quantize_act_kernel<7, false, kItems><<<blocks, 256, 0, st>>>(x, b, m, ldx, xq, sx);
}

cudaError_t launch_quantize_act(const uint16_t* x, int64_t b, int64_t m, int64_t ldx, uint8_t* xq,
                                float* sx, cudaStream_t st, bool a8, bool bytes4) {
  // Four items per warp once there are enough of them for about 4 blocks per SM.
  const int64_t items = b * ((m / 128 + 1) / 2);
  if (items >= 148 * 4 * 8 * 4)
    launch_quantize_items<4>(x, b, static_cast<int>(m), ldx, xq, sx, st, a8, bytes4);
  else
    launch_quantize_items<1>(x, b, static_cast<int>(m), ldx, xq, sx, st, a8, bytes4);
  return cudaGetLastError();
}

cudaError_t launch_pack_cols(const uint16_t* w, int64_t m, int64_t cols, uint8_t* q, float* s,
                             cudaStream_t st) {
  dim3 grid(static_cast<unsigned>((cols + 127) / 128), static_cast<unsigned>(m / 128));
  pack_cols_kernel<<<grid, 128, 0, st>>>(w, static_cast<int>(m), static_cast<int>(cols), q, s);
  return cudaGetLastError();
}

cudaError_t launch_transpose_bf16(const uint16_t* in, int64_t rows, int64_t cols, uint16_t* out,
                                  cudaStream_t st) {
  dim3 grid(static_cast<unsigned>((cols + 31) / 32), static_cast<unsigned>((rows + 31) / 32));
  transpose16_kernel<<<grid, dim3(32, 8), 0, st>>>(in, static_cast<int>(rows),
                                                    static_cast<int>(cols), out);
  return cudaGetLastError();
}

cudaError_t launch_add_cast(const float* a, const float* b, int64_t count, uint16_t* y,
                            cudaStream_t st) {
  const int64_t n4 = count / 4;
  int64_t blocks = (n4 + 255) / 256;
  if (blocks > 148 * 16) blocks = 148 * 16;
  if (blocks < 1) blocks = 1;
  add_cast_kernel<<<static_cast<unsigned>(blocks), 256, 0, st>>>(
      reinterpret_cast<const float4*>(a), reinterpret_cast<const float4*>(b), n4,
      reinterpret_cast<uint2*>(y));
  return cudaGetLastError();
}

}  // namespace twq
