// Internal interface between the C-ABI layer (twq_api.cu) and the kernels.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/twq.h"

namespace twq {

// What one launch of the tensor-core kernel computes.
enum GemmMode : int {
  kModeFused = 0,    // Y = bf16(Q(X)Q(R) + bf16(Q(X)Q(L1)) L2)
  kModeW4A4 = 1,     // Y = bf16(Q(X)Q(R))
  kModeLowRank = 2,  // Y = bf16(bf16(Q(X)Q(L1)) L2)
  kModeResF32 = 3,   // out = Q(X)Q(R) in fp32            (unfused comparator, step 1)
  kModeHOnly = 4,    // out = bf16(Q(X)Q(L1)), b x r      (unfused comparator, step 2)
  kModeS2F32 = 5,    // out = H L2 in fp32, H read from HBM (unfused comparator, step 3)
  kModeFusedS2Q = 6, // Y = bf16(Q(X)Q(R) + Q(bf16(Q(X)Q(L1))) Q(L2)): the INT4 stage 2
};

struct GemmCall {
  int mode;
  const uint8_t* xq;
  const float* sx;
  int64_t b;
  const twq_weights* w;
  void* out;                // bf16 Y, fp32 b x n, or bf16 H (b x r)
  const uint16_t* h_global; // kModeS2F32 only: bf16 H, b x r
  const uint16_t* x = nullptr;  // decode kernel only: BF16 X, quantized in the kernel
  int64_t ldx = 0;
  bool a8 = false;  // xq holds one int8 code per element, b x m (W4A8's 8-bit codes, or
                    // 4-bit codes stored in bytes)
  const uint8_t* l2q = nullptr;  // kModeFusedS2Q: L2 as 4-bit codes, n x r/2 (K-major)
  const float* sl2q = nullptr;   // kModeFusedS2Q: their scales, (r/128) x n
};

// Host-side launchers; all return cudaSuccess or the launch error.
cudaError_t launch_gemm(const GemmCall& call, cudaStream_t stream, int* launches);
// a8: int8 codes with q_max = 127 (b x m bytes); bytes4: 4-bit codes (q_max = 7) one
// per byte (b x m bytes); else packed nibbles (b x m/2 bytes).
cudaError_t launch_quantize_act(const uint16_t* x, int64_t b, int64_t m, int64_t ldx, uint8_t* xq,
                                float* sx, cudaStream_t stream, bool a8 = false,
                                bool bytes4 = false);
cudaError_t launch_pack_cols(const uint16_t* w, int64_t m, int64_t cols, uint8_t* q, float* s,
                             cudaStream_t stream);
cudaError_t launch_transpose_bf16(const uint16_t* in, int64_t rows, int64_t cols, uint16_t* out,
                                  cudaStream_t stream);
cudaError_t launch_add_cast(const float* a, const float* b, int64_t count, uint16_t* y,
                            cudaStream_t stream);

// Prefill kernel on CTA pairs (256 x 256 tiles, tcgen05 cta_group::2): the fused,
// W4A4-only and low-rank-only layers with 4-bit X codes, n % 256 == 0, m >= 256,
// b > 16.
bool pair_eligible(const GemmCall& call);
cudaError_t launch_pair(const GemmCall& call, cudaStream_t stream);
// Self-test of the bounded waits: the kernel with its X copies withheld and the
// given wait limit, so that every wait on X runs out and the kernel leaves through
// its abort path (status site codes 41-52 in the pair status word).
cudaError_t launch_pair_stall_selftest(const GemmCall& call, cudaStream_t stream,
                                       unsigned long long wait_ns);
cudaError_t read_and_clear_pair_status(int* code);

// Decode-shape kernel (b <= 16, split K over a 4- or 8-CTA cluster).
bool decode_eligible(const GemmCall& call);
cudaError_t launch_decode(const GemmCall& call, cudaStream_t stream);

// twq_release_cache: drop the decode path's cached tensor maps, and the
// allocation-free entry point's resolved scratch addresses.
void release_decode_cache();
void release_noalloc_cache();

// Device status words (first wait site that gave up), one per kernel family.
cudaError_t read_and_clear_device_status(int* code);
cudaError_t read_and_clear_decode_status(int* code);

}  // namespace twq
