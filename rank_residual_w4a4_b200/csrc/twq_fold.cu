// Offline fold of the learned transforms into the layer's factors (TwinQuant
// §4.1, "Theory-Guided Re-parameterization over Dual Decomposed Subspaces",
// Eq. (6) and the factors after it): U' = Q^-1 U G, V' = G^-1 V, R' = Q^-1 R.
// Q is orthogonal (§4.2: Q is kept on the Stiefel manifold, Q^T Q = I), so
// Q^-1 = Q^T; G is invertible and is inverted here (Gauss-Jordan elimination
// with partial pivoting in fp64). The products accumulate in fp32 and the
// outputs are BF16 (round to nearest even), ready for twq_pack_weights.
// Offline work: plain CUDA-core kernels, no tensor cores.
#include <cuda_bf16.h>

#include "twq_internal.h"

namespace twq {
namespace {

constexpr int kInvThreads = 256;

// [G | I] -> [I | G^-1] in place in `aug` (r x 2r doubles, row-major), one CTA.
// *singular = 1 if a pivot column has no nonzero (finite) entry.
__global__ void __launch_bounds__(kInvThreads) gj_invert_kernel(const float* __restrict__ g, int r,
                                                                double* __restrict__ aug,
                                                                float* __restrict__ ginv,
                                                                int* __restrict__ singular) {
  __shared__ double s_val[kInvThreads];
  __shared__ int s_idx[kInvThreads];
  __shared__ double s_fac[1024];  // column k of every row before the update (r <= 1024)
  const int tid = threadIdx.x;
  const int w = 2 * r;
  for (int e = tid; e < r * w; e += kInvThreads) {
    const int i = e / w, j = e % w;
    aug[e] = j < r ? static_cast<double>(g[i * r + j]) : (j - r == i ? 1.0 : 0.0);
  }
  if (tid == 0) *singular = 0;
  __syncthreads();
  for (int k = 0; k < r; ++k) {
    // pivot: the row i >= k with the largest |aug[i][k]| (lowest index on ties)
    double best = -1.0;
    int bi = k;
    for (int i = k + tid; i < r; i += kInvThreads) {
      const double v = fabs(aug[i * w + k]);
      if (v > best) {
        best = v;
        bi = i;
      }
    }
    s_val[tid] = best;
    s_idx[tid] = bi;
    __syncthreads();
    for (int off = kInvThreads / 2; off > 0; off >>= 1) {
      if (tid < off) {
        const double a = s_val[tid], b = s_val[tid + off];
        if (b > a || (b == a && s_idx[tid + off] < s_idx[tid])) {
          s_val[tid] = b;
          s_idx[tid] = s_idx[tid + off];
        }
      }
      __syncthreads();
    }
    const int p = s_idx[0];
    const double pv = s_val[0];
    __syncthreads();
    if (!(pv > 0.0) || !isfinite(pv)) {
      if (tid == 0) *singular = 1;
      return;  // uniform: every thread read the same pivot value
    }
    if (p != k)
      for (int j = tid; j < w; j += kInvThreads) {
        const double t = aug[k * w + j];
        aug[k * w + j] = aug[p * w + j];
        aug[p * w + j] = t;
      }
    __syncthreads();
    const double inv = 1.0 / aug[k * w + k];
    for (int j = tid; j < w; j += kInvThreads) aug[k * w + j] *= inv;
    __syncthreads();
    for (int i = tid; i < r; i += kInvThreads) s_fac[i] = aug[i * w + k];
    __syncthreads();
    for (int e = tid; e < r * w; e += kInvThreads) {
      const int i = e / w, j = e % w;
      if (i != k) aug[e] -= s_fac[i] * aug[k * w + j];
    }
    __syncthreads();
  }
  for (int e = tid; e < r * r; e += kInvThreads) {
    const int i = e / r, j = e % r;
    ginv[e] = static_cast<float>(aug[i * w + r + j]);
  }
}

__device__ __forceinline__ float load_f(const float* p, int64_t i) { return p[i]; }
__device__ __forceinline__ float load_f(const uint16_t* p, int64_t i) {
  return __uint_as_float(static_cast<uint32_t>(p[i]) << 16);
}
__device__ __forceinline__ void store_out(float* p, int64_t i, float v) { p[i] = v; }
__device__ __forceinline__ void store_out(uint16_t* p, int64_t i, float v) {
  p[i] = __bfloat16_as_ushort(__float2bfloat16_rn(v));
}

constexpr int kFT = 64;   // output tile
constexpr int kFK = 16;   // K step
constexpr int kFThreads = 256;

// C (M x N, row-major) = op(A) (M x K) * B (K x N, row-major), fp32 accumulation.
// op(A) = A (M x K row-major), or A^T when kTransA (A stored K x M row-major).
template <typename TA, typename TB, typename TC, bool kTransA>
__global__ void __launch_bounds__(kFThreads) fold_gemm_kernel(const TA* __restrict__ a,
                                                              const TB* __restrict__ b,
                                                              TC* __restrict__ c, int M, int N,
                                                              int K) {
  __shared__ float as[kFK][kFT + 1];
  __shared__ float bs[kFK][kFT];
  const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
  const int m0 = blockIdx.y * kFT, n0 = blockIdx.x * kFT;
  float acc[4][4] = {};
  for (int k0 = 0; k0 < K; k0 += kFK) {
    for (int e = threadIdx.x; e < kFK * kFT; e += kFThreads) {
      const int kk = e / kFT, mm = e % kFT;  // as[kk][mm] = op(A)[m0 + mm][k0 + kk]
      const int gm = m0 + mm, gk = k0 + kk;
      float v = 0.0f;
      if (gm < M && gk < K)
        v = kTransA ? load_f(a, static_cast<int64_t>(gk) * M + gm)
                    : load_f(a, static_cast<int64_t>(gm) * K + gk);
      as[kk][mm] = v;
      const int gn = n0 + mm;
      bs[kk][mm] = (gk < K && gn < N) ? load_f(b, static_cast<int64_t>(gk) * N + gn) : 0.0f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < kFK; ++kk) {
      float av[4], bv[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) av[i] = as[kk][ty + 16 * i];
#pragma unroll
      for (int j = 0; j < 4; ++j) bv[j] = bs[kk][tx + 16 * j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int gm = m0 + ty + 16 * i, gn = n0 + tx + 16 * j;
      if (gm < M && gn < N) store_out(c, static_cast<int64_t>(gm) * N + gn, acc[i][j]);
    }
}

template <typename TA, typename TB, typename TC, bool kTransA>
cudaError_t fold_gemm(const TA* a, const TB* b, TC* c, int M, int N, int K, cudaStream_t st) {
  dim3 grid(static_cast<unsigned>((N + kFT - 1) / kFT), static_cast<unsigned>((M + kFT - 1) / kFT));
  fold_gemm_kernel<TA, TB, TC, kTransA><<<grid, kFThreads, 0, st>>>(a, b, c, M, N, K);
  return cudaGetLastError();
}

inline size_t up256(size_t v) { return (v + 255) & ~size_t(255); }

struct FoldWorkspace {
  size_t aug, ginv, t, flag, total;
};

FoldWorkspace fold_layout(int64_t m, int64_t r) {
  FoldWorkspace w;
  w.aug = 0;
  w.ginv = w.aug + up256(static_cast<size_t>(2 * r * r) * 8);
  w.t = w.ginv + up256(static_cast<size_t>(r * r) * 4);
  w.flag = w.t + up256(static_cast<size_t>(m * r) * 4);
  w.total = w.flag + 256;
  return w;
}

}  // namespace
}  // namespace twq

extern "C" {

size_t twq_fold_workspace_bytes(int64_t m, int64_t n, int64_t r) {
  (void)n;
  if (m <= 0 || r <= 0) return 0;
  return twq::fold_layout(m, r).total;
}

twq_status twq_fold_transforms(const float* Q, const float* G, const uint16_t* U,
                               const uint16_t* V, const uint16_t* R, int64_t m, int64_t n,
                               int64_t r, uint16_t* L1_out, uint16_t* L2_out, uint16_t* R_out,
                               void* workspace, size_t workspace_bytes, twq_stream_t stream) {
  if (m <= 0 || n <= 0 || r <= 0) return TWQ_ERR_INVALID_ARG;
  // r <= 1024 (the inversion's shared buffer); m / 64 output tiles fit a grid's y extent
  if (r > 1024 || m > 65535 * 64 || n > (int64_t(1) << 24)) return TWQ_ERR_UNSUPPORTED;
  if (!Q || !G || !U || !V || !R || !L1_out || !L2_out || !R_out || !workspace)
    return TWQ_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return TWQ_ERR_MISALIGNED;
  const twq::FoldWorkspace lay = twq::fold_layout(m, r);
  if (workspace_bytes < lay.total) return TWQ_ERR_INVALID_ARG;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  double* aug = reinterpret_cast<double*>(ws + lay.aug);
  float* ginv = reinterpret_cast<float*>(ws + lay.ginv);
  float* t = reinterpret_cast<float*>(ws + lay.t);
  int* flag = reinterpret_cast<int*>(ws + lay.flag);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int M = static_cast<int>(m), N = static_cast<int>(n), Rk = static_cast<int>(r);
  twq::gj_invert_kernel<<<1, twq::kInvThreads, 0, st>>>(G, Rk, aug, ginv, flag);
  cudaError_t e = cudaGetLastError();
  // U' = Q^T (U G)
  if (e == cudaSuccess) e = twq::fold_gemm<uint16_t, float, float, false>(U, G, t, M, Rk, Rk, st);
  if (e == cudaSuccess) e = twq::fold_gemm<float, float, uint16_t, true>(Q, t, L1_out, M, Rk, M, st);
  // V' = G^-1 V
  if (e == cudaSuccess) e = twq::fold_gemm<float, uint16_t, uint16_t, false>(ginv, V, L2_out, Rk, N, Rk, st);
  // R' = Q^T R
  if (e == cudaSuccess) e = twq::fold_gemm<float, uint16_t, uint16_t, true>(Q, R, R_out, M, N, M, st);
  if (e != cudaSuccess) return TWQ_ERR_CUDA;
  int singular = 0;
  if (cudaMemcpyAsync(&singular, flag, sizeof(int), cudaMemcpyDeviceToHost, st) != cudaSuccess ||
      cudaStreamSynchronize(st) != cudaSuccess)
    return TWQ_ERR_CUDA;
  return singular ? TWQ_ERR_INVALID_ARG : TWQ_OK;
}

}  // extern "C"
