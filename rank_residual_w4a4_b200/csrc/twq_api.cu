// C ABI of the library (include/twq.h): argument validation on the host, then
// stream-ordered launches. No entry point allocates device memory.
#include <string.h>

#include "twq_internal.h"

namespace {

constexpr int kVersion = 100;  // 0.1.0

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

twq_status shape_ok(int64_t m, int64_t n, int64_t r) {
  if (m <= 0 || n <= 0 || r < 0) return TWQ_ERR_INVALID_ARG;
  if (m % 128 || n % 128) return TWQ_ERR_INVALID_ARG;
  if (r % 16) return TWQ_ERR_INVALID_ARG;
  if (r > 256) return TWQ_ERR_UNSUPPORTED;
  // TMA coordinates and element offsets are 32-bit in the kernels.
  if (m > (int64_t(1) << 24) || n > (int64_t(1) << 24)) return TWQ_ERR_UNSUPPORTED;
  return TWQ_OK;
}

twq_status from_cuda(cudaError_t e) { return e == cudaSuccess ? TWQ_OK : TWQ_ERR_CUDA; }

// Checks shared by the three layer entry points. `need_res` / `need_lr` say
// which weight buffers the call reads.
twq_status check_layer(const uint8_t* xq, const float* sx, int64_t b, const twq_weights* w,
                       const void* y, bool need_res, bool need_lr) {
  if (!w) return TWQ_ERR_INVALID_ARG;
  twq_status s = shape_ok(w->m, w->n, w->r);
  if (s != TWQ_OK) return s;
  if (b < 0) return TWQ_ERR_INVALID_ARG;
  if (b > (int64_t(1) << 30)) return TWQ_ERR_UNSUPPORTED;
  if (b == 0) return TWQ_OK;
  if (!xq || !sx || !y) return TWQ_ERR_INVALID_ARG;
  if (!aligned16(xq) || !aligned16(sx) || !aligned16(y)) return TWQ_ERR_MISALIGNED;
  if (need_res) {
    if (!w->rq || !w->sr) return TWQ_ERR_INVALID_ARG;
    if (!aligned16(w->rq) || !aligned16(w->sr)) return TWQ_ERR_MISALIGNED;
  }
  if (need_lr) {
    if (w->r == 0) return TWQ_ERR_INVALID_ARG;
    if (!w->l1q || !w->sl1 || !w->l2t) return TWQ_ERR_INVALID_ARG;
    if (!aligned16(w->l1q) || !aligned16(w->sl1) || !aligned16(w->l2t)) return TWQ_ERR_MISALIGNED;
  }
  return TWQ_OK;
}

twq_status run(int mode, const uint8_t* xq, const float* sx, int64_t b, const twq_weights* w,
               void* out, const uint16_t* h, twq_stream_t stream) {
  twq::GemmCall c{mode, xq, sx, b, w, out, h};
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (twq::decode_eligible(c)) return from_cuda(twq::launch_decode(c, st));
  return from_cuda(twq::launch_gemm(c, st, nullptr));
}

}  // namespace

extern "C" {

int twq_version(void) { return kVersion; }

const char* twq_status_string(twq_status s) {
  switch (s) {
    case TWQ_OK: return "ok";
    case TWQ_ERR_INVALID_ARG: return "invalid argument";
    case TWQ_ERR_UNSUPPORTED: return "unsupported shape";
    case TWQ_ERR_MISALIGNED: return "misaligned pointer or stride";
    case TWQ_ERR_CUDA: return "CUDA error";
    case TWQ_ERR_NOT_IMPLEMENTED: return "not implemented";
    case TWQ_ERR_DEVICE: return "device wait timed out";
  }
  return "unknown status";
}

twq_status twq_weights_sizes(int64_t m, int64_t n, int64_t r, size_t bytes_out[5]) {
  if (!bytes_out) return TWQ_ERR_INVALID_ARG;
  twq_status s = shape_ok(m, n, r);
  if (s != TWQ_OK) return s;
  const int64_t G = m / 128;
  bytes_out[0] = static_cast<size_t>(n * (m / 2));
  bytes_out[1] = static_cast<size_t>(G * n * 4);
  bytes_out[2] = static_cast<size_t>(r * (m / 2));
  bytes_out[3] = static_cast<size_t>(G * r * 4);
  bytes_out[4] = static_cast<size_t>(n * r * 2);
  return TWQ_OK;
}

twq_status twq_act_sizes(int64_t b, int64_t m, size_t bytes_out[2]) {
  if (!bytes_out || b < 0 || m <= 0 || m % 128) return TWQ_ERR_INVALID_ARG;
  if (m > (int64_t(1) << 24) || b > (int64_t(1) << 30)) return TWQ_ERR_UNSUPPORTED;
  bytes_out[0] = static_cast<size_t>(b * (m / 2));
  bytes_out[1] = static_cast<size_t>(b * (m / 128) * 4);
  return TWQ_OK;
}

twq_status twq_quantize_act(const uint16_t* x, int64_t b, int64_t m, int64_t ldx, uint8_t* xq,
                            float* sx, twq_stream_t stream) {
  if (b < 0 || m <= 0 || m % 128 || ldx < m) return TWQ_ERR_INVALID_ARG;
  if (m > (int64_t(1) << 24) || b > (int64_t(1) << 30)) return TWQ_ERR_UNSUPPORTED;
  if (b == 0) return TWQ_OK;
  if (!x || !xq || !sx) return TWQ_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(xq) || !aligned16(sx) || ldx % 8) return TWQ_ERR_MISALIGNED;
  return from_cuda(twq::launch_quantize_act(x, b, m, ldx, xq, sx,
                                            reinterpret_cast<cudaStream_t>(stream)));
}

twq_status twq_quantize_act_a8(const uint16_t* x, int64_t b, int64_t m, int64_t ldx, int8_t* xq8,
                               float* sx, twq_stream_t stream) {
  if (b < 0 || m <= 0 || m % 128 || ldx < m) return TWQ_ERR_INVALID_ARG;
  if (m > (int64_t(1) << 24) || b > (int64_t(1) << 30)) return TWQ_ERR_UNSUPPORTED;
  if (b == 0) return TWQ_OK;
  if (!x || !xq8 || !sx) return TWQ_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(xq8) || !aligned16(sx) || ldx % 8) return TWQ_ERR_MISALIGNED;
  return from_cuda(twq::launch_quantize_act(x, b, m, ldx, reinterpret_cast<uint8_t*>(xq8), sx,
                                            reinterpret_cast<cudaStream_t>(stream), true));
}

twq_status twq_quantize_act_i8(const uint16_t* x, int64_t b, int64_t m, int64_t ldx, int8_t* xq8,
                               float* sx, twq_stream_t stream) {
  if (b < 0 || m <= 0 || m % 128 || ldx < m) return TWQ_ERR_INVALID_ARG;
  if (m > (int64_t(1) << 24) || b > (int64_t(1) << 30)) return TWQ_ERR_UNSUPPORTED;
  if (b == 0) return TWQ_OK;
  if (!x || !xq8 || !sx) return TWQ_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(xq8) || !aligned16(sx) || ldx % 8) return TWQ_ERR_MISALIGNED;
  return from_cuda(twq::launch_quantize_act(x, b, m, ldx, reinterpret_cast<uint8_t*>(xq8), sx,
                                            reinterpret_cast<cudaStream_t>(stream), false, true));
}

twq_status twq_pack_weights(const uint16_t* R, const uint16_t* L1, const uint16_t* L2,
                            const twq_weights* w, twq_stream_t stream) {
  if (!w) return TWQ_ERR_INVALID_ARG;
  twq_status s = shape_ok(w->m, w->n, w->r);
  if (s != TWQ_OK) return s;
  if (!R || !w->rq || !w->sr) return TWQ_ERR_INVALID_ARG;
  if (!aligned16(R) || !aligned16(w->rq) || !aligned16(w->sr)) return TWQ_ERR_MISALIGNED;
  if (w->r > 0) {
    if (!L1 || !L2 || !w->l1q || !w->sl1 || !w->l2t) return TWQ_ERR_INVALID_ARG;
    if (!aligned16(L1) || !aligned16(L2) || !aligned16(w->l1q) || !aligned16(w->sl1) ||
        !aligned16(w->l2t))
      return TWQ_ERR_MISALIGNED;
  }
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = twq::launch_pack_cols(R, w->m, w->n, w->rq, w->sr, st);
  if (e == cudaSuccess && w->r > 0) e = twq::launch_pack_cols(L1, w->m, w->r, w->l1q, w->sl1, st);
  if (e == cudaSuccess && w->r > 0) e = twq::launch_transpose_bf16(L2, w->r, w->n, w->l2t, st);
  return from_cuda(e);
}

twq_status twq_fused_linear(const uint8_t* xq, const float* sx, int64_t b, const twq_weights* w,
                            uint16_t* y, twq_stream_t stream) {
  const bool lr = w && w->r > 0;
  twq_status s = check_layer(xq, sx, b, w, y, true, lr);
  if (s != TWQ_OK || b == 0) return s;
  return run(lr ? twq::kModeFused : twq::kModeW4A4, xq, sx, b, w, y, nullptr, stream);
}

twq_status twq_w4a4_only(const uint8_t* xq, const float* sx, int64_t b, const twq_weights* w,
                         uint16_t* y, twq_stream_t stream) {
  twq_status s = check_layer(xq, sx, b, w, y, true, false);
  if (s != TWQ_OK || b == 0) return s;
  return run(twq::kModeW4A4, xq, sx, b, w, y, nullptr, stream);
}

twq_status twq_lowrank_only(const uint8_t* xq, const float* sx, int64_t b, const twq_weights* w,
                            uint16_t* y, twq_stream_t stream) {
  twq_status s = check_layer(xq, sx, b, w, y, false, true);
  if (s != TWQ_OK || b == 0) return s;
  return run(twq::kModeLowRank, xq, sx, b, w, y, nullptr, stream);
}

twq_status twq_fused_linear_a8(const int8_t* xq8, const float* sx, int64_t b, const twq_weights* w,
                               uint16_t* y, twq_stream_t stream) {
  const bool lr = w && w->r > 0;
  const uint8_t* xq = reinterpret_cast<const uint8_t*>(xq8);
  twq_status s = check_layer(xq, sx, b, w, y, true, lr);
  if (s != TWQ_OK || b == 0) return s;
  twq::GemmCall c{lr ? twq::kModeFused : twq::kModeW4A4, xq, sx, b, w, y, nullptr};
  c.a8 = true;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (twq::decode_eligible(c)) return from_cuda(twq::launch_decode(c, st));
  return from_cuda(twq::launch_gemm(c, st, nullptr));
}

twq_status twq_fused_linear_i8(const int8_t* xq8, const float* sx, int64_t b, const twq_weights* w,
                               uint16_t* y, twq_stream_t stream) {
  return twq_fused_linear_a8(xq8, sx, b, w, y, stream);
}

twq_status twq_pack_l2_int4(const uint16_t* L2, int64_t r, int64_t n, uint8_t* l2q, float* sl2q,
                            twq_stream_t stream) {
  if (r <= 0 || r % 128 || n <= 0 || n % 128) return TWQ_ERR_INVALID_ARG;
  if (r > 256 || n > (int64_t(1) << 24)) return TWQ_ERR_UNSUPPORTED;
  if (!L2 || !l2q || !sl2q) return TWQ_ERR_INVALID_ARG;
  if (!aligned16(L2) || !aligned16(l2q) || !aligned16(sl2q)) return TWQ_ERR_MISALIGNED;
  return from_cuda(twq::launch_pack_cols(L2, r, n, l2q, sl2q, reinterpret_cast<cudaStream_t>(stream)));
}

twq_status twq_fused_linear_s2q(const uint8_t* xq, const float* sx, int64_t b, const twq_weights* w,
                                const uint8_t* l2q, const float* sl2q, uint16_t* y,
                                twq_stream_t stream) {
  if (!w) return TWQ_ERR_INVALID_ARG;
  if (w->r <= 0 || w->r % 128) return w->r > 0 ? TWQ_ERR_UNSUPPORTED : TWQ_ERR_INVALID_ARG;
  twq_status s = check_layer(xq, sx, b, w, y, true, false);
  if (s != TWQ_OK || b == 0) return s;
  if (!w->l1q || !w->sl1 || !l2q || !sl2q) return TWQ_ERR_INVALID_ARG;
  if (!aligned16(w->l1q) || !aligned16(w->sl1) || !aligned16(l2q) || !aligned16(sl2q))
    return TWQ_ERR_MISALIGNED;
  twq::GemmCall c{twq::kModeFusedS2Q, xq, sx, b, w, y, nullptr};
  c.l2q = l2q;
  c.sl2q = sl2q;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (twq::decode_eligible(c)) return from_cuda(twq::launch_decode(c, st));
  return from_cuda(twq::launch_gemm(c, st, nullptr));
}

// Validates a twq_fused_linear_x call (b >= 1) and fills the decode launch.
static twq_status prepare_fused_x(const uint16_t* x, int64_t ldx, int64_t b, const twq_weights* w,
                                  uint16_t* y, twq::GemmCall* out, bool a8 = false) {
  if (!x || !y || !w->rq || !w->sr) return TWQ_ERR_INVALID_ARG;
  if (!aligned16(x) || ldx % 8 || !aligned16(y) || !aligned16(w->rq) || !aligned16(w->sr))
    return TWQ_ERR_MISALIGNED;
  const bool lr = w->r > 0;
  if (lr) {
    if (!w->l1q || !w->sl1 || !w->l2t) return TWQ_ERR_INVALID_ARG;
    if (!aligned16(w->l1q) || !aligned16(w->sl1) || !aligned16(w->l2t)) return TWQ_ERR_MISALIGNED;
  }
  twq::GemmCall c{lr ? twq::kModeFused : twq::kModeW4A4, nullptr, nullptr, b, w, y, nullptr};
  c.x = x;
  c.ldx = ldx;
  c.a8 = a8;
  if (!twq::decode_eligible(c)) return TWQ_ERR_UNSUPPORTED;
  *out = c;
  return TWQ_OK;
}

twq_status twq_fused_linear_x(const uint16_t* x, int64_t ldx, int64_t b, const twq_weights* w,
                              uint16_t* y, twq_stream_t stream) {
  if (!w) return TWQ_ERR_INVALID_ARG;
  twq_status s = shape_ok(w->m, w->n, w->r);
  if (s != TWQ_OK) return s;
  if (b < 0 || ldx < w->m) return TWQ_ERR_INVALID_ARG;
  if (b == 0) return TWQ_OK;
  twq::GemmCall c{};
  if ((s = prepare_fused_x(x, ldx, b, w, y, &c)) != TWQ_OK) return s;
  return from_cuda(twq::launch_decode(c, reinterpret_cast<cudaStream_t>(stream)));
}

twq_status twq_fused_linear_x_a8(const uint16_t* x, int64_t ldx, int64_t b, const twq_weights* w,
                                 uint16_t* y, twq_stream_t stream) {
  if (!w) return TWQ_ERR_INVALID_ARG;
  twq_status s = shape_ok(w->m, w->n, w->r);
  if (s != TWQ_OK) return s;
  if (b < 0 || ldx < w->m) return TWQ_ERR_INVALID_ARG;
  if (b == 0) return TWQ_OK;
  twq::GemmCall c{};
  if ((s = prepare_fused_x(x, ldx, b, w, y, &c, true)) != TWQ_OK) return s;
  return from_cuda(twq::launch_decode(c, reinterpret_cast<cudaStream_t>(stream)));
}

twq_status twq_fused_linear_x_host(const uint16_t* x_host, int64_t b, const twq_weights* w,
                                   uint16_t* x_dev, uint16_t* y_dev, uint16_t* y_host,
                                   twq_stream_t stream) {
  if (!w) return TWQ_ERR_INVALID_ARG;
  twq_status s = shape_ok(w->m, w->n, w->r);
  if (s != TWQ_OK) return s;
  if (b < 0) return TWQ_ERR_INVALID_ARG;
  if (b == 0) return TWQ_OK;
  if (!x_host || !y_host) return TWQ_ERR_INVALID_ARG;
  twq::GemmCall c{};
  if ((s = prepare_fused_x(x_dev, w->m, b, w, y_dev, &c)) != TWQ_OK) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const size_t xb = static_cast<size_t>(b) * w->m * 2, yb = static_cast<size_t>(b) * w->n * 2;
  if (cudaMemcpyAsync(x_dev, x_host, xb, cudaMemcpyHostToDevice, st) != cudaSuccess)
    return TWQ_ERR_CUDA;
  cudaError_t e = twq::launch_decode(c, st);
  if (e != cudaSuccess) return from_cuda(e);
  if (cudaMemcpyAsync(y_host, y_dev, yb, cudaMemcpyDeviceToHost, st) != cudaSuccess)
    return TWQ_ERR_CUDA;
  return TWQ_OK;
}

twq_status twq_linear_host(const uint16_t* x_host, int64_t b, const twq_weights* w,
                           uint16_t* x_dev, int8_t* xq8, float* sx, uint16_t* y_dev,
                           uint16_t* y_host, twq_stream_t stream) {
  if (!w) return TWQ_ERR_INVALID_ARG;
  twq_status s = shape_ok(w->m, w->n, w->r);
  if (s != TWQ_OK) return s;
  if (b < 0) return TWQ_ERR_INVALID_ARG;
  if (b > (int64_t(1) << 30)) return TWQ_ERR_UNSUPPORTED;
  if (b == 0) return TWQ_OK;
  if (!x_host || !y_host || !x_dev || !y_dev) return TWQ_ERR_INVALID_ARG;
  if (!aligned16(x_dev)) return TWQ_ERR_MISALIGNED;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const size_t xb = static_cast<size_t>(b) * w->m * 2, yb = static_cast<size_t>(b) * w->n * 2;
  // Decode batches that the one-launch layer takes: no codes in HBM at all.
  twq::GemmCall c{};
  const bool one = prepare_fused_x(x_dev, w->m, b, w, y_dev, &c) == TWQ_OK;
  const uint8_t* xq = reinterpret_cast<const uint8_t*>(xq8);
  if (!one) {
    const bool lr = w->r > 0;
    if ((s = check_layer(xq, sx, b, w, y_dev, true, lr)) != TWQ_OK) return s;
  }
  if (cudaMemcpyAsync(x_dev, x_host, xb, cudaMemcpyHostToDevice, st) != cudaSuccess)
    return TWQ_ERR_CUDA;
  cudaError_t e;
  if (one) {
    e = twq::launch_decode(c, st);
  } else {
    // the codes one per byte (twq_quantize_act_i8), which the layer reads as they lie
    e = twq::launch_quantize_act(x_dev, b, w->m, w->m, reinterpret_cast<uint8_t*>(xq8), sx, st,
                                 false, true);
    if (e == cudaSuccess) {
      twq::GemmCall g{w->r > 0 ? twq::kModeFused : twq::kModeW4A4, xq, sx, b, w, y_dev, nullptr};
      g.a8 = true;
      e = twq::decode_eligible(g) ? twq::launch_decode(g, st) : twq::launch_gemm(g, st, nullptr);
    }
  }
  if (e != cudaSuccess) return from_cuda(e);
  if (cudaMemcpyAsync(y_host, y_dev, yb, cudaMemcpyDeviceToHost, st) != cudaSuccess)
    return TWQ_ERR_CUDA;
  return TWQ_OK;
}

size_t twq_unfused_workspace_bytes(int64_t b, int64_t n, int64_t r) {
  if (b <= 0 || n <= 0 || r < 0) return 0;
  // Y_res fp32 (b x n) | Y_lr fp32 (b x n) | H bf16 (b x r), each 256-byte aligned
  auto up = [](size_t v) { return (v + 255) & ~size_t(255); };
  return up(size_t(b) * n * 4) * 2 + up(size_t(b) * r * 2);
}

twq_status twq_unfused_linear(const uint8_t* xq, const float* sx, int64_t b, const twq_weights* w,
                              uint16_t* y, void* workspace, size_t workspace_bytes,
                              twq_stream_t stream) {
  const bool lr = w && w->r > 0;
  twq_status s = check_layer(xq, sx, b, w, y, true, lr);
  if (s != TWQ_OK || b == 0) return s;
  if (!workspace) return TWQ_ERR_INVALID_ARG;
  if (!aligned16(workspace)) return TWQ_ERR_MISALIGNED;
  if (workspace_bytes < twq_unfused_workspace_bytes(b, w->n, w->r)) return TWQ_ERR_INVALID_ARG;
  auto up = [](size_t v) { return (v + 255) & ~size_t(255); };
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  float* yres = reinterpret_cast<float*>(ws);
  float* ylr = reinterpret_cast<float*>(ws + up(size_t(b) * w->n * 4));
  uint16_t* h = reinterpret_cast<uint16_t*>(ws + 2 * up(size_t(b) * w->n * 4));
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (!lr) return run(twq::kModeW4A4, xq, sx, b, w, y, nullptr, stream);
  s = run(twq::kModeResF32, xq, sx, b, w, yres, nullptr, stream);
  if (s == TWQ_OK) s = run(twq::kModeHOnly, xq, sx, b, w, h, nullptr, stream);
  if (s == TWQ_OK) s = run(twq::kModeS2F32, xq, sx, b, w, ylr, h, stream);
  if (s == TWQ_OK) s = from_cuda(twq::launch_add_cast(yres, ylr, b * w->n, y, st));
  return s;
}

twq_status twq_device_status(int* code) {
  if (!code) return TWQ_ERR_INVALID_ARG;
  cudaError_t e = cudaDeviceSynchronize();
  if (e != cudaSuccess) return TWQ_ERR_CUDA;
  int c1 = 0, c2 = 0, c3 = 0;
  e = twq::read_and_clear_device_status(&c1);
  if (e == cudaSuccess) e = twq::read_and_clear_decode_status(&c2);
  if (e == cudaSuccess) e = twq::read_and_clear_pair_status(&c3);
  if (e != cudaSuccess) return TWQ_ERR_CUDA;
  *code = c1 ? c1 : (c2 ? c2 : c3);
  return *code ? TWQ_ERR_DEVICE : TWQ_OK;
}

twq_status twq_selftest_wait_timeout(const uint8_t* xq, const float* sx, int64_t b,
                                     const twq_weights* w, uint16_t* y, int64_t wait_limit_ns,
                                     twq_stream_t stream) {
  twq_status s = check_layer(xq, sx, b, w, y, true, false);
  if (s != TWQ_OK) return s;
  if (wait_limit_ns < 1000 || wait_limit_ns > 1000000000) return TWQ_ERR_INVALID_ARG;
  twq::GemmCall c{twq::kModeW4A4, xq, sx, b, w, y, nullptr};
  if (!twq::pair_eligible(c)) return TWQ_ERR_UNSUPPORTED;
  return from_cuda(twq::launch_pair_stall_selftest(c, reinterpret_cast<cudaStream_t>(stream),
                                                   static_cast<unsigned long long>(wait_limit_ns)));
}

void twq_release_cache(void) {
  twq::release_decode_cache();
  twq::release_noalloc_cache();
}

int twq_launches_per_call(const char* ep) {
  if (!ep) return -1;
  if (!strcmp(ep, "twq_quantize_act") || !strcmp(ep, "twq_quantize_act_a8")) return 1;
  if (!strcmp(ep, "twq_pack_weights")) return 3;
  if (!strcmp(ep, "twq_pack_l2_int4") || !strcmp(ep, "twq_fused_linear_s2q")) return 1;
  if (!strcmp(ep, "twq_fused_linear") || !strcmp(ep, "twq_w4a4_only") ||
      !strcmp(ep, "twq_lowrank_only") || !strcmp(ep, "twq_fused_linear_x") ||
      !strcmp(ep, "twq_fused_linear_x_host") || !strcmp(ep, "twq_fused_linear_a8") ||
      !strcmp(ep, "twq_fused_linear_x_a8") || !strcmp(ep, "twq_quantize_act_i8") ||
      !strcmp(ep, "twq_fused_linear_i8"))
    return 1;
  if (!strcmp(ep, "twq_linear_host")) return 2;
  if (!strcmp(ep, "twq_selftest_wait_timeout")) return 1;  // 1 for the batches twq_fused_linear_x takes
  if (!strcmp(ep, "twq_unfused_linear") || !strcmp(ep, "twq_unfused_linear_noalloc")) return 4;
  if (!strcmp(ep, "twq_fold_transforms")) return 5;
  return -1;
}

}  // extern "C"
