// An entry point for callers that may not allocate device memory.
//
// Some callers cannot call cudaMalloc: a plugin inside a host framework that
// owns the whole device-memory budget, or a latency-critical service that must
// not let an allocation synchronize the device in the middle of its work. The
// unfused comparator needs scratch space (fp32 Y_res and Y_lr, BF16 H); this
// variant takes it from a fixed array that the library itself holds, so the
// caller passes only its inputs and outputs.
//
// The array is a file-scope __device__ object: every GPU that loads this
// library holds its kNoAllocScratchBytes until the process exits. In host code
// its name is only a host-side stand-in; the device address is obtained once
// per device, with that device current, through cudaGetSymbolAddress.
#include <mutex>

#include "twq_internal.h"

namespace {

constexpr size_t kNoAllocScratchBytes = size_t(16) << 20;  // 16 MiB
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

std::mutex g_setup_mutex;
void* g_scratch_addr[kMaxDevices];  // device address of g_noalloc_scratch, per device

// Set-up, once per device: resolve the scratch array's device address with
// that device current (the caller's current device).
twq_status scratch_address(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return TWQ_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return TWQ_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return TWQ_ERR_CUDA;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return TWQ_OK;
}

}  // namespace

namespace twq {
// Forgets the resolved addresses, so that the next call on each device resolves
// the array again (needed after the caller's cudaDeviceReset, which ends the
// context that the old address belonged to).
void release_noalloc_cache() {
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  for (void*& p : g_scratch_addr) p = nullptr;
}
}  // namespace twq

extern "C" twq_status twq_unfused_linear_noalloc(const uint8_t* xq, const float* sx, int64_t b,
                                                 const twq_weights* w, uint16_t* y,
                                                 twq_stream_t stream) {
  if (!w || b < 0) return TWQ_ERR_INVALID_ARG;
  if (b == 0) return twq_unfused_linear(xq, sx, b, w, y, nullptr, 0, stream);
  if (w->m <= 0 || w->n <= 0 || w->r < 0) return TWQ_ERR_INVALID_ARG;
  // Without a low-rank part the comparator is the W4A4 kernel alone (what
  // twq_unfused_linear runs for r == 0), which uses no scratch: no size limit then.
  if (w->r == 0) return twq_w4a4_only(xq, sx, b, w, y, stream);
  const size_t need = twq_unfused_workspace_bytes(b, w->n, w->r);
  if (need == 0) return TWQ_ERR_INVALID_ARG;
  if (need > kNoAllocScratchBytes) return TWQ_ERR_UNSUPPORTED;  // beyond the fixed 16 MiB
  void* scratch = nullptr;
  twq_status s = scratch_address(&scratch);
  if (s != TWQ_OK) return s;
  return twq_unfused_linear(xq, sx, b, w, y, scratch, kNoAllocScratchBytes, stream);
}
