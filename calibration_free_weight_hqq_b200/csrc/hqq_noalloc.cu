// hqq_noalloc.cu - hqq_quantize_ex_noalloc: the second-level (8-bit scale/zero) quantize
// path with its scratch in a fixed array compiled into the library, for callers that cannot
// allocate device memory themselves. It forwards to hqq_quantize_ex with that array as the
// workspace; nothing here allocates.
#include <mutex>

#include "../../include/hqq/hqq.h"

#define HQQ_EXPORT extern "C" __attribute__((visibility("default")))

namespace {

// The scratch: fp32 scale and zero of every group (256-byte aligned parts), written in full
// by the solver before the second-level kernel reads them, so nothing in it needs clearing.
constexpr size_t kScratchBytes = HQQ_NOALLOC_SCRATCH_BYTES;
static __device__ __align__(256) unsigned char g_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_setup_mutex;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of g_scratch on the current device. In host code g_scratch only names a
// host-side stand-in, so its address must come from the runtime, once per device, with that
// device current.
cudaError_t scratch_on_current_device(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  if (g_scratch_ptr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return cudaSuccess;
}

}  // namespace

HQQ_EXPORT hqq_status hqq_quantize_ex_noalloc(const void* W, int64_t rows, int64_t cols,
                                              const hqq_params* params, void* Wq_packed,
                                              void* scale, void* zero, void* scale_mm,
                                              void* zero_mm, cudaStream_t stream) {
  if (!params) return HQQ_ERR_INVALID_ARG;
  const size_t need = hqq_workspace_bytes(rows, cols, params);
  if (need == (size_t)-1 || need == 0) {
    // invalid arguments (reported by the regular path before any launch) or no scratch needed
    return hqq_quantize_ex(W, rows, cols, params, Wq_packed, scale, zero, scale_mm, zero_mm,
                           nullptr, 0, stream);
  }
  if (need > kScratchBytes) return HQQ_ERR_WORKSPACE;
  void* scratch = nullptr;
  if (scratch_on_current_device(&scratch) != cudaSuccess) return HQQ_ERR_CUDA;
  return hqq_quantize_ex(W, rows, cols, params, Wq_packed, scale, zero, scale_mm, zero_mm,
                         scratch, kScratchBytes, stream);
}
