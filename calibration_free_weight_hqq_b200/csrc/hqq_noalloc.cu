// hqq_noalloc.cu - hqq_quantize_ex_noalloc: the second-level (8-bit scale/zero) quantize
// path with its scratch in a fixed array compiled into the library, for callers that cannot
// allocate device memory themselves. It validates the call exactly as hqq_quantize_ex does,
// then forwards to it with that array as the workspace; nothing here allocates.
#include <mutex>

#include "../../include/hqq/hqq.h"
#include "hqq_abi_internal.h"

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
// host-side stand-in, so its address must come from the runtime: once per device (the
// first call on it), with that device current, and then from this table.
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
  // The same checks, in the same order, as hqq_quantize_ex, so that an invalid call reports
  // the same status through either entry point; then the size, then the device of W.
  hqq_status st = hqqabi::validate_quantize(W, rows, cols, *params, Wq_packed, scale, zero,
                                            scale_mm, zero_mm);
  if (st != HQQ_OK) return st;
  const size_t need = hqq_workspace_bytes(rows, cols, params);
  if (need == 0 || rows * cols == 0)  // no second level: no scratch at all
    return hqq_quantize_ex(W, rows, cols, params, Wq_packed, scale, zero, scale_mm, zero_mm,
                           nullptr, 0, stream);
  if (need > kScratchBytes) return HQQ_ERR_WORKSPACE;
  if ((st = hqqabi::check_device(W)) != HQQ_OK) return st;
  // The current device is the one W lives on (checked just above).
  void* scratch = nullptr;
  st = hqqabi::cuda_status(scratch_on_current_device(&scratch));
  if (st != HQQ_OK) return st;
  return hqq_quantize_ex(W, rows, cols, params, Wq_packed, scale, zero, scale_mm, zero_mm,
                         scratch, kScratchBytes, stream);
}
