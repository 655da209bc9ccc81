// hqq_abi_internal.h - helpers of the C ABI layer shared between its translation units
// (hidden symbols of libhqq_b200.so, not part of the public interface).
#pragma once

#include "../../include/hqq/hqq.h"

namespace hqqabi {

// HQQ_OK for cudaSuccess; otherwise records the CUDA error name and message for
// hqq_last_cuda_error() and returns HQQ_ERR_CUDA.
hqq_status cuda_status(cudaError_t e);

// The argument checks hqq_quantize_ex makes first, in its order: shapes, parameters, dtypes,
// null and misaligned pointers (then come the workspace and the device of W, checked by the
// caller). HQQ_OK also for an empty matrix (nothing to launch).
hqq_status validate_quantize(const void* W, int64_t rows, int64_t cols, const hqq_params& prm,
                             const void* Wq_packed, const void* scale, const void* zero,
                             const void* scale_mm, const void* zero_mm);

// HQQ_ERR_INVALID_ARG when p is device memory of another device than the current one, or
// host memory the GPU cannot address (neither pinned nor managed); HQQ_OK otherwise.
hqq_status check_device(const void* p);

}  // namespace hqqabi
