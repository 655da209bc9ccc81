// hqq_kernels.h - host-side launch interface between the C ABI layer and the kernels.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace hqqk {

// Element types; the values equal the public hqq_dtype enumerators.
enum Dt : int { kF16 = 0, kBF16 = 1, kF32 = 2, kU8 = 3 };

// One matrix of the quantize path.
struct QuantJob {
  const void* W;     // device, row-major [rows, cols]
  int64_t rows, cols, n_groups;
  int w_dtype;       // Dt
  int nbits, group_size, axis, iters;
  float p, beta0, kappa;
  uint8_t* packed;   // device, packed code stream
  void* scale;       // device, n_groups values of scale_dtype
  void* zero;        // device, n_groups values of zero_dtype
  int scale_dtype;   // Dt (kF32 when the second level follows)
  int zero_dtype;
  int flags;         // HQQ_FLAG_* bits
};

// One matrix of the dequantize path.
struct DequantJob {
  const uint8_t* packed;
  const void* scale;  // meta_dtype values, or uint8 codes when scale_mm != nullptr
  const void* zero;   // meta_dtype values, or uint8 codes when zero_mm != nullptr
  const float* scale_mm;  // second-level (step2, zero2) pairs or nullptr
  const float* zero_mm;
  int meta_group_size;
  int meta_dtype;
  int64_t rows, cols, n_groups;
  int nbits, group_size, axis;
  int out_dtype;
  void* out;
};

// Matrices per batched launch (their pointers and tile prefix sums travel as kernel
// parameters); larger batches are split into several launches.
constexpr int kMaxBatch = 256;

cudaError_t launch_quantize(const QuantJob& job, cudaStream_t stream);
// All jobs share nbits, group_size, axis, iters, p, beta0, kappa and the dtypes.
cudaError_t launch_quantize_batched(const QuantJob* jobs, int n, cudaStream_t stream);
cudaError_t launch_dequantize(const DequantJob& job, cudaStream_t stream);
// All jobs share the settings and dtypes; only pointers and shapes differ.
cudaError_t launch_dequantize_batched(const DequantJob* jobs, int n, cudaStream_t stream);
// Y[M, N] = X[M, K] · W'^T (+ bias) with W' the dequantized 4-bit, group-64, axis-1 weight
// [N, K]; X, bias and Y share x_dtype (kBF16 or kF16). Shapes and alignment are validated by
// the caller: K % 64 == 0, N % 8 == 0, 16-byte aligned X, packed and Y.
struct GemmJob {
  const void* X;
  const uint8_t* packed;
  const void* scale;
  const void* zero;
  const void* bias;  // nullptr or [N]
  void* Y;
  int64_t M, N, K;
  int x_dtype;
  int meta_dtype;
  bool overlap_weights;  // HQQ_FLAG_OVERLAP_WEIGHTS: the decode kernel may overlap the
                         // previous kernel on the stream (programmatic dependent launch)
};
cudaError_t launch_w4a16_gemm(const GemmJob& job, cudaStream_t stream);
// Number of bounded waits inside the GEMM kernel that ran out of time since the library was
// loaded (0 on every healthy run).
cudaError_t read_gemm_timeouts(unsigned int* out);

// MXFP4: n = rows*cols elements (n % 32 == 0), blocks of 32 consecutive elements.
cudaError_t launch_mxfp4_quantize(const void* W, int dtype, int64_t n, uint8_t* codes,
                                  uint8_t* scales, cudaStream_t stream);
cudaError_t launch_mxfp4_dequantize(const uint8_t* codes, const uint8_t* scales, int64_t n,
                                    int out_dtype, void* out, cudaStream_t stream);

cudaError_t launch_quantize_meta(const void* meta, int dtype, int64_t n, int group, uint8_t* q,
                                 float* mm, cudaStream_t stream);
cudaError_t launch_dequantize_meta(const uint8_t* q, const float* mm, int64_t n, int group,
                                   float* out, cudaStream_t stream);

}  // namespace hqqk
