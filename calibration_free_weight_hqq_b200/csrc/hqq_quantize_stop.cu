// hqq_quantize_stop.cu - the solver with HQQ_FLAG_STOP_AT_FIXED_POINT compiled in: a warp
// stops iterating once every group in it sits at a fixed point of the zero update with the
// shrinkage provably zero, after which every remaining evaluation would repeat the last one
// exactly (results bit-identical to running all iterations).
#include "hqq_quantize_impl.cuh"

namespace hqqk {

cudaError_t launch_quantize_stop(const QuantJob* jobs, int n, bool batched, cudaStream_t st) {
  if (!batched) return launch_batch<1, true>(jobs, n, st);
  for (int i = 0; i < n; i += kMaxBatch) {
    const int k = n - i < kMaxBatch ? n - i : kMaxBatch;
    const cudaError_t e = launch_batch<kMaxBatch, true>(jobs + i, k, st);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace hqqk
