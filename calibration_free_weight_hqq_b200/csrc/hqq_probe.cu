// hqq_probe.cu - throughput probe of the special-function unit (MUFU lg2/ex2) on this GPU,
// the unit that bounds the HQQ solver. Built into a separate library (libhqq_probe.so), not
// the quantization ABI; bench.py --probe-sfu runs it to justify the roofline's peak.
//
// Every thread runs 8 independent dependency chains of approximate lg2/ex2 (and nothing
// else but one FADD/FMUL per step), so the SFU issue rate, not latency, limits the kernel.
// out must hold blocks*threads floats (one store per thread, so the work is not removed).
#include <cuda_runtime.h>

namespace {

__device__ __forceinline__ float ex2a(float x) {
  float y;
  asm volatile("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float lg2a(float x) {
  float y;
  asm volatile("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

template <int OP>
__global__ void sfu_probe_kernel(float* out, int iters) {
  float x[8];
#pragma unroll
  for (int c = 0; c < 8; ++c) x[c] = 0.6f + 0.01f * c + 1e-7f * threadIdx.x;
  for (int i = 0; i < iters; ++i) {
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      if (OP == 0) x[c] = ex2a(-x[c]);                // 1 SFU op; stays in [0.5, 0.71]
      else if (OP == 1) x[c] = lg2a(x[c]) + 1.7f;     // 1 SFU op; converges near 3.4
      else x[c] = ex2a(0.7f * lg2a(x[c]));            // 2 SFU ops: x^0.7, as in the solver
    }
  }
  float s = 0.f;
#pragma unroll
  for (int c = 0; c < 8; ++c) s += x[c];
  out[(size_t)blockIdx.x * blockDim.x + threadIdx.x] = s;
}

}  // namespace

// op: 0 = ex2 only, 1 = lg2 only, 2 = lg2 then ex2. Returns the cudaError_t of the launch.
extern "C" __attribute__((visibility("default"))) int hqq_probe_sfu(int op, float* out,
                                                                    int blocks, int threads,
                                                                    int iters, void* stream) {
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (op == 0) sfu_probe_kernel<0><<<blocks, threads, 0, st>>>(out, iters);
  else if (op == 1) sfu_probe_kernel<1><<<blocks, threads, 0, st>>>(out, iters);
  else sfu_probe_kernel<2><<<blocks, threads, 0, st>>>(out, iters);
  return (int)cudaGetLastError();
}
