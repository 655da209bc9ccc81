// hqq_probe.cu - throughput probes behind the rooflines: the special-function unit (MUFU
// lg2/ex2, which bounds the HQQ solver) and HBM read-only / write-only / copy bandwidth (the
// dequantizer writes 4 bytes for every byte it reads at 4 bits). Built into a separate
// library (bench_probes/libhqq_probe.so), not the quantization ABI; run by
// `python bench_probes/probe.py sfu` / `python bench_probes/probe.py hbm`.
//
// Every thread runs 8 independent dependency chains of approximate lg2/ex2 (and nothing
// else but one FADD/FMUL per step), so the SFU issue rate, not latency, limits the kernel.
// out must hold blocks*threads floats (one store per thread, so the work is not removed).
#include <cuda_runtime.h>
#include <stdint.h>

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

// HBM probes: 16-byte accesses, 4 per thread per pass in flight, grid-stride.
__global__ void hbm_write_kernel(uint4* dst, size_t n16) {
  const size_t stride = (size_t)gridDim.x * blockDim.x;
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n16; i += 4 * stride) {
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const size_t j = i + k * stride;
      if (j < n16) dst[j] = make_uint4((uint32_t)j, 1u, 2u, 3u);
    }
  }
}
__global__ void hbm_read_kernel(const uint4* src, size_t n16, uint32_t* out) {
  const size_t stride = (size_t)gridDim.x * blockDim.x;
  uint32_t acc = 0;
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n16; i += 4 * stride) {
    uint4 v[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const size_t j = i + k * stride;
      v[k] = j < n16 ? __ldcs(src + j) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int k = 0; k < 4; ++k) acc ^= v[k].x ^ v[k].y ^ v[k].z ^ v[k].w;
  }
  out[(size_t)blockIdx.x * blockDim.x + threadIdx.x] = acc;
}
__global__ void hbm_copy_kernel(const uint4* src, uint4* dst, size_t n16) {
  const size_t stride = (size_t)gridDim.x * blockDim.x;
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n16; i += 4 * stride) {
    uint4 v[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const size_t j = i + k * stride;
      if (j < n16) v[k] = __ldcs(src + j);
    }
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const size_t j = i + k * stride;
      if (j < n16) dst[j] = v[k];
    }
  }
}

}  // namespace

// op: 0 = write `bytes` to a, 1 = read `bytes` from a (one uint32 per thread to b),
// 2 = copy `bytes` from a to b. bytes must be a multiple of 16; b must hold blocks*threads
// uint32 for op 1.
extern "C" __attribute__((visibility("default"))) int hqq_probe_hbm(int op, void* a, void* b,
                                                                    size_t bytes, int blocks,
                                                                    int threads, void* stream) {
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const size_t n16 = bytes / 16;
  if (op == 0) hbm_write_kernel<<<blocks, threads, 0, st>>>(reinterpret_cast<uint4*>(a), n16);
  else if (op == 1)
    hbm_read_kernel<<<blocks, threads, 0, st>>>(reinterpret_cast<const uint4*>(a), n16,
                                                reinterpret_cast<uint32_t*>(b));
  else
    hbm_copy_kernel<<<blocks, threads, 0, st>>>(reinterpret_cast<const uint4*>(a),
                                                reinterpret_cast<uint4*>(b), n16);
  return (int)cudaGetLastError();
}

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
