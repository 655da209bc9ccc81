// hqq_mx.cu - MXFP4 weight-only encoding and decoding.
//
// What is computed ("HQQ calibration-free guide" (lnwmold.com) §5.1 lists an mxfp4 weight-only
// mode; the encoding is the Open Compute Project Microscaling format MXFP4): a row-major
// [rows, cols] weight is cut into blocks of 32 consecutive elements of a row. Each block gets
// one E8M0 scale 2^e, e = floor(log2(max |v|)) - 2 clamped to [-127, 127] (an all-zero block
// takes -127), stored as the byte e + 127; each element is v / 2^e rounded to the nearest FP4
// E2M1 value (ties to the even mantissa bit, magnitudes above 6 saturating to 6, sign kept),
// two codes per byte with element 2j in the low nibble. Decoding is E2M1 value * 2^e.
//
// Both kernels are HBM-bound elementwise passes (encode: read 2 B, write 0.53 B per bf16
// weight). A warp covers 8 blocks: lane l holds elements 8l .. 8l+7 of the warp's 256 (one
// 16-byte load for 16-bit inputs), the 4 lanes of a block reduce its maximum with two
// shuffles, and the lane writes its 8 codes as one 32-bit word (a warp writes 128 contiguous
// bytes). The division by 2^e is an exact multiplication by a power of two; the rounding to
// E2M1 is the hardware conversion cvt.rn.satfinite.e2m1x2.f32, whose result the tests check
// against the definition element by element.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "hqq_device.cuh"
#include "hqq_kernels.h"

namespace hqqk {
namespace {

#ifndef HQQ_MX_UNROLL
#define HQQ_MX_UNROLL 4
#endif
constexpr int kMxThreads = 256;
constexpr int kMxUnroll = HQQ_MX_UNROLL;  // 256-element chunks per warp per iteration

template <int DT>
__device__ __forceinline__ void load8(const void* W, int64_t i, float (&v)[8]) {
  if constexpr (DT == kF32) {
    const float4* p = reinterpret_cast<const float4*>(static_cast<const float*>(W) + i);
    const float4 a = __ldcs(p), b = __ldcs(p + 1);
    v[0] = a.x, v[1] = a.y, v[2] = a.z, v[3] = a.w, v[4] = b.x, v[5] = b.y, v[6] = b.z,
    v[7] = b.w;
  } else {
    const uint4 u =
        __ldcs(reinterpret_cast<const uint4*>(static_cast<const unsigned short*>(W) + i));
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      if constexpr (DT == kBF16) {
        v[2 * k] = __uint_as_float(w[k] << 16);
        v[2 * k + 1] = __uint_as_float(w[k] & 0xFFFF0000u);
      } else {
        v[2 * k] = f16_bits_to_f32(w[k] & 0xFFFFu);
        v[2 * k + 1] = f16_bits_to_f32(w[k] >> 16);
      }
    }
  }
}

// floor(log2 amax) - 2, clamped to [-127, 127]; amax is finite and >= 0.
__device__ __forceinline__ int mx_exponent(float amax) {
  const uint32_t b = __float_as_uint(amax);
  const int E = static_cast<int>(b >> 23);
  int fl;
  if (E != 0)
    fl = E - 127;
  else if (b == 0)
    return -127;
  else
    fl = (31 - __clz(static_cast<int>(b))) - 149;  // subnormal: value = b * 2^-149
  return min(127, max(-127, fl - 2));
}

// 2^k as fp32 for k in [-127, 127] (2^-127 is the subnormal 0x00400000).
__device__ __forceinline__ float pow2i(int k) {
  return k > -127 ? __uint_as_float(static_cast<uint32_t>(k + 127) << 23)
                  : __uint_as_float(0x00400000u);
}

// Two fp32 values to two E2M1 codes in one byte, `lo` in the low nibble.
__device__ __forceinline__ uint32_t e2m1x2(float lo, float hi) {
  uint16_t r;
  asm("{\n\t.reg .b8 t;\n\tcvt.rn.satfinite.e2m1x2.f32 t, %1, %2;\n\tcvt.u16.u8 %0, t;\n\t}"
      : "=h"(r)
      : "f"(hi), "f"(lo));
  return r;
}

// One byte of two E2M1 codes to two halves (exact), the low nibble in the low half.
__device__ __forceinline__ __half2 e2m1x2_to_half2(uint32_t byte) {
  uint32_t h;
  asm("{\n\t.reg .b8 t;\n\tcvt.u8.u32 t, %1;\n\tcvt.rn.f16x2.e2m1x2 %0, t;\n\t}"
      : "=r"(h)
      : "r"(byte));
  return *reinterpret_cast<__half2*>(&h);
}

// Encode the 8 elements v of one lane (its block = 4 lanes) and store them.
__device__ __forceinline__ void encode8(const float (&v)[8], int64_t i, bool in,
                                        uint8_t* __restrict__ codes,
                                        uint8_t* __restrict__ scales, int lane) {
  float amax = 0.0f;
#pragma unroll
  for (int k = 0; k < 8; ++k) amax = fmaxf(amax, fabsf(v[k]));
  amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, 1));
  amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, 2));
  const int e = mx_exponent(amax);
  const float inv = pow2i(-e);
  uint32_t packed = 0;
#pragma unroll
  for (int k = 0; k < 4; ++k)
    packed |= e2m1x2(__fmul_rn(v[2 * k], inv), __fmul_rn(v[2 * k + 1], inv)) << (8 * k);
  if (in) {
    *reinterpret_cast<uint32_t*>(codes + i / 2) = packed;
    if ((lane & 3) == 0) scales[i / 32] = static_cast<uint8_t>(e + 127);
  }
}

// Each warp takes kMxUnroll consecutive 256-element chunks per iteration and issues all their
// loads before converting any (more bytes in flight per SM).
template <int DT>
__global__ void __launch_bounds__(kMxThreads) mxfp4_quantize_kernel(const void* __restrict__ W,
                                                                     int64_t n,
                                                                     uint8_t* __restrict__ codes,
                                                                     uint8_t* __restrict__ scales) {
  const int lane = threadIdx.x & 31;
  const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  for (int64_t w = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
       w * 256 * kMxUnroll < n; w += nwarps) {
    float v[kMxUnroll][8];
#pragma unroll
    for (int u = 0; u < kMxUnroll; ++u) {
      const int64_t i = (w * kMxUnroll + u) * 256 + lane * 8;
      if (i < n) {  // n % 32 == 0: the 4 lanes of a block are all in or all out
        load8<DT>(W, i, v[u]);
      } else {
#pragma unroll
        for (int k = 0; k < 8; ++k) v[u][k] = 0.0f;
      }
    }
#pragma unroll
    for (int u = 0; u < kMxUnroll; ++u) {
      const int64_t i = (w * kMxUnroll + u) * 256 + lane * 8;
      encode8(v[u], i, i < n, codes, scales, lane);
    }
  }
}

template <int OUT>
__global__ void __launch_bounds__(kMxThreads) mxfp4_dequantize_kernel(
    const uint8_t* __restrict__ codes, const uint8_t* __restrict__ scales, int64_t n,
    void* __restrict__ out) {
  const int lane = threadIdx.x & 31;
  const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  for (int64_t w = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
       w * 256 * kMxUnroll < n; w += nwarps) {
    uint32_t c[kMxUnroll];
    int sc[kMxUnroll];
#pragma unroll
    for (int u = 0; u < kMxUnroll; ++u) {
      const int64_t i = (w * kMxUnroll + u) * 256 + lane * 8;
      c[u] = i < n ? __ldcs(reinterpret_cast<const unsigned int*>(codes + i / 2)) : 0u;
      sc[u] = i < n ? static_cast<int>(__ldg(scales + i / 32)) : 127;
    }
#pragma unroll
    for (int u = 0; u < kMxUnroll; ++u) {
      const int64_t i = (w * kMxUnroll + u) * 256 + lane * 8;
      if (i >= n) continue;
      const float x = pow2i(sc[u] - 127);
      float v[8];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float2 f = __half22float2(e2m1x2_to_half2((c[u] >> (8 * k)) & 0xFFu));
        v[2 * k] = __fmul_rn(f.x, x);  // exact: an E2M1 value times a power of two
        v[2 * k + 1] = __fmul_rn(f.y, x);
      }
      if constexpr (OUT == kF32) {
        float4* p = reinterpret_cast<float4*>(static_cast<float*>(out) + i);
        __stcs(p, make_float4(v[0], v[1], v[2], v[3]));
        __stcs(p + 1, make_float4(v[4], v[5], v[6], v[7]));
      } else {
        const uint4 o = make_uint4(pack2_16<OUT>(v[0], v[1]), pack2_16<OUT>(v[2], v[3]),
                                   pack2_16<OUT>(v[4], v[5]), pack2_16<OUT>(v[6], v[7]));
        __stcs(reinterpret_cast<uint4*>(static_cast<unsigned short*>(out) + i), o);
      }
    }
  }
}

unsigned mx_grid(int64_t n) {
  const int64_t warps = (n + 256 * kMxUnroll - 1) / (256 * kMxUnroll);
  const int64_t blocks = (warps + kMxThreads / 32 - 1) / (kMxThreads / 32);
  return static_cast<unsigned>(blocks < 148 * 16 ? blocks : 148 * 16);
}

}  // namespace

cudaError_t launch_mxfp4_quantize(const void* W, int dtype, int64_t n, uint8_t* codes,
                                  uint8_t* scales, cudaStream_t stream) {
  if (n == 0) return cudaSuccess;
  const unsigned g = mx_grid(n);
  if (dtype == kF32)
    mxfp4_quantize_kernel<kF32><<<g, kMxThreads, 0, stream>>>(W, n, codes, scales);
  else if (dtype == kBF16)
    mxfp4_quantize_kernel<kBF16><<<g, kMxThreads, 0, stream>>>(W, n, codes, scales);
  else
    mxfp4_quantize_kernel<kF16><<<g, kMxThreads, 0, stream>>>(W, n, codes, scales);
  return cudaGetLastError();
}

cudaError_t launch_mxfp4_dequantize(const uint8_t* codes, const uint8_t* scales, int64_t n,
                                    int out_dtype, void* out, cudaStream_t stream) {
  if (n == 0) return cudaSuccess;
  const unsigned g = mx_grid(n);
  if (out_dtype == kF32)
    mxfp4_dequantize_kernel<kF32><<<g, kMxThreads, 0, stream>>>(codes, scales, n, out);
  else if (out_dtype == kBF16)
    mxfp4_dequantize_kernel<kBF16><<<g, kMxThreads, 0, stream>>>(codes, scales, n, out);
  else
    mxfp4_dequantize_kernel<kF16><<<g, kMxThreads, 0, stream>>>(codes, scales, n, out);
  return cudaGetLastError();
}

}  // namespace hqqk
