// hqq_device.cuh - device helpers shared by the quantize, dequantize and meta kernels of
// the B200 (sm_100a) HQQ library: dtype conversion, MUFU wrappers, rounding, packing.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "hqq_kernels.h"

namespace hqqk {

// 1.5 * 2^23: adding then subtracting it rounds an fp32 value |v| < 2^22 to the nearest
// integer, ties to even (the sum lands in [2^23, 2^24) where the spacing is 1). Both adds
// run on the FMA pipe, unlike a separate round instruction.
constexpr float kRoundMagic = 12582912.0f;

__device__ __forceinline__ float rint_magic(float v) {
  return __fsub_rn(__fadd_rn(v, kRoundMagic), kRoundMagic);
}

// MUFU base-2 logarithm / exponential (documented PTX approximations, ftz).
__device__ __forceinline__ float lg2_approx(float x) {
  float y;
  asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// fp32 pairs (sm_100 add/mul .f32x2: one instruction, two lanes, each lane rounded to
// nearest even exactly as the scalar operation), written as PTX with the explicit .rn
// modifier. Measured on sm_100a: the float2 intrinsics (__fmul2_rn feeding __fadd2_rn) were
// contracted into a fused multiply-add, one rounding instead of two, and so were these PTX
// forms inside a large unrolled loop. So an f32x2 product must never feed an f32x2 addition
// where the definition rounds both; callers keep such products scalar (__fmul_rn, which is
// never fused). A product feeding nothing but a multiplication or a special function is safe.
__device__ __forceinline__ float2 fadd2_rn(float2 a, float2 b) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "add.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return d;
}
__device__ __forceinline__ float2 fmul2_rn(float2 a, float2 b) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "mul.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return d;
}

// Exact fp32 -> fp64 widening built from the bit fields on the integer pipes (no conversion
// instruction, which would share the SFU pipe with lg2/ex2). Zero and subnormal inputs, which
// need renormalisation, take the conversion instruction.
__device__ __forceinline__ double f32_to_f64_exact(float x) {
  const uint32_t b = __float_as_uint(x);
  const uint32_t e = (b >> 23) & 0xffu;
  if (e == 0u || e == 0xffu) return (double)x;
  const uint32_t hi = (b & 0x80000000u) | ((e + 896u) << 20) | ((b >> 3) & 0x000fffffu);
  const uint32_t lo = b << 29;
  return __hiloint2double((int)hi, (int)lo);
}

// A non-negative integer below 2^23 held exactly in an fp32, widened to fp64 without a
// conversion instruction (2^52 + i built from bits, minus 2^52; both exact).
__device__ __forceinline__ double small_int_f32_to_f64(float x) {
  const uint32_t i = __float_as_uint(__fadd_rn(x, 8388608.0f)) - 0x4B000000u;
  return __dsub_rn(__hiloint2double(0x43300000, (int)i), 4503599627370496.0);
}

__device__ __forceinline__ float bf16_bits_to_f32(uint32_t h) { return __uint_as_float(h << 16); }
__device__ __forceinline__ float f16_bits_to_f32(uint32_t h) {
  return __half2float(__ushort_as_half((unsigned short)h));
}

// Load one element of dtype DT at index i as fp32 (exact upcast).
template <int DT>
__device__ __forceinline__ float load_elem(const void* p, int64_t i) {
  if constexpr (DT == kF32) {
    return __ldg(reinterpret_cast<const float*>(p) + i);
  } else {
    unsigned short h = __ldg(reinterpret_cast<const unsigned short*>(p) + i);
    return DT == kBF16 ? bf16_bits_to_f32(h) : f16_bits_to_f32(h);
  }
}

__device__ __forceinline__ float load_meta(const void* p, int dt, int64_t i) {
  if (dt == kF32) return reinterpret_cast<const float*>(p)[i];
  unsigned short h = reinterpret_cast<const unsigned short*>(p)[i];
  return dt == kBF16 ? bf16_bits_to_f32(h) : f16_bits_to_f32(h);
}

// Store an fp32 value rounded once (nearest even) to dtype dt.
__device__ __forceinline__ void store_meta(void* p, int dt, int64_t i, float v) {
  if (dt == kF32) {
    reinterpret_cast<float*>(p)[i] = v;
  } else if (dt == kBF16) {
    reinterpret_cast<__nv_bfloat16*>(p)[i] = __float2bfloat16_rn(v);
  } else {
    reinterpret_cast<__half*>(p)[i] = __float2half_rn(v);
  }
}

// Round two fp32 values to 16-bit storage and pack them (low half = a).
template <int DT>
__device__ __forceinline__ uint32_t pack2_16(float a, float b) {
  if constexpr (DT == kBF16) {
    __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&h);
  } else {
    __half2 h = __floats2half2_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&h);
  }
}

// Eight consecutive 4-bit codes (LSB-first in a little-endian word: code 2b in the low
// nibble of byte b, code 2b+1 in its high nibble) to eight dequantized 16-bit values of type
// OUT (kBF16 or kF16): (float(q) - zero) * scale with the dequantizer's three roundings. Each
// code becomes the float 2^23 + q by placing its byte under the exponent bits (0x4B000000);
// subtracting 2^23 is exact; q - zero is computed as q + (-zero) (identical rounding). The
// arithmetic runs on fp32 pairs (sm_100 FADD2/FMUL2: one instruction, two lanes, the same
// rounding as two scalar operations, fadd2_rn / fmul2_rn).
template <int OUT>
__device__ __forceinline__ uint4 dequant8_4bit(uint32_t w, float2 neg_zero, float2 scale) {
  const uint32_t lo = w & 0x0F0F0F0Fu, hi = (w >> 4) & 0x0F0F0F0Fu;
  const float2 neg_magic = make_float2(-8388608.0f, -8388608.0f);
  uint32_t o[4];
#pragma unroll
  for (int b = 0; b < 4; ++b) {
    const float2 m = make_float2(__uint_as_float(__byte_perm(lo, 0x4B000000u, 0x7540 + b)),
                                 __uint_as_float(__byte_perm(hi, 0x4B000000u, 0x7540 + b)));
    const float2 v = fmul2_rn(fadd2_rn(fadd2_rn(m, neg_magic), neg_zero), scale);
    o[b] = pack2_16<OUT>(v.x, v.y);
  }
  return make_uint4(o[0], o[1], o[2], o[3]);
}

}  // namespace hqqk
