// hqq_quantize_impl.cuh - the HQQ solver kernel and its launchers (templates). Included by
// hqq_quantize.cu (iterations run to the end) and hqq_quantize_stop.cu (iterations stop at a
// fixed point, HQQ_FLAG_STOP_AT_FIXED_POINT), so that each set compiles in its own unit and
// the unused option costs the other nothing (a runtime test inside the loop measured 8.7 %).
#pragma once

#include <math.h>

#include "hqq_device.cuh"
#include "hqq_kernels.h"

namespace hqqk {

// Threads per block: 160 (5 warps) for 3-bit codes, where 160*E codes per block must be a
// multiple of 10 so that 10-code words never straddle blocks; HQQ_QBLOCK (4 warps by default)
// otherwise, which with 128 registers a thread lets 16 warps share an SM instead of 15.
#ifndef HQQ_QBLOCK
#define HQQ_QBLOCK 128
#endif
template <bool PACK3>
__host__ __device__ constexpr int qblock() { return PACK3 ? 160 : HQQ_QBLOCK; }

// Tuning knobs (compile-time): minimum resident blocks per SM (0: the per-shape table
// min_blocks below; a positive value forces it for every shape), and whether to round with
// the hardware round instruction instead of the magic-number add.
#ifndef HQQ_MINB
#define HQQ_MINB 0
#endif
#ifndef HQQ_USE_FRND
#define HQQ_USE_FRND 0
#endif
// 1: keep the scaled weights Ws = w*s in registers; 0: recompute w*s at each use (fewer
// registers, one more FMA-pipe op per element and evaluation).
#ifndef HQQ_STORE_WS
#define HQQ_STORE_WS 1
#endif
// 1: run the per-element arithmetic of an evaluation on fp32 pairs (sm_100 FADD2/FMUL2: one
// issue slot for two elements, each lane rounded exactly as the scalar operation); 0: scalar.
#ifndef HQQ_PAIRED
#define HQQ_PAIRED 1
#endif
// 1: take the zero update's exact fp32 form when it applies (no shrinkage, |S_ws| not tiny);
// 0: always the fp64 form.
#ifndef HQQ_F32_UPDATE
#define HQQ_F32_UPDATE 1
#endif
// axis-0 group loader: 2 = per-warp shared-memory tiles filled with 16-byte loads (no block
// barrier), 1 = one tile per block (block barrier), 0 = each lane loads its column directly
// (2- or 4-byte loads, one per element). The tiles apply where the shape allows them.
#ifndef HQQ_AXIS0_TILE
#define HQQ_AXIS0_TILE 2
#endif

// Resident blocks per SM the register budget is sized for (measured on B200, every shape of
// the shipped workloads): with 32 elements per lane the raw and scaled weights take 48
// registers, and 128 registers a thread (no spills) ran faster than 96 or 72 (spills); with
// 16 or fewer elements per lane 96 registers fit without spills.
template <int G, int L, int BLOCK>
__host__ __device__ constexpr int min_blocks() {
  // 32-element lanes: 128 registers (15 or 16 warps an SM); fewer elements: 96 (20 warps)
  return HQQ_MINB > 0 ? HQQ_MINB : (G / L < 32 ? 640 : 512) / BLOCK;
}

__device__ __forceinline__ float round_even(float v) {
#if HQQ_USE_FRND
  return rintf(v);
#else
  return rint_magic(v);
#endif
}

// Shrinkage cut-offs of the updates: We = max(|r| - |r|^(p-1)/beta_k, 0) is nonzero only
// where |r|^(2-p) > 1/beta_k. cut[k] = (1/beta_k)^(1/(2-p)) * (1 - 1e-5) for update k, with
// beta_k and 1/beta_k formed by the same fp32 operations as the kernel's, evaluated on the host
// in fp64 and rounded down to fp32. Below cut[k] every rounded |r|^(p-1)/beta_k still exceeds
// |r| (the margin covers the power's, the product's and the difference's roundings), so We is
// exactly 0. Updates past the table use cut_min, the last update's cut-off (beta only grows,
// so it is the smallest), which also decides when a group can never shrink again.
constexpr int kCutTable = 64;
struct ShrinkCut {
  float cut[kCutTable];
  float cut_min;
};

struct QArgs {
  const void* W;
  int64_t rows, cols, n_groups;
  int nbits, iters;
  float qmax, p, beta0, kappa;
  uint8_t* packed;
  void* scale;
  void* zero;
  int scale_dtype, zero_dtype;
  int flags;  // bit 0: stop a warp's iterations once all its groups sit at a fixed point
};

template <int L>
__device__ __forceinline__ float group_sum(float x, unsigned m) {
#pragma unroll
  for (int o = 1; o < L; o <<= 1) x += __shfl_xor_sync(m, x, o);
  return x;
}
template <int L>
__device__ __forceinline__ double group_sum_d(double x, unsigned m) {
#pragma unroll
  for (int o = 1; o < L; o <<= 1) x += __shfl_xor_sync(m, x, o);
  return x;
}
template <int L>
__device__ __forceinline__ float group_min(float x, unsigned m) {
#pragma unroll
  for (int o = 1; o < L; o <<= 1) x = fminf(x, __shfl_xor_sync(m, x, o));
  return x;
}
template <int L>
__device__ __forceinline__ float group_max(float x, unsigned m) {
#pragma unroll
  for (int o = 1; o < L; o <<= 1) x = fmaxf(x, __shfl_xor_sync(m, x, o));
  return x;
}

// Flat index of element j (0..G) of group g.
template <int G, int AXIS>
__device__ __forceinline__ int64_t elem_index(const QArgs& a, int64_t g, int j) {
  if constexpr (AXIS == 1) {
    return g * G + j;  // cols is a multiple of G, so groups tile memory contiguously
  } else {
    int64_t rb = g / a.cols, c = g - rb * a.cols;
    return (rb * G + j) * a.cols + c;
  }
}

// A lane's E raw weights: fp32, or two 16-bit values per 32-bit register (low half first),
// widened to fp32 at each use (exact).
template <int WDT, int E>
struct WRaw {
  static constexpr bool kPacked = WDT != kF32;
  uint32_t u[kPacked ? E / 2 : E];
  __device__ __forceinline__ float get(int j) const {
    if constexpr (!kPacked) {
      return __uint_as_float(u[j]);
    } else {
      const uint32_t x = u[j >> 1];
      if constexpr (WDT == kBF16) {
        return (j & 1) ? __uint_as_float(x & 0xffff0000u) : __uint_as_float(x << 16);
      } else {
        return f16_bits_to_f32((j & 1) ? (x >> 16) : (x & 0xffffu));
      }
    }
  }
};

// Load this lane's E elements of group g (16-byte vector loads for axis=1; for axis=0 the
// lanes of a warp hold consecutive columns, so each row access is coalesced).
template <int G, int E, int AXIS, int WDT>
__device__ __forceinline__ void load_group(const QArgs& a, int64_t g, int lane, WRaw<WDT, E>& w) {
  constexpr int PER16 = WDT == kF32 ? 4 : 8;  // elements per 16-byte vector
  if constexpr (AXIS == 1) {
    const int64_t base = g * G + (int64_t)lane * E;
    const char* src = reinterpret_cast<const char*>(a.W) + base * (WDT == kF32 ? 4 : 2);
#pragma unroll
    for (int i = 0; i < E / PER16; ++i) {
      const uint4 v = __ldg(reinterpret_cast<const uint4*>(src) + i);
      w.u[4 * i] = v.x; w.u[4 * i + 1] = v.y; w.u[4 * i + 2] = v.z; w.u[4 * i + 3] = v.w;
    }
  } else {
    const int64_t rb = g / a.cols, c = g - rb * a.cols;
    const int64_t base = (rb * G + (int64_t)lane * E) * a.cols + c;
    if constexpr (WDT == kF32) {
      const uint32_t* src = reinterpret_cast<const uint32_t*>(a.W);
#pragma unroll
      for (int j = 0; j < E; ++j) w.u[j] = __ldg(src + base + (int64_t)j * a.cols);
    } else {
      const unsigned short* src = reinterpret_cast<const unsigned short*>(a.W);
#pragma unroll
      for (int i = 0; i < E / 2; ++i) {
        const uint32_t lo = __ldg(src + base + (int64_t)(2 * i) * a.cols);
        const uint32_t hi = __ldg(src + base + (int64_t)(2 * i + 1) * a.cols);
        w.u[i] = lo | (hi << 16);
      }
    }
  }
}

// axis 0 through shared memory: the block's NGB groups are NGB consecutive columns of one
// row block (or of two, where the tile wraps), each G elements down its column. The block
// reads the G element rows of the tile with 16-byte loads (consecutive threads take
// consecutive 16-byte pieces of a row: coalesced), stores them to shared memory as a
// [G][NGB] tile, and each lane then gathers its column's E elements from the tile.
// Requires every 16-byte piece to lie in one row block: cols and NGB multiples of the
// elements per 16 bytes (then n_groups and every tile start are too).
template <int WDT>
__host__ __device__ constexpr int elems_per_16B() { return WDT == kF32 ? 4 : 8; }

template <int G, int NGB, int WDT, int BLOCK>
__device__ __forceinline__ void load_tile_axis0(const QArgs& a, int64_t g0, unsigned char* s_tile) {
  constexpr int PERV = elems_per_16B<WDT>();
  constexpr int ESZ = WDT == kF32 ? 4 : 2;
  constexpr int CPR = NGB / PERV;  // 16-byte pieces per element row of the tile
  const char* W = reinterpret_cast<const char*>(a.W);
#pragma unroll 1
  for (int k = threadIdx.x; k < G * CPR; k += BLOCK) {
    const int j = k / CPR, i0 = (k - j * CPR) * PERV;
    const int64_t gg = g0 + i0;
    if (gg < a.n_groups) {
      const int64_t rb = gg / a.cols, c = gg - rb * a.cols;
      const uint4 v = __ldg(reinterpret_cast<const uint4*>(W + ((rb * G + j) * a.cols + c) * ESZ));
      *reinterpret_cast<uint4*>(s_tile + (j * NGB + i0) * ESZ) = v;
    }
  }
}

template <int G, int NGB, int E, int WDT>
__device__ __forceinline__ void gather_tile_axis0(const unsigned char* s_tile, int gi, int lane,
                                                  WRaw<WDT, E>& w) {
  if constexpr (WDT == kF32) {
    const uint32_t* t = reinterpret_cast<const uint32_t*>(s_tile);
#pragma unroll
    for (int j = 0; j < E; ++j) w.u[j] = t[(lane * E + j) * NGB + gi];
  } else {
    const unsigned short* t = reinterpret_cast<const unsigned short*>(s_tile);
#pragma unroll
    for (int i = 0; i < E / 2; ++i) {
      const uint32_t lo = t[(lane * E + 2 * i) * NGB + gi];
      const uint32_t hi = t[(lane * E + 2 * i + 1) * NGB + gi];
      w.u[i] = lo | (hi << 16);
    }
  }
}

// axis 0 through shared memory, one warp at a time: a warp's 32/L groups are 32/L consecutive
// columns of one row block (the tile start and 32/L are multiples of the elements per 16
// bytes, and so is cols). The warp reads the G element rows of its columns with 16-byte loads
// (32/L columns = 64/L bytes of a row: 4/L lanes per row, 8L rows per load instruction), stores
// them to its own shared-memory region and, after a warp barrier only, each lane gathers its
// E elements. Lane block l (rows l*E .. l*E+E-1) is stored after l spare rows, so that the L
// lanes of a group read from disjoint banks.
template <int G, int L, int WDT>
__device__ __forceinline__ void load_warp_tile_axis0(const QArgs& a, int64_t gw0, int wl,
                                                     unsigned char* s_w) {
  constexpr int PERV = elems_per_16B<WDT>();
  constexpr int ESZ = WDT == kF32 ? 4 : 2;
  constexpr int WG = 32 / L, E = G / L;
  constexpr int CPR = WG / PERV;  // 16-byte pieces per element row of the warp's columns
  const char* W = reinterpret_cast<const char*>(a.W);
#pragma unroll
  for (int k = wl; k < G * CPR; k += 32) {
    const int j = k / CPR, i0 = (k - j * CPR) * PERV;
    const int64_t gg = gw0 + i0;
    if (gg < a.n_groups) {
      const int64_t rb = gg / a.cols, c = gg - rb * a.cols;
      const uint4 v = __ldg(reinterpret_cast<const uint4*>(W + ((rb * G + j) * a.cols + c) * ESZ));
      *reinterpret_cast<uint4*>(s_w + ((j + j / E) * WG + i0) * ESZ) = v;
    }
  }
}

template <int G, int L, int WDT>
__device__ __forceinline__ void gather_warp_tile_axis0(const unsigned char* s_w, int gi, int lane,
                                                       WRaw<WDT, G / L>& w) {
  constexpr int WG = 32 / L, E = G / L;
  const int r0 = lane * E + lane;  // first stored row of this lane's block
  if constexpr (WDT == kF32) {
    const uint32_t* t = reinterpret_cast<const uint32_t*>(s_w);
#pragma unroll
    for (int j = 0; j < E; ++j) w.u[j] = t[(r0 + j) * WG + gi];
  } else {
    const unsigned short* t = reinterpret_cast<const unsigned short*>(s_w);
#pragma unroll
    for (int i = 0; i < E / 2; ++i) {
      const uint32_t lo = t[(r0 + 2 * i) * WG + gi];
      const uint32_t hi = t[(r0 + 2 * i + 1) * WG + gi];
      w.u[i] = lo | (hi << 16);
    }
  }
}

// Exact shrinkage sum over this lane's elements, recomputed from memory (rare path).
// `cut` is this update's cut-off with its rounding margin (ShrinkCut): elements whose
// residual is below it have We == 0 exactly and are skipped before the power.
template <int G, int E, int AXIS, int WDT>
__device__ __noinline__ double shrink_sum_exact(const QArgs& a, int64_t g, int lane, float s,
                                                float step, float z, float inv_beta,
                                                float cut) {
  const float slack = 1e-3f * (fabsf(z) + a.qmax + 1.0f);
  const float pm1 = a.p - 1.0f;
  double acc = 0.0;
#pragma unroll 1
  for (int j = 0; j < E; ++j) {
    const float w = load_elem<WDT>(a.W, elem_index<G, AXIS>(a, g, lane * E + j));
    const float v = __fadd_rn(__fmul_rn(w, s), z);
    const float q = fminf(fmaxf(rintf(v), 0.0f), a.qmax);
    const float d = __fsub_rn(v, q);
    if (step * (fabsf(d) * 1.001f + slack) < cut) continue;
    const float r = __fsub_rn(w, __fmul_rn(__fsub_rn(q, z), step));
    const float ar = fabsf(r);
    if (!(ar >= cut)) continue;  // below the cut-off (or zero): We == 0 exactly
    // |r|^(p-1) rounded once to fp32: the fp64 power, then one rounding (the correctly
    // rounded fp32 value except within a few fp64 ulps of an fp32 rounding boundary)
    const float t = __double2float_rn(pow((double)ar, (double)pm1));
    const float m = fmaxf(__fsub_rn(ar, __fmul_rn(t, inv_beta)), 0.0f);
    acc += (double)copysignf(m, r);
  }
  return acc;
}

// Store E codes of NB bits (NB in {1,2,4,8}) starting at code index code0.
template <int NB, int E>
__device__ __forceinline__ void store_codes(uint8_t* packed, int64_t code0, const uint32_t (&q)[E]) {
  constexpr int BITS = E * NB;
  uint8_t* dst = packed + code0 * NB / 8;
  if constexpr (BITS >= 32) {
    constexpr int NW = BITS / 32;
    uint32_t w[NW];
#pragma unroll
    for (int i = 0; i < NW; ++i) w[i] = 0;
#pragma unroll
    for (int j = 0; j < E; ++j) w[(j * NB) / 32] |= q[j] << ((j * NB) % 32);
    if constexpr (NW % 4 == 0) {
#pragma unroll
      for (int i = 0; i < NW / 4; ++i)
        reinterpret_cast<uint4*>(dst)[i] = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
    } else if constexpr (NW % 2 == 0) {
#pragma unroll
      for (int i = 0; i < NW / 2; ++i) reinterpret_cast<uint2*>(dst)[i] = make_uint2(w[2 * i], w[2 * i + 1]);
    } else {
      reinterpret_cast<uint32_t*>(dst)[0] = w[0];
    }
  } else {
    uint32_t w = 0;
#pragma unroll
    for (int j = 0; j < E; ++j) w |= q[j] << (j * NB);
    if constexpr (BITS == 16) {
      reinterpret_cast<unsigned short*>(dst)[0] = (unsigned short)w;
    } else {
      dst[0] = (uint8_t)w;
    }
  }
}

// One evaluation of candidate zero z over this lane's elements: the lp error (four
// partial sums) and the code sum.
template <int E, int WDT, bool CLAMP, bool P_ONE, bool TRACK>
__device__ __forceinline__ void evaluate(const float (&ws)[HQQ_STORE_WS ? E : 1],
                                         const WRaw<WDT, E>& w, float s,
                                         float z, float step, float qmax, float pp, float& e,
                                         float& sq, float& rmax) {
  float ea[4] = {0.f, 0.f, 0.f, 0.f};
  float qa[2] = {0.f, 0.f};
  float rm = 0.0f;
#pragma unroll
  for (int j = 0; j < E; ++j) {
    const float wsj = HQQ_STORE_WS ? ws[j] : __fmul_rn(w.get(j), s);
    const float v = __fadd_rn(wsj, z);
    const float q = round_even(CLAMP ? fminf(fmaxf(v, 0.0f), qmax) : v);
    const float r = __fsub_rn(w.get(j), __fmul_rn(__fsub_rn(q, z), step));
    const float term = P_ONE ? fabsf(r) : ex2_approx(__fmul_rn(pp, lg2_approx(fabsf(r))));
    ea[j & 3] = __fadd_rn(ea[j & 3], term);
    qa[j & 1] += q;
    if (TRACK) rm = fmaxf(rm, fabsf(r));
  }
  e = __fadd_rn(__fadd_rn(ea[0], ea[1]), __fadd_rn(ea[2], ea[3]));
  sq = qa[0] + qa[1];
  rmax = rm;
}

// The same evaluation on pairs of elements (j, j+1): the fp32 adds of the definition and the
// exponent product are lanes of add/mul.rn.f32x2, the residual's product is two scalar
// multiplies (see below), so every rounding is that of the scalar code;
// subtractions are additions of the negated operand (identical IEEE result), and
// w - (q - z)*step is formed as w + (q - z)*(-step) (the product's rounding is symmetric).
// The clamp, when needed, is applied per element before the rounding, as in the scalar path.
template <int E, int WDT, bool CLAMP, bool P_ONE, bool TRACK>
__device__ __forceinline__ void evaluate_paired(const float (&ws)[HQQ_STORE_WS ? E : 1],
                                                const WRaw<WDT, E>& w, float s, float z,
                                                float step, float qmax, float pp, float& e,
                                                float& sq, float& rmax) {
  static_assert(E % 2 == 0, "pairs of elements");
  const float2 z2 = make_float2(z, z), nz2 = make_float2(-z, -z);
  const float2 pp2 = make_float2(pp, pp);
  const float2 magic2 = make_float2(kRoundMagic, kRoundMagic);
  const float2 nmagic2 = make_float2(-kRoundMagic, -kRoundMagic);
  float2 ea[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
  float2 qa = make_float2(0.f, 0.f);
  float rm0 = 0.0f, rm1 = 0.0f;
#pragma unroll
  for (int j = 0; j < E; j += 2) {
    const float2 wsj = HQQ_STORE_WS ? make_float2(ws[j], ws[j + 1])
                                    : fmul2_rn(make_float2(w.get(j), w.get(j + 1)),
                                                 make_float2(s, s));
    float2 v = fadd2_rn(wsj, z2);
    if (CLAMP) v = make_float2(fminf(fmaxf(v.x, 0.0f), qmax), fminf(fmaxf(v.y, 0.0f), qmax));
#if HQQ_USE_FRND
    const float2 q = make_float2(rintf(v.x), rintf(v.y));
#else
    const float2 q = fadd2_rn(fadd2_rn(v, magic2), nmagic2);
#endif
    // the product stays two scalar multiplies: an f32x2 multiply feeding an f32x2 add was
    // fused into one multiply-add by the code generator (one rounding instead of two), even
    // with explicit .rn on both; __fmul_rn is never fused
    const float2 d = fadd2_rn(q, nz2);
    const float2 r = fadd2_rn(make_float2(w.get(j), w.get(j + 1)),
                              make_float2(__fmul_rn(d.x, -step), __fmul_rn(d.y, -step)));
    float2 term;
    if (P_ONE) {
      term = make_float2(fabsf(r.x), fabsf(r.y));
    } else {
      const float2 l = fmul2_rn(make_float2(lg2_approx(fabsf(r.x)), lg2_approx(fabsf(r.y))), pp2);
      term = make_float2(ex2_approx(l.x), ex2_approx(l.y));
    }
    ea[(j >> 1) & 1] = fadd2_rn(ea[(j >> 1) & 1], term);
    qa = fadd2_rn(qa, q);
    if (TRACK) {
      rm0 = fmaxf(rm0, fabsf(r.x));
      rm1 = fmaxf(rm1, fabsf(r.y));
    }
  }
  // ea[0] holds the partial sums of j = 0, 1 (mod 4), ea[1] those of j = 2, 3: combined in
  // the scalar path's order, so both variants return the same bits
  e = __fadd_rn(__fadd_rn(ea[0].x, ea[0].y), __fadd_rn(ea[1].x, ea[1].y));
  sq = qa.x + qa.y;
  rmax = fmaxf(rm0, rm1);
}

// One evaluation, dispatched on the warp-uniform flags to the compiled variants.
template <int E, int WDT, bool TRACK>
__device__ __forceinline__ void evaluate_any(const float (&ws)[HQQ_STORE_WS ? E : 1],
                                             const WRaw<WDT, E>& w, float s, float z, float step,
                                             float qmax, float pp, bool p_one, bool clamp,
                                             float& e, float& sq, float& rmax) {
  if constexpr (HQQ_PAIRED && E % 2 == 0) {
    if (p_one) {
      if (clamp) evaluate_paired<E, WDT, true, true, TRACK>(ws, w, s, z, step, qmax, pp, e, sq, rmax);
      else evaluate_paired<E, WDT, false, true, TRACK>(ws, w, s, z, step, qmax, pp, e, sq, rmax);
    } else {
      if (clamp) evaluate_paired<E, WDT, true, false, TRACK>(ws, w, s, z, step, qmax, pp, e, sq, rmax);
      else evaluate_paired<E, WDT, false, false, TRACK>(ws, w, s, z, step, qmax, pp, e, sq, rmax);
    }
  } else {
    if (p_one) {
      if (clamp) evaluate<E, WDT, true, true, TRACK>(ws, w, s, z, step, qmax, pp, e, sq, rmax);
      else evaluate<E, WDT, false, true, TRACK>(ws, w, s, z, step, qmax, pp, e, sq, rmax);
    } else {
      if (clamp) evaluate<E, WDT, true, false, TRACK>(ws, w, s, z, step, qmax, pp, e, sq, rmax);
      else evaluate<E, WDT, false, false, TRACK>(ws, w, s, z, step, qmax, pp, e, sq, rmax);
    }
  }
}

// The solver for the group this lane belongs to, from its raw weights in registers.
// Returns the group's final codes (this lane's E of them), step and best zero.
template <int G, int L, int AXIS, int WDT, bool STOP>
__device__ __forceinline__ void solve_group(const QArgs& a, int64_t g, int lane, unsigned gmask,
                                            unsigned wmask, const ShrinkCut& sc,
                                            const WRaw<WDT, G / L>& w, uint32_t (&q)[G / L],
                                            float& step_out, float& zbest_out) {
  constexpr int E = G / L;
  // ---- min/max round-to-nearest initialisation
  float mn = w.get(0), mx = w.get(0);
#pragma unroll
  for (int j = 1; j < E; ++j) {
    mn = fminf(mn, w.get(j));
    mx = fmaxf(mx, w.get(j));
  }
  if constexpr (L > 1) {
    mn = group_min<L>(mn, gmask);
    mx = group_max<L>(mx, gmask);
  }
  const float qmax = a.qmax;
  float s = 1.0f, step = 1.0f;
  if (mx > mn) {
    const float range = __fsub_rn(mx, mn);
    s = __fdiv_rn(qmax, range);
    step = __fdiv_rn(range, qmax);
  }
  const float z0 = __fmul_rn(-mn, s);
  float ws[HQQ_STORE_WS ? E : 1];  // scaled weights Ws = w*s, resident for all evaluations
  double acc = 0.0;
#pragma unroll
  for (int j = 0; j < E; ++j) {
    const float wsj = __fmul_rn(w.get(j), s);
    if constexpr (HQQ_STORE_WS) ws[j] = wsj;
    acc = __dadd_rn(acc, f32_to_f64_exact(wsj));
  }
  if constexpr (L > 1) acc = group_sum_d<L>(acc, gmask);
  const float S_ws_f = __double2float_rn(acc);  // rounded once to fp32
  // Without shrinkage (sum We = 0) the definition's update is fp32(fp64(sumQ - S_ws) / G).
  // sumQ is an integer below 2^16 and S_ws an fp32 value; when S_ws is 0 or |S_ws| >= 2^-12
  // both fit in 53 bits counted from the larger one's top bit down to S_ws's last bit, so the
  // fp64 difference is exact and the update equals one fp32 subtraction (the exact difference
  // rounded once) times the power of two 1/G (exact): no fp64 work on the common path.
  const bool f32_update_exact = S_ws_f == 0.0f || fabsf(S_ws_f) >= 0x1p-12f;
  const float wsmin = __fmul_rn(mn, s), wsmax = __fmul_rn(mx, s);

  // ---- iterations
  const float pp = a.p;
  const bool p_one = pp == 1.0f;  // |r|^1 needs no transcendental (and is then exact)
  float z = z0, zbest = z0, best = __int_as_float(0x7f800000), beta = a.beta0;
  for (int k = 0;; ++k) {
    // Codes stay inside [0, qmax] without clamping iff the group's extreme values do:
    // rint(v) >= 0 for v >= -0.5 and rint(v) <= qmax for v < qmax + 0.5.
    const bool inside = __fadd_rn(wsmin, z) >= -0.5f && __fadd_rn(wsmax, z) < qmax + 0.5f;
    const bool clamp = __any_sync(wmask, !inside);
    // Bound on max_j |r_j| at this zero: unclamped codes leave |v - Q| <= 1/2, clamped ones at
    // most the distance of the group's extreme scaled weight from the code range.
    const float hi = fmaxf(0.5f, fmaxf(-__fadd_rn(wsmin, z), __fsub_rn(__fadd_rn(wsmax, z), qmax)));
    const float bound = step * (hi * 1.001f + 1e-3f * (fabsf(z) + qmax + 1.0f));
    const float cutk = k < kCutTable ? sc.cut[k] : sc.cut_min;
    // A group whose bound reaches this update's cut-off has its largest residual measured
    // during the evaluation (warps with such a group run the tracking variant).
    const bool may_shrink = k < a.iters && !(bound < cutk);
    float e, sq, rmax;
    if (__any_sync(wmask, may_shrink))
      evaluate_any<E, WDT, true>(ws, w, s, z, step, qmax, pp, p_one, clamp, e, sq, rmax);
    else
      evaluate_any<E, WDT, false>(ws, w, s, z, step, qmax, pp, p_one, clamp, e, sq, rmax);
    if constexpr (L > 1) {
      e = group_sum<L>(e, gmask);
      sq = group_sum<L>(sq, gmask);
    }
    if (e < best) {
      best = e;
      zbest = z;
    }
    if (k == a.iters) break;

    // The exact shrinkage runs only where a residual reaches the cut-off (then it also skips
    // the elements below it); elsewhere every We is exactly 0.
    bool shrink = false;
    if (may_shrink) {
      if constexpr (L > 1) rmax = group_max<L>(rmax, gmask);
      shrink = !(rmax < cutk);
    }
    // Closed-form zero. Every lane computes it (a masked warp instruction costs the pipe as
    // much as a full one, so one lane computing and broadcasting would only add a shuffle).
    float znew;
    if (HQQ_F32_UPDATE && !shrink && f32_update_exact) {
      znew = __fmul_rn(__fsub_rn(sq, S_ws_f), 1.0f / (float)G);
    } else {
      // the definition's fp64 form z = fp32((sumQ - S_ws + s*sumWe) / G) (G = 2^k: the
      // division is exact), with the exact shrinkage sum where a residual reaches the cut-off
      double swe = 0.0;
      if (shrink) {
        swe = shrink_sum_exact<G, E, AXIS, WDT>(a, g, lane, s, step, z, __fdiv_rn(1.0f, beta),
                                                cutk);
        if constexpr (L > 1) swe = group_sum_d<L>(swe, gmask);
      }
      const double num = __dadd_rn(__dsub_rn(small_int_f32_to_f64(sq), (double)S_ws_f),
                                   __dmul_rn((double)s, swe));
      znew = __double2float_rn(__dmul_rn(num, 1.0 / (double)G));
    }
    beta = __fmul_rn(beta, a.kappa);
    if constexpr (STOP) {
      // Fixed point: same zero, and the bound is below every later update's cut-off, so
      // every remaining evaluation repeats this one exactly (same codes and error, never a
      // new best).
      const bool settled = bound < sc.cut_min && __float_as_uint(znew) == __float_as_uint(z);
      z = znew;
      if (__all_sync(wmask, settled)) break;
    } else {
      z = znew;
    }
  }

  // ---- final codes: the integer is read from the low mantissa bits of v + 1.5*2^23
#pragma unroll
  for (int j = 0; j < E; ++j) {
    const float wsj = HQQ_STORE_WS ? ws[j] : __fmul_rn(w.get(j), s);
    const float v = fminf(fmaxf(__fadd_rn(wsj, zbest), 0.0f), qmax);
    q[j] = __float_as_uint(__fadd_rn(v, kRoundMagic)) - 0x4B400000u;
  }
  step_out = step;
  zbest_out = zbest;
}

// A batch of matrices sharing one configuration, passed by value as kernel parameters
// (no device allocation): per-matrix pointers and shapes, and the prefix sums of their
// tile counts, so that a block finds its matrix with a binary search in parameter space.
template <int MAXB>
struct QBatch {
  QArgs c;                         // shared settings; pointers/shape fields unused
  ShrinkCut sc;                    // cut-offs of the updates (host-computed)
  int n;                           // matrices in this launch
  int64_t tile_start[MAXB + 1];    // tile_start[i] = first tile of matrix i
  const void* W[MAXB];
  int64_t cols[MAXB], n_groups[MAXB];
  uint8_t* packed[MAXB];
  void* scale[MAXB];
  void* zero[MAXB];
};

template <int MAXB>
__device__ __forceinline__ int find_matrix(const QBatch<MAXB>& b, int64_t tile) {
  int lo = 0, hi = b.n - 1;  // the last i with tile_start[i] <= tile
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (b.tile_start[mid] <= tile) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// One block solves a tile of NGB consecutive groups of one matrix. Blocks are short (tens of
// us) and many, so resident blocks sit at different phases and the MUFU stays fed through
// each block's load / min-max / packing phases (a persistent grid-stride variant, where all
// warps of an SM reach those phases together, measured 28 % slower).
template <int G, int L, int AXIS, int WDT, bool PACK3, int MAXB, bool STOP>
__global__ void __launch_bounds__(qblock<PACK3>(), min_blocks<G, L, qblock<PACK3>()>())
    quantize_kernel(const __grid_constant__ QBatch<MAXB> batch) {
  constexpr int kQBlock = qblock<PACK3>();
  constexpr int E = G / L;
  constexpr int NGB = kQBlock / L;  // groups per block
  __shared__ uint8_t s_codes[PACK3 ? NGB * G : 1];
  constexpr bool kTile = HQQ_AXIS0_TILE == 1 && AXIS == 0 && NGB % elems_per_16B<WDT>() == 0;
  constexpr bool kWTile =
      HQQ_AXIS0_TILE == 2 && AXIS == 0 && (32 / L) % elems_per_16B<WDT>() == 0;
  constexpr int kTileBytes = kTile ? G * NGB * (WDT == kF32 ? 4 : 2)
                             : kWTile ? (kQBlock / 32) * (G + L) * (32 / L) * (WDT == kF32 ? 4 : 2)
                                      : 16;
  __shared__ __align__(16) unsigned char s_tile[kTileBytes];

  const int mi = MAXB == 1 ? 0 : find_matrix(batch, (int64_t)blockIdx.x);
  const int64_t tile = (int64_t)blockIdx.x - batch.tile_start[mi];
  QArgs a = batch.c;
  a.W = batch.W[mi];
  a.cols = batch.cols[mi];
  a.n_groups = batch.n_groups[mi];
  a.packed = batch.packed[mi];
  a.scale = batch.scale[mi];
  a.zero = batch.zero[mi];

  const int tid = threadIdx.x;
  const int lane = tid % L;
  const int64_t g = tile * NGB + tid / L;
  const bool valid = g < a.n_groups;
  const unsigned wmask = __ballot_sync(0xffffffffu, valid);  // live lanes of this warp
  const unsigned gmask = L == 1 ? 0u : (((1u << L) - 1u) << ((tid & 31) & ~(L - 1)));

  // axis 0: the tile paths when every 16-byte piece stays in one row block (block-uniform)
  const bool tiled = (kTile || kWTile) && a.cols % elems_per_16B<WDT>() == 0;
  constexpr int kWRegion = (G + L) * (32 / L) * (WDT == kF32 ? 4 : 2);  // per warp
  unsigned char* s_w = s_tile + (tid / 32) * (kWTile ? kWRegion : 0);
  if (tiled) {
    if constexpr (kTile) {
      load_tile_axis0<G, NGB, WDT, kQBlock>(a, tile * NGB, s_tile);
      __syncthreads();
    } else if constexpr (kWTile) {
      load_warp_tile_axis0<G, L, WDT>(a, tile * NGB + (tid / 32) * (32 / L), tid & 31, s_w);
      __syncwarp();
    }
  }
  if (valid) {
    WRaw<WDT, E> w;  // raw weights, resident for all evaluations
    if (tiled) {
      if constexpr (kTile) gather_tile_axis0<G, NGB, E, WDT>(s_tile, tid / L, lane, w);
      if constexpr (kWTile) gather_warp_tile_axis0<G, L, WDT>(s_w, (tid & 31) / L, lane, w);
    } else {
      load_group<G, E, AXIS, WDT>(a, g, lane, w);
    }
    uint32_t q[E];
    float step, zbest;
    solve_group<G, L, AXIS, WDT, STOP>(a, g, lane, gmask, wmask, batch.sc, w, q, step, zbest);
    if (lane == 0) {
      store_meta(a.scale, a.scale_dtype, g, step);
      store_meta(a.zero, a.zero_dtype, g, zbest);
    }
    const int64_t code0 = g * G + (int64_t)lane * E;
    if constexpr (PACK3) {
      uint8_t* sc = s_codes + (tid / L) * G + lane * E;
#pragma unroll
      for (int j = 0; j < E; ++j) sc[j] = (uint8_t)q[j];
    } else {
      switch (a.nbits) {
        case 1: store_codes<1, E>(a.packed, code0, q); break;
        case 2: store_codes<2, E>(a.packed, code0, q); break;
        case 4: store_codes<4, E>(a.packed, code0, q); break;
        default: store_codes<8, E>(a.packed, code0, q); break;
      }
    }
  }

  if constexpr (PACK3) {
    // 10 codes of 3 bits per little-endian word; this block's codes start on a word.
    __syncthreads();
    const int64_t code_base = tile * NGB * G;
    const int64_t left = a.n_groups * G - code_base;
    const int n_valid = (int)(left < (int64_t)NGB * G ? left : (int64_t)NGB * G);
    const int n_words = (n_valid + 9) / 10;
    uint32_t* out = reinterpret_cast<uint32_t*>(a.packed) + code_base / 10;
    for (int wi = tid; wi < n_words; wi += kQBlock) {
      uint32_t word = 0;
#pragma unroll
      for (int i = 0; i < 10; ++i) {
        const int idx = wi * 10 + i;
        if (idx < n_valid) word |= (uint32_t)s_codes[idx] << (3 * i);
      }
      out[wi] = word;
    }
  }
}

#ifndef HQQ_G64_LANES
#define HQQ_G64_LANES 2
#endif

// Host side of ShrinkCut: beta_k and 1/beta_k by the kernel's fp32 operations (IEEE single
// precision, round to nearest, on the host too), the power in fp64, rounded down to fp32.
static void fill_cutoffs(int iters, float p, float beta0, float kappa, ShrinkCut* sc) {
  const double e = 1.0 / (2.0 - (double)p);
  float beta = beta0;
  float last = 0.0f;
  for (int k = 0; k < iters; ++k) {
    const float ib = 1.0f / beta;
    const double c = pow((double)ib, e) * (1.0 - 1e-5);
    float cf = (float)c;
    if ((double)cf > c) cf = nextafterf(cf, 0.0f);
    if (k < kCutTable) sc->cut[k] = cf;
    last = cf;
    beta = beta * kappa;
  }
  for (int k = iters < kCutTable ? iters : kCutTable; k < kCutTable; ++k) sc->cut[k] = last;
  sc->cut_min = last;
}

template <int MAXB>
static cudaError_t fill_batch(const QuantJob* jobs, int n, int ngb, QBatch<MAXB>* b,
                              int64_t* tiles_out) {
  const QuantJob& j0 = jobs[0];
  QArgs& c = b->c;
  c.W = nullptr;
  c.rows = c.cols = c.n_groups = 0;
  c.nbits = j0.nbits;
  c.iters = j0.iters;
  c.qmax = (float)((1 << j0.nbits) - 1);
  c.p = j0.p;
  c.beta0 = j0.beta0;
  c.kappa = j0.kappa;
  c.packed = nullptr;
  c.scale = c.zero = nullptr;
  c.scale_dtype = j0.scale_dtype;
  c.zero_dtype = j0.zero_dtype;
  c.flags = j0.flags;
  fill_cutoffs(j0.iters, j0.p, j0.beta0, j0.kappa, &b->sc);
  int64_t tiles = 0;
  int k = 0;
  for (int i = 0; i < n; ++i) {
    const QuantJob& j = jobs[i];
    if (j.n_groups == 0) continue;
    b->tile_start[k] = tiles;
    b->W[k] = j.W;
    b->cols[k] = j.cols;
    b->n_groups[k] = j.n_groups;
    b->packed[k] = j.packed;
    b->scale[k] = j.scale;
    b->zero[k] = j.zero;
    tiles += (j.n_groups + ngb - 1) / ngb;
    ++k;
  }
  b->tile_start[k] = tiles;
  b->n = k;
  *tiles_out = tiles;
  return tiles > 0x7fffffffLL ? cudaErrorInvalidValue : cudaSuccess;
}

template <int G, int L, int AXIS, int WDT, int MAXB, bool STOP>
static cudaError_t launch_g(const QuantJob* jobs, int n, cudaStream_t st) {
  const bool pack3 = jobs[0].nbits == 3;
  const int block = pack3 ? qblock<true>() : qblock<false>();
  QBatch<MAXB> b;
  int64_t tiles = 0;
  cudaError_t e = fill_batch<MAXB>(jobs, n, block / L, &b, &tiles);
  if (e != cudaSuccess) return e;
  if (tiles == 0) return cudaSuccess;
  if (pack3) {
    quantize_kernel<G, L, AXIS, WDT, true, MAXB, STOP><<<(unsigned)tiles, block, 0, st>>>(b);
  } else {
    quantize_kernel<G, L, AXIS, WDT, false, MAXB, STOP><<<(unsigned)tiles, block, 0, st>>>(b);
  }
  return cudaGetLastError();
}

template <int AXIS, int WDT, int MAXB, bool STOP>
static cudaError_t launch_axis_dt(const QuantJob* jobs, int n, cudaStream_t st) {
  switch (jobs[0].group_size) {
    case 8: return launch_g<8, 1, AXIS, WDT, MAXB, STOP>(jobs, n, st);
    case 16: return launch_g<16, 1, AXIS, WDT, MAXB, STOP>(jobs, n, st);
    case 32: return launch_g<32, 1, AXIS, WDT, MAXB, STOP>(jobs, n, st);
    case 64: return launch_g<64, HQQ_G64_LANES, AXIS, WDT, MAXB, STOP>(jobs, n, st);
    case 128: return launch_g<128, 2 * HQQ_G64_LANES, AXIS, WDT, MAXB, STOP>(jobs, n, st);
    case 256: return launch_g<256, 4 * HQQ_G64_LANES, AXIS, WDT, MAXB, STOP>(jobs, n, st);
    default: return cudaErrorInvalidValue;
  }
}

template <int MAXB, bool STOP>
static cudaError_t launch_batch(const QuantJob* jobs, int n, cudaStream_t st) {
  const QuantJob& j = jobs[0];
  if (j.axis == 1) {
    switch (j.w_dtype) {
      case kF16: return launch_axis_dt<1, kF16, MAXB, STOP>(jobs, n, st);
      case kBF16: return launch_axis_dt<1, kBF16, MAXB, STOP>(jobs, n, st);
      default: return launch_axis_dt<1, kF32, MAXB, STOP>(jobs, n, st);
    }
  }
  switch (j.w_dtype) {
    case kF16: return launch_axis_dt<0, kF16, MAXB, STOP>(jobs, n, st);
    case kBF16: return launch_axis_dt<0, kBF16, MAXB, STOP>(jobs, n, st);
    default: return launch_axis_dt<0, kF32, MAXB, STOP>(jobs, n, st);
  }
}

}  // namespace hqqk
