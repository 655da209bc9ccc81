// hqq_dequantize.cu - dequantization and second-level (8-bit meta) kernels for sm_100a.
//
// Dequantize ("HQQ calibration-free guide" (lnwmold.com) §3.2, dequantize(); "hqq-quantization
// skill summary" (nav.superapi.store), usage): W'[i] = (float(Q_i) - zero_g)*scale_g in fp32,
// two separate roundings, then one rounding to nearest even to the output dtype.
// With the second level ("HQQ tutorial" (devpress.csdn.net) §3.3, quant_scale/quant_zero),
// scale_g (zero_g) is first rebuilt in fp32 as (code - zero2)*step2 of its run.
//
// Layout on B200: HBM-bound (about 2.5 bytes per weight at 4 bits). A lane writes chunks of 8
// consecutive outputs with one 16-byte streaming store each (two for fp32), so a warp stores
// 512 contiguous bytes per instruction, and a warp issues the loads of several chunks before
// converting any. Codes become floats through the 2^23 mantissa trick and group indices
// through shifts, keeping the slow conversion/XU pipe and 64-bit division out of the
// per-element work. Kernels: dequant4_axis1_kernel (4 bits, plain meta, 16-bit output: the
// bench layout), dequant_axis1_kernel (every other axis-1 layout), dequant_axis0_cols_kernel
// (axis 0, groups of at most 64 bits, width a multiple of 8) and dequant_axis0_kernel (the
// remaining axis-0 layouts, element by element).
#include "hqq_device.cuh"
#include "hqq_kernels.h"

namespace hqqk {

constexpr int kDBlock = 256;

// Output stores are streaming (evict-first): the result is not read back by this pass.
template <typename T>
__device__ __forceinline__ void st_out(T* p, const T& v) {
  __stcs(p, v);
}

struct DArgs {
  const uint8_t* packed;
  const void* scale;
  const void* zero;
  const float* scale_mm;
  const float* zero_mm;
  int meta_group_size, meta_dtype;
  int log2_meta_group;    // log2(meta_group_size) when it is a power of two, else -1
  int64_t rows, cols, n;  // n = rows*cols
  int group_size, log2_group;
  void* out;
};

// A batch of matrices sharing one configuration, passed by value as kernel parameters (no
// device allocation): per-matrix pointers and shapes and the prefix sums of their tile
// counts; a block finds its matrix with a binary search in parameter space.
template <int MAXB>
struct DBatch {
  DArgs c;  // shared settings (meta dtype, run length, group size); pointer fields unused
  int n;
  int64_t tile_start[MAXB + 1];
  const uint8_t* packed[MAXB];
  const void* scale[MAXB];
  const void* zero[MAXB];
  const float* scale_mm[MAXB];
  const float* zero_mm[MAXB];
  int64_t rows[MAXB], cols[MAXB];
  void* out[MAXB];
};

template <int MAXB>
__device__ __forceinline__ DArgs batch_args(const DBatch<MAXB>& b, int64_t tile, int64_t* local) {
  int lo = 0, hi = b.n - 1;  // the last i with tile_start[i] <= tile
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (b.tile_start[mid] <= tile) lo = mid; else hi = mid - 1;
  }
  DArgs a = b.c;
  a.packed = b.packed[lo];
  a.scale = b.scale[lo];
  a.zero = b.zero[lo];
  a.scale_mm = b.scale_mm[lo];
  a.zero_mm = b.zero_mm[lo];
  a.rows = b.rows[lo];
  a.cols = b.cols[lo];
  a.n = a.rows * a.cols;
  a.out = b.out[lo];
  *local = tile - b.tile_start[lo];
  return a;
}

// The tiles of a persistent block. HQQ_DQ_ORDER 0: grid-stride order (tiles b, b + grid, ...),
// so that the resident blocks work on one contiguous band of the output at a time; 1: a
// contiguous range of ceil(total / grid) tiles per block. Either way a block's tile index only
// grows, so it finds its first matrix with one binary search and afterwards only steps forward
// over matrix boundaries (a search per tile cost as many instructions as the conversion of the
// tile's 32 elements per thread).
#ifndef HQQ_DQ_ORDER
#define HQQ_DQ_ORDER 0
#endif
template <int MAXB>
__device__ __forceinline__ DArgs matrix_args(const DBatch<MAXB>& b, int i) {
  DArgs a = b.c;
  a.packed = b.packed[i];
  a.scale = b.scale[i];
  a.zero = b.zero[i];
  a.scale_mm = b.scale_mm[i];
  a.zero_mm = b.zero_mm[i];
  a.rows = b.rows[i];
  a.cols = b.cols[i];
  a.n = a.rows * a.cols;
  a.out = b.out[i];
  return a;
}

// The cursor holds only the matrix index and its tile range; a tile's arguments are read from
// the parameter space when the tile starts (holding them across tiles cost up to 23 registers
// and occupancy in these memory-bound kernels).
template <int MAXB>
struct TileCursor {
  const DBatch<MAXB>& b;
  int64_t t, t_end, stride;  // next tile, end, step between a block's tiles
  int64_t mstart;            // first tile of the current matrix
  int64_t mend;              // first tile past the current matrix
  int mi;                    // current matrix

  __device__ explicit TileCursor(const DBatch<MAXB>& batch) : b(batch) {
    const int64_t total = b.tile_start[b.n];
    if (HQQ_DQ_ORDER == 0) {
      t = blockIdx.x;
      t_end = total;
      stride = gridDim.x;
    } else {
      const int64_t per = (total + gridDim.x - 1) / gridDim.x;
      t = (int64_t)blockIdx.x * per;
      t_end = t + per < total ? t + per : total;
      stride = 1;
    }
    mi = 0;
    if (t < t_end) {
      int lo = 0, hi = b.n - 1;  // the last i with tile_start[i] <= t
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (b.tile_start[mid] <= t) lo = mid; else hi = mid - 1;
      }
      mi = lo;
    }
    mstart = b.tile_start[mi];
    mend = b.tile_start[mi + 1];
  }
  // Moves to the block's next tile; false when there is none. *local = the tile's index
  // within its matrix, *matrix = the matrix.
  __device__ bool next(int64_t* local, int* matrix) {
    if (t >= t_end) return false;
    while (t >= mend) {  // empty matrices have no tiles
      ++mi;
      mstart = mend;
      mend = b.tile_start[mi + 1];
    }
    *local = t - mstart;
    *matrix = mi;
    t += stride;
    return true;
  }
};

// Small non-negative integer (< 2^23) to fp32 without a conversion instruction: OR it into
// the mantissa of 2^23 and subtract 2^23 (exact; stays on the FMA/ALU pipes).
__device__ __forceinline__ float u2f_small(uint32_t q) {
  return __fsub_rn(__uint_as_float(q | 0x4B000000u), 8388608.0f);
}

// Scale or zero of group g: stored directly, or as an 8-bit code of the second level
// decoded with its run's (step, zero) pair. The run index is a shift for power-of-two runs
// (a 64-bit division otherwise).
__device__ __forceinline__ float meta_value(const DArgs& a, const void* p, const float* mm,
                                            int64_t g) {
  if (mm) {
    const int64_t run = a.log2_meta_group >= 0 ? g >> a.log2_meta_group : g / a.meta_group_size;
    const float q = u2f_small(__ldg(reinterpret_cast<const uint8_t*>(p) + g));
    const float2 sz = __ldg(reinterpret_cast<const float2*>(mm) + run);
    return __fmul_rn(__fsub_rn(q, sz.y), sz.x);
  }
  return load_meta(p, a.meta_dtype, g);
}

// Code with stream index k (layout of the header).
template <int NB>
__device__ __forceinline__ uint32_t code_at(const uint8_t* packed, int64_t k) {
  if constexpr (NB == 3) {
    const uint32_t w = __ldg(reinterpret_cast<const uint32_t*>(packed) + k / 10);
    return (w >> (3 * (int)(k % 10))) & 7u;
  } else {
    constexpr int PER = 8 / NB;
    return (__ldg(packed + k / PER) >> ((int)(k % PER) * NB)) & ((1u << NB) - 1u);
  }
}

template <int OUT_DT>
__device__ __forceinline__ void store8(void* out, int64_t k0, const float (&v)[8]) {
  if constexpr (OUT_DT == kF32) {
    float4* dst = reinterpret_cast<float4*>(reinterpret_cast<float*>(out) + k0);
    st_out(dst, make_float4(v[0], v[1], v[2], v[3]));
    st_out(dst + 1, make_float4(v[4], v[5], v[6], v[7]));
  } else {
    uint4 u;
    u.x = pack2_16<OUT_DT>(v[0], v[1]);
    u.y = pack2_16<OUT_DT>(v[2], v[3]);
    u.z = pack2_16<OUT_DT>(v[4], v[5]);
    u.w = pack2_16<OUT_DT>(v[6], v[7]);
    st_out(reinterpret_cast<uint4*>(reinterpret_cast<unsigned short*>(out) + k0), u);
  }
}

template <int OUT_DT>
__device__ __forceinline__ void store1(void* out, int64_t k, float v) {
  store_meta(out, OUT_DT, k, v);
}

// axis=1: 8 consecutive elements share one group and have consecutive codes. A warp covers
// 256 consecutive elements per chunk (lane l: elements 8l .. 8l+7: their codes in one load of
// 1..8 bytes, or two 32-bit words for 3 bits, their group's meta, one 16- or 32-byte store),
// kD1Unroll chunks per warp per tile with every load of the tile issued before any conversion.
// Any nbits, plain or second-level meta, any output type. A tile (kDTile1 elements, a multiple
// of every group size) starts on a group and on a byte of the code stream, so its 64-bit
// bases are formed once and the per-chunk index work is 32-bit.
#ifndef HQQ_DQ1_UNROLL
#define HQQ_DQ1_UNROLL 4
#endif
constexpr int kD1Unroll = HQQ_DQ1_UNROLL;
constexpr int kDTile1 = kDBlock * 8 * kD1Unroll;

// The 8 codes of a lane as one bit field, code j in bits NB*j .. NB*j+NB-1. `tile_codes`
// points at the tile's first code byte (for 3 bits: `words` at the 32-bit word holding the
// tile's first code, whose slot is r0); li is the lane's first element within the tile.
template <int NB>
__device__ __forceinline__ uint64_t codes8_field(const uint8_t* tile_codes, const uint32_t* words,
                                                 int r0, int li) {
  if constexpr (NB == 3) {
    // 10 codes per 32-bit word (bits 30..31 unused): join the two words the 8 codes can
    // span into 60 contiguous bits, then drop the slots before the lane's first code.
    const uint32_t k = (uint32_t)(r0 + li);
    const uint32_t w = k / 10u, off = k - 10u * w;
    const uint32_t lo = __ldg(words + w);
    const uint32_t hi = off >= 3u ? __ldg(words + w + 1) : 0u;  // code 8 is in the next word
    return (((uint64_t)hi << 30) | (lo & 0x3FFFFFFFu)) >> (3u * off);
  } else if constexpr (NB == 8) {
    const uint2 v = __ldg(reinterpret_cast<const uint2*>(tile_codes + li));
    return (uint64_t)v.x | ((uint64_t)v.y << 32);
  } else if constexpr (NB == 4) {
    return __ldg(reinterpret_cast<const uint32_t*>(tile_codes + li / 2));
  } else if constexpr (NB == 2) {
    return __ldg(reinterpret_cast<const unsigned short*>(tile_codes + li / 4));
  } else {
    return __ldg(tile_codes + li / 8);
  }
}

// Code j of a field as the fp32 bit pattern 2^23 + code (the exact value 2^23 + code).
template <int NB>
__device__ __forceinline__ float code_magic(uint64_t field, int j) {
  if constexpr (NB == 8) {
    const uint32_t w = j < 4 ? (uint32_t)field : (uint32_t)(field >> 32);
    return __uint_as_float(__byte_perm(w, 0x4B000000u, 0x7540 + (j & 3)));
  } else {
    return __uint_as_float(((uint32_t)(field >> (NB * j)) & ((1u << NB) - 1u)) | 0x4B000000u);
  }
}

// META 1: scale and zero both second-level 8-bit codes in runs of a power-of-two length (the
// quant_scale + quant_zero layout): the tile's code and run bases are formed once and a chunk's
// group and run are 32-bit offsets from them (the per-chunk 64-bit index work and the meta-kind
// branches were most of this kernel's integer instructions, which bound it). META 0: any meta.
template <int NB, int OUT_DT, int MAXB, int META>
__global__ void __launch_bounds__(kDBlock) dequant_axis1_kernel(
    const __grid_constant__ DBatch<MAXB> batch) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const float2 neg_magic = make_float2(-8388608.0f, -8388608.0f);
  TileCursor<MAXB> cur(batch);
  int64_t local;
  int mi;
  while (cur.next(&local, &mi)) {
    const DArgs a = matrix_args(batch, mi);
    const int64_t e0 = local * kDTile1;  // the tile's first element
    const int64_t left = a.n - e0;
    const int rem = left < kDTile1 ? (int)left : kDTile1;
    const uint8_t* tile_codes = a.packed + (NB == 3 ? 0 : e0 / 8 * NB);
    const int64_t w0 = NB == 3 ? e0 / 10 : 0;
    const int r0 = NB == 3 ? (int)(e0 - 10 * w0) : 0;
    const uint32_t* words = reinterpret_cast<const uint32_t*>(a.packed) + w0;
    const int64_t g0 = e0 >> a.log2_group;
    const int lane0 = warp * (kD1Unroll * 256) + lane * 8;
    // META 1: this tile's 8-bit codes from group g0, its runs from run g0 >> L (rem0 groups in)
    const uint8_t* qs = static_cast<const uint8_t*>(a.scale) + g0;
    const uint8_t* qz = static_cast<const uint8_t*>(a.zero) + g0;
    const int L = a.log2_meta_group;
    const int64_t run0 = META ? g0 >> L : 0;
    const int rem0 = META ? static_cast<int>(g0 - (run0 << L)) : 0;
    const float2* ms = reinterpret_cast<const float2*>(a.scale_mm) + run0;
    const float2* mz = reinterpret_cast<const float2*>(a.zero_mm) + run0;
    uint64_t field[kD1Unroll];
    float sc[kD1Unroll], zr[kD1Unroll];
#pragma unroll
    for (int u = 0; u < kD1Unroll; ++u) {
      const int li = lane0 + u * 256;
      if (li < rem) {  // n and G are multiples of 8: a lane's 8 elements share one group
        field[u] = codes8_field<NB>(tile_codes, words, r0, li);
        if constexpr (META == 1) {
          // meta_value's arithmetic: (code - zero2) * step2 of the group's run
          const int gi = li >> a.log2_group;
          const int ri = (rem0 + gi) >> L;
          const float2 s2 = __ldg(ms + ri), z2 = __ldg(mz + ri);
          sc[u] = __fmul_rn(__fsub_rn(u2f_small(__ldg(qs + gi)), s2.y), s2.x);
          zr[u] = __fmul_rn(__fsub_rn(u2f_small(__ldg(qz + gi)), z2.y), z2.x);
        } else {
          const int64_t g = g0 + (li >> a.log2_group);
          sc[u] = meta_value(a, a.scale, a.scale_mm, g);
          zr[u] = meta_value(a, a.zero, a.zero_mm, g);
        }
      }
    }
#pragma unroll
    for (int u = 0; u < kD1Unroll; ++u) {
      const int li = lane0 + u * 256;
      if (li < rem) {
        // (code - zero) * scale, each operation rounded once as in the scalar form: the
        // subtraction of 2^23 is exact, x - z equals x + (-z), and the pair instructions
        // round each lane like the scalar ones
        const float2 nz = make_float2(-zr[u], -zr[u]), s2 = make_float2(sc[u], sc[u]);
        float v[8];
#pragma unroll
        for (int j = 0; j < 8; j += 2) {
          const float2 m = make_float2(code_magic<NB>(field[u], j), code_magic<NB>(field[u], j + 1));
          const float2 r = fmul2_rn(fadd2_rn(fadd2_rn(m, neg_magic), nz), s2);
          v[j] = r.x;
          v[j + 1] = r.y;
        }
        store8<OUT_DT>(a.out, e0 + li, v);
      }
    }
  }
}

// 4-bit codes, plain (not second-level) meta, 16-bit output - the layout every bench step
// and the linear layer use. A warp covers 256 consecutive elements per chunk (lane l: elements
// 8l .. 8l+7, one 32-bit code load, one 16-byte store), kD4Unroll chunks per warp per tile;
// all of a tile's loads are issued before any conversion, which keeps more bytes in flight
// than the generic kernel's two 8-element chunks per thread.
constexpr int kD4Unroll = 4;
constexpr int64_t kDTile4 = (int64_t)kDBlock * 8 * kD4Unroll;

template <int OUT_DT, int MAXB>
__global__ void __launch_bounds__(kDBlock) dequant4_axis1_kernel(
    const __grid_constant__ DBatch<MAXB> batch) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  TileCursor<MAXB> cur(batch);
  int64_t local;
  int mi;
  while (cur.next(&local, &mi)) {
    const DArgs a = matrix_args(batch, mi);
    const int64_t base = local * kDTile4 + (int64_t)warp * (kD4Unroll * 256) + lane * 8;
    uint32_t w[kD4Unroll];
    float sc[kD4Unroll], zr[kD4Unroll];
#pragma unroll
    for (int u = 0; u < kD4Unroll; ++u) {
      const int64_t i = base + u * 256;
      if (i < a.n) {  // n and G are multiples of 8: a lane's 8 elements share one group
        w[u] = __ldcs(reinterpret_cast<const unsigned int*>(a.packed + i / 2));
        const int64_t g = i >> a.log2_group;
        sc[u] = load_meta(a.scale, a.meta_dtype, g);
        zr[u] = load_meta(a.zero, a.meta_dtype, g);
      }
    }
#pragma unroll
    for (int u = 0; u < kD4Unroll; ++u) {
      const int64_t i = base + u * 256;
      if (i < a.n)
        st_out(reinterpret_cast<uint4*>(reinterpret_cast<unsigned short*>(a.out) + i),
               dequant8_4bit<OUT_DT>(w[u], make_float2(-zr[u], -zr[u]),
                                     make_float2(sc[u], sc[u])));
    }
  }
}

// axis=0 (groups run down columns): element (r, c) is code j = r % G of group
// g = (r / G)*cols + c. Rows with cols % 8 == 0 take 8 columns per thread; a block covers
// one tile of kDBlock*8 elements of one matrix.
constexpr int64_t kDTile0 = (int64_t)kDBlock * 8;

template <int NB, int OUT_DT, int MAXB>
__global__ void __launch_bounds__(kDBlock)
    dequant_axis0_kernel(const __grid_constant__ DBatch<MAXB> batch) {
  int64_t local;
  const DArgs a = batch_args(batch, (int64_t)blockIdx.x, &local);
  const int64_t k0 = (local * kDBlock + threadIdx.x) * 8;
  if (k0 >= a.n) return;
  const int G = a.group_size;
  if ((a.cols & 7) == 0) {
    const int64_t r = k0 / a.cols, c0 = k0 - r * a.cols;
    const int64_t rb = r >> a.log2_group;
    const int j = (int)(r - (rb << a.log2_group));
    float v[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int64_t g = rb * a.cols + c0 + i;
      const float sc = meta_value(a, a.scale, a.scale_mm, g);
      const float zr = meta_value(a, a.zero, a.zero_mm, g);
      const float q = u2f_small(code_at<NB>(a.packed, (g << a.log2_group) + j));
      v[i] = __fmul_rn(__fsub_rn(q, zr), sc);
    }
    store8<OUT_DT>(a.out, k0, v);
    return;
  }
  const int64_t kend = k0 + 8 < a.n ? k0 + 8 : a.n;
  for (int64_t k = k0; k < kend; ++k) {
    const int64_t r = k / a.cols, c = k - r * a.cols;
    const int64_t rb = r / G;
    const int j = (int)(r - rb * G);
    const int64_t g = rb * a.cols + c;
    const float sc = meta_value(a, a.scale, a.scale_mm, g);
    const float zr = meta_value(a, a.zero, a.zero_mm, g);
    const float q = u2f_small(code_at<NB>(a.packed, g * G + j));
    store1<OUT_DT>(a.out, k, __fmul_rn(__fsub_rn(q, zr), sc));
  }
}

// axis=0 with small groups (G*NB <= 64 bits) and a 16-bit output: a group is one column's G
// consecutive rows and its G*NB bits are contiguous in the stream, so a lane takes 8 adjacent
// columns of one row block, loads their 8 groups' codes (8*G*NB/8 bytes, one to four 16-byte
// loads) and meta once, and writes one 16-byte run per row of the block: a warp (256 columns)
// writes 512 contiguous bytes per row. Work unit = (row block, 256 columns), one per warp.
constexpr int kD0Cols = 256;  // columns per warp unit

template <int NB, int G, int OUT_DT, int MAXB>
__global__ void __launch_bounds__(kDBlock) dequant_axis0_cols_kernel(
    const __grid_constant__ DBatch<MAXB> batch) {
  constexpr int kBg = G * NB / 8;  // bytes per group: 1, 2, 4 or 8
  constexpr int kWords = 2 * kBg;  // 8 groups
  static_assert(kBg == 1 || kBg == 2 || kBg == 4 || kBg == 8, "group bytes");
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  TileCursor<MAXB> cur(batch);
  int64_t local;
  int mi;
  while (cur.next(&local, &mi)) {
    const DArgs a = matrix_args(batch, mi);
    const int64_t cunits = (a.cols + kD0Cols - 1) / kD0Cols;
    const int64_t unit = local * (kDBlock / 32) + warp;
    const int64_t rb = unit / cunits;
    if (rb >= a.rows / G) continue;
    const int64_t c0 = (unit - rb * cunits) * kD0Cols + lane * 8;
    if (c0 >= a.cols) continue;  // cols % 8 == 0 on this path: 8 columns are all in or out
    const int64_t g0 = rb * a.cols + c0;
    const uint8_t* src = a.packed + g0 * kBg;  // 8 consecutive groups, 8*kBg-byte aligned
    uint32_t wd[kWords];
    if constexpr (kBg == 1) {
      const uint2 v = __ldg(reinterpret_cast<const uint2*>(src));
      wd[0] = v.x;
      wd[1] = v.y;
    } else {
#pragma unroll
      for (int q = 0; q < kWords / 4; ++q) {
        const uint4 v = __ldg(reinterpret_cast<const uint4*>(src) + q);
        wd[4 * q] = v.x;
        wd[4 * q + 1] = v.y;
        wd[4 * q + 2] = v.z;
        wd[4 * q + 3] = v.w;
      }
    }
    // group i's G*NB bits (stream bits i*G*NB ..) in one 64-bit register, compile-time indices
    uint64_t gw[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      if constexpr (kBg == 8)
        gw[i] = static_cast<uint64_t>(wd[2 * i]) | (static_cast<uint64_t>(wd[2 * i + 1]) << 32);
      else
        gw[i] = (wd[i * kBg / 4] >> (8 * ((i * kBg) % 4))) & ((1ull << (8 * kBg)) - 1ull);
    }
    float sc[8], nz[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      sc[i] = meta_value(a, a.scale, a.scale_mm, g0 + i);
      nz[i] = -meta_value(a, a.zero, a.zero_mm, g0 + i);
    }
#pragma unroll 4
    for (int j = 0; j < G; ++j) {
      float v[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const uint32_t q = static_cast<uint32_t>(gw[i] >> (j * NB)) & ((1u << NB) - 1u);
        v[i] = __fmul_rn(__fadd_rn(u2f_small(q), nz[i]), sc[i]);
      }
      store8<OUT_DT>(a.out, (rb * G + j) * a.cols + c0, v);
    }
  }
}

// SMs x resident blocks per SM of `kernel` on the current device (host-side query).
template <typename K>
static cudaError_t resident_blocks(K kernel, int* out) {
  int dev = 0, sms = 0, per_sm = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e == cudaSuccess) e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, kDBlock, 0);
  *out = sms * (per_sm > 0 ? per_sm : 1);
  return e;
}

template <int MAXB>
static void fill_dbatch(const DequantJob* jobs, int n, int64_t tile_elems, DBatch<MAXB>* b) {
  const DequantJob& j0 = jobs[0];
  DArgs& c = b->c;
  c.packed = nullptr;
  c.scale = c.zero = nullptr;
  c.scale_mm = c.zero_mm = nullptr;
  c.meta_group_size = j0.meta_group_size > 0 ? j0.meta_group_size : 1;
  c.meta_dtype = j0.meta_dtype;
  c.log2_meta_group = -1;
  for (int l = 0; l < 31; ++l)
    if ((1 << l) == c.meta_group_size) c.log2_meta_group = l;
  c.rows = c.cols = c.n = 0;
  c.group_size = j0.group_size;
  c.log2_group = 0;
  while ((1 << c.log2_group) < j0.group_size) ++c.log2_group;
  c.out = nullptr;
  int64_t tiles = 0;
  int k = 0;
  for (int i = 0; i < n; ++i) {
    const DequantJob& j = jobs[i];
    const int64_t elems = j.rows * j.cols;
    if (elems == 0) continue;
    b->tile_start[k] = tiles;
    b->packed[k] = j.packed;
    b->scale[k] = j.scale;
    b->zero[k] = j.zero;
    b->scale_mm[k] = j.scale_mm;
    b->zero_mm[k] = j.zero_mm;
    b->rows[k] = j.rows;
    b->cols[k] = j.cols;
    b->out[k] = j.out;
    tiles += (elems + tile_elems - 1) / tile_elems;
    ++k;
  }
  b->tile_start[k] = tiles;
  b->n = k;
}

// The axis-0 column kernel for groups of G (G >= 8; G * NB <= 64 bits); tiles count its warp
// units (row block, 256 columns), kDBlock / 32 per block.
template <int NB, int G, int OUT_DT, int MAXB>
static cudaError_t launch_axis0_cols(const DequantJob* jobs, int n, cudaStream_t st) {
  if constexpr (G < 8) {
    return cudaErrorNotSupported;
  } else {
    DBatch<MAXB> b;
    fill_dbatch<MAXB>(jobs, n, kDTile0, &b);
    int64_t tiles = 0;
    for (int k = 0; k < b.n; ++k) {
      b.tile_start[k] = tiles;
      const int64_t units = (b.rows[k] / G) * ((b.cols[k] + kD0Cols - 1) / kD0Cols);
      tiles += (units + kDBlock / 32 - 1) / (kDBlock / 32);
    }
    b.tile_start[b.n] = tiles;
    if (tiles == 0) return cudaSuccess;
    int resident = 0;
    const cudaError_t e = resident_blocks(dequant_axis0_cols_kernel<NB, G, OUT_DT, MAXB>, &resident);
    if (e != cudaSuccess) return e;
    const int64_t blocks = tiles < resident ? tiles : resident;
    dequant_axis0_cols_kernel<NB, G, OUT_DT, MAXB><<<(unsigned)blocks, kDBlock, 0, st>>>(b);
    return cudaGetLastError();
  }
}

template <int NB, int OUT_DT, int MAXB>
static cudaError_t launch_nb_dt(const DequantJob* jobs, int n, cudaStream_t st) {
  DBatch<MAXB> b;
  if constexpr (NB == 4 && OUT_DT != kF32) {
    bool plain_meta = jobs[0].axis == 1;
    for (int i = 0; i < n; ++i) plain_meta = plain_meta && !jobs[i].scale_mm && !jobs[i].zero_mm;
    if (plain_meta) {
      fill_dbatch<MAXB>(jobs, n, kDTile4, &b);
      const int64_t tiles = b.tile_start[b.n];
      if (tiles == 0) return cudaSuccess;
      int resident = 0;
      const cudaError_t e = resident_blocks(dequant4_axis1_kernel<OUT_DT, MAXB>, &resident);
      if (e != cudaSuccess) return e;
      const int64_t blocks = tiles < resident ? tiles : resident;
      dequant4_axis1_kernel<OUT_DT, MAXB><<<(unsigned)blocks, kDBlock, 0, st>>>(b);
      return cudaGetLastError();
    }
  }
  if (jobs[0].axis == 1) {
    fill_dbatch<MAXB>(jobs, n, kDTile1, &b);
    const int64_t tiles = b.tile_start[b.n];
    if (tiles == 0) return cudaSuccess;
    bool both_runs = b.c.log2_meta_group >= 0;  // every matrix: 8-bit scale and zero
    for (int i = 0; i < n; ++i) both_runs = both_runs && jobs[i].scale_mm && jobs[i].zero_mm;
    int resident = 0;
    cudaError_t e = both_runs
                        ? resident_blocks(dequant_axis1_kernel<NB, OUT_DT, MAXB, 1>, &resident)
                        : resident_blocks(dequant_axis1_kernel<NB, OUT_DT, MAXB, 0>, &resident);
    if (e != cudaSuccess) return e;
    const int64_t blocks = tiles < resident ? tiles : resident;
    if (both_runs)
      dequant_axis1_kernel<NB, OUT_DT, MAXB, 1><<<(unsigned)blocks, kDBlock, 0, st>>>(b);
    else
      dequant_axis1_kernel<NB, OUT_DT, MAXB, 0><<<(unsigned)blocks, kDBlock, 0, st>>>(b);
  } else {
    if constexpr (OUT_DT != kF32 && NB != 3) {
      bool cols8 = true;
      for (int i = 0; i < n; ++i) cols8 = cols8 && jobs[i].cols % 8 == 0;
      const int G = jobs[0].group_size;
      cudaError_t e = cudaErrorNotSupported;
      if (cols8) {
        if (NB * G == 16) e = launch_axis0_cols<NB, 16 / NB, OUT_DT, MAXB>(jobs, n, st);
        else if (NB * G == 32) e = launch_axis0_cols<NB, 32 / NB, OUT_DT, MAXB>(jobs, n, st);
        else if (NB * G == 64) e = launch_axis0_cols<NB, 64 / NB, OUT_DT, MAXB>(jobs, n, st);
        else if (NB * G == 8) e = launch_axis0_cols<NB, 8 / NB, OUT_DT, MAXB>(jobs, n, st);
      }
      if (e != cudaErrorNotSupported) return e;
    }
    fill_dbatch<MAXB>(jobs, n, kDTile0, &b);
    const int64_t tiles = b.tile_start[b.n];
    if (tiles == 0) return cudaSuccess;
    if (tiles > 0x7fffffffLL) return cudaErrorInvalidValue;
    dequant_axis0_kernel<NB, OUT_DT, MAXB><<<(unsigned)tiles, kDBlock, 0, st>>>(b);
  }
  return cudaGetLastError();
}

template <int OUT_DT, int MAXB>
static cudaError_t launch_dt(const DequantJob* jobs, int n, cudaStream_t st) {
  switch (jobs[0].nbits) {
    case 1: return launch_nb_dt<1, OUT_DT, MAXB>(jobs, n, st);
    case 2: return launch_nb_dt<2, OUT_DT, MAXB>(jobs, n, st);
    case 3: return launch_nb_dt<3, OUT_DT, MAXB>(jobs, n, st);
    case 4: return launch_nb_dt<4, OUT_DT, MAXB>(jobs, n, st);
    default: return launch_nb_dt<8, OUT_DT, MAXB>(jobs, n, st);
  }
}

template <int MAXB>
static cudaError_t launch_dq(const DequantJob* jobs, int n, cudaStream_t st) {
  switch (jobs[0].out_dtype) {
    case kF16: return launch_dt<kF16, MAXB>(jobs, n, st);
    case kBF16: return launch_dt<kBF16, MAXB>(jobs, n, st);
    default: return launch_dt<kF32, MAXB>(jobs, n, st);
  }
}

cudaError_t launch_dequantize(const DequantJob& j, cudaStream_t st) {
  return launch_dq<1>(&j, 1, st);
}

cudaError_t launch_dequantize_batched(const DequantJob* jobs, int n, cudaStream_t st) {
  for (int i = 0; i < n; i += kMaxBatch) {
    const int k = n - i < kMaxBatch ? n - i : kMaxBatch;
    const cudaError_t e = launch_dq<kMaxBatch>(jobs + i, k, st);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

// ------------------------------------------------------------------ second level

// One warp per run of `group` values: min/max, step2/zero2, 8-bit codes
// ("HQQ tutorial" (devpress.csdn.net) §3.3; round-to-nearest only, no solver).
__global__ void __launch_bounds__(256) quantize_meta_kernel(const void* meta, int dt, int64_t n,
                                                            int group, uint8_t* q, float* mm) {
  const int64_t run = ((int64_t)blockIdx.x * 256 + threadIdx.x) / 32;
  const int lane = threadIdx.x & 31;
  const int64_t runs = (n + group - 1) / group;
  if (run >= runs) return;
  const int64_t b = run * group;
  const int64_t e = b + group < n ? b + group : n;
  float mn = __int_as_float(0x7f800000), mx = -mn;
  for (int64_t k = b + lane; k < e; k += 32) {
    const float v = load_meta(meta, dt, k);
    mn = fminf(mn, v);
    mx = fmaxf(mx, v);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  }
  float s2 = 1.0f, st2 = 1.0f;
  if (mx > mn) {
    const float range = __fsub_rn(mx, mn);
    s2 = __fdiv_rn(255.0f, range);
    st2 = __fdiv_rn(range, 255.0f);
  }
  const float z2 = __fmul_rn(-mn, s2);
  for (int64_t k = b + lane; k < e; k += 32) {
    const float v = __fadd_rn(__fmul_rn(load_meta(meta, dt, k), s2), z2);
    q[k] = (uint8_t)(__float_as_uint(__fadd_rn(fminf(fmaxf(v, 0.0f), 255.0f), kRoundMagic)) -
                     0x4B400000u);
  }
  if (lane == 0) {
    mm[2 * run] = st2;
    mm[2 * run + 1] = z2;
  }
}

__global__ void __launch_bounds__(256) dequantize_meta_kernel(const uint8_t* q, const float* mm,
                                                              int64_t n, int group, float* out) {
  const int64_t k = (int64_t)blockIdx.x * 256 + threadIdx.x;
  if (k >= n) return;
  const int64_t run = k / group;
  out[k] = __fmul_rn(__fsub_rn(u2f_small(q[k]), mm[2 * run + 1]), mm[2 * run]);
}

cudaError_t launch_quantize_meta(const void* meta, int dtype, int64_t n, int group, uint8_t* q,
                                 float* mm, cudaStream_t st) {
  const int64_t runs = (n + group - 1) / group;
  const int64_t blocks = (runs * 32 + 255) / 256;
  if (blocks == 0) return cudaSuccess;
  if (blocks > 0x7fffffffLL) return cudaErrorInvalidValue;
  quantize_meta_kernel<<<(unsigned)blocks, 256, 0, st>>>(meta, dtype, n, group, q, mm);
  return cudaGetLastError();
}

cudaError_t launch_dequantize_meta(const uint8_t* q, const float* mm, int64_t n, int group,
                                   float* out, cudaStream_t st) {
  const int64_t blocks = (n + 255) / 256;
  if (blocks == 0) return cudaSuccess;
  if (blocks > 0x7fffffffLL) return cudaErrorInvalidValue;
  dequantize_meta_kernel<<<(unsigned)blocks, 256, 0, st>>>(q, mm, n, group, out);
  return cudaGetLastError();
}

}  // namespace hqqk
