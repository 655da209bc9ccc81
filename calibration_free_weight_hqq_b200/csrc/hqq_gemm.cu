// hqq_gemm.cu - the consumer of the packed format: Y = X · W'^T (+ bias) for a 4-bit, group-64,
// axis-1 quantized weight, with W' dequantized on the fly into the tensor-core operand.
//
// What is computed: an HQQ-quantized linear layer computes its output in the compute dtype from
// the dequantized weight ("HQQ calibration-free guide" (lnwmold.com) §3.2, HQQLinear forward
// with compute_dtype; §4.2, the axis=1 backends fuse dequantization into the matrix product).
// W'[n, k] = dtype((float(Q[n, k]) - zero[g]) * scale[g]), g = n*(K/64) + k/64, rounded once to
// the activation dtype exactly as hqq_dequantize writes it; Y[m, n] = dtype(Σ_k X[m,k]·W'[n,k]
// accumulated in fp32 (+ bias[n])).
//
// Blackwell design, one 256 x 256 output tile per CTA, 64 + 32*HQQ_GEMM_DQ_WARPS threads, one
// CTA per SM:
//   warp 0      TMA producer: X tile (two 128 x 64 boxes, 128-byte swizzle, which is the UMMA
//               K-major SW128 layout) and the packed-code tile (256 rows x 32 bytes) into a
//               3-stage ring.
//   warp 1      allocates 512 TMEM columns (two 128 x 256 fp32 accumulators); lane 0 issues
//               tcgen05.mma (kind::f16, M=128, N=256, K=16) - 8 per k-block - and releases
//               ring slots with tcgen05.commit.
//   warps 2-    dequantize: (scale, zero) of their rows fetched 8 k-blocks ahead (one group
//               per row per k-block: BK = 64 = group size), 4-bit codes to bf16/fp16 straight
//               into a 2-stage ring in the SW128 K-major layout
//               (16-byte stores, conflict-free); after the last k-block, the epilogue:
//               tcgen05.ld of the accumulators, bias, rounding, 32 x 32 blocks staged in
//               shared memory and written by TMA stores.
// Every wait is bounded (about two seconds of %globaltimer); on expiry the CTA raises an abort
// flag, counts a timeout in g_gemm_timeouts, skips its remaining work, waits (bounded) for
// its own asynchronous operations and frees its TMEM.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>
#include <type_traits>

#include "hqq_device.cuh"
#include "hqq_kernels.h"

namespace hqqk {

__device__ unsigned int g_gemm_timeouts = 0;

namespace {

#ifndef HQQ_GEMM_DQ_WARPS
#define HQQ_GEMM_DQ_WARPS 16
#endif
#ifndef HQQ_GEMM_B_STAGES
#define HQQ_GEMM_B_STAGES 2
#endif
#ifndef HQQ_GEMM_TMA_STORE
#define HQQ_GEMM_TMA_STORE 1
#endif
#ifndef HQQ_GEMM_2SM
#define HQQ_GEMM_2SM 1
#endif

constexpr int kBM = 256, kBN = 256, kBK = 64;
constexpr int kStagesL = 3;                  // X + packed codes + meta
constexpr int kStagesB = HQQ_GEMM_B_STAGES;  // dequantized operand
constexpr int kDqWarps = HQQ_GEMM_DQ_WARPS;  // 8 or 16
static_assert(kDqWarps == 8 || kDqWarps == 16, "dequantize warps");
constexpr int kDqIters = kBN * (kBK / 8) / (32 * kDqWarps);  // 8-code chunks per thread
constexpr int kThreads = 64 + 32 * kDqWarps;
constexpr uint32_t kAHalf = 128 * kBK * 2;
constexpr uint32_t kABytes = 2 * kAHalf;
constexpr uint32_t kPBytes = kBN * kBK / 2;
constexpr uint32_t kBBytes = kBN * kBK * 2;
constexpr uint32_t kOffA = 0;
constexpr uint32_t kOffB = kOffA + kStagesL * kABytes;
constexpr uint32_t kOffP = kOffB + kStagesB * kBBytes;
constexpr uint32_t kOffBar = kOffP + kStagesL * kPBytes;
// Epilogue staging (reuses the X ring once the last MMA has completed): per dequantize warp two
// 32 x 32 output blocks of 64-byte rows, stored by TMA.
constexpr uint32_t kStageBytes = 32 * 32 * 2;
static_assert(kDqWarps * 2 * kStageBytes <= kStagesL * kABytes, "staging fits the X ring");
constexpr int kBarFullL = 0, kBarEmptyL = kStagesL, kBarFullB = 2 * kStagesL,
              kBarEmptyB = 2 * kStagesL + kStagesB, kBarAcc = 2 * kStagesL + 2 * kStagesB;
constexpr int kNumBars = kBarAcc + 1;
constexpr uint32_t kOffTmem = kOffBar + 8 * kNumBars;
constexpr uint32_t kOffAbort = kOffTmem + 4;
constexpr uint32_t kSmemBytes = kOffAbort + 4 + 1024;  // + slack to align the base to 1024
constexpr uint32_t kTmemCols = 512;
constexpr unsigned long long kWaitLimitNs = 2000000000ull;
static_assert(kOffB % 1024 == 0 && kABytes % 1024 == 0 && kBBytes % 1024 == 0, "SW128 tiles");
static_assert(kSmemBytes <= 232448, "shared memory per CTA");

struct GemmArgs {
  const void* scale;
  const void* zero;
  const void* bias;  // nullptr or [N] of the activation dtype
  void* Y;           // [M, N] of the activation dtype
  int M, N, K;
};

// ---------------------------------------------------------------- PTX wrappers
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ uint64_t globaltimer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void mbar_arrive_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
// Wait for the phase of `bar` with the given parity to complete. Returns false when the CTA
// aborted (another role gave up) or this wait ran out of time (it then raises the abort).
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity,
                                          volatile uint32_t* abort_flag) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*abort_flag) return false;
    if (globaltimer() - t0 > kWaitLimitNs) {
      *abort_flag = 1;
      atomicAdd(&g_gemm_timeouts, 1u);
      return false;
    }
  }
}
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int x, int y,
                                            uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar)
      : "memory");
}
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, uint32_t src, int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%1, %2}], [%3];" ::"l"(
          reinterpret_cast<uint64_t>(map)),
      "r"(x), "r"(y), "r"(src)
      : "memory");
}
__device__ __forceinline__ void bulk_commit() {
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void bulk_wait_read() {
  asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   bar)
               : "memory");
}
__device__ __forceinline__ void tc_mma(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc,
                                       uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d),
      "l"(a), "l"(b), "r"(idesc), "r"(accumulate)
      : "memory");
}
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11,"
      " %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29,"
      " %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// Shared-memory matrix descriptor of a K-major operand tile in the 128-byte swizzle layout:
// rows of 64 16-bit elements (128 B), 8-row atoms 1024 B apart (stride byte offset), tile
// base 1024-byte aligned. Fields: start address >> 4 (bits 0-13), leading byte offset >> 4
// (16-29, unused by this layout, set to 1), stride byte offset >> 4 (32-45), descriptor
// version 1 (46-47), layout 2 = SWIZZLE_128B (61-63).
__device__ __forceinline__ uint64_t sw128_kmajor_desc(uint32_t saddr) {
  return static_cast<uint64_t>((saddr >> 4) & 0x3FFFu) | (1ull << 16) |
         (static_cast<uint64_t>(1024 >> 4) << 32) | (1ull << 46) | (2ull << 61);
}

// Instruction descriptor of kind::f16: fp32 accumulator (bits 4-5 = 1), A and B format
// (bits 7-9, 10-12: 0 = f16, 1 = bf16), both K-major (bits 15, 16 = 0), N >> 3 (bits 17-22),
// M >> 4 (bits 24-28).
template <bool F16>
__device__ __forceinline__ uint32_t mma_idesc() {
  constexpr uint32_t fmt = F16 ? 0u : 1u;
  return (1u << 4) | (fmt << 7) | (fmt << 10) | (static_cast<uint32_t>(kBN >> 3) << 17) |
         (static_cast<uint32_t>(128 >> 4) << 24);
}

// The 4-bit conversion of the operand tile is dequant8_4bit (hqq_device.cuh): the same three
// roundings as hqq_dequantize.
template <bool F16>
__device__ __forceinline__ uint4 dequant8(uint32_t w, float2 neg_zero, float2 scale) {
  return dequant8_4bit<F16 ? kF16 : kBF16>(w, neg_zero, scale);
}

template <int MT>
__device__ __forceinline__ uint32_t meta_load(const uint8_t* p) {
  if constexpr (MT == kF32) return __ldg(reinterpret_cast<const unsigned int*>(p));
  return __ldg(reinterpret_cast<const unsigned short*>(p));
}
template <int MT>
__device__ __forceinline__ float meta_f32(uint32_t h) {
  if constexpr (MT == kF32) return __uint_as_float(h);
  return MT == kBF16 ? bf16_bits_to_f32(h) : f16_bits_to_f32(h);
}

template <bool F16, int MT>
__global__ void __launch_bounds__(kThreads, 1)
    w4a16_gemm_kernel(const __grid_constant__ CUtensorMap tmap_x,
                      const __grid_constant__ CUtensorMap tmap_w,
                      const __grid_constant__ CUtensorMap tmap_y, const GemmArgs args) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_u32(smem);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n0 = blockIdx.x * kBN, m0 = blockIdx.y * kBM;
  const int KB = args.K / kBK;
  volatile uint32_t* abort_flag = reinterpret_cast<volatile uint32_t*>(smem + kOffAbort);
  auto bar = [&](int i) { return sbase + kOffBar + 8u * static_cast<uint32_t>(i); };

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStagesL; ++s) {
      mbar_init(bar(kBarFullL + s), 1);  // producer's expect_tx (+ the copies' bytes)
      mbar_init(bar(kBarEmptyL + s), 1);  // MMA commit
    }
    for (int t = 0; t < kStagesB; ++t) {
      mbar_init(bar(kBarFullB + t), kDqWarps);
      mbar_init(bar(kBarEmptyB + t), 1);
    }
    mbar_init(bar(kBarAcc), 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmap_x)) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmap_w)) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmap_y)) : "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     sbase + kOffTmem),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(smem + kOffTmem);

  if (warp == 0) {
    // ------------------------------------------------------------ producer (TMA only)
    int issued = 0;
    for (int kb = 0; kb < KB; ++kb) {
      const int s = kb % kStagesL;
      const uint32_t ph = (kb / kStagesL) & 1;
      if (!mbar_wait(bar(kBarEmptyL + s), ph ^ 1, abort_flag)) break;
      if (lane == 0) {
        const uint32_t full = bar(kBarFullL + s);
        mbar_arrive_tx(full, kABytes + kPBytes);
        const uint32_t a = sbase + kOffA + s * kABytes;
        tma_load_2d(a, &tmap_x, kb * kBK, m0, full);
        tma_load_2d(a + kAHalf, &tmap_x, kb * kBK, m0 + 128, full);
        tma_load_2d(sbase + kOffP + s * kPBytes, &tmap_w, kb * (kBK / 2), n0, full);
      }
      ++issued;
    }
    // Before leaving, make sure no copy of ours is still landing in shared memory: wait for
    // the last use of every slot (already complete on the normal path).
    if (lane == 0) {
      for (int kb = issued - 1; kb >= 0 && kb >= issued - kStagesL; --kb) {
        const uint64_t t0 = globaltimer();
        while (!mbar_try_wait(bar(kBarFullL + kb % kStagesL), (kb / kStagesL) & 1) &&
               globaltimer() - t0 < kWaitLimitNs) {
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc = mma_idesc<F16>();
      for (int kb = 0; kb < KB; ++kb) {
        const int s = kb % kStagesL, t = kb % kStagesB;
        if (!mbar_wait(bar(kBarFullL + s), (kb / kStagesL) & 1, abort_flag)) break;
        if (!mbar_wait(bar(kBarFullB + t), (kb / kStagesB) & 1, abort_flag)) break;
        tc_fence_after();
        const uint32_t a = sbase + kOffA + s * kABytes;
        const uint64_t da0 = sw128_kmajor_desc(a), da1 = sw128_kmajor_desc(a + kAHalf);
        const uint64_t db = sw128_kmajor_desc(sbase + kOffB + t * kBBytes);
#pragma unroll
        for (int k = 0; k < kBK / 16; ++k) {
          // K step of 16 elements = 32 bytes inside the swizzled 128-byte row.
          const uint32_t acc = (kb | k) != 0;
          tc_mma(tmem, da0 + 2 * k, db + 2 * k, idesc, acc);
          tc_mma(tmem + kBN, da1 + 2 * k, db + 2 * k, idesc, acc);
        }
        tc_commit(bar(kBarEmptyL + s));
        tc_commit(bar(kBarEmptyB + t));
      }
      tc_commit(bar(kBarAcc));  // also the last word on any aborted run
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ dequantize
    // Thread (d, lane) converts 8-code chunk `chunk` of rows d*4*kDqIters + 4j + lane/8. The
    // 8 lanes that share a row also share its (scale, zero): each fetches the values of one
    // of the next 8 k-blocks (lane & 7 = offset) from global memory a full 8 k-blocks ahead,
    // and every k-block the value is taken from the lane that holds it with a shuffle. For
    // 16-bit meta scale and zero travel packed in one word.
    const int d = warp - 2;
    const int chunk = lane & 7;
    constexpr int kMB = MT == kF32 ? 4 : 2;
    constexpr int kWords = MT == kF32 ? 2 : 1;  // shuffled words per row and k-block
    const int64_t groups_per_row = args.K / kBK;
    const uint8_t* row_s[kDqIters];
    const uint8_t* row_z[kDqIters];
#pragma unroll
    for (int j = 0; j < kDqIters; ++j) {
      const int n = n0 + d * (4 * kDqIters) + j * 4 + (lane >> 3);
      const int64_t off = static_cast<int64_t>(n) * groups_per_row * kMB;
      row_s[j] = n < args.N ? static_cast<const uint8_t*>(args.scale) + off : nullptr;
      row_z[j] = n < args.N ? static_cast<const uint8_t*>(args.zero) + off : nullptr;
    }
    uint32_t nxt_s[kDqIters], nxt_z[kDqIters], cur[kDqIters][kWords];
    auto fetch8 = [&](int kb8) {  // this lane's k-block of the 8-block window kb8
      const int kk = kb8 * 8 + chunk;
#pragma unroll
      for (int j = 0; j < kDqIters; ++j) {
        const bool in = row_s[j] != nullptr && kk < KB;  // rows past N dequantize to 0
        nxt_s[j] = in ? meta_load<MT>(row_s[j] + static_cast<int64_t>(kk) * kMB) : 0u;
        nxt_z[j] = in ? meta_load<MT>(row_z[j] + static_cast<int64_t>(kk) * kMB) : 0u;
      }
    };
    if (KB > 0) fetch8(0);
    for (int kb = 0; kb < KB; ++kb) {
      const int s = kb % kStagesL, t = kb % kStagesB;
      if ((kb & 7) == 0) {  // the window's values arrived during the previous 8 k-blocks
#pragma unroll
        for (int j = 0; j < kDqIters; ++j) {
          if constexpr (kWords == 1) {
            cur[j][0] = nxt_s[j] | (nxt_z[j] << 16);
          } else {
            cur[j][0] = nxt_s[j];
            cur[j][kWords - 1] = nxt_z[j];
          }
        }
        if (kb + 8 < KB) fetch8((kb >> 3) + 1);
      }
      const int src = (lane & ~7) | (kb & 7);
      float sc[kDqIters], nz[kDqIters];
#pragma unroll
      for (int j = 0; j < kDqIters; ++j) {
        if constexpr (kWords == 1) {
          const uint32_t v = __shfl_sync(0xFFFFFFFFu, cur[j][0], src);
          sc[j] = meta_f32<MT>(v & 0xFFFFu);
          nz[j] = -meta_f32<MT>(v >> 16);
        } else {
          sc[j] = meta_f32<MT>(__shfl_sync(0xFFFFFFFFu, cur[j][0], src));
          nz[j] = -meta_f32<MT>(__shfl_sync(0xFFFFFFFFu, cur[j][kWords - 1], src));
        }
      }
      // warp-uniform outcome: the shuffles above and below take every lane
      if (!__all_sync(0xFFFFFFFFu, mbar_wait(bar(kBarFullL + s), (kb / kStagesL) & 1, abort_flag)))
        break;
      if (!__all_sync(0xFFFFFFFFu,
                      mbar_wait(bar(kBarEmptyB + t), ((kb / kStagesB) & 1) ^ 1, abort_flag)))
        break;
      const uint8_t* P = smem + kOffP + s * kPBytes;
      uint8_t* B = smem + kOffB + t * kBBytes;
      uint32_t w[kDqIters];
#pragma unroll
      for (int j = 0; j < kDqIters; ++j) {
        const int row = d * (4 * kDqIters) + j * 4 + (lane >> 3);
        w[j] = *reinterpret_cast<const uint32_t*>(P + row * 32 + chunk * 4);
      }
#pragma unroll
      for (int j = 0; j < kDqIters; ++j) {
        const int row = d * (4 * kDqIters) + j * 4 + (lane >> 3);
        *reinterpret_cast<uint4*>(B + row * 128 + ((chunk ^ (row & 7)) << 4)) =
            dequant8<F16>(w[j], make_float2(nz[j], nz[j]), make_float2(sc[j], sc[j]));
      }
      fence_proxy_async_smem();  // generic-proxy writes -> read by the tensor core
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(kBarFullB + t));
    }

    // ------------------------------------------------------------ epilogue
    // 4 consecutive warps cover the four TMEM lane quarters; groups of four alternate
    // between the two accumulators and split the 8 column chunks between them
    constexpr int kChunksPerWarp = (kBN / 32) * 8 / kDqWarps;
    const int h = (d >> 2) & 1;    // which 128-row accumulator
    const int c0 = (d >> 3) * kChunksPerWarp;
    const int quarter = warp & 3;  // TMEM lanes this warp may read: 32*quarter ..
    // warp-uniform: tcgen05.ld below is a .sync.aligned instruction
    const bool ok =
        __all_sync(0xFFFFFFFFu, mbar_wait(bar(kBarAcc), 0, abort_flag) && !*abort_flag);
    tc_fence_after();
    const int row0 = m0 + h * 128 + quarter * 32;
    const unsigned short* bias = reinterpret_cast<const unsigned short*>(args.bias);
#if HQQ_GEMM_TMA_STORE
    uint8_t* stage0 = smem + kOffA + static_cast<uint32_t>(d) * 2u * kStageBytes;
#else
    const int m = row0 + lane;
    typedef typename std::conditional<F16, __half, __nv_bfloat16>::type T;
    T* Yrow = reinterpret_cast<T*>(args.Y) + static_cast<int64_t>(m) * args.N;
#endif
#pragma unroll 1
    for (int c = c0; c < c0 + kChunksPerWarp; ++c) {
      uint32_t r[32];
      if (ok && KB > 0) {
        tmem_ld32(tmem + (static_cast<uint32_t>(quarter * 32) << 16) + h * kBN + c * 32, r);
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) r[i] = 0u;  // empty sum (K = 0)
      }
      const int nc = n0 + c * 32;
      uint32_t o[16];
#pragma unroll
      for (int i = 0; i < 32; i += 2) {
        float v0 = __uint_as_float(r[i]), v1 = __uint_as_float(r[i + 1]);
        if (bias != nullptr && nc + i < args.N) {  // N % 8 == 0: pairs never straddle
          v0 = __fadd_rn(v0, F16 ? f16_bits_to_f32(bias[nc + i]) : bf16_bits_to_f32(bias[nc + i]));
          v1 = __fadd_rn(v1, F16 ? f16_bits_to_f32(bias[nc + i + 1])
                                 : bf16_bits_to_f32(bias[nc + i + 1]));
        }
        o[i / 2] = pack2_16<F16 ? kF16 : kBF16>(v0, v1);
      }
#if HQQ_GEMM_TMA_STORE
      // Stage the warp's 32 x 32 block (row = lane, 64 bytes) in the 64-byte swizzle the
      // output tensor map uses (16-byte chunk q of row r at chunk q ^ ((r >> 1) & 3)), which
      // makes the four 16-byte stores conflict-free; one lane then stores it with TMA.
      // Rows past M and columns past N are clipped by the copy itself.
      uint8_t* stage = stage0 + ((c - c0) & 1) * kStageBytes;
      if (lane == 0 && c - c0 >= 2) bulk_wait_read<1>();  // this buffer's previous store
      __syncwarp();
#pragma unroll
      for (int q = 0; q < 4; ++q)
        *reinterpret_cast<uint4*>(stage + lane * 64 + ((q ^ ((lane >> 1) & 3)) << 4)) =
            make_uint4(o[4 * q], o[4 * q + 1], o[4 * q + 2], o[4 * q + 3]);
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0 && ok) {
        tma_store_2d(&tmap_y, smem_u32(stage), nc, row0);
        bulk_commit();
      }
#else
      if (!ok || m >= args.M || nc >= args.N) continue;
      if (nc + 32 <= args.N) {
        uint4* dst = reinterpret_cast<uint4*>(Yrow + nc);
#pragma unroll
        for (int q = 0; q < 4; ++q)
          dst[q] = make_uint4(o[4 * q], o[4 * q + 1], o[4 * q + 2], o[4 * q + 3]);
      } else {
#pragma unroll
        for (int i = 0; i < 16; ++i)
          if (nc + 2 * i < args.N) reinterpret_cast<uint32_t*>(Yrow + nc)[i] = o[i];
      }
#endif
    }
#if HQQ_GEMM_TMA_STORE
    if (lane == 0) bulk_wait_read<0>();  // shared memory stays ours until the stores read it
    __syncwarp();
#endif
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(kTmemCols)
                 : "memory");
  }
}

// ================================================================ 2-SM kernel
// A CTA pair (cluster of 2 along x, rank 0 = leader) computes a 512 x 256 output tile with
// tcgen05.mma.cta_group::2 (M = 256 = 128 rows from each CTA, N = 256 split 128 / 128):
//   * each CTA TMA-loads its own two 128 x 64 X boxes (rows m0 + h*256 + rank*128) per k-block;
//     those copies complete on the leader's barrier (cta_group::2 form);
//   * each CTA dequantizes only its own 128 rows of the W' tile (n0 + rank*128 ..) into its own
//     shared memory, so the conversion work per output is half that of one CTA doing all 256,
//     and each SM's tensor core reads only its own half of W';
//   * the leader's single thread issues the MMAs into two 256-column accumulators per SM and
//     multicasts its commits to both CTAs' barriers; one thread of the follower relays "our
//     half is written" to the leader with one cluster-scope arrive per k-block.
namespace sm2 {
constexpr int kStagesL = 4;   // X boxes + packed codes
constexpr int kStagesB = 3;   // dequantized half operand
constexpr int kDqWarps = 16;
constexpr int kRows = kBN / 2;                                   // W' rows per CTA
constexpr int kDqIters = kRows * (kBK / 8) / (32 * kDqWarps);   // 2
constexpr int kThreads = 64 + 32 * kDqWarps;
constexpr uint32_t kAHalf = 128 * kBK * 2;
constexpr uint32_t kABytes = 2 * kAHalf;
constexpr uint32_t kPBytes = kRows * kBK / 2;
constexpr uint32_t kBBytes = kRows * kBK * 2;
constexpr uint32_t kOffA = 0;
constexpr uint32_t kOffB = kOffA + kStagesL * kABytes;
constexpr uint32_t kOffP = kOffB + kStagesB * kBBytes;
constexpr uint32_t kOffBar = kOffP + kStagesL * kPBytes;
constexpr int kFullA = 0, kFullP = kStagesL, kEmptyL = 2 * kStagesL, kFullB = 3 * kStagesL,
              kHalfB = kFullB + kStagesB, kEmptyB = kHalfB + kStagesB, kAcc = kEmptyB + kStagesB;
constexpr int kNumBars = kAcc + 1;
constexpr uint32_t kOffTmem = kOffBar + 8 * kNumBars;
constexpr uint32_t kOffAbort = kOffTmem + 4;
constexpr uint32_t kSmemBytes = kOffAbort + 4 + 1024;
static_assert(kOffB % 1024 == 0 && kBBytes % 1024 == 0, "SW128 tiles");
static_assert(kSmemBytes <= 232448, "shared memory per CTA");
static_assert(kDqWarps * 2 * kStageBytes <= kStagesL * kABytes, "staging fits the X ring");
}  // namespace sm2

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::
                   : "memory");
}
// Address of the same shared-memory location in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t cluster_addr(uint32_t local, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(local), "r"(rank));
  return r;
}
__device__ __forceinline__ bool mbar_try_wait_cluster(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
// As mbar_wait, acquiring at cluster scope (arrivals from the peer CTA or its commits).
__device__ __forceinline__ bool mbar_wait_cl(uint32_t bar, uint32_t parity,
                                             volatile uint32_t* abort_flag) {
  if (mbar_try_wait_cluster(bar, parity)) return true;
  const uint64_t t0 = globaltimer();
  while (true) {
    if (mbar_try_wait_cluster(bar, parity)) return true;
    if (*abort_flag) return false;
    if (globaltimer() - t0 > kWaitLimitNs) {
      *abort_flag = 1;
      atomicAdd(&g_gemm_timeouts, 1u);
      return false;
    }
  }
}
__device__ __forceinline__ void mbar_arrive_remote(uint32_t cluster_bar) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_bar)
               : "memory");
}
// TMA load whose completion is counted on a barrier of either CTA of the pair.
__device__ __forceinline__ void tma_load_2d_pair(uint32_t dst, const CUtensorMap* map, int x,
                                                 int y, uint32_t cluster_bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(cluster_bar)
      : "memory");
}
__device__ __forceinline__ void tc_mma_pair(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc,
                                            uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d),
      "l"(a), "l"(b), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Arrive on `bar` (same offset) in both CTAs of the pair once the issued MMAs complete.
__device__ __forceinline__ void tc_commit_pair(uint32_t bar) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
      " [%0], %1;" ::"r"(bar),
      "h"(static_cast<unsigned short>(3))
      : "memory");
}
template <bool F16>
__device__ __forceinline__ uint32_t mma_idesc_m256() {
  constexpr uint32_t fmt = F16 ? 0u : 1u;
  return (1u << 4) | (fmt << 7) | (fmt << 10) | (static_cast<uint32_t>(kBN >> 3) << 17) |
         (static_cast<uint32_t>(256 >> 4) << 24);
}

template <bool F16, int MT>
__global__ void __launch_bounds__(sm2::kThreads, 1)
    w4a16_gemm_2sm_kernel(const __grid_constant__ CUtensorMap tmap_x,
                          const __grid_constant__ CUtensorMap tmap_w,
                          const __grid_constant__ CUtensorMap tmap_y, const GemmArgs args) {
  // this kernel's layout (shadows the one-CTA kernel's constants)
  constexpr auto kStagesL = sm2::kStagesL;
  constexpr auto kStagesB = sm2::kStagesB;
  constexpr auto kDqWarps = sm2::kDqWarps;
  constexpr auto kRows = sm2::kRows;
  constexpr auto kDqIters = sm2::kDqIters;
  constexpr auto kAHalf = sm2::kAHalf;
  constexpr auto kABytes = sm2::kABytes;
  constexpr auto kPBytes = sm2::kPBytes;
  constexpr auto kBBytes = sm2::kBBytes;
  constexpr auto kOffA = sm2::kOffA;
  constexpr auto kOffB = sm2::kOffB;
  constexpr auto kOffP = sm2::kOffP;
  constexpr auto kOffBar = sm2::kOffBar;
  constexpr auto kFullA = sm2::kFullA;
  constexpr auto kFullP = sm2::kFullP;
  constexpr auto kEmptyL = sm2::kEmptyL;
  constexpr auto kFullB = sm2::kFullB;
  constexpr auto kHalfB = sm2::kHalfB;
  constexpr auto kEmptyB = sm2::kEmptyB;
  constexpr auto kAcc = sm2::kAcc;
  constexpr auto kOffTmem = sm2::kOffTmem;
  constexpr auto kOffAbort = sm2::kOffAbort;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_u32(smem);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();  // 0: leader, issues the MMAs
  const bool leader = rank == 0;
  const int m0 = static_cast<int>(blockIdx.x >> 1) * 512, n0 = blockIdx.y * kBN;
  const int KB = args.K / kBK;
  volatile uint32_t* abort_flag = reinterpret_cast<volatile uint32_t*>(smem + kOffAbort);
  auto bar = [&](int i) { return sbase + kOffBar + 8u * static_cast<uint32_t>(i); };

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStagesL; ++s) {
      mbar_init(bar(kFullA + s), 1);   // leader: expect_tx for both CTAs' X boxes
      mbar_init(bar(kFullP + s), 1);   // own packed codes
      mbar_init(bar(kEmptyL + s), 1);  // leader's commit
    }
    for (int t = 0; t < kStagesB; ++t) {
      mbar_init(bar(kFullB + t), kDqWarps + 1);  // leader: own warps + the follower's relay
      mbar_init(bar(kHalfB + t), kDqWarps);      // follower: own warps
      mbar_init(bar(kEmptyB + t), 1);            // leader's commit
    }
    mbar_init(bar(kAcc), 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmap_x)) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmap_w)) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmap_y)) : "memory");
  }
  if (warp == 1) {  // the same warp in both CTAs, as the paired allocation requires
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     sbase + kOffTmem),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // barriers of both CTAs initialised, TMEM address written in both
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(smem + kOffTmem);
  const uint32_t leader_bars = cluster_addr(sbase + kOffBar, 0);
  auto lbar = [&](int i) { return leader_bars + 8u * static_cast<uint32_t>(i); };

  if (warp == 0) {
    // ------------------------------------------------------------ producer (both CTAs)
    int issued = 0;
    for (int kb = 0; kb < KB; ++kb) {
      const int s = kb % kStagesL;
      if (!mbar_wait_cl(bar(kEmptyL + s), ((kb / kStagesL) & 1) ^ 1, abort_flag)) break;
      if (lane == 0) {
        if (leader) mbar_arrive_tx(bar(kFullA + s), 2 * kABytes);
        const uint32_t a = sbase + kOffA + s * kABytes;
        tma_load_2d_pair(a, &tmap_x, kb * kBK, m0 + static_cast<int>(rank) * 128, lbar(kFullA + s));
        tma_load_2d_pair(a + kAHalf, &tmap_x, kb * kBK, m0 + 256 + static_cast<int>(rank) * 128,
                         lbar(kFullA + s));
        mbar_arrive_tx(bar(kFullP + s), kPBytes);
        tma_load_2d(sbase + kOffP + s * kPBytes, &tmap_w, kb * (kBK / 2),
                    n0 + static_cast<int>(rank) * kRows, bar(kFullP + s));
      }
      ++issued;
    }
    if (lane == 0) {  // own packed-code copies landed before leaving (complete on the normal path)
      for (int kb = issued - 1; kb >= 0 && kb >= issued - kStagesL; --kb) {
        const uint64_t t0 = globaltimer();
        while (!mbar_try_wait(bar(kFullP + kb % kStagesL), (kb / kStagesL) & 1) &&
               globaltimer() - t0 < kWaitLimitNs) {
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      if (leader) {
        // -------------------------------------------------------- MMA issuer (leader)
        const uint32_t idesc = mma_idesc_m256<F16>();
        for (int kb = 0; kb < KB; ++kb) {
          const int s = kb % kStagesL, t = kb % kStagesB;
          if (!mbar_wait_cl(bar(kFullA + s), (kb / kStagesL) & 1, abort_flag)) break;
          if (!mbar_wait_cl(bar(kFullB + t), (kb / kStagesB) & 1, abort_flag)) break;
          tc_fence_after();
          const uint32_t a = sbase + kOffA + s * kABytes;
          const uint64_t da0 = sw128_kmajor_desc(a), da1 = sw128_kmajor_desc(a + kAHalf);
          const uint64_t db = sw128_kmajor_desc(sbase + kOffB + t * kBBytes);
#pragma unroll
          for (int k = 0; k < kBK / 16; ++k) {
            const uint32_t acc = (kb | k) != 0;
            tc_mma_pair(tmem, da0 + 2 * k, db + 2 * k, idesc, acc);
            tc_mma_pair(tmem + kBN, da1 + 2 * k, db + 2 * k, idesc, acc);
          }
          tc_commit_pair(bar(kEmptyL + s));
          tc_commit_pair(bar(kEmptyB + t));
        }
        tc_commit_pair(bar(kAcc));  // also the last word on any aborted run
      } else {
        // -------------------------------------------------------- relay (follower)
        for (int kb = 0; kb < KB; ++kb) {
          const int t = kb % kStagesB;
          if (!mbar_wait(bar(kHalfB + t), (kb / kStagesB) & 1, abort_flag)) break;
          mbar_arrive_remote(lbar(kFullB + t));
        }
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ dequantize (both CTAs)
    const int d = warp - 2;
    const int chunk = lane & 7;
    constexpr int kMB = MT == kF32 ? 4 : 2;
    constexpr int kWords = MT == kF32 ? 2 : 1;
    const int64_t groups_per_row = args.K / kBK;
    const int nbase = n0 + static_cast<int>(rank) * kRows;
    const uint8_t* row_s[kDqIters];
    const uint8_t* row_z[kDqIters];
#pragma unroll
    for (int j = 0; j < kDqIters; ++j) {
      const int n = nbase + d * (4 * kDqIters) + j * 4 + (lane >> 3);
      const int64_t off = static_cast<int64_t>(n) * groups_per_row * kMB;
      row_s[j] = n < args.N ? static_cast<const uint8_t*>(args.scale) + off : nullptr;
      row_z[j] = n < args.N ? static_cast<const uint8_t*>(args.zero) + off : nullptr;
    }
    uint32_t nxt_s[kDqIters], nxt_z[kDqIters], cur[kDqIters][kWords];
    auto fetch8 = [&](int kb8) {
      const int kk = kb8 * 8 + chunk;
#pragma unroll
      for (int j = 0; j < kDqIters; ++j) {
        const bool in = row_s[j] != nullptr && kk < KB;
        nxt_s[j] = in ? meta_load<MT>(row_s[j] + static_cast<int64_t>(kk) * kMB) : 0u;
        nxt_z[j] = in ? meta_load<MT>(row_z[j] + static_cast<int64_t>(kk) * kMB) : 0u;
      }
    };
    if (KB > 0) fetch8(0);
    for (int kb = 0; kb < KB; ++kb) {
      const int s = kb % kStagesL, t = kb % kStagesB;
      if ((kb & 7) == 0) {
#pragma unroll
        for (int j = 0; j < kDqIters; ++j) {
          if constexpr (kWords == 1) {
            cur[j][0] = nxt_s[j] | (nxt_z[j] << 16);
          } else {
            cur[j][0] = nxt_s[j];
            cur[j][kWords - 1] = nxt_z[j];
          }
        }
        if (kb + 8 < KB) fetch8((kb >> 3) + 1);
      }
      const int src = (lane & ~7) | (kb & 7);
      float sc[kDqIters], nz[kDqIters];
#pragma unroll
      for (int j = 0; j < kDqIters; ++j) {
        if constexpr (kWords == 1) {
          const uint32_t v = __shfl_sync(0xFFFFFFFFu, cur[j][0], src);
          sc[j] = meta_f32<MT>(v & 0xFFFFu);
          nz[j] = -meta_f32<MT>(v >> 16);
        } else {
          sc[j] = meta_f32<MT>(__shfl_sync(0xFFFFFFFFu, cur[j][0], src));
          nz[j] = -meta_f32<MT>(__shfl_sync(0xFFFFFFFFu, cur[j][kWords - 1], src));
        }
      }
      if (!__all_sync(0xFFFFFFFFu, mbar_wait(bar(kFullP + s), (kb / kStagesL) & 1, abort_flag)))
        break;
      if (!__all_sync(0xFFFFFFFFu,
                      mbar_wait_cl(bar(kEmptyB + t), ((kb / kStagesB) & 1) ^ 1, abort_flag)))
        break;
      const uint8_t* P = smem + kOffP + s * kPBytes;
      uint8_t* B = smem + kOffB + t * kBBytes;
      uint32_t w[kDqIters];
#pragma unroll
      for (int j = 0; j < kDqIters; ++j) {
        const int row = d * (4 * kDqIters) + j * 4 + (lane >> 3);
        w[j] = *reinterpret_cast<const uint32_t*>(P + row * 32 + chunk * 4);
      }
#pragma unroll
      for (int j = 0; j < kDqIters; ++j) {
        const int row = d * (4 * kDqIters) + j * 4 + (lane >> 3);
        *reinterpret_cast<uint4*>(B + row * 128 + ((chunk ^ (row & 7)) << 4)) =
            dequant8<F16>(w[j], make_float2(nz[j], nz[j]), make_float2(sc[j], sc[j]));
      }
      fence_proxy_async_smem();  // generic-proxy writes -> read by the tensor core
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(leader ? kFullB + t : kHalfB + t));
    }

    // ------------------------------------------------------------ epilogue (both CTAs)
    constexpr int kChunksPerWarp = (kBN / 32) * 8 / kDqWarps;
    const int h = (d >> 2) & 1;
    const int c0 = (d >> 3) * kChunksPerWarp;
    const int quarter = warp & 3;
    const bool ok =
        __all_sync(0xFFFFFFFFu, mbar_wait_cl(bar(kAcc), 0, abort_flag) && !*abort_flag);
    tc_fence_after();
    const int row0 = m0 + h * 256 + static_cast<int>(rank) * 128 + quarter * 32;
    const unsigned short* bias = reinterpret_cast<const unsigned short*>(args.bias);
    uint8_t* stage0 = smem + kOffA + static_cast<uint32_t>(d) * 2u * kStageBytes;
#pragma unroll 1
    for (int c = c0; c < c0 + kChunksPerWarp; ++c) {
      uint32_t r[32];
      if (ok && KB > 0) {
        tmem_ld32(tmem + (static_cast<uint32_t>(quarter * 32) << 16) + h * kBN + c * 32, r);
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) r[i] = 0u;
      }
      const int nc = n0 + c * 32;
      uint32_t o[16];
#pragma unroll
      for (int i = 0; i < 32; i += 2) {
        float v0 = __uint_as_float(r[i]), v1 = __uint_as_float(r[i + 1]);
        if (bias != nullptr && nc + i < args.N) {
          v0 = __fadd_rn(v0, F16 ? f16_bits_to_f32(bias[nc + i]) : bf16_bits_to_f32(bias[nc + i]));
          v1 = __fadd_rn(v1, F16 ? f16_bits_to_f32(bias[nc + i + 1])
                                 : bf16_bits_to_f32(bias[nc + i + 1]));
        }
        o[i / 2] = pack2_16<F16 ? kF16 : kBF16>(v0, v1);
      }
      uint8_t* stage = stage0 + ((c - c0) & 1) * kStageBytes;
      if (lane == 0 && c - c0 >= 2) bulk_wait_read<1>();
      __syncwarp();
#pragma unroll
      for (int q = 0; q < 4; ++q)
        *reinterpret_cast<uint4*>(stage + lane * 64 + ((q ^ ((lane >> 1) & 3)) << 4)) =
            make_uint4(o[4 * q], o[4 * q + 1], o[4 * q + 2], o[4 * q + 3]);
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0 && ok) {
        tma_store_2d(&tmap_y, smem_u32(stage), nc, row0);
        bulk_commit();
      }
    }
    if (lane == 0) bulk_wait_read<0>();
    __syncwarp();
  }

  // The leader's commits land in both CTAs' barriers asynchronously: see the last use of every
  // slot completed before the pair parts.
  if (warp == 1 && lane == 0) {
    for (int kb = KB - 1; kb >= 0 && kb >= KB - kStagesL; --kb) {
      const uint64_t t0 = globaltimer();
      while (!mbar_try_wait_cluster(bar(kEmptyL + kb % kStagesL), (kb / kStagesL) & 1) &&
             globaltimer() - t0 < kWaitLimitNs) {
      }
    }
    for (int kb = KB - 1; kb >= 0 && kb >= KB - kStagesB; --kb) {
      const uint64_t t0 = globaltimer();
      while (!mbar_try_wait_cluster(bar(kEmptyB + kb % kStagesB), (kb / kStagesB) & 1) &&
             globaltimer() - t0 < kWaitLimitNs) {
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(kTmemCols)
                 : "memory");
  }
}

// ---------------------------------------------------------------- host side
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

template <bool F16, int MT>
cudaError_t launch_typed(const GemmJob& job, cudaStream_t stream) {
  PFN_cuTensorMapEncodeTiled_v12000 encode = tensor_map_encoder();
  if (encode == nullptr) return cudaErrorNotSupported;
  CUtensorMap mx, mw;
  {
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(job.K), static_cast<cuuint64_t>(job.M)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(job.K) * 2};
    const cuuint32_t box[2] = {kBK, 128};
    const cuuint32_t estr[2] = {1, 1};
    if (encode(&mx, F16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
               const_cast<void*>(job.X), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  {
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(job.K / 2),
                                static_cast<cuuint64_t>(job.N)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(job.K / 2)};
    const cuuint32_t box[2] = {kBK / 2, HQQ_GEMM_2SM ? static_cast<cuuint32_t>(sm2::kRows) : kBN};
    const cuuint32_t estr[2] = {1, 1};
    if (encode(&mw, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(job.packed), dims,
               strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  CUtensorMap my;
  {
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(job.N), static_cast<cuuint64_t>(job.M)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(job.N) * 2};
    const cuuint32_t box[2] = {32, 32};
    const cuuint32_t estr[2] = {1, 1};
    if (encode(&my, F16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
               job.Y, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
               CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  // per device and cheap: set on every call rather than cached
  cudaError_t e = cudaFuncSetAttribute(w4a16_gemm_kernel<F16, MT>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(kSmemBytes));
  if (e != cudaSuccess) return e;
  GemmArgs a;
  a.scale = job.scale;
  a.zero = job.zero;
  a.bias = job.bias;
  a.Y = job.Y;
  a.M = static_cast<int>(job.M);
  a.N = static_cast<int>(job.N);
  a.K = static_cast<int>(job.K);
#if HQQ_GEMM_2SM
  e = cudaFuncSetAttribute(w4a16_gemm_2sm_kernel<F16, MT>,
                           cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(sm2::kSmemBytes));
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * static_cast<unsigned>((job.M + 511) / 512),
                     static_cast<unsigned>((job.N + kBN - 1) / kBN));
  cfg.blockDim = dim3(sm2::kThreads);
  cfg.dynamicSmemBytes = sm2::kSmemBytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, w4a16_gemm_2sm_kernel<F16, MT>, mx, mw, my, a);
#else
  const dim3 grid(static_cast<unsigned>((job.N + kBN - 1) / kBN),
                  static_cast<unsigned>((job.M + kBM - 1) / kBM));
  w4a16_gemm_kernel<F16, MT><<<grid, kThreads, kSmemBytes, stream>>>(mx, mw, my, a);
  return cudaGetLastError();
#endif
}

// K = 0: the sum is empty, Y[m, n] = bias[n] (or 0).
__global__ void empty_sum_kernel(const unsigned short* bias, unsigned short* Y, int64_t M,
                                 int64_t N) {
  const int64_t total = M * N;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x)
    Y[i] = bias != nullptr ? bias[i % N] : static_cast<unsigned short>(0);
}

}  // namespace

cudaError_t launch_w4a16_gemm(const GemmJob& job, cudaStream_t stream) {
  if (job.M == 0 || job.N == 0) return cudaSuccess;
  if (job.K == 0) {
    empty_sum_kernel<<<296, 256, 0, stream>>>(static_cast<const unsigned short*>(job.bias),
                                              static_cast<unsigned short*>(job.Y), job.M, job.N);
    return cudaGetLastError();
  }
  const bool f16 = job.x_dtype == kF16;
  switch (job.meta_dtype) {
    case kF16:
      return f16 ? launch_typed<true, kF16>(job, stream) : launch_typed<false, kF16>(job, stream);
    case kBF16:
      return f16 ? launch_typed<true, kBF16>(job, stream) : launch_typed<false, kBF16>(job, stream);
    default:
      return f16 ? launch_typed<true, kF32>(job, stream) : launch_typed<false, kF32>(job, stream);
  }
}

cudaError_t read_gemm_timeouts(unsigned int* out) {
  return cudaMemcpyFromSymbol(out, g_gemm_timeouts, sizeof(unsigned int));
}

}  // namespace hqqk
