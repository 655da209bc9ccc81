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
// Three kernels, picked by the number of rows M of X (tokens):
//   * w4a16_gemm_2sm_kernel (M > 128): a CTA pair computes a 512 x 256 output tile with the
//     2-SM tensor-core MMA; each CTA dequantizes its own 128 rows of the W' tile (description
//     at the kernel).
//   * w4a16_skinny_kernel (16 < M <= 128): the roles swap - W' (128 rows per CTA) is the
//     MMA's M operand and the tokens its N - and a cluster of 4 CTAs splits K, reducing the
//     partial sums over distributed shared memory (description at the kernel).
//   * w4a16_gemv_kernel (M <= 16, decode): W' is dequantized straight into the register
//     fragments of the warp-level MMA; a cluster of up to 8 CTAs splits K (description at the
//     kernel); K up to 32768, larger K goes to the split-K kernel.
// Every wait of the first two is bounded (about two seconds of %globaltimer); on expiry the
// CTA raises an abort flag, counts a timeout in g_gemm_timeouts, skips its remaining work,
// waits (bounded) for its own asynchronous operations and frees its TMEM. The third has no
// waits besides the hardware cluster barrier.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <algorithm>
#include <mutex>
#include <type_traits>

#include "hqq_device.cuh"
#include "hqq_kernels.h"

namespace hqqk {

__device__ unsigned int g_gemm_timeouts = 0;

namespace {

constexpr int kBN = 256, kBK = 64;  // W' rows per 2-SM pair tile; K per k-block = group size
// Epilogue staging (reuses the X ring once the last MMA has completed): per dequantize warp two
// 32 x 32 output blocks of 64-byte rows, stored by TMA.
constexpr uint32_t kStageBytes = 32 * 32 * 2;
constexpr uint32_t kTmemCols = 512;
constexpr unsigned long long kWaitLimitNs = 2000000000ull;

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
#ifndef HQQ_GEMM_STAGES_B
#define HQQ_GEMM_STAGES_B 4
#endif
constexpr int kStagesL = 4;                  // X boxes + packed codes
constexpr int kStagesB = HQQ_GEMM_STAGES_B;  // dequantized half operand
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
__device__ __forceinline__ void cluster_arrive() {
  asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait() {
  asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
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
// Arrive on a barrier of the peer CTA. The default semantics (release at CTA scope) suffice for
// a "your operand half is written" signal: the data it announces is the peer's own shared
// memory, complete before this thread acquired its local barrier. A cluster-scope release
// measured about 0.9 us per arrive on B200 when one is relayed per k-block.
__device__ __forceinline__ void mbar_arrive_remote(uint32_t cluster_bar) {
  asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(cluster_bar) : "memory");
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

// ================================================================ skinny kernel (M <= 128)
// Decode-sized batches: too few output tiles for the 2-SM kernel to fill the GPU, and the
// weight is read once per token batch, so the work is the dequantization of W' and its HBM
// read. Roles swap: D[n, m] = sum_k W'[n, k] * X[m, k] with W' (128 rows per CTA, dequantized
// into shared memory in the SW128 K-major layout) as the MMA's A operand (M = 128) and the
// ntok <= 128 token rows of X (TMA, SW128) as its B operand (N = ntok, a multiple of 16); the
// accumulator is 128 TMEM lanes x ntok columns. A cluster of kSkS CTAs shares one W' row tile
// and splits K into contiguous slices; after its slice each CTA reads its partial D and writes
// rows 16r .. 16r+15 of it into a per-source slot of cluster CTA r (distributed shared memory,
// plain stores); after a cluster barrier CTA r sums its kSkS slots in rank order (fixed order:
// deterministic), adds bias, rounds and stores its 16 output rows for every token.
namespace skinny {
constexpr int kS = 4;            // CTAs per cluster = K slices
constexpr int kRows = 128;       // W' rows per CTA
constexpr int kTokMax = 64;      // tokens per CTA (MMA N); larger batches take several tiles
constexpr int kMaxM = 128;       // the skinny kernel serves M <= kMaxM
constexpr int kSub = 4;          // k-blocks per load stage: 128-byte rows of packed codes
constexpr int kStagesL = 2;      // load stages (X boxes + packed codes of kSub k-blocks)
constexpr int kStagesB = 3;      // dequantized W' stages, one k-block each
constexpr int kDqWarps = 8;
constexpr int kDqIters = kRows * (kBK / 8) / (32 * kDqWarps);  // chunks per thread
constexpr int kThreads = 64 + 32 * kDqWarps;
constexpr uint32_t kPBytes = kRows * kBK / 2 * kSub;  // 16 KB: 128 rows x 128 bytes
constexpr uint32_t kWBytes = kRows * kBK * 2;      // 16 KB
constexpr int kOwnRows = kRows / kS;                // output rows reduced per CTA
constexpr int kFullL = 0, kEmptyL = kStagesL, kFullW = 2 * kStagesL, kEmptyW = kFullW + kStagesB,
              kAcc = kEmptyW + kStagesB;
constexpr int kNumBars = kAcc + 1;
constexpr uint32_t kTmemCols = 128;
// Shared-memory layout for ntok tokens (a multiple of 16): the X ring holds ntok rows per stage
// and the reduction slots ntok columns, so small batches leave room for two CTAs per SM.
struct Layout {
  uint32_t x_stage, off_w, off_p, off_red, slot, off_bar, off_tmem, off_abort, bytes;
};
__host__ __device__ constexpr Layout layout(int ntok) {
  Layout L{};
  L.x_stage = static_cast<uint32_t>(ntok) * kBK * 2 * kSub;  // kSub SW128 boxes of ntok rows
  L.off_w = kStagesL * L.x_stage;
  L.off_p = L.off_w + kStagesB * kWBytes;
  L.off_red = L.off_p + kStagesL * kPBytes;
  L.slot = static_cast<uint32_t>(kOwnRows) * static_cast<uint32_t>(ntok) * 4;
  L.off_bar = L.off_red + kS * L.slot;
  L.off_tmem = L.off_bar + 8 * kNumBars;
  L.off_abort = L.off_tmem + 4;
  L.bytes = L.off_abort + 4 + 1024;  // + slack to align the base to 1024
  return L;
}
static_assert(kWBytes % 1024 == 0, "SW128 tiles");
static_assert(layout(kTokMax).bytes <= 232448, "shared memory per CTA");
}  // namespace skinny

// Instruction descriptor of kind::f16, M = 128, N = ntok (a multiple of 16, <= 256).
template <bool F16>
__device__ __forceinline__ uint32_t mma_idesc_m128(int ntok) {
  constexpr uint32_t fmt = F16 ? 0u : 1u;
  return (1u << 4) | (fmt << 7) | (fmt << 10) | (static_cast<uint32_t>(ntok >> 3) << 17) |
         (static_cast<uint32_t>(128 >> 4) << 24);
}
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11,"
      " %12, %13, %14, %15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void st_cluster_v4f(uint32_t addr, float a, float b, float c, float d) {
  asm volatile("st.shared::cluster.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "f"(a), "f"(b),
               "f"(c), "f"(d)
               : "memory");
}

template <bool F16, int MT>
__global__ void __launch_bounds__(skinny::kThreads, 2)
    w4a16_skinny_kernel(const __grid_constant__ CUtensorMap tmap_x,
                        const __grid_constant__ CUtensorMap tmap_w, const GemmArgs args,
                        int ntok) {
  // this kernel's layout (shadows the 2-SM kernel's constants)
  constexpr int kS = skinny::kS, kStagesL = skinny::kStagesL, kStagesB = skinny::kStagesB;
  constexpr int kSub = skinny::kSub;
  constexpr int kDqWarps = skinny::kDqWarps, kDqIters = skinny::kDqIters;
  constexpr int kOwnRows = skinny::kOwnRows, kTokMax = skinny::kTokMax;
  constexpr uint32_t kPBytes = skinny::kPBytes, kWBytes = skinny::kWBytes;
  const skinny::Layout lay = skinny::layout(ntok);
  const uint32_t kXBytes = lay.x_stage, kSlotBytes = lay.slot;
  const uint32_t kOffX = 0, kOffW = lay.off_w, kOffP = lay.off_p, kOffRed = lay.off_red,
                 kOffBar = lay.off_bar, kOffTmem = lay.off_tmem, kOffAbort = lay.off_abort;
  constexpr int kFullL = skinny::kFullL, kEmptyL = skinny::kEmptyL, kFullW = skinny::kFullW,
                kEmptyW = skinny::kEmptyW, kAcc = skinny::kAcc;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_u32(smem);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();  // K slice of this CTA; also which 16 rows it reduces
  const int n0 = static_cast<int>(blockIdx.x / kS) * skinny::kRows;
  const int m0 = blockIdx.y * kTokMax;
  const int KB = args.K / kBK;
  const int per = (KB + kS - 1) / kS;
  const int kb0 = min(KB, static_cast<int>(rank) * per), kb1 = min(KB, kb0 + per);
  const int nkb = kb1 - kb0;
  volatile uint32_t* abort_flag = reinterpret_cast<volatile uint32_t*>(smem + kOffAbort);
  auto bar = [&](int i) { return sbase + kOffBar + 8u * static_cast<uint32_t>(i); };

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStagesL; ++s) {
      mbar_init(bar(kFullL + s), 1);
      mbar_init(bar(kEmptyL + s), 1);
    }
    for (int t = 0; t < kStagesB; ++t) {
      mbar_init(bar(kFullW + t), kDqWarps);
      mbar_init(bar(kEmptyW + t), 1);
    }
    mbar_init(bar(kAcc), 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmap_x)) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmap_w)) : "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     sbase + kOffTmem),
                 "r"(skinny::kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // every CTA of the cluster is running before anyone writes into another
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(smem + kOffTmem);
  const uint32_t xbox = static_cast<uint32_t>(ntok) * kBK * 2;  // one X box (one k-block)
  const int nsb = (nkb + kSub - 1) / kSub;                        // load stages of the slice

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    // one stage = kSub k-blocks: kSub X boxes and one box of 128 packed-code rows x 128 bytes
    // (boxes reaching past K read zeros; k-blocks past the slice are loaded but not used)
    int issued = 0;
    for (int j = 0; j < nsb; ++j) {
      const int s = j % kStagesL, kb = kb0 + j * kSub;
      if (!mbar_wait(bar(kEmptyL + s), ((j / kStagesL) & 1) ^ 1, abort_flag)) break;
      if (lane == 0) {
        const uint32_t full = bar(kFullL + s);
        mbar_arrive_tx(full, kSub * xbox + kPBytes);
#pragma unroll
        for (int u = 0; u < kSub; ++u)
          tma_load_2d(sbase + kOffX + s * kXBytes + u * xbox, &tmap_x, (kb + u) * kBK, m0, full);
        tma_load_2d(sbase + kOffP + s * kPBytes, &tmap_w, kb * (kBK / 2), n0, full);
      }
      ++issued;
    }
    if (lane == 0) {
      for (int j = issued - 1; j >= 0 && j >= issued - kStagesL; --j) {
        const uint64_t t0 = globaltimer();
        while (!mbar_try_wait(bar(kFullL + j % kStagesL), (j / kStagesL) & 1) &&
               globaltimer() - t0 < kWaitLimitNs) {
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc = mma_idesc_m128<F16>(ntok);
      for (int j = 0; j < nkb; ++j) {
        const int sb = j / kSub, sub = j % kSub, s = sb % kStagesL, t = j % kStagesB;
        if (!mbar_wait(bar(kFullL + s), (sb / kStagesL) & 1, abort_flag)) break;
        if (!mbar_wait(bar(kFullW + t), (j / kStagesB) & 1, abort_flag)) break;
        tc_fence_after();
        const uint64_t dw = sw128_kmajor_desc(sbase + kOffW + t * kWBytes);
        const uint64_t dx = sw128_kmajor_desc(sbase + kOffX + s * kXBytes + sub * xbox);
#pragma unroll
        for (int k = 0; k < kBK / 16; ++k) tc_mma(tmem, dw + 2 * k, dx + 2 * k, idesc, (j | k) != 0);
        if (sub == kSub - 1 || j == nkb - 1) tc_commit(bar(kEmptyL + s));
        tc_commit(bar(kEmptyW + t));
      }
      tc_commit(bar(kAcc));  // also the last word on any aborted run
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ dequantize
    const int d = warp - 2;
    const int chunk = lane & 7;
    constexpr int kMB = MT == kF32 ? 4 : 2;
    constexpr int kWords = MT == kF32 ? 2 : 1;
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
    auto fetch8 = [&](int w8) {  // this lane's k-block of the 8-block window w8 of the slice
      const int kk = kb0 + w8 * 8 + chunk;
#pragma unroll
      for (int j = 0; j < kDqIters; ++j) {
        const bool in = row_s[j] != nullptr && kk < kb1;
        nxt_s[j] = in ? meta_load<MT>(row_s[j] + static_cast<int64_t>(kk) * kMB) : 0u;
        nxt_z[j] = in ? meta_load<MT>(row_z[j] + static_cast<int64_t>(kk) * kMB) : 0u;
      }
    };
    if (nkb > 0) fetch8(0);
    for (int j8 = 0; j8 < nkb; ++j8) {
      const int sb = j8 / kSub, sub = j8 % kSub, s = sb % kStagesL, t = j8 % kStagesB;
      if ((j8 & 7) == 0) {  // the window's values arrived during the previous 8 k-blocks
#pragma unroll
        for (int j = 0; j < kDqIters; ++j) {
          if constexpr (kWords == 1) {
            cur[j][0] = nxt_s[j] | (nxt_z[j] << 16);
          } else {
            cur[j][0] = nxt_s[j];
            cur[j][kWords - 1] = nxt_z[j];
          }
        }
        if (j8 + 8 < nkb) fetch8((j8 >> 3) + 1);
      }
      const int src = (lane & ~7) | (j8 & 7);
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
      if (!__all_sync(0xFFFFFFFFu, mbar_wait(bar(kFullL + s), (sb / kStagesL) & 1, abort_flag)))
        break;
      if (!__all_sync(0xFFFFFFFFu,
                      mbar_wait(bar(kEmptyW + t), ((j8 / kStagesB) & 1) ^ 1, abort_flag)))
        break;
      const uint8_t* P = smem + kOffP + s * kPBytes;
      uint8_t* Wt = smem + kOffW + t * kWBytes;
      uint32_t w[kDqIters];
#pragma unroll
      for (int j = 0; j < kDqIters; ++j) {
        const int row = d * (4 * kDqIters) + j * 4 + (lane >> 3);
        w[j] = *reinterpret_cast<const uint32_t*>(P + row * 128 + sub * 32 + chunk * 4);
      }
#pragma unroll
      for (int j = 0; j < kDqIters; ++j) {
        const int row = d * (4 * kDqIters) + j * 4 + (lane >> 3);
        *reinterpret_cast<uint4*>(Wt + row * 128 + ((chunk ^ (row & 7)) << 4)) =
            dequant8<F16>(w[j], make_float2(nz[j], nz[j]), make_float2(sc[j], sc[j]));
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(kFullW + t));
    }

    // ------------------------------------------------------------ partial sums -> owners
    // Warps 2..5 read the four TMEM lane quarters (rows 32q .. 32q+31 of the W' tile); row
    // 16r + i goes to slot `rank` of cluster CTA r: float [kOwnRows][kTokMax] at i.
    if (d < 4) {
      const int quarter = warp & 3;
      const bool ok =
          __all_sync(0xFFFFFFFFu, mbar_wait(bar(kAcc), 0, abort_flag) && !*abort_flag);
      tc_fence_after();
      const int row = quarter * 32 + lane;  // W' row within the tile
      const uint32_t owner = static_cast<uint32_t>(row / kOwnRows);
      const uint32_t slot = sbase + kOffRed + rank * kSlotBytes +
                            static_cast<uint32_t>(row % kOwnRows) * static_cast<uint32_t>(ntok) * 4;
      const uint32_t dst = cluster_addr(slot, owner);
      for (int c = 0; c < ntok; c += 16) {
        uint32_t r[16];
        if (ok && nkb > 0) {
          tmem_ld16(tmem + (static_cast<uint32_t>(quarter * 32) << 16) + c, r);
        } else {
#pragma unroll
          for (int i = 0; i < 16; ++i) r[i] = 0u;  // empty slice: its partial sum is 0
        }
#pragma unroll
        for (int i = 0; i < 16; i += 4)
          st_cluster_v4f(dst + (c + i) * 4, __uint_as_float(r[i]), __uint_as_float(r[i + 1]),
                         __uint_as_float(r[i + 2]), __uint_as_float(r[i + 3]));
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync();  // every partial row has landed in its owner's slots
  // ------------------------------------------------------------ owner: reduce and store
  if (warp >= 2 && !*abort_flag) {
    typedef typename std::conditional<F16, __half, __nv_bfloat16>::type T;
    const float* red = reinterpret_cast<const float*>(smem + kOffRed);
    const unsigned short* bias = reinterpret_cast<const unsigned short*>(args.bias);
    const int nbase = n0 + static_cast<int>(rank) * kOwnRows;
    // pairs (m, 2p) .. (m, 2p+1) of this CTA's 16 rows: 8 pairs per token
    for (int idx = threadIdx.x - 64; idx < ntok * (kOwnRows / 2); idx += 32 * kDqWarps) {
      const int m = idx / (kOwnRows / 2), pr = 2 * (idx % (kOwnRows / 2));
      if (m0 + m >= args.M || nbase + pr >= args.N) continue;
      float v0 = 0.0f, v1 = 0.0f;
#pragma unroll
      for (int src = 0; src < kS; ++src) {  // fixed order
        v0 = __fadd_rn(v0, red[src * (kSlotBytes / 4) + pr * ntok + m]);
        v1 = __fadd_rn(v1, red[src * (kSlotBytes / 4) + (pr + 1) * ntok + m]);
      }
      if (bias != nullptr) {
        v0 = __fadd_rn(v0, F16 ? f16_bits_to_f32(bias[nbase + pr]) : bf16_bits_to_f32(bias[nbase + pr]));
        v1 = __fadd_rn(v1, F16 ? f16_bits_to_f32(bias[nbase + pr + 1])
                               : bf16_bits_to_f32(bias[nbase + pr + 1]));
      }
      *reinterpret_cast<uint32_t*>(reinterpret_cast<T*>(args.Y) +
                                   static_cast<int64_t>(m0 + m) * args.N + nbase + pr) =
          pack2_16<F16 ? kF16 : kBF16>(v0, v1);
    }
  }
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(skinny::kTmemCols)
                 : "memory");
  }
}

// ================================================================ decode kernel (M <= 16)
// For up to 16 tokens the product is bound by reading the packed weight (0.5 B per weight),
// not by the math, and the tensor-core operand round trip through shared memory of the
// kernels above costs more than the arithmetic. Here each warp dequantizes W' straight into
// the B fragments of the warp-level MMA (mma.sync m16n8k16, fp32 accumulation) in registers;
// the tokens are the MMA's M = 16 rows (zero rows past M) and X comes from shared memory.
//   * A warp owns 16 W' rows (2 n-tiles of 8) and a K-slice; 8 warps per CTA share the slice
//     (115 registers a thread: 2 CTAs, 16 warps per SM); a cluster of S CTAs (S = 1, 2, 4 or 8,
//     along x) splits K, one slice per CTA.
//   * k-blocks of 128: lane (g, t) (g = lane / 4, t = lane % 4) loads, per n-tile, the 16 code
//     bytes of row 8r + g at k = 32t .. 32t+31 (one group: t / 2) and that group's (scale,
//     zero); the loads of the next 4 k-blocks are in flight while one is converted.
//   * The contraction order inside a k-block is permuted (the same permutation on both
//     operands): MMA step s (0..7) takes k = 32t + 4s + {0, 1, 2, 3} at the k slots
//     {2t, 2t+1, 2t+8, 2t+9} that lane t holds, so each lane's 8 codes of one 32-bit word give
//     the B fragments of two steps and its X fragments are 16-byte pieces of one token row.
//     X is staged in shared memory with those pieces reordered so that the fragment loads are
//     free of bank conflicts (rows padded to 64 mod 128 bytes).
//   * Partial sums go over distributed shared memory to the CTA of the cluster that owns the
//     rows (128 / S rows each), which adds the S slots in rank order (deterministic), adds bias,
//     rounds once and stores. No waits other than the cluster barrier.
// Tile shape (compile-time): warps per CTA, n-tiles per warp, k-blocks in flight. The defaults
// were the best or equal among 4/8/16 warps, 1/2/4 n-tiles and 2/4 k-blocks on B200.
#ifndef HQQ_GEMV_WARPS
#define HQQ_GEMV_WARPS 8
#endif
#ifndef HQQ_GEMV_NT
#define HQQ_GEMV_NT 2
#endif
#ifndef HQQ_GEMV_DEPTH
#define HQQ_GEMV_DEPTH 4
#endif
// Where the next row tile's first code loads are issued: 1 = between the arrive and the wait of
// the tile's cluster barrier, 0 = before the barrier.
#ifndef HQQ_GEMV_SPLIT_SYNC
#define HQQ_GEMV_SPLIT_SYNC 1
#endif
// When the next kernel on the stream may launch (HQQ_FLAG_OVERLAP_WEIGHTS): 1 = after this
// kernel's last tile, 0 = at entry. At entry the dependent's persistent grid, sized for an idle
// GPU, started partly late and its clusters then carried several tiles each (measured slower,
// also when only the grids with one row tile per cluster triggered at entry).
#ifndef HQQ_GEMV_TRIGGER_LATE
#define HQQ_GEMV_TRIGGER_LATE 1
#endif

namespace gemv {
constexpr int kKB = 128;                     // k per k-block
constexpr int kDepth = HQQ_GEMV_DEPTH;       // k-blocks of codes in flight per warp
constexpr int kMaxKbPerSlice = 32;           // X tile <= 16 x 8256 B
constexpr int kMaxM = 16;
__host__ __device__ constexpr uint32_t x_row_bytes(int kb_per) { return kb_per * 256 + 64; }
// Tile shape: WARPS warps of NT n-tiles (8 W' rows each) per CTA.
template <int WARPS, int NT>
struct Shape {
  static constexpr int kWarps = WARPS;
  static constexpr int kThreads = 32 * WARPS;
  static constexpr int kNT = NT;
  static constexpr int kRowsCta = WARPS * NT * 8;
  static constexpr int kLgRowsCta =
      kRowsCta == 256 ? 8 : kRowsCta == 128 ? 7 : kRowsCta == 64 ? 6 : 5;
  static_assert((1 << kLgRowsCta) == kRowsCta, "power-of-two CTA rows");
  static constexpr uint32_t kRedBytes = kRowsCta * 16 * 4;
  static constexpr uint32_t smem_bytes(int kb_per) {
    return 16 * x_row_bytes(kb_per) + 2 * kRedBytes;  // X slice + two reduction buffers
  }
};
// The shapes built: 128-row tiles (the default), and 64-row tiles for layers so wide that the
// 128-row tiles outnumber the clusters that fit at once.
using Wide = Shape<HQQ_GEMV_WARPS, HQQ_GEMV_NT>;
using Narrow = Shape<4, 2>;
}  // namespace gemv

template <bool F16>
__device__ __forceinline__ void mma_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                          uint32_t a3, uint32_t b0, uint32_t b1) {
  if constexpr (F16) {
    asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
        "{%8, %9}, {%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
  } else {
    asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
        "{%8, %9}, {%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
  }
}

__device__ __forceinline__ void st_cluster_f32(uint32_t addr, float v) {
  asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(addr), "f"(v) : "memory");
}

// grid (S, ceil(N / 128)), cluster (S, 1, 1) with S = 2^lg_s; kb_per = k-blocks per slice;
// M <= 16.
template <bool F16, int MT, int WARPS, int NT>
__global__ void __launch_bounds__(32 * WARPS) w4a16_gemv_kernel(
    const void* __restrict__ X, const uint8_t* __restrict__ packed, const GemmArgs args,
    int lg_s, int kb_per) {
  using namespace gemv;
  using Sh = Shape<WARPS, NT>;
  constexpr int kWarps = Sh::kWarps, kThreads = Sh::kThreads, kNT = Sh::kNT;
  constexpr int kRowsCta = Sh::kRowsCta, kLgRowsCta = Sh::kLgRowsCta;
  constexpr uint32_t kRedBytes = Sh::kRedBytes;
  (void)kWarps;
  extern __shared__ __align__(16) uint8_t smem[];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int g = lane >> 2, t = lane & 3;
  const int rank = static_cast<int>(cluster_rank());
  const int M = args.M, N = args.N, K = args.K;
  const int nkb = (K + kKB - 1) / kKB;
  const int kb0 = rank * kb_per;
  const int nloc = max(0, min(kb_per, nkb - kb0));  // k-blocks of this slice
  const int n_tiles = (N + kRowsCta - 1) / kRowsCta;
  const int64_t row_bytes = K / 2, groups_per_row = K / 64;
  constexpr int kMsz = MT == kF32 ? 4 : 2;
  const uint8_t* sc_base = static_cast<const uint8_t*>(args.scale);
  const uint8_t* zr_base = static_cast<const uint8_t*>(args.zero);

  // this lane's n-tile rows (8r + g of the warp's 16) of row tile `tile` at the slice start:
  // code and meta pointers; invalid rows read nothing (codes and meta 0 -> W' = +0)
  const uint8_t* crow[kNT];
  const uint8_t* srow[kNT];
  const uint8_t* zrow[kNT];
  bool rin[kNT];
  auto set_rows = [&](int tile) {
#pragma unroll
    for (int r = 0; r < kNT; ++r) {
      const int row = tile * kRowsCta + warp * (kNT * 8) + 8 * r + g;
      rin[r] = row < N;
      crow[r] = packed + row * row_bytes + static_cast<int64_t>(kb0) * 64 + 16 * t;
      const int64_t gi = row * groups_per_row + 2 * static_cast<int64_t>(kb0) + (t >> 1);
      srow[r] = sc_base + gi * kMsz;
      zrow[r] = zr_base + gi * kMsz;
    }
  };

  uint4 code[kDepth][kNT];
  uint32_t msc[kDepth][kNT], mzr[kDepth][kNT];
  auto load_kb = [&](int i, uint4 (&c)[kNT], uint32_t (&s)[kNT], uint32_t (&z)[kNT]) {
    const bool kin = (kb0 + i) * kKB + 32 * t < K;  // K % 64 == 0: lane t's 32 k all in or out
#pragma unroll
    for (int r = 0; r < kNT; ++r) {
      if (kin && rin[r]) {
        c[r] = __ldg(reinterpret_cast<const uint4*>(crow[r] + i * 64));
        s[r] = meta_load<MT>(srow[r] + i * (2 * kMsz));
        z[r] = meta_load<MT>(zrow[r] + i * (2 * kMsz));
      } else {
        c[r] = make_uint4(0u, 0u, 0u, 0u);
        s[r] = 0u;
        z[r] = 0u;
      }
    }
  };
  auto load_first = [&]() {
#pragma unroll
    for (int i = 0; i < kDepth; ++i)
      if (i < nloc) load_kb(i, code[i], msc[i], mzr[i]);
  };

  // Programmatic dependent launch (HQQ_FLAG_OVERLAP_WEIGHTS): this kernel may start before the
  // previous one on the stream has finished; it loads its weight codes and meta (which no
  // earlier work writes, by the flag's promise) and then waits for the previous kernel's
  // completion and memory before it reads X or writes anything. It lets the next kernel
  // launch once its own tiles are done (HQQ_GEMV_TRIGGER_LATE). Without the launch attribute
  // these instructions are no-ops.
  int tile = static_cast<int>(blockIdx.y);
  if (!HQQ_GEMV_TRIGGER_LATE) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  set_rows(tile);
  load_first();
  asm volatile("griddepcontrol.wait;" ::: "memory");

  // X[0..15][slice] -> shared memory, once for every row tile of this CTA: 16-byte piece q
  // (k = 8q within the slice) of token m at m * rs + (q / 16) * 256 + (q % 4) * 64 +
  // ((q / 4) % 4) * 16; zeros past M and past K
  const uint32_t rs = x_row_bytes(kb_per);
  {
    // asynchronous 16-byte copies (all issued before one wait; 0 source bytes = zero fill);
    // thread = (token m = tid / kTpr, piece column tid % kTpr)
    constexpr int kTpr = kThreads / 16;
    const int m = threadIdx.x / kTpr;
    const int kc0 = kb0 * kKB;
    const bool mrow = m < M;
    const unsigned short* xrow = static_cast<const unsigned short*>(X) +
                                 (mrow ? static_cast<int64_t>(m) * K + kc0 : 0);
    const uint32_t xs = smem_u32(smem) + m * rs;
    for (int q = threadIdx.x % kTpr; q < kb_per * 16; q += kTpr) {
      const bool in = mrow && kc0 + 8 * q < K;
      const int kk = q & 15;
      const uint32_t dst = xs + (q >> 4) * 256 + (kk & 3) * 64 + (kk >> 2) * 16;
      asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst),
                   "l"(xrow + (in ? 8 * q : 0)), "r"(in ? 16 : 0)
                   : "memory");
    }
    asm volatile("cp.async.wait_all;" ::: "memory");
  }
  __syncthreads();

  const uint8_t* xa_row = smem + g * rs + t * 16;
  const uint8_t* xb_row = smem + (g + 8) * rs + t * 16;
  const int S = 1 << lg_s, lg_rpo = kLgRowsCta - lg_s, rpo = kRowsCta >> lg_s;
  typedef typename std::conditional<F16, __half, __nv_bfloat16>::type T;
  const unsigned short* bias = reinterpret_cast<const unsigned short*>(args.bias);

  // Row tiles blockIdx.y, blockIdx.y + gridDim.y, ... (the same sequence in every CTA of the
  // cluster, so all of them take the same barriers). The reduction slots alternate between
  // two buffers: a tile's partial sums are written after the barrier that ends the previous
  // tile, and its buffer is written again only two tiles later, after the barrier that the
  // owner passes once it has read it.
  for (int it = 0; tile < n_tiles; tile += static_cast<int>(gridDim.y), ++it) {
    float acc[kNT][4];
#pragma unroll
    for (int r = 0; r < kNT; ++r) acc[r][0] = acc[r][1] = acc[r][2] = acc[r][3] = 0.0f;

    for (int base = 0; base < nloc; base += kDepth) {
#pragma unroll
      for (int d = 0; d < kDepth; ++d) {
        const int i = base + d;
        if (i < nloc) {
          float2 nz2[kNT], sc2[kNT];
#pragma unroll
          for (int r = 0; r < kNT; ++r) {
            const float sc = meta_f32<MT>(msc[d][r]), z = meta_f32<MT>(mzr[d][r]);
            nz2[r] = make_float2(-z, -z);
            sc2[r] = make_float2(sc, sc);
          }
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            // word j: k = 32t + 8j .. +7 -> steps 2j (k +0..3) and 2j+1 (k +4..7)
            const uint4 xa = *reinterpret_cast<const uint4*>(xa_row + i * 256 + j * 64);
            const uint4 xb = *reinterpret_cast<const uint4*>(xb_row + i * 256 + j * 64);
#pragma unroll
            for (int r = 0; r < kNT; ++r) {
              const uint32_t w = j == 0 ? code[d][r].x : j == 1 ? code[d][r].y
                               : j == 2 ? code[d][r].z : code[d][r].w;
              const uint4 o = dequant8<F16>(w, nz2[r], sc2[r]);
              mma_16816<F16>(acc[r], xa.x, xb.x, xa.y, xb.y, o.x, o.y);
              mma_16816<F16>(acc[r], xa.z, xb.z, xa.w, xb.w, o.z, o.w);
            }
          }
          if (i + kDepth < nloc) load_kb(i + kDepth, code[d], msc[d], mzr[d]);
        }
      }
    }

    const int row_cta = tile * kRowsCta;
#if !HQQ_GEMV_SPLIT_SYNC
    if (tile + static_cast<int>(gridDim.y) < n_tiles) {
      set_rows(tile + static_cast<int>(gridDim.y));
      load_first();
    }
#endif

    // partial sums -> the owner CTA's slot for this rank:
    // red[(src * RPO + row_local) * 16 + m], buffer it & 1
    const uint32_t red_local = smem_u32(smem + 16 * rs + (it & 1) * kRedBytes);
#pragma unroll
    for (int r = 0; r < kNT; ++r) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int rho = warp * (kNT * 8) + 8 * r + 2 * t + (e & 1);
        const int m = g + 8 * (e >> 1);
        const int owner = rho >> lg_rpo, rl = rho & (rpo - 1);
        const uint32_t off = static_cast<uint32_t>(((rank * rpo + rl) * 16 + m) * 4);
        st_cluster_f32(cluster_addr(red_local + off, static_cast<uint32_t>(owner)), acc[r][e]);
      }
    }
#if HQQ_GEMV_SPLIT_SYNC
    // The barrier's release orders this thread's earlier loads too, so the next tile's first
    // codes are requested after the arrive: they are in flight during the wait and the
    // reduction instead of delaying the arrive until they return.
    cluster_arrive();
    if (tile + static_cast<int>(gridDim.y) < n_tiles) {
      set_rows(tile + static_cast<int>(gridDim.y));
      load_first();
    }
    cluster_wait();
#else
    cluster_sync();
#endif

    // owner: rows row_cta + rank * rpo .. + rpo - 1, every token < M, two rows per store
    const float* red = reinterpret_cast<const float*>(smem + 16 * rs + (it & 1) * kRedBytes);
    const int nbase = row_cta + rank * rpo;
    for (int idx = threadIdx.x; idx < (M << (lg_rpo - 1)); idx += kThreads) {
      const int m = idx >> (lg_rpo - 1), pr = 2 * (idx & ((rpo >> 1) - 1));
      if (nbase + pr >= N) continue;
      float v0 = 0.0f, v1 = 0.0f;
      for (int src = 0; src < S; ++src) {  // fixed order
        v0 = __fadd_rn(v0, red[(src * rpo + pr) * 16 + m]);
        v1 = __fadd_rn(v1, red[(src * rpo + pr + 1) * 16 + m]);
      }
      if (bias != nullptr) {
        v0 = __fadd_rn(v0, F16 ? f16_bits_to_f32(bias[nbase + pr]) : bf16_bits_to_f32(bias[nbase + pr]));
        v1 = __fadd_rn(v1, F16 ? f16_bits_to_f32(bias[nbase + pr + 1])
                               : bf16_bits_to_f32(bias[nbase + pr + 1]));
      }
      *reinterpret_cast<uint32_t*>(reinterpret_cast<T*>(args.Y) + static_cast<int64_t>(m) * N +
                                   nbase + pr) = pack2_16<F16 ? kF16 : kBF16>(v0, v1);
    }
  }
  // No remote write follows the last barrier (each CTA then reads only its own slots), so
  // the CTAs of the cluster may leave independently.
  if (HQQ_GEMV_TRIGGER_LATE) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
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

// 2-D row-major tensor map: `inner` elements per row (x), `outer` rows (y), box {bx, by}.
bool make_map(CUtensorMap* m, CUtensorMapDataType dt, size_t elem, const void* base,
              uint64_t inner, uint64_t outer, uint32_t bx, uint32_t by,
              CUtensorMapSwizzle swz) {
  PFN_cuTensorMapEncodeTiled_v12000 encode = tensor_map_encoder();
  if (encode == nullptr) return false;
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {inner * elem};
  const cuuint32_t box[2] = {bx, by};
  const cuuint32_t estr[2] = {1, 1};
  return encode(m, dt, 2, const_cast<void*>(base), dims, strides, box, estr,
                CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Clusters of S CTAs of `kernel` (`threads` a CTA, `smem` bytes of dynamic shared memory)
// that fit on the device at once (0 if the runtime cannot tell); cached per (kernel, S, smem).
int gemv_resident_clusters(const void* kernel, int S, uint32_t smem, int threads) {
  struct Entry { const void* k; int s; uint32_t smem; int n; };
  static std::mutex mu;
  static Entry cache[64];
  static int used = 0;
  std::lock_guard<std::mutex> lock(mu);
  for (int i = 0; i < used; ++i)
    if (cache[i].k == kernel && cache[i].s == S && cache[i].smem == smem) return cache[i].n;
  cudaLaunchConfig_t c = {};
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = static_cast<unsigned>(S);
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  c.attrs = at;
  c.numAttrs = 1;
  c.gridDim = dim3(static_cast<unsigned>(S), 1, 1);
  c.blockDim = dim3(static_cast<unsigned>(threads));
  c.dynamicSmemBytes = smem;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, kernel, &c) != cudaSuccess) {
    (void)cudaGetLastError();  // an unanswered query only means one cluster per row tile
    n = 0;
  }
  if (used < 64) cache[used++] = Entry{kernel, S, smem, n};
  return n;
}

template <bool F16, int MT, typename Sh>
cudaError_t set_gemv_smem() {
  return cudaFuncSetAttribute(w4a16_gemv_kernel<F16, MT, Sh::kWarps, Sh::kNT>,
                              cudaFuncAttributeMaxDynamicSharedMemorySize,
                              static_cast<int>(Sh::smem_bytes(gemv::kMaxKbPerSlice)));
}

// The decode kernel with tile shape Sh: one wave of clusters, each looping over row tiles.
template <bool F16, int MT, typename Sh>
cudaError_t launch_gemv(const GemmJob& job, const GemmArgs& a, cudaLaunchConfig_t* cfg, int S,
                        int lg_s, int kb_per) {
  cudaError_t e = set_gemv_smem<F16, MT, Sh>();
  if (e != cudaSuccess) return e;
  const uint32_t smem = Sh::smem_bytes(kb_per);
  const int64_t tiles = (job.N + Sh::kRowsCta - 1) / Sh::kRowsCta;
  const int resident = gemv_resident_clusters(
      reinterpret_cast<const void*>(&w4a16_gemv_kernel<F16, MT, Sh::kWarps, Sh::kNT>), S, smem,
      Sh::kThreads);
  const int64_t ny = resident > 0 && tiles > resident ? resident : tiles;
  cfg->blockDim = dim3(Sh::kThreads);
  cfg->dynamicSmemBytes = smem;
  cfg->gridDim = dim3(static_cast<unsigned>(S), static_cast<unsigned>(ny));
  const uint8_t* packed = job.packed;
  return cudaLaunchKernelEx(cfg, w4a16_gemv_kernel<F16, MT, Sh::kWarps, Sh::kNT>, job.X, packed,
                            a, lg_s, kb_per);
}

template <bool F16, int MT>
cudaError_t launch_typed(const GemmJob& job, cudaStream_t stream) {
  const CUtensorMapDataType xdt =
      F16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  GemmArgs a;
  a.scale = job.scale;
  a.zero = job.zero;
  a.bias = job.bias;
  a.Y = job.Y;
  a.M = static_cast<int>(job.M);
  a.N = static_cast<int>(job.N);
  a.K = static_cast<int>(job.K);
  cudaLaunchConfig_t cfg = {};
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  CUtensorMap mx, mw;
  const int nkb = static_cast<int>((job.K + gemv::kKB - 1) / gemv::kKB);
  const int S = nkb >= 16 ? 8 : nkb >= 8 ? 4 : nkb >= 4 ? 2 : 1;
  const int kb_per = (nkb + S - 1) / S;
  if (job.M <= gemv::kMaxM && kb_per <= gemv::kMaxKbPerSlice &&
      (job.N + gemv::Narrow::kRowsCta - 1) / gemv::Narrow::kRowsCta <= 65535) {
    attr[0].val.clusterDim.x = static_cast<unsigned>(S);
    if (job.overlap_weights) cfg.numAttrs = 2;  // the decode kernel waits before reading X
    const int lg_s = S == 8 ? 3 : S == 4 ? 2 : S == 2 ? 1 : 0;
    // 128-row tiles when one wave of clusters covers the rows (or nearly), 64-row tiles for
    // wider layers (measured: the 11008-row layers 30.7 -> 26.6 us, the 4096-row ones slower)
    const int64_t wide_tiles = (job.N + gemv::Wide::kRowsCta - 1) / gemv::Wide::kRowsCta;
    cudaError_t e = set_gemv_smem<F16, MT, gemv::Wide>();
    if (e != cudaSuccess) return e;
    const int wide_resident = gemv_resident_clusters(
        reinterpret_cast<const void*>(&w4a16_gemv_kernel<F16, MT, gemv::Wide::kWarps, gemv::Wide::kNT>),
        S, gemv::Wide::smem_bytes(kb_per), gemv::Wide::kThreads);
    if (wide_resident > 0 && wide_tiles > wide_resident)
      return launch_gemv<F16, MT, gemv::Narrow>(job, a, &cfg, S, lg_s, kb_per);
    return launch_gemv<F16, MT, gemv::Wide>(job, a, &cfg, S, lg_s, kb_per);
  }
  if (job.M <= skinny::kMaxM) {
    const int ntok = static_cast<int>(
        (std::min<int64_t>(job.M, skinny::kTokMax) + 15) / 16 * 16);
    if (!make_map(&mx, xdt, 2, job.X, job.K, job.M, kBK, ntok, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map(&mw, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, job.packed, job.K / 2, job.N,
                  kBK / 2 * skinny::kSub, skinny::kRows, CU_TENSOR_MAP_SWIZZLE_NONE))
      return cudaErrorInvalidValue;
    const uint32_t smem = skinny::layout(ntok).bytes;
    cudaError_t e = cudaFuncSetAttribute(w4a16_skinny_kernel<F16, MT>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(skinny::layout(skinny::kTokMax).bytes));
    if (e != cudaSuccess) return e;
    cfg.gridDim = dim3(skinny::kS * static_cast<unsigned>((job.N + skinny::kRows - 1) / skinny::kRows),
                       static_cast<unsigned>((job.M + skinny::kTokMax - 1) / skinny::kTokMax));
    cfg.blockDim = dim3(skinny::kThreads);
    cfg.dynamicSmemBytes = smem;
    attr[0].val.clusterDim.x = skinny::kS;
    return cudaLaunchKernelEx(&cfg, w4a16_skinny_kernel<F16, MT>, mx, mw, a, ntok);
  }
  CUtensorMap my;
  if (!make_map(&mx, xdt, 2, job.X, job.K, job.M, kBK, 128, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_map(&mw, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, job.packed, job.K / 2, job.N, kBK / 2,
                sm2::kRows, CU_TENSOR_MAP_SWIZZLE_NONE) ||
      !make_map(&my, xdt, 2, job.Y, job.N, job.M, 32, 32, CU_TENSOR_MAP_SWIZZLE_64B))
    return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(w4a16_gemm_2sm_kernel<F16, MT>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(sm2::kSmemBytes));
  if (e != cudaSuccess) return e;
  cfg.gridDim = dim3(2 * static_cast<unsigned>((job.M + 511) / 512),
                     static_cast<unsigned>((job.N + kBN - 1) / kBN));
  cfg.blockDim = dim3(sm2::kThreads);
  cfg.dynamicSmemBytes = sm2::kSmemBytes;
  attr[0].val.clusterDim.x = 2;
  return cudaLaunchKernelEx(&cfg, w4a16_gemm_2sm_kernel<F16, MT>, mx, mw, my, a);
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
