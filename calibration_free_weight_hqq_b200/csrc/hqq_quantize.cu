// hqq_quantize.cu - the HQQ solver kernel for sm_100a.
//
// What it computes (per group of G weights; the pages give no equations, so this is the
// plainest reading of "HQQ calibration-free guide" (lnwmold.com) §2.1, "HQQ tutorial"
// (devpress.csdn.net) §2 and §3.3 and "Dropbox HQQ analysis" (ainews.cool), technical deep
// dive): min/max round-to-nearest init, then iters+1 evaluations of candidate zeros, each
// scored by the lp error sum|r|^p, with the lp generalised soft-threshold of the residual
// (auxiliary error variable) and the closed-form mean zero update between evaluations,
// beta *= kappa, and the earliest best candidate kept. Final codes are bit-packed and the
// scale (the quantization step) and zero written once.
//
// How it maps to B200:
//   * A lane owns E = min(G, 32) consecutive weights of a group; L = G/E adjacent lanes
//     share a group and combine sums with shuffles. The group's scaled weights Ws = w*s
//     (fp32) and raw weights (two 16-bit values per register) stay in registers for all
//     iterations, so HBM sees one read of W and one write of the packed codes and meta: the
//     kernel is bound by the MUFU (lg2/ex2 of |r|^p) and issue rate, not by memory.
//   * Per element and evaluation: v = Ws + z, round-half-even by the 1.5*2^23 magic add
//     (FMA pipe), r = w - (Q - z)*step with the definition's roundings (so residuals are
//     bit-identical to the definition's), MUFU lg2 + ex2 for |r|^p, four partial sums of the
//     error (only comparisons use it), the code sum. The clamp to [0, qmax] is skipped when
//     a warp vote shows that no element of the warp's groups can leave the code range
//     (v is monotone in Ws, so the group's extreme values decide). p == 1 skips the MUFU.
//   * Shrinkage: We_j is nonzero only where |r_j| > beta^(-1/(2-p)). A per-group bound on
//     max|r_j| (from the group's min/max and the zero, no per-element work) proves We == 0
//     exactly for almost every group and iteration; otherwise a per-element path computes
//     We exactly as the definition does (fp32; the power is the fp64 power rounded once;
//     fp64 sum).
//   * The zero update uses the same fp64 expression as the definition,
//     z = fp32(((double)sumQ - (double)sum(Ws) + (double)s*sum(We)) / G), with sumQ exact in
//     fp32, so given identical codes the zero is bit-identical whatever the summation order.
//   * Packing: 8/4/2/1-bit codes are packed in registers and stored with 4..16-byte stores;
//     3-bit codes (10 per 32-bit word, crossing group boundaries) are staged in shared memory
//     per block (160*E codes, a multiple of 10) and emitted as whole words.
#include "hqq_quantize_impl.cuh"

namespace hqqk {

// Defined in hqq_quantize_stop.cu: the same launches with the fixed-point stop compiled in.
cudaError_t launch_quantize_stop(const QuantJob* jobs, int n, bool batched, cudaStream_t st);

cudaError_t launch_quantize(const QuantJob& j, cudaStream_t st) {
  if (j.flags & 1) return launch_quantize_stop(&j, 1, false, st);
  return launch_batch<1, false>(&j, 1, st);
}

cudaError_t launch_quantize_batched(const QuantJob* jobs, int n, cudaStream_t st) {
  if (n > 0 && (jobs[0].flags & 1)) return launch_quantize_stop(jobs, n, true, st);
  for (int i = 0; i < n; i += kMaxBatch) {
    const int k = n - i < kMaxBatch ? n - i : kMaxBatch;
    const cudaError_t e = launch_batch<kMaxBatch, false>(jobs + i, k, st);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace hqqk
