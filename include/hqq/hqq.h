/*
 * hqq.h - C ABI of the calibration-free HQQ (Half-Quadratic Quantization) weight
 * quantize / dequantize path, written for NVIDIA B200 (sm_100a).
 *
 * What the operation is (sources, by page title and section):
 *   - "HQQ calibration-free guide" (lnwmold.com) §2.1: HQQ needs no calibration data; it
 *     splits the hard, non-convex quantization problem into two simpler sub-problems that
 *     are solved alternately through an auxiliary variable.
 *   - same page §2.2: nbits in {8,4,3,2,1}; group_size = weights per group sharing one
 *     scale/zero; axis selects the direction groups run along a [out_features,in_features]
 *     weight.
 *   - same page §3.2: a quantized layer keeps packed low-bit weights (`unpack(dtype=uint8)`)
 *     and can `dequantize()` back to the compute dtype.
 *   - "hqq-quantization skill summary" (nav.superapi.store), usage paragraph: the results
 *     of quantization are W_q, scale and zero, and dequantize() reconstructs W.
 *   - "HQQ tutorial" (devpress.csdn.net) §3.3: quant_zero / quant_scale quantize the zero
 *     and scale themselves with a higher precision such as 8 bits.
 * The pages print no solver formula. The solver computed here is the plainest reading of
 * their description, written out in full in the comment on hqq_quantize below.
 *
 * Conventions for every entry point
 *   Ownership  The caller owns every buffer. Nothing here allocates, frees or synchronises
 *              device memory or streams; all device work is enqueued on `stream`.
 *   Pointers   Arguments documented "device" must be device (or managed) memory on the
 *              current device. Before it launches, each call checks its first device
 *              argument (W, Wq_packed, X, meta, codes or Y) with cudaPointerGetAttributes
 *              and returns HQQ_ERR_INVALID_ARG when that buffer lives on another device or
 *              is pageable host memory; the other buffers of a call are the caller's
 *              responsibility (host pointers there are undefined behaviour).
 *   Errors     Argument errors are returned synchronously before any launch, and nothing
 *              is written. When there is nothing to do (rows*cols == 0, n == 0) a call with
 *              otherwise valid arguments returns HQQ_OK at once; its pointers may be NULL.
 *              A failed launch returns HQQ_ERR_CUDA (the CUDA error string is available
 *              from hqq_last_cuda_error()). Nothing throws across this ABI.
 *   Threads    All entry points are re-entrant. hqq_last_cuda_error() is thread-local.
 *
 * Packed code layout (fixed here; the pages fix none)
 *   Group order g:  axis=1: g = r*(cols/gs) + cb, group elements W[r, cb*gs + j]
 *                   axis=0: g = rb*cols + c,      group elements W[rb*gs + j, c]
 *   scale/zero are arrays of n_groups values in g order (row-major [rows, cols/gs] for
 *   axis=1, [rows/gs, cols] for axis=0).
 *   Code stream:    code k = g*gs + j (row-major W order for axis=1).
 *     nbits 8,4,2,1: code k sits in byte k/(8/nbits), bits [(k%(8/nbits))*nbits, +nbits),
 *                    least significant first.
 *     nbits 3:       code k sits in the little-endian 32-bit word k/10, bits [(k%10)*3, +3);
 *                    bits 30..31 and unused tail slots are zero.
 *   Second level (quant_scale / quant_zero): the n_groups meta values, in g order, are cut
 *   into runs of meta_group_size consecutive values (the last run may be short). Each run
 *   has uint8 codes and one fp32 pair (step2, zero2), stored interleaved as
 *   mm[2*i] = step2, mm[2*i+1] = zero2.
 */
#ifndef HQQ_HQQ_H_
#define HQQ_HQQ_H_

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

#define HQQ_ABI_VERSION 5

typedef enum {
  HQQ_OK = 0,
  HQQ_ERR_INVALID_ARG = 1, /* null pointer, negative size, p/beta0/kappa out of range */
  HQQ_ERR_UNSUPPORTED = 2, /* nbits, group_size, axis or dtype outside the supported set */
  HQQ_ERR_SHAPE = 3,       /* grouped dimension not divisible by group_size, or too large */
  HQQ_ERR_ALIGNMENT = 4,   /* a pointer is not aligned as documented */
  HQQ_ERR_CUDA = 5,        /* a CUDA launch or runtime call failed */
  HQQ_ERR_WORKSPACE = 6    /* workspace missing or smaller than hqq_workspace_bytes() */
} hqq_status;

typedef enum { HQQ_F16 = 0, HQQ_BF16 = 1, HQQ_F32 = 2, HQQ_U8 = 3 } hqq_dtype;

/* Supported set (checked on every call):
 *   nbits       1, 2, 3, 4, 8
 *   group_size  8, 16, 32, 64, 128, 256
 *   axis        0 or 1
 *   iters       0 .. HQQ_MAX_ITERS
 *   p           0 < p <= 1;  beta0 > 0 and finite;  kappa >= 1 and finite
 *   W dtype     HQQ_F16, HQQ_BF16, HQQ_F32;  meta dtype HQQ_F16, HQQ_BF16, HQQ_F32
 *   meta_group_size (second level) 8 .. 1024 */
#define HQQ_MAX_ITERS 1000

/* Quantization parameters; mirrors BaseQuantizeConfig(nbits, group_size, quant_zero,
 * quant_scale, axis) of the "HQQ tutorial" (devpress.csdn.net) §3.3, plus the solver
 * constants p (lp exponent), beta0 (initial penalty) and kappa (penalty growth). */
typedef struct {
  int nbits;
  int group_size;
  int axis;
  int iters;
  float p;
  float beta0;
  float kappa;
  hqq_dtype w_dtype;    /* dtype of W (input of quantize) */
  hqq_dtype meta_dtype; /* dtype of first-level scale/zero when they are not quantized */
  int quant_scale;      /* nonzero: scale is stored as uint8 codes + fp32 (step2, zero2) */
  int quant_zero;       /* nonzero: zero is stored as uint8 codes + fp32 (step2, zero2) */
  int meta_group_size;  /* run length of the second level (128 in the shipped workloads) */
  int flags;            /* HQQ_FLAG_* bits (0: none) */
} hqq_params;

/* Stop a group's iterations once they can only repeat themselves: when an update returns the
 * zero bit-for-bit unchanged and the group's residual bound proves that the shrinkage stays
 * zero for every remaining update, every later evaluation reproduces the last one exactly
 * (same codes, same error, no new best), so the results are bit-identical to running all
 * iters. Applied per warp of groups (a warp stops when all its groups have settled). Off by
 * default: with it, the work done depends on the data rather than being iters+1
 * evaluations per group. */
#define HQQ_FLAG_STOP_AT_FIXED_POINT 1

/* hqq_linear only (the quantize entry points refuse it): the caller promises that no work
 * enqueued earlier on the stream, and possibly still running, writes this call's weight
 * (Wq_packed, scale, zero) - as in a sequence of decode steps over weights quantized and
 * synchronised beforehand. The decode kernel (M <= 16) may then start while the previous
 * kernel on the stream is finishing (programmatic dependent launch): it loads its weight codes
 * and meta first and waits for the previous kernel to complete, with its writes visible,
 * before it reads X, bias or anything else and before it writes Y. Results are identical with
 * or without the flag; other kernels ignore it. Without the promise (say, a quantize call just
 * before on the same stream), leave it off. */
#define HQQ_FLAG_OVERLAP_WEIGHTS 2

/* Number of quantization groups of a [rows, cols] weight: rows*cols/group_size.
 * Returns -1 if the grouped dimension (cols for axis=1, rows for axis=0) is not a multiple
 * of group_size or an argument is out of range. Host only; no CUDA call. */
int64_t hqq_num_groups(int64_t rows, int64_t cols, int group_size, int axis);

/* Bytes of the packed code stream for rows*cols codes (layout above):
 * ceil(N*nbits/8) for nbits 8,4,2,1 and 4*ceil(N/10) for nbits 3. Returns 0 for an
 * unsupported nbits or a negative size. Host only. */
size_t hqq_packed_bytes(int64_t rows, int64_t cols, int nbits, int group_size, int axis);

/* Number of second-level runs for n meta values: ceil(n / meta_group_size). Host only. */
int64_t hqq_num_meta_groups(int64_t n, int meta_group_size);

/* Device workspace hqq_quantize_ex needs for these arguments, in bytes (0 when neither
 * quant_scale nor quant_zero is set). Host only. Returns (size_t)-1 on invalid params. */
size_t hqq_workspace_bytes(int64_t rows, int64_t cols, const hqq_params* params);

/* Quantize one weight matrix with the HQQ solver.
 *
 * Per group of gs weights w_0..w_{gs-1} (upcast to fp32), with qmax = 2^nbits - 1:
 *   1. min/max round-to-nearest init: mn, mx; s = qmax/(mx-mn), step = (mx-mn)/qmax
 *      (s = step = 1 when mx == mn); z = -mn*s; Ws_j = w_j*s.
 *   2. iters+1 evaluations k = 0..iters of the candidate zero z_k (z_0 is the RTN zero):
 *      codes Q_j = clamp(rint(Ws_j + z_k), 0, qmax) (round half to even), residual
 *      r_j = w_j - (Q_j - z_k)*step, lp error e_k = sum_j |r_j|^p. The first candidate
 *      with the smallest e_k is kept (best-error tracking).
 *   3. after evaluations 0..iters-1, the auxiliary error variable is the lp generalised
 *      soft-threshold of the residual, We_j = sign(r_j)*max(|r_j| - |r_j|^(p-1)/beta_k, 0),
 *      the zero is updated in closed form as a group mean,
 *      z_{k+1} = mean_j(Q_j - Ws_j + s*We_j), and beta_{k+1} = beta_k*kappa (beta_0 = beta0).
 *   4. final codes Q*_j = clamp(rint(Ws_j + z_best), 0, qmax); scale = step; zero = z_best.
 *   Dequantization is then W'_j = (Q*_j - zero)*scale.
 * Sources: auxiliary variable and alternating minimisation, "HQQ calibration-free guide"
 * (lnwmold.com) §2.1 and "Dropbox HQQ analysis" (ainews.cool), technical deep dive; a
 * loss that is lenient on small errors and protects outliers, "HQQ tutorial"
 * (devpress.csdn.net) §2. The exact steps above are this library's reading of those
 * passages (the pages give no equations).
 *
 * W          device, row-major [rows, cols] of `dtype` (F16, BF16 or F32), 16-byte aligned.
 * Wq_packed  device, hqq_packed_bytes(...) bytes, 16-byte aligned; fully overwritten.
 * scale,zero device, n_groups values each of `dtype` (meta dtype = W dtype), naturally
 *            aligned; written in g order.
 * Requires cols % group_size == 0 (axis=1) or rows % group_size == 0 (axis=0), and
 * rows*cols < 2^40. The result is deterministic (bitwise identical run to run). */
hqq_status hqq_quantize(const void* W, hqq_dtype dtype, int64_t rows, int64_t cols, int nbits,
                        int group_size, int axis, int iters, float p, float beta0, float kappa,
                        void* Wq_packed, void* scale, void* zero, cudaStream_t stream);

/* Dequantize: W_out[...] = (float(Q) - zero)*scale in fp32, rounded once (to nearest even)
 * to `out_dtype`. ("HQQ calibration-free guide" (lnwmold.com) §3.2, dequantize().)
 * Wq_packed  device, layout above. scale, zero: device, n_groups values of `meta_dtype`.
 * W_out      device, row-major [rows, cols] of out_dtype (F16, BF16, F32), 16-byte aligned. */
hqq_status hqq_dequantize(const void* Wq_packed, const void* scale, const void* zero,
                          hqq_dtype meta_dtype, hqq_dtype out_dtype, int64_t rows, int64_t cols,
                          int nbits, int group_size, int axis, void* W_out, cudaStream_t stream);

/* Quantize with the full parameter set, including the second level of the "HQQ tutorial"
 * (devpress.csdn.net) §3.3 (quant_scale / quant_zero: 8-bit min/max round-to-nearest of
 * the fp32 scale and zero values, runs of meta_group_size values in g order).
 * scale      device. quant_scale == 0: n_groups values of params->meta_dtype.
 *                    quant_scale != 0: n_groups uint8 codes.
 * zero       device, likewise with quant_zero.
 * scale_mm   device fp32 [n_meta_groups][2] (step2, zero2) when quant_scale, else ignored.
 * zero_mm    device fp32 [n_meta_groups][2] when quant_zero, else ignored.
 * workspace  device, >= hqq_workspace_bytes(...) bytes, 16-byte aligned (may be NULL when
 *            that size is 0). Its contents on entry do not matter and on exit are undefined.
 *            Two calls that use the same workspace concurrently race. */
hqq_status hqq_quantize_ex(const void* W, int64_t rows, int64_t cols, const hqq_params* params,
                           void* Wq_packed, void* scale, void* zero, void* scale_mm, void* zero_mm,
                           void* workspace, size_t workspace_bytes, cudaStream_t stream);

/* Size of the fixed device scratch that hqq_quantize_ex_noalloc uses in place of a workspace:
 * 32 MiB, enough for 4,194,304 groups when both quant_scale and quant_zero are set and
 * 8,388,608 groups when one of them is. */
#define HQQ_NOALLOC_SCRATCH_BYTES ((size_t)32 << 20)

/* hqq_quantize_ex for callers that cannot allocate device memory. (The pages have no
 * counterpart; this is a deployment convenience of this library.)
 * Some callers can't call cudaMalloc: a plugin or extension that its host framework hands
 * only a stream and the tensors, code that runs where every byte of device memory belongs to
 * another allocator (a caching allocator or a fixed-size pool), or a serving process that
 * forbids allocation once it has started. The second level needs fp32 scratch for the scale
 * and zero of every group; this entry point takes it from a fixed array compiled into the
 * library instead of a caller-supplied workspace, and calls no allocating routine.
 *   Arguments, outputs and results are those of hqq_quantize_ex without the workspace; the
 *   arguments are checked first, exactly as hqq_quantize_ex checks them, so an invalid call
 *   returns the same status through either entry point.
 *   The array holds HQQ_NOALLOC_SCRATCH_BYTES; a valid call that needs more
 *   (hqq_workspace_bytes() > HQQ_NOALLOC_SCRATCH_BYTES) returns HQQ_ERR_WORKSPACE and
 *   launches nothing. Calls without quant_scale/quant_zero use no scratch.
 *   Every GPU that loads the array holds it (32 MiB) until the process exits.
 *   The first call on a device sets up the array's device address for that device (a host
 *   runtime query, with the device current); make that first call before any stream capture.
 *   If that query fails the call returns HQQ_ERR_CUDA and hqq_last_cuda_error() names the
 *   error. The address is kept for the life of the process: after cudaDeviceReset() (or
 *   anything else that replaces the device's primary context) this entry point must not be
 *   called again in that process.
 *   All calls on a device share the one array and it keeps the last call's contents (each
 *   call writes the parts it reads first, so nothing needs clearing). Calls that overlap on
 *   the GPU - on different streams, or from different host threads, at the same time on one
 *   device - race on it: keep such calls ordered, e.g. on one stream. */
hqq_status hqq_quantize_ex_noalloc(const void* W, int64_t rows, int64_t cols,
                                   const hqq_params* params, void* Wq_packed, void* scale,
                                   void* zero, void* scale_mm, void* zero_mm,
                                   cudaStream_t stream);

/* Inverse of hqq_quantize_ex. When quant_scale (quant_zero) is set, the scale (zero) of each
 * group is first rebuilt in fp32 as (code - zero2)*step2 of its run, and that fp32 value is
 * used directly. W_out as in hqq_dequantize. */
hqq_status hqq_dequantize_ex(const void* Wq_packed, const void* scale, const void* zero,
                             const void* scale_mm, const void* zero_mm, int64_t rows, int64_t cols,
                             const hqq_params* params, hqq_dtype out_dtype, void* W_out,
                             cudaStream_t stream);

/* One matrix of a batched call. */
typedef struct {
  void* W;          /* device, row-major [rows, cols]: quantize reads it (params->w_dtype);
                       dequantize writes it (out_dtype). 16-byte aligned. */
  int64_t rows, cols;
  void* Wq_packed;  /* device, hqq_packed_bytes(rows, cols, ...) bytes, 16-byte aligned */
  void* scale;      /* device, rows*cols/group_size values of params->meta_dtype */
  void* zero;       /* device, likewise */
} hqq_matrix;

/* Quantize n matrices that share one configuration (params: nbits, group_size, axis, solver
 * constants, w_dtype, meta_dtype; quant_scale/quant_zero must be 0) with as few launches as
 * possible: up to 256 matrices per launch, their pointers and shapes passed as kernel
 * parameters, so one tail instead of one per matrix and no device allocation. Shapes may
 * differ. Each matrix's results are identical to hqq_quantize_ex on it alone. This is the
 * whole-model driver: a model with per-layer configurations ("HQQ tutorial"
 * (devpress.csdn.net) §4.2 layer_configs; "HQQ calibration-free guide" (lnwmold.com) §3.4)
 * makes one call per configuration. mats: host array of n descriptors (copied before the
 * call returns). Every matrix is validated before anything is launched. */
hqq_status hqq_quantize_batched(const hqq_matrix* mats, int n, const hqq_params* params,
                                cudaStream_t stream);

/* Dequantize n matrices of one configuration into their W fields (out_dtype), batched like
 * hqq_quantize_batched; results identical to hqq_dequantize_ex per matrix. */
hqq_status hqq_dequantize_batched(const hqq_matrix* mats, int n, const hqq_params* params,
                                  hqq_dtype out_dtype, cudaStream_t stream);

/* Per-layer mixed precision in one call: matrix i is quantized with its own configuration
 * params[i] (host array of n). The pages configure layers by name pattern - 8-bit group 128 for
 * the first block and the output head, 4-bit group 64 elsewhere ("HQQ tutorial"
 * (devpress.csdn.net) §4.2, layer_configs) - or by layer type, e.g. 4-bit attention and 2-bit
 * MLP weights ("hqq-quantization skill summary" (nav.superapi.store), dynamic_config).
 * Matrices whose configurations are equal in every field form one group; the groups are
 * issued in order of first appearance, each as hqq_quantize_batched (same rules:
 * quant_scale/quant_zero must be 0, up to 256 matrices per launch), so a model with k
 * distinct configurations takes k batched launches (more only past 256 matrices a group).
 * Each matrix's results are identical to hqq_quantize_ex with its configuration. Every matrix
 * and configuration is validated before anything is launched; on an invalid argument nothing
 * is launched. */
hqq_status hqq_quantize_mixed(const hqq_matrix* mats, const hqq_params* params, int n,
                              cudaStream_t stream);

/* Inverse of hqq_quantize_mixed: matrix i dequantized with params[i] into its W field
 * (out_dtype), grouped and launched like hqq_quantize_mixed; results identical to
 * hqq_dequantize_ex per matrix. */
hqq_status hqq_dequantize_mixed(const hqq_matrix* mats, const hqq_params* params, int n,
                                hqq_dtype out_dtype, cudaStream_t stream);

/* Host only (no device work): the grouping hqq_quantize_mixed / hqq_dequantize_mixed use.
 * group_of (host array of n ints) receives, for each matrix, the index of its configuration
 * group, numbered by first appearance; *n_groups their count. HQQ_ERR_INVALID_ARG on n < 0 or
 * a null pointer that n requires. */
hqq_status hqq_mixed_plan(const hqq_params* params, int n, int* group_of, int* n_groups);

/* Second level on its own: 8-bit min/max round-to-nearest of n fp32/f16/bf16 values `meta`
 * (device) in runs of `group` values ("HQQ tutorial" (devpress.csdn.net) §3.3). Per run:
 * step2 = (max-min)/255, s2 = 255/(max-min) (both 1 when max == min), zero2 = -min*s2,
 * q = clamp(rint(m*s2 + zero2), 0, 255). q_u8: device, n bytes. mm: device fp32 [runs][2]. */
hqq_status hqq_quantize_meta(const void* meta, hqq_dtype dtype, int64_t n, int group, void* q_u8,
                             void* mm, cudaStream_t stream);

/* out_f32[i] = (q_u8[i] - zero2)*step2 of its run, in fp32. All pointers device. */
hqq_status hqq_dequantize_meta(const void* q_u8, const void* mm, int64_t n, int group,
                               void* out_f32, cudaStream_t stream);

/* The consumer of the packed format: the forward pass of an HQQ-quantized linear layer,
 *     Y[m, n] = dtype( sum_k X[m, k] * W'[n, k]  (+ bias[n]) ),
 * with W' the dequantized weight rounded once to the activation dtype exactly as
 * hqq_dequantize writes it, W'[n, k] = dtype((float(Q[n, k]) - zero[g]) * scale[g]),
 * g = n*(K/64) + k/64, and the sum accumulated in fp32 on the tensor cores ("HQQ
 * calibration-free guide" (lnwmold.com) §3.2: a quantized layer computes in its compute
 * dtype from the dequantized weight; §4.2: the axis=1 backends fuse the dequantization
 * into the matrix product). The dequantized weight is never written to memory.
 *   X          device, row-major [M, K] of x_dtype (HQQ_BF16 or HQQ_F16), 16-byte aligned.
 *   Wq_packed, scale, zero
 *              the outputs of hqq_quantize / hqq_quantize_ex for W of shape [N, K]
 *              (rows = N output features, cols = K input features) with params->nbits 4,
 *              group_size 64, axis 1 and no second level; scale and zero are
 *              params->meta_dtype (F16, BF16 or F32). Wq_packed 16-byte aligned.
 *   bias       NULL or device [N] of x_dtype.
 *   Y          device, row-major [M, N] of x_dtype, 16-byte aligned; must not overlap the
 *              inputs.
 * Shapes: K % 64 == 0 and N % 8 == 0 (HQQ_ERR_SHAPE otherwise), M, K < 2^31, N <= 65535*256.
 * K == 0 gives
 * Y = bias (or 0). Other nbits / group_size / axis, or quant_scale / quant_zero, return
 * HQQ_ERR_UNSUPPORTED. The solver fields of params are ignored; params->flags may hold
 * HQQ_FLAG_OVERLAP_WEIGHTS (and HQQ_FLAG_STOP_AT_FIXED_POINT, ignored), other bits return
 * HQQ_ERR_INVALID_ARG. */
hqq_status hqq_linear(const void* X, int64_t M, int64_t K, hqq_dtype x_dtype,
                      const void* Wq_packed, const void* scale, const void* zero,
                      const void* bias, int64_t N, const hqq_params* params, void* Y,
                      cudaStream_t stream);

/* MXFP4 weight-only encoding ("HQQ calibration-free guide" (lnwmold.com) §5.1 lists an
 * mxfp4 weight-only mode; the encoding is the Open Compute Project Microscaling format
 * MXFP4). W: device, row-major [rows, cols] of dtype (F16, BF16 or F32), 16-byte aligned,
 * finite values; cols % 32 == 0 (HQQ_ERR_SHAPE otherwise). Blocks of 32 consecutive elements
 * of a row share one scale 2^e, e = floor(log2(max |v|)) - 2 clamped to [-127, 127] (an
 * all-zero block takes -127), written as the byte e + 127 to scales[block] (block = r*cols/32
 * + c/32; rows*cols/32 bytes). Each element is v / 2^e rounded to the nearest FP4 E2M1 value
 * (magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6; ties to the even mantissa bit; above 6 saturates to
 * 6; sign kept), as a 4-bit code sign<<3 | magnitude index, two per byte with element 2j in
 * the low nibble (codes: rows*cols/2 bytes, 4-byte aligned). */
hqq_status hqq_mxfp4_quantize(const void* W, hqq_dtype dtype, int64_t rows, int64_t cols,
                              void* codes, void* scales, cudaStream_t stream);

/* W_out[k] = E2M1 value of code k * 2^(scales[k/32] - 127), computed exactly and rounded once
 * to out_dtype (F16, BF16 or F32); W_out: device [rows, cols], 16-byte aligned. */
hqq_status hqq_mxfp4_dequantize(const void* codes, const void* scales, int64_t rows,
                                int64_t cols, hqq_dtype out_dtype, void* W_out,
                                cudaStream_t stream);

/* Kernels that wait on barriers inside a CTA (hqq_linear) bound each wait by about two
 * seconds; a wait that runs out sets the CTA's outputs aside (not written), frees its
 * resources and is counted. *count receives the number counted since the library was
 * loaded on the current device (0 on every healthy run). Synchronises the device. */
hqq_status hqq_wait_timeouts(unsigned int* count);

/* Human-readable name of a status code (static storage). */
const char* hqq_status_string(hqq_status status);

/* Message of the last CUDA error seen by this thread inside the library ("" if none). */
const char* hqq_last_cuda_error(void);

/* HQQ_ABI_VERSION of the loaded library. */
int hqq_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* HQQ_HQQ_H_ */
