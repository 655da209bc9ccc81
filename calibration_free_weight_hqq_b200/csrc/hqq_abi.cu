// hqq_abi.cu - extern "C" entry points of libhqq_b200.so: argument validation (pure host
// arithmetic, no CUDA call before the arguments are known to be valid) and dispatch to the
// kernels. Declarations and the full contract are in include/hqq/hqq.h.
#include <math.h>
#include <stdio.h>
#include <string.h>

#include <vector>

#include "../../include/hqq/hqq.h"
#include "hqq_abi_internal.h"
#include "hqq_kernels.h"

#define HQQ_EXPORT extern "C" __attribute__((visibility("default")))

static_assert((int)HQQ_F16 == hqqk::kF16 && (int)HQQ_BF16 == hqqk::kBF16 &&
                  (int)HQQ_F32 == hqqk::kF32 && (int)HQQ_U8 == hqqk::kU8,
              "dtype enumerators must match");

namespace {
thread_local char g_last_cuda_error[256] = "";
}  // namespace

hqq_status hqqabi::cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return HQQ_OK;
  snprintf(g_last_cuda_error, sizeof(g_last_cuda_error), "%s: %s", cudaGetErrorName(e),
           cudaGetErrorString(e));
  return HQQ_ERR_CUDA;
}

hqq_status hqqabi::check_device(const void* p) {
  cudaPointerAttributes at;
  cudaError_t e = cudaPointerGetAttributes(&at, p);
  if (e != cudaSuccess) return cuda_status(e);
  if (at.type == cudaMemoryTypeUnregistered) return HQQ_ERR_INVALID_ARG;  // pageable host
  if (at.type != cudaMemoryTypeDevice) return HQQ_OK;  // pinned host or managed memory
  int dev = -1;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return cuda_status(e);
  return at.device == dev ? HQQ_OK : HQQ_ERR_INVALID_ARG;
}

using hqqabi::check_device;
using hqqabi::cuda_status;

namespace {

constexpr int64_t kMaxElems = int64_t(1) << 40;

bool nbits_ok(int nbits) {
  return nbits == 1 || nbits == 2 || nbits == 3 || nbits == 4 || nbits == 8;
}
bool group_ok(int g) { return g == 8 || g == 16 || g == 32 || g == 64 || g == 128 || g == 256; }
bool wdtype_ok(int dt) { return dt == HQQ_F16 || dt == HQQ_BF16 || dt == HQQ_F32; }
size_t dtype_size(int dt) { return dt == HQQ_F32 ? 4 : dt == HQQ_U8 ? 1 : 2; }
bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// Shape checks shared by quantize and dequantize.
hqq_status check_shape(int64_t rows, int64_t cols, int nbits, int group_size, int axis) {
  if (rows < 0 || cols < 0) return HQQ_ERR_INVALID_ARG;
  if (!nbits_ok(nbits) || !group_ok(group_size) || (axis != 0 && axis != 1))
    return HQQ_ERR_UNSUPPORTED;
  if (cols > 0 && rows > kMaxElems / cols) return HQQ_ERR_SHAPE;
  if (axis == 1 && cols % group_size) return HQQ_ERR_SHAPE;
  if (axis == 0 && rows % group_size) return HQQ_ERR_SHAPE;
  return HQQ_OK;
}

bool flags_ok(int flags) { return (flags & ~HQQ_FLAG_STOP_AT_FIXED_POINT) == 0; }

hqq_status check_solver(int iters, float p, float beta0, float kappa) {
  if (iters < 0 || iters > HQQ_MAX_ITERS) return HQQ_ERR_INVALID_ARG;
  if (!(p > 0.0f && p <= 1.0f)) return HQQ_ERR_INVALID_ARG;
  if (!(beta0 > 0.0f) || !isfinite(beta0)) return HQQ_ERR_INVALID_ARG;
  if (!(kappa >= 1.0f) || !isfinite(kappa)) return HQQ_ERR_INVALID_ARG;
  return HQQ_OK;
}

hqq_status check_meta_group(int g) { return (g >= 8 && g <= 1024) ? HQQ_OK : HQQ_ERR_UNSUPPORTED; }

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

}  // namespace

HQQ_EXPORT int hqq_abi_version(void) { return HQQ_ABI_VERSION; }

HQQ_EXPORT const char* hqq_last_cuda_error(void) { return g_last_cuda_error; }

HQQ_EXPORT const char* hqq_status_string(hqq_status s) {
  switch (s) {
    case HQQ_OK: return "HQQ_OK";
    case HQQ_ERR_INVALID_ARG: return "HQQ_ERR_INVALID_ARG";
    case HQQ_ERR_UNSUPPORTED: return "HQQ_ERR_UNSUPPORTED";
    case HQQ_ERR_SHAPE: return "HQQ_ERR_SHAPE";
    case HQQ_ERR_ALIGNMENT: return "HQQ_ERR_ALIGNMENT";
    case HQQ_ERR_CUDA: return "HQQ_ERR_CUDA";
    case HQQ_ERR_WORKSPACE: return "HQQ_ERR_WORKSPACE";
  }
  return "HQQ_ERR_UNKNOWN";
}

HQQ_EXPORT int64_t hqq_num_groups(int64_t rows, int64_t cols, int group_size, int axis) {
  if (!group_ok(group_size) || (axis != 0 && axis != 1) || rows < 0 || cols < 0) return -1;
  if (cols > 0 && rows > kMaxElems / cols) return -1;
  if (axis == 1 && cols % group_size) return -1;
  if (axis == 0 && rows % group_size) return -1;
  return rows * cols / group_size;
}

HQQ_EXPORT size_t hqq_packed_bytes(int64_t rows, int64_t cols, int nbits, int group_size, int axis) {
  (void)group_size;
  (void)axis;
  if (!nbits_ok(nbits) || rows < 0 || cols < 0) return 0;
  if (cols > 0 && rows > kMaxElems / cols) return 0;
  const int64_t n = rows * cols;
  if (nbits == 3) return (size_t)(4 * ((n + 9) / 10));
  return (size_t)((n * nbits + 7) / 8);
}

HQQ_EXPORT int64_t hqq_num_meta_groups(int64_t n, int meta_group_size) {
  if (n < 0 || meta_group_size <= 0) return -1;
  return (n + meta_group_size - 1) / meta_group_size;
}

// Workspace: fp32 scale then fp32 zero (only the quantized ones), each part 256-aligned.
HQQ_EXPORT size_t hqq_workspace_bytes(int64_t rows, int64_t cols, const hqq_params* prm) {
  if (!prm) return (size_t)-1;
  const int64_t ng = hqq_num_groups(rows, cols, prm->group_size, prm->axis);
  if (ng < 0) return (size_t)-1;
  const size_t part = round_up((size_t)ng * 4, 256);
  return part * ((prm->quant_scale ? 1 : 0) + (prm->quant_zero ? 1 : 0));
}

hqq_status hqqabi::validate_quantize(const void* W, int64_t rows, int64_t cols,
                                     const hqq_params& prm, const void* Wq_packed,
                                     const void* scale, const void* zero, const void* scale_mm,
                                     const void* zero_mm) {
  hqq_status st = check_shape(rows, cols, prm.nbits, prm.group_size, prm.axis);
  if (st != HQQ_OK) return st;
  if ((st = check_solver(prm.iters, prm.p, prm.beta0, prm.kappa)) != HQQ_OK) return st;
  if (!flags_ok(prm.flags)) return HQQ_ERR_INVALID_ARG;
  if (!wdtype_ok(prm.w_dtype) || !wdtype_ok(prm.meta_dtype)) return HQQ_ERR_UNSUPPORTED;
  const bool qs = prm.quant_scale != 0, qz = prm.quant_zero != 0;
  if ((qs || qz) && (st = check_meta_group(prm.meta_group_size)) != HQQ_OK) return st;
  if (rows * cols == 0) return HQQ_OK;  // nothing to read or write; pointers may be NULL
  if (!W || !Wq_packed || !scale || !zero) return HQQ_ERR_INVALID_ARG;
  if ((qs && !scale_mm) || (qz && !zero_mm)) return HQQ_ERR_INVALID_ARG;
  if (!aligned(W, 16) || !aligned(Wq_packed, 16)) return HQQ_ERR_ALIGNMENT;
  const size_t msz = dtype_size(prm.meta_dtype);
  if (!qs && !aligned(scale, msz)) return HQQ_ERR_ALIGNMENT;
  if (!qz && !aligned(zero, msz)) return HQQ_ERR_ALIGNMENT;
  if ((qs && !aligned(scale_mm, 8)) || (qz && !aligned(zero_mm, 8))) return HQQ_ERR_ALIGNMENT;
  return HQQ_OK;
}

static hqq_status quantize_impl(const void* W, int64_t rows, int64_t cols, const hqq_params& prm,
                                void* Wq_packed, void* scale, void* zero, void* scale_mm,
                                void* zero_mm, void* workspace, size_t workspace_bytes,
                                cudaStream_t stream) {
  hqq_status st =
      hqqabi::validate_quantize(W, rows, cols, prm, Wq_packed, scale, zero, scale_mm, zero_mm);
  if (st != HQQ_OK || rows * cols == 0) return st;
  const bool qs = prm.quant_scale != 0, qz = prm.quant_zero != 0;
  const size_t need = hqq_workspace_bytes(rows, cols, &prm);
  if (need > 0) {
    if (!workspace || workspace_bytes < need) return HQQ_ERR_WORKSPACE;
    if (!aligned(workspace, 16)) return HQQ_ERR_ALIGNMENT;
  }
  if ((st = check_device(W)) != HQQ_OK) return st;
  const int64_t ng = rows * cols / prm.group_size;

  const size_t part = round_up((size_t)ng * 4, 256);
  float* ws_scale = qs ? reinterpret_cast<float*>(workspace) : nullptr;
  float* ws_zero = qz ? reinterpret_cast<float*>(reinterpret_cast<char*>(workspace) + (qs ? part : 0))
                      : nullptr;

  hqqk::QuantJob j;
  j.W = W;
  j.rows = rows;
  j.cols = cols;
  j.n_groups = ng;
  j.w_dtype = prm.w_dtype;
  j.nbits = prm.nbits;
  j.group_size = prm.group_size;
  j.axis = prm.axis;
  j.iters = prm.iters;
  j.p = prm.p;
  j.beta0 = prm.beta0;
  j.kappa = prm.kappa;
  j.packed = reinterpret_cast<uint8_t*>(Wq_packed);
  j.scale = qs ? static_cast<void*>(ws_scale) : scale;
  j.zero = qz ? static_cast<void*>(ws_zero) : zero;
  j.scale_dtype = qs ? static_cast<int>(hqqk::kF32) : static_cast<int>(prm.meta_dtype);
  j.zero_dtype = qz ? static_cast<int>(hqqk::kF32) : static_cast<int>(prm.meta_dtype);
  j.flags = prm.flags;
  if ((st = cuda_status(hqqk::launch_quantize(j, stream))) != HQQ_OK) return st;
  if (qs) {
    st = cuda_status(hqqk::launch_quantize_meta(ws_scale, hqqk::kF32, ng, prm.meta_group_size,
                                                reinterpret_cast<uint8_t*>(scale),
                                                reinterpret_cast<float*>(scale_mm), stream));
    if (st != HQQ_OK) return st;
  }
  if (qz) {
    st = cuda_status(hqqk::launch_quantize_meta(ws_zero, hqqk::kF32, ng, prm.meta_group_size,
                                                reinterpret_cast<uint8_t*>(zero),
                                                reinterpret_cast<float*>(zero_mm), stream));
    if (st != HQQ_OK) return st;
  }
  return HQQ_OK;
}

HQQ_EXPORT hqq_status hqq_quantize(const void* W, hqq_dtype dtype, int64_t rows, int64_t cols,
                                   int nbits, int group_size, int axis, int iters, float p,
                                   float beta0, float kappa, void* Wq_packed, void* scale,
                                   void* zero, cudaStream_t stream) {
  hqq_params prm;
  prm.nbits = nbits;
  prm.group_size = group_size;
  prm.axis = axis;
  prm.iters = iters;
  prm.p = p;
  prm.beta0 = beta0;
  prm.kappa = kappa;
  prm.w_dtype = dtype;
  prm.meta_dtype = dtype;
  prm.quant_scale = 0;
  prm.quant_zero = 0;
  prm.meta_group_size = 128;
  prm.flags = 0;
  return quantize_impl(W, rows, cols, prm, Wq_packed, scale, zero, nullptr, nullptr, nullptr, 0,
                       stream);
}

HQQ_EXPORT hqq_status hqq_quantize_ex(const void* W, int64_t rows, int64_t cols,
                                      const hqq_params* params, void* Wq_packed, void* scale,
                                      void* zero, void* scale_mm, void* zero_mm, void* workspace,
                                      size_t workspace_bytes, cudaStream_t stream) {
  if (!params) return HQQ_ERR_INVALID_ARG;
  return quantize_impl(W, rows, cols, *params, Wq_packed, scale, zero, scale_mm, zero_mm,
                       workspace, workspace_bytes, stream);
}

static hqq_status dequantize_impl(const void* Wq_packed, const void* scale, const void* zero,
                                  const void* scale_mm, const void* zero_mm, int meta_dtype,
                                  int meta_group_size, int64_t rows, int64_t cols, int nbits,
                                  int group_size, int axis, int out_dtype, void* W_out,
                                  cudaStream_t stream) {
  hqq_status st = check_shape(rows, cols, nbits, group_size, axis);
  if (st != HQQ_OK) return st;
  if (!wdtype_ok(out_dtype)) return HQQ_ERR_UNSUPPORTED;
  if ((!scale_mm || !zero_mm) && !wdtype_ok(meta_dtype)) return HQQ_ERR_UNSUPPORTED;
  if ((scale_mm || zero_mm) && (st = check_meta_group(meta_group_size)) != HQQ_OK) return st;
  if (rows * cols == 0) return HQQ_OK;
  if (!Wq_packed || !scale || !zero || !W_out) return HQQ_ERR_INVALID_ARG;
  if (!aligned(Wq_packed, 16) || !aligned(W_out, 16)) return HQQ_ERR_ALIGNMENT;
  const size_t msz = dtype_size(meta_dtype);
  if ((!scale_mm && !aligned(scale, msz)) || (!zero_mm && !aligned(zero, msz)))
    return HQQ_ERR_ALIGNMENT;
  if ((scale_mm && !aligned(scale_mm, 8)) || (zero_mm && !aligned(zero_mm, 8)))
    return HQQ_ERR_ALIGNMENT;
  if ((st = check_device(Wq_packed)) != HQQ_OK) return st;
  hqqk::DequantJob j;
  j.packed = reinterpret_cast<const uint8_t*>(Wq_packed);
  j.scale = scale;
  j.zero = zero;
  j.scale_mm = reinterpret_cast<const float*>(scale_mm);
  j.zero_mm = reinterpret_cast<const float*>(zero_mm);
  j.meta_group_size = meta_group_size;
  j.meta_dtype = meta_dtype;
  j.rows = rows;
  j.cols = cols;
  j.n_groups = rows * cols / group_size;
  j.nbits = nbits;
  j.group_size = group_size;
  j.axis = axis;
  j.out_dtype = out_dtype;
  j.out = W_out;
  return cuda_status(hqqk::launch_dequantize(j, stream));
}

HQQ_EXPORT hqq_status hqq_dequantize(const void* Wq_packed, const void* scale, const void* zero,
                                     hqq_dtype meta_dtype, hqq_dtype out_dtype, int64_t rows,
                                     int64_t cols, int nbits, int group_size, int axis,
                                     void* W_out, cudaStream_t stream) {
  return dequantize_impl(Wq_packed, scale, zero, nullptr, nullptr, meta_dtype, 128, rows, cols,
                         nbits, group_size, axis, out_dtype, W_out, stream);
}

HQQ_EXPORT hqq_status hqq_dequantize_ex(const void* Wq_packed, const void* scale, const void* zero,
                                        const void* scale_mm, const void* zero_mm, int64_t rows,
                                        int64_t cols, const hqq_params* params,
                                        hqq_dtype out_dtype, void* W_out, cudaStream_t stream) {
  if (!params) return HQQ_ERR_INVALID_ARG;
  const void* smm = params->quant_scale ? scale_mm : nullptr;
  const void* zmm = params->quant_zero ? zero_mm : nullptr;
  if ((params->quant_scale && !scale_mm) || (params->quant_zero && !zero_mm))
    return HQQ_ERR_INVALID_ARG;
  return dequantize_impl(Wq_packed, scale, zero, smm, zmm, params->meta_dtype,
                         params->meta_group_size, rows, cols, params->nbits, params->group_size,
                         params->axis, out_dtype, W_out, stream);
}

// Per-matrix checks shared by the batched calls (shape, pointers, alignment).
static hqq_status check_matrix(const hqq_matrix& m, const hqq_params& prm, size_t w_align,
                               int out_dtype) {
  hqq_status st = check_shape(m.rows, m.cols, prm.nbits, prm.group_size, prm.axis);
  if (st != HQQ_OK) return st;
  if (m.rows * m.cols == 0) return HQQ_OK;
  if (!m.W || !m.Wq_packed || !m.scale || !m.zero) return HQQ_ERR_INVALID_ARG;
  if (!aligned(m.W, w_align) || !aligned(m.Wq_packed, 16)) return HQQ_ERR_ALIGNMENT;
  const size_t msz = dtype_size(prm.meta_dtype);
  if (!aligned(m.scale, msz) || !aligned(m.zero, msz)) return HQQ_ERR_ALIGNMENT;
  (void)out_dtype;
  return HQQ_OK;
}

static hqq_status check_batch_params(const hqq_matrix* mats, int n, const hqq_params* prm) {
  if (!prm || n < 0 || (n > 0 && !mats)) return HQQ_ERR_INVALID_ARG;
  if (!nbits_ok(prm->nbits) || !group_ok(prm->group_size) || (prm->axis != 0 && prm->axis != 1))
    return HQQ_ERR_UNSUPPORTED;
  if (!wdtype_ok(prm->w_dtype) || !wdtype_ok(prm->meta_dtype)) return HQQ_ERR_UNSUPPORTED;
  if (prm->quant_scale || prm->quant_zero) return HQQ_ERR_UNSUPPORTED;
  return HQQ_OK;
}

HQQ_EXPORT hqq_status hqq_quantize_batched(const hqq_matrix* mats, int n, const hqq_params* prm,
                                           cudaStream_t stream) {
  hqq_status st = check_batch_params(mats, n, prm);
  if (st != HQQ_OK) return st;
  if ((st = check_solver(prm->iters, prm->p, prm->beta0, prm->kappa)) != HQQ_OK) return st;
  if (!flags_ok(prm->flags)) return HQQ_ERR_INVALID_ARG;
  std::vector<hqqk::QuantJob> jobs;
  jobs.reserve((size_t)n);
  for (int i = 0; i < n; ++i) {
    const hqq_matrix& m = mats[i];
    if ((st = check_matrix(m, *prm, 16, -1)) != HQQ_OK) return st;
    if (m.rows * m.cols == 0) continue;
    hqqk::QuantJob j;
    j.W = m.W;
    j.rows = m.rows;
    j.cols = m.cols;
    j.n_groups = m.rows * m.cols / prm->group_size;
    j.w_dtype = prm->w_dtype;
    j.nbits = prm->nbits;
    j.group_size = prm->group_size;
    j.axis = prm->axis;
    j.iters = prm->iters;
    j.p = prm->p;
    j.beta0 = prm->beta0;
    j.kappa = prm->kappa;
    j.packed = reinterpret_cast<uint8_t*>(m.Wq_packed);
    j.scale = m.scale;
    j.zero = m.zero;
    j.scale_dtype = prm->meta_dtype;
    j.zero_dtype = prm->meta_dtype;
    j.flags = prm->flags;
    jobs.push_back(j);
  }
  if (jobs.empty()) return HQQ_OK;
  for (const hqqk::QuantJob& j : jobs)  // every matrix's arguments are valid: now its device
    if ((st = check_device(j.W)) != HQQ_OK) return st;
  return cuda_status(hqqk::launch_quantize_batched(jobs.data(), (int)jobs.size(), stream));
}

HQQ_EXPORT hqq_status hqq_dequantize_batched(const hqq_matrix* mats, int n, const hqq_params* prm,
                                             hqq_dtype out_dtype, cudaStream_t stream) {
  hqq_status st = check_batch_params(mats, n, prm);
  if (st != HQQ_OK) return st;
  if (!wdtype_ok(out_dtype)) return HQQ_ERR_UNSUPPORTED;
  std::vector<hqqk::DequantJob> jobs;
  jobs.reserve((size_t)n);
  for (int i = 0; i < n; ++i) {
    const hqq_matrix& m = mats[i];
    if ((st = check_matrix(m, *prm, 16, out_dtype)) != HQQ_OK) return st;
    if (m.rows * m.cols == 0) continue;
    hqqk::DequantJob j;
    j.packed = reinterpret_cast<const uint8_t*>(m.Wq_packed);
    j.scale = m.scale;
    j.zero = m.zero;
    j.scale_mm = nullptr;
    j.zero_mm = nullptr;
    j.meta_group_size = 128;
    j.meta_dtype = prm->meta_dtype;
    j.rows = m.rows;
    j.cols = m.cols;
    j.n_groups = m.rows * m.cols / prm->group_size;
    j.nbits = prm->nbits;
    j.group_size = prm->group_size;
    j.axis = prm->axis;
    j.out_dtype = out_dtype;
    j.out = m.W;
    jobs.push_back(j);
  }
  if (jobs.empty()) return HQQ_OK;
  for (const hqqk::DequantJob& j : jobs)
    if ((st = check_device(j.packed)) != HQQ_OK) return st;
  return cuda_status(hqqk::launch_dequantize_batched(jobs.data(), (int)jobs.size(), stream));
}

// ---------------------------------------------------------------- mixed configurations
// Two configurations are the same when every field that reaches a kernel is equal.
static bool same_config(const hqq_params& a, const hqq_params& b) {
  return a.nbits == b.nbits && a.group_size == b.group_size && a.axis == b.axis &&
         a.iters == b.iters && a.p == b.p && a.beta0 == b.beta0 && a.kappa == b.kappa &&
         a.w_dtype == b.w_dtype && a.meta_dtype == b.meta_dtype &&
         a.quant_scale == b.quant_scale && a.quant_zero == b.quant_zero &&
         a.meta_group_size == b.meta_group_size && a.flags == b.flags;
}

// group_of[i] = index (by first appearance) of the configuration of matrix i; rep[g] = the
// first matrix of group g.
static void plan_mixed(const hqq_params* prm, int n, std::vector<int>* group_of,
                       std::vector<int>* rep) {
  group_of->assign((size_t)n, -1);
  rep->clear();
  for (int i = 0; i < n; ++i) {
    int g = -1;
    for (size_t k = 0; k < rep->size(); ++k)
      if (same_config(prm[(*rep)[k]], prm[i])) { g = (int)k; break; }
    if (g < 0) {
      g = (int)rep->size();
      rep->push_back(i);
    }
    (*group_of)[i] = g;
  }
}

HQQ_EXPORT hqq_status hqq_mixed_plan(const hqq_params* params, int n, int* group_of,
                                     int* n_groups) {
  if (n < 0 || !n_groups || (n > 0 && (!params || !group_of))) return HQQ_ERR_INVALID_ARG;
  std::vector<int> g, rep;
  plan_mixed(params, n, &g, &rep);
  for (int i = 0; i < n; ++i) group_of[i] = g[(size_t)i];
  *n_groups = (int)rep.size();
  return HQQ_OK;
}

// Validate every matrix against its own configuration, then issue one batched call per
// configuration group (matrices in their original order within a group).
template <typename Batched>
static hqq_status run_mixed(const hqq_matrix* mats, const hqq_params* prm, int n, int out_dtype,
                            Batched batched) {
  if (n < 0 || (n > 0 && (!mats || !prm))) return HQQ_ERR_INVALID_ARG;
  for (int i = 0; i < n; ++i) {
    hqq_status st = check_batch_params(&mats[i], 1, &prm[i]);
    if (st != HQQ_OK) return st;
    if (out_dtype < 0) {
      if ((st = check_solver(prm[i].iters, prm[i].p, prm[i].beta0, prm[i].kappa)) != HQQ_OK)
        return st;
      if (!flags_ok(prm[i].flags)) return HQQ_ERR_INVALID_ARG;
    } else if (!wdtype_ok(out_dtype)) {
      return HQQ_ERR_UNSUPPORTED;
    }
    if ((st = check_matrix(mats[i], prm[i], 16, out_dtype)) != HQQ_OK) return st;
  }
  for (int i = 0; i < n; ++i) {  // all arguments are valid: now the devices, before any launch
    if (mats[i].rows * mats[i].cols == 0) continue;
    const hqq_status st = check_device(out_dtype < 0 ? mats[i].W : mats[i].Wq_packed);
    if (st != HQQ_OK) return st;
  }
  std::vector<int> group_of, rep;
  plan_mixed(prm, n, &group_of, &rep);
  std::vector<hqq_matrix> sub;
  sub.reserve((size_t)n);
  for (size_t g = 0; g < rep.size(); ++g) {
    sub.clear();
    for (int i = 0; i < n; ++i)
      if (group_of[(size_t)i] == (int)g) sub.push_back(mats[i]);
    const hqq_status st = batched(sub.data(), (int)sub.size(), &prm[rep[g]]);
    if (st != HQQ_OK) return st;
  }
  return HQQ_OK;
}

HQQ_EXPORT hqq_status hqq_quantize_mixed(const hqq_matrix* mats, const hqq_params* params, int n,
                                         cudaStream_t stream) {
  return run_mixed(mats, params, n, -1, [&](const hqq_matrix* m, int k, const hqq_params* p) {
    return hqq_quantize_batched(m, k, p, stream);
  });
}

HQQ_EXPORT hqq_status hqq_dequantize_mixed(const hqq_matrix* mats, const hqq_params* params,
                                           int n, hqq_dtype out_dtype, cudaStream_t stream) {
  if (!wdtype_ok(out_dtype)) return HQQ_ERR_UNSUPPORTED;
  return run_mixed(mats, params, n, static_cast<int>(out_dtype),
                   [&](const hqq_matrix* m, int k, const hqq_params* p) {
                     return hqq_dequantize_batched(m, k, p, out_dtype, stream);
                   });
}

HQQ_EXPORT hqq_status hqq_quantize_meta(const void* meta, hqq_dtype dtype, int64_t n, int group,
                                        void* q_u8, void* mm, cudaStream_t stream) {
  if (n < 0) return HQQ_ERR_INVALID_ARG;
  if (!wdtype_ok(dtype)) return HQQ_ERR_UNSUPPORTED;
  hqq_status st = check_meta_group(group);
  if (st != HQQ_OK) return st;
  if (n == 0) return HQQ_OK;
  if (!meta || !q_u8 || !mm) return HQQ_ERR_INVALID_ARG;
  if (!aligned(meta, dtype_size(dtype)) || !aligned(mm, 8)) return HQQ_ERR_ALIGNMENT;
  if ((st = check_device(meta)) != HQQ_OK) return st;
  return cuda_status(hqqk::launch_quantize_meta(meta, dtype, n, group,
                                                reinterpret_cast<uint8_t*>(q_u8),
                                                reinterpret_cast<float*>(mm), stream));
}

HQQ_EXPORT hqq_status hqq_dequantize_meta(const void* q_u8, const void* mm, int64_t n, int group,
                                          void* out_f32, cudaStream_t stream) {
  if (n < 0) return HQQ_ERR_INVALID_ARG;
  hqq_status st = check_meta_group(group);
  if (st != HQQ_OK) return st;
  if (n == 0) return HQQ_OK;
  if (!q_u8 || !mm || !out_f32) return HQQ_ERR_INVALID_ARG;
  if (!aligned(mm, 8) || !aligned(out_f32, 4)) return HQQ_ERR_ALIGNMENT;
  if ((st = check_device(q_u8)) != HQQ_OK) return st;
  return cuda_status(hqqk::launch_dequantize_meta(reinterpret_cast<const uint8_t*>(q_u8),
                                                  reinterpret_cast<const float*>(mm), n, group,
                                                  reinterpret_cast<float*>(out_f32), stream));
}

HQQ_EXPORT hqq_status hqq_linear(const void* X, int64_t M, int64_t K, hqq_dtype x_dtype,
                                 const void* Wq_packed, const void* scale, const void* zero,
                                 const void* bias, int64_t N, const hqq_params* params, void* Y,
                                 cudaStream_t stream) {
  if (!params) return HQQ_ERR_INVALID_ARG;
  const hqq_params& prm = *params;
  if (M < 0 || N < 0 || K < 0) return HQQ_ERR_INVALID_ARG;
  if (x_dtype != HQQ_BF16 && x_dtype != HQQ_F16) return HQQ_ERR_UNSUPPORTED;
  if (prm.nbits != 4 || prm.group_size != 64 || prm.axis != 1 || prm.quant_scale ||
      prm.quant_zero)
    return HQQ_ERR_UNSUPPORTED;
  if (!wdtype_ok(prm.meta_dtype)) return HQQ_ERR_INVALID_ARG;
  if ((prm.flags & ~(HQQ_FLAG_STOP_AT_FIXED_POINT | HQQ_FLAG_OVERLAP_WEIGHTS)) != 0)
    return HQQ_ERR_INVALID_ARG;
  if (K % 64 != 0 || N % 8 != 0) return HQQ_ERR_SHAPE;
  if (M >= (int64_t(1) << 31) || N >= (int64_t(1) << 31) || K >= (int64_t(1) << 31) ||
      (N + 255) / 256 > 65535)
    return HQQ_ERR_SHAPE;
  if (M == 0 || N == 0) return HQQ_OK;
  if (!Y) return HQQ_ERR_INVALID_ARG;
  if (K > 0 && (!X || !Wq_packed || !scale || !zero)) return HQQ_ERR_INVALID_ARG;
  if (!aligned(Y, 16) || !aligned(bias, 2)) return HQQ_ERR_ALIGNMENT;
  if (K > 0 && (!aligned(X, 16) || !aligned(Wq_packed, 16) ||
                !aligned(scale, dtype_size(prm.meta_dtype)) ||
                !aligned(zero, dtype_size(prm.meta_dtype))))
    return HQQ_ERR_ALIGNMENT;
  const hqq_status dst = check_device(Y);
  if (dst != HQQ_OK) return dst;
  hqqk::GemmJob j;
  j.X = X;
  j.packed = reinterpret_cast<const uint8_t*>(Wq_packed);
  j.scale = scale;
  j.zero = zero;
  j.bias = bias;
  j.Y = Y;
  j.M = M;
  j.N = N;
  j.K = K;
  j.x_dtype = x_dtype;
  j.meta_dtype = prm.meta_dtype;
  j.overlap_weights = (prm.flags & HQQ_FLAG_OVERLAP_WEIGHTS) != 0;
  return cuda_status(hqqk::launch_w4a16_gemm(j, stream));
}

HQQ_EXPORT hqq_status hqq_wait_timeouts(unsigned int* count) {
  if (!count) return HQQ_ERR_INVALID_ARG;
  return cuda_status(hqqk::read_gemm_timeouts(count));
}

static hqq_status check_mx_shape(int64_t rows, int64_t cols) {
  if (rows < 0 || cols < 0) return HQQ_ERR_INVALID_ARG;
  if (cols % 32 != 0) return HQQ_ERR_SHAPE;
  if (rows > 0 && cols > 0 && rows > kMaxElems / cols) return HQQ_ERR_SHAPE;
  return HQQ_OK;
}

HQQ_EXPORT hqq_status hqq_mxfp4_quantize(const void* W, hqq_dtype dtype, int64_t rows,
                                         int64_t cols, void* codes, void* scales,
                                         cudaStream_t stream) {
  hqq_status st = check_mx_shape(rows, cols);
  if (st != HQQ_OK) return st;
  if (!wdtype_ok(dtype)) return HQQ_ERR_UNSUPPORTED;
  if (rows * cols == 0) return HQQ_OK;
  if (!W || !codes || !scales) return HQQ_ERR_INVALID_ARG;
  if (!aligned(W, 16) || !aligned(codes, 4)) return HQQ_ERR_ALIGNMENT;
  if ((st = check_device(W)) != HQQ_OK) return st;
  return cuda_status(hqqk::launch_mxfp4_quantize(W, dtype, rows * cols,
                                                 reinterpret_cast<uint8_t*>(codes),
                                                 reinterpret_cast<uint8_t*>(scales), stream));
}

HQQ_EXPORT hqq_status hqq_mxfp4_dequantize(const void* codes, const void* scales, int64_t rows,
                                           int64_t cols, hqq_dtype out_dtype, void* W_out,
                                           cudaStream_t stream) {
  hqq_status st = check_mx_shape(rows, cols);
  if (st != HQQ_OK) return st;
  if (!wdtype_ok(out_dtype)) return HQQ_ERR_UNSUPPORTED;
  if (rows * cols == 0) return HQQ_OK;
  if (!codes || !scales || !W_out) return HQQ_ERR_INVALID_ARG;
  if (!aligned(codes, 4) || !aligned(W_out, 16)) return HQQ_ERR_ALIGNMENT;
  if ((st = check_device(codes)) != HQQ_OK) return st;
  return cuda_status(hqqk::launch_mxfp4_dequantize(reinterpret_cast<const uint8_t*>(codes),
                                                   reinterpret_cast<const uint8_t*>(scales),
                                                   rows * cols, out_dtype, W_out, stream));
}
