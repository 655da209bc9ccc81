"""calibration_free_weight_hqq_b200 - HQQ weight quantize / dequantize on NVIDIA B200.

A thin Python binding over the C ABI of ``libhqq_b200.so`` (declared in
``include/hqq/hqq.h``). The functions carry the C names and only marshal arguments:
PyTorch supplies device memory and the current stream, and every step of quantization and
dequantization runs in the library's CUDA kernels. There is no CPU fallback: if the
library is missing or the tensors are not on a CUDA device, the calls raise.

    import torch, calibration_free_weight_hqq_b200 as hqq
    W = torch.randn(4096, 1024, device="cuda", dtype=torch.float16) * 0.02
    Wq, scale, zero = hqq.hqq_quantize(W, nbits=4, group_size=64, axis=1)
    W2 = hqq.hqq_dequantize(Wq, scale, zero, 4096, 1024, nbits=4, group_size=64, axis=1,
                            out_dtype=torch.float16)

Parameters mirror BaseQuantizeConfig(nbits, group_size, quant_zero, quant_scale, axis)
("HQQ tutorial" (devpress.csdn.net) §3.3) plus the solver constants iters, p, beta0, kappa.
"""
from __future__ import annotations

import ctypes
import os
import threading
from typing import Optional

import torch

__all__ = [
    "HQQError", "HQQParams", "lib", "library_path", "hqq_quantize", "hqq_quantize_ex",
    "hqq_dequantize", "hqq_dequantize_ex", "hqq_quantize_meta", "hqq_dequantize_meta",
    "hqq_packed_bytes", "hqq_num_groups", "hqq_num_meta_groups", "hqq_workspace_bytes",
    "HQQ_F16", "HQQ_BF16", "HQQ_F32", "HQQ_U8",
]

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "libhqq_b200.so")
_lock = threading.Lock()
_lib = None

HQQ_F16, HQQ_BF16, HQQ_F32, HQQ_U8 = 0, 1, 2, 3
_TORCH_DT = {torch.float16: HQQ_F16, torch.bfloat16: HQQ_BF16, torch.float32: HQQ_F32,
             torch.uint8: HQQ_U8}
_DT_TORCH = {v: k for k, v in _TORCH_DT.items()}


class HQQError(RuntimeError):
    def __init__(self, status: int, where: str, detail: str = ""):
        self.status = status
        name = lib().hqq_status_string(status).decode()
        super().__init__(f"{where}: {name}" + (f" ({detail})" if detail else ""))


class HQQMatrix(ctypes.Structure):
    """Mirror of the C struct hqq_matrix (one matrix of a batched call)."""
    _fields_ = [("W", ctypes.c_void_p), ("rows", ctypes.c_int64), ("cols", ctypes.c_int64),
                ("Wq_packed", ctypes.c_void_p), ("scale", ctypes.c_void_p),
                ("zero", ctypes.c_void_p)]


class HQQParams(ctypes.Structure):
    """Mirror of the C struct hqq_params."""
    _fields_ = [("nbits", ctypes.c_int), ("group_size", ctypes.c_int), ("axis", ctypes.c_int),
                ("iters", ctypes.c_int), ("p", ctypes.c_float), ("beta0", ctypes.c_float),
                ("kappa", ctypes.c_float), ("w_dtype", ctypes.c_int),
                ("meta_dtype", ctypes.c_int), ("quant_scale", ctypes.c_int),
                ("quant_zero", ctypes.c_int), ("meta_group_size", ctypes.c_int),
                ("flags", ctypes.c_int)]

HQQ_FLAG_STOP_AT_FIXED_POINT = 1
HQQ_FLAG_OVERLAP_WEIGHTS = 2


def library_path() -> str:
    return _LIB_PATH


def lib() -> ctypes.CDLL:
    """The loaded C library (raises if it has not been built)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(_LIB_PATH):
                raise RuntimeError(
                    f"{_LIB_PATH} is missing: build it with "
                    "`python -m calibration_free_weight_hqq_b200.build` (nvcc, sm_100a)")
            L = ctypes.CDLL(_LIB_PATH)
            P, i64, i32, f32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_float
            sz = ctypes.c_size_t
            L.hqq_quantize.argtypes = [P, i32, i64, i64, i32, i32, i32, i32, f32, f32, f32, P, P,
                                       P, P]
            L.hqq_dequantize.argtypes = [P, P, P, i32, i32, i64, i64, i32, i32, i32, P, P]
            L.hqq_quantize_ex.argtypes = [P, i64, i64, ctypes.POINTER(HQQParams), P, P, P, P, P,
                                          P, sz, P]
            L.hqq_dequantize_ex.argtypes = [P, P, P, P, P, i64, i64, ctypes.POINTER(HQQParams),
                                            i32, P, P]
            L.hqq_quantize_ex_noalloc.argtypes = [P, i64, i64, ctypes.POINTER(HQQParams), P, P,
                                                  P, P, P, P]
            L.hqq_quantize_batched.argtypes = [ctypes.POINTER(HQQMatrix), i32,
                                               ctypes.POINTER(HQQParams), P]
            L.hqq_dequantize_batched.argtypes = [ctypes.POINTER(HQQMatrix), i32,
                                                 ctypes.POINTER(HQQParams), i32, P]
            L.hqq_quantize_mixed.argtypes = [ctypes.POINTER(HQQMatrix),
                                             ctypes.POINTER(HQQParams), i32, P]
            L.hqq_dequantize_mixed.argtypes = [ctypes.POINTER(HQQMatrix),
                                               ctypes.POINTER(HQQParams), i32, i32, P]
            L.hqq_mixed_plan.argtypes = [ctypes.POINTER(HQQParams), i32,
                                         ctypes.POINTER(ctypes.c_int), ctypes.POINTER(ctypes.c_int)]
            L.hqq_quantize_meta.argtypes = [P, i32, i64, i32, P, P, P]
            L.hqq_dequantize_meta.argtypes = [P, P, i64, i32, P, P]
            L.hqq_linear.argtypes = [P, i64, i64, i32, P, P, P, P, i64,
                                     ctypes.POINTER(HQQParams), P, P]
            L.hqq_wait_timeouts.argtypes = [ctypes.POINTER(ctypes.c_uint)]
            L.hqq_mxfp4_quantize.argtypes = [P, i32, i64, i64, P, P, P]
            L.hqq_mxfp4_dequantize.argtypes = [P, P, i64, i64, i32, P, P]
            for f in ("hqq_quantize", "hqq_dequantize", "hqq_quantize_ex", "hqq_dequantize_ex",
                      "hqq_quantize_meta", "hqq_dequantize_meta", "hqq_quantize_ex_noalloc",
                      "hqq_quantize_batched", "hqq_dequantize_batched", "hqq_linear",
                      "hqq_wait_timeouts", "hqq_mxfp4_quantize", "hqq_mxfp4_dequantize",
                      "hqq_quantize_mixed", "hqq_dequantize_mixed", "hqq_mixed_plan"):
                getattr(L, f).restype = i32
            L.hqq_packed_bytes.argtypes = [i64, i64, i32, i32, i32]
            L.hqq_packed_bytes.restype = sz
            L.hqq_num_groups.argtypes = [i64, i64, i32, i32]
            L.hqq_num_groups.restype = i64
            L.hqq_num_meta_groups.argtypes = [i64, i32]
            L.hqq_num_meta_groups.restype = i64
            L.hqq_workspace_bytes.argtypes = [i64, i64, ctypes.POINTER(HQQParams)]
            L.hqq_workspace_bytes.restype = sz
            L.hqq_status_string.argtypes = [i32]
            L.hqq_status_string.restype = ctypes.c_char_p
            L.hqq_last_cuda_error.argtypes = []
            L.hqq_last_cuda_error.restype = ctypes.c_char_p
            L.hqq_abi_version.argtypes = []
            L.hqq_abi_version.restype = i32
            _lib = L
    return _lib


def _check(status: int, where: str):
    if status != 0:
        detail = lib().hqq_last_cuda_error().decode() if status == 5 else ""
        raise HQQError(status, where, detail)


def _cuda(t: torch.Tensor, name: str, dev: Optional[torch.device] = None) -> int:
    """Device pointer of a contiguous CUDA tensor; with `dev`, the tensor must live there."""
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor (no CPU path exists)")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dev is not None:
        _same_device(dev, t, name)
    return t.data_ptr()


def _same_device(dev: torch.device, t: torch.Tensor, name: str) -> None:
    """Every buffer of a call lives on the device of its first input: the library launches on
    the current device, which the wrappers set to that one."""
    if t.device != dev:
        raise ValueError(f"{name} is on {t.device}, but this call runs on {dev}")


def _stream(stream: Optional[torch.cuda.Stream], dev: torch.device) -> int:
    if stream is None:
        return torch.cuda.current_stream(dev).cuda_stream
    if stream.device != dev:
        raise ValueError(f"stream belongs to {stream.device}, but this call runs on {dev}")
    return stream.cuda_stream


def hqq_packed_bytes(rows: int, cols: int, nbits: int, group_size: int = 64, axis: int = 1) -> int:
    return int(lib().hqq_packed_bytes(rows, cols, nbits, group_size, axis))


def hqq_num_groups(rows: int, cols: int, group_size: int, axis: int) -> int:
    return int(lib().hqq_num_groups(rows, cols, group_size, axis))


def hqq_num_meta_groups(n: int, meta_group_size: int) -> int:
    return int(lib().hqq_num_meta_groups(n, meta_group_size))


def _meta_shape(rows: int, cols: int, group_size: int, axis: int):
    return (rows, cols // group_size) if axis == 1 else (rows // group_size, cols)


def make_params(nbits=4, group_size=64, axis=1, iters=20, p=0.7, beta0=10.0, kappa=1.01,
                w_dtype=torch.bfloat16, meta_dtype=None, quant_scale=False, quant_zero=False,
                meta_group_size=128, stop_at_fixed_point=False,
                overlap_weights=False) -> HQQParams:
    """The C struct hqq_params. stop_at_fixed_point: HQQ_FLAG_STOP_AT_FIXED_POINT (quantize);
    overlap_weights: HQQ_FLAG_OVERLAP_WEIGHTS (hqq_linear; see the header for its promise)."""
    meta_dtype = w_dtype if meta_dtype is None else meta_dtype
    flags = (HQQ_FLAG_STOP_AT_FIXED_POINT if stop_at_fixed_point else 0) | \
        (HQQ_FLAG_OVERLAP_WEIGHTS if overlap_weights else 0)
    return HQQParams(nbits, group_size, axis, iters, p, beta0, kappa, _TORCH_DT[w_dtype],
                     _TORCH_DT[meta_dtype], int(bool(quant_scale)), int(bool(quant_zero)),
                     meta_group_size, flags)


def hqq_workspace_bytes(rows: int, cols: int, params: HQQParams) -> int:
    n = lib().hqq_workspace_bytes(rows, cols, ctypes.byref(params))
    if n == ctypes.c_size_t(-1).value:
        raise ValueError("invalid parameters")
    return int(n)


def hqq_quantize(W: torch.Tensor, nbits: int = 4, group_size: int = 64, axis: int = 1,
                 iters: int = 20, p: float = 0.7, beta0: float = 10.0, kappa: float = 1.01, *,
                 Wq_packed: Optional[torch.Tensor] = None, scale: Optional[torch.Tensor] = None,
                 zero: Optional[torch.Tensor] = None, stream=None):
    """Quantize a 2-D CUDA weight (fp16/bf16/fp32). Returns (Wq_packed uint8, scale, zero),
    scale/zero in W's dtype, shaped [rows, cols/G] (axis=1) or [rows/G, cols] (axis=0)."""
    if W.dim() != 2:
        raise ValueError("W must be 2-D [out_features, in_features]")
    rows, cols = W.shape
    wp = _cuda(W, "W")
    dev = W.device
    if Wq_packed is None:
        Wq_packed = torch.empty(hqq_packed_bytes(rows, cols, nbits, group_size, axis),
                                dtype=torch.uint8, device=W.device)
    ms = _meta_shape(rows, cols, group_size, axis) if hqq_num_groups(rows, cols, group_size, axis) >= 0 else (0,)
    if scale is None:
        scale = torch.empty(ms, dtype=W.dtype, device=W.device)
    if zero is None:
        zero = torch.empty(ms, dtype=W.dtype, device=W.device)
    with torch.cuda.device(dev):
        st = lib().hqq_quantize(wp, _TORCH_DT.get(W.dtype, -1), rows, cols, nbits, group_size,
                                axis, iters, p, beta0, kappa, _cuda(Wq_packed, "Wq_packed", dev),
                                _cuda(scale, "scale", dev), _cuda(zero, "zero", dev),
                                _stream(stream, dev))
    _check(st, "hqq_quantize")
    return Wq_packed, scale, zero


def hqq_quantize_ex(W: torch.Tensor, params: HQQParams, *, stream=None, workspace=None,
                    out: Optional[dict] = None):
    """Full parameter set (second-level 8-bit scale/zero). Returns a dict with Wq_packed,
    scale, zero (uint8 codes when quantized) and scale_mm / zero_mm (fp32 [runs, 2]); `out`,
    a dict of that form from an earlier call, is written in place."""
    rows, cols = W.shape
    wp = _cuda(W, "W")
    dev = W.device
    ng = hqq_num_groups(rows, cols, params.group_size, params.axis)
    if ng < 0:
        raise HQQError(3, "hqq_quantize_ex")
    ms = _meta_shape(rows, cols, params.group_size, params.axis)
    mdt = _DT_TORCH[params.meta_dtype]
    runs = max(hqq_num_meta_groups(ng, params.meta_group_size), 0)
    out = out if out is not None else {
        "Wq_packed": torch.empty(hqq_packed_bytes(rows, cols, params.nbits), dtype=torch.uint8,
                                 device=dev),
        "scale": torch.empty(ms, dtype=torch.uint8 if params.quant_scale else mdt, device=dev),
        "zero": torch.empty(ms, dtype=torch.uint8 if params.quant_zero else mdt, device=dev),
        "scale_mm": torch.empty((runs, 2), dtype=torch.float32, device=dev)
        if params.quant_scale else None,
        "zero_mm": torch.empty((runs, 2), dtype=torch.float32, device=dev)
        if params.quant_zero else None,
    }
    need = hqq_workspace_bytes(rows, cols, params)
    if workspace is None and need:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    for k in ("scale_mm", "zero_mm"):
        if out[k] is not None:
            _same_device(dev, out[k], k)
    if workspace is not None:
        _same_device(dev, workspace, "workspace")
    with torch.cuda.device(dev):
        st = lib().hqq_quantize_ex(
            wp, rows, cols, ctypes.byref(params), _cuda(out["Wq_packed"], "Wq_packed", dev),
            _cuda(out["scale"], "scale", dev), _cuda(out["zero"], "zero", dev),
            out["scale_mm"].data_ptr() if out["scale_mm"] is not None else None,
            out["zero_mm"].data_ptr() if out["zero_mm"] is not None else None,
            workspace.data_ptr() if workspace is not None else None,
            workspace.numel() if workspace is not None else 0, _stream(stream, dev))
    _check(st, "hqq_quantize_ex")
    return out


def hqq_quantize_ex_noalloc(W: torch.Tensor, params: HQQParams, *, stream=None):
    """hqq_quantize_ex whose second-level scratch is the library's fixed device array
    (HQQ_NOALLOC_SCRATCH_BYTES) instead of a workspace; the outputs are still allocated here
    (by torch) unless a caller passes its own through the C entry point."""
    rows, cols = W.shape
    dev = W.device
    ng = hqq_num_groups(rows, cols, params.group_size, params.axis)
    if ng < 0:
        raise HQQError(3, "hqq_quantize_ex_noalloc")
    ms = _meta_shape(rows, cols, params.group_size, params.axis)
    mdt = _DT_TORCH[params.meta_dtype]
    runs = max(hqq_num_meta_groups(ng, params.meta_group_size), 0)
    out = {
        "Wq_packed": torch.empty(hqq_packed_bytes(rows, cols, params.nbits), dtype=torch.uint8,
                                 device=dev),
        "scale": torch.empty(ms, dtype=torch.uint8 if params.quant_scale else mdt, device=dev),
        "zero": torch.empty(ms, dtype=torch.uint8 if params.quant_zero else mdt, device=dev),
        "scale_mm": torch.empty((runs, 2), dtype=torch.float32, device=dev)
        if params.quant_scale else None,
        "zero_mm": torch.empty((runs, 2), dtype=torch.float32, device=dev)
        if params.quant_zero else None,
    }
    with torch.cuda.device(dev):
        st = lib().hqq_quantize_ex_noalloc(
            _cuda(W, "W"), rows, cols, ctypes.byref(params),
            _cuda(out["Wq_packed"], "Wq_packed", dev), _cuda(out["scale"], "scale", dev),
            _cuda(out["zero"], "zero", dev),
            out["scale_mm"].data_ptr() if out["scale_mm"] is not None else None,
            out["zero_mm"].data_ptr() if out["zero_mm"] is not None else None,
            _stream(stream, dev))
    _check(st, "hqq_quantize_ex_noalloc")
    return out


def alloc_outputs(shapes, params: HQQParams, device="cuda"):
    """(packed, scale, zero) tensors for each (rows, cols) in `shapes`."""
    mdt = _DT_TORCH[params.meta_dtype]
    outs = []
    for rows, cols in shapes:
        ms = _meta_shape(rows, cols, params.group_size, params.axis)
        outs.append((torch.empty(hqq_packed_bytes(rows, cols, params.nbits), dtype=torch.uint8,
                                 device=device),
                     torch.empty(ms, dtype=mdt, device=device),
                     torch.empty(ms, dtype=mdt, device=device)))
    return outs


def matrix_batch(Ws, outs):
    """ctypes array of hqq_matrix descriptors for tensors Ws[i] (inputs of a quantize or
    outputs of a dequantize) and their (packed, scale, zero) outs[i]; build it once and
    reuse it across calls to skip the per-call marshalling."""
    arr = (HQQMatrix * len(Ws))()
    dev = Ws[0].device if len(Ws) else None
    for i, (W, (pk, sc, zr)) in enumerate(zip(Ws, outs)):
        arr[i] = HQQMatrix(_cuda(W, "W", dev), W.shape[0], W.shape[1],
                           _cuda(pk, "Wq_packed", dev), _cuda(sc, "scale", dev),
                           _cuda(zr, "zero", dev))
    return arr


def _batch_device(tensors) -> torch.device:
    if not len(tensors):
        return torch.device("cuda", torch.cuda.current_device())
    return tensors[0].device


def hqq_quantize_batched(Ws, params: HQQParams, *, outs=None, batch=None, stream=None):
    """Quantize a list of 2-D CUDA weights sharing one configuration in as few launches as
    possible (the whole-model driver). Returns the list of (packed, scale, zero)."""
    if outs is None:
        outs = alloc_outputs([tuple(W.shape) for W in Ws], params, Ws[0].device)
    if batch is None:
        batch = matrix_batch(Ws, outs)
    dev = _batch_device(Ws)
    with torch.cuda.device(dev):
        st = lib().hqq_quantize_batched(batch, len(Ws), ctypes.byref(params),
                                        _stream(stream, dev))
    _check(st, "hqq_quantize_batched")
    return outs


def hqq_dequantize_batched(outs, shapes, params: HQQParams, out_dtype=torch.bfloat16, *,
                           W_out=None, batch=None, stream=None):
    """Dequantize a list of (packed, scale, zero) of one configuration into new (or given)
    [rows, cols] tensors of out_dtype."""
    if W_out is None:
        W_out = [torch.empty(sh, dtype=out_dtype, device=outs[0][0].device) for sh in shapes]
    if batch is None:
        batch = matrix_batch(W_out, outs)
    dev = _batch_device(W_out)
    with torch.cuda.device(dev):
        st = lib().hqq_dequantize_batched(
            batch, len(W_out), ctypes.byref(params),
            _TORCH_DT.get(W_out[0].dtype if W_out else out_dtype, -1), _stream(stream, dev))
    _check(st, "hqq_dequantize_batched")
    return W_out


def _params_array(params_list):
    arr = (HQQParams * len(params_list))()
    for i, p in enumerate(params_list):
        arr[i] = p
    return arr


def hqq_mixed_plan(params_list):
    """The grouping of a mixed call (host only): (group index per matrix, number of groups)."""
    n = len(params_list)
    g = (ctypes.c_int * max(n, 1))()
    k = ctypes.c_int(0)
    _check(lib().hqq_mixed_plan(_params_array(params_list), n, g, ctypes.byref(k)),
           "hqq_mixed_plan")
    return [g[i] for i in range(n)], k.value


def hqq_quantize_mixed(Ws, params_list, *, outs=None, batch=None, stream=None):
    """Quantize a list of 2-D CUDA weights, weight i with its own configuration params_list[i]
    (per-layer mixed precision), one batched launch per distinct configuration. Returns the
    list of (packed, scale, zero). `batch` = matrix_batch(Ws, outs), built once, skips the
    per-call marshalling."""
    if outs is None:
        outs = [alloc_outputs([tuple(W.shape)], p, W.device)[0] for W, p in zip(Ws, params_list)]
    if batch is None:
        batch = matrix_batch(Ws, outs)
    dev = _batch_device(Ws)
    with torch.cuda.device(dev):
        st = lib().hqq_quantize_mixed(batch, _params_array(params_list), len(Ws),
                                      _stream(stream, dev))
    _check(st, "hqq_quantize_mixed")
    return outs


def hqq_dequantize_mixed(outs, shapes, params_list, out_dtype=torch.bfloat16, *, W_out=None,
                         batch=None, stream=None):
    """Dequantize (packed, scale, zero) i with params_list[i] into new (or given) [rows, cols]
    tensors of out_dtype (`batch` as in hqq_quantize_mixed, over W_out and outs)."""
    if W_out is None:
        W_out = [torch.empty(sh, dtype=out_dtype, device=outs[0][0].device) for sh in shapes]
    if batch is None:
        batch = matrix_batch(W_out, outs)
    dev = _batch_device(W_out)
    with torch.cuda.device(dev):
        st = lib().hqq_dequantize_mixed(
            batch, _params_array(params_list), len(W_out),
            _TORCH_DT.get(W_out[0].dtype if W_out else out_dtype, -1), _stream(stream, dev))
    _check(st, "hqq_dequantize_mixed")
    return W_out


def hqq_dequantize(Wq_packed, scale, zero, rows: int, cols: int, nbits: int = 4,
                   group_size: int = 64, axis: int = 1, out_dtype=torch.bfloat16, *, out=None,
                   stream=None):
    """Dequantize to a [rows, cols] CUDA tensor of out_dtype."""
    if out is None:
        out = torch.empty((rows, cols), dtype=out_dtype, device=Wq_packed.device)
    dev = Wq_packed.device
    with torch.cuda.device(dev):
        st = lib().hqq_dequantize(_cuda(Wq_packed, "Wq_packed"), _cuda(scale, "scale", dev),
                                  _cuda(zero, "zero", dev), _TORCH_DT.get(scale.dtype, -1),
                                  _TORCH_DT.get(out.dtype, -1), rows, cols, nbits, group_size,
                                  axis, _cuda(out, "out", dev), _stream(stream, dev))
    _check(st, "hqq_dequantize")
    return out


def hqq_dequantize_ex(q: dict, rows: int, cols: int, params: HQQParams, out_dtype=torch.bfloat16,
                      *, out=None, stream=None):
    """Inverse of hqq_quantize_ex (q is its result dict)."""
    if out is None:
        out = torch.empty((rows, cols), dtype=out_dtype, device=q["Wq_packed"].device)
    smm, zmm = q.get("scale_mm"), q.get("zero_mm")
    dev = q["Wq_packed"].device
    for name, t in (("scale_mm", smm), ("zero_mm", zmm)):
        if t is not None:
            _same_device(dev, t, name)
    with torch.cuda.device(dev):
        st = lib().hqq_dequantize_ex(
            _cuda(q["Wq_packed"], "Wq_packed"), _cuda(q["scale"], "scale", dev),
            _cuda(q["zero"], "zero", dev),
            smm.data_ptr() if smm is not None else None,
            zmm.data_ptr() if zmm is not None else None, rows, cols, ctypes.byref(params),
            _TORCH_DT.get(out.dtype, -1), _cuda(out, "out", dev), _stream(stream, dev))
    _check(st, "hqq_dequantize_ex")
    return out


def hqq_quantize_meta(meta: torch.Tensor, group: int = 128, *, stream=None):
    """Second level alone: returns (uint8 codes [n], fp32 [runs, 2] (step2, zero2))."""
    n = meta.numel()
    q = torch.empty(n, dtype=torch.uint8, device=meta.device)
    mm = torch.empty((max(hqq_num_meta_groups(n, group), 0), 2), dtype=torch.float32,
                     device=meta.device)
    dev = meta.device
    with torch.cuda.device(dev):
        st = lib().hqq_quantize_meta(_cuda(meta, "meta"), _TORCH_DT.get(meta.dtype, -1), n,
                                     group, _cuda(q, "q", dev), _cuda(mm, "mm", dev),
                                     _stream(stream, dev))
    _check(st, "hqq_quantize_meta")
    return q, mm


def hqq_dequantize_meta(q: torch.Tensor, mm: torch.Tensor, group: int = 128, *, stream=None):
    out = torch.empty(q.numel(), dtype=torch.float32, device=q.device)
    dev = q.device
    with torch.cuda.device(dev):
        st = lib().hqq_dequantize_meta(_cuda(q, "q"), _cuda(mm, "mm", dev), q.numel(), group,
                                       _cuda(out, "out", dev), _stream(stream, dev))
    _check(st, "hqq_dequantize_meta")
    return out


def hqq_linear(X: torch.Tensor, Wq_packed: torch.Tensor, scale: torch.Tensor,
               zero: torch.Tensor, N: int, params: Optional[HQQParams] = None, *,
               bias: Optional[torch.Tensor] = None, Y: Optional[torch.Tensor] = None,
               stream=None) -> torch.Tensor:
    """Forward pass of a 4-bit, group-64, axis-1 HQQ linear layer on the tensor cores:
    Y = X @ W'.T (+ bias), W' = the weight [N, K] dequantized to X's dtype (bf16 or fp16).
    X is [M, K] (or any [..., K]); scale/zero come from hqq_quantize* of W [N, K]."""
    if params is None:
        params = make_params(4, 64, 1, w_dtype=X.dtype, meta_dtype=scale.dtype)
    lead = X.shape[:-1]
    K = X.shape[-1]
    M = 1
    for d in lead:
        M *= d
    X2 = X.reshape(M, K)
    if Y is None:
        Y = torch.empty(*lead, N, dtype=X.dtype, device=X.device)
    dev = X.device
    with torch.cuda.device(dev):
        st = lib().hqq_linear(_cuda(X2, "X"), M, K, _TORCH_DT.get(X.dtype, -1),
                              _cuda(Wq_packed, "Wq_packed", dev), _cuda(scale, "scale", dev),
                              _cuda(zero, "zero", dev),
                              _cuda(bias, "bias", dev) if bias is not None else None,
                              N, ctypes.byref(params), _cuda(Y, "Y", dev), _stream(stream, dev))
    _check(st, "hqq_linear")
    return Y


def hqq_wait_timeouts() -> int:
    """Bounded in-kernel waits that ran out of time since load (0 on healthy runs)."""
    n = ctypes.c_uint(0)
    _check(lib().hqq_wait_timeouts(ctypes.byref(n)), "hqq_wait_timeouts")
    return int(n.value)


def hqq_mxfp4_quantize(W: torch.Tensor, *, codes: Optional[torch.Tensor] = None,
                       scales: Optional[torch.Tensor] = None, stream=None):
    """MXFP4 encoding of a 2-D CUDA weight (fp16/bf16/fp32, cols % 32 == 0): returns
    (codes uint8 [rows, cols/2], scales uint8 [rows, cols/32] = e + 127)."""
    if W.dim() != 2:
        raise ValueError("W must be 2-D")
    rows, cols = W.shape
    if codes is None:
        codes = torch.empty(rows, cols // 2, dtype=torch.uint8, device=W.device)
    if scales is None:
        scales = torch.empty(rows, cols // 32, dtype=torch.uint8, device=W.device)
    dev = W.device
    with torch.cuda.device(dev):
        st = lib().hqq_mxfp4_quantize(_cuda(W, "W"), _TORCH_DT.get(W.dtype, -1), rows, cols,
                                      _cuda(codes, "codes", dev), _cuda(scales, "scales", dev),
                                      _stream(stream, dev))
    _check(st, "hqq_mxfp4_quantize")
    return codes, scales


def hqq_mxfp4_dequantize(codes: torch.Tensor, scales: torch.Tensor, rows: int, cols: int,
                         out_dtype=torch.bfloat16, *, out: Optional[torch.Tensor] = None,
                         stream=None) -> torch.Tensor:
    """Decode MXFP4 codes and scales to a [rows, cols] CUDA tensor of out_dtype."""
    if out is None:
        out = torch.empty(rows, cols, dtype=out_dtype, device=codes.device)
    dev = codes.device
    with torch.cuda.device(dev):
        st = lib().hqq_mxfp4_dequantize(_cuda(codes, "codes"), _cuda(scales, "scales", dev),
                                        rows, cols, _TORCH_DT.get(out.dtype, -1),
                                        _cuda(out, "out", dev), _stream(stream, dev))
    _check(st, "hqq_mxfp4_dequantize")
    return out
