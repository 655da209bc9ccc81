"""CPU oracle of the calibration-free HQQ quantize / dequantize path.

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg
of ``bench.py`` may import this package; the product path (the CUDA library and its
binding in ``calibration_free_weight_hqq_b200``) never does, and the two share no code.

The arithmetic lives in ``hqq_oracle.c`` (plain scalar C, fp32 with fp64 only for the sums
the definition pins, no FMA contraction). This module builds it with gcc and wraps it with
ctypes + numpy. Every function cites its source in the C file.

Parity pins: the oracle is checked against closed forms, invariants, special cases and
brute force in ``tests/test_oracle_pins.py``. One part is not pinned by an independent
value: the solver's *optimality* (no closed form exists for the best zero; only
"no worse than RTN" and brute force on tiny groups are checked) - parity unpinned for
optimality.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "hqq_oracle.c")
_LIB = os.path.join(_HERE, "libhqq_oracle.so")
_lock = threading.Lock()
_lib = None

CFLAGS = ["-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off", "-fno-fast-math",
          "-fno-finite-math-only", "-pthread"]


def build(force: bool = False) -> str:
    """Compile the oracle into ``oracle/libhqq_oracle.so`` (gcc)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp.%d" % os.getpid()
        subprocess.check_call(["gcc", *CFLAGS, _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            P = ctypes.c_void_p
            i64, i32, f32 = ctypes.c_int64, ctypes.c_int, ctypes.c_float
            lib.hqq_oracle_quantize.argtypes = [P, i64, i64, i32, i32, i32, i32, f32, f32, f32,
                                                P, i64, P, P, P, P, i32]
            lib.hqq_oracle_quantize.restype = i32
            lib.hqq_oracle_quantize_group.argtypes = [P, i32, i32, i32, f32, f32, f32, P, P, P, P,
                                                      P]
            lib.hqq_oracle_quantize_group.restype = f32
            lib.hqq_oracle_codes_at_zero.argtypes = [P, i32, i32, f32, P]
            lib.hqq_oracle_codes_at_zero.restype = None
            lib.hqq_oracle_shrink.argtypes = [f32, f32, f32]
            lib.hqq_oracle_shrink.restype = f32
            lib.hqq_oracle_pow_pm1.argtypes = [f32, f32]
            lib.hqq_oracle_pow_pm1.restype = f32
            lib.hqq_oracle_packed_bytes.argtypes = [i64, i32]
            lib.hqq_oracle_packed_bytes.restype = i64
            lib.hqq_oracle_pack.argtypes = [P, i64, i32, P]
            lib.hqq_oracle_pack.restype = None
            lib.hqq_oracle_unpack.argtypes = [P, i64, i32, P]
            lib.hqq_oracle_unpack.restype = None
            lib.hqq_oracle_dequantize.argtypes = [P, P, P, i64, i64, i32, i32, P]
            lib.hqq_oracle_dequantize.restype = None
            lib.hqq_oracle_quantize_meta.argtypes = [P, i64, i32, P, P]
            lib.hqq_oracle_quantize_meta.restype = None
            lib.hqq_oracle_dequantize_meta.argtypes = [P, P, i64, i32, P]
            lib.hqq_oracle_dequantize_meta.restype = None
            _lib = lib
    return _lib


def _ptr(a: np.ndarray) -> int:
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data


def _f32(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.float32))


def default_threads() -> int:
    return max(1, len(os.sched_getaffinity(0)))


def quantize(W, nbits: int, group_size: int, axis: int, iters: int, p: float, beta0: float,
             kappa: float, group_ids=None, nthreads: int = 1, with_err: bool = False):
    """Quantize the fp32 matrix W (2-D).

    Returns (codes [n_sel, G] uint8 in group order, scale [n_sel] f32, zero [n_sel] f32)
    and, if ``with_err``, the best lp error per group. With ``group_ids`` only those groups
    (g order indices) are solved; outputs follow the order of ``group_ids``.
    """
    W = _f32(W)
    rows, cols = W.shape
    lib = _load()
    if group_ids is None:
        n = rows * cols // group_size
        ids_ptr, n_sel = None, 0
    else:
        ids = np.ascontiguousarray(np.asarray(group_ids, dtype=np.int64))
        n = ids.size
        ids_ptr, n_sel = _ptr(ids), n
    codes = np.zeros((n, group_size), np.uint8)
    scale = np.zeros(n, np.float32)
    zero = np.zeros(n, np.float32)
    err = np.zeros(n, np.float32) if with_err else None
    rc = lib.hqq_oracle_quantize(_ptr(W), rows, cols, nbits, group_size, axis, iters, p, beta0,
                                 kappa, ids_ptr, n_sel, _ptr(codes), _ptr(scale), _ptr(zero),
                                 _ptr(err) if with_err else None, nthreads)
    if rc != 0:
        raise ValueError("oracle rejected the arguments")
    if with_err:
        return codes, scale, zero, err
    return codes, scale, zero


def quantize_group(w, nbits: int, iters: int, p: float, beta0: float, kappa: float):
    """Solve one group; returns dict(codes, scale, zero, best_err, z_trace, e_trace)."""
    w = _f32(w).ravel()
    G = w.size
    lib = _load()
    codes = np.zeros(G, np.uint8)
    s = np.zeros(1, np.float32)
    z = np.zeros(1, np.float32)
    zt = np.zeros(iters + 1, np.float32)
    et = np.zeros(iters + 1, np.float32)
    best = lib.hqq_oracle_quantize_group(_ptr(w), G, nbits, iters, p, beta0, kappa, _ptr(codes),
                                         _ptr(s), _ptr(z), _ptr(zt), _ptr(et))
    return dict(codes=codes, scale=np.float32(s[0]), zero=np.float32(z[0]),
                best_err=np.float32(best), z_trace=zt, e_trace=et)


def codes_at_zero(w, nbits: int, zero: float) -> np.ndarray:
    """Final-code step alone for one group at a given zero."""
    w = _f32(w).ravel()
    out = np.zeros(w.size, np.uint8)
    _load().hqq_oracle_codes_at_zero(_ptr(w), w.size, nbits, float(zero), _ptr(out))
    return out


def pow_pm1(a: float, p: float) -> np.float32:
    """a^(p-1) (a > 0) rounded once to fp32, as the solver's shrinkage and error use it."""
    return np.float32(_load().hqq_oracle_pow_pm1(a, p))


def shrink(r: float, beta: float, p: float) -> np.float32:
    return np.float32(_load().hqq_oracle_shrink(r, beta, p))


def packed_bytes(n: int, nbits: int) -> int:
    return int(_load().hqq_oracle_packed_bytes(n, nbits))


def pack(codes, nbits: int) -> np.ndarray:
    c = np.ascontiguousarray(np.asarray(codes, dtype=np.uint8).ravel())
    out = np.zeros(packed_bytes(c.size, nbits), np.uint8)
    _load().hqq_oracle_pack(_ptr(c), c.size, nbits, _ptr(out))
    return out


def unpack(packed, n: int, nbits: int) -> np.ndarray:
    pk = np.ascontiguousarray(np.asarray(packed, dtype=np.uint8).ravel())
    assert pk.size >= packed_bytes(n, nbits)
    out = np.zeros(n, np.uint8)
    _load().hqq_oracle_unpack(_ptr(pk), n, nbits, _ptr(out))
    return out


def dequantize(codes, scale, zero, rows: int, cols: int, group_size: int, axis: int):
    """fp32 [rows, cols] reconstruction (float(Q) - zero) * scale from g-order codes."""
    c = np.ascontiguousarray(np.asarray(codes, dtype=np.uint8).ravel())
    s, z = _f32(scale).ravel(), _f32(zero).ravel()
    out = np.zeros((rows, cols), np.float32)
    _load().hqq_oracle_dequantize(_ptr(c), _ptr(s), _ptr(z), rows, cols, group_size, axis,
                                  _ptr(out))
    return out


def quantize_meta(m, group: int):
    """Second level: returns (q uint8 [n], mm f32 [runs, 2] = (step2, zero2))."""
    m = _f32(m).ravel()
    runs = (m.size + group - 1) // group
    q = np.zeros(m.size, np.uint8)
    mm = np.zeros((runs, 2), np.float32)
    _load().hqq_oracle_quantize_meta(_ptr(m), m.size, group, _ptr(q), _ptr(mm))
    return q, mm


def dequantize_meta(q, mm, group: int) -> np.ndarray:
    q = np.ascontiguousarray(np.asarray(q, dtype=np.uint8).ravel())
    mm = _f32(mm)
    out = np.zeros(q.size, np.float32)
    _load().hqq_oracle_dequantize_meta(_ptr(q), _ptr(mm), q.size, group, _ptr(out))
    return out


def round_to_dtype(a, dtype: str) -> np.ndarray:
    """Round fp32 values once, to nearest with ties to even, to ``"bf16"`` or ``"f16"``;
    returned as fp32 (which holds every such value exactly). ``"f32"`` returns a copy.

    bf16 keeps the upper 16 bits of the fp32 pattern: adding 0x7FFF plus the lowest kept bit
    and truncating rounds half to even (finite inputs; the path produces no NaN)."""
    x = _f32(a)
    if dtype == "f32":
        return x.copy()
    if dtype == "f16":
        return x.astype(np.float16).astype(np.float32)
    if dtype != "bf16":
        raise ValueError(dtype)
    b = x.view(np.uint32).astype(np.uint64)
    r = (b + 0x7FFF + ((b >> 16) & 1)) & 0xFFFF0000
    return r.astype(np.uint32).view(np.float32).reshape(x.shape)


def linear(X, codes, scale, zero, N: int, K: int, dtype: str, bias=None) -> np.ndarray:
    """Forward pass of a quantized linear layer, in fp64: Y[m, n] = sum_k X[m, k]·W'[n, k]
    (+ bias[n]), where W' is the axis-1, group-64 weight [N, K] dequantized by
    ``dequantize`` and rounded once to the compute dtype ("HQQ calibration-free guide"
    (lnwmold.com) §3.2: the layer dequantizes to compute_dtype and multiplies; §4.2: the
    axis=1 backends fuse the two). X holds the activations' exact values (fp32 array of
    bf16/fp16 numbers) [M, K]; codes are in g order. The product is numpy's float64 matmul:
    a library primitive whose result differs from the exact sum by far less than any fp32
    accumulation does. The caller rounds Y to the compute dtype where it compares bits."""
    Wd = round_to_dtype(dequantize(codes, scale, zero, N, K, 64, 1), dtype)
    Y = np.asarray(X, dtype=np.float64) @ Wd.astype(np.float64).T
    if bias is not None:
        Y = Y + np.asarray(bias, dtype=np.float64)[None, :]
    return Y


def _mx_sigs(L):
    u8p = ctypes.c_void_p
    L.hqq_oracle_e2m1_encode.argtypes = [ctypes.c_float]
    L.hqq_oracle_e2m1_encode.restype = ctypes.c_uint8
    L.hqq_oracle_e2m1_decode.argtypes = [ctypes.c_uint8]
    L.hqq_oracle_e2m1_decode.restype = ctypes.c_float
    L.hqq_oracle_mx_exponent.argtypes = [u8p, ctypes.c_int]
    L.hqq_oracle_mx_exponent.restype = ctypes.c_int
    L.hqq_oracle_mxfp4_quantize.argtypes = [u8p, ctypes.c_int64, ctypes.c_int64, u8p, u8p]
    L.hqq_oracle_mxfp4_dequantize.argtypes = [u8p, u8p, ctypes.c_int64, ctypes.c_int64, u8p]


def e2m1_encode(v: float) -> int:
    """One FP4 E2M1 code (sign bit 3, magnitude index 0..7) for an fp32 value: nearest
    E2M1 value, ties to the even mantissa bit, saturating at 6 (MX conversion)."""
    L = _load()
    _mx_sigs(L)
    return int(L.hqq_oracle_e2m1_encode(float(np.float32(v))))


def e2m1_decode(code: int) -> float:
    L = _load()
    _mx_sigs(L)
    return float(L.hqq_oracle_e2m1_decode(code))


def mx_exponent(v) -> int:
    """Shared exponent of one block: floor(log2 max|v|) - 2, clamped to [-127, 127]."""
    L = _load()
    _mx_sigs(L)
    a = _f32(v).ravel()
    return int(L.hqq_oracle_mx_exponent(_ptr(a), a.size))


def mxfp4_quantize(W):
    """MXFP4 encoding of the fp32 matrix W [rows, cols] (cols % 32 == 0), blocks of 32 along
    rows: returns (codes uint8 [rows*cols/2], scales uint8 [rows*cols/32] = e + 127)."""
    L = _load()
    _mx_sigs(L)
    W = _f32(W)
    rows, cols = W.shape
    assert cols % 32 == 0
    codes = np.zeros(rows * cols // 2, np.uint8)
    scales = np.zeros(rows * cols // 32, np.uint8)
    L.hqq_oracle_mxfp4_quantize(_ptr(W), rows, cols, _ptr(codes), _ptr(scales))
    return codes, scales


def mxfp4_dequantize(codes, scales, rows: int, cols: int) -> np.ndarray:
    """fp32 [rows, cols]: E2M1 value x 2^(scale - 127)."""
    L = _load()
    _mx_sigs(L)
    c = np.ascontiguousarray(np.asarray(codes, np.uint8).ravel())
    s = np.ascontiguousarray(np.asarray(scales, np.uint8).ravel())
    out = np.zeros((rows, cols), np.float32)
    L.hqq_oracle_mxfp4_dequantize(_ptr(c), _ptr(s), rows, cols, _ptr(out))
    return out
