"""Host-side checks of the C ABI (no GPU): the library loads, exports every function that
include/hqq/hqq.h declares, its size helpers agree with the layout, and argument errors are
reported synchronously before any CUDA call (fake non-null pointers are never dereferenced
because every call here fails validation or has nothing to do)."""
import ctypes
import math
import os
import re

import pytest
import torch

import calibration_free_weight_hqq_b200 as hqq

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "hqq", "hqq.h")

OK, INVALID, UNSUPPORTED, SHAPE, ALIGN, CUDA, WORKSPACE = range(7)
FAKE = 0x100000  # 16-byte aligned, never dereferenced
FAKE_ODD = 0x100002


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(hqq_\w+)\s*\(", text)))


@pytest.fixture(scope="module")
def L():
    return hqq.lib()


def test_exports_every_declared_symbol(L):
    names = declared_functions()
    assert "hqq_quantize" in names and "hqq_dequantize" in names and len(names) >= 12
    for n in names:
        assert hasattr(L, n), n
    assert L.hqq_abi_version() == 5


def test_size_helpers_match_layout(L):
    import oracle
    for nbits in (1, 2, 3, 4, 8):
        for rows, cols in ((0, 0), (1, 64), (37, 128), (4096, 1024)):
            n = rows * cols
            assert hqq.hqq_packed_bytes(rows, cols, nbits) == oracle.packed_bytes(n, nbits)
    assert hqq.hqq_packed_bytes(4096, 1024, 5) == 0
    assert hqq.hqq_num_groups(4096, 1024, 64, 1) == 65536
    assert hqq.hqq_num_groups(4096, 1024, 64, 0) == 65536
    assert hqq.hqq_num_groups(100, 1024, 64, 0) == -1
    assert hqq.hqq_num_groups(100, 1000, 64, 1) == -1
    assert hqq.hqq_num_groups(64, 64, 48, 1) == -1
    assert hqq.hqq_num_meta_groups(300, 128) == 3
    p = hqq.make_params(nbits=3, group_size=64, quant_scale=True, quant_zero=True)
    ng = 28672 * 8192 // 64
    assert hqq.hqq_workspace_bytes(28672, 8192, p) == 2 * math.ceil(ng * 4 / 256) * 256
    p0 = hqq.make_params()
    assert hqq.hqq_workspace_bytes(28672, 8192, p0) == 0


def test_status_strings(L):
    for code, name in enumerate(["HQQ_OK", "HQQ_ERR_INVALID_ARG", "HQQ_ERR_UNSUPPORTED",
                                 "HQQ_ERR_SHAPE", "HQQ_ERR_ALIGNMENT", "HQQ_ERR_CUDA",
                                 "HQQ_ERR_WORKSPACE"]):
        assert L.hqq_status_string(code).decode() == name


def q(L, **kw):
    a = dict(W=FAKE, dtype=1, rows=64, cols=128, nbits=4, G=64, axis=1, iters=20, p=0.7,
             beta0=10.0, kappa=1.01, packed=FAKE, scale=FAKE, zero=FAKE)
    a.update(kw)
    return L.hqq_quantize(a["W"], a["dtype"], a["rows"], a["cols"], a["nbits"], a["G"],
                          a["axis"], a["iters"], a["p"], a["beta0"], a["kappa"], a["packed"],
                          a["scale"], a["zero"], None)


@pytest.mark.parametrize("kw,status", [
    (dict(nbits=5), UNSUPPORTED), (dict(nbits=0), UNSUPPORTED), (dict(G=48), UNSUPPORTED),
    (dict(G=512), UNSUPPORTED), (dict(axis=2), UNSUPPORTED), (dict(dtype=3), UNSUPPORTED),
    (dict(cols=100), SHAPE), (dict(axis=0, rows=100), SHAPE), (dict(rows=-1), INVALID),
    (dict(iters=-1), INVALID), (dict(iters=100000), INVALID), (dict(p=0.0), INVALID),
    (dict(p=1.5), INVALID), (dict(p=float("nan")), INVALID), (dict(beta0=0.0), INVALID),
    (dict(beta0=float("inf")), INVALID), (dict(kappa=0.5), INVALID), (dict(W=0), INVALID),
    (dict(packed=0), INVALID), (dict(scale=0), INVALID), (dict(W=FAKE_ODD), ALIGN),
    (dict(packed=FAKE + 8), ALIGN), (dict(scale=FAKE + 1), ALIGN),
    (dict(rows=1 << 30, cols=1 << 30), SHAPE),
])
def test_quantize_rejects_bad_arguments(L, kw, status):
    assert q(L, **kw) == status


def test_empty_matrix_is_a_no_op(L):
    assert q(L, rows=0) == OK
    assert q(L, cols=0) == OK


def test_quantize_ex_workspace_and_meta_checks(L):
    p = hqq.make_params(quant_scale=True, quant_zero=True)
    call = lambda **kw: L.hqq_quantize_ex(kw.get("W", FAKE), 64, 128, ctypes.byref(p), FAKE,
                                          FAKE, FAKE, kw.get("smm", FAKE), kw.get("zmm", FAKE),
                                          kw.get("ws", FAKE), kw.get("wsb", 0), None)
    assert call() == WORKSPACE
    assert call(ws=None, wsb=1 << 20) == WORKSPACE
    assert call(smm=None, wsb=1 << 20) == INVALID
    assert call(ws=FAKE + 4, wsb=1 << 20) == ALIGN
    bad = hqq.make_params(quant_scale=True, meta_group_size=4)
    assert L.hqq_quantize_ex(FAKE, 64, 128, ctypes.byref(bad), FAKE, FAKE, FAKE, FAKE, FAKE,
                             FAKE, 1 << 20, None) == UNSUPPORTED
    assert L.hqq_quantize_ex(FAKE, 64, 128, None, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 0,
                             None) == INVALID


def test_dequantize_rejects_bad_arguments(L):
    d = lambda **kw: L.hqq_dequantize(kw.get("pk", FAKE), FAKE, FAKE, kw.get("mdt", 1),
                                      kw.get("odt", 1), 64, kw.get("cols", 128),
                                      kw.get("nbits", 4), 64, 1, kw.get("out", FAKE), None)
    assert d(nbits=6) == UNSUPPORTED
    assert d(odt=3) == UNSUPPORTED
    assert d(cols=96) == SHAPE
    assert d(out=0) == INVALID
    assert d(out=FAKE + 2) == ALIGN
    assert L.hqq_dequantize_meta(FAKE, FAKE, 100, 3, FAKE, None) == UNSUPPORTED
    assert L.hqq_quantize_meta(FAKE, 1, -1, 128, FAKE, FAKE, None) == INVALID


def test_binding_has_no_cpu_path():
    W = torch.zeros(64, 128, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="CUDA"):
        hqq.hqq_quantize(W)


def test_batched_calls_validate_before_launch(L):
    m = hqq.HQQMatrix(FAKE, 64, 128, FAKE, FAKE, FAKE)
    bad = hqq.HQQMatrix(FAKE, 64, 100, FAKE, FAKE, FAKE)   # cols not a multiple of 64
    arr = (hqq.HQQMatrix * 2)(m, bad)
    p = hqq.make_params()
    assert L.hqq_quantize_batched(arr, 2, ctypes.byref(p), None) == SHAPE
    assert L.hqq_dequantize_batched(arr, 2, ctypes.byref(p), 1, None) == SHAPE
    assert L.hqq_quantize_batched(None, 3, ctypes.byref(p), None) == INVALID
    assert L.hqq_quantize_batched(arr, -1, ctypes.byref(p), None) == INVALID
    q = hqq.make_params(quant_scale=True)
    assert L.hqq_quantize_batched(arr, 1, ctypes.byref(q), None) == UNSUPPORTED
    empty = (hqq.HQQMatrix * 1)(hqq.HQQMatrix(None, 0, 128, None, None, None))
    assert L.hqq_quantize_batched(empty, 1, ctypes.byref(p), None) == OK
    assert L.hqq_quantize_batched(arr, 0, ctypes.byref(p), None) == OK
    odd = (hqq.HQQMatrix * 1)(hqq.HQQMatrix(FAKE + 8, 64, 128, FAKE, FAKE, FAKE))
    assert L.hqq_quantize_batched(odd, 1, ctypes.byref(p), None) == ALIGN


def test_mixed_plan_groups_equal_configurations():
    # the pages' per-layer recipes: 8-bit g128 for the first block / output head, 4-bit g64
    # elsewhere ("HQQ tutorial" §4.2), 2-bit g16 MLP ("hqq-quantization skill summary")
    c8 = hqq.make_params(8, 128)
    c4 = hqq.make_params(4, 64)
    c2 = hqq.make_params(2, 16)
    c4b = hqq.make_params(4, 64)  # equal to c4 field by field: the same group
    assert hqq.hqq_mixed_plan([c8, c4, c2, c4b, c2, c8]) == ([0, 1, 2, 1, 2, 0], 3)
    # any field that reaches a kernel separates configurations
    variants = [hqq.make_params(4, 64, axis=0), hqq.make_params(4, 64, iters=5),
                hqq.make_params(4, 64, p=0.5), hqq.make_params(4, 64, w_dtype=torch.float16),
                hqq.make_params(4, 64, meta_dtype=torch.float32),
                hqq.make_params(4, 64, stop_at_fixed_point=True)]
    groups, k = hqq.hqq_mixed_plan([c4] + variants)
    assert groups == list(range(1 + len(variants))) and k == 1 + len(variants)
    assert hqq.hqq_mixed_plan([]) == ([], 0)


def test_mixed_calls_validate_every_matrix_before_launch(L):
    good = hqq.HQQMatrix(FAKE, 64, 128, FAKE, FAKE, FAKE)
    arr = (hqq.HQQMatrix * 2)(good, good)
    ok4, bad5 = hqq.make_params(4, 64), hqq.make_params(4, 64)
    bad5.nbits = 5
    prm = (hqq.HQQParams * 2)(ok4, bad5)
    assert L.hqq_quantize_mixed(arr, prm, 2, None) == UNSUPPORTED
    assert L.hqq_dequantize_mixed(arr, prm, 2, 1, None) == UNSUPPORTED
    # the second matrix does not fit its own configuration (cols % 256)
    prm = (hqq.HQQParams * 2)(ok4, hqq.make_params(8, 256))
    assert L.hqq_quantize_mixed(arr, prm, 2, None) == SHAPE
    assert L.hqq_dequantize_mixed(arr, prm, 2, 1, None) == SHAPE
    q = hqq.make_params(4, 64, quant_scale=True)
    prm = (hqq.HQQParams * 2)(ok4, q)
    assert L.hqq_quantize_mixed(arr, prm, 2, None) == UNSUPPORTED
    prm = (hqq.HQQParams * 2)(ok4, ok4)
    assert L.hqq_dequantize_mixed(arr, prm, 2, 7, None) == UNSUPPORTED
    assert L.hqq_quantize_mixed(None, prm, 2, None) == INVALID
    assert L.hqq_quantize_mixed(arr, None, 2, None) == INVALID
    assert L.hqq_quantize_mixed(arr, prm, -1, None) == INVALID
    assert L.hqq_quantize_mixed(arr, prm, 0, None) == OK
    empty = (hqq.HQQMatrix * 1)(hqq.HQQMatrix(None, 0, 128, None, None, None))
    assert L.hqq_quantize_mixed(empty, prm, 1, None) == OK
    assert L.hqq_mixed_plan(prm, -1, None, None) == INVALID


def test_unknown_flags_are_rejected(L):
    p = hqq.make_params()
    p.flags = 2
    assert L.hqq_quantize_ex(FAKE, 64, 128, ctypes.byref(p), FAKE, FAKE, FAKE, None, None, None,
                             0, None) == INVALID
    arr = (hqq.HQQMatrix * 1)(hqq.HQQMatrix(FAKE, 64, 128, FAKE, FAKE, FAKE))
    assert L.hqq_quantize_batched(arr, 1, ctypes.byref(p), None) == INVALID


def test_linear_validates_before_launch(L):
    BF16, F16, F32 = 1, 0, 2
    good = hqq.make_params(4, 64, 1, w_dtype=torch.bfloat16)

    def call(M=256, K=128, xdt=BF16, X=FAKE, W=FAKE, s=FAKE, z=FAKE, b=None, N=256,
             prm=good, Y=FAKE):
        return L.hqq_linear(X, M, K, xdt, W, s, z, b, N,
                            ctypes.byref(prm) if prm is not None else None, Y, None)

    assert call(prm=None) == INVALID
    assert call(M=-1) == INVALID
    assert call(xdt=F32) == UNSUPPORTED
    for kw in ({"nbits": 3}, {"group_size": 32}, {"axis": 0}, {"quant_scale": True}):
        args = dict(nbits=4, group_size=64, axis=1, w_dtype=torch.bfloat16)
        args.update(kw)
        assert call(prm=hqq.make_params(**args)) == UNSUPPORTED, kw
    bad_meta = hqq.make_params(4, 64, 1, w_dtype=torch.bfloat16)
    bad_meta.meta_dtype = 3
    assert call(prm=bad_meta) == INVALID
    # flags: the overlap promise (and the solver's fixed-point flag, ignored) are accepted
    # (the call then fails only for its fake pointers, after validation); other bits are not
    bad_flags = hqq.make_params(4, 64, 1, w_dtype=torch.bfloat16)
    bad_flags.flags = 4
    assert call(prm=bad_flags) == INVALID
    ok_flags = hqq.make_params(4, 64, 1, w_dtype=torch.bfloat16, overlap_weights=True,
                               stop_at_fixed_point=True)
    assert call(prm=ok_flags, K=96) == SHAPE  # validation continues past the flags
    # the quantize entry points refuse the linear layer's flag
    ovl = hqq.make_params(4, 64, 1, w_dtype=torch.bfloat16, overlap_weights=True)
    assert L.hqq_quantize_ex(FAKE, 64, 128, ctypes.byref(ovl), FAKE, FAKE, FAKE, None, None,
                             None, 0, None) == INVALID
    assert call(K=96) == SHAPE
    assert call(N=260) == SHAPE
    assert call(M=1 << 31) == SHAPE
    assert call(Y=None) == INVALID
    assert call(X=None) == INVALID
    assert call(X=FAKE_ODD) == ALIGN
    assert call(Y=FAKE + 8) == ALIGN
    assert call(b=FAKE + 1) == ALIGN
    # nothing to do: valid arguments with M == 0 or N == 0 return at once, pointers unused
    assert call(M=0, X=None, W=None, s=None, z=None, Y=None) == OK
    assert call(N=0, X=None, W=None, s=None, z=None, Y=None) == OK


def test_mxfp4_validates_before_launch(L):
    BF16, U8 = 1, 3
    assert L.hqq_mxfp4_quantize(FAKE, BF16, 4, 48, FAKE, FAKE, None) == SHAPE
    assert L.hqq_mxfp4_quantize(FAKE, U8, 4, 64, FAKE, FAKE, None) == UNSUPPORTED
    assert L.hqq_mxfp4_quantize(FAKE, BF16, -1, 64, FAKE, FAKE, None) == INVALID
    assert L.hqq_mxfp4_quantize(None, BF16, 4, 64, FAKE, FAKE, None) == INVALID
    assert L.hqq_mxfp4_quantize(FAKE_ODD, BF16, 4, 64, FAKE, FAKE, None) == ALIGN
    assert L.hqq_mxfp4_quantize(None, BF16, 0, 64, None, None, None) == OK
    assert L.hqq_mxfp4_dequantize(FAKE, FAKE, 4, 40, BF16, FAKE, None) == SHAPE
    assert L.hqq_mxfp4_dequantize(FAKE, FAKE, 4, 64, BF16, FAKE + 8, None) == ALIGN
    assert L.hqq_mxfp4_dequantize(FAKE, FAKE, 4, 64, U8, FAKE, None) == UNSUPPORTED
    assert L.hqq_mxfp4_dequantize(None, None, 4, 0, BF16, None, None) == OK


def test_mixed_model_workload_is_valid_for_its_configurations():
    # the --mixed bench workload: block 0 at 8-bit g128, attention 4-bit g64, MLP 2-bit g16;
    # every matrix fits its own configuration and the plan makes three launch groups
    from calibration_free_weight_hqq_b200 import workloads
    wl = workloads.llama7b_model_mixed()
    uniform = workloads.llama7b_model_4b()
    assert [(m.rows, m.cols, m.seed) for m in wl.matrices] == \
        [(m.rows, m.cols, m.seed) for m in uniform.matrices]
    counts = {}
    for m in wl.matrices:
        counts[(m.nbits, m.group_size)] = counts.get((m.nbits, m.group_size), 0) + 1
        assert hqq.hqq_num_groups(m.rows, m.cols, m.group_size, m.axis) > 0
    assert counts == {(8, 128): 7, (4, 64): 4 * 31, (2, 16): 3 * 31}
    cfgs = [hqq.make_params(m.nbits, m.group_size, m.axis, m.iters, m.p, m.beta0, m.kappa,
                            w_dtype=m.dtype) for m in wl.matrices]
    groups, k = hqq.hqq_mixed_plan(cfgs)
    assert k == 3 and groups[:7] == [0] * 7 and groups[7:11] == [1] * 4 and groups[11:14] == [2] * 3


def test_binding_rejects_buffers_from_another_device():
    # every buffer of a call must live on the device of its first input (the wrappers make
    # that device current for the launch); the check itself needs no GPU
    t = torch.zeros(4)
    hqq._same_device(torch.device("cpu"), t, "scale")
    with pytest.raises(ValueError, match="cuda:1"):
        hqq._same_device(torch.device("cuda", 1), t, "scale")

    class FakeStream:
        device = torch.device("cuda", 0)
        cuda_stream = 0
    with pytest.raises(ValueError, match="stream belongs to cuda:0"):
        hqq._stream(FakeStream(), torch.device("cuda", 1))
    assert hqq._stream(FakeStream(), torch.device("cuda", 0)) == 0


def test_noalloc_checks_arguments_before_its_size(L):
    # an oversized call (59 MB of scratch needed, the array holds 32 MiB) that is also invalid
    # reports what hqq_quantize_ex reports for it; only a valid oversized call is refused for
    # its size
    rows, cols = 28672, 8192

    def call(W=FAKE, **kw):
        p = hqq.make_params(**{**dict(nbits=1, group_size=32, quant_scale=True,
                                      quant_zero=True), **kw})
        na = L.hqq_quantize_ex_noalloc(W, rows, cols, ctypes.byref(p), FAKE, FAKE, FAKE, FAKE,
                                       FAKE, None)
        ex = L.hqq_quantize_ex(W, rows, cols, ctypes.byref(p), FAKE, FAKE, FAKE, FAKE, FAKE,
                               FAKE, 1 << 30, None)
        return na, ex

    assert call(p=0.0) == (INVALID, INVALID)
    assert call(nbits=5) == (UNSUPPORTED, UNSUPPORTED)
    assert call(W=FAKE_ODD) == (ALIGN, ALIGN)
    assert call(meta_group_size=4) == (UNSUPPORTED, UNSUPPORTED)
    assert call()[0] == WORKSPACE
