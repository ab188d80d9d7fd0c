"""Host-side checks of the C ABI: the library loads, exports every entry point
include/q8.h declares, and rejects bad arguments before touching a device.

None of these launch a kernel.  Pointers passed here are never dereferenced:
each call returns from host validation (or from the device check, which finds
no usable sm_100a device on a CPU-only machine).
"""
import ctypes
import os
import re

import pytest
import torch

from bit_quantized_b200 import build as q8build

q8build.build()
from bit_quantized_b200 import q8  # noqa: E402

HEADER = os.path.join(os.path.dirname(os.path.dirname(__file__)), "include", "q8.h")
FAKE = 0x10000          # 16-byte aligned, never dereferenced
MIS = 0x10008           # 8-byte aligned only
# Calls with valid arguments and fake pointers are made only where no GPU is
# visible: there they stop at the device check; on a GPU they would launch.
NO_GPU = not torch.cuda.is_available()


def _declared():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(q8_[a-z0-9_]+)\s*\(", text)))


def test_every_declared_symbol_is_exported():
    names = _declared()
    assert len(names) >= 12
    lib = ctypes.CDLL(q8.LIB_PATH)
    for name in names:
        assert hasattr(lib, name), name
    assert sorted(q8.EXPORTED) == names


def test_version_matches_header():
    m = re.search(r"#define Q8_VERSION (\d+)", open(HEADER).read())
    assert q8.q8_version() == int(m.group(1))


def test_status_strings():
    for s in range(11):
        assert q8.q8_status_string(s) not in ("", "unknown status")
    assert q8.q8_status_string(99) == "unknown status"


def test_workspace_size():
    ws = q8.q8_workspace_size(q8.Q8_OP_LINEAR_INT8_MIXED, 512, 4096, 4096)
    up = lambda v, a: (v + a - 1) // a * a
    kp = 4096
    want = (up(4096, 256) + up(4 * 4096, 256) + 256 + up(512 * 4096, 256) + 2 * up(4 * 512, 256)
            + up(2 * 512 * kp, 256) + up(2 * 4096 * kp, 256))
    assert ws == want
    assert q8.q8_workspace_size(q8.Q8_OP_LINEAR_W8A8, 16, 4096, 4096) == 0
    assert q8.q8_workspace_size(q8.Q8_OP_LINEAR_INT8_MIXED, 1, 16, 32) > 0


def test_workspace_size_out_of_range_sizes():
    # Sizes beyond 2^31 - 1 are never valid: the size function answers
    # SIZE_MAX instead of a product that could overflow into a small number.
    size_max = 2**64 - 1
    big = 2**31
    assert q8.q8_workspace_size(q8.Q8_OP_LINEAR_INT8_MIXED, big, 16, 32) == size_max
    assert q8.q8_workspace_size(q8.Q8_OP_LINEAR_INT8_MIXED, 16, 2**62, 32) == size_max
    assert q8.q8_workspace_size(q8.Q8_OP_LINEAR_INT8_MIXED, 16, 16, 2**62) == size_max
    assert q8.q8_workspace_size(q8.Q8_OP_LINEAR_INT8_MIXED, -1, 16, 32) == 0


def test_noalloc_validation_before_sizing():
    # The allocation-free entry point checks K against the weight and the
    # INT32 bound, and M against 2^31 - 1, before it sizes its scratch; all of
    # these fail without touching the device.
    f = L.q8_linear_int8_mixed_noalloc
    w = _weight(k=128, ld=128)

    def call(m=16, k=128, w=w):
        return f(FAKE, q8.Q8_F16, m, k, k, ctypes.byref(w), None, 6.0, None, FAKE, w.n, None, None,
                 None, None, _ns)
    assert f(FAKE, q8.Q8_F16, 16, 128, 128, None, None, 6.0, None, FAKE, 64, None, None, None,
             None, _ns) == q8.Q8_ERR_NULL
    assert call(k=256) == q8.Q8_ERR_SHAPE                       # k != w->k
    assert call(m=-1) == q8.Q8_ERR_SHAPE
    assert call(m=2**40) == q8.Q8_ERR_SHAPE                     # beyond 2^31 - 1
    wk = _weight(k=65536, ld=65536)
    assert call(k=65536, w=wk) == q8.Q8_ERR_SHAPE               # beyond the INT32 bound
    assert call(m=2**20, k=128) == q8.Q8_ERR_SHAPE              # scratch does not fit


def test_selftest_wait_timeout_validation():
    assert L.q8_selftest_wait_timeout(0, _ns) == q8.Q8_ERR_SHAPE
    assert L.q8_selftest_wait_timeout(-5, _ns) == q8.Q8_ERR_SHAPE
    assert L.q8_selftest_wait_timeout(1000001, _ns) == q8.Q8_ERR_SHAPE
    if NO_GPU:
        assert L.q8_selftest_wait_timeout(1000, _ns) in (q8.Q8_ERR_CUDA,
                                                         q8.Q8_ERR_UNSUPPORTED_ARCH)


L = q8.lib()
_ns = None


def qw(**kw):
    args = dict(W=FAKE, w_dtype=q8.Q8_BF16, n=64, k=128, ldw=128, scheme=q8.Q8_ASYM_INT8,
                code_dtype=q8.Q8_S8, codes=FAKE, scale=FAKE, zp=FAKE)
    args.update(kw)
    return L.q8_quantize_weight(args["W"], args["w_dtype"], args["n"], args["k"], args["ldw"],
                                args["scheme"], args["code_dtype"], args["codes"], args["scale"],
                                args["zp"], _ns)


def test_quantize_weight_validation():
    assert qw(W=None) == q8.Q8_ERR_NULL
    assert qw(zp=None) == q8.Q8_ERR_NULL                       # asymmetric needs Z
    assert qw(k=100, ldw=100) == q8.Q8_ERR_SHAPE               # K % 32
    assert qw(ldw=64) == q8.Q8_ERR_SHAPE                       # ld < k
    assert qw(n=-1) == q8.Q8_ERR_SHAPE
    assert qw(w_dtype=q8.Q8_S8) == q8.Q8_ERR_DTYPE
    assert qw(code_dtype=q8.Q8_E4M3) == q8.Q8_ERR_SCHEME
    assert qw(scheme=q8.Q8_SYM_INT8, code_dtype=q8.Q8_U8) == q8.Q8_ERR_SCHEME
    assert qw(scheme=7) == q8.Q8_ERR_SCHEME
    assert qw(W=MIS) == q8.Q8_ERR_ALIGN
    assert qw(ldw=132) == q8.Q8_ERR_ALIGN                      # 264 bytes
    # valid arguments reach the device check: no sm_100a device here
    if NO_GPU:
        assert qw() in (q8.Q8_ERR_CUDA, q8.Q8_ERR_UNSUPPORTED_ARCH)
    if NO_GPU:
        assert qw(scheme=q8.Q8_SYM_INT8, zp=None) in (q8.Q8_ERR_CUDA, q8.Q8_ERR_UNSUPPORTED_ARCH)


def qa(**kw):
    args = dict(X=FAKE, x_dtype=q8.Q8_F16, m=16, k=256, ldx=256, scheme=q8.Q8_SYM_INT8, ub=0.0,
                codes=FAKE, scale=FAKE, rowsum=FAKE)
    args.update(kw)
    return L.q8_quantize_act(args["X"], args["x_dtype"], args["m"], args["k"], args["ldx"],
                             args["scheme"], args["ub"], args["codes"], args["scale"],
                             args["rowsum"], _ns)


def test_quantize_act_validation():
    assert qa(codes=None) == q8.Q8_ERR_NULL
    assert qa(k=48, ldx=48) == q8.Q8_ERR_SHAPE
    assert qa(scheme=q8.Q8_ASYM_INT8) == q8.Q8_ERR_SCHEME
    assert qa(x_dtype=q8.Q8_E4M3) == q8.Q8_ERR_DTYPE
    assert qa(codes=MIS) == q8.Q8_ERR_ALIGN
    if NO_GPU:
        assert qa() in (q8.Q8_ERR_CUDA, q8.Q8_ERR_UNSUPPORTED_ARCH)
    assert qa(m=0) == q8.Q8_OK                                  # empty call: nothing launched
    assert qa(m=0, X=None, codes=None, scale=None) == q8.Q8_OK


def _weight(code_dtype=q8.Q8_S8, zp=FAKE, n=64, k=128, ld=128):
    return q8.CWeight(FAKE, code_dtype, FAKE, zp, n, k, ld)


def _act(code_dtype=q8.Q8_S8, m=16, k=128, ld=128, rowsum=FAKE):
    return q8.CAct(FAKE, code_dtype, FAKE, rowsum, m, k, ld)


def lin(x=None, w=None, Y=FAKE, ldy=64):
    x = x or _act()
    w = w or _weight()
    return L.q8_linear_w8a8(ctypes.byref(x), ctypes.byref(w), None, Y, ldy, None, None, 0, _ns)


def test_linear_w8a8_validation():
    assert lin(Y=None) == q8.Q8_ERR_NULL
    assert lin(x=_act(rowsum=None)) == q8.Q8_ERR_NULL          # zero point needs row sums
    assert lin(x=_act(k=256, ld=256)) == q8.Q8_ERR_SHAPE       # K mismatch
    assert lin(w=_weight(n=40)) == q8.Q8_ERR_SHAPE             # N % 16
    assert lin(ldy=32) == q8.Q8_ERR_SHAPE
    assert lin(x=_act(code_dtype=q8.Q8_E4M3)) == q8.Q8_ERR_DTYPE   # fp8 x int8
    assert lin(w=_weight(code_dtype=q8.Q8_E4M3)) == q8.Q8_ERR_SCHEME  # fp8 with zero point
    assert lin(x=_act(k=65536, ld=65536), w=_weight(k=65536, ld=65536)) == q8.Q8_ERR_SHAPE
    assert lin(Y=MIS) == q8.Q8_ERR_ALIGN
    assert lin(ldy=68) == q8.Q8_ERR_ALIGN
    if NO_GPU:
        assert lin() in (q8.Q8_ERR_CUDA, q8.Q8_ERR_UNSUPPORTED_ARCH)
    fx = _act(code_dtype=q8.Q8_E4M3, rowsum=None)
    if NO_GPU:
        assert lin(x=fx, w=_weight(code_dtype=q8.Q8_E4M3, zp=None)) in (
            q8.Q8_ERR_CUDA, q8.Q8_ERR_UNSUPPORTED_ARCH)


def mixed(w=None, ws=FAKE, ws_bytes=None, x_dtype=q8.Q8_F16, m=16, k=128, W16=None):
    w = w or _weight(k=k, ld=k)
    if ws_bytes is None:
        ws_bytes = q8.q8_workspace_size(q8.Q8_OP_LINEAR_INT8_MIXED, m, w.n, k)
    return L.q8_linear_int8_mixed(FAKE, x_dtype, m, k, k, ctypes.byref(w), W16, 6.0, None, FAKE,
                                  w.n, None, None, None, None, ws, ws_bytes, _ns)


def test_linear_int8_mixed_validation():
    assert mixed(ws=None) == q8.Q8_ERR_WORKSPACE
    assert mixed(ws_bytes=100) == q8.Q8_ERR_WORKSPACE
    assert mixed(ws=FAKE + 16) == q8.Q8_ERR_ALIGN              # workspace must be 256-aligned
    assert mixed(x_dtype=q8.Q8_BF16) == q8.Q8_ERR_DTYPE
    assert mixed(w=_weight(code_dtype=q8.Q8_E4M3, zp=None)) == q8.Q8_ERR_DTYPE
    assert mixed(W16=MIS) == q8.Q8_ERR_ALIGN
    if NO_GPU:
        assert mixed() in (q8.Q8_ERR_CUDA, q8.Q8_ERR_UNSUPPORTED_ARCH)


def test_outlier_act_validation():
    f = L.q8_outlier_quantize_act
    args = [FAKE, q8.Q8_F16, 16, 128, 128, 6.0, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 128, _ns]
    a = list(args); a[10] = None
    assert f(*a) == q8.Q8_ERR_NULL
    a = list(args); a[13] = 64
    assert f(*a) == q8.Q8_ERR_SHAPE                             # ldo < round_up(k, 64)
    a = list(args); a[1] = q8.Q8_BF16
    assert f(*a) == q8.Q8_ERR_DTYPE
    a = list(args); a[12] = MIS
    assert f(*a) == q8.Q8_ERR_ALIGN
    if NO_GPU:
        assert f(*args) in (q8.Q8_ERR_CUDA, q8.Q8_ERR_UNSUPPORTED_ARCH)


def test_device_calls_report_no_device():
    assert q8.q8_device_check() in (q8.Q8_ERR_CUDA, q8.Q8_ERR_UNSUPPORTED_ARCH, q8.Q8_OK)
    v = ctypes.c_int32(0)
    assert L.q8_get_device_status(None, _ns) == q8.Q8_ERR_NULL


def rq(x=None, w=None, Y=FAKE, ldy=64, out_scale=0.05):
    x = x or _act()
    w = w or _weight()
    return L.q8_linear_w8a8_requant(ctypes.byref(x), ctypes.byref(w), None, out_scale, Y, ldy, None, _ns)


def test_linear_w8a8_requant_validation():
    assert rq(Y=None) == q8.Q8_ERR_NULL
    assert rq(x=_act(rowsum=None)) == q8.Q8_ERR_NULL           # zero point needs row sums
    assert rq(ldy=32) == q8.Q8_ERR_SHAPE
    assert rq(x=_act(code_dtype=q8.Q8_E4M3)) == q8.Q8_ERR_DTYPE   # INT8 codes only
    for bad in (0.0, -1.0, float("inf"), float("nan")):
        assert rq(out_scale=bad) == q8.Q8_ERR_SCHEME
    assert rq(ldy=72) == q8.Q8_ERR_ALIGN                        # int8 rows: ldy % 16
    assert rq(Y=MIS) == q8.Q8_ERR_ALIGN
    assert rq(x=_act(m=0)) == q8.Q8_OK                          # empty call
    if NO_GPU:
        assert rq() in (q8.Q8_ERR_CUDA, q8.Q8_ERR_UNSUPPORTED_ARCH)


def qs(X=FAKE, m=16, k=128, ldx=128, scale=0.02, codes=FAKE, sc=FAKE, rs=FAKE, dt=q8.Q8_BF16):
    return L.q8_quantize_act_static(X, dt, m, k, ldx, scale, codes, sc, rs, _ns)


def test_quantize_act_static_validation():
    assert qs(X=None) == q8.Q8_ERR_NULL
    assert qs(sc=None) == q8.Q8_ERR_NULL
    assert qs(k=100, ldx=100) == q8.Q8_ERR_SHAPE                 # K % 32
    assert qs(ldx=64) == q8.Q8_ERR_SHAPE
    assert qs(dt=q8.Q8_S8) == q8.Q8_ERR_DTYPE
    for bad in (0.0, -0.5, float("inf"), float("nan")):
        assert qs(scale=bad) == q8.Q8_ERR_SCHEME
    assert qs(X=MIS) == q8.Q8_ERR_ALIGN
    assert qs(m=0, X=None, codes=None, sc=None) == q8.Q8_OK     # empty call
    if NO_GPU:
        assert qs(rs=None) in (q8.Q8_ERR_CUDA, q8.Q8_ERR_UNSUPPORTED_ARCH)


def qsm(X=FAKE, m=16, k=128, ldx=128, mult=FAKE, codes=FAKE, sc=FAKE, rs=FAKE, dt=q8.Q8_BF16):
    return L.q8_quantize_act_smooth(X, dt, m, k, ldx, mult, codes, sc, rs, _ns)


def test_quantize_act_smooth_validation():
    assert qsm(mult=None) == q8.Q8_ERR_NULL
    assert qsm(X=None) == q8.Q8_ERR_NULL
    assert qsm(k=100, ldx=100) == q8.Q8_ERR_SHAPE
    assert qsm(dt=q8.Q8_U8) == q8.Q8_ERR_DTYPE
    assert qsm(mult=MIS) == q8.Q8_ERR_ALIGN
    assert qsm(m=0, X=None, mult=None) == q8.Q8_OK               # empty call
    if NO_GPU:
        assert qsm() in (q8.Q8_ERR_CUDA, q8.Q8_ERR_UNSUPPORTED_ARCH)


def qg4(W=FAKE, dt=q8.Q8_BF16, n=256, k=512, ldw=512, group=128, codes=FAKE, ldc=256, sc=FAKE):
    return L.q8_quantize_weight_g4(W, dt, n, k, ldw, group, codes, ldc, sc, _ns)


def test_quantize_weight_g4_validation():
    assert qg4(W=None) == q8.Q8_ERR_NULL
    assert qg4(sc=None) == q8.Q8_ERR_NULL
    assert qg4(dt=q8.Q8_F32) == q8.Q8_ERR_DTYPE
    for bad in (16, 48, 256):
        assert qg4(group=bad) == q8.Q8_ERR_SCHEME
    assert qg4(k=480, ldw=480) == q8.Q8_ERR_SHAPE               # k % group
    assert qg4(n=200) == q8.Q8_ERR_SHAPE                         # n % 16
    assert qg4(ldc=128) == q8.Q8_ERR_SHAPE                       # ldc < k / 2
    assert qg4(ldc=264) == q8.Q8_ERR_ALIGN                       # ldc % 16
    assert qg4(codes=MIS) == q8.Q8_ERR_ALIGN
    assert qg4(n=0, W=None, codes=None, sc=None) == q8.Q8_OK      # empty call
    if NO_GPU:
        assert qg4() in (q8.Q8_ERR_CUDA, q8.Q8_ERR_UNSUPPORTED_ARCH)


def _wg4(n=256, k=512, ld=256, group=64, codes=FAKE, scale=FAKE):
    return q8.CWeightG4(codes, scale, n, k, ld, group)


def lw4(X=FAKE, dt=q8.Q8_BF16, m=16, k=512, ldx=512, w=None, bias=None, Y=FAKE, ldy=256):
    w = w or _wg4()
    return L.q8_linear_w4a16(X, dt, m, k, ldx, ctypes.byref(w), bias, Y, ldy, _ns)


def test_linear_w4a16_validation():
    assert L.q8_linear_w4a16(FAKE, q8.Q8_BF16, 16, 512, 512, None, None, FAKE, 256, _ns) == q8.Q8_ERR_NULL
    assert lw4(Y=None) == q8.Q8_ERR_NULL
    assert lw4(w=_wg4(scale=None)) == q8.Q8_ERR_NULL
    assert lw4(dt=q8.Q8_S8) == q8.Q8_ERR_DTYPE
    assert lw4(dt=q8.Q8_F32) == q8.Q8_ERR_DTYPE
    assert lw4(w=_wg4(group=96)) == q8.Q8_ERR_SCHEME
    assert lw4(k=256, ldx=256) == q8.Q8_ERR_SHAPE                # k != w.k
    assert lw4(w=_wg4(ld=128)) == q8.Q8_ERR_SHAPE                # ld < k / 2
    assert lw4(w=_wg4(n=200, ld=256)) == q8.Q8_ERR_SHAPE         # n % 16
    assert lw4(ldy=128) == q8.Q8_ERR_SHAPE                       # ldy < n
    assert lw4(m=65535 * 256 + 1) == q8.Q8_ERR_SHAPE
    assert lw4(ldy=260) == q8.Q8_ERR_ALIGN
    assert lw4(X=MIS) == q8.Q8_ERR_ALIGN
    assert lw4(bias=MIS) == q8.Q8_ERR_ALIGN
    assert lw4(w=_wg4(ld=264)) == q8.Q8_ERR_ALIGN
    assert lw4(m=0, X=None, Y=None) == q8.Q8_OK                  # empty call
    if NO_GPU:
        assert lw4() in (q8.Q8_ERR_CUDA, q8.Q8_ERR_UNSUPPORTED_ARCH)


def q4k(W=FAKE, dt=q8.Q8_BF16, n=256, k=512, ldw=512, codes=FAKE, ldc=256, sc=FAKE, sub=FAKE, sup=FAKE):
    return L.q8_quantize_weight_q4k(W, dt, n, k, ldw, codes, ldc, sc, sub, sup, _ns)


def test_quantize_weight_q4k_validation():
    assert q4k(sub=None) == q8.Q8_ERR_NULL
    assert q4k(sup=None) == q8.Q8_ERR_NULL
    assert q4k(dt=q8.Q8_F32) == q8.Q8_ERR_DTYPE
    assert q4k(k=384, ldw=384, ldc=192) == q8.Q8_ERR_SHAPE      # k % 256
    assert q4k(n=40) == q8.Q8_ERR_SHAPE
    assert q4k(ldc=128) == q8.Q8_ERR_SHAPE
    assert q4k(sub=MIS) == q8.Q8_ERR_ALIGN
    assert q4k(ldc=264) == q8.Q8_ERR_ALIGN
    assert q4k(n=0, W=None) == q8.Q8_OK
    if NO_GPU:
        assert q4k() in (q8.Q8_ERR_CUDA, q8.Q8_ERR_UNSUPPORTED_ARCH)


def test_expand_q4k_scales_validation():
    f = L.q8_expand_q4k_scales
    assert f(None, FAKE, 256, 512, FAKE, _ns) == q8.Q8_ERR_NULL
    assert f(FAKE, FAKE, 256, 320, FAKE, _ns) == q8.Q8_ERR_SHAPE
    assert f(FAKE, MIS, 256, 512, FAKE, _ns) == q8.Q8_ERR_ALIGN
    assert f(None, None, 0, 512, None, _ns) == q8.Q8_OK
    if NO_GPU:
        assert f(FAKE, FAKE, 256, 512, FAKE, _ns) in (q8.Q8_ERR_CUDA, q8.Q8_ERR_UNSUPPORTED_ARCH)


def lmoe(x=None, w=None, E=4, offsets=FAKE, bias=None, Y=FAKE, ldy=64):
    x = x or _act(code_dtype=q8.Q8_E4M3, rowsum=None)
    w = w or _weight(code_dtype=q8.Q8_E4M3, zp=None, n=256)
    return L.q8_linear_fp8_grouped(ctypes.byref(x), ctypes.byref(w), E, offsets, bias, Y, ldy, _ns)


def test_linear_fp8_grouped_validation():
    assert L.q8_linear_fp8_grouped(None, None, 4, FAKE, None, FAKE, 64, _ns) == q8.Q8_ERR_NULL
    assert lmoe(offsets=None) == q8.Q8_ERR_NULL
    assert lmoe(Y=None) == q8.Q8_ERR_NULL
    assert lmoe(x=_act()) == q8.Q8_ERR_DTYPE                     # INT8 activations
    assert lmoe(w=_weight(zp=None, n=256)) == q8.Q8_ERR_DTYPE    # INT8 weights
    assert lmoe(E=0) == q8.Q8_ERR_SHAPE
    assert lmoe(E=3) == q8.Q8_ERR_SHAPE                          # n not divisible by experts
    assert lmoe(E=32) == q8.Q8_ERR_SHAPE                         # 8 channels per expert
    assert lmoe(ldy=16) == q8.Q8_ERR_SHAPE                       # ldy < n
    assert lmoe(ldy=68) == q8.Q8_ERR_ALIGN
    assert lmoe(offsets=FAKE + 2) == q8.Q8_ERR_ALIGN
    assert lmoe(bias=MIS) == q8.Q8_ERR_ALIGN
    assert lmoe(x=_act(code_dtype=q8.Q8_E4M3, rowsum=None, m=0), Y=None) == q8.Q8_OK
    if NO_GPU:
        assert lmoe() in (q8.Q8_ERR_CUDA, q8.Q8_ERR_UNSUPPORTED_ARCH)


def test_injected_failure_propagates_and_disarms():
    inj = L.q8_inject_failure
    try:
        assert inj(99, 0) == q8.Q8_ERR_SCHEME
        assert inj(q8.Q8_ERR_LAUNCH, -1) == q8.Q8_ERR_SHAPE
        assert inj(q8.Q8_ERR_LAUNCH, 0) == q8.Q8_OK
        assert qs(X=None) == q8.Q8_ERR_NULL            # failed validation: not counted
        assert q8.q8_device_check() != q8.Q8_ERR_LAUNCH # status calls are not affected
        assert qs() == q8.Q8_ERR_LAUNCH                # the next validated call fails ...
        if NO_GPU:                                      # ... once
            assert qs() in (q8.Q8_ERR_CUDA, q8.Q8_ERR_UNSUPPORTED_ARCH)
            assert inj(q8.Q8_ERR_WORKSPACE, 1) == q8.Q8_OK
            assert lw4() in (q8.Q8_ERR_CUDA, q8.Q8_ERR_UNSUPPORTED_ARCH)   # skipped
            assert lmoe() == q8.Q8_ERR_WORKSPACE
        assert inj(q8.Q8_ERR_DEVICE_TIMEOUT, 0) == q8.Q8_OK
        with pytest.raises(q8.Q8Error) as e:           # the binding raises the injected status
            q8._check(lw4(), "q8_linear_w4a16")
        assert e.value.status == q8.Q8_ERR_DEVICE_TIMEOUT
        q8.q8_inject_failure(q8.Q8_ERR_LAUNCH, 3)
        q8.q8_inject_failure(q8.Q8_OK)                 # disarm
        if NO_GPU:
            assert qs() in (q8.Q8_ERR_CUDA, q8.Q8_ERR_UNSUPPORTED_ARCH)
    finally:
        inj(q8.Q8_OK, 0)
