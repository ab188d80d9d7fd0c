"""Thin Python binding of libq8.so (include/q8.h), same names as the C ABI.

Argument marshalling only: each function checks that tensors are CUDA tensors
of the expected dtype, allocates outputs with torch when the caller does not
pass them, and calls the C entry point with raw device pointers and the
current torch CUDA stream.  Every step of the computation runs in the
library's kernels; there is no fallback.  If libq8.so is missing, importing
this module raises.
"""
from __future__ import annotations

import ctypes
import dataclasses
import os
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libq8.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with `python -m bit_quantized_b200.build` "
        "(the q8 CUDA library has no fallback)")

_lib = ctypes.CDLL(LIB_PATH)

# ---------------------------------------------------------------- C types

Q8_OK, Q8_ERR_NULL, Q8_ERR_SHAPE, Q8_ERR_ALIGN, Q8_ERR_DTYPE, Q8_ERR_SCHEME = range(6)
Q8_ERR_UNSUPPORTED_ARCH, Q8_ERR_LAUNCH, Q8_ERR_DEVICE_TIMEOUT, Q8_ERR_WORKSPACE, Q8_ERR_CUDA = range(6, 11)
Q8_S8, Q8_U8, Q8_E4M3, Q8_F16, Q8_BF16, Q8_F32, Q8_S32 = range(7)
Q8_ASYM_INT8, Q8_SYM_INT8, Q8_FP8_E4M3 = range(3)
Q8_OP_LINEAR_W8A8, Q8_OP_LINEAR_INT8_MIXED = 0, 1
Q8_NOALLOC_SCRATCH_BYTES = 64 << 20

EXPORTED = [
    "q8_quantize_weight", "q8_dequantize_weight", "q8_quantize_act", "q8_quantize_act_static",
    "q8_quantize_act_smooth",
    "q8_outlier_quantize_act",
    "q8_linear_w8a8", "q8_linear_w8a8_requant", "q8_linear_w8a8_dynamic", "q8_linear_int8_mixed",
    "q8_linear_int8_mixed_noalloc",
    "q8_quantize_weight_g4", "q8_quantize_weight_q4k", "q8_expand_q4k_scales", "q8_linear_w4a16",
    "q8_linear_fp8_grouped",
    "q8_workspace_size", "q8_status_string",
    "q8_get_device_status", "q8_clear_device_status", "q8_device_check", "q8_version",
    "q8_inject_failure", "q8_selftest_wait_timeout",
]


class CWeight(ctypes.Structure):
    _fields_ = [("codes", ctypes.c_void_p), ("code_dtype", ctypes.c_int),
                ("scale", ctypes.c_void_p), ("zero_point", ctypes.c_void_p),
                ("n", ctypes.c_int64), ("k", ctypes.c_int64), ("ld", ctypes.c_int64)]


class CAct(ctypes.Structure):
    _fields_ = [("codes", ctypes.c_void_p), ("code_dtype", ctypes.c_int),
                ("scale", ctypes.c_void_p), ("rowsum", ctypes.c_void_p),
                ("m", ctypes.c_int64), ("k", ctypes.c_int64), ("ld", ctypes.c_int64)]


class CWeightG4(ctypes.Structure):
    _fields_ = [("codes", ctypes.c_void_p), ("scale", ctypes.c_void_p),
                ("n", ctypes.c_int64), ("k", ctypes.c_int64), ("ld", ctypes.c_int64),
                ("group", ctypes.c_int32)]


_i64, _int, _f, _vp, _sz = ctypes.c_int64, ctypes.c_int, ctypes.c_float, ctypes.c_void_p, ctypes.c_size_t
_SIG = {
    "q8_quantize_weight": ([_vp, _int, _i64, _i64, _i64, _int, _int, _vp, _vp, _vp, _vp], _int),
    "q8_dequantize_weight": ([ctypes.POINTER(CWeight), _int, _vp, _vp], _int),
    "q8_quantize_act": ([_vp, _int, _i64, _i64, _i64, _int, _f, _vp, _vp, _vp, _vp], _int),
    "q8_quantize_act_static": ([_vp, _int, _i64, _i64, _i64, _f, _vp, _vp, _vp, _vp], _int),
    "q8_quantize_act_smooth": ([_vp, _int, _i64, _i64, _i64, _vp, _vp, _vp, _vp, _vp], _int),
    "q8_outlier_quantize_act": ([_vp, _int, _i64, _i64, _i64, _f, _vp, _vp, _vp, _vp, _vp, _vp,
                                 _vp, _i64, _vp], _int),
    "q8_linear_w8a8": ([ctypes.POINTER(CAct), ctypes.POINTER(CWeight), _vp, _vp, _i64, _vp, _vp,
                        _sz, _vp], _int),
    "q8_linear_w8a8_requant": ([ctypes.POINTER(CAct), ctypes.POINTER(CWeight), _vp, _f, _vp, _i64,
                                _vp, _vp], _int),
    "q8_linear_w8a8_dynamic": ([_vp, _int, _i64, _i64, _i64, _int, _f, ctypes.POINTER(CWeight),
                                _vp, _vp, _i64, _vp, _vp, _vp, _vp, _vp], _int),
    "q8_linear_int8_mixed": ([_vp, _int, _i64, _i64, _i64, ctypes.POINTER(CWeight), _vp, _f, _vp,
                              _vp, _i64, _vp, _vp, _vp, _vp, _vp, _sz, _vp], _int),
    "q8_linear_int8_mixed_noalloc": ([_vp, _int, _i64, _i64, _i64, ctypes.POINTER(CWeight), _vp,
                                      _f, _vp, _vp, _i64, _vp, _vp, _vp, _vp, _vp], _int),
    "q8_quantize_weight_g4": ([_vp, _int, _i64, _i64, _i64, ctypes.c_int32, _vp, _i64, _vp, _vp],
                              _int),
    "q8_quantize_weight_q4k": ([_vp, _int, _i64, _i64, _i64, _vp, _i64, _vp, _vp, _vp, _vp], _int),
    "q8_expand_q4k_scales": ([_vp, _vp, _i64, _i64, _vp, _vp], _int),
    "q8_linear_fp8_grouped": ([ctypes.POINTER(CAct), ctypes.POINTER(CWeight), _i64, _vp, _vp, _vp,
                               _i64, _vp], _int),
    "q8_linear_w4a16": ([_vp, _int, _i64, _i64, _i64, ctypes.POINTER(CWeightG4), _vp, _vp, _i64,
                         _vp], _int),
    "q8_workspace_size": ([_int, _i64, _i64, _i64], _sz),
    "q8_status_string": ([_int], ctypes.c_char_p),
    "q8_get_device_status": ([_vp, _vp], _int),
    "q8_clear_device_status": ([_vp], _int),
    "q8_device_check": ([], _int),
    "q8_inject_failure": ([_int, ctypes.c_int32], _int),
    "q8_selftest_wait_timeout": ([ctypes.c_int32, _vp], _int),
    "q8_version": ([], _int),
}
for _name, (_args, _res) in _SIG.items():
    _fn = getattr(_lib, _name)
    _fn.argtypes = _args
    _fn.restype = _res


def lib():
    """The loaded ctypes library (raw C entry points)."""
    return _lib


class Q8Error(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {q8_status_string(status)} (status {status})")


def _check(status: int, where: str) -> None:
    if status != Q8_OK:
        raise Q8Error(status, where)


def q8_status_string(status: int) -> str:
    return _lib.q8_status_string(int(status)).decode()


def q8_version() -> int:
    return int(_lib.q8_version())


def q8_device_check() -> int:
    return int(_lib.q8_device_check())


def q8_inject_failure(code: int, skip: int = 0) -> None:
    """Arm a one-shot host-side failure: after `skip` more validated calls, the
    next one returns `code` (raised as Q8Error by this binding); Q8_OK disarms."""
    _check(_lib.q8_inject_failure(int(code), int(skip)), "q8_inject_failure")


def q8_workspace_size(op: int, m: int, n: int, k: int) -> int:
    return int(_lib.q8_workspace_size(op, m, n, k))


# ---------------------------------------------------------------- helpers

_FLOAT_DT = {torch.float16: Q8_F16, torch.bfloat16: Q8_BF16, torch.float32: Q8_F32}


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _cuda(t: torch.Tensor, name: str) -> torch.Tensor:
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dim() != 2 or t.stride(1) != 1:
        raise ValueError(f"{name} must be 2-D with unit column stride")
    return t


@dataclasses.dataclass
class QWeight:
    """A per-output-channel quantized weight (device tensors)."""
    codes: torch.Tensor          # n x k int8 / uint8 / float8_e4m3fn
    scale: torch.Tensor          # [n] fp32
    zero_point: Optional[torch.Tensor]  # [n] fp32 (integer-valued) or None
    code_dtype: int

    def c(self) -> CWeight:
        n, k = self.codes.shape
        return CWeight(self.codes.data_ptr(), self.code_dtype, self.scale.data_ptr(),
                       None if self.zero_point is None else self.zero_point.data_ptr(),
                       n, k, self.codes.stride(0))


@dataclasses.dataclass
class QAct:
    """A per-token quantized activation (device tensors)."""
    codes: torch.Tensor          # m x k int8 / float8_e4m3fn
    scale: torch.Tensor          # [m] fp32
    rowsum: Optional[torch.Tensor]  # [m] int32 or None
    code_dtype: int

    def c(self) -> CAct:
        m, k = self.codes.shape
        return CAct(self.codes.data_ptr(), self.code_dtype, self.scale.data_ptr(),
                    None if self.rowsum is None else self.rowsum.data_ptr(), m, k,
                    self.codes.stride(0))


# ---------------------------------------------------------------- entry points

_SCHEME = {"asym": Q8_ASYM_INT8, "sym": Q8_SYM_INT8, "fp8": Q8_FP8_E4M3}
_CODES = {"s8": (Q8_S8, torch.int8), "u8": (Q8_U8, torch.uint8),
          "e4m3": (Q8_E4M3, torch.float8_e4m3fn)}


def q8_quantize_weight(W: torch.Tensor, scheme: str = "asym", codes: str = "s8",
                       stream=None) -> QWeight:
    """Per-output-channel weight quantization (see q8_quantize_weight in q8.h)."""
    _cuda(W, "W")
    n, k = W.shape
    cdt, tdt = _CODES[codes]
    q = torch.empty((n, k), dtype=tdt, device=W.device)
    S = torch.empty(n, dtype=torch.float32, device=W.device)
    Z = torch.empty(n, dtype=torch.float32, device=W.device) if scheme == "asym" else None
    _check(_lib.q8_quantize_weight(_ptr(W), _FLOAT_DT[W.dtype], n, k, W.stride(0),
                                   _SCHEME[scheme], cdt, _ptr(q), _ptr(S), _ptr(Z),
                                   _stream(stream)), "q8_quantize_weight")
    return QWeight(q, S, Z, cdt)


def q8_dequantize_weight(w: QWeight, out_dtype=torch.float32, stream=None) -> torch.Tensor:
    out = torch.empty(w.codes.shape, dtype=out_dtype, device=w.codes.device)
    cw = w.c()
    _check(_lib.q8_dequantize_weight(ctypes.byref(cw), _FLOAT_DT[out_dtype], _ptr(out),
                                     _stream(stream)), "q8_dequantize_weight")
    return out


def q8_quantize_act(X: torch.Tensor, scheme: str = "int8", clip_ub: float = 0.0,
                    out: Optional[QAct] = None, stream=None) -> QAct:
    """Dynamic per-token quantization: scheme "int8" (symmetric, row sums) or "fp8"."""
    _cuda(X, "X")
    m, k = X.shape
    if out is None:
        if scheme == "int8":
            out = QAct(torch.empty((m, k), dtype=torch.int8, device=X.device),
                       torch.empty(m, dtype=torch.float32, device=X.device),
                       torch.empty(m, dtype=torch.int32, device=X.device), Q8_S8)
        else:
            out = QAct(torch.empty((m, k), dtype=torch.float8_e4m3fn, device=X.device),
                       torch.empty(m, dtype=torch.float32, device=X.device), None, Q8_E4M3)
    _check(_lib.q8_quantize_act(_ptr(X), _FLOAT_DT[X.dtype], m, k, X.stride(0),
                                Q8_SYM_INT8 if scheme == "int8" else Q8_FP8_E4M3, float(clip_ub),
                                _ptr(out.codes), _ptr(out.scale), _ptr(out.rowsum),
                                _stream(stream)), "q8_quantize_act")
    return out


def q8_quantize_act_static(X: torch.Tensor, scale: float, out: Optional[QAct] = None,
                           stream=None) -> QAct:
    """Static INT8 quantization with a calibrated per-tensor scale (row sums included)."""
    _cuda(X, "X")
    m, k = X.shape
    if out is None:
        out = QAct(torch.empty((m, k), dtype=torch.int8, device=X.device),
                   torch.empty(m, dtype=torch.float32, device=X.device),
                   torch.empty(m, dtype=torch.int32, device=X.device), Q8_S8)
    _check(_lib.q8_quantize_act_static(_ptr(X), _FLOAT_DT[X.dtype], m, k, X.stride(0), float(scale),
                                       _ptr(out.codes), _ptr(out.scale), _ptr(out.rowsum),
                                       _stream(stream)), "q8_quantize_act_static")
    return out


def q8_quantize_act_smooth(X: torch.Tensor, mult: torch.Tensor, out: Optional[QAct] = None,
                           stream=None) -> QAct:
    """Dynamic INT8 quantization of X * mult (per-column smoothing multipliers, fp32 [k])."""
    _cuda(X, "X")
    m, k = X.shape
    if not mult.is_cuda or mult.dtype != torch.float32 or mult.shape != (k,) or not mult.is_contiguous():
        raise ValueError("mult must be a contiguous CUDA float32 tensor of shape (k,)")
    if out is None:
        out = QAct(torch.empty((m, k), dtype=torch.int8, device=X.device),
                   torch.empty(m, dtype=torch.float32, device=X.device),
                   torch.empty(m, dtype=torch.int32, device=X.device), Q8_S8)
    _check(_lib.q8_quantize_act_smooth(_ptr(X), _FLOAT_DT[X.dtype], m, k, X.stride(0), _ptr(mult),
                                       _ptr(out.codes), _ptr(out.scale), _ptr(out.rowsum),
                                       _stream(stream)), "q8_quantize_act_smooth")
    return out


def q8_outlier_quantize_act(X: torch.Tensor, threshold: float = 6.0, gather: bool = True,
                            stream=None) -> dict:
    """LLM.int8 outlier columns + regular-stream INT8 quantization."""
    _cuda(X, "X")
    m, k = X.shape
    dev = X.device
    kp = (k + 63) // 64 * 64
    r = {
        "codes": torch.empty((m, k), dtype=torch.int8, device=dev),
        "scale": torch.empty(m, dtype=torch.float32, device=dev),
        "rowsum": torch.empty(m, dtype=torch.int32, device=dev),
        "mask": torch.empty(k, dtype=torch.uint8, device=dev),
        "idx": torch.empty(k, dtype=torch.int32, device=dev),
        "count": torch.empty(1, dtype=torch.int32, device=dev),
        "x_outlier": torch.empty((m, kp), dtype=torch.float16, device=dev) if gather else None,
    }
    _check(_lib.q8_outlier_quantize_act(
        _ptr(X), _FLOAT_DT[X.dtype], m, k, X.stride(0), float(threshold), _ptr(r["codes"]),
        _ptr(r["scale"]), _ptr(r["rowsum"]), _ptr(r["mask"]), _ptr(r["idx"]), _ptr(r["count"]),
        _ptr(r["x_outlier"]), kp, _stream(stream)), "q8_outlier_quantize_act")
    return r


def q8_linear_w8a8(x: QAct, w: QWeight, bias: Optional[torch.Tensor] = None,
                   out: Optional[torch.Tensor] = None, acc_debug: Optional[torch.Tensor] = None,
                   stream=None) -> torch.Tensor:
    """W8A8 linear with the dequant epilogue; returns the bf16 M x N output."""
    m, n = x.codes.shape[0], w.codes.shape[0]
    if out is None:
        out = torch.empty((m, n), dtype=torch.bfloat16, device=x.codes.device)
    cx, cw = x.c(), w.c()
    _check(_lib.q8_linear_w8a8(ctypes.byref(cx), ctypes.byref(cw), _ptr(bias), _ptr(out),
                               out.stride(0), _ptr(acc_debug), None, 0, _stream(stream)),
           "q8_linear_w8a8")
    return out


def q8_linear_w8a8_requant(x: QAct, w: QWeight, out_scale: float, bias: Optional[torch.Tensor] = None,
                           out: Optional[torch.Tensor] = None, acc_debug: Optional[torch.Tensor] = None,
                           stream=None) -> torch.Tensor:
    """INT8 W8A8 linear with the output re-quantized to int8 codes (scale out_scale)."""
    m, n = x.codes.shape[0], w.codes.shape[0]
    if out is None:
        out = torch.empty((m, n), dtype=torch.int8, device=x.codes.device)
    cx, cw = x.c(), w.c()
    _check(_lib.q8_linear_w8a8_requant(ctypes.byref(cx), ctypes.byref(cw), _ptr(bias), float(out_scale),
                                       _ptr(out), out.stride(0), _ptr(acc_debug), _stream(stream)),
           "q8_linear_w8a8_requant")
    return out


def q8_linear_w8a8_dynamic(X: torch.Tensor, w: QWeight, scheme: str = "int8",
                           clip_ub: float = 0.0, bias: Optional[torch.Tensor] = None,
                           out: Optional[torch.Tensor] = None, act: Optional[QAct] = None,
                           acc_debug: Optional[torch.Tensor] = None, stream=None):
    """Activation quantization + W8A8 linear in one call; returns (Y, QAct)."""
    _cuda(X, "X")
    m, k = X.shape
    n = w.codes.shape[0]
    dev = X.device
    if out is None:
        out = torch.empty((m, n), dtype=torch.bfloat16, device=dev)
    if act is None:
        if scheme == "int8":
            act = QAct(torch.empty((m, k), dtype=torch.int8, device=dev),
                       torch.empty(m, dtype=torch.float32, device=dev),
                       torch.empty(m, dtype=torch.int32, device=dev), Q8_S8)
        else:
            act = QAct(torch.empty((m, k), dtype=torch.float8_e4m3fn, device=dev),
                       torch.empty(m, dtype=torch.float32, device=dev), None, Q8_E4M3)
    cw = w.c()
    _check(_lib.q8_linear_w8a8_dynamic(
        _ptr(X), _FLOAT_DT[X.dtype], m, k, X.stride(0),
        Q8_SYM_INT8 if scheme == "int8" else Q8_FP8_E4M3, float(clip_ub), ctypes.byref(cw),
        _ptr(bias), _ptr(out), out.stride(0), _ptr(act.codes), _ptr(act.scale),
        _ptr(act.rowsum), _ptr(acc_debug), _stream(stream)), "q8_linear_w8a8_dynamic")
    return out, act


def q8_linear_int8_mixed(X: torch.Tensor, w: QWeight, threshold: float = 6.0,
                         W16: Optional[torch.Tensor] = None, bias: Optional[torch.Tensor] = None,
                         out: Optional[torch.Tensor] = None,
                         workspace: Optional[torch.Tensor] = None, debug: bool = False,
                         stream=None):
    """LLM.int8 mixed-decomposition linear.  Returns Y, or (Y, debug dict) with debug=True."""
    _cuda(X, "X")
    m, k = X.shape
    n = w.codes.shape[0]
    dev = X.device
    if out is None:
        out = torch.empty((m, n), dtype=torch.bfloat16, device=dev)
    need = q8_workspace_size(Q8_OP_LINEAR_INT8_MIXED, m, n, k)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=dev)
    dbg = None
    if debug:
        dbg = {"mask": torch.empty(k, dtype=torch.uint8, device=dev),
               "count": torch.empty(1, dtype=torch.int32, device=dev),
               "acc": torch.empty((m, n), dtype=torch.int32, device=dev),
               "y16": torch.empty((m, n), dtype=torch.float32, device=dev)}
    cw = w.c()
    _check(_lib.q8_linear_int8_mixed(
        _ptr(X), _FLOAT_DT[X.dtype], m, k, X.stride(0), ctypes.byref(cw), _ptr(W16),
        float(threshold), _ptr(bias), _ptr(out), out.stride(0),
        _ptr(dbg["mask"]) if dbg else None, _ptr(dbg["count"]) if dbg else None,
        _ptr(dbg["acc"]) if dbg else None, _ptr(dbg["y16"]) if dbg else None,
        _ptr(workspace), workspace.numel(), _stream(stream)), "q8_linear_int8_mixed")
    return (out, dbg) if debug else out


@dataclasses.dataclass
class QWeightG4:
    """A group-wise 4-bit weight (device tensors): codes n x k/2 uint8 (two
    nibbles q + 8 per byte, low nibble first), scale (k/group) x n fp32."""
    codes: torch.Tensor
    scale: torch.Tensor
    group: int

    @property
    def n(self) -> int:
        return self.codes.shape[0]

    @property
    def k(self) -> int:
        return self.scale.shape[0] * self.group

    def c(self) -> CWeightG4:
        return CWeightG4(self.codes.data_ptr(), self.scale.data_ptr(), self.n, self.k,
                         self.codes.stride(0), self.group)


def q8_quantize_weight_g4(W: torch.Tensor, group: int = 128, stream=None) -> QWeightG4:
    """Group-wise symmetric 4-bit weight quantization (see q8_quantize_weight_g4 in q8.h)."""
    _cuda(W, "W")
    n, k = W.shape
    codes = torch.empty((n, k // 2), dtype=torch.uint8, device=W.device)
    scale = torch.empty((max(k // group, 1) if k % group == 0 else 1, n), dtype=torch.float32,
                        device=W.device)
    _check(_lib.q8_quantize_weight_g4(_ptr(W), _FLOAT_DT.get(W.dtype, -1), n, k, W.stride(0),
                                      int(group), _ptr(codes), codes.stride(0), _ptr(scale),
                                      _stream(stream)), "q8_quantize_weight_g4")
    return QWeightG4(codes, scale, int(group))


def q8_quantize_weight_q4k(W: torch.Tensor, stream=None):
    """GGUF Q4_K-style weights (see q8_quantize_weight_q4k in q8.h).

    Returns (QWeightG4 with group 32 and the effective scales, sub_codes
    (k/64) x n uint8, super_scale (k/256) x n fp32)."""
    _cuda(W, "W")
    n, k = W.shape
    dev = W.device
    codes = torch.empty((n, k // 2), dtype=torch.uint8, device=dev)
    scale = torch.empty((k // 32, n), dtype=torch.float32, device=dev)
    sub = torch.empty((max(k // 64, 1), n), dtype=torch.uint8, device=dev)
    sup = torch.empty((max(k // 256, 1), n), dtype=torch.float32, device=dev)
    _check(_lib.q8_quantize_weight_q4k(_ptr(W), _FLOAT_DT.get(W.dtype, -1), n, k, W.stride(0),
                                       _ptr(codes), codes.stride(0), _ptr(scale), _ptr(sub),
                                       _ptr(sup), _stream(stream)), "q8_quantize_weight_q4k")
    return QWeightG4(codes, scale, 32), sub, sup


def q8_expand_q4k_scales(sub_codes: torch.Tensor, super_scale: torch.Tensor, k: int,
                         out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """The (k/32) x n effective scales of compact Q4_K scales."""
    n = super_scale.shape[1]
    if out is None:
        out = torch.empty((k // 32, n), dtype=torch.float32, device=super_scale.device)
    _check(_lib.q8_expand_q4k_scales(_ptr(sub_codes), _ptr(super_scale), n, k, _ptr(out),
                                     _stream(stream)), "q8_expand_q4k_scales")
    return out


def q8_linear_w4a16(X: torch.Tensor, w: QWeightG4, bias: Optional[torch.Tensor] = None,
                    out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """W4A16 linear: bf16/fp16 X times the group-wise 4-bit weight; bf16 M x N output."""
    _cuda(X, "X")
    m, k = X.shape
    if out is None:
        out = torch.empty((m, w.n), dtype=torch.bfloat16, device=X.device)
    cw = w.c()
    _check(_lib.q8_linear_w4a16(_ptr(X), _FLOAT_DT.get(X.dtype, -1), m, k, X.stride(0),
                                ctypes.byref(cw), _ptr(bias), _ptr(out), out.stride(0),
                                _stream(stream)), "q8_linear_w4a16")
    return out


def q8_linear_fp8_grouped(x: QAct, w: QWeight, num_experts: int, offsets: torch.Tensor,
                          bias: Optional[torch.Tensor] = None, out: Optional[torch.Tensor] = None,
                          stream=None) -> torch.Tensor:
    """Grouped FP8 rowwise linear (mixture of experts): tokens sorted by expert,
    offsets a CUDA int32 tensor of num_experts + 1 entries; returns bf16 M x n."""
    if not offsets.is_cuda or offsets.dtype != torch.int32 or offsets.numel() != num_experts + 1:
        raise ValueError("offsets must be a CUDA int32 tensor of num_experts + 1 entries")
    m = x.codes.shape[0]
    n = w.codes.shape[0] // num_experts
    if out is None:
        out = torch.empty((m, n), dtype=torch.bfloat16, device=x.codes.device)
    cx, cw = x.c(), w.c()
    _check(_lib.q8_linear_fp8_grouped(ctypes.byref(cx), ctypes.byref(cw), int(num_experts),
                                      _ptr(offsets.contiguous()), _ptr(bias), _ptr(out),
                                      out.stride(0), _stream(stream)), "q8_linear_fp8_grouped")
    return out


def q8_get_device_status(stream=None) -> int:
    v = ctypes.c_int32(0)
    _check(_lib.q8_get_device_status(ctypes.cast(ctypes.pointer(v), ctypes.c_void_p),
                                     _stream(stream)), "q8_get_device_status")
    return int(v.value)


def q8_clear_device_status(stream=None) -> None:
    _check(_lib.q8_clear_device_status(_stream(stream)), "q8_clear_device_status")


def q8_selftest_wait_timeout(limit_us: int, stream=None) -> None:
    """Enqueue the failure-detection self-test: a kernel whose bounded barrier
    wait runs out after `limit_us` microseconds and records
    Q8_ERR_DEVICE_TIMEOUT in the device status word (q8_get_device_status)."""
    _check(_lib.q8_selftest_wait_timeout(int(limit_us), _stream(stream)),
           "q8_selftest_wait_timeout")
