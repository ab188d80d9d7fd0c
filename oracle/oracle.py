"""Python driver for the q8 CPU oracle (``q8_oracle.c``).

TEST INFRASTRUCTURE.  Only the tests, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` import this module.  The CUDA library never
does, and this module imports nothing from it.

The C file holds every arithmetic step; this driver only marshals numpy arrays
and chains the steps in the order the pages give them:

  weights (offline)  : per-row scale/zero-point, codes
  activations (call) : [outlier columns] -> per-token scale, codes, row sums
  int8 linear        : int64 dot products -> zero-point correction -> S_x -> S_w
  fp8 linear         : double dot products -> fp32 -> S_x -> S_w
  LLM.int8 merge     : fp32(y_int8 + y16), y16 from the fp16 outlier columns
  group-wise 4-bit   : per-group absmax / 7 codes; Q4_K second-level scales
  W4A16 linear       : 16-bit dequantized weight, double dot products -> fp32
  grouped FP8 (MoE)  : the FP8 linear over each expert's token rows and weight block
  output             : bf16 round-to-nearest-even of the fp32 result

All inputs are numpy arrays on the host.  16-bit float tensors are passed as
their raw uint16 bit patterns with a format tag ("f16" or "bf16").
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "q8_oracle.c")
_LIB = os.path.join(_HERE, "libq8_oracle.so")
_FMT = {"f16": 0, "bf16": 1}
_lib = None

CFLAGS = ["-O2", "-ffp-contract=off", "-fno-fast-math", "-fopenmp", "-fPIC", "-shared",
          "-Wall", "-Wextra", "-std=c11"]


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (no fast-math, no contraction)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", *CFLAGS, "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _P(t):
    return ctypes.POINTER(t)


def lib():
    global _lib
    if _lib is None:
        L = ctypes.CDLL(build())
        i64, i32, f, vp = ctypes.c_int64, ctypes.c_int, ctypes.c_float, ctypes.c_void_p
        sig = {
            "or_init": [],
            "or_max_threads": [],
            "or_set_threads": [i32],
            "or_widen16": [vp, i32, vp, i64],
            "or_widen_e4m3": [vp, vp, i64],
            "or_round16": [vp, i32, vp, i64],
            "or_round_e4m3": [vp, vp, i64],
            "or_quant_weight_asym": [vp, i64, i64, i32, vp, vp, vp],
            "or_quant_weight_sym": [vp, i64, i64, i32, vp, vp],
            "or_quant_weight_fp8": [vp, i64, i64, vp, vp],
            "or_quant_weight_group": [vp, i64, i64, i32, i64, vp, vp],
            "or_dequant_group16": [vp, vp, i64, i64, i64, i32, vp],
            "or_quant_weight_q4k": [vp, i64, i64, vp, vp, vp, vp, vp],
            "or_quant_act_int8": [vp, i64, i64, vp, vp, vp, vp],
            "or_quant_act_fp8": [vp, i64, i64, f, vp, vp],
            "or_quant_act_static": [vp, i64, i64, f, vp, vp, vp],
            "or_quant_act_smooth": [vp, i64, i64, vp, vp, vp, vp],
            "or_smooth_weight": [vp, i64, i64, vp, vp],
            "or_requant": [vp, i64, f, vp],
            "or_outlier_columns": [vp, i64, i64, f, vp, vp, vp],
            "or_gemm_int": [vp, i32, i64, vp, i32, i64, i64, vp, i64, vp, i64, vp],
            "or_epilogue_int": [vp, vp, i64, vp, i64, vp, vp, vp, vp, vp, vp],
            "or_gemm_fp8": [vp, i64, vp, i64, i64, vp, i64, vp, i64, vp, vp, vp, vp, vp],
            "or_dequant_weight_f16": [vp, i32, i64, vp, vp, vp, i64, vp, i64, vp],
            "or_dequant_weight": [vp, i32, i64, i64, i64, vp, vp, vp],
            "or_outlier_gemm": [vp, i64, vp, i64, vp, i64, vp, i64, vp, i64, vp],
            "or_merge": [vp, vp, i64, vp, i64, vp, vp],
        }
        for name, args in sig.items():
            fn = getattr(L, name)
            fn.argtypes = args
            fn.restype = ctypes.c_int if name == "or_max_threads" else None
        L.or_init()
        _lib = L
    return _lib


def _ptr(a: Optional[np.ndarray]):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return a.ctypes.data_as(ctypes.c_void_p)


def threads() -> int:
    return int(lib().or_max_threads())


def set_threads(n: int) -> None:
    lib().or_set_threads(int(n))


# ---------------------------------------------------------------- formats

def widen16(bits: np.ndarray, fmt: str) -> np.ndarray:
    b = np.ascontiguousarray(bits, dtype=np.uint16)
    out = np.empty(b.shape, np.float32)
    lib().or_widen16(_ptr(b), _FMT[fmt], _ptr(out), b.size)
    return out


def widen_e4m3(codes: np.ndarray) -> np.ndarray:
    c = np.ascontiguousarray(codes, dtype=np.uint8)
    out = np.empty(c.shape, np.float32)
    lib().or_widen_e4m3(_ptr(c), _ptr(out), c.size)
    return out


def round16(x: np.ndarray, fmt: str) -> np.ndarray:
    a = np.ascontiguousarray(x, dtype=np.float32)
    out = np.empty(a.shape, np.uint16)
    lib().or_round16(_ptr(a), _FMT[fmt], _ptr(out), a.size)
    return out


def round_e4m3(x: np.ndarray) -> np.ndarray:
    a = np.ascontiguousarray(x, dtype=np.float32)
    out = np.empty(a.shape, np.uint8)
    lib().or_round_e4m3(_ptr(a), _ptr(out), a.size)
    return out


# ---------------------------------------------------------------- weights

def quant_weight(w: np.ndarray, scheme: str, codes: str = "s8", bits: int = 8):
    """Quantize an N x K fp32 weight (values exact in its 16-bit dtype).

    scheme "asym": returns (q, S, Z) with int8 codes and Z in [-128, 127];
        codes "u8" stores q + 128 as uint8 and Z + 128 as its zero point.
    scheme "sym" : returns (q, S, None), q in [-qmax, qmax].
    scheme "fp8" : returns (q e4m3 codes uint8, S, None).
    """
    w = np.ascontiguousarray(w, dtype=np.float32)
    n, k = w.shape
    S = np.empty(n, np.float32)
    L = lib()
    if scheme == "asym":
        q = np.empty((n, k), np.int8)
        Z = np.empty(n, np.float32)
        L.or_quant_weight_asym(_ptr(w), n, k, bits, _ptr(q), _ptr(S), _ptr(Z))
        if codes == "u8":
            assert bits == 8
            return (q.astype(np.int16) + 128).astype(np.uint8), S, (Z + 128.0).astype(np.float32)
        return q, S, Z
    if scheme == "sym":
        q = np.empty((n, k), np.int8)
        L.or_quant_weight_sym(_ptr(w), n, k, bits, _ptr(q), _ptr(S))
        return q, S, None
    if scheme == "fp8":
        q = np.empty((n, k), np.uint8)
        L.or_quant_weight_fp8(_ptr(w), n, k, _ptr(q), _ptr(S))
        return q, S, None
    raise ValueError(scheme)


def quant_weight_group(w: np.ndarray, g: int, bits: int = 4):
    """Group-wise symmetric weights: every g consecutive values of a row share
    one absmax scale.  Returns (q int8 N x K in [-qmax, qmax], S N x K/g)."""
    w = np.ascontiguousarray(w, dtype=np.float32)
    n, k = w.shape
    assert k % g == 0
    q = np.empty((n, k), np.int8)
    S = np.empty((n, k // g), np.float32)
    lib().or_quant_weight_group(_ptr(w), n, k, bits, g, _ptr(q), _ptr(S))
    return q, S


def quant_weight_q4k(w: np.ndarray):
    """Q4_K two-level scales over super blocks of 8 x 32 weights.

    Returns a dict: q (int8 N x K), s_sub, q_sub, S_eff (N x K/32) and
    s_super (N x K/256).  S_eff is the per-32 scale the weight is dequantized
    with (dequant_group16 / linear_w4a16 with g = 32)."""
    w = np.ascontiguousarray(w, dtype=np.float32)
    n, k = w.shape
    assert k % 256 == 0
    out = {"q": np.empty((n, k), np.int8), "s_sub": np.empty((n, k // 32), np.float32),
           "s_super": np.empty((n, k // 256), np.float32),
           "q_sub": np.empty((n, k // 32), np.uint8), "S_eff": np.empty((n, k // 32), np.float32)}
    lib().or_quant_weight_q4k(_ptr(w), n, k, _ptr(out["q"]), _ptr(out["s_sub"]),
                              _ptr(out["s_super"]), _ptr(out["q_sub"]), _ptr(out["S_eff"]))
    return out


def dequant_group16(q: np.ndarray, S: np.ndarray, g: int, fmt: str) -> np.ndarray:
    """16-bit bits of fl32(S[n, k/g] * q[n, k]) rounded to fmt ("f16"/"bf16")."""
    q = np.ascontiguousarray(q, dtype=np.int8)
    S = np.ascontiguousarray(S, dtype=np.float32)
    n, k = q.shape
    out = np.empty((n, k), np.uint16)
    lib().or_dequant_group16(_ptr(q), _ptr(S), n, k, g, _FMT[fmt], _ptr(out))
    return out


def linear_w4a16(x: np.ndarray, q: np.ndarray, S: np.ndarray, g: int, fmt: str,
                 bias=None, rows=None, cols=None):
    """Group-quantized weight times 16-bit activations.

    x: M x K fp32 holding fmt values.  The weight is dequantized to fmt
    (dequant_group16), the products are summed in double and rounded once to
    fp32, then y = fl32(y + bias[n]); Y = bf16_rne(y).  Returns (y, Y)."""
    k = q.shape[1]
    w16 = widen16(dequant_group16(q, S, g, fmt), fmt)
    c = _index(cols, q.shape[0])
    y = outlier_gemm(x, w16, np.arange(k, dtype=np.int32), rows, c)
    if bias is not None:
        y = (y + np.asarray(bias, np.float32)[c][None, :]).astype(np.float32)
    return y, round16(y, "bf16")


# ---------------------------------------------------------------- activations

def quant_act_int8(x: np.ndarray, skip: Optional[np.ndarray] = None):
    x = np.ascontiguousarray(x, dtype=np.float32)
    m, k = x.shape
    q = np.empty((m, k), np.int8)
    S = np.empty(m, np.float32)
    rs = np.empty(m, np.int32)
    sk = None if skip is None else np.ascontiguousarray(skip, dtype=np.uint8)
    lib().or_quant_act_int8(_ptr(x), m, k, _ptr(sk), _ptr(q), _ptr(S), _ptr(rs))
    return q, S, rs


def quant_act_static(x: np.ndarray, S: float):
    """Static per-tensor symmetric INT8: (codes, per-row scale copies, row sums)."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    m, k = x.shape
    q = np.empty((m, k), np.int8)
    Sr = np.empty(m, np.float32)
    rs = np.empty(m, np.int32)
    lib().or_quant_act_static(_ptr(x), m, k, float(np.float32(S)), _ptr(q), _ptr(Sr), _ptr(rs))
    return q, Sr, rs


def quant_act_smooth(x: np.ndarray, mult: np.ndarray):
    """Dynamic INT8 quantization of fl32(x * mult[col]): (codes, scales, row sums)."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    m, k = x.shape
    mu = np.ascontiguousarray(mult, dtype=np.float32)
    assert mu.shape == (k,)
    q = np.empty((m, k), np.int8)
    S = np.empty(m, np.float32)
    rs = np.empty(m, np.int32)
    lib().or_quant_act_smooth(_ptr(x), m, k, _ptr(mu), _ptr(q), _ptr(S), _ptr(rs))
    return q, S, rs


def smooth_weight(w: np.ndarray, s: np.ndarray) -> np.ndarray:
    """fl32(w * s[col]): the weight side of the smoothing (offline)."""
    w = np.ascontiguousarray(w, dtype=np.float32)
    n, k = w.shape
    out = np.empty((n, k), np.float32)
    lib().or_smooth_weight(_ptr(w), n, k, _ptr(np.ascontiguousarray(s, dtype=np.float32)), _ptr(out))
    return out


def requant(y: np.ndarray, S: float) -> np.ndarray:
    """INT8 codes of a layer's fp32 output with the next layer's input scale."""
    y = np.ascontiguousarray(y, dtype=np.float32)
    q = np.empty(y.shape, np.int8)
    lib().or_requant(_ptr(y), y.size, float(np.float32(S)), _ptr(q))
    return q


def quant_act_fp8(x: np.ndarray, ub: float):
    x = np.ascontiguousarray(x, dtype=np.float32)
    m, k = x.shape
    q = np.empty((m, k), np.uint8)
    S = np.empty(m, np.float32)
    lib().or_quant_act_fp8(_ptr(x), m, k, float(ub), _ptr(q), _ptr(S))
    return q, S


def outlier_columns(x: np.ndarray, threshold: float):
    x = np.ascontiguousarray(x, dtype=np.float32)
    m, k = x.shape
    mask = np.empty(k, np.uint8)
    idx = np.empty(max(k, 1), np.int32)
    cnt = ctypes.c_int32(0)
    lib().or_outlier_columns(_ptr(x), m, k, float(threshold), _ptr(mask), _ptr(idx),
                             ctypes.cast(ctypes.pointer(cnt), ctypes.c_void_p))
    return mask, idx[: cnt.value].copy(), int(cnt.value)


# ---------------------------------------------------------------- GEMMs

def _index(sel, size):
    if sel is None:
        return np.arange(size, dtype=np.int64)
    return np.ascontiguousarray(sel, dtype=np.int64)


def gemm_int(a: np.ndarray, b: np.ndarray, rows=None, cols=None) -> np.ndarray:
    """int64 sum_k a[m, k] * b[n, k] over the selected rows/cols (int8/uint8 codes)."""
    a = np.ascontiguousarray(a)
    b = np.ascontiguousarray(b)
    assert a.dtype in (np.int8, np.uint8) and b.dtype in (np.int8, np.uint8)
    r = _index(rows, a.shape[0])
    c = _index(cols, b.shape[0])
    acc = np.empty((r.size, c.size), np.int64)
    lib().or_gemm_int(_ptr(a), int(a.dtype == np.int8), a.shape[1], _ptr(b),
                      int(b.dtype == np.int8), b.shape[1], a.shape[1], _ptr(r), r.size,
                      _ptr(c), c.size, _ptr(acc))
    return acc


def epilogue_int(acc, rows, cols, Zw, rowsum, Sx, Sw, bias=None):
    r = _index(rows, acc.shape[0])
    c = _index(cols, acc.shape[1])
    y = np.empty((r.size, c.size), np.float32)
    f32 = lambda v: None if v is None else np.ascontiguousarray(v, dtype=np.float32)
    lib().or_epilogue_int(_ptr(np.ascontiguousarray(acc, dtype=np.int64)), _ptr(r), r.size,
                          _ptr(c), c.size, _ptr(f32(Zw)),
                          _ptr(np.ascontiguousarray(rowsum, dtype=np.int32)),
                          _ptr(f32(Sx)), _ptr(f32(Sw)), _ptr(f32(bias)), _ptr(y))
    return y


INT32_MAX = 2**31 - 1


def linear_w8a8_int8(xq, Sx, rowsum, wq, Sw, Zw=None, bias=None, rows=None, cols=None):
    """INT8 W8A8 linear over the selected outputs.

    Returns (acc int64, y fp32, Y bf16 bits).  acc is asserted to fit in int32,
    the accumulator width the pages name.
    """
    acc = gemm_int(xq, wq, rows, cols)
    assert np.abs(acc).max(initial=0) <= INT32_MAX, "INT32 accumulator bound exceeded"
    r = _index(rows, xq.shape[0])
    c = _index(cols, wq.shape[0])
    y = epilogue_int(acc, r, c, Zw, rowsum, Sx, Sw, bias)
    return acc, y, round16(y, "bf16")


def linear_w8a8_fp8(xq, Sx, wq, Sw, bias=None, rows=None, cols=None):
    """FP8 rowwise linear.  Returns (acc fp32, y fp32, Y bf16 bits)."""
    xq = np.ascontiguousarray(xq, dtype=np.uint8)
    wq = np.ascontiguousarray(wq, dtype=np.uint8)
    r = _index(rows, xq.shape[0])
    c = _index(cols, wq.shape[0])
    acc = np.empty((r.size, c.size), np.float32)
    y = np.empty((r.size, c.size), np.float32)
    f32 = lambda v: None if v is None else np.ascontiguousarray(v, dtype=np.float32)
    lib().or_gemm_fp8(_ptr(xq), xq.shape[1], _ptr(wq), wq.shape[1], xq.shape[1], _ptr(r),
                      r.size, _ptr(c), c.size, _ptr(f32(Sx)), _ptr(f32(Sw)),
                      _ptr(f32(bias)), _ptr(acc), _ptr(y))
    return acc, y, round16(y, "bf16")


def linear_moe_fp8(xq, Sx, wq, Sw, offsets, n: int, bias=None, rows=None):
    """Grouped FP8 rowwise linear of a mixture-of-experts layer.

    [FBGEMM] 5.4 (Llama4 experts): the experts' weights sit in one tensor, one
    FP8 block with per-row scales per expert, and each expert's tokens are
    quantized and multiplied with f8f8bf16_rowwise on their own.  Tokens are
    sorted by expert: rows offsets[e] .. offsets[e+1]-1 of xq use expert e,
    whose weight is rows e*n .. e*n+n-1 of the stacked wq (scales Sw, bias
    stacked the same way).  Each block is linear_w8a8_fp8.  Returns
    (y fp32 len(rows) x n, Y bf16 bits)."""
    off = [int(v) for v in offsets]
    m = np.asarray(xq).shape[0]
    r_all = _index(rows, m)
    y = np.zeros((r_all.size, n), np.float32)
    for e in range(len(off) - 1):
        sel = np.nonzero((r_all >= off[e]) & (r_all < off[e + 1]))[0]
        if sel.size == 0:
            continue
        _, ye, _ = linear_w8a8_fp8(xq, Sx, wq, Sw, bias, rows=r_all[sel],
                                   cols=np.arange(e * n, (e + 1) * n))
        y[sel] = ye
    return y, round16(y, "bf16")


def dequant_weight_f16(wq, Sw, Zw, colidx, rows=None) -> np.ndarray:
    """fp16 bits of S (q - Z) for the given weight columns (nr x ncols)."""
    wq = np.ascontiguousarray(wq)
    r = _index(rows, wq.shape[0])
    ci = np.ascontiguousarray(colidx, dtype=np.int32)
    out = np.empty((r.size, ci.size), np.uint16)
    f32 = lambda v: None if v is None else np.ascontiguousarray(v, dtype=np.float32)
    lib().or_dequant_weight_f16(_ptr(wq), int(wq.dtype == np.int8), wq.shape[1],
                                _ptr(f32(Sw)), _ptr(f32(Zw)), _ptr(r), r.size, _ptr(ci),
                                ci.size, _ptr(out))
    return out


def dequant_weight_codes(wq, kind: str, Sw, Zw=None) -> np.ndarray:
    """fp32 S (q - Z) for every element.  kind: "s8", "u8" or "e4m3"."""
    wq = np.ascontiguousarray(wq)
    n, k = wq.shape
    out = np.empty((n, k), np.float32)
    f32 = lambda v: None if v is None else np.ascontiguousarray(v, dtype=np.float32)
    lib().or_dequant_weight(_ptr(wq), {"s8": 0, "u8": 1, "e4m3": 2}[kind], n, k, wq.shape[1],
                            _ptr(f32(Sw)), _ptr(f32(Zw)), _ptr(out))
    return out


def outlier_gemm(x: np.ndarray, w16_cols: np.ndarray, idx, rows=None, cols=None):
    """fp32(sum_j x[m, idx[j]] * w16_cols[n, j]) with double accumulation.

    x: M x K fp32 (fp16 values); w16_cols: N x count fp32 (fp16 values)."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    w = np.ascontiguousarray(w16_cols, dtype=np.float32)
    ix = np.ascontiguousarray(idx, dtype=np.int32)
    r = _index(rows, x.shape[0])
    c = _index(cols, w.shape[0])
    y = np.empty((r.size, c.size), np.float32)
    lib().or_outlier_gemm(_ptr(x), x.shape[1], _ptr(w) if w.size else None,
                          max(w.shape[1], 1), _ptr(ix) if ix.size else None, ix.size, _ptr(r),
                          r.size, _ptr(c), c.size, _ptr(y))
    return y


def merge(y_int8, y16, cols, bias=None):
    a = np.ascontiguousarray(y_int8, dtype=np.float32)
    b = np.ascontiguousarray(y16, dtype=np.float32)
    c = np.ascontiguousarray(cols, dtype=np.int64)
    y = np.empty(a.shape, np.float32)
    f32 = lambda v: None if v is None else np.ascontiguousarray(v, dtype=np.float32)
    lib().or_merge(_ptr(a), _ptr(b), a.shape[0], _ptr(c), a.shape[1], _ptr(f32(bias)), _ptr(y))
    return y


def linear_int8_mixed(x: np.ndarray, wq, Sw, Zw, threshold: float, w16_full=None,
                      bias=None, rows=None, cols=None):
    """LLM.int8 mixed decomposition over the selected outputs.

    x: M x K fp32 holding fp16 values.  wq: N x K int8/uint8 codes with per-row
    S/Z.  w16_full: the original N x K fp16 weight as fp32 values
    (llm_int8_has_fp16_weight), else the outlier columns are dequantized to fp16.
    Returns a dict with every intermediate the GPU path exposes.
    """
    m, k = x.shape
    mask, idx, count = outlier_columns(x, threshold)
    xq, Sx, rowsum = quant_act_int8(x, skip=mask)
    r = _index(rows, m)
    c = _index(cols, wq.shape[0])
    acc, y_int8, _ = linear_w8a8_int8(xq, Sx, rowsum, wq, Sw, Zw, None, r, c)
    if w16_full is not None:
        w16 = np.ascontiguousarray(np.asarray(w16_full, np.float32)[:, idx])
    else:
        w16 = widen16(dequant_weight_f16(wq, Sw, Zw, idx), "f16")
    y16 = outlier_gemm(x, w16, idx, r, c)
    y = merge(y_int8, y16, c, bias)
    return {"mask": mask, "idx": idx, "count": count, "xq": xq, "Sx": Sx, "rowsum": rowsum,
            "acc": acc, "y_int8": y_int8, "w16": w16, "y16": y16, "y": y,
            "Y": round16(y, "bf16")}
