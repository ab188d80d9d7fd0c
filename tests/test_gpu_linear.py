"""GPU parity of the W8A8 and LLM.int8 linears against the CPU oracle.

INT8 accumulators and INT8 W8A8 outputs are compared bit for bit; FP8 and
mixed outputs under the 2-ulp contract of tests/parity.py (check_fp_output,
which prints the largest error in ulps).  The workloads are compared in full
at their own sizes, in the launch configuration the benchmark uses; smaller
shapes span several tiles, ragged tails and the decode path.
"""
import numpy as np
import pytest
import torch

import workloads
from oracle import oracle as O
from tests import parity as P

pytestmark = pytest.mark.gpu

from bit_quantized_b200 import q8  # noqa: E402

DEV = "cuda:0"


def _int8_case(x32, w32, scheme, codes, X_dev, W_dev, bias=None, rows=None, cols=None,
               what=""):
    """Runs quantize + linear on the GPU and checks codes, acc and Y against the oracle."""
    qa = q8.q8_quantize_act(X_dev, "int8")
    qw = q8.q8_quantize_weight(W_dev, scheme, codes)
    m, n = X_dev.shape[0], W_dev.shape[0]
    acc = torch.empty((m, n), dtype=torch.int32, device=DEV)
    b_dev = None if bias is None else torch.from_numpy(bias).to(DEV)
    Y = q8.q8_linear_w8a8(qa, qw, bias=b_dev, acc_debug=acc)
    torch.cuda.synchronize()
    xq, Sx, rs = O.quant_act_int8(x32)
    wq, Sw, Zw = O.quant_weight(w32, scheme, codes)
    r = np.arange(m) if rows is None else rows
    c = np.arange(n) if cols is None else cols
    acc_ref, y_ref, Y_ref = O.linear_w8a8_int8(xq, Sx, rs, wq, Sw, Zw, bias, r, c)
    P.assert_equal(acc.cpu().numpy()[np.ix_(r, c)], acc_ref.astype(np.int32), what + " acc")
    Yb = P.bf16_bits(Y)[np.ix_(r, c)]
    P.assert_equal(Yb, Y_ref, what + " Y")
    P.assert_bf16_within(Yb, y_ref, 0.0, what)


def _rand(m, k, dtype, seed, std=1.0):
    X = workloads.random_matrix(m, k, dtype, seed, std)
    return X, P.host_f32(X)


# ------------------------------------------------------------------ INT8 W8A8, full size

def test_decode_q_proj_full():
    X, W, info, x32, w32 = P.workload("decode_q_proj")
    _int8_case(x32, w32, "asym", "u8", X.to(DEV), W.to(DEV), what="decode_q_proj")


@pytest.mark.slow
def test_prefill_ffn_up_full():
    # every output of the 2048 x 14336 x 4096 workload (the oracle's int64 GEMM
    # takes seconds on the host cores)
    X, W, info, x32, w32 = P.workload("prefill_ffn_up")
    _int8_case(x32, w32, "sym", "s8", X.to(DEV), W.to(DEV), what="prefill_ffn_up")


# ------------------------------------------------------------------ INT8 W8A8, shapes

@pytest.mark.parametrize("m,n,k", [
    (1, 128, 256),          # single token, decode kernel
    (16, 4096, 4096),       # decode shape, s8 weights
    (17, 272, 160),         # decode kernel NT=32, N % 32 == 16, ragged K block
    (64, 512, 1024),        # decode kernel NT=64
    (65, 384, 512),         # tile kernel, one partial M tile
    (300, 640, 1024),       # tile kernel, several tiles, ragged M
    (384, 2304, 384),       # tile kernel BN=256 path (tiles >= SMs)
    (130, 48, 32),          # K = 32: one K block mostly out of bounds; N = 48
    (512, 8288, 256),       # tile kernel BN=224 path (37 x 224-wide tiles, ragged N)
])
@pytest.mark.parametrize("scheme,codes", [("asym", "s8"), ("asym", "u8"), ("sym", "s8")])
def test_int8_shapes(m, n, k, scheme, codes):
    X, x32 = _rand(m, k, torch.bfloat16, seed=m + n + k)
    W, w32 = _rand(n, k, torch.bfloat16, seed=m * n + k, std=0.02)
    _int8_case(x32, w32, scheme, codes, X.to(DEV), W.to(DEV), what=f"{m}x{n}x{k} {scheme}/{codes}")


@pytest.mark.parametrize("m", [8, 256])
def test_int8_bias(m):
    X, x32 = _rand(m, 512, torch.bfloat16, seed=41)
    W, w32 = _rand(320, 512, torch.bfloat16, seed=42, std=0.02)
    bias = np.linspace(-3, 3, 320).astype(np.float32)
    _int8_case(x32, w32, "asym", "s8", X.to(DEV), W.to(DEV), bias=bias, what=f"bias m={m}")


def test_int8_empty_m():
    W = workloads.random_matrix(64, 64, torch.bfloat16, 1, 0.02).to(DEV)
    qw = q8.q8_quantize_weight(W, "asym", "s8")
    qa = q8.q8_quantize_act(torch.empty((0, 64), dtype=torch.bfloat16, device=DEV), "int8")
    Y = q8.q8_linear_w8a8(qa, qw)
    torch.cuda.synchronize()
    assert Y.shape == (0, 64)


def test_int8_strided_output():
    X, x32 = _rand(20, 256, torch.bfloat16, seed=43)
    W, w32 = _rand(64, 256, torch.bfloat16, seed=44, std=0.02)
    qa = q8.q8_quantize_act(X.to(DEV), "int8")
    qw = q8.q8_quantize_weight(W.to(DEV), "sym", "s8")
    big = torch.full((20, 96), 7.0, dtype=torch.bfloat16, device=DEV)
    q8.q8_linear_w8a8(qa, qw, out=big[:, 16:80])
    torch.cuda.synchronize()
    xq, Sx, rs = O.quant_act_int8(x32)
    wq, Sw, _ = O.quant_weight(w32, "sym")
    _, _, Y_ref = O.linear_w8a8_int8(xq, Sx, rs, wq, Sw)
    P.assert_equal(P.bf16_bits(big[:, 16:80]), Y_ref, "strided Y")
    assert (big[:, :16] == 7).all() and (big[:, 80:] == 7).all(), "write outside the output view"


# ------------------------------------------------------------------ FP8

def _fp8_case(x32, w32, X_dev, W_dev, ub, bias=None, rows=None, cols=None, what=""):
    qa = q8.q8_quantize_act(X_dev, "fp8", clip_ub=ub)
    qw = q8.q8_quantize_weight(W_dev, "fp8", "e4m3")
    m, n = X_dev.shape[0], W_dev.shape[0]
    b_dev = None if bias is None else torch.from_numpy(bias).to(DEV)
    acc = torch.empty((m, n), dtype=torch.float32, device=DEV)
    Y = q8.q8_linear_w8a8(qa, qw, bias=b_dev, acc_debug=acc)
    torch.cuda.synchronize()
    xq, Sx = O.quant_act_fp8(x32, ub)
    wq, Sw, _ = O.quant_weight(w32, "fp8")
    r = np.arange(m) if rows is None else rows
    c = np.arange(n) if cols is None else cols
    acc_ref, y_ref, _ = O.linear_w8a8_fp8(xq, Sx, wq, Sw, bias, r, c)
    a_abs = np.abs(O.widen_e4m3(xq[r])).astype(np.float64)
    b_abs = np.abs(O.widen_e4m3(wq[c])).astype(np.float64)
    mag = a_abs @ b_abs.T
    k = x32.shape[1]
    P.check_fp_acc(acc.cpu().numpy()[np.ix_(r, c)], acc_ref, mag, k, 32, what + " acc")
    term = (P.accumulation_bound(mag, k, 32) * Sx[r][:, None].astype(np.float64)
            * Sw[c][None, :].astype(np.float64))
    return P.check_fp_output(P.bf16_bits(Y)[np.ix_(r, c)], y_ref, term, what)


@pytest.mark.slow
def test_fp8_rowwise_full():
    # every output of the 4096 x 8192 x 8192 workload
    X, W, info, x32, w32 = P.workload("fp8_rowwise")
    _fp8_case(x32, w32, X.to(DEV), W.to(DEV), 1200.0, what="fp8_rowwise")


@pytest.mark.parametrize("m,n,k", [(5, 256, 512), (16, 1024, 2048), (200, 528, 1024),
                                   (256, 2560, 512)])
def test_fp8_shapes(m, n, k):
    X, x32 = _rand(m, k, torch.bfloat16, seed=m + 7 * k)
    X[0, 0] = 3000.0                        # beyond the upper bound: saturates
    x32 = P.host_f32(X)
    W, w32 = _rand(n, k, torch.bfloat16, seed=n + k, std=0.02)
    bias = np.linspace(-1, 1, n).astype(np.float32)
    _fp8_case(x32, w32, X.to(DEV), W.to(DEV), 1200.0, bias=bias, what=f"fp8 {m}x{n}x{k}")


# ------------------------------------------------------------------ LLM.int8 mixed

def _mixed_case(X, W, threshold, codes="s8", has_fp16_weight=False, bias=None, rows=None,
                cols=None, what=""):
    x32, w32 = P.host_f32(X), P.host_f32(W)
    Wd = W.to(DEV)
    qw = q8.q8_quantize_weight(Wd, "asym", codes)
    b_dev = None if bias is None else torch.from_numpy(bias).to(DEV)
    Y, dbg = q8.q8_linear_int8_mixed(X.to(DEV), qw, threshold,
                                     W16=Wd if has_fp16_weight else None, bias=b_dev, debug=True)
    torch.cuda.synchronize()
    wq, Sw, Zw = O.quant_weight(w32, "asym", codes)
    m, n = X.shape[0], W.shape[0]
    r = np.arange(m) if rows is None else rows
    c = np.arange(n) if cols is None else cols
    ref = O.linear_int8_mixed(x32, wq, Sw, Zw, threshold, w16_full=w32 if has_fp16_weight else None,
                              bias=bias, rows=r, cols=c)
    P.assert_equal(dbg["mask"].cpu().numpy(), ref["mask"], what + " mask")
    assert int(dbg["count"].item()) == ref["count"], what + " count"
    P.assert_equal(dbg["acc"].cpu().numpy()[np.ix_(r, c)], ref["acc"].astype(np.int32), what + " acc")
    # outlier stream: fp32 accumulation of fp16 products over count columns
    # (kind::f16, 16 products per MMA instruction)
    y16 = dbg["y16"].cpu().numpy()[np.ix_(r, c)].astype(np.float64)
    mag16 = np.abs(x32[np.ix_(r, ref["idx"])]).astype(np.float64) @ np.abs(ref["w16"][c]).T.astype(np.float64)
    P.check_fp_acc(y16, ref["y16"], mag16, max(ref["count"], 1), 16, what + " y16")
    if ref["count"] > 0:
        fro = np.linalg.norm(y16 - ref["y16"]) / max(np.linalg.norm(ref["y16"]), 1e-30)
        assert fro <= 1e-3, what + f" y16 relative Frobenius {fro}"
    term = P.accumulation_bound(mag16, max(ref["count"], 1), 16)
    stats = P.check_fp_output(P.bf16_bits(Y)[np.ix_(r, c)], ref["y"], term, what)
    return stats, ref["count"]


def test_tiny_mixed_full():
    X, W, info, x32, w32 = P.workload("tiny_mixed")
    _, count = _mixed_case(X, W, 6.0, what="tiny_mixed")
    assert count == 2


def test_mixed_512_full():
    X, W, info, x32, w32 = P.workload("mixed_512")
    _mixed_case(X, W, 6.0, what="mixed_512")


@pytest.mark.parametrize("threshold", [0.0, float("inf"), 1e-30, 2.5])
def test_mixed_thresholds(threshold):
    X = workloads.random_matrix(40, 320, torch.float16, seed=51)
    X[:, 17] *= 20
    W = workloads.random_matrix(96, 320, torch.float16, seed=52, std=0.02)
    _mixed_case(X, W, threshold, what=f"T={threshold}")


def test_mixed_off_equals_w8a8_bit_exact():
    X = workloads.random_matrix(48, 256, torch.float16, seed=53)
    X[:, 9] *= 15
    W = workloads.random_matrix(128, 256, torch.float16, seed=54, std=0.02)
    Wd = W.to(DEV)
    qw = q8.q8_quantize_weight(Wd, "asym", "s8")
    Ym = q8.q8_linear_int8_mixed(X.to(DEV), qw, 0.0)
    Yp = q8.q8_linear_w8a8(q8.q8_quantize_act(X.to(DEV), "int8"), qw)
    torch.cuda.synchronize()
    P.assert_equal(P.bf16_bits(Ym), P.bf16_bits(Yp), "threshold 0 vs W8A8")


@pytest.mark.parametrize("codes,fp16w", [("u8", False), ("s8", True)])
def test_mixed_variants(codes, fp16w):
    X = workloads.random_matrix(130, 512, torch.float16, seed=55)
    X[:, [1, 300, 301]] *= 12
    W = workloads.random_matrix(272, 512, torch.float16, seed=56, std=0.02)
    bias = np.linspace(-1, 1, 272).astype(np.float32)
    _mixed_case(X, W, 6.0, codes=codes, has_fp16_weight=fp16w, bias=bias,
                what=f"mixed {codes} fp16w={fp16w}")


def test_mixed_many_outliers():
    # 100 outlier columns: two fp16 K blocks of 64 in the outlier GEMM
    X = workloads.random_matrix(64, 1024, torch.float16, seed=57)
    X[:, ::10] *= 10
    W = workloads.random_matrix(128, 1024, torch.float16, seed=58, std=0.02)
    _, count = _mixed_case(X, W, 6.0, what="many outliers")
    assert count > 64


def test_mixed_more_tiles_than_sms():
    # 1152 x 2560: 9 x 20 = 180 tiles of 128 x 128, more than one wave of the
    # persistent grid (148 CTAs), so CTAs run two tiles with both TMEM buffers.
    X = workloads.random_matrix(1152, 512, torch.float16, seed=59)
    X[:, [5, 77, 300]] *= 14
    W = workloads.random_matrix(2560, 512, torch.float16, seed=60, std=0.02)
    rows = P.sample_indices(1152, 256, 3)
    cols = P.sample_indices(2560, 512, 4)
    _mixed_case(X, W, 6.0, rows=rows, cols=cols, what="mixed 1152x2560")


def test_device_status_clean():
    assert q8.q8_get_device_status() == 0


# ------------------------------------------------------------------ one-call activation quant + linear

def _dynamic_vs_two_step(X, W, scheme, codes, wscheme, ub=0.0, bias=None, what=""):
    Xd, Wd = X.to(DEV), W.to(DEV)
    qw = q8.q8_quantize_weight(Wd, wscheme, codes)
    m, n = X.shape[0], W.shape[0]
    b = None if bias is None else torch.from_numpy(bias).to(DEV)
    acc_dt = torch.float32 if scheme == "fp8" else torch.int32
    acc1 = torch.empty((m, n), dtype=acc_dt, device=DEV)
    acc2 = torch.empty((m, n), dtype=acc_dt, device=DEV)
    Y1, act = q8.q8_linear_w8a8_dynamic(Xd, qw, scheme, clip_ub=ub, bias=b, acc_debug=acc1)
    qa = q8.q8_quantize_act(Xd, scheme, clip_ub=ub)
    Y2 = q8.q8_linear_w8a8(qa, qw, bias=b, acc_debug=acc2)
    torch.cuda.synchronize()
    P.assert_equal(P.codes_u8(act.codes), P.codes_u8(qa.codes), what + " codes")
    P.assert_equal(act.scale.cpu().numpy().view(np.uint32), qa.scale.cpu().numpy().view(np.uint32),
                   what + " scale")
    if scheme == "int8":
        P.assert_equal(act.rowsum.cpu().numpy(), qa.rowsum.cpu().numpy(), what + " rowsum")
        P.assert_equal(acc1.cpu().numpy(), acc2.cpu().numpy(), what + " acc")
        P.assert_equal(P.bf16_bits(Y1), P.bf16_bits(Y2), what + " Y")
    else:
        # the same kernels on the same codes: identical accumulators and outputs
        P.assert_equal(acc1.cpu().numpy().view(np.uint32), acc2.cpu().numpy().view(np.uint32),
                       what + " acc")
        P.assert_equal(P.bf16_bits(Y1), P.bf16_bits(Y2), what + " Y")
    return Y1, qw, act


@pytest.mark.parametrize("m,n,k,dtype", [
    (16, 4096, 4096, torch.bfloat16),   # decode workload shape
    (1, 128, 256, torch.float16),
    (17, 272, 160, torch.bfloat16),     # NT=32, ragged last K block
    (33, 512, 1024, torch.float16),     # NT=64
    (64, 384, 4096, torch.bfloat16),
    (65, 256, 256, torch.bfloat16),     # tile kernel
    (8, 256, 512, torch.float32),       # fp32 input
    (3, 208, 160, torch.bfloat16),      # ragged N and last K block
    (12, 1008, 3008, torch.float16),    # fp16, 12 token rows
])
@pytest.mark.parametrize("codes,wscheme", [("u8", "asym"), ("s8", "sym")])
def test_dynamic_int8_matches_two_step(m, n, k, dtype, codes, wscheme):
    X = workloads.random_matrix(m, k, dtype, seed=m * 7 + k)
    W = workloads.random_matrix(n, k, dtype, seed=n + 3 * k, std=0.02)
    bias = np.linspace(-1, 1, n).astype(np.float32) if m % 2 else None
    _dynamic_vs_two_step(X, W, "int8", codes, wscheme, bias=bias, what=f"dyn {m}x{n}x{k} {codes}")


@pytest.mark.parametrize("m,n,k", [(16, 1024, 2048), (5, 256, 512), (40, 512, 1024)])
def test_dynamic_fp8_matches_two_step(m, n, k):
    X = workloads.random_matrix(m, k, torch.bfloat16, seed=m + k) * 3
    X[0, 1] = 5000.0                         # beyond the upper bound
    W = workloads.random_matrix(n, k, torch.bfloat16, seed=n + k, std=0.02)
    _dynamic_vs_two_step(X, W, "fp8", "e4m3", "fp8", ub=1200.0, what=f"dyn fp8 {m}x{n}x{k}")


def test_dynamic_decode_workload_against_oracle():
    X, W, info, x32, w32 = P.workload("decode_q_proj")
    Y, qw, act = _dynamic_vs_two_step(X, W, "int8", "u8", "asym", what="decode workload")
    xq, Sx, rs = O.quant_act_int8(x32)
    wq, Sw, Zw = O.quant_weight(w32, "asym", "u8")
    _, _, Y_ref = O.linear_w8a8_int8(xq, Sx, rs, wq, Sw, Zw)
    P.assert_equal(P.bf16_bits(Y), Y_ref, "decode workload Y vs oracle")
