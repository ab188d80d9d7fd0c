"""GPU parity of the quantize kernels against the CPU oracle, bit-exact.

Every call goes through the C ABI (bit_quantized_b200.q8 marshals torch tensors
into raw pointers).  Inputs are the seeded workloads at full size plus edge
shapes: one row, K = 32, rows that do not fill a thread group, rows longer
than the register-cached path, fp32 inputs.
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
ACT_WORKLOADS = ["tiny_mixed", "decode_q_proj", "prefill_ffn_up", "mixed_512"]


def _act_int8_check(X: torch.Tensor, x32: np.ndarray, what: str):
    qa = q8.q8_quantize_act(X.to(DEV), "int8")
    torch.cuda.synchronize()
    q, S, rs = O.quant_act_int8(x32)
    P.assert_equal(qa.codes.cpu().numpy(), q, what + " codes")
    P.assert_equal(qa.scale.cpu().numpy().view(np.uint32), S.view(np.uint32), what + " scale")
    P.assert_equal(qa.rowsum.cpu().numpy(), rs, what + " rowsum")


@pytest.mark.parametrize("name", ACT_WORKLOADS)
def test_act_int8_workloads(name):
    X, W, info, x32, w32 = P.workload(name)
    _act_int8_check(X, x32, name)


@pytest.mark.parametrize("m,k,dtype", [(1, 32, torch.bfloat16), (3, 96, torch.float16),
                                       (7, 4096 + 32, torch.bfloat16), (2, 32768, torch.float16),
                                       (5, 160, torch.float32), (33, 8192, torch.bfloat16)])
def test_act_int8_edges(m, k, dtype):
    X = workloads.random_matrix(m, k, dtype, seed=m * 1000 + k)
    X[0, k // 2] = 0.0
    _act_int8_check(X, P.host_f32(X), f"{m}x{k} {dtype}")


def test_act_int8_zero_rows_and_ties():
    X = torch.zeros(4, 64, dtype=torch.float32)
    X[1, :8] = torch.tensor([127.0, 62.5, 63.5, -62.5, -63.5, 0.5, 1.5, -0.5])
    X[2, 3] = -1e-30
    _act_int8_check(X, P.host_f32(X), "zeros/ties")


def test_act_int8_strided_input():
    base = workloads.random_matrix(24, 512, torch.bfloat16, seed=5)
    view = base[:, 128:384]          # row stride 512, 16-byte aligned start
    qa = q8.q8_quantize_act(base.to(DEV)[:, 128:384], "int8")
    torch.cuda.synchronize()
    q, S, rs = O.quant_act_int8(P.host_f32(view.contiguous()))
    P.assert_equal(qa.codes.cpu().numpy(), q, "strided codes")


def _act_fp8_check(X, x32, ub, what):
    qa = q8.q8_quantize_act(X.to(DEV), "fp8", clip_ub=ub)
    torch.cuda.synchronize()
    q, S = O.quant_act_fp8(x32, ub)
    P.assert_equal(P.codes_u8(qa.codes), q, what + " codes")
    P.assert_equal(qa.scale.cpu().numpy().view(np.uint32), S.view(np.uint32), what + " scale")


def test_act_fp8_workload():
    X, W, info, x32, w32 = P.workload("fp8_rowwise")
    _act_fp8_check(X, x32, 1200.0, "fp8_rowwise")


def test_act_fp8_clip_binds():
    X = workloads.random_matrix(9, 256, torch.bfloat16, seed=11)
    X[0, 3] = 5000.0
    X[1, 7] = -1300.0
    X[2, 9] = 1199.0
    X[3, :] = 0.0
    x32 = P.host_f32(X)
    for ub in (1200.0, 0.0, 100.0):
        _act_fp8_check(X, x32, ub, f"ub={ub}")


@pytest.mark.parametrize("m,k", [(1, 32), (17, 8192 + 64), (4, 20000 // 32 * 32)])
def test_act_fp8_edges(m, k):
    X = workloads.random_matrix(m, k, torch.bfloat16, seed=k) * 30
    _act_fp8_check(X, P.host_f32(X), 1200.0, f"{m}x{k}")


WEIGHT_CASES = [("tiny_mixed", "asym", "s8"), ("decode_q_proj", "asym", "u8"),
                ("prefill_ffn_up", "sym", "s8"), ("mixed_512", "asym", "s8"),
                ("fp8_rowwise", "fp8", "e4m3")]


def _weight_check(W: torch.Tensor, w32: np.ndarray, scheme: str, codes: str, what: str):
    qw = q8.q8_quantize_weight(W.to(DEV), scheme, codes)
    torch.cuda.synchronize()
    q, S, Z = O.quant_weight(w32, scheme, codes)
    got = P.codes_u8(qw.codes) if codes in ("u8", "e4m3") else qw.codes.cpu().numpy()
    P.assert_equal(got, q, what + " codes")
    P.assert_equal(qw.scale.cpu().numpy().view(np.uint32), S.view(np.uint32), what + " scale")
    if Z is not None:
        P.assert_equal(qw.zero_point.cpu().numpy(), Z, what + " zero point")
    return qw, (q, S, Z)


@pytest.mark.parametrize("name,scheme,codes", WEIGHT_CASES)
def test_weight_workloads(name, scheme, codes):
    X, W, info, x32, w32 = P.workload(name)
    _weight_check(W, w32, scheme, codes, name)


@pytest.mark.parametrize("scheme,codes", [("asym", "s8"), ("asym", "u8"), ("sym", "s8"),
                                          ("fp8", "e4m3")])
def test_weight_edge_rows(scheme, codes):
    W = workloads.random_matrix(16, 96, torch.float16, seed=3, std=0.02)
    W[0] = 0.0                                   # zero range: eps scale
    W[1] = 0.25                                  # constant row
    W[2] = W[2].abs() + 0.1                      # no zero crossing
    W[3, 5] = 3.0                                # one large entry
    _weight_check(W, P.host_f32(W), scheme, codes, f"edges {scheme}/{codes}")


def test_weight_fp32_input_and_stride():
    base = workloads.random_matrix(48, 320, torch.float32, seed=8, std=0.05)
    Wd = base.to(DEV)[:, 32:288]
    qw = q8.q8_quantize_weight(Wd, "asym", "s8")
    torch.cuda.synchronize()
    q, S, Z = O.quant_weight(base[:, 32:288].contiguous().numpy(), "asym")
    P.assert_equal(qw.codes.cpu().numpy(), q, "fp32 strided codes")


@pytest.mark.parametrize("codes,kind,out", [("s8", "s8", torch.float32), ("u8", "u8", torch.bfloat16),
                                            ("e4m3", "e4m3", torch.float16)])
def test_dequantize_weight(codes, kind, out):
    W = workloads.random_matrix(64, 256, torch.bfloat16, seed=21, std=0.02)
    scheme = "fp8" if codes == "e4m3" else "asym"
    qw, (q, S, Z) = _weight_check(W, P.host_f32(W), scheme, codes, "dequant input")
    d = q8.q8_dequantize_weight(qw, out)
    torch.cuda.synchronize()
    ref = O.dequant_weight_codes(q, kind, S, Z)
    if out == torch.float32:
        P.assert_equal(d.cpu().numpy().view(np.uint32), ref.view(np.uint32), "dequant f32")
    else:
        fmt = "bf16" if out == torch.bfloat16 else "f16"
        P.assert_equal(d.cpu().view(torch.int16).numpy().view(np.uint16), O.round16(ref, fmt),
                       "dequant " + fmt)


# ------------------------------------------------------------------ LLM.int8 activation side

def _outlier_check(X: torch.Tensor, threshold: float, what: str):
    x32 = P.host_f32(X)
    r = q8.q8_outlier_quantize_act(X.to(DEV), threshold)
    torch.cuda.synchronize()
    mask, idx, count = O.outlier_columns(x32, threshold)
    q, S, rs = O.quant_act_int8(x32, skip=mask)
    P.assert_equal(r["mask"].cpu().numpy(), mask, what + " mask")
    assert int(r["count"].item()) == count, what + " count"
    P.assert_equal(r["idx"].cpu().numpy()[:count], idx, what + " idx")
    P.assert_equal(r["codes"].cpu().numpy(), q, what + " codes")
    P.assert_equal(r["scale"].cpu().numpy().view(np.uint32), S.view(np.uint32), what + " scale")
    P.assert_equal(r["rowsum"].cpu().numpy(), rs, what + " rowsum")
    xo = r["x_outlier"].cpu()
    cpad = (count + 63) // 64 * 64
    want = workloads.bits16(X.contiguous())[:, idx]
    P.assert_equal(xo.view(torch.int16).numpy().view(np.uint16)[:, :count], want, what + " x_outlier")
    assert (xo[:, count:cpad] == 0).all(), what + " x_outlier padding"
    return count


@pytest.mark.parametrize("name", ["tiny_mixed", "mixed_512"])
def test_outlier_act_workloads(name):
    X, W, info, x32, w32 = P.workload(name)
    count = _outlier_check(X, 6.0, name)
    assert count >= len(info["planted_columns"])


@pytest.mark.parametrize("threshold", [0.0, -1.0, float("inf"), 1e-30, 6.0])
def test_outlier_act_thresholds(threshold):
    X = workloads.random_matrix(40, 320, torch.float16, seed=31)
    X[3, 100] = 6.0            # exactly the threshold: not an outlier
    X[7, 200] = -6.01
    _outlier_check(X, threshold, f"T={threshold}")


def test_outlier_act_one_row():
    X = workloads.random_matrix(1, 64, torch.float16, seed=32)
    X[0, 63] = 7.0
    assert _outlier_check(X, 6.0, "one row") == 1


def test_quotient_rounding_at_exact_midpoints():
    """Rows whose scale is exactly 1 put x / S on integer and E4M3 rounding
    midpoints, which must round half to even."""
    ints = [127.0, 62.5, 63.5, -62.5, -63.5, 0.5, 1.5, -0.5, 2.5, -2.5, 100.5, -126.5]
    Xi = torch.zeros(2, 64, dtype=torch.bfloat16)
    Xi[0, :len(ints)] = torch.tensor(ints)
    Xi[1, :len(ints)] = -torch.tensor(ints)
    _act_int8_check(Xi, P.host_f32(Xi), "integer midpoints")
    # E4M3 midpoints: 1.0625 (1 | 1.125), 3.125 (3 | 3.25), 0.0029296875 (subnormal 3*2^-10),
    # 240 (224 | 256), 432 (416 | 448)
    mids = [448.0, 1.0625, 3.125, 0.0029296875, 240.0, 432.0, -1.0625, -240.0, 1.1875, 13.0]
    Xf = torch.zeros(2, 64, dtype=torch.bfloat16)
    Xf[0, :len(mids)] = torch.tensor(mids)
    Xf[1, :len(mids)] = -torch.tensor(mids)
    _act_fp8_check(Xf, P.host_f32(Xf), 0.0, "e4m3 midpoints")
    W = torch.zeros(16, 64, dtype=torch.bfloat16)
    W[0, :len(mids)] = torch.tensor(mids)
    _weight_check(W, P.host_f32(W), "fp8", "e4m3", "weight e4m3 midpoints")
    Wa = torch.zeros(16, 64, dtype=torch.float32)
    Wa[:, 0] = 0.0
    Wa[:, 1] = 255.0            # S = 1 exactly, Z = -128
    Wa[:, 2:14] = torch.tensor([0.5, 1.5, 2.5, 100.5, 127.5, 128.5, 200.5, 254.5, 3.5, 4.5, 5.5, 6.5])
    _weight_check(Wa, P.host_f32(Wa), "asym", "s8", "asym integer midpoints")


def test_ties_with_non_power_of_two_scale():
    """absmax = 127 * 9/64 (fp16-exact) gives S = 9/64 exactly, so
    x = (n + 1/2) * 9/128 lies exactly on a rounding midpoint of x / S: whole
    16-byte vectors of such elements, and single ones among regular values."""
    m, k = 6, 256
    g = torch.Generator().manual_seed(41)
    n = torch.randint(-100, 100, (m, k), generator=g).to(torch.float32)
    X = ((2 * n + 1) * 9 / 128).to(torch.float16)
    X[:, 0] = 127 * 9 / 64
    X[3:, 1:] = (torch.randn(3, k - 1, generator=g) * 4).to(torch.float16)
    X[3, 37] = 0.5 * 9 / 64                 # one midpoint among regular values
    X[4, 200] = -2.5 * 9 / 64
    _act_int8_check(X, P.host_f32(X), "int8 ties, S = 9/64")
    # E4M3 midpoints times S = 63 / 448 = 9/64
    mids = torch.tensor([1.0625, 3.125, 240.0, 432.0, -1.0625, -13.0, 1.1875, 0.0029296875])
    Xf = (mids.repeat(m, k // 8) * 9 / 64).to(torch.float16)
    Xf[:, 0] = 63.0
    Xf[3:, 1:] = (torch.randn(3, k - 1, generator=g) * 4).to(torch.float16)
    Xf[3, 9] = 3.125 * 9 / 64
    _act_fp8_check(Xf, P.host_f32(Xf), 0.0, "e4m3 ties, S = 9/64")
    W = Xf.clone()
    _weight_check(W, P.host_f32(W), "fp8", "e4m3", "weight e4m3 ties")
    _weight_check(X.clone(), P.host_f32(X), "sym", "s8", "weight sym ties")
