"""Pins for the oracle's GEMMs, epilogues and the LLM.int8 merge.

Integer dot products are checked against numpy's int64 matmul; the dequant
epilogue against an fp64 matmul of the dequantized operands (so a dropped
zero-point term, a wrong sign or a transposed operand fails); the FP8 and
fp16 streams against fp64 matmuls of torch-decoded values; and the mixed
decomposition against its special cases (threshold off, everything outlier).
"""
import numpy as np
import pytest
import torch

import workloads
from oracle import oracle as O


def _codes(seed, m, k, signed=True):
    rng = np.random.default_rng(seed)
    if signed:
        return rng.integers(-128, 128, (m, k), dtype=np.int64).astype(np.int8)
    return rng.integers(0, 256, (m, k), dtype=np.int64).astype(np.uint8)


@pytest.mark.parametrize("signed_b", [True, False])
def test_gemm_int_matches_numpy(signed_b):
    a = _codes(1, 37, 96)
    b = _codes(2, 53, 96, signed_b)
    ref = a.astype(np.int64) @ b.astype(np.int64).T
    assert np.array_equal(O.gemm_int(a, b), ref)
    rows, cols = np.array([0, 36, 5]), np.array([52, 1])
    assert np.array_equal(O.gemm_int(a, b, rows, cols), ref[np.ix_(rows, cols)])


def test_int32_bound_holds_at_k4096():
    # worst case |acc| <= K * 127 * 255 for int8 x uint8 codes
    a = np.full((1, 4096), 127, np.int8)
    b = np.full((1, 4096), 255, np.uint8)
    acc = O.gemm_int(a, b)
    assert acc[0, 0] == 4096 * 127 * 255 < 2**31 - 1


def _quantized_pair(seed, m, n, k, scheme="asym", codes="s8"):
    x = workloads.random_matrix(m, k, torch.bfloat16, seed).float().numpy()
    w = workloads.random_matrix(n, k, torch.bfloat16, seed + 1, 0.02).float().numpy()
    xq, Sx, rs = O.quant_act_int8(x)
    wq, Sw, Zw = O.quant_weight(w, scheme, codes)
    return x, w, xq, Sx, rs, wq, Sw, Zw


@pytest.mark.parametrize("scheme,codes", [("asym", "s8"), ("asym", "u8"), ("sym", "s8")])
def test_epilogue_matches_fp64_of_dequantized_operands(scheme, codes):
    x, w, xq, Sx, rs, wq, Sw, Zw = _quantized_pair(3, 24, 40, 256, scheme, codes)
    bias = np.linspace(-1, 1, 40).astype(np.float32)
    acc, y, Y = O.linear_w8a8_int8(xq, Sx, rs, wq, Sw, Zw, bias)
    xd = Sx[:, None].astype(np.float64) * xq
    z = 0.0 if Zw is None else Zw[:, None].astype(np.float64)
    wd = Sw[:, None].astype(np.float64) * (wq.astype(np.float64) - z)
    y64 = xd @ wd.T + bias
    mag = np.abs(xd) @ np.abs(wd).T + np.abs(bias)
    assert np.all(np.abs(y - y64) <= 4 * 2.0**-24 * mag + 1e-30)
    # the quantized product is a plausible approximation of the real one
    rel = np.linalg.norm(y64 - (x.astype(np.float64) @ w.T + bias)) / np.linalg.norm(y64)
    assert rel < 0.05


def test_zero_point_identity():
    x, w, xq, Sx, rs, wq, Sw, Zw = _quantized_pair(4, 5, 7, 64)
    acc = O.gemm_int(xq, wq)
    for m in range(5):
        for n in range(7):
            direct = sum(int(xq[m, t]) * (int(wq[n, t]) - int(Zw[n])) for t in range(64))
            assert acc[m, n] - int(Zw[n]) * int(rs[m]) == direct


def test_bf16_output_is_rne_of_fp32():
    x, w, xq, Sx, rs, wq, Sw, Zw = _quantized_pair(5, 8, 16, 128)
    acc, y, Y = O.linear_w8a8_int8(xq, Sx, rs, wq, Sw, Zw)
    ref = torch.from_numpy(y).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(Y, ref)


def test_fp8_gemm_matches_fp64():
    rng = np.random.default_rng(6)
    a = rng.integers(0, 256, (20, 128), dtype=np.int64).astype(np.uint8)
    b = rng.integers(0, 256, (12, 128), dtype=np.int64).astype(np.uint8)
    a[(a & 0x7F) == 0x7F] = 0   # no NaN codes
    b[(b & 0x7F) == 0x7F] = 0
    dec = lambda c: torch.from_numpy(c.view(np.int8)).view(torch.float8_e4m3fn).double().numpy()
    ref = dec(a) @ dec(b).T
    Sx = np.full(20, 0.5, np.float32)
    Sw = np.full(12, 0.25, np.float32)
    acc, y, _ = O.linear_w8a8_fp8(a, Sx, b, Sw)
    mag = np.abs(dec(a)) @ np.abs(dec(b)).T
    assert np.all(np.abs(acc - ref) <= 2.0**-24 * np.abs(ref) + 2.0**-50 * mag)
    assert np.array_equal(y, (acc * np.float32(0.5) * np.float32(0.25)).astype(np.float32))


def test_fp8_linear_plausible():
    x = workloads.random_matrix(32, 512, torch.bfloat16, 7).float().numpy()
    w = workloads.random_matrix(48, 512, torch.bfloat16, 8, 0.02).float().numpy()
    xq, Sx = O.quant_act_fp8(x, 1200.0)
    wq, Sw, _ = O.quant_weight(w, "fp8")
    _, y, _ = O.linear_w8a8_fp8(xq, Sx, wq, Sw)
    ref = x.astype(np.float64) @ w.T
    assert np.linalg.norm(y - ref) / np.linalg.norm(ref) < 0.05


def test_dequant_f16_within_half_ulp():
    x, w, xq, Sx, rs, wq, Sw, Zw = _quantized_pair(9, 4, 32, 64)
    cols = np.array([0, 5, 63], np.int32)
    w16 = O.widen16(O.dequant_weight_f16(wq, Sw, Zw, cols), "f16").astype(np.float64)
    exact = Sw[:, None].astype(np.float64) * (wq[:, cols].astype(np.float64) - Zw[:, None])
    ulp = np.spacing(np.abs(exact).astype(np.float16)).astype(np.float64)
    assert np.all(np.abs(w16 - exact) <= 0.5 * ulp + 2.0**-24 * np.abs(exact))


def test_outlier_gemm_matches_fp64():
    X, W, info = workloads.make_inputs("tiny_mixed")
    x = X.float().numpy()
    w = W.float().numpy()
    idx = np.array(info["planted_columns"], np.int32)
    y16 = O.outlier_gemm(x, w[:, idx], idx)
    ref = x[:, idx].astype(np.float64) @ w[:, idx].T.astype(np.float64)
    assert np.all(np.abs(y16 - ref) <= 2.0**-24 * np.abs(ref) + 1e-30)


def _mixed_inputs():
    X, W, info = workloads.make_inputs("tiny_mixed")
    x = X.float().numpy()
    w = W.float().numpy()
    wq, Sw, Zw = O.quant_weight(w, "asym")
    return x, w, wq, Sw, Zw


@pytest.mark.parametrize("threshold", [0.0, -3.0, float("inf")])
def test_mixed_without_outliers_is_plain_w8a8(threshold):
    x, w, wq, Sw, Zw = _mixed_inputs()
    r = O.linear_int8_mixed(x, wq, Sw, Zw, threshold)
    xq, Sx, rs = O.quant_act_int8(x)
    acc, y, Y = O.linear_w8a8_int8(xq, Sx, rs, wq, Sw, Zw)
    assert r["count"] == 0
    assert np.array_equal(r["acc"], acc) and np.array_equal(r["Y"], Y)
    assert np.array_equal(r["y"].view(np.uint32), y.view(np.uint32))


def test_mixed_everything_outlier_is_fp16_gemm():
    x, w, wq, Sw, Zw = _mixed_inputs()
    r = O.linear_int8_mixed(x, wq, Sw, Zw, 1e-30)
    assert r["count"] == np.count_nonzero(np.abs(x).max(0) > 0)
    assert np.all(r["xq"] == 0) and np.all(r["acc"] == 0)
    ref = x.astype(np.float64) @ r["w16"].astype(np.float64).T if r["count"] == x.shape[1] else None
    if ref is not None:
        assert np.all(np.abs(r["y"] - ref) <= 2.0**-23 * (np.abs(x) @ np.abs(r["w16"]).T) + 1e-30)


def test_mixed_decomposition_beats_plain_int8_on_outliers():
    x, w, wq, Sw, Zw = _mixed_inputs()
    ref = x.astype(np.float64) @ w.T.astype(np.float64)
    mixed = O.linear_int8_mixed(x, wq, Sw, Zw, 6.0)["y"]
    plain = O.linear_int8_mixed(x, wq, Sw, Zw, 0.0)["y"]
    e_mixed = np.linalg.norm(mixed - ref) / np.linalg.norm(ref)
    e_plain = np.linalg.norm(plain - ref) / np.linalg.norm(ref)
    assert e_mixed < 0.5 * e_plain and e_mixed < 0.05


def test_mixed_has_fp16_weight_uses_original_columns():
    x, w, wq, Sw, Zw = _mixed_inputs()
    r = O.linear_int8_mixed(x, wq, Sw, Zw, 6.0, w16_full=w)
    assert np.array_equal(r["w16"], w[:, r["idx"]])
    r2 = O.linear_int8_mixed(x, wq, Sw, Zw, 6.0)
    assert np.array_equal(r["acc"], r2["acc"])          # the int8 stream is unchanged
    assert not np.array_equal(r["y16"], r2["y16"])      # the fp16 stream's weight differs


def test_mixed_bias_added_after_merge():
    x, w, wq, Sw, Zw = _mixed_inputs()
    bias = np.linspace(-2, 2, w.shape[0]).astype(np.float32)
    r = O.linear_int8_mixed(x, wq, Sw, Zw, 6.0, bias=bias)
    r0 = O.linear_int8_mixed(x, wq, Sw, Zw, 6.0)
    assert np.array_equal(r["y"], (r0["y"] + bias).astype(np.float32))


@pytest.mark.parametrize("kind", ["s8", "u8", "e4m3"])
def test_dequant_weight_codes(kind):
    w = workloads.random_matrix(16, 64, torch.bfloat16, 12, 0.02).float().numpy()
    scheme = {"s8": "asym", "u8": "asym", "e4m3": "fp8"}[kind]
    q, S, Z = O.quant_weight(w, scheme, {"s8": "s8", "u8": "u8", "e4m3": "e4m3"}[kind])
    d = O.dequant_weight_codes(q, kind, S, Z)
    if kind == "e4m3":
        vals = torch.from_numpy(q.view(np.int8)).view(torch.float8_e4m3fn).double().numpy()
        exact = S[:, None].astype(np.float64) * vals
    else:
        exact = S[:, None].astype(np.float64) * (q.astype(np.float64) - Z[:, None])
    assert np.all(np.abs(d - exact) <= 2.0**-24 * np.abs(exact))
    # dequantized weights sit within the quantization error of the originals
    assert np.all(np.abs(d - w) <= np.maximum(S[:, None] * 0.51, np.abs(w) * 2.0**-3))
