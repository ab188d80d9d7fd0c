"""Pins for the oracle's weight and activation quantizers.

Each check rests on something other than the oracle itself: the pages' worked
examples (tests/golden), closed-form invariants of absmax / min-max
quantization, brute-force nearest-code search in exact rational arithmetic,
and the outlier rule checked by brute force over columns.
"""
import json
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import workloads
from oracle import oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


# ------------------------------------------------------------------ worked examples

def test_worked_example_per_channel_row_4bit():
    g = _golden("worked_examples_4bit.json")["per_channel_row"]
    w = np.float32([g["values"]])
    q, S, _ = O.quant_weight(w, "sym", bits=4)
    assert abs(S[0] - g["scale_printed"]) < 0.005
    assert q[0].tolist() == [0, 0, 0, 7, 7, 7]
    assert q[0][0] == g["codes_printed"]["0.0002"] and q[0][3] == g["codes_printed"]["48.5"]


def test_worked_example_q4k_sub_blocks():
    g = _golden("worked_examples_4bit.json")["q4k_sub_blocks"]
    w = np.float32(g["blocks"])
    q, S, _ = O.quant_weight(w, "sym", bits=4)
    assert np.allclose(S, g["scales_printed"], atol=0.0006)
    assert q.tolist() == g["codes_by_rule"]
    # the printed codes differ from the rule in exactly one place (recorded in the fixture)
    diff = np.argwhere(np.array(g["codes_printed"]) != np.array(g["codes_by_rule"]))
    assert diff.tolist() == [[2, 3]]
    # the super-block scale re-quantizes the sub-block scales by absmax / 15
    assert abs(float(S.max()) / 15 - g["super_scale_printed"]) < 5e-5


# ------------------------------------------------------------------ helpers

def _rne_fraction(t: Fraction) -> int:
    f = t.numerator // t.denominator
    d = t - f
    if d > Fraction(1, 2):
        return f + 1
    if d < Fraction(1, 2):
        return f
    return f if f % 2 == 0 else f + 1


def _near_half(t: Fraction) -> bool:
    """True when t is within fp32 rounding distance of a half-integer, where the
    rounded quotient fl32(x / S) may fall on either side."""
    f = t.numerator // t.denominator
    return abs((t - f) - Fraction(1, 2)) <= abs(t) * Fraction(1, 2**22)


def _rows(seed, n, k, std=1.0, dtype=torch.bfloat16):
    return workloads.random_matrix(n, k, dtype, seed, std).float().numpy()


# ------------------------------------------------------------------ symmetric

@pytest.mark.parametrize("bits", [3, 4, 8])
def test_sym_brute_force_nearest_code(bits):
    w = _rows(10 + bits, 6, 64)
    q, S, _ = O.quant_weight(w, "sym", bits=bits)
    qmax = 2 ** (bits - 1) - 1
    for r in range(w.shape[0]):
        s = Fraction(float(S[r]))
        for j in range(w.shape[1]):
            t = Fraction(float(w[r, j])) / s
            if _near_half(t):
                continue
            want = max(-qmax, min(qmax, _rne_fraction(t)))
            assert q[r, j] == want, (r, j, float(t))


def test_sym_invariants():
    w = _rows(20, 64, 512, std=0.02)
    q, S, _ = O.quant_weight(w, "sym")
    a = np.abs(w).max(axis=1)
    arg = np.abs(w).argmax(axis=1)
    # the row absmax element lands on +-127 exactly
    assert np.array_equal(np.abs(q[np.arange(64), arg]), np.full(64, 127))
    # per-element error at most S/2 (plus fp32 rounding of the quotient)
    err = np.abs(w.astype(np.float64) - S[:, None].astype(np.float64) * q)
    assert np.all(err <= S[:, None] * (0.5 + 2.0**-16))
    # S = alpha / 127 up to one fp32 rounding (the pages' s = 127 / alpha as a divisor)
    assert np.allclose(S.astype(np.float64), a.astype(np.float64) / 127, rtol=2.0**-23, atol=0)
    # odd symmetry: quantizing -w gives -q with the same scale
    q2, S2, _ = O.quant_weight(-w, "sym")
    assert np.array_equal(S2, S) and np.array_equal(q2, -q)


def test_sym_zero_row_uses_eps():
    q, S, _ = O.quant_weight(np.zeros((2, 32), np.float32), "sym")
    assert np.all(q == 0) and np.all(S == np.float32(1e-8))


# ------------------------------------------------------------------ asymmetric

@pytest.mark.parametrize("bits", [3, 4, 8])
def test_asym_brute_force_nearest_code(bits):
    w = _rows(30 + bits, 6, 64, std=0.5)
    q, S, Z = O.quant_weight(w, "asym", bits=bits)
    qmin, qmax = -(2 ** (bits - 1)), 2 ** (bits - 1) - 1
    for r in range(w.shape[0]):
        s = Fraction(float(S[r]))
        z = int(Z[r])
        for j in range(w.shape[1]):
            t = Fraction(float(w[r, j])) / s
            if _near_half(t):
                continue
            want = max(qmin, min(qmax, _rne_fraction(t) + z))
            assert q[r, j] == want, (r, j)


def test_asym_invariants():
    w = _rows(40, 64, 512, std=0.02)
    q, S, Z = O.quant_weight(w, "asym")
    r = np.arange(64)
    lo, hi = w.min(axis=1), w.max(axis=1)
    # the row minimum maps to -128 exactly; the maximum to 127 (126 from rounding slop)
    assert np.all(q[r, w.argmin(axis=1)] == -128)
    assert np.all(np.isin(q[r, w.argmax(axis=1)], [126, 127]))
    # S = (max - min) / 255 up to two fp32 roundings
    assert np.allclose(S, (hi.astype(np.float64) - lo) / 255, rtol=2.0**-22, atol=0)
    # min-max calibration form: Z = Qmin - round(Rmin / S), i.e. RNE is odd-symmetric
    zmm = -128 - np.round((lo / S).astype(np.float32))
    assert np.array_equal(Z, zmm.astype(np.float32))
    # 0.0 maps exactly to Z
    q0, _, _ = O.quant_weight(np.concatenate([w, np.zeros((64, 1), np.float32)], 1), "asym")
    assert np.array_equal(q0[:, -1].astype(np.float32), Z)
    # dequant error within S/2, except where the top code was clamped
    deq = S[:, None].astype(np.float64) * (q.astype(np.float64) - Z[:, None])
    err = np.abs(w - deq)
    clamped = q == 127
    assert np.all(err[~clamped] <= (S[:, None] * (0.5 + 2.0**-16)).repeat(512, 1)[~clamped])
    assert np.all(err <= S[:, None] * 1.5)


def test_asym_dequant_mse_below_page_bound():
    bound = _golden("page_constants.json")["dequant_mse_bound"]["value"]
    X, W, _ = workloads.make_inputs("decode_q_proj", k=512, n=256)
    w = W.float().numpy()
    q, S, Z = O.quant_weight(w, "asym")
    deq = S[:, None] * (q.astype(np.float32) - Z[:, None])
    assert float(np.mean((deq - w) ** 2)) < bound


def test_asym_uint8_convention_matches_int8():
    w = _rows(41, 8, 64, std=0.02)
    q8, S8, Z8 = O.quant_weight(w, "asym", codes="s8")
    qu, Su, Zu = O.quant_weight(w, "asym", codes="u8")
    assert np.array_equal(Su, S8)
    assert np.array_equal(qu.astype(np.int32) - Zu.astype(np.int32)[:, None],
                          q8.astype(np.int32) - Z8.astype(np.int32)[:, None])
    # the uint8 zero point is the Fabric article's round(-min / scale)
    lo = w.min(axis=1)
    assert np.array_equal(Zu, np.round((-lo / S8).astype(np.float32)).astype(np.float32))


def test_asym_rows_without_zero_crossing_and_constant_rows():
    w = np.float32([[0.5, 0.6, 0.7, 0.9] * 8, [2.0] * 32, [-1.0, -0.5] * 16, [0.0] * 32])
    q, S, Z = O.quant_weight(w, "asym")
    assert np.all((Z >= -128) & (Z <= 127))
    assert S[1] == np.float32(1e-8) and S[3] == np.float32(1e-8)
    assert np.all(q[3] == Z[3])


# ------------------------------------------------------------------ fp8

def test_fp8_weight_codes_are_nearest_e4m3():
    w = _rows(50, 32, 256, std=0.02)
    q, S, _ = O.quant_weight(w, "fp8")
    t = (w / S[:, None]).astype(np.float32)
    ref = torch.from_numpy(t).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(q, ref)
    # the row absmax element lands on +-448 (code 0x7E / 0xFE)
    arg = np.abs(w).argmax(axis=1)
    assert np.all((q[np.arange(32), arg] & 0x7F) == 0x7E)


def test_fp8_act_clip_at_upper_bound():
    ub = _golden("page_constants.json")["activation_scale_ub"]["value"]
    x = _rows(51, 8, 256)
    x[0, 5] = 5000.0
    x[1, 7] = -1300.0
    x[2, 9] = 1199.0
    q, S = O.quant_act_fp8(x, ub)
    assert S[0] == np.float32(np.float32(ub) / np.float32(448))
    assert q[0, 5] == 0x7E and q[1, 7] == 0xFE       # beyond ub: saturated
    assert S[2] == np.float32(np.float32(1199.0) / np.float32(448))
    assert (q[2, 9] & 0x7F) == 0x7E
    # without a bound the scale follows the absmax
    q2, S2 = O.quant_act_fp8(x, 0.0)
    assert S2[0] == np.float32(np.float32(5000.0) / np.float32(448))
    t = (x / S[:, None]).astype(np.float32)
    t = np.clip(t, -448, 448)   # torch's cast gives NaN past 448; saturation checked above
    ref = torch.from_numpy(t).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(q, ref)


# ------------------------------------------------------------------ activations (int8)

def test_act_int8_rowsum_and_skip():
    x = _rows(60, 16, 256)
    skip = np.zeros(256, np.uint8)
    skip[[3, 77, 200]] = 1
    x[:, 77] = 40.0
    q, S, rs = O.quant_act_int8(x, skip)
    assert np.array_equal(rs, q.astype(np.int64).sum(1).astype(np.int32))
    assert np.all(q[:, skip == 1] == 0)
    a = np.abs(x[:, skip == 0]).max(1)
    assert np.allclose(S, a / 127, rtol=2.0**-23, atol=0)
    q0, S0, _ = O.quant_act_int8(x)
    assert np.all(S0 >= S)
    assert np.all(np.abs(q[np.arange(16), np.abs(np.where(skip == 1, 0, x)).argmax(1)]) == 127)


def test_act_int8_ties_round_half_even():
    # alpha = 127 gives S = 1 exactly, so x / S is x itself.
    x = np.float32([[127.0, 62.5, 63.5, -62.5, -63.5, 0.5, 1.5, -0.5] + [0.0] * 24])
    q, S, _ = O.quant_act_int8(x)
    assert S[0] == 1.0
    assert q[0, :8].tolist() == [127, 62, 64, -62, -64, 0, 2, 0]


# ------------------------------------------------------------------ outliers

def test_outlier_columns_brute_force():
    x = _rows(70, 64, 300)
    x[5, 11] = 6.5
    x[9, 200] = -7.0
    x[3, 150] = 6.0         # exactly the threshold: not an outlier ("exceeds")
    x[:, 150] = np.clip(x[:, 150], -6.0, 6.0)
    mask, idx, count = O.outlier_columns(x, 6.0)
    ref = np.flatnonzero((np.abs(x) > 6.0).any(axis=0))
    assert idx.tolist() == ref.tolist() and count == ref.size
    assert np.array_equal(mask, (np.abs(x) > 6.0).any(axis=0).astype(np.uint8))
    assert 150 not in idx and 11 in idx and 200 in idx


def test_outlier_threshold_zero_turns_decomposition_off():
    x = _rows(71, 8, 64)
    for t in (0.0, -1.0):
        mask, idx, count = O.outlier_columns(x, t)
        assert count == 0 and not mask.any()
    mask, idx, count = O.outlier_columns(x, float("inf"))
    assert count == 0


def test_tiny_workload_planted_outliers():
    const = _golden("page_constants.json")
    X, W, info = workloads.make_inputs("tiny_mixed")
    x = X.float().numpy()
    mask, idx, count = O.outlier_columns(x, const["llm_int8_threshold"]["value"])
    assert idx.tolist() == [3, 77] == info["planted_columns"]
    lo, hi = const["outlier_range"]["value"]
    assert np.all((np.abs(x[:, idx]) >= lo) & (np.abs(x[:, idx]) <= hi))


def test_mixed_workload_planted_outliers_found():
    X, W, info = workloads.make_inputs("mixed_512")
    mask, idx, count = O.outlier_columns(X.float().numpy(), 6.0)
    assert set(info["planted_columns"]) <= set(idx.tolist())
