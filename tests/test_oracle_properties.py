"""Property-based pins of the oracle's quantizers (hypothesis).

Random rows of finite fp32 values are checked against what absmax / min-max
quantization guarantees by construction ("大模型量化" (Xilyfe), symmetric and
asymmetric sections; "大模型量化技术" overview 2.3): code ranges, the end
points of a row landing on the end codes, half-step error bounds, odd
symmetry, row sums, the e4m3 rounding's monotonicity and saturation (OCP
FP8 E4M3 definition), the LLM.int8 outlier rule by brute force, the FP8
clip and static scales.  Exact rational arithmetic decides the codes away
from ties.
"""
from fractions import Fraction

import numpy as np
from hypothesis import HealthCheck, given, settings
from hypothesis import strategies as st
from hypothesis.extra.numpy import arrays

from oracle import oracle as O

SETTINGS = settings(max_examples=60, deadline=None, derandomize=True,
                    suppress_health_check=[HealthCheck.too_slow])

finite = st.floats(min_value=-3.0e4, max_value=3.0e4, allow_nan=False, allow_infinity=False,
                   width=32)
rows = st.integers(1, 4).flatmap(
    lambda r: st.integers(1, 8).flatmap(
        lambda c: arrays(np.float32, (r, 32 * c), elements=finite)))


def _near_tie(t: Fraction) -> bool:
    f = t - (t.numerator // t.denominator)
    return abs(f - Fraction(1, 2)) < Fraction(1, 2 ** 18)


@SETTINGS
@given(rows)
def test_symmetric_int8_properties(x):
    q, S, rs = O.quant_act_int8(x)
    assert np.abs(q.astype(np.int32)).max() <= 127
    assert np.array_equal(rs, q.astype(np.int32).sum(axis=1))
    for r in range(x.shape[0]):
        a = float(np.abs(x[r]).max())
        s = float(S[r])
        if a == 0.0:
            assert s == np.float32(1e-8) and not q[r].any()
            continue
        raw = np.float32(np.float32(a) / np.float32(127))
        assert s == float(max(raw, np.float32(1e-8)))               # eps floor
        if raw >= np.float32(1e-8):
            j = int(np.abs(x[r]).argmax())
            assert abs(int(q[r, j])) == 127
        for jj in range(0, x.shape[1], 7):
            t = Fraction(float(x[r, jj])) / Fraction(s)
            if not _near_tie(t):
                want = min(range(-127, 128), key=lambda c: abs(t - c))
                assert q[r, jj] == want
    qn, Sn, _ = O.quant_act_int8(-x)
    assert np.array_equal(Sn, S) and np.array_equal(qn, -q)


@SETTINGS
@given(rows)
def test_asymmetric_int8_properties(w):
    q, S, Z = O.quant_weight(w, "asym")
    assert q.min() >= -128 and q.max() <= 127
    for r in range(w.shape[0]):
        lo, hi = float(w[r].min()), float(w[r].max())
        s = float(S[r])
        if hi == lo:
            continue
        jlo = int(w[r].argmin())
        if lo <= 0.0 <= hi:
            assert q[r, jlo] == -128
            # dequantized values sit within half a step (plus rounding slop of S)
            deq = s * (q[r].astype(np.float64) - float(Z[r]))
            assert np.all(np.abs(deq - w[r].astype(np.float64)) <= s * (0.5 + 2.0 ** -18) + 1e-30)


@SETTINGS
@given(rows)
def test_group_quant_is_blockwise_symmetric(w):
    g = 32
    q, S = O.quant_weight_group(w, g)
    n, k = w.shape
    qb, Sb, _ = O.quant_weight(w.reshape(n * (k // g), g), "sym", bits=4)
    assert np.array_equal(q.reshape(n * (k // g), g), qb)
    assert np.array_equal(S.reshape(-1), Sb)


@SETTINGS
@given(arrays(np.float32, (64,), elements=st.floats(min_value=-2000.0, max_value=2000.0,
                                                    allow_nan=False, width=32)))
def test_e4m3_rounding_properties(v):
    codes = O.round_e4m3(v)
    back = O.widen_e4m3(codes).astype(np.float64)
    x = v.astype(np.float64)
    order = np.argsort(x, kind="stable")
    assert np.all(np.diff(back[order]) >= 0)                      # monotone
    assert np.all(np.abs(back) <= 448.0)                          # saturates
    assert np.array_equal(O.round_e4m3(back.astype(np.float32)), codes)   # idempotent
    inside = np.abs(x) <= 448.0
    # nearest: no finite e4m3 value is strictly closer (spacing 2^(e-3), subnormals 2^-9)
    e = np.floor(np.log2(np.maximum(np.abs(x), 2.0 ** -6)))
    half = np.exp2(e - 3) / 2
    assert np.all(np.abs(back - x)[inside] <= half[inside] + 1e-12)


@SETTINGS
@given(rows, st.floats(min_value=0.5, max_value=40.0, width=32))
def test_outlier_columns_brute_force(x, T):
    mask, idx, count = O.outlier_columns(x, T)
    want = (np.abs(x.astype(np.float64)) > T).any(axis=0)
    assert np.array_equal(mask.astype(bool), want)
    assert idx.tolist() == np.nonzero(want)[0].tolist() and count == int(want.sum())
    # the regular stream's per-token scale ignores those columns; their codes are 0
    q, S, _ = O.quant_act_int8(x, skip=mask)
    assert not q[:, want].any()
    rest = np.where(want[None, :], 0.0, np.abs(x))
    expect = np.maximum((rest.max(axis=1).astype(np.float32) / np.float32(127)).astype(np.float32),
                        np.float32(1e-8))
    assert np.array_equal(S, expect)


@SETTINGS
@given(rows, st.sampled_from([0.0, 1200.0, 50.0]))
def test_fp8_activation_clip(x, ub):
    q, S = O.quant_act_fp8(x, ub)
    a = np.abs(x).max(axis=1)
    if ub > 0:
        a = np.minimum(a, np.float32(ub))
    expect = np.maximum((a.astype(np.float32) / np.float32(448)).astype(np.float32), np.float32(1e-8))
    assert np.array_equal(S, expect)
    back = np.abs(O.widen_e4m3(q))
    assert back.max() <= 448.0
    over = np.abs(x) > (a[:, None] if ub > 0 else np.inf)
    assert np.all(back[over] == 448.0)                 # values past the clip saturate


@SETTINGS
@given(rows, st.floats(min_value=0.0009765625, max_value=50.0, width=32))
def test_static_scale_and_requant(x, S):
    q, Sr, rs = O.quant_act_static(x, S)
    assert np.all(Sr == np.float32(S)) and np.array_equal(rs, q.astype(np.int32).sum(axis=1))
    assert np.abs(q.astype(np.int32)).max() <= 127
    assert np.array_equal(O.requant(x, S), q)          # the same rule on a layer output
    s = Fraction(float(np.float32(S)))
    flat = x.reshape(-1)
    for j in range(0, flat.size, 5):
        t = Fraction(float(flat[j])) / s
        if not _near_tie(t):
            want = max(-127, min(127, min(range(-128, 129), key=lambda c: abs(t - c))))
            assert q.reshape(-1)[j] == want


blocks256 = st.integers(1, 3).flatmap(
    lambda r: st.integers(1, 2).flatmap(
        lambda c: arrays(np.float32, (r, 256 * c),
                         elements=st.floats(min_value=-100.0, max_value=100.0, width=32))))


@SETTINGS
@given(blocks256)
def test_q4k_scale_properties(w):
    r = O.quant_weight_q4k(w)
    n, k = w.shape
    ss = r["s_sub"].reshape(n, k // 256, 8)
    qs = r["q_sub"].reshape(n, k // 256, 8)
    sup = r["s_super"]
    assert qs.max() <= 15
    assert np.array_equal(sup, (ss.max(axis=2) / np.float32(15)).astype(np.float32))
    top = np.take_along_axis(qs, ss.argmax(axis=2)[..., None], 2)[..., 0]
    assert np.all(top == 15)
    eff = r["S_eff"].reshape(n, k // 256, 8).astype(np.float64)
    assert np.all(np.abs(eff - ss) <= sup[..., None].astype(np.float64) * (0.5 + 2.0 ** -18))


@SETTINGS
@given(st.integers(1, 5), st.integers(1, 3), st.sampled_from([32, 64]), st.integers(0, 2 ** 31 - 1))
def test_w4a16_product_matches_fp64(m, nk, g, seed):
    rng = np.random.default_rng(seed)
    n, k = 16, 64 * nk
    x = O.widen16(O.round16(rng.standard_normal((m, k)).astype(np.float32), "bf16"), "bf16")
    w = (rng.standard_normal((n, k)) * 0.05).astype(np.float32)
    q, S = O.quant_weight_group(w, g)
    y, _ = O.linear_w4a16(x, q, S, g, "bf16")
    wd = O.widen16(O.dequant_group16(q, S, g, "bf16"), "bf16").astype(np.float64)
    ref = x.astype(np.float64) @ wd.T
    assert np.all(np.abs(y.astype(np.float64) - ref) <= np.spacing(np.abs(ref.astype(np.float32))))
