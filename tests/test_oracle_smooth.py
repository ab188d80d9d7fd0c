"""Pins of the oracle's activation smoothing ("大模型量化" (Xilyfe), algorithm
list, SmoothQuant: outlier channels of the activation are moved onto the
weight so the activation quantizes easily).

The smoothing step is checked against numpy's IEEE float32 multiply (the rest
of the quantizer is pinned in test_oracle_quant.py); the convention (divide the
activation column, multiply the weight column) against the exact invariance of
X W^T under power-of-two factors; and the purpose, a smaller activation
quantization error once an outlier column is smoothed.
"""
import numpy as np

from oracle import oracle as O


def _x(seed=0, m=6, k=256):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((m, k)).astype(np.float32)
    x[:, 17] *= 40.0          # an outlier channel
    return x


def test_unit_multipliers_give_the_dynamic_quantizer():
    x = _x()
    q, S, rs = O.quant_act_smooth(x, np.ones(x.shape[1], np.float32))
    q2, S2, rs2 = O.quant_act_int8(x)
    assert np.array_equal(q, q2) and np.array_equal(S, S2) and np.array_equal(rs, rs2)


def test_the_smoothing_step_is_an_ieee_float32_multiply():
    x = _x(1)
    rng = np.random.default_rng(2)
    mult = rng.uniform(0.05, 3.0, x.shape[1]).astype(np.float32)
    q, S, rs = O.quant_act_smooth(x, mult)
    q2, S2, rs2 = O.quant_act_int8((x * mult[None, :]).astype(np.float32))
    assert np.array_equal(q, q2) and np.array_equal(S, S2) and np.array_equal(rs, rs2)


def test_power_of_two_smoothing_leaves_the_product_unchanged():
    x = _x(3)
    rng = np.random.default_rng(4)
    w = (rng.standard_normal((32, x.shape[1])) * 0.02).astype(np.float32)
    e = rng.integers(-3, 4, x.shape[1])
    s = np.exp2(e).astype(np.float32)
    xs = (x * (1.0 / s)[None, :]).astype(np.float32)
    ws = O.smooth_weight(w, s)
    assert np.array_equal(ws, (w * s[None, :]).astype(np.float32))
    assert np.array_equal(xs.astype(np.float64) @ ws.T.astype(np.float64),
                          x.astype(np.float64) @ w.T.astype(np.float64))


def test_smoothing_an_outlier_channel_reduces_the_activation_error():
    x = _x(5)
    k = x.shape[1]
    s = np.ones(k, np.float32)
    s[17] = 40.0                                   # absorb the outlier into the weight
    mult = (1.0 / s).astype(np.float32)
    q0, S0, _ = O.quant_act_int8(x)
    q1, S1, _ = O.quant_act_smooth(x, mult)
    err0 = np.abs(q0 * S0[:, None] - x)                          # plain
    err1 = np.abs(q1 * S1[:, None] * s[None, :] - x)             # smoothed, mapped back
    keep = np.arange(k) != 17
    assert err1[:, keep].mean() < 0.2 * err0[:, keep].mean()
