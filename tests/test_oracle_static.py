"""Pins of the oracle's static activation quantizer and output re-quantizer
("大模型量化" (Xilyfe): the paragraph on 静态量化, and the re-quantization step
of 量化对象 / INT8 这么小的范围不会导致溢出吗).

Checked against what the definition q = clamp(rne(fl32(x / S)), -127, 127)
fixes independently of the oracle's code: integer multiples of a power-of-two
scale, ties that round to even, saturation, an independent evaluation with
numpy's IEEE float32 division and Python's round-half-even, and agreement with
the (separately pinned) dynamic quantizer when the static scale equals a row's
dynamic scale.
"""
import numpy as np
import pytest

from oracle import oracle as O


def _independent(x: np.ndarray, S: float) -> np.ndarray:
    t = (np.asarray(x, np.float32) / np.float32(S)).astype(np.float32)   # fl32(x / S)
    r = np.array([round(float(v)) for v in t.ravel()], dtype=np.float64).reshape(t.shape)
    return np.clip(r, -127, 127).astype(np.int8)


def test_integer_multiples_of_a_power_of_two_scale():
    S = 0.125
    n = np.arange(-127, 128, dtype=np.float32)
    q, Sr, rs = O.quant_act_static((n * S)[None, :], S)
    assert (q[0] == n.astype(np.int8)).all()
    assert Sr[0] == np.float32(S) and rs[0] == int(n.sum())


def test_ties_round_to_even_and_saturation():
    x = np.array([[0.5, 1.5, 2.5, -0.5, -1.5, -2.5, 126.5, -126.5, 127.4, 127.6, 1e30, -1e30, 0.0, -0.0]],
                 np.float32)
    q, _, rs = O.quant_act_static(x, 1.0)
    assert q[0].tolist() == [0, 2, 2, 0, -2, -2, 126, -126, 127, 127, 127, -127, 0, 0]
    assert rs[0] == sum(q[0].tolist())


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_matches_an_independent_evaluation(seed):
    rng = np.random.default_rng(seed)
    x = (rng.standard_normal((7, 300)) * rng.choice([0.01, 1.0, 50.0])).astype(np.float32)
    x[0, :20] = np.float32(0.03125) * (np.arange(20) + 0.5)   # near ties for S = 1/32
    for S in (np.float32(rng.uniform(0.001, 0.5)), np.float32(1 / 32), np.float32(3.0)):
        q, Sr, rs = O.quant_act_static(x, float(S))
        want = _independent(x, float(S))
        assert np.array_equal(q, want)
        assert (Sr == S).all()
        assert np.array_equal(rs, want.astype(np.int64).sum(axis=1).astype(np.int32))


def test_static_with_the_dynamic_scale_gives_the_dynamic_codes():
    rng = np.random.default_rng(7)
    x = rng.standard_normal((5, 256)).astype(np.float32)
    qd, Sd, rsd = O.quant_act_int8(x)
    for r in range(5):
        q, _, rs = O.quant_act_static(x[r:r + 1], float(Sd[r]))
        assert np.array_equal(q[0], qd[r]) and rs[0] == rsd[r]


def test_requant_is_the_static_code_of_the_output():
    rng = np.random.default_rng(3)
    y = (rng.standard_normal((4, 64)) * 3).astype(np.float32)
    S = np.float32(0.0234)
    assert np.array_equal(O.requant(y, float(S)), _independent(y, float(S)))
    assert np.array_equal(O.requant(y, float(S)), O.quant_act_static(y, float(S))[0])
    assert O.requant(np.array([2.0 ** 20, -(2.0 ** 20)], np.float32), 1.0).tolist() == [127, -127]
