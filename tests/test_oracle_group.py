"""Pins for the oracle's group-wise low-bit weights and the W4A16 product.

Group-wise symmetric quantization ("大模型量化技术" overview, 2.2 granularity
table: one scale per group of 64-128 parameters; "大模型量化" (Xilyfe), GGUF
section: each block of a row gets its own absmax scale, qmax = 7 for 4 bits).
The checks rest on the page's printed Q4_K block example, exact rational
nearest-code search, closed-form invariants of absmax quantization, torch's
16-bit casts and numpy's fp64 matmul.
"""
import json
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

from oracle import oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def _rne_fraction(t: Fraction) -> int:
    f = t.numerator // t.denominator
    d = t - f
    if d > Fraction(1, 2):
        return f + 1
    if d < Fraction(1, 2):
        return f
    return f if f % 2 == 0 else f + 1


def test_q4k_example_as_one_row_of_blocks():
    # The page's three sub-blocks, laid end to end in one row with a group of 4.
    g = _golden("worked_examples_4bit.json")["q4k_sub_blocks"]
    w = np.float32([sum(g["blocks"], [])])
    q, S = O.quant_weight_group(w, 4, bits=4)
    assert S.shape == (1, 3)
    assert np.allclose(S[0], g["scales_printed"], atol=0.0006)
    assert q[0].tolist() == sum(g["codes_by_rule"], [])


def test_scale_layout_and_empty_groups():
    # Row 1, group 2 holds the only non-zero value: its scale is that value / 7
    # and every other group gets the eps floor with zero codes.
    n, k, g = 3, 256, 64
    w = np.zeros((n, k), np.float32)
    w[1, 2 * g + 5] = -3.5
    q, S = O.quant_weight_group(w, g)
    expect = np.full((n, k // g), np.float32(1e-8))
    expect[1, 2] = np.float32(3.5) / np.float32(7)
    assert np.array_equal(S, expect)
    assert q[1, 2 * g + 5] == -7
    assert np.count_nonzero(q) == 1


@pytest.mark.parametrize("g", [32, 64, 128])
def test_absmax_invariants(g):
    rng = np.random.default_rng(5)
    w = (rng.standard_normal((24, 512)) * 0.02).astype(np.float32)
    q, S = O.quant_weight_group(w, g)
    wg = w.reshape(24, -1, g)
    qg = q.reshape(24, -1, g).astype(np.int32)
    assert np.abs(q).max() <= 7
    # the absmax element of every group maps to +-7
    i = np.abs(wg).argmax(axis=2)
    top = np.take_along_axis(qg, i[..., None], 2)[..., 0]
    assert np.all(np.abs(top) == 7)
    # scale is max|w| / 7 per group, every error within half a step
    assert np.array_equal(S, (np.abs(wg).max(axis=2) / np.float32(7)).astype(np.float32))
    err = np.abs(wg.astype(np.float64) - S[..., None].astype(np.float64) * qg)
    assert np.all(err <= S[..., None] * (0.5 + 2.0 ** -20))
    # odd symmetry
    qn, Sn = O.quant_weight_group(-w, g)
    assert np.array_equal(Sn, S) and np.array_equal(qn, -q)


def test_groups_are_independent():
    rng = np.random.default_rng(6)
    n, k, g = 8, 384, 128
    w = (rng.standard_normal((n, k)) * 0.02).astype(np.float32)
    q, S = O.quant_weight_group(w, g)
    w2 = w.copy()
    w2[:, g:2 * g] *= np.float32(4.0)            # exact power-of-two change of group 1
    q2, S2 = O.quant_weight_group(w2, g)
    assert np.array_equal(q2, q)
    assert np.array_equal(S2[:, 1], S[:, 1] * np.float32(4.0))
    assert np.array_equal(S2[:, [0, 2]], S[:, [0, 2]])


def test_whole_row_group_is_per_channel_symmetric():
    rng = np.random.default_rng(7)
    w = (rng.standard_normal((16, 256)) * 0.02).astype(np.float32)
    q, S = O.quant_weight_group(w, 256)
    qs, Ss, _ = O.quant_weight(w, "sym", bits=4)
    assert np.array_equal(q, qs) and np.array_equal(S[:, 0], Ss)


def test_codes_are_nearest_by_exact_search():
    rng = np.random.default_rng(8)
    w = rng.standard_normal((6, 64)).astype(np.float32)
    w[0, :4] = [3.5, -3.5, 1.5, 0.5]             # ties once divided by 1.0 below
    w[0, 4] = 7.0                                 # absmax of group 0 -> S = 1
    q, S = O.quant_weight_group(w, 32)
    ties = 0
    for r in range(w.shape[0]):
        for j in range(w.shape[1]):
            s = Fraction(float(S[r, j // 32]))
            t = Fraction(float(w[r, j])) / s
            best = min(range(-7, 8), key=lambda c: (abs(t - c), c % 2))
            frac_part = t - (t.numerator // t.denominator)
            if abs(frac_part - Fraction(1, 2)) < Fraction(1, 2 ** 20):
                ties += 1
                assert q[r, j] == max(-7, min(7, _rne_fraction(t)))
            else:
                assert q[r, j] == best
    assert ties >= 4


@pytest.mark.parametrize("fmt,tdt", [("bf16", torch.bfloat16), ("f16", torch.float16)])
def test_dequant_group16_matches_torch_cast(fmt, tdt):
    rng = np.random.default_rng(9)
    w = (rng.standard_normal((10, 256)) * 0.05).astype(np.float32)
    q, S = O.quant_weight_group(w, 64)
    got = O.dequant_group16(q, S, 64, fmt)
    prod = np.repeat(S, 64, axis=1) * q.astype(np.float32)        # fl32 products
    want = torch.from_numpy(prod).to(tdt).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(got, want)


@pytest.mark.parametrize("fmt", ["bf16", "f16"])
def test_linear_w4a16_matches_fp64_matmul(fmt):
    rng = np.random.default_rng(10)
    m, n, k, g = 7, 48, 384, 128
    x = O.widen16(O.round16(rng.standard_normal((m, k)).astype(np.float32), fmt), fmt)
    w = (rng.standard_normal((n, k)) * 0.02).astype(np.float32)
    q, S = O.quant_weight_group(w, g)
    bias = rng.standard_normal(n).astype(np.float32)
    y0, _ = O.linear_w4a16(x, q, S, g, fmt)
    y, Y = O.linear_w4a16(x, q, S, g, fmt, bias=bias)
    wd = O.widen16(O.dequant_group16(q, S, g, fmt), fmt).astype(np.float64)
    ref = (x.astype(np.float64) @ wd.T).astype(np.float32)
    ulp = np.spacing(np.abs(ref)).astype(np.float64)
    assert np.all(np.abs(y0.astype(np.float64) - ref) <= ulp)
    assert np.array_equal(y, (y0 + bias[None, :]).astype(np.float32))
    assert np.array_equal(Y, O.round16(y, "bf16"))
    # selecting rows and columns picks the same values
    ys, _ = O.linear_w4a16(x, q, S, g, fmt, bias=bias, rows=[6, 0], cols=[47, 3, 5])
    assert np.array_equal(ys, y[[6, 0]][:, [47, 3, 5]])


# ------------------------------------------------------------------ Q4_K two-level scales

def test_q4k_page_example_super_scale():
    # The page's three sub-blocks (4 values each, padded with zeros to the
    # 32-value sub-blocks of Q4_K; zeros leave each absmax unchanged) and five
    # empty sub-blocks make one 256-value super block.
    g = _golden("worked_examples_4bit.json")["q4k_sub_blocks"]
    w = np.zeros((1, 256), np.float32)
    for j, blk in enumerate(g["blocks"]):
        w[0, 32 * j:32 * j + 4] = blk
    r = O.quant_weight_q4k(w)
    assert np.allclose(r["s_sub"][0, :3], g["scales_printed"], atol=0.0006)
    assert abs(float(r["s_super"][0, 0]) - g["super_scale_printed"]) < 5e-5
    assert r["q_sub"][0].tolist() == [5, 15, 1, 0, 0, 0, 0, 0]      # 0.457/0.0857, 15, 0.071/0.0857
    for j, codes in enumerate(g["codes_by_rule"]):
        assert r["q"][0, 32 * j:32 * j + 4].tolist() == codes


def test_q4k_invariants_and_nearest_sub_codes():
    rng = np.random.default_rng(11)
    w = (rng.standard_normal((12, 512)) * 0.02).astype(np.float32)
    w[:, 40:72] *= np.float32(8.0)                  # uneven sub-block ranges
    r = O.quant_weight_q4k(w)
    q32, S32 = O.quant_weight_group(w, 32)
    assert np.array_equal(r["q"], q32) and np.array_equal(r["s_sub"], S32)
    ss = r["s_sub"].reshape(12, 2, 8)
    sup = r["s_super"]
    assert np.array_equal(sup, (ss.max(axis=2) / np.float32(15)).astype(np.float32))
    qs = r["q_sub"].reshape(12, 2, 8)
    assert qs.max() <= 15
    top = np.take_along_axis(qs, ss.argmax(axis=2)[..., None], 2)[..., 0]
    assert np.all(top == 15)
    for i in range(12):
        for b in range(2):
            s = Fraction(float(sup[i, b]))
            for j in range(8):
                t = Fraction(float(ss[i, b, j])) / s
                best = min(range(16), key=lambda c: (abs(t - c), c % 2))
                assert qs[i, b, j] == best
    eff = r["S_eff"].reshape(12, 2, 8).astype(np.float64)
    assert np.all(np.abs(eff - ss) <= sup[..., None] * (0.5 + 2.0 ** -20))
    assert np.array_equal(eff, (sup[..., None] * qs.astype(np.float32)).astype(np.float64))


def test_q4k_all_zero_super_block():
    # Every sub-block at the eps floor: s_super = 1e-8 / 15, every sub-scale
    # code 15, so the effective scale is the floor again; codes are 0.
    w = np.zeros((2, 512), np.float32)
    w[1, 300] = 0.5                               # second super block of row 1 is not empty
    r = O.quant_weight_q4k(w)
    assert np.all(r["q"][0] == 0)
    assert np.all(r["s_super"][0] == np.float32(np.float32(1e-8) / np.float32(15)))
    assert np.all(r["q_sub"][0] == 15)
    assert np.all(np.abs(r["S_eff"][0] - np.float32(1e-8)) <= np.float32(1e-8) * 2.0 ** -22)
    # row 1: block 0 empty as above; block 1 holds 0.5 in sub-block 1 (values 288..319)
    assert r["q"][1, 300] == 7 and r["q_sub"][1, 9] == 15
    assert np.all(r["q_sub"][1, 8:16][[0, 2, 3, 4, 5, 6, 7]] == 0)
