"""Pins for the oracle's grouped (mixture-of-experts) FP8 rowwise linear.

Transformers FP8 / FBGEMM page, 5.4: one FP8 weight block with per-row scales
per expert, each expert's tokens multiplied on their own.  The checks use
torch's float8_e4m3fn decoding and numpy's fp64 matmul for the products, so
they test which expert block each token meets, independently of the
oracle's C routines.
"""
import numpy as np
import torch

from oracle import oracle as O


def _decode(codes: np.ndarray) -> np.ndarray:
    return torch.from_numpy(codes).view(torch.float8_e4m3fn).float().numpy().astype(np.float64)


def _case(seed=3, E=4, n=16, k=64, counts=(5, 0, 7, 2)):
    rng = np.random.default_rng(seed)
    m = sum(counts)
    x = rng.standard_normal((m, k)).astype(np.float32)
    w = (rng.standard_normal((E * n, k)) * 0.05).astype(np.float32)
    xq, Sx = O.quant_act_fp8(x, 0.0)
    wq, Sw, _ = O.quant_weight(w, "fp8")
    off = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    return xq, Sx, wq, Sw, off, n


def test_each_token_meets_its_own_expert():
    xq, Sx, wq, Sw, off, n = _case()
    bias = np.arange(4 * n, dtype=np.float32) * np.float32(0.01)
    y, Y = O.linear_moe_fp8(xq, Sx, wq, Sw, off, n, bias=bias)
    X = _decode(xq)
    Wd = _decode(wq)
    for e in range(len(off) - 1):
        for m in range(off[e], off[e + 1]):
            acc = (X[m] @ Wd[e * n:(e + 1) * n].T).astype(np.float32)
            ref = (acc * Sx[m]).astype(np.float32) * Sw[e * n:(e + 1) * n]
            ref = ref.astype(np.float32) + bias[e * n:(e + 1) * n]
            ulp = np.spacing(np.abs(ref.astype(np.float32)))
            assert np.all(np.abs(y[m] - ref) <= 2 * ulp), (e, m)
    assert np.array_equal(Y, O.round16(y, "bf16"))


def test_reordering_experts_reorders_outputs():
    xq, Sx, wq, Sw, off, n = _case(seed=4)
    y, _ = O.linear_moe_fp8(xq, Sx, wq, Sw, off, n)
    # swap experts 0 and 2 together with their tokens
    order = [2, 1, 0, 3]
    rows = np.concatenate([np.arange(off[e], off[e + 1]) for e in order])
    wrows = np.concatenate([np.arange(e * n, (e + 1) * n) for e in order])
    cnt = [off[e + 1] - off[e] for e in order]
    off2 = np.concatenate([[0], np.cumsum(cnt)]).astype(np.int32)
    y2, _ = O.linear_moe_fp8(xq[rows], Sx[rows], wq[wrows], Sw[wrows], off2, n)
    assert np.array_equal(y2, y[rows])


def test_single_expert_is_the_dense_linear_and_rows_select():
    xq, Sx, wq, Sw, off, n = _case(seed=5, E=1, counts=(9,))
    y, _ = O.linear_moe_fp8(xq, Sx, wq, Sw, off, n)
    _, yd, _ = O.linear_w8a8_fp8(xq, Sx, wq, Sw)
    assert np.array_equal(y, yd)
    xq, Sx, wq, Sw, off, n = _case(seed=6)
    y, _ = O.linear_moe_fp8(xq, Sx, wq, Sw, off, n)
    ys, _ = O.linear_moe_fp8(xq, Sx, wq, Sw, off, n, rows=[13, 0, 6])
    assert np.array_equal(ys, y[[13, 0, 6]])


def test_zero_expert_weight_gives_bias_only():
    xq, Sx, wq, Sw, off, n = _case(seed=7)
    wq = wq.copy()
    wq[2 * n:3 * n] = 0                           # expert 2: e4m3 zeros
    bias = np.full(4 * n, np.float32(0.25))
    y, _ = O.linear_moe_fp8(xq, Sx, wq, Sw, off, n, bias=bias)
    assert np.all(y[off[2]:off[3]] == np.float32(0.25))
