"""Pins for the oracle's float-format conversions.

The oracle decodes and rounds fp16, bf16 and FP8 E4M3 from the formats'
definitions.  Here each conversion is checked against an independent library
routine (numpy's float16 casts, torch's bfloat16 and float8_e4m3fn casts), over
every bit pattern where that is cheap and on seeded values and exact ties
otherwise.
"""
import numpy as np
import pytest
import torch

from oracle import oracle as O

ALL16 = np.arange(65536, dtype=np.uint32).astype(np.uint16)


def test_widen_f16_all_patterns():
    got = O.widen16(ALL16, "f16")
    ref = ALL16.view(np.float16).astype(np.float32)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan].view(np.uint32), ref[~nan].view(np.uint32))


def test_widen_bf16_all_patterns():
    got = O.widen16(ALL16, "bf16")
    ref = torch.from_numpy(ALL16.view(np.int16)).view(torch.bfloat16).float().numpy()
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan].view(np.uint32), ref[~nan].view(np.uint32))


def _probe_values(seed, n=200000):
    rng = np.random.default_rng(seed)
    mags = np.exp2(rng.uniform(-30, 20, n)).astype(np.float32)
    sgn = np.where(rng.random(n) < 0.5, -1.0, 1.0).astype(np.float32)
    return mags * sgn


def _midpoints(values: np.ndarray) -> np.ndarray:
    """Exact midpoints between consecutive finite values, as fp32 when exact."""
    v = np.unique(values[np.isfinite(values)].astype(np.float64))
    mid = (v[1:] + v[:-1]) / 2
    mid32 = mid.astype(np.float32)
    return mid32[mid32.astype(np.float64) == mid]


def test_round_f16_matches_numpy():
    x = np.concatenate([_probe_values(1), np.float32([0.0, -0.0, 65504, 65519.996, 65520,
                                                      1e6, -1e6, 2.0**-25, 2.0**-24, 3e-8])])
    f16_vals = ALL16.view(np.float16).astype(np.float32)
    x = np.concatenate([x, _midpoints(f16_vals)])
    got = O.round16(x, "f16")
    ref = x.astype(np.float16).view(np.uint16)
    assert np.array_equal(got, ref)


def test_round_bf16_matches_torch():
    x = np.concatenate([_probe_values(2), np.float32([0.0, -0.0, 3.389e38, 3.4e38, -3.4e38])])
    bf_vals = torch.from_numpy(ALL16.view(np.int16)).view(torch.bfloat16).float().numpy()
    x = np.concatenate([x, _midpoints(bf_vals)])
    got = O.round16(x, "bf16")
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(got, ref)


def test_bf16_ties_go_to_even():
    # 1 + 2^-8 lies halfway between bf16 1.0 (0x3F80) and 1 + 2^-7 (0x3F81).
    x = np.float32([1.0 + 2.0**-8, 1.0 + 3 * 2.0**-8])
    assert O.round16(x, "bf16").tolist() == [0x3F80, 0x3F82]


E4M3_CODES = np.arange(256, dtype=np.uint8)


def _torch_e4m3_values():
    return torch.from_numpy(E4M3_CODES.view(np.int8)).view(torch.float8_e4m3fn).float().numpy()


def test_widen_e4m3_all_codes():
    got = O.widen_e4m3(E4M3_CODES)
    ref = _torch_e4m3_values()
    nan = np.isnan(ref)
    assert nan.sum() == 2  # 0x7F and 0xFF
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])
    assert got[0x7E] == 448.0 and got[0x01] == 2.0**-9


def test_round_e4m3_in_range_matches_torch():
    x = _probe_values(3) / np.float32(2.0**8)
    x = x[np.abs(x) <= 448]
    # every finite fp16 and bf16 pattern inside the E4M3 range, plus exact ties
    f16 = ALL16.view(np.float16).astype(np.float32)
    bf = torch.from_numpy(ALL16.view(np.int16)).view(torch.bfloat16).float().numpy()
    pool = np.concatenate([x, f16, bf, _midpoints(_torch_e4m3_values())])
    pool = pool[np.isfinite(pool) & (np.abs(pool) <= 448)]
    got = O.round_e4m3(pool)
    ref = torch.from_numpy(pool).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(got, ref)


def test_round_e4m3_saturates():
    x = np.float32([448.0, 463.99, 464.0, 480.0, 1e4, 3e38, -500.0, -1e30])
    got = O.round_e4m3(x)
    assert got.tolist() == [0x7E, 0x7E, 0x7E, 0x7E, 0x7E, 0x7E, 0xFE, 0xFE]


def test_round_e4m3_subnormal_ties():
    # 2^-10 is halfway between 0 and the smallest subnormal 2^-9: ties to even -> 0.
    x = np.float32([2.0**-10, 3 * 2.0**-10, 2.0**-10 * 1.0001, -(2.0**-10)])
    assert O.round_e4m3(x).tolist() == [0x00, 0x02, 0x01, 0x80]
