"""Helpers shared by the GPU parity tests: seeded inputs, oracle references and
the comparison rules.

Comparison rules
  * codes, scales, zero points, row sums, outlier masks/indices/counts and
    INT32 accumulators: bit-exact;
  * INT8 W8A8 bf16 outputs: bit-exact (the epilogue's fp32 steps are the
    oracle's, in the same order), which is inside the 2-ulp contract;
  * fp32-accumulated outputs (FP8, the LLM.int8 outlier stream, W4A16, the
    grouped FP8 linear): the tensor cores add into the fp32 accumulator once
    per MMA instruction, a K step of 32 products for 8-bit operands and 16 for
    16-bit ones, where the oracle sums every product in double and rounds
    once.  With mag = (|A| |B|^T)[m, n] and n_add = ceil(K_acc / k_step) + 8
    roundings (8 more for a split-K reduction), each erring by at most 2^-24
    of a partial sum no larger than mag, plus as much again for the rounding
    inside one MMA's dot product:
        |acc - acc_ref| <= n_add 2^-23 mag                 (accumulation_bound)
    On the output the contract is 2 bf16 ulp of the oracle's fp32 result.
    Where that accumulation term (times the scales) is at most one bf16 ulp
    of y_ref, it holds as it stands (a rounding of y within 1 ulp, then bf16's
    half ulp); where it is larger, y_ref lies in a cancellation (|y| far below
    the magnitude of its products) and the term is added:
        |Y - y_ref| <= 2 ulp_bf16(y_ref) + 4 2^-24 |y_ref|  [+ term, cancellation only]
    check_fp_output reports the maximum error in ulps, the share of outputs
    beyond 2 ulp and the share that needed the cancellation term.
  * Exact-arithmetic inputs (tests/test_gpu_exact.py): small-integer operands
    and power-of-two scales make every partial sum exact in fp32 in any order,
    so accumulators and outputs are compared bit for bit at full K.
"""
from __future__ import annotations

import functools

import numpy as np
import torch

import workloads
from oracle import oracle as O

FMT = {torch.float16: "f16", torch.bfloat16: "bf16"}


def host_f32(t: torch.Tensor) -> np.ndarray:
    """Exact fp32 values of a CPU fp16/bf16/fp32 tensor, decoded by the oracle."""
    if t.dtype == torch.float32:
        return t.numpy().astype(np.float32)
    return O.widen16(workloads.bits16(t), FMT[t.dtype])


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def f32(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().numpy().astype(np.float32)


def codes_u8(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().view(torch.uint8).numpy()


def bf16_ulp(y: np.ndarray) -> np.ndarray:
    """Spacing of bf16 numbers at |y| (normal range), 2^(floor(log2|y|) - 7)."""
    a = np.abs(y.astype(np.float64))
    a = np.maximum(a, 2.0**-126)
    return np.exp2(np.floor(np.log2(a)) - 7)


def bf16_values(bits: np.ndarray) -> np.ndarray:
    return O.widen16(bits, "bf16").astype(np.float64)


def assert_bf16_within(Y_bits: np.ndarray, y_ref: np.ndarray, extra: np.ndarray | float = 0.0,
                       what: str = "") -> float:
    """Checks |Y - y_ref| <= 2 ulp_bf16(y_ref) + extra; returns the max error in ulps."""
    got = bf16_values(Y_bits)
    err = np.abs(got - y_ref.astype(np.float64))
    bound = 2 * bf16_ulp(y_ref) + extra
    bad = err > bound
    if bad.any():
        i = np.argwhere(bad)[0]
        raise AssertionError(f"{what}: {bad.sum()} outputs outside the bound; first at {i.tolist()}: "
                             f"got {got[tuple(i)]!r} ref {y_ref[tuple(i)]!r} bound {np.broadcast_to(bound, err.shape)[tuple(i)]!r}")
    return float((err / bf16_ulp(y_ref)).max(initial=0.0))


def accumulation_bound(mag: np.ndarray, k_acc: int, k_step: int = 32) -> np.ndarray:
    """Bound of |acc - acc_ref| for an fp32 tensor-core accumulation of k_acc
    products with sum of magnitudes `mag` (see the module docstring)."""
    n_add = -(-int(k_acc) // int(k_step)) + 8
    return n_add * 2.0**-23 * np.asarray(mag, np.float64)


def check_fp_acc(acc: np.ndarray, acc_ref: np.ndarray, mag: np.ndarray, k_acc: int,
                 k_step: int, what: str) -> float:
    """Asserts the accumulation bound on an fp32 accumulator; returns the
    largest error in units of 2^-24 mag (the per-rounding error scale)."""
    acc = np.asarray(acc, np.float64)
    ref = np.asarray(acc_ref, np.float64)
    err = np.abs(acc - ref)
    bound = accumulation_bound(mag, k_acc, k_step) + 2.0**-24 * np.abs(ref)
    bad = err > bound
    if bad.any():
        i = tuple(np.argwhere(bad)[0])
        raise AssertionError(f"{what}: {int(bad.sum())} accumulators outside the bound; first at "
                             f"{list(i)}: got {acc[i]!r} ref {ref[i]!r} bound {bound[i]!r}")
    unit = 2.0**-24 * np.maximum(np.asarray(mag, np.float64), 1e-300)
    ratio = float((err / unit).max(initial=0.0))
    print(f"[parity] {what}: accumulator error max {ratio:.2f} x 2^-24 mag "
          f"(bound {-(-int(k_acc) // int(k_step)) + 8} x 2^-23 mag)")
    return ratio


def check_fp_output(Y_bits: np.ndarray, y_ref: np.ndarray, term: np.ndarray | float,
                    what: str) -> dict:
    """The 2-ulp output contract with the cancellation rule of the module
    docstring.  `term` is the accumulation bound already multiplied by the
    output's scales.  Returns and prints the error statistics."""
    got = bf16_values(Y_bits)
    yr = np.asarray(y_ref, np.float64)
    ulp = bf16_ulp(yr)
    err = np.abs(got - yr)
    term = np.broadcast_to(np.asarray(term, np.float64), err.shape)
    cancel = term > ulp
    bound = 2 * ulp + 4 * 2.0**-24 * np.abs(yr) + np.where(cancel, term, 0.0)
    bad = err > bound
    if bad.any():
        i = tuple(np.argwhere(bad)[0])
        raise AssertionError(f"{what}: {int(bad.sum())} outputs outside the bound; first at "
                             f"{list(i)}: got {got[i]!r} ref {yr[i]!r} bound {bound[i]!r}"
                             f" (cancellation term {'on' if cancel[i] else 'off'})")
    e_ulp = err / ulp
    stats = {"max_ulp": float(e_ulp.max(initial=0.0)),
             "max_ulp_outside_cancellation": float(e_ulp[~cancel].max(initial=0.0)),
             "frac_beyond_2ulp": float((e_ulp > 2.0).mean()) if e_ulp.size else 0.0,
             "frac_cancellation": float(cancel.mean()) if cancel.size else 0.0,
             "outputs": int(e_ulp.size)}
    print(f"[parity] {what}: max {stats['max_ulp']:.3f} ulp, "
          f"{stats['max_ulp_outside_cancellation']:.3f} ulp outside cancellation, "
          f"{100 * stats['frac_beyond_2ulp']:.4f}% beyond 2 ulp, "
          f"{100 * stats['frac_cancellation']:.4f}% in cancellation, {stats['outputs']} outputs")
    return stats


def assert_equal(a: np.ndarray, b: np.ndarray, what: str) -> None:
    a = np.asarray(a)
    b = np.asarray(b)
    assert a.shape == b.shape, f"{what}: shape {a.shape} vs {b.shape}"
    if not np.array_equal(a, b):
        diff = np.argwhere(a != b)
        i = tuple(diff[0])
        raise AssertionError(f"{what}: {len(diff)} mismatches; first at {list(i)}: {a[i]!r} vs {b[i]!r}")


@functools.lru_cache(maxsize=8)
def workload(name: str):
    """CPU inputs of a named workload plus their exact fp32 values."""
    X, W, info = workloads.make_inputs(name)
    return X, W, info, host_f32(X), host_f32(W)


def sample_indices(size: int, count: int, seed: int) -> np.ndarray:
    """Sorted sample of indices that always includes both ends."""
    if count >= size:
        return np.arange(size, dtype=np.int64)
    rng = np.random.default_rng(seed)
    pick = rng.choice(size, count - 2, replace=False)
    return np.unique(np.concatenate([[0, size - 1], pick])).astype(np.int64)
