"""Helpers shared by the GPU parity tests: seeded inputs, oracle references and
the comparison rules.

Comparison rules
  * codes, scales, zero points, row sums, outlier masks/indices/counts and
    INT32 accumulators: bit-exact;
  * INT8 W8A8 bf16 outputs: bit-exact (the epilogue's fp32 steps are the
    oracle's, in the same order), which is inside the 2-ulp contract;
  * FP8 and LLM.int8 outputs (fp32 accumulation order differs between the
    tensor cores and the oracle's double sum):
        |Y - y_ref| <= 2 ulp_bf16(y_ref) + K_acc 2^-22 (|A| |B|^T)[m, n] * scales
    where K_acc is the fp32-accumulated depth.
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
