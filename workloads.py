"""Seeded synthetic workloads for the 8-bit quantized linear layer.

This module only draws random inputs.  It holds none of the quantization
arithmetic, so both the CPU oracle and the CUDA path can take their inputs from
it without sharing any of the method's code.

Every draw uses a CPU ``torch.Generator`` seeded with 0, in a fixed order:
X first, then W, then the structure draws (outlier columns, heavy tails).
Values are drawn in fp32 and cast once to the workload's 16-bit dtype.

The value structure follows the pages:
  * hidden states are mostly regular, about N(0, 1) (|x| within ~3.5), and a
    few systematic outlier feature columns sit in [-60, -6] U [6, 60]
    (bitsandbytes LLM.int8 page, "核心思想" section);
  * weights are small, N(0, 0.02), sized like Llama-3-8B's q_proj (4096x4096)
    and FFN up projection (14336x4096) (8-Bit LLM Quantization with Lightning
    Fabric, section 2.1).
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    kind: str            # "int8_mixed" | "w8a8_int8" | "w8a8_fp8"
    m: int
    n: int
    k: int
    x_dtype: torch.dtype
    w_dtype: torch.dtype
    weight_scheme: str   # "asym" | "sym" | "fp8"
    weight_codes: str    # "s8" | "u8" | "e4m3"
    threshold: float = 6.0
    clip_ub: float = 0.0
    description: str = ""


WORKLOADS = {
    "tiny_mixed": Workload(
        "tiny_mixed", "int8_mixed", 16, 256, 256, torch.float16, torch.float16,
        "asym", "s8", threshold=6.0,
        description="LLM.int8 linear 16x256x256 fp16, outlier columns 3 and 77"),
    "decode_q_proj": Workload(
        "decode_q_proj", "w8a8_int8", 16, 4096, 4096, torch.bfloat16, torch.bfloat16,
        "asym", "u8",
        description="q_proj-shaped decode W8A8: 16 tokens x 4096 -> 4096, asymmetric uint8 weights"),
    "prefill_ffn_up": Workload(
        "prefill_ffn_up", "w8a8_int8", 2048, 14336, 4096, torch.bfloat16, torch.bfloat16,
        "sym", "s8",
        description="prefill FFN-up W8A8 INT8: 2048 tokens x 4096 -> 14336, symmetric weights"),
    "mixed_512": Workload(
        "mixed_512", "int8_mixed", 512, 4096, 4096, torch.float16, torch.float16,
        "asym", "s8", threshold=6.0,
        description="LLM.int8 mixed decomposition 512x4096x4096 fp16, 6 outlier columns"),
    "fp8_rowwise": Workload(
        "fp8_rowwise", "w8a8_fp8", 4096, 8192, 8192, torch.bfloat16, torch.bfloat16,
        "fp8", "e4m3", clip_ub=1200.0,
        description="FP8 e4m3 rowwise W8A8 4096x8192x8192, activation clip 1200"),
}

ORDER = ["tiny_mixed", "decode_q_proj", "prefill_ffn_up", "mixed_512", "fp8_rowwise"]


def _outlier_values(g: torch.Generator, shape) -> torch.Tensor:
    mag = torch.empty(shape).uniform_(6.0, 60.0, generator=g)
    sign = torch.randint(0, 2, shape, generator=g).float() * 2.0 - 1.0
    return mag * sign


def make_inputs(name: str, seed: int = 0, m: Optional[int] = None,
                n: Optional[int] = None, k: Optional[int] = None):
    """Return (X, W, info) for a named workload as CPU tensors in its dtypes.

    ``m``, ``n`` and ``k`` override the sizes (same recipe, other shapes);
    ``info`` records the planted structure (outlier columns, if any).
    """
    w = WORKLOADS[name]
    m = w.m if m is None else m
    n = w.n if n is None else n
    k = w.k if k is None else k
    g = torch.Generator().manual_seed(seed)
    X = torch.randn(m, k, generator=g)
    W = torch.randn(n, k, generator=g) * 0.02
    info = {}
    if name == "tiny_mixed":
        cols = [c for c in (3, 77) if c < k]
        X[:, cols] = _outlier_values(g, (m, len(cols)))
        info["planted_columns"] = cols
    elif name == "mixed_512":
        cols = torch.randperm(k, generator=g)[:6].tolist()
        X[:, cols] = _outlier_values(g, (m, len(cols)))
        info["planted_columns"] = sorted(cols)
    elif name == "decode_q_proj":
        heavy = torch.rand(n, k, generator=g) < 0.01
        W = torch.where(heavy, torch.randn(n, k, generator=g) * 0.2, W)
    elif name == "fp8_rowwise":
        spikes = torch.rand(m, k, generator=g) < 0.001
        X = torch.where(spikes, X * 100.0, X)
    return X.to(w.x_dtype), W.to(w.w_dtype), info


def random_matrix(rows: int, cols: int, dtype: torch.dtype, seed: int,
                  std: float = 1.0) -> torch.Tensor:
    """A seeded N(0, std) matrix, for edge-case shapes in the tests."""
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(rows, cols, generator=g) * std).to(dtype)


def bits16(t: torch.Tensor):
    """The raw 16-bit patterns of an fp16/bf16 CPU tensor as a uint16 numpy array."""
    import numpy as np
    assert t.dtype in (torch.float16, torch.bfloat16)
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


# ---------------------------------------------------------------- exact-arithmetic inputs
#
# Inputs whose products and partial sums are all exactly representable in
# fp32, so that any summation order gives the same accumulator.  They carry
# no quantization arithmetic: small integers, powers of two, and weights laid
# on a grid whose per-row (or per-group) range is fixed by construction.

def small_int_matrix(rows: int, cols: int, seed: int, lim: int) -> torch.Tensor:
    """Seeded fp32 matrix of integers drawn uniformly from [-lim, lim]."""
    g = torch.Generator().manual_seed(seed)
    return torch.randint(-lim, lim + 1, (rows, cols), generator=g).float()


def pow2_vector(n: int, seed: int, lo: int, hi: int) -> torch.Tensor:
    """Seeded fp32 vector of powers of two 2^e, e drawn uniformly from [lo, hi)."""
    g = torch.Generator().manual_seed(seed)
    return torch.exp2(torch.randint(lo, hi, (n,), generator=g).float())


def grid_rows(rows: int, cols: int, seed: int, step_exp: int) -> torch.Tensor:
    """Rows of integers in [-128, 127] times 2^step_exp, each row holding both
    -128 and 127 (at seeded positions), so every row spans exactly 255 grid
    steps."""
    g = torch.Generator().manual_seed(seed)
    v = torch.randint(-128, 128, (rows, cols), generator=g)
    perm = torch.argsort(torch.rand(rows, cols, generator=g), dim=1)
    r = torch.arange(rows)
    v[r, perm[:, 0]] = -128
    v[r, perm[:, 1]] = 127
    return v.float() * 2.0 ** step_exp


def group_grid(rows: int, cols: int, group: int, seed: int, lo: int, hi: int) -> torch.Tensor:
    """Each run of `group` consecutive values along a row is 2^e times integers
    in [-7, 7] (e drawn from [lo, hi) per run), and holds +-7 * 2^e at a seeded
    position, so the run's absolute maximum is exactly 7 * 2^e."""
    assert cols % group == 0
    g = torch.Generator().manual_seed(seed)
    v = torch.randint(-7, 8, (rows, cols // group, group), generator=g).float()
    e = torch.randint(lo, hi, (rows, cols // group, 1), generator=g).float()
    pos = torch.randint(0, group, (rows, cols // group), generator=g)
    sign = torch.randint(0, 2, (rows, cols // group), generator=g).float() * 2 - 1
    v.scatter_(2, pos.unsqueeze(2), (7 * sign).unsqueeze(2))
    return (v * torch.exp2(e)).reshape(rows, cols)
