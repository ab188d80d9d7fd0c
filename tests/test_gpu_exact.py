"""Exact-arithmetic parity of the fp32-accumulated paths, compared bit for bit.

The tensor cores add into an fp32 accumulator in their own order, so on
general inputs the FP8, LLM.int8 outlier, W4A16 and grouped FP8 accumulators
can only be compared with the oracle's once-rounded double sum within a
bound.  A dropped, duplicated or misplaced K slice can hide inside such a
bound.  These cases choose operands whose products and partial sums are all
exactly representable in fp32 (small integers, weights on a power-of-two
grid, power-of-two scales), so every summation order gives the same result:
accumulators and bf16 outputs must equal the oracle's bit for bit, at the full
K of the workloads and with M spanning several tiles.  A missing or repeated
slice changes an integer sum and fails.

Pages: FP8 rowwise linear, "Transformers FP8 (W8A8) 量化实战：基于 FBGEMM"
section 5.3 (f8f8bf16_rowwise) and 5.4 (Llama4 experts); the LLM.int8 outlier
stream, the bitsandbytes LLM.int8 page, 核心思想; group-wise 4-bit weights,
the "大模型量化技术" overview section 2.2 and "大模型量化" (Xilyfe) GGUF section.
"""
import numpy as np
import pytest
import torch

import workloads
from oracle import oracle as O
from tests import parity as P

pytestmark = pytest.mark.gpu

from bit_quantized_b200 import q8  # noqa: E402

DEV = "cuda:0"


def _e4m3_codes(values: torch.Tensor) -> np.ndarray:
    """e4m3 codes of small integers (exactly representable), via the oracle."""
    v = values.numpy().astype(np.float32)
    c = O.round_e4m3(v)
    assert np.array_equal(O.widen_e4m3(c), v)
    return c


def _dev_e4m3(codes: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(codes).to(DEV).view(torch.float8_e4m3fn)


def _fp8_operands(m, n, k, seed):
    xq = _e4m3_codes(workloads.small_int_matrix(m, k, seed, 4))
    wq = _e4m3_codes(workloads.small_int_matrix(n, k, seed + 1, 4))
    Sx = workloads.pow2_vector(m, seed + 2, -9, -3).numpy()
    Sw = workloads.pow2_vector(n, seed + 3, -12, -6).numpy()
    return xq, wq, Sx, Sw


# ------------------------------------------------------------------ dense FP8

@pytest.mark.parametrize("m,n,k", [
    (4096, 8192, 8192),     # the FP8 rowwise workload's shape and launch configuration
    (640, 1280, 8192),      # 5 x 5 tiles of 128 x 256 (fewer tiles than SMs)
    (300, 2000, 4096),      # ragged M and N tails
    (16, 4096, 8192),       # decode kernel: K split over a cluster
    (48, 1024, 8192),       # decode kernel, 64-token tile, ragged
])
def test_fp8_exact(m, n, k):
    xq, wq, Sx, Sw = _fp8_operands(m, n, k, seed=m + n + k)
    qa = q8.QAct(_dev_e4m3(xq), torch.from_numpy(Sx).to(DEV), None, q8.Q8_E4M3)
    qw = q8.QWeight(_dev_e4m3(wq), torch.from_numpy(Sw).to(DEV), None, q8.Q8_E4M3)
    acc = torch.empty((m, n), dtype=torch.float32, device=DEV)
    Y = q8.q8_linear_w8a8(qa, qw, acc_debug=acc)
    torch.cuda.synchronize()
    assert q8.q8_get_device_status() == 0
    acc_ref, y_ref, Y_ref = O.linear_w8a8_fp8(xq, Sx, wq, Sw)
    P.assert_equal(acc.cpu().numpy().view(np.uint32), acc_ref.view(np.uint32), f"fp8 {m}x{n}x{k} acc")
    P.assert_equal(P.bf16_bits(Y), Y_ref, f"fp8 {m}x{n}x{k} Y")


# ------------------------------------------------------------------ grouped FP8 (MoE)

@pytest.mark.parametrize("counts,n,k", [
    ((130, 0, 7, 300, 64), 256, 8192),          # empty and sub-tile experts, straddling tiles
    ((600, 520, 300, 700), 512, 4096),          # several tiles per expert
])
def test_grouped_fp8_exact(counts, n, k):
    E, m = len(counts), int(sum(counts))
    xq, wq, Sx, Sw = _fp8_operands(m, E * n, k, seed=m + n)
    off = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    qa = q8.QAct(_dev_e4m3(xq), torch.from_numpy(Sx).to(DEV), None, q8.Q8_E4M3)
    qw = q8.QWeight(_dev_e4m3(wq), torch.from_numpy(Sw).to(DEV), None, q8.Q8_E4M3)
    Y = q8.q8_linear_fp8_grouped(qa, qw, E, torch.from_numpy(off).to(DEV))
    torch.cuda.synchronize()
    assert q8.q8_get_device_status() == 0
    _, Y_ref = O.linear_moe_fp8(xq, Sx, wq, Sw, off, n)
    P.assert_equal(P.bf16_bits(Y), Y_ref, f"grouped fp8 {counts} Y")


# ------------------------------------------------------------------ LLM.int8 outlier stream

@pytest.mark.parametrize("fp16_weight", [False, True])
def test_mixed_outlier_stream_exact(fp16_weight):
    # 512 x 1024 x 4096 (4 x 8 tiles): 100 integer-valued outlier columns (two
    # fp16 K blocks of 64, the second half padding), regular columns below the
    # threshold; weights on a 2^-6 grid spanning exactly 255 steps per row, so
    # S = 2^-6, Z = 0 and the dequantized fp16 weight equals the weight.
    m, n, k = 512, 1024, 4096
    g = torch.Generator().manual_seed(77)
    X = workloads.random_matrix(m, k, torch.float32, 78).clamp_(-5.5, 5.5)
    cols = torch.randperm(k, generator=g)[:100]
    Xo = workloads.small_int_matrix(m, 100, 79, 40)
    Xo[0] = torch.where(Xo[0] >= 0, Xo[0].clamp(min=7), Xo[0].clamp(max=-7))
    X[:, cols] = Xo
    X16 = X.to(torch.float16)
    W16 = workloads.grid_rows(n, k, 80, -6).to(torch.float16)
    x32, w32 = P.host_f32(X16), P.host_f32(W16)
    bias = workloads.pow2_vector(n, 81, -4, 0).numpy()
    Wd = W16.to(DEV)
    qw = q8.q8_quantize_weight(Wd, "asym", "s8")
    Y, dbg = q8.q8_linear_int8_mixed(X16.to(DEV), qw, 6.0, W16=Wd if fp16_weight else None,
                                     bias=torch.from_numpy(bias).to(DEV), debug=True)
    torch.cuda.synchronize()
    assert q8.q8_get_device_status() == 0
    wq, Sw, Zw = O.quant_weight(w32, "asym", "s8")
    assert np.all(Sw == 2.0**-6) and np.all(Zw == 0)
    ref = O.linear_int8_mixed(x32, wq, Sw, Zw, 6.0, w16_full=w32 if fp16_weight else None,
                              bias=bias)
    assert ref["count"] == 100
    what = f"mixed exact fp16_weight={fp16_weight}"
    P.assert_equal(dbg["mask"].cpu().numpy(), ref["mask"], what + " mask")
    P.assert_equal(dbg["acc"].cpu().numpy(), ref["acc"].astype(np.int32), what + " acc")
    P.assert_equal(dbg["y16"].cpu().numpy().view(np.uint32), ref["y16"].view(np.uint32), what + " y16")
    P.assert_equal(P.bf16_bits(Y), ref["Y"], what + " Y")


# ------------------------------------------------------------------ W4A16

@pytest.mark.parametrize("m,n,k,g", [
    (16, 1024, 4096, 128),     # decode: K split over a cluster
    (300, 512, 4096, 64),      # two 256-token tiles, ragged
    (16, 128, 8192, 128),      # 16 K slices per split CTA: staging rings wrap
    (1, 256, 4096, 32),
])
def test_w4a16_exact(m, n, k, g):
    # Each group of g weights is 2^e times integers in [-7, 7] with |max| = 7 * 2^e,
    # so S = 2^e, the codes are the integers and the 16-bit weight is exact;
    # activations are small integers.
    W = workloads.group_grid(n, k, g, seed=m + n, lo=-9, hi=-4).to(torch.bfloat16)
    X = workloads.small_int_matrix(m, k, m + n + 1, 8).to(torch.bfloat16)
    w32, x32 = P.host_f32(W), P.host_f32(X)
    qw = q8.q8_quantize_weight_g4(W.to(DEV), g)
    Y = q8.q8_linear_w4a16(X.to(DEV), qw)
    torch.cuda.synchronize()
    assert q8.q8_get_device_status() == 0
    q_ref, S_ref = O.quant_weight_group(w32, g)
    assert np.all(np.log2(S_ref) == np.round(np.log2(S_ref)))
    _, Y_ref = O.linear_w4a16(x32, q_ref, S_ref, g, "bf16")
    P.assert_equal(P.bf16_bits(Y), Y_ref, f"w4a16 exact {m}x{n}x{k} g{g}")
