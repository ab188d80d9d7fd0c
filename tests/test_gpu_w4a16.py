"""GPU parity of the group-wise 4-bit weight quantizer and the W4A16 linear.

Codes and scales are compared bit for bit with the oracle.  Outputs are
compared with the oracle's double-accumulated product of the same 16-bit
dequantized weight under the 2-ulp contract of tests/parity.py
(check_fp_output), the accumulation term ceil(K / 16) + 8 roundings of
2^-23 (|x| |w~|^T)[m, n] applying only to outputs in cancellation; the
maximum error in ulps is printed for every case.
Shapes cover every token tile (16, 32, 64, 128, 256), K split across a
cluster and not, a half-filled last K slice (K = 96 with groups of 32),
ragged token and channel tails, both 16-bit activation formats, and the
q_proj-sized decode case in full.  Q4_K two-level scales (codes, sub-scale
codes, super scales, effective scales, and their expansion from the compact
form) are bit-exact too.
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


def _unpack(codes: torch.Tensor) -> np.ndarray:
    b = codes.cpu().numpy().astype(np.int16)
    q = np.empty((b.shape[0], 2 * b.shape[1]), np.int16)
    q[:, 0::2] = (b & 15) - 8
    q[:, 1::2] = (b >> 4) - 8
    return q.astype(np.int8)


def _quant_case(W: torch.Tensor, g: int, what: str):
    w32 = P.host_f32(W)
    qw = q8.q8_quantize_weight_g4(W.to(DEV), g)
    torch.cuda.synchronize()
    q_ref, S_ref = O.quant_weight_group(w32, g)
    P.assert_equal(_unpack(qw.codes), q_ref, what + " codes")
    P.assert_equal(qw.scale.cpu().numpy().T, S_ref, what + " scales")
    return qw, w32, q_ref, S_ref


@pytest.mark.parametrize("n,k,g,dt", [(256, 512, 32, torch.bfloat16),
                                      (272, 384, 128, torch.float16),
                                      (48, 96, 32, torch.bfloat16),
                                      (4096, 4096, 128, torch.bfloat16)])
def test_group_quant_bit_exact(n, k, g, dt):
    W = workloads.random_matrix(n, k, dt, seed=n + k + g, std=0.02)
    _quant_case(W, g, f"{n}x{k} g{g}")


def test_group_quant_ties_zero_groups_and_saturation():
    k, g = 128, 32
    W = torch.zeros(16, k)
    W[0, :32] = torch.tensor([7.0, 3.5, -3.5, 2.5, 0.5, -0.5, 1.5] + [0.0] * 25)   # S = 1, ties
    W[1, 32:64] = torch.linspace(-1.0, 1.0, 32)
    W[2, 64:96] = 3.0e4                         # one value repeated: every code 7
    W[3, 96:] = -1.0e-9                         # below the eps floor: S = 1e-8, codes -0 -> 0
    qw, _, q_ref, S_ref = _quant_case(W.to(torch.bfloat16), g, "ties")
    assert q_ref[0, :7].tolist() == [7, 4, -4, 2, 0, 0, 2]


def _linear_case(m, n, k, g, dt, seed, bias=False, what=""):
    X = workloads.random_matrix(m, k, dt, seed)
    W = workloads.random_matrix(n, k, dt, seed + 1, std=0.02)
    qw, w32, q_ref, S_ref = _quant_case(W, g, what)
    x32 = P.host_f32(X)
    b = (np.random.default_rng(seed).standard_normal(n) * 0.1).astype(np.float32) if bias else None
    Y = q8.q8_linear_w4a16(X.to(DEV), qw, bias=None if b is None else torch.from_numpy(b).to(DEV))
    torch.cuda.synchronize()
    assert q8.q8_get_device_status() == 0
    fmt = P.FMT[dt]
    y_ref, _ = O.linear_w4a16(x32, q_ref, S_ref, g, fmt, bias=b)
    wd = O.widen16(O.dequant_group16(q_ref, S_ref, g, fmt), fmt).astype(np.float64)
    term = P.accumulation_bound(np.abs(x32.astype(np.float64)) @ np.abs(wd).T, k, 16)
    return P.check_fp_output(P.bf16_bits(Y), y_ref, term, what)


@pytest.mark.parametrize("m,n,k,g,dt", [
    (1, 256, 512, 64, torch.bfloat16),       # one token, K split
    (3, 208, 160, 32, torch.bfloat16),       # ragged channels and a half K slice
    (16, 384, 96, 32, torch.float16),        # two K slices, the second half empty
    (30, 512, 1024, 128, torch.bfloat16),    # token tile 32
    (40, 272, 512, 64, torch.float16),       # token tile 64, ragged channels
    (100, 256, 512, 32, torch.bfloat16),     # token tile 128, no split
    (300, 384, 256, 128, torch.float16),     # two token tiles of 256, ragged
    (260, 256, 2048, 32, torch.bfloat16),    # tile 256 with 32 K slices: staging rings wrap
    (16, 128, 8192, 128, torch.bfloat16),    # K split over 8 CTAs of 16 slices each: rings wrap
])
def test_linear_w4a16_shapes(m, n, k, g, dt):
    _linear_case(m, n, k, g, dt, seed=m * 7 + n, bias=(m % 2 == 0), what=f"{m}x{n}x{k} g{g}")


def test_linear_w4a16_decode_q_proj_full():
    # The decode weight recipe at q_proj size, 16 tokens, groups of 128.
    X, W, _ = workloads.make_inputs("decode_q_proj")
    qw, w32, q_ref, S_ref = _quant_case(W, 128, "decode weights")
    x32 = P.host_f32(X)
    Y = q8.q8_linear_w4a16(X.to(DEV), qw)
    torch.cuda.synchronize()
    y_ref, _ = O.linear_w4a16(x32, q_ref, S_ref, 128, "bf16")
    wd = O.widen16(O.dequant_group16(q_ref, S_ref, 128, "bf16"), "bf16").astype(np.float64)
    term = P.accumulation_bound(np.abs(x32.astype(np.float64)) @ np.abs(wd).T, 4096, 16)
    P.check_fp_output(P.bf16_bits(Y), y_ref, term, "decode w4a16")


def test_linear_w4a16_after_producer_kernel():
    # X written by the kernel just before the linear on the same stream: the
    # linear's early start must still read the finished X.
    m, n, k, g = 16, 512, 1024, 64
    W = workloads.random_matrix(n, k, torch.bfloat16, 5, std=0.02)
    qw = q8.q8_quantize_weight_g4(W.to(DEV), g)
    X0 = workloads.random_matrix(m, k, torch.bfloat16, 6).to(DEV)
    for _ in range(3):
        X = X0 * 2.0                            # producer kernel
        Y = q8.q8_linear_w4a16(X, qw)
    Y_sep = q8.q8_linear_w4a16(X0 * 2.0, qw)
    torch.cuda.synchronize()
    assert torch.equal(Y.view(torch.int16), Y_sep.view(torch.int16))
    assert q8.q8_get_device_status() == 0


# ------------------------------------------------------------------ Q4_K two-level scales

def _unpack_sub(sub: torch.Tensor) -> np.ndarray:
    b = sub.cpu().numpy()
    out = np.empty((2 * b.shape[0], b.shape[1]), np.uint8)
    out[0::2] = b & 15
    out[1::2] = b >> 4
    return out.T                                   # n x k/32


@pytest.mark.parametrize("n,k,dt", [(256, 512, torch.bfloat16), (48, 1024, torch.float16),
                                    (4096, 4096, torch.bfloat16)])
def test_q4k_quant_bit_exact(n, k, dt):
    W = workloads.random_matrix(n, k, dt, seed=n + 3 * k, std=0.02)
    W[:, 40:72] *= 8.0                             # uneven sub-block ranges
    w32 = P.host_f32(W)
    qw, sub, sup = q8.q8_quantize_weight_q4k(W.to(DEV))
    torch.cuda.synchronize()
    r = O.quant_weight_q4k(w32)
    P.assert_equal(_unpack(qw.codes), r["q"], "q4k codes")
    P.assert_equal(_unpack_sub(sub), r["q_sub"], "q4k sub-scale codes")
    P.assert_equal(sup.cpu().numpy().T, r["s_super"], "q4k super scales")
    P.assert_equal(qw.scale.cpu().numpy().T, r["S_eff"], "q4k effective scales")
    again = q8.q8_expand_q4k_scales(sub, sup, k)
    torch.cuda.synchronize()
    P.assert_equal(again.cpu().numpy(), qw.scale.cpu().numpy(), "expanded scales")


def test_q4k_linear():
    m, n, k = 16, 512, 1024
    X = workloads.random_matrix(m, k, torch.bfloat16, 21)
    W = workloads.random_matrix(n, k, torch.bfloat16, 22, std=0.02)
    W[:, 64:96] *= 20.0                            # one loud sub-block per row
    qw, sub, sup = q8.q8_quantize_weight_q4k(W.to(DEV))
    Y = q8.q8_linear_w4a16(X.to(DEV), qw)
    torch.cuda.synchronize()
    r = O.quant_weight_q4k(P.host_f32(W))
    x32 = P.host_f32(X)
    y_ref, _ = O.linear_w4a16(x32, r["q"], r["S_eff"], 32, "bf16")
    wd = O.widen16(O.dequant_group16(r["q"], r["S_eff"], 32, "bf16"), "bf16").astype(np.float64)
    term = P.accumulation_bound(np.abs(x32.astype(np.float64)) @ np.abs(wd).T, k, 16)
    P.check_fp_output(P.bf16_bits(Y), y_ref, term, "q4k linear")


def test_w4a16_strided_output_leaves_guard_bands():
    # Y is a view into a larger buffer (row stride n + 40, two extra rows):
    # the padding, filled with a sentinel, must stay untouched.
    m, n, k, g = 37, 272, 512, 64
    X = workloads.random_matrix(m, k, torch.bfloat16, 31)
    W = workloads.random_matrix(n, k, torch.bfloat16, 32, std=0.02)
    qw = q8.q8_quantize_weight_g4(W.to(DEV), g)
    big = torch.full((m + 2, n + 40), -3.0, dtype=torch.bfloat16, device=DEV)
    Y = q8.q8_linear_w4a16(X.to(DEV), qw, out=big[:m, :n])
    ref = q8.q8_linear_w4a16(X.to(DEV), qw)
    torch.cuda.synchronize()
    assert Y.stride(0) == n + 40
    assert torch.equal(big[:m, :n].view(torch.int16), ref.view(torch.int16))
    assert (big[:m, n:] == -3.0).all() and (big[m:] == -3.0).all()
