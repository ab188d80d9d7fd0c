"""GPU parity of the smoothed activation quantizer and of a smoothed W8A8
linear against the CPU oracle, bit-exact ("大模型量化" (Xilyfe), algorithm list,
SmoothQuant: activation outlier channels moved onto the weight).

Seeded inputs; multipliers drawn per column, with the outlier columns of the
LLM.int8-style inputs smoothed hardest.  Shapes cover every kernel
configuration (short rows, one wave, several waves) and fp32 input.
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


def _mult(k, seed, outliers=()):
    rng = np.random.default_rng(seed)
    s = rng.uniform(0.3, 3.0, k).astype(np.float32)
    for j in outliers:
        s[j] = 40.0
    return s, (1.0 / s).astype(np.float32)


def _check(X: torch.Tensor, mult: np.ndarray, what: str):
    qa = q8.q8_quantize_act_smooth(X.to(DEV), torch.from_numpy(mult).to(DEV))
    torch.cuda.synchronize()
    q, S, rs = O.quant_act_smooth(P.host_f32(X), mult)
    P.assert_equal(qa.codes.cpu().numpy(), q, what + " codes")
    P.assert_equal(qa.scale.cpu().numpy().view(np.uint32), S.view(np.uint32), what + " scale")
    P.assert_equal(qa.rowsum.cpu().numpy(), rs, what + " rowsum")
    return qa


@pytest.mark.parametrize("m,k,dtype", [(16, 4096, torch.bfloat16), (2048, 4096, torch.bfloat16),
                                       (4096, 8192, torch.bfloat16), (5, 160, torch.float32),
                                       (33, 8192, torch.float16), (2, 32768, torch.float16)])
def test_smooth_act(m, k, dtype):
    X = workloads.random_matrix(m, k, dtype, seed=3 * m + k)
    _, mult = _mult(k, seed=k)
    _check(X, mult, f"{m}x{k} {dtype}")


def test_smooth_act_outlier_workload():
    X, W, info, x32, w32 = P.workload("mixed_512")
    _, mult = _mult(X.shape[1], 9, info["planted_columns"])
    _check(X, mult, "mixed_512 with smoothed outlier columns")


def test_smoothed_linear_matches_oracle():
    m, n, k = 16, 1024, 2048
    X = workloads.random_matrix(m, k, torch.bfloat16, seed=21)
    X[:, 100] *= 30
    W = workloads.random_matrix(n, k, torch.bfloat16, seed=22, std=0.02)
    s, mult = _mult(k, 23, outliers=(100,))
    Ws = O.smooth_weight(P.host_f32(W), s)                       # offline, fp32
    qw = q8.q8_quantize_weight(torch.from_numpy(Ws).to(DEV), "asym", "u8")
    qa = q8.q8_quantize_act_smooth(X.to(DEV), torch.from_numpy(mult).to(DEV))
    Y = q8.q8_linear_w8a8(qa, qw)
    torch.cuda.synchronize()
    xq, Sx, rs = O.quant_act_smooth(P.host_f32(X), mult)
    wq, Sw, Zw = O.quant_weight(Ws, "asym", "u8")
    _, _, Yr = O.linear_w8a8_int8(xq, Sx, rs, wq, Sw, Zw)
    P.assert_equal(P.bf16_bits(Y), Yr, "smoothed linear")
    assert q8.q8_get_device_status() == 0
