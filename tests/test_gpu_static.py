"""GPU parity of the static activation quantizer and of the re-quantizing
W8A8 linear against the CPU oracle, bit-exact ("大模型量化" (Xilyfe): static
quantization with calibrated scales; re-quantization of a layer's INT32 result
back to INT8 before the next layer).

Inputs are seeded (workloads.random_matrix).  Scales cover: a calibrated scale
with headroom (no saturation), one that makes rows saturate (those rows take
the exact path), a power of two (exact reciprocal), and a scale for which many
inputs sit exactly on rounding midpoints.
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


def _static_check(X: torch.Tensor, S: float, what: str):
    qa = q8.q8_quantize_act_static(X.to(DEV), S)
    torch.cuda.synchronize()
    q, Sr, rs = O.quant_act_static(P.host_f32(X), S)
    P.assert_equal(qa.codes.cpu().numpy(), q, what + " codes")
    P.assert_equal(qa.scale.cpu().numpy().view(np.uint32), Sr.view(np.uint32), what + " scale")
    P.assert_equal(qa.rowsum.cpu().numpy(), rs, what + " rowsum")
    return qa


@pytest.mark.parametrize("m,k,dtype", [(16, 4096, torch.bfloat16), (2048, 4096, torch.bfloat16),
                                       (4096, 8192, torch.bfloat16), (5, 160, torch.float32),
                                       (3, 96, torch.float16), (33, 8192, torch.float16),
                                       (2, 32768, torch.bfloat16)])   # longer than the register cache
def test_static_act_scales(m, k, dtype):
    X = workloads.random_matrix(m, k, dtype, seed=m + k)
    amax = float(X.float().abs().max())
    for name, S in [("headroom", 1.25 * amax / 127), ("saturating", 0.5 * amax / 127),
                    ("power of two", 2.0 ** np.floor(np.log2(amax / 127)))]:
        _static_check(X, float(np.float32(S)), f"{m}x{k} {dtype} {name}")


def test_static_act_midpoints():
    S = np.float32(9 / 64)
    g = torch.Generator().manual_seed(5)
    n = torch.randint(-150, 150, (8, 512), generator=g).to(torch.float32)
    X = ((2 * n + 1) * float(S) / 2).to(torch.float16)      # x / S on half-integers, some beyond 127
    _static_check(X, float(S), "midpoints")


@pytest.mark.parametrize("m,n,k,codes,wscheme", [(16, 4096, 4096, "u8", "asym"),
                                                 (256, 512, 1024, "s8", "sym"),
                                                 (3, 208, 160, "s8", "asym"),
                                                 (40, 512, 1024, "u8", "asym")])   # NT = 64 decode
def test_requant_linear(m, n, k, codes, wscheme):
    X = workloads.random_matrix(m, k, torch.bfloat16, seed=m + 2 * n)
    W = workloads.random_matrix(n, k, torch.bfloat16, seed=n + k, std=0.02)
    qw = q8.q8_quantize_weight(W.to(DEV), wscheme, codes)
    Sx = float(np.float32(1.1 * float(X.float().abs().max()) / 127))
    qa = q8.q8_quantize_act_static(X.to(DEV), Sx)
    bias = torch.linspace(-0.5, 0.5, n, device=DEV) if m % 2 else None
    Y16 = q8.q8_linear_w8a8(qa, qw, bias=bias)
    torch.cuda.synchronize()
    yabs = float(Y16.float().abs().max())
    wq, Sw, Zw = O.quant_weight(P.host_f32(W), wscheme, codes)
    xq, Sxr, rs = O.quant_act_static(P.host_f32(X), Sx)
    b = None if bias is None else bias.cpu().numpy()
    _, y_ref, _ = O.linear_w8a8_int8(xq, Sxr, rs, wq, Sw, None if wscheme == "sym" else Zw, bias=b)
    for name, So in [("headroom", 1.2 * yabs / 127), ("saturating", 0.3 * yabs / 127)]:
        So = float(np.float32(So))
        acc = torch.empty((m, n), dtype=torch.int32, device=DEV)
        Yq = q8.q8_linear_w8a8_requant(qa, qw, So, bias=bias, acc_debug=acc)
        torch.cuda.synchronize()
        P.assert_equal(Yq.cpu().numpy(), O.requant(y_ref, So), f"requant {m}x{n}x{k} {name}")
    assert q8.q8_get_device_status() == 0
