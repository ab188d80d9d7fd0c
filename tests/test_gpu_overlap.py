"""Launch overlap: a weight re-quantized in place right before a linear.

The GEMM kernels request their first weight slices before their
programmatic-launch wait, relying on the weight quantizer not triggering an
early launch.  Here the weight's code, scale and zero-point buffers are
re-quantized from a different matrix immediately before the linear, eagerly
and inside one CUDA graph, and the output must equal (bit for bit) the output
of the same linear on a freshly quantized copy of that matrix: a stale weight
slice would change it.  Shapes cover the pair GEMM (more than 256 tokens), the
one-CTA GEMM and the decode GEMM, INT8 and FP8.
"""
import ctypes

import pytest
import torch

import workloads
from tests import parity as P

pytestmark = pytest.mark.gpu

from bit_quantized_b200 import q8  # noqa: E402

DEV = "cuda:0"


def _quantize_into(W, qw, scheme):
    """q8_quantize_weight through the C ABI into qw's existing buffers."""
    n, k = W.shape
    cdt = qw.code_dtype
    z = None if qw.zero_point is None else ctypes.c_void_p(qw.zero_point.data_ptr())
    st = q8.lib().q8_quantize_weight(
        ctypes.c_void_p(W.data_ptr()), q8.Q8_BF16, n, k, W.stride(0),
        {"asym": q8.Q8_ASYM_INT8, "sym": q8.Q8_SYM_INT8, "fp8": q8.Q8_FP8_E4M3}[scheme], cdt,
        ctypes.c_void_p(qw.codes.data_ptr()), ctypes.c_void_p(qw.scale.data_ptr()), z,
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == q8.Q8_OK


@pytest.mark.parametrize("m,n,k,scheme,codes,act", [
    (512, 1024, 2048, "asym", "s8", "int8"),     # pair GEMM
    (200, 768, 1024, "sym", "s8", "int8"),       # one-CTA GEMM
    (16, 1024, 2048, "asym", "u8", "int8"),      # decode GEMM
    (640, 1280, 2048, "fp8", "e4m3", "fp8"),     # pair GEMM, FP8
])
def test_weight_requantized_in_place_before_linear(m, n, k, scheme, codes, act):
    X = workloads.random_matrix(m, k, torch.bfloat16, seed=m + k).to(DEV)
    Wa = workloads.random_matrix(n, k, torch.bfloat16, seed=n, std=0.02).to(DEV)
    Wb = workloads.random_matrix(n, k, torch.bfloat16, seed=n + 1, std=0.03).to(DEV)
    clip = 1200.0 if act == "fp8" else 0.0
    ref = {}
    for name, W in (("a", Wa), ("b", Wb)):
        Y, _ = q8.q8_linear_w8a8_dynamic(X, q8.q8_quantize_weight(W, scheme, codes), act, clip_ub=clip)
        ref[name] = P.bf16_bits(Y)
    qw = q8.q8_quantize_weight(Wa, scheme, codes)
    Y = torch.empty((m, n), dtype=torch.bfloat16, device=DEV)
    qa = None

    def step(W):
        nonlocal qa
        _quantize_into(W, qw, scheme)
        _, qa = q8.q8_linear_w8a8_dynamic(X, qw, act, clip_ub=clip, out=Y, act=qa)

    # eager: a -> b -> a
    for name, W in (("b", Wb), ("a", Wa), ("b", Wb)):
        step(W)
        torch.cuda.synchronize()
        P.assert_equal(P.bf16_bits(Y), ref[name], f"eager {name}")
    # one CUDA graph holding both re-quantizations and both linears
    outs = []
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        step(Wa)
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    Ya = torch.empty_like(Y)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        step(Wb)
        Ya.copy_(Y)
        step(Wa)
    for _ in range(3):
        g.replay()
        torch.cuda.synchronize()
        outs.append((P.bf16_bits(Ya), P.bf16_bits(Y)))
    for yb, ya in outs:
        P.assert_equal(yb, ref["b"], "graph b")
        P.assert_equal(ya, ref["a"], "graph a")
    assert q8.q8_get_device_status() == 0
