"""q8_linear_int8_mixed_noalloc, the LLM.int8 linear for callers that cannot
allocate device memory, against q8_linear_int8_mixed with a caller workspace.

The allocation-free entry point runs the same kernels on a scratch array the
library owns, so on the same inputs its output must equal the workspace entry
point's: the output and the debug copies (outlier mask and count, INT32
accumulators, fp32 outlier stream) that come out of the library's scratch.
The calls go straight through the C ABI.  Two different problems are
run back to back (the scratch keeps the previous call's contents), then the
first one again.  This file is collected last on purpose.
"""
import ctypes

import numpy as np
import pytest
import torch

import workloads
from tests import parity as P

pytestmark = pytest.mark.gpu

from bit_quantized_b200 import q8  # noqa: E402

DEV = "cuda:0"


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _noalloc(X, qw, threshold, Y, bias=None, mask=None, count=None, acc=None, y16=None):
    cw = qw.c()
    m, k = X.shape
    return q8.lib().q8_linear_int8_mixed_noalloc(
        _ptr(X), q8.Q8_F16, m, k, X.stride(0), ctypes.byref(cw), None, float(threshold),
        _ptr(bias), _ptr(Y), Y.stride(0), _ptr(mask), _ptr(count), _ptr(acc), _ptr(y16), _stream())


def _case(seed, m, n, k, outlier_cols):
    X = workloads.random_matrix(m, k, torch.float16, seed)
    X[:, outlier_cols] *= 12
    W = workloads.random_matrix(n, k, torch.float16, seed + 1, 0.02)
    return X.to(DEV), q8.q8_quantize_weight(W.to(DEV), "asym", "s8")


def _check(X, qw, threshold, what, bias=None):
    """The allocation-free call against the workspace entry point: output,
    outlier mask and count, INT32 accumulators and the fp32 outlier stream,
    all copied out of the library's scratch, must be bit-identical."""
    m, k = X.shape
    n = qw.codes.shape[0]
    Y_ref, dbg = q8.q8_linear_int8_mixed(X, qw, threshold, bias=bias, debug=True)
    Y = torch.full((m, n), float("nan"), dtype=torch.bfloat16, device=DEV)
    mask = torch.full((k,), 0xAB, dtype=torch.uint8, device=DEV)
    count = torch.full((1,), -1, dtype=torch.int32, device=DEV)
    acc = torch.full((m, n), 0x7EADBEEF, dtype=torch.int32, device=DEV)
    y16 = torch.full((m, n), float("nan"), dtype=torch.float32, device=DEV)
    assert _noalloc(X, qw, threshold, Y, bias, mask, count, acc, y16) == q8.Q8_OK, what
    torch.cuda.synchronize()
    ref_bits = P.bf16_bits(Y_ref)
    got_bits = P.bf16_bits(Y)
    P.assert_bf16_within(got_bits, P.bf16_values(ref_bits), 0.0, what)
    P.assert_equal(got_bits, ref_bits, what + " Y")
    P.assert_equal(mask.cpu().numpy(), dbg["mask"].cpu().numpy(), what + " mask")
    assert int(count.item()) == int(dbg["count"].item()), what + " count"
    P.assert_equal(acc.cpu().numpy(), dbg["acc"].cpu().numpy(), what + " acc")
    P.assert_equal(y16.cpu().numpy().view(np.uint32), dbg["y16"].cpu().numpy().view(np.uint32),
                   what + " y16")


def test_noalloc_matches_workspace_entry_point_on_consecutive_calls():
    Xt, Wt, _ = workloads.make_inputs("tiny_mixed")
    first = (Xt.to(DEV), q8.q8_quantize_weight(Wt.to(DEV), "asym", "s8"))
    second = _case(71, 130, 272, 512, [1, 300, 301, 450])
    bias = torch.linspace(-1, 1, 272, device=DEV)
    _check(*first, 6.0, "first call (16x256x256)")
    _check(*second, 6.0, "second call (130x272x512, bias)", bias=bias)
    _check(*first, 6.0, "third call, first problem again")
    assert q8.q8_get_device_status() == 0


def test_noalloc_rejects_sizes_beyond_its_scratch():
    # n = k = 8192 needs 2 * 8192 * 8192 bytes for the outlier weight columns
    # alone (128 MiB) > Q8_NOALLOC_SCRATCH_BYTES: refused before any launch.
    n = k = 8192
    assert q8.q8_workspace_size(q8.Q8_OP_LINEAR_INT8_MIXED, 16, n, k) > q8.Q8_NOALLOC_SCRATCH_BYTES
    X = torch.zeros((16, k), dtype=torch.float16, device=DEV)
    codes = torch.zeros((n, k), dtype=torch.int8, device=DEV)
    scale = torch.ones(n, dtype=torch.float32, device=DEV)
    qw = q8.QWeight(codes, scale, None, q8.Q8_S8)
    Y = torch.zeros((16, n), dtype=torch.bfloat16, device=DEV)
    assert _noalloc(X, qw, 6.0, Y) == q8.Q8_ERR_SHAPE
    torch.cuda.synchronize()
    assert (Y == 0).all()
