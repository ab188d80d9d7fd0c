"""Device-side failure detection on the GPU, without a fault.

q8_selftest_wait_timeout runs a CTA with the GEMM kernels' roles whose
producer waits on a barrier nothing arrives on, bounded by a short limit.  The
wait runs out, the status word reads Q8_ERR_DEVICE_TIMEOUT, the other roles
leave on the abort flag, the CTA frees its tensor memory and returns.  The
test then checks that the status clears and that the next calls (a tile
kernel that allocates all 512 TMEM columns, and the decode kernel) still give
bit-exact results: the context stayed usable and no TMEM was left allocated.
"""
import time

import numpy as np
import pytest
import torch

import workloads
from oracle import oracle as O
from tests import parity as P

pytestmark = pytest.mark.gpu

from bit_quantized_b200 import q8  # noqa: E402

DEV = "cuda:0"


@pytest.fixture(autouse=True)
def _clear_status_after():
    yield
    q8.q8_clear_device_status()     # later test files expect a clean status word


def _int8_linear_matches_oracle(m, n, k, seed):
    X = workloads.random_matrix(m, k, torch.bfloat16, seed)
    W = workloads.random_matrix(n, k, torch.bfloat16, seed + 1, std=0.02)
    qa = q8.q8_quantize_act(X.to(DEV), "int8")
    qw = q8.q8_quantize_weight(W.to(DEV), "sym", "s8")
    Y = q8.q8_linear_w8a8(qa, qw)
    torch.cuda.synchronize()
    xq, Sx, rs = O.quant_act_int8(P.host_f32(X))
    wq, Sw, _ = O.quant_weight(P.host_f32(W), "sym")
    _, _, Y_ref = O.linear_w8a8_int8(xq, Sx, rs, wq, Sw)
    P.assert_equal(P.bf16_bits(Y), Y_ref, f"{m}x{n}x{k} after the timeout")


@pytest.mark.parametrize("limit_us", [2000, 50])
def test_bounded_wait_runs_out_and_context_stays_usable(limit_us):
    q8.q8_clear_device_status()
    assert q8.q8_get_device_status() == q8.Q8_OK
    t0 = time.perf_counter()
    q8.q8_selftest_wait_timeout(limit_us)
    status = q8.q8_get_device_status()          # waits for the stream
    elapsed = time.perf_counter() - t0
    assert status == q8.Q8_ERR_DEVICE_TIMEOUT
    assert elapsed < 0.5, f"self-test took {elapsed:.3f} s for a {limit_us} us limit"
    # The status word keeps the first error until it is cleared.
    _int8_linear_matches_oracle(16, 256, 512, 3)
    assert q8.q8_get_device_status() == q8.Q8_ERR_DEVICE_TIMEOUT
    q8.q8_clear_device_status()
    assert q8.q8_get_device_status() == q8.Q8_OK
    # Both GEMM kernels run normally afterwards: 300 tokens take the tile
    # kernel (512 TMEM columns per CTA), 16 the decode kernel.
    _int8_linear_matches_oracle(300, 2304, 1024, 5)
    _int8_linear_matches_oracle(16, 1024, 2048, 7)
    assert q8.q8_get_device_status() == q8.Q8_OK


def test_status_word_reported_to_python_as_error_code():
    q8.q8_selftest_wait_timeout(100)
    assert q8.q8_get_device_status() == q8.Q8_ERR_DEVICE_TIMEOUT
    assert "bounded device-side wait" in q8.q8_status_string(q8.q8_get_device_status())
    q8.q8_clear_device_status()
    assert q8.q8_get_device_status() == q8.Q8_OK
