"""Every finite 16-bit input through every quantizer, bit-exact against the oracle.

The kernels form each code from the IEEE quotient fl32(x / S) without a
division (one multiply by RN(1/S) and two FMA corrections), so the codes of
every representable bf16 and fp16 value are checked here, under many row
scales: for each absmax A in a list, the rows hold all finite values v of the
type with |v| <= A (A itself in every row), so every rounding boundary of the
integer and E4M3 codes below A is crossed.  Static scales include ones small
enough to overflow the quotient and ones below the exact-quotient domain;
smoothed rows multiply by per-column factors first.  Rows of 4096 take the
register-cached path, rows of 65536 the re-read path.
"""
import numpy as np
import pytest
import torch

from oracle import oracle as O
from tests import parity as P

pytestmark = pytest.mark.gpu

from bit_quantized_b200 import q8  # noqa: E402

DEV = "cuda:0"
K = 4096


def _finite(dtype):
    """All finite values of a 16-bit float type (both zeros included)."""
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    emask = 0x7F80 if dtype == torch.bfloat16 else 0x7C00
    bits = bits[(bits & emask) != emask]
    return torch.from_numpy(bits.view(np.int16)).view(dtype)


def _amax_list(dtype, seed):
    """Row absmax values: fixed ones (1, 127, 448, the largest finite value,
    the smallest normal, a subnormal, scales that are exact) and random
    finite positive values of the type spread over its exponents."""
    vals = _finite(dtype)
    pos = vals[(vals.float() > 0)]
    fixed = [1.0, 127.0, 448.0, 0.75, 1.0 / 3.0, 127.0 * 9 / 64, 63.0, 3.0e-3]
    g = torch.Generator().manual_seed(seed)
    rnd = pos[torch.randint(0, pos.numel(), (14,), generator=g)]
    out = torch.cat([torch.tensor(fixed).to(dtype), rnd, pos[-1:], pos[:1]])
    smallest_normal = 2.0 ** -14 if dtype == torch.float16 else 2.0 ** -126
    out = torch.cat([out, torch.tensor([smallest_normal]).to(dtype)])
    return out


def _rows(dtype, amax, k, seed):
    """Rows of length k holding every finite value with |v| <= A for each A,
    shuffled, A appended to every row, zero-padded."""
    vals = _finite(dtype)
    g = torch.Generator().manual_seed(seed)
    rows = []
    for A in amax:
        a = float(A)
        sel = vals[vals.float().abs() <= a]
        sel = sel[torch.randperm(sel.numel(), generator=g)]
        per = k - 1
        for s in range(0, sel.numel(), per):
            chunk = sel[s:s + per]
            row = torch.zeros(k, dtype=dtype)
            row[:chunk.numel()] = chunk
            row[-1] = A
            rows.append(row)
    return torch.stack(rows)


@pytest.fixture(scope="module", params=[torch.bfloat16, torch.float16], ids=["bf16", "fp16"])
def matrix(request):
    dtype = request.param
    X = _rows(dtype, _amax_list(dtype, 7), K, 11)
    return X, P.host_f32(X)


def _act_int8(X, x32, what):
    qa = q8.q8_quantize_act(X.to(DEV), "int8")
    torch.cuda.synchronize()
    q, S, rs = O.quant_act_int8(x32)
    P.assert_equal(qa.scale.cpu().numpy().view(np.uint32), S.view(np.uint32), what + " scale")
    P.assert_equal(qa.codes.cpu().numpy(), q, what + " codes")
    P.assert_equal(qa.rowsum.cpu().numpy(), rs, what + " rowsum")


def _act_fp8(X, x32, ub, what):
    qa = q8.q8_quantize_act(X.to(DEV), "fp8", clip_ub=ub)
    torch.cuda.synchronize()
    q, S = O.quant_act_fp8(x32, ub)
    P.assert_equal(qa.scale.cpu().numpy().view(np.uint32), S.view(np.uint32), what + " scale")
    P.assert_equal(P.codes_u8(qa.codes), q, what + " codes")


def test_act_int8_every_value(matrix):
    X, x32 = matrix
    _act_int8(X, x32, f"int8 {X.dtype} {X.shape[0]} rows")


def test_act_fp8_every_value(matrix):
    X, x32 = matrix
    _act_fp8(X, x32, 0.0, "fp8")
    # A clip bound below most rows' absmax: quotients above 448 saturate,
    # and the rows with the largest values leave the exact-quotient domain.
    _act_fp8(X, x32, 1.5, "fp8 clipped at 1.5")
    _act_fp8(X, x32, 2.0 ** -100, "fp8 clipped at 2^-100")


@pytest.mark.parametrize("scheme,codes", [("sym", "s8"), ("asym", "s8"), ("asym", "u8"), ("fp8", "e4m3")])
def test_weight_every_value(matrix, scheme, codes):
    W, w32 = matrix
    qw = q8.q8_quantize_weight(W.to(DEV), scheme, codes)
    torch.cuda.synchronize()
    q, S, Z = O.quant_weight(w32, scheme, codes)
    got = P.codes_u8(qw.codes) if codes in ("u8", "e4m3") else qw.codes.cpu().numpy()
    what = f"weight {scheme}/{codes} {W.dtype}"
    P.assert_equal(qw.scale.cpu().numpy().view(np.uint32), S.view(np.uint32), what + " scale")
    if Z is not None:
        P.assert_equal(qw.zero_point.cpu().numpy(), Z, what + " zero point")
    P.assert_equal(got, q, what + " codes")


def test_weight_asym_one_signed_rows(matrix):
    """Rows that do not cross zero (only the positive, then only the negative
    values): Z sits at a clamp bound and most quotients saturate."""
    W, w32 = matrix
    for sign in (1.0, -1.0):
        Wp = W.abs() * sign
        for codes in ("s8", "u8"):
            qw = q8.q8_quantize_weight(Wp.to(DEV), "asym", codes)
            torch.cuda.synchronize()
            q, S, Z = O.quant_weight(P.host_f32(Wp), "asym", codes)
            got = P.codes_u8(qw.codes) if codes == "u8" else qw.codes.cpu().numpy()
            what = f"asym {codes} sign {sign:+.0f} {W.dtype}"
            P.assert_equal(qw.zero_point.cpu().numpy(), Z, what + " zero point")
            P.assert_equal(got, q, what + " codes")


@pytest.mark.parametrize("S", [0.0123, 1.0, 9.0 / 64.0, 3.7e4, 1e-20, 2.0 ** -95, 1e-40])
def test_static_every_value(matrix, S):
    """Static scales from ordinary to tiny: at 1e-20 large inputs' quotients
    overflow fp32; 2^-95 and the subnormal 1e-40 lie below the exact-quotient
    domain and are coded by division."""
    X, x32 = matrix
    qa = q8.q8_quantize_act_static(X.to(DEV), S)
    torch.cuda.synchronize()
    q, Sr, rs = O.quant_act_static(x32, S)
    what = f"static S={S} {X.dtype}"
    P.assert_equal(qa.codes.cpu().numpy(), q, what + " codes")
    P.assert_equal(qa.rowsum.cpu().numpy(), rs, what + " rowsum")


def test_smooth_every_value(matrix):
    """Rows whose smoothed values stay finite (x * m overflows fp32 in the
    rows with the type's largest values, which no scale can code)."""
    X, x32 = matrix
    g = np.random.default_rng(5)
    mult = np.exp(g.uniform(-4.0, 4.0, K)).astype(np.float32)
    with np.errstate(over="ignore"):
        finite = np.isfinite(x32 * mult[None, :]).all(axis=1)
    assert finite.sum() >= 0.8 * finite.size
    X, x32 = X[torch.from_numpy(finite)], np.ascontiguousarray(x32[finite])
    qa = q8.q8_quantize_act_smooth(X.to(DEV), torch.from_numpy(mult).to(DEV))
    torch.cuda.synchronize()
    q, S, rs = O.quant_act_smooth(x32, mult)
    what = f"smooth {X.dtype}"
    P.assert_equal(qa.scale.cpu().numpy().view(np.uint32), S.view(np.uint32), what + " scale")
    P.assert_equal(qa.codes.cpu().numpy(), q, what + " codes")
    P.assert_equal(qa.rowsum.cpu().numpy(), rs, what + " rowsum")


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16], ids=["bf16", "fp16"])
def test_long_rows_every_value(dtype):
    """Rows of 65536 values (longer than the register cache: read twice)."""
    amax = _amax_list(dtype, 13)[[0, 1, 2, 8, -3]]
    X = _rows(dtype, amax, 65536, 17)
    x32 = P.host_f32(X)
    _act_int8(X, x32, f"long int8 {dtype}")
    _act_fp8(X, x32, 0.0, f"long fp8 {dtype}")
