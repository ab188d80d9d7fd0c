"""GPU parity of the grouped FP8 rowwise linear (mixture-of-experts layers).

Activation and weight codes are bit-exact with the oracle (the FP8 quantizers
are the ones of the dense path); outputs meet the 2-ulp contract of
tests/parity.py (check_fp_output) for every token against its own expert's
block, the accumulation term ceil(K / 32) + 8 roundings of
2^-23 (|xq| |wq|^T) Sx Sw applying only to outputs in cancellation.  Cases cover empty experts,
experts smaller than one tile, tiles that straddle two experts, a ragged
channel tail, bias, and offsets that leave rows uncovered (those rows must
stay untouched).
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


def _moe_case(counts, n, k, seed, bias=False, rows=None, offsets=None, what=""):
    E = len(counts)
    m = int(sum(counts))
    X = workloads.random_matrix(m, k, torch.bfloat16, seed)
    W = workloads.random_matrix(E * n, k, torch.bfloat16, seed + 1, std=0.02)
    x32, w32 = P.host_f32(X), P.host_f32(W)
    off = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32) if offsets is None \
        else np.asarray(offsets, np.int32)
    b = (np.random.default_rng(seed).standard_normal(E * n) * 0.1).astype(np.float32) if bias else None
    qa = q8.q8_quantize_act(X.to(DEV), "fp8", clip_ub=1200.0)
    qw = q8.q8_quantize_weight(W.to(DEV), "fp8", "e4m3")
    Y = torch.full((m, n), 7.0, dtype=torch.bfloat16, device=DEV)     # sentinel
    q8.q8_linear_fp8_grouped(qa, qw, E, torch.from_numpy(off).to(DEV),
                             bias=None if b is None else torch.from_numpy(b).to(DEV), out=Y)
    torch.cuda.synchronize()
    assert q8.q8_get_device_status() == 0
    xq, Sx = O.quant_act_fp8(x32, 1200.0)
    wq, Sw, _ = O.quant_weight(w32, "fp8")
    P.assert_equal(P.codes_u8(qa.codes), xq, what + " act codes")
    P.assert_equal(P.codes_u8(qw.codes), wq, what + " weight codes")
    r = np.arange(m) if rows is None else np.asarray(rows)
    covered = (r >= max(off[0], 0)) & (r < min(off[-1], m))
    y_ref, _ = O.linear_moe_fp8(xq, Sx, wq, Sw, off, n, bias=b, rows=r[covered])
    # per-row magnitude bound against the row's own expert block
    Xa = np.abs(O.widen_e4m3(xq)).astype(np.float64)
    Wa = np.abs(O.widen_e4m3(wq)).astype(np.float64)
    extra = np.zeros(y_ref.shape)
    for i, row in enumerate(r[covered]):
        e = int(np.searchsorted(off, row, side="right") - 1)
        mag = Xa[row] @ Wa[e * n:(e + 1) * n].T
        extra[i] = (P.accumulation_bound(mag, k, 32) * float(Sx[row])
                    * Sw[e * n:(e + 1) * n].astype(np.float64))
    Yb = P.bf16_bits(Y)
    P.check_fp_output(Yb[r[covered]], y_ref, extra, what)
    if (~covered).any():                       # uncovered rows keep the sentinel
        assert np.all(Y.float().cpu().numpy()[r[~covered]] == 7.0)


@pytest.mark.parametrize("counts,n,k", [
    ((130, 0, 7, 300), 256, 512),            # empty expert, sub-tile expert, straddling tiles
    ((1,), 128, 256),                         # one token, one expert
    ((64, 64, 64, 64, 64, 64, 64, 64), 144, 1024),   # ragged channel tail (16 of 144)
    ((3, 250, 0, 0, 129), 512, 160),          # K not a multiple of 128
])
def test_grouped_fp8_shapes(counts, n, k):
    _moe_case(counts, n, k, seed=sum(counts) + n, bias=(n % 256 == 0), what=f"moe {counts} n{n} k{k}")


def test_grouped_fp8_llama4_like_sampled():
    # 16 experts of a Llama4-like FFN (gate_up 2 x 1024 wide) over 2048 routed tokens.
    rng = np.random.default_rng(12)
    counts = rng.multinomial(2048, np.ones(16) / 16)
    rows = P.sample_indices(2048, 160, 13)
    _moe_case(tuple(int(c) for c in counts), 2048, 1024, seed=40, rows=rows, what="moe llama4-like")


def test_grouped_fp8_offsets_leave_rows_uncovered():
    # offsets cover rows 0..99 only: rows 100..149 are never written
    _moe_case((40, 60, 50), 128, 256, seed=9, offsets=[0, 40, 100, 100], what="moe uncovered")


def test_grouped_fp8_strided_output_leaves_guard_bands():
    counts, n, k = (70, 0, 140), 144, 256
    E, m = len(counts), sum(counts)
    X = workloads.random_matrix(m, k, torch.bfloat16, 51)
    W = workloads.random_matrix(E * n, k, torch.bfloat16, 52, std=0.02)
    off = torch.tensor(np.concatenate([[0], np.cumsum(counts)]), dtype=torch.int32, device=DEV)
    qa = q8.q8_quantize_act(X.to(DEV), "fp8", clip_ub=1200.0)
    qw = q8.q8_quantize_weight(W.to(DEV), "fp8", "e4m3")
    big = torch.full((m + 3, n + 24), -5.0, dtype=torch.bfloat16, device=DEV)
    q8.q8_linear_fp8_grouped(qa, qw, E, off, out=big[:m, :n])
    ref = q8.q8_linear_fp8_grouped(qa, qw, E, off)
    torch.cuda.synchronize()
    assert torch.equal(big[:m, :n].view(torch.int16), ref.view(torch.int16))
    assert (big[:m, n:] == -5.0).all() and (big[m:] == -5.0).all()
