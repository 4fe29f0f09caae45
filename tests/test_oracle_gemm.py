"""Pins for the oracle's fp64 GEMM reference (W4A4 NVFP4 linear layers: LongLive-2.0 abstract,
fugumt.com; "W4A4 NVFP4 inference" and NVFP4 training GEMMs).

The reference is the plain definition Y = Adeq . Bdeq^T (+bias | +R).  It is checked against
numpy's BLAS matmul on operands decoded with ml_dtypes/torch tables (a different summation order
and different decode code), against closed forms, and on bias/residual handling.
"""
import ml_dtypes
import numpy as np
import pytest
import torch

from bit_kv_cache_24_b200 import synth

E2M1 = np.arange(16, dtype=np.uint8).view(ml_dtypes.float4_e2m1fn).astype(np.float64)
E4M3 = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).to(torch.float64).numpy()


def _deq(q):
    c = np.stack([q.codes & 0xF, q.codes >> 4], axis=-1).reshape(q.codes.shape[0], -1)[:, : q.cols]
    return E2M1[c] * np.repeat(E4M3[q.sf], 16, axis=1)[:, : q.cols] * np.float64(q.g)


@pytest.mark.parametrize("M,N,K", [(1, 1, 16), (1, 16, 16), (17, 8, 32), (16, 24, 544), (37, 40, 96), (5, 3, 17)])
def test_gemm_matches_blas_on_independent_decode(orc, M, N, K):
    a = synth.ragged(M * 7 + K, M, K, "outliers")
    w = synth.ragged(N * 3 + K, N, K, "normal")
    _, qa = orc.quantize(a)
    _, qb = orc.quantize(w)
    y = orc.gemm_rows(qa, qb)
    ref = _deq(qa) @ _deq(qb).T
    scale = np.abs(_deq(qa)).max() * np.abs(_deq(qb)).max() * K + 1e-300
    assert np.max(np.abs(y - ref)) <= 1e-12 * scale


def test_gemm_all_ones_closed_form(orc):
    # x = 1: g = fp32(1/2688), sf = 448, d = fp32(448 g), r = fp32(1/d) = 6, every code 6.0, so
    # Adeq = 6*448*g = 2688 g exactly and Y = K (2688 g)^2.
    M, N, K = 4, 5, 256
    _, qa = orc.quantize(torch.ones(M, K, dtype=torch.bfloat16))
    _, qb = orc.quantize(torch.ones(N, K, dtype=torch.bfloat16))
    g = np.float64(np.float32(1.0) / np.float32(2688.0))
    assert qa.g == np.float32(g)
    assert np.all(qa.sf == 0x7E) and np.all(qa.codes == 0x77)
    y = orc.gemm_rows(qa, qb)
    want = K * (2688.0 * g) ** 2            # (2688 g)^2 needs ~58 bits: fp64 rounding only
    assert np.all(np.abs(y - want) <= K * 2.0 ** -52 * want)
    assert abs(want - K * (1 + 2.0 ** -25)) < 1e-3 * K  # 2688 fp32(1/2688) is 1 + O(2^-25)


def test_gemm_scaled_identity_closed_form(orc):
    # W = 6 I: every diagonal block has b = amax = 6 -> sf 448, d = 448 fp32(6/2688) = 1, code 6;
    # Bdeq = 2688 fp32(6/2688) I, so Y = Adeq * 2688 fp32(6/2688).
    K = 64
    w = torch.zeros(K, K, dtype=torch.bfloat16)
    w.diagonal().fill_(6.0)
    a = synth.ragged(2, 9, K, "normal")
    _, qa = orc.quantize(a)
    _, qb = orc.quantize(w)
    c = 2688.0 * np.float64(np.float32(6.0) / np.float32(2688.0))
    y = orc.gemm_rows(qa, qb)
    assert np.array_equal(y, _deq(qa) * c)


def test_gemm_bias_residual_and_row_subset(orc):
    M, N, K = 12, 16, 64
    a = synth.ragged(4, M, K, "normal")
    w = synth.ragged(5, N, K, "normal")
    bias = synth.ragged(6, 1, N, "normal")[0]
    resid = synth.ragged(7, M, N, "normal")
    _, qa = orc.quantize(a)
    _, qb = orc.quantize(w)
    base = _deq(qa) @ _deq(qb).T
    yb = orc.gemm_rows(qa, qb, bias=bias)
    yr = orc.gemm_rows(qa, qb, resid=resid)
    tol = 1e-12 * np.abs(base).max()
    assert np.max(np.abs(yb - (base + bias.to(torch.float64).numpy()[None, :]))) <= tol
    assert np.max(np.abs(yr - (base + resid.to(torch.float64).numpy()))) <= tol
    rows = np.array([11, 0, 5])
    ys = orc.gemm_rows(qa, qb, rows=rows, resid=resid)
    assert np.array_equal(ys, yr[rows])


@pytest.mark.parametrize("M,N,K,extra", [(37, 40, 96, None), (130, 24, 544, "bias"), (64, 16, 1008, "resid")])
def test_gemm_full_equals_the_row_loop(orc, M, N, K, extra):
    """gemm_full (one fp64 matmul of the dequantized operands, for full-size outputs) against the
    plain per-element sequential sum of gemm_rows: only the fp64 summation order differs."""
    a = synth.ragged(M + 2 * K, M, K, "outliers")
    w = synth.ragged(N + 5 * K, N, K, "lognormal")
    _, qa = orc.quantize(a)
    _, qb = orc.quantize(w)
    kw = {}
    if extra == "bias":
        kw["bias"] = synth.ragged(8, 1, N, "normal")[0]
    elif extra == "resid":
        kw["resid"] = synth.ragged(9, M, N, "normal")
    full = orc.gemm_full(qa, qb, **kw)
    rows = orc.gemm_rows(qa, qb, **kw)
    scale = np.abs(_deq(qa)).max() * np.abs(_deq(qb)).max() * K
    assert full.shape == (M, N)
    assert np.max(np.abs(full - rows)) <= 1e-12 * scale


def test_gemm_full_all_ones_closed_form(orc):
    M, N, K = 3, 8, 512
    _, qa = orc.quantize(torch.ones(M, K, dtype=torch.bfloat16))
    _, qb = orc.quantize(torch.ones(N, K, dtype=torch.bfloat16))
    g = np.float64(np.float32(1.0) / np.float32(2688.0))
    want = K * (2688.0 * g) ** 2
    y = orc.gemm_full(qa, qb)
    assert np.all(np.abs(y - want) <= K * 2.0 ** -52 * want)


def test_bf16_from_f64_rounds_once(orc):
    """Direct fp64 -> BF16 rounding (to nearest, ties to even) against the oracle's FP32 -> BF16
    on values that are exact in FP32 (one rounding either way), and on cases where rounding
    through FP32 first would round twice."""
    rng = np.random.default_rng(5)
    bits = rng.integers(0x00800000, 0x7F000000, 200_000, dtype=np.uint64).astype(np.uint32)
    f = bits.view(np.float32)
    f = np.concatenate([f, -f, np.float32([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, 3.0, 448.0])])
    assert np.array_equal(orc.bf16_from_f64(f.astype(np.float64)), orc.bf16_from_float_array(f))
    # 1 + 2^-8 is a tie between 1 (0x3F80, even) and 1 + 2^-7 (0x3F81): the even one
    assert orc.bf16_from_f64(1.0 + 2.0 ** -8) == 0x3F80
    assert orc.bf16_from_f64(1.0 + 3 * 2.0 ** -8) == 0x3F82
    # just above the tie: BF16 rounds up; through FP32 the 2^-30 would vanish first (-> 0x3F80)
    x = 1.0 + 2.0 ** -8 + 2.0 ** -30
    assert orc.bf16_from_f64(x) == 0x3F81
    assert orc.bf16_from_float(np.float32(x)) == 0x3F80
    assert orc.bf16_from_f64(-x) == 0xBF81
    assert orc.bf16_from_f64(-(1.0 + 2.0 ** -8)) == 0xBF80
