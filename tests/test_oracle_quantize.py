"""Pins for the oracle's quantizer / dequantizer: hand-derived worked examples (tests/golden),
exact special cases, the round-trip error bound of round-to-nearest, and structural invariants.

The method (W4A4 NVFP4 activations/weights and an NVFP4 KV cache, LongLive-2.0 abstract on
fugumt.com; d9249.github.io review, section "핵심 아이디어 / 구조 / 동작 방식") fixes no numeric
example, so the expected values below come from the format definitions, worked by hand.
"""
import os

import ml_dtypes
import numpy as np
import pytest
import torch

from bit_kv_cache_24_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "nvfp4_worked_examples.txt")

E2M1 = np.arange(16, dtype=np.uint8).view(ml_dtypes.float4_e2m1fn).astype(np.float64)
E4M3 = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).to(torch.float64).numpy()


def _bf16(a):
    return torch.tensor(np.asarray(a, dtype=np.float32)).to(torch.bfloat16)


def _unpack(codes, cols):
    lo = codes & 0xF
    hi = codes >> 4
    out = np.stack([lo, hi], axis=-1).reshape(codes.shape[0], -1)
    return out[:, :cols]


def _deq_independent(q):
    """fp64 dequant from the codes with decode tables taken from ml_dtypes/torch."""
    c = _unpack(q.codes, q.cols)
    sf = np.repeat(E4M3[q.sf], 16, axis=1)[:, : q.cols]
    return E2M1[c] * sf * np.float64(q.g)


def _golden():
    rows = []
    for line in open(GOLDEN, encoding="utf-8"):
        if line.startswith("#") or not line.strip():
            continue
        name, xs, gbits, sfs, codes, packed = [f.strip() for f in line.split("|")]
        rows.append((name, [float(v) for v in xs.split()], int(gbits, 16),
                     [int(v, 16) for v in sfs.split()], [int(v, 16) for v in codes.split()],
                     [int(v, 16) for v in packed.split()]))
    return rows


@pytest.mark.parametrize("case", _golden(), ids=lambda c: c[0])
def test_worked_examples(orc, case):
    name, xs, gbits, sfs, codes, packed = case
    st, q = orc.quantize(_bf16([xs]))
    assert st == 0
    assert int(np.float32(q.g).view(np.uint32)) == gbits
    assert list(q.sf[0]) == sfs
    assert list(_unpack(q.codes, len(xs))[0]) == codes
    assert list(q.codes[0][: len(packed)]) == packed
    assert not q.codes[0][len(packed):].any()            # row padding is zero


def test_worked_example_saturation_dequant(orc):
    _, xs, *_ = _golden()[1]
    st, q = orc.quantize(_bf16([xs]))
    y = orc.bf16_bits_to_f32(orc.dequant(q))[0]
    # 4.0 saturates: 6 * 288 * g = 3.857143 -> BF16 3.859375
    assert y[16] == np.float32(3.859375)
    assert _deq_independent(q)[0, 16] == pytest.approx(3.857142857, rel=1e-7)


def test_power_of_two_scales_round_trip_and_ties(orc):
    # With amax_in = 2688 * 2^e the tensor scale g = 2^e exactly, and a block whose max is
    # 6 * 2^k gets sf = 2^(k-e) and d = 2^k exactly: grid values round-trip, midpoints go even.
    e = -3
    amax_in = float(2688.0 * 2.0 ** e)
    rng = np.random.default_rng(1)
    rows = []
    for k in (-9, -4, 0, 3):
        d = 2.0 ** k
        grid = np.array([6, 0.5, 1, 1.5, 2, 3, 4, 0, -0.5, -1, -1.5, -2, -3, -4, -6, 6.0])
        rows.append(grid * d)
        ties = np.array([6, 0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5, -0.25, -0.75, -1.25, -1.75, -2.5, -3.5, -5, 0])
        rows.append(ties * d)
    x = np.array(rows)
    st, q = orc.quantize(_bf16(x), amax_in=amax_in)
    assert st == 0 and q.g == np.float32(2.0 ** e)
    deq = _deq_independent(q)
    for r in range(0, len(rows), 2):
        assert np.array_equal(deq[r], x[r])                       # exact round trip
        want = np.array([6, 0, 1, 1, 2, 2, 4, 4, -0, -1, -1, -2, -2, -4, -4, 0]) * x[r + 1][0] / 6
        assert np.array_equal(deq[r + 1], want)                   # ties to even


def test_zero_tensor_and_zero_blocks(orc):
    x = np.zeros((3, 48))
    x[1, 20] = -2.0                                               # one non-zero block
    st, q = orc.quantize(_bf16(x))
    assert st == 0
    assert q.sf[0].tolist() == [0, 0, 0] and q.sf[2].tolist() == [0, 0, 0]
    assert q.sf[1, 0] == 0 and q.sf[1, 2] == 0 and q.sf[1, 1] == 0x7E
    st, q0 = orc.quantize(_bf16(np.zeros((2, 32))))
    assert q0.g == 1.0 and not q0.codes.any() and not q0.sf.any()


def test_nonfinite_input_reports_status(orc):
    for bad in (np.inf, -np.inf, np.nan):
        x = np.ones((2, 32))
        x[1, 7] = bad
        st, _ = orc.quantize(_bf16(x))
        assert st == orc.ORC_NONFINITE
    st, _ = orc.quantize(_bf16(np.ones((1, 16))), amax_in=float("inf"))
    assert st == orc.ORC_NONFINITE


@pytest.mark.parametrize("rows,cols,kind", [(1, 16, "normal"), (7, 40, "outliers"), (64, 256, "lognormal"),
                                            (33, 1000, "wide"), (130, 96, "wide"), (257, 3072, "outliers")])
def test_round_trip_error_bound(orc, rows, cols, kind):
    """Round to nearest: |x - deq| <= d*h(|q|) (+ saturation excess), h = half the E2M1 gap."""
    x = synth.ragged(7 + rows, rows, cols, kind)
    st, q = orc.quantize(x)
    assert st == 0
    xf = x.to(torch.float64).numpy()
    deq = _deq_independent(q)
    nb = q.sf.shape[1]
    d = np.repeat((E4M3[q.sf] * np.float64(q.g)), 16, axis=1)[:, :cols]
    a = np.abs(xf) / np.where(d == 0, 1, d)
    h = np.where(a < 2, 0.25, np.where(a < 4, 0.5, 1.0))
    bound = d * (h + a * 2.0 ** -21) + np.maximum(0.0, np.abs(xf) - 6 * d)
    err = np.abs(xf - deq)
    assert np.all(err <= bound + 1e-300), float(np.max(err - bound))
    # zero blocks are exact; a block holding the tensor's amax gets the top scale 448
    assert np.all(deq[d == 0] == 0)
    am = np.max(np.abs(xf))
    if q.g > 2.0 ** -120:
        i, j = np.unravel_index(np.argmax(np.abs(xf)), xf.shape)
        assert q.sf[i, j // 16] == 0x7E


def test_nearest_code_is_optimal(orc):
    """Brute force on small tensors: every code is a nearest E2M1 value of q = x*r (FP32)."""
    x = synth.ragged(3, 40, 64, "outliers")
    st, q = orc.quantize(x)
    xf = x.to(torch.float32).numpy()
    codes = _unpack(q.codes, 64)
    d = (E4M3[q.sf].astype(np.float32) * np.float32(q.g)).astype(np.float32)
    for i in range(40):
        for b in range(4):
            if d[i, b] == 0:
                assert not codes[i, 16 * b:16 * b + 16].any()
                continue
            r = np.float32(1.0) / d[i, b]
            qq = (xf[i, 16 * b:16 * b + 16] * r).astype(np.float64)
            dist = np.abs(qq[:, None] - E2M1[None, :8] * np.sign(qq)[:, None])
            chosen = np.abs(qq - E2M1[codes[i, 16 * b:16 * b + 16]])
            assert np.all(chosen <= dist.min(axis=1) + 0.0)


def test_requantize_reproduces_codes_of_saturated_blocks(orc):
    x = synth.ragged(11, 32, 256, "normal")
    st, q = orc.quantize(x)
    amax = float(np.max(np.abs(x.to(torch.float32).numpy())))
    y = torch.from_numpy(orc.dequant(q).view(np.int16)).view(torch.bfloat16)
    st, q2 = orc.quantize(y, amax_in=amax)
    c1, c2 = _unpack(q.codes, 256), _unpack(q2.codes, 256)
    for i in range(32):
        for b in range(16):
            blk = c1[i, 16 * b:16 * b + 16]
            if np.any((blk & 7) == 7):
                assert q2.sf[i, b] == q.sf[i, b]
                assert np.array_equal(c2[i, 16 * b:16 * b + 16], blk)


@pytest.mark.parametrize("rows,cols", [(16, 32), (40, 24), (4680 // 10, 96), (37, 5)])
def test_colwise_is_rowwise_of_transpose(orc, rows, cols):
    x = synth.ragged(5, rows, cols, "lognormal")
    st, qc = orc.quantize(x, colwise=True)
    st2, qr = orc.quantize(x.t().contiguous())
    assert st == st2 == 0
    assert np.array_equal(qc.codes, qr.codes) and np.array_equal(qc.sf, qr.sf) and qc.g == qr.g
    assert qc.rows == cols and qc.cols == rows
    # a trailing partial block (rows % 16 != 0) is zero-padded: padded codes stay 0
    if rows % 16:
        c = _unpack(qc.codes, qc.codes.shape[1] * 2)
        assert not c[:, rows:].any()


def test_dequant_is_fp32_product_then_bf16(orc):
    """Dequant = BF16(FP32(e2m1*sf) * g): checked against torch's FP32 multiply and BF16 cast."""
    x = synth.ragged(9, 64, 512, "wide")
    st, q = orc.quantize(x)
    c = _unpack(q.codes, 512)
    prod = (E2M1[c] * np.repeat(E4M3[q.sf], 16, axis=1)).astype(np.float32)   # exact
    ref = (torch.from_numpy(prod) * torch.tensor(np.float32(q.g))).to(torch.bfloat16)
    ours = orc.dequant(q)
    assert np.array_equal(ours, ref.view(torch.int16).numpy().view(np.uint16))


def test_kv_model_append_then_dequant(orc):
    kv = orc.KVCacheModel(layers=2, heads=4, head_dim=32, slots=3, slot_tokens=20)
    chunks = [synth.kv_chunk(0, s, tokens=20)[0][:, :4, :32].contiguous() for s in range(3)]
    for s, k in enumerate(chunks):
        assert kv.append(1, s, k, k) == 0
    K, V = kv.dequant(1, [2, 0])
    for part, s in zip((K[:20], K[20:]), (2, 0)):
        st, q = orc.quantize(chunks[s].reshape(20, 128))
        assert np.array_equal(part.reshape(20, 128), orc.dequant(q))
    assert np.array_equal(K, V)
