"""Pins for the oracle's number formats against sources other than the oracle itself.

E2M1 / E4M3 / BF16 are not defined numerically on the pages (landx.limxdynamics.com, section
"什么是 NVFP4?", only names NVFP4 as Blackwell's 4-bit float).  The reading is the OCP format
definition; the independent references here are torch's float8_e4m3fn and bfloat16 casts and
ml_dtypes' float4_e2m1fn / float8_e4m3fn casts (all round-to-nearest-even), plus literal tables.
"""
import ml_dtypes
import numpy as np
import pytest
import torch


def _sweep_f32(n_stride, lo_bits=0, hi_bits=0x7F800000):
    bits = np.arange(lo_bits, hi_bits, n_stride, dtype=np.uint64).astype(np.uint32)
    return bits.view(np.float32)


def _midpoints_and_neighbours(values):
    """Exact midpoints of adjacent values plus the fp32 numbers just below/above them."""
    v = np.asarray(sorted(set(values)), dtype=np.float64)
    mids = ((v[:-1] + v[1:]) / 2).astype(np.float32)
    out = [mids, np.nextafter(mids, np.float32(-np.inf)), np.nextafter(mids, np.float32(np.inf)),
           v.astype(np.float32)]
    return np.concatenate(out)


def test_e2m1_decode_table(orc):
    # OCP MX E2M1 magnitudes, literal
    mags = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
    for c in range(8):
        assert orc.e2m1_value(c) == mags[c]
        v = orc.e2m1_value(c | 8)
        assert v == -mags[c] and np.signbit(v)
    # and against ml_dtypes' decoder
    table = np.arange(16, dtype=np.uint8).view(ml_dtypes.float4_e2m1fn).astype(np.float32)
    assert np.array_equal(table, np.array([orc.e2m1_value(c) for c in range(16)], np.float32))


def test_e4m3_decode_table(orc):
    ours = np.array([orc.e4m3_value(b) for b in range(256)], dtype=np.float64)
    ref_t = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    ref_m = np.arange(256, dtype=np.uint8).view(ml_dtypes.float8_e4m3fn).astype(np.float64)
    for ref in (ref_t, ref_m):
        assert np.array_equal(np.isnan(ours), np.isnan(ref))
        ok = ~np.isnan(ref)
        assert np.array_equal(ours[ok], ref[ok])
    assert np.isnan(ours[0x7F]) and np.isnan(ours[0xFF])
    # spot values of the format
    assert orc.e4m3_value(0x7E) == 448.0
    assert orc.e4m3_value(0x79) == 288.0
    assert orc.e4m3_value(0x08) == 2.0 ** -6
    assert orc.e4m3_value(0x01) == 2.0 ** -9


def test_e4m3_encode_matches_torch(orc):
    finite = [orc.e4m3_value(b) for b in range(0x7F)]
    x = np.concatenate([
        _sweep_f32(911),                                         # dense over all positive fp32
        _midpoints_and_neighbours(finite),
        np.array([448.0, 464.0, 465.0, 480.0, 1e6, 2.0 ** -10, 2.0 ** -11], np.float32),
    ]).astype(np.float32)
    x = np.concatenate([x, -x])
    ours = orc.e4m3_encode_array(x)
    # torch's cast does not saturate: clamp to the max finite first (RNE of a clamped value is
    # the satfinite result because everything above 448 rounds to 448 or overflows)
    ref = torch.from_numpy(np.clip(x, -448.0, 448.0)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    bad = np.nonzero(ours != ref)[0]
    assert bad.size == 0, [(float(x[i]), int(ours[i]), int(ref[i])) for i in bad[:10]]
    assert orc.e4m3_encode(float("inf")) == 0x7E
    assert orc.e4m3_encode(float("-inf")) == 0xFE


def test_e2m1_encode_matches_ml_dtypes(orc):
    grid = [orc.e2m1_value(c) for c in range(8)]
    x = np.concatenate([
        _sweep_f32(1021),
        _midpoints_and_neighbours(grid),
        np.array([6.0, 6.5, 7.0, 1e30, np.inf, 0.0, 1e-45], np.float32),
    ]).astype(np.float32)
    x = np.concatenate([x, -x])
    ours = orc.e2m1_encode_array(x)
    ref = x.astype(ml_dtypes.float4_e2m1fn).view(np.uint8) & 0xF
    bad = np.nonzero(ours != ref)[0]
    assert bad.size == 0, [(float(x[i]), int(ours[i]), int(ref[i])) for i in bad[:10]]


def test_e2m1_ties_and_saturation_literal(orc):
    # exact midpoints go to the even code (OCP: round to nearest, ties to even)
    cases = {0.25: 0x0, 0.75: 0x2, 1.25: 0x2, 1.75: 0x4, 2.5: 0x4, 3.5: 0x6, 5.0: 0x6,
             6.0: 0x7, 6.22: 0x7, 1e9: 0x7, -0.1: 0x8, -0.25: 0x8, -0.75: 0xA, 0.2500001: 0x1}
    for q, c in cases.items():
        assert orc.e2m1_encode(q) == c, q
    assert orc.e2m1_encode(float("nan")) == 0x0          # reading: NaN products encode as +0


def test_bf16_rne_matches_torch(orc):
    rng = np.random.default_rng(0)
    hi = rng.integers(0, 1 << 16, size=200_000, dtype=np.uint32) << 16
    low = np.array([0x0000, 0x7FFF, 0x8000, 0x8001, 0xFFFF, 0x1234], dtype=np.uint32)
    bits = (hi[:, None] | low[None, :]).ravel()
    x = bits.view(np.float32)
    x = x[~np.isnan(x)]
    ours = orc.bf16_from_float_array(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    bad = np.nonzero(ours != ref)[0]
    assert bad.size == 0, [(float(x[i]), hex(ours[i]), hex(ref[i])) for i in bad[:10]]


@pytest.mark.parametrize("rows,cols", [(1, 16), (128, 64), (130, 80), (300, 1000)])
def test_sf_mma_layout_is_a_padded_bijection(orc, rows, cols):
    nb = orc.sf_pitch(cols)
    offs = np.array([[orc.lib().orc_sf_mma_offset(i, b, cols) for b in range(nb)] for i in range(rows)])
    total = orc.sf_mma_bytes(rows, cols)
    assert offs.min() >= 0 and offs.max() < total
    assert len(np.unique(offs)) == rows * nb
    assert total % 512 == 0


def test_sf_mma_layout_literal_offsets(orc):
    # 128x4 atoms of 512 bytes: row i -> (i%32)*16 + ((i%128)/32)*4, block b -> b%4, atoms
    # ordered block-column fastest (tcgen05 scale-factor layout of the PTX ISA)
    off = orc.lib().orc_sf_mma_offset
    assert off(0, 0, 64) == 0
    assert off(0, 1, 64) == 1
    assert off(1, 0, 64) == 16
    assert off(32, 0, 64) == 4
    assert off(33, 2, 64) == 22
    assert off(127, 3, 64) == 511
    assert off(0, 4, 128) == 512          # next block-column atom
    assert off(128, 0, 128) == 1024       # next row atom, after the 2 block-column atoms
    assert off(200, 5, 128) == 1024 + 512 + (200 % 32) * 16 + ((200 % 128) // 32) * 4 + 1
