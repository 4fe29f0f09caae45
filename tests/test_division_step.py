"""The quantizer's shortcut for the block-scale quotient, checked on the host.

The CUDA quantizer computes the scale quotient q = RN(b / den) of the published NVFP4 format
(b = block max, a BF16 value; den = 6 g) without an IEEE division:
    y = RN(1 / den),  q0 = RN(b * y),  q = RN(q0 + RN(b - q0 * den) * y)   (both steps fused)
which is the last step of Markstein's division.  It is used only when b >= 2^-100 and
den >= 2^-125 (the residual then stays normal); other blocks divide.  This test emulates those
FP32 steps exactly in float64 (a product of two FP32 values and the sums involved are exact
there, so one final rounding to FP32 reproduces each fused operation) for every positive finite
BF16 b against a spread of den values, and requires the quotient to equal RN(b / den).
"""
import numpy as np
import pytest


def _rn32(x64):
    return x64.astype(np.float32)


def _dens(rng):
    d = np.concatenate([
        rng.uniform(1e-6, 10.0, 60),
        2.0 ** rng.uniform(-125.0, 60.0, 60),
        np.array([6.0, 6.0 / 2688.0, 1.0, 3.0, 2.0 ** -125, 448.0 * 6.0]),
    ]).astype(np.float32)
    return d[(d >= np.float32(2.0 ** -125)) & np.isfinite(d)]


@pytest.mark.parametrize("seed", [0, 1])
def test_markstein_step_equals_rounded_quotient(seed):
    rng = np.random.default_rng(seed)
    bits = np.arange(1, 0x7F80, dtype=np.uint32)              # positive finite BF16 (with subnormals)
    b32 = (bits << 16).view(np.float32)
    b32 = b32[b32 >= np.float32(2.0 ** -100)]
    b = b32.astype(np.float64)
    checked = 0
    for den in _dens(rng):
        den64 = np.float64(den)
        y = np.float64(_rn32(np.float64(1.0) / den64))
        exact = b / den64
        keep = exact <= 449.0                                  # quotients the quantizer can see
        if not keep.any():
            continue
        q_true = _rn32(exact[keep])
        bk = b[keep]
        q0 = _rn32(bk * y).astype(np.float64)
        r = _rn32(bk - q0 * den64).astype(np.float64)          # fma(-q0, den, b)
        q = _rn32(q0 + r * y)                                  # fma(r, y, q0)
        bad = np.nonzero(q != q_true)[0]
        assert bad.size == 0, (float(den), float(bk[bad[0]]), float(q[bad[0]]), float(q_true[bad[0]]))
        checked += bk.size
    assert checked > 1_000_000
