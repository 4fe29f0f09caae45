"""GPU parity of the element encoders (hardware cvt E2M1 / E4M3) against the oracle's
definition-based encoders, on a dense FP32 sweep including every tie point."""
import numpy as np
import pytest
import torch

import bit_kv_cache_24_b200 as nv

pytestmark = pytest.mark.gpu


def _sweep():
    bits = np.arange(0, 0x7F800000, 613, dtype=np.uint64).astype(np.uint32)
    x = bits.view(np.float32)
    grid = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6], np.float64)
    mids = ((grid[:-1] + grid[1:]) / 2).astype(np.float32)
    e4 = np.array([2.0 ** -9 * k for k in range(1, 8)] + [2.0 ** e * (1 + m / 8) for e in range(-6, 9) for m in range(8)])
    e4 = np.sort(e4[e4 <= 448])
    e4m = ((e4[:-1] + e4[1:]) / 2).astype(np.float32)
    pts = np.concatenate([mids, e4m, e4.astype(np.float32), grid.astype(np.float32)])
    near = np.concatenate([pts, np.nextafter(pts, np.float32(0)), np.nextafter(pts, np.float32(np.inf))])
    x = np.concatenate([x, near, np.array([np.inf, 448, 464, 465, 1e30], np.float32)])
    return np.concatenate([x, -x]).astype(np.float32)


def test_encoders_match_oracle(orc):
    x = _sweep()
    e2, e4 = nv.encode_elements(torch.from_numpy(x).cuda())
    e2, e4 = e2.cpu().numpy(), e4.cpu().numpy()
    want2 = orc.e2m1_encode_array(x)
    want4 = orc.e4m3_encode_array(np.abs(x))
    bad = np.nonzero(e2 != want2)[0]
    assert bad.size == 0, [(float(x[i]), int(e2[i]), int(want2[i])) for i in bad[:8]]
    bad = np.nonzero(e4 != want4)[0]
    assert bad.size == 0, [(float(x[i]), int(e4[i]), int(want4[i])) for i in bad[:8]]


def test_bounded_wait_gives_up_and_reports_timeout():
    assert nv.selftest_wait_timeout(limit_ns=2_000_000) == nv.NVFP4_ERR_TIMEOUT
    # the context is still usable afterwards
    x = torch.ones(4, device="cuda")
    assert float(x.sum()) == 4.0
