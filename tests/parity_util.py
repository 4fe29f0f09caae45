"""Helpers shared by the GPU parity tests (CPU oracle vs CUDA path on the same seeded inputs)."""
import numpy as np
import torch

import bit_kv_cache_24_b200 as nv


def gpu_bytes(t):
    return t.detach().cpu().numpy()


def assert_quantized_equal(orc, gq, oq, label=""):
    """Bit-exact: codes (all bytes, padding included), scales (in the GPU's layout, padding
    included) and the per-tensor scale g."""
    assert gq.rows == oq.rows and gq.cols == oq.cols
    g_gpu = np.float32(gq.g.item())
    assert g_gpu.view(np.uint32) == np.float32(oq.g).view(np.uint32), (label, g_gpu, oq.g)
    codes = gpu_bytes(gq.codes)
    bad = np.argwhere(codes != oq.codes)
    assert bad.size == 0, (label, "codes differ", bad[:5].tolist(), codes[tuple(bad[0])], oq.codes[tuple(bad[0])])
    want_sf = oq.sf_mma() if gq.sf_layout == nv.SF_MMA else oq.sf.reshape(-1)
    sf = gpu_bytes(gq.sf)
    bad = np.nonzero(sf != want_sf)[0]
    assert bad.size == 0, (label, "scales differ", bad[:5].tolist(), sf[bad[:5]].tolist(), want_sf[bad[:5]].tolist())


def gemm_tolerance(A_deq_max, B_deq_max, K):
    """max-abs bound: 1e-3 * sqrt(K) * max|Adeq| * max|Bdeq| (FP32 accumulation-order slack)."""
    return 1e-3 * np.sqrt(K) * A_deq_max * B_deq_max


def rel_fro(y, ref):
    return float(np.linalg.norm(y - ref) / max(np.linalg.norm(ref), 1e-300))
