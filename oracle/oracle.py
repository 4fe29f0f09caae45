"""Python face of the CPU oracle (test infrastructure only).

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg may import this
module.  It loads ``oracle/liboracle.so`` (plain C, see nvfp4_oracle.c for the reading of the
format it follows) and wraps it for numpy / torch-CPU tensors.  It never touches the CUDA
library.

Parity status: every function here is pinned by ``tests/test_oracle_*.py`` (format tables against
torch and ml_dtypes, worked examples in ``tests/golden/``, invariants, brute force).  Nothing here
is "parity unpinned".
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from concurrent.futures import ThreadPoolExecutor

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "nvfp4_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

ORC_OK = 0
ORC_NONFINITE = 3

_P = ctypes.c_void_p
_I64 = ctypes.c_int64


def build(force: bool = False) -> str:
    """Compile the oracle with strict IEEE single-precision semantics (no contraction)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        subprocess.check_call([
            "gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared",
            "-o", _LIB, _SRC, "-lm",
        ])
    return _LIB


_lib = None


def lib():
    global _lib
    if _lib is None:
        L = ctypes.CDLL(build())
        L.orc_e2m1_value.restype = ctypes.c_double
        L.orc_e2m1_value.argtypes = [ctypes.c_int]
        L.orc_e4m3_value.restype = ctypes.c_double
        L.orc_e4m3_value.argtypes = [ctypes.c_int]
        L.orc_e2m1_encode.restype = ctypes.c_uint8
        L.orc_e2m1_encode.argtypes = [ctypes.c_float]
        L.orc_e4m3_encode.restype = ctypes.c_uint8
        L.orc_e4m3_encode.argtypes = [ctypes.c_float]
        L.orc_bf16_from_float.restype = ctypes.c_uint16
        L.orc_bf16_from_float.argtypes = [ctypes.c_float]
        L.orc_bf16_to_float.restype = ctypes.c_float
        L.orc_bf16_to_float.argtypes = [ctypes.c_uint16]
        L.orc_global_scale.restype = ctypes.c_float
        L.orc_global_scale.argtypes = [ctypes.c_float]
        for f in ("orc_codes_pitch", "orc_sf_pitch"):
            getattr(L, f).restype = _I64
            getattr(L, f).argtypes = [_I64]
        L.orc_sf_mma_bytes.restype = _I64
        L.orc_sf_mma_bytes.argtypes = [_I64, _I64]
        L.orc_sf_mma_offset.restype = _I64
        L.orc_sf_mma_offset.argtypes = [_I64, _I64, _I64]
        L.orc_sf_linear_to_mma.restype = None
        L.orc_sf_linear_to_mma.argtypes = [_P, _I64, _I64, _P]
        L.orc_amax.restype = ctypes.c_int
        L.orc_amax.argtypes = [_P, _I64, _I64, _I64, _P]
        for f in ("orc_quantize_rows", "orc_quantize_cols"):
            getattr(L, f).restype = ctypes.c_int
            getattr(L, f).argtypes = [_P, _I64, _I64, _I64, _P, _P, _P, _P]
        L.orc_dequant.restype = None
        L.orc_dequant.argtypes = [_P, _P, ctypes.c_float, _I64, _I64, _P, _I64]
        L.orc_dequant_f64.restype = None
        L.orc_dequant_f64.argtypes = [_P, _P, ctypes.c_float, _I64, _I64, _P]
        for f in ("orc_e2m1_encode_n", "orc_e4m3_encode_n", "orc_bf16_from_float_n"):
            getattr(L, f).restype = None
            getattr(L, f).argtypes = [_P, _I64, _P]
        L.orc_gemm_rows.restype = None
        L.orc_gemm_rows.argtypes = [_P, _P, ctypes.c_float, _P, _I64, _I64, _P, _P, _I64, _P, _I64, _P]
        _lib = L
    return _lib


def _ptr(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(_P)


def as_u16(x) -> np.ndarray:
    """BF16 torch tensor (CPU) or uint16 numpy array -> contiguous uint16 numpy array."""
    if hasattr(x, "view") and hasattr(x, "dtype") and str(x.dtype) == "torch.bfloat16":
        import torch
        return x.contiguous().view(torch.int16).numpy().view(np.uint16)
    return np.ascontiguousarray(x, dtype=np.uint16)


# ---- scalar codecs ---------------------------------------------------------------------------

def e2m1_value(code: int) -> float:
    return lib().orc_e2m1_value(code)


def e4m3_value(byte: int) -> float:
    return lib().orc_e4m3_value(byte)


def e2m1_encode(q: float) -> int:
    return lib().orc_e2m1_encode(q)


def e4m3_encode(v: float) -> int:
    return lib().orc_e4m3_encode(v)


def bf16_from_float(f: float) -> int:
    return lib().orc_bf16_from_float(f)


def _encode_n(fn, x, dtype):
    x = np.ascontiguousarray(x, dtype=np.float32).ravel()
    out = np.empty(x.size, dtype=dtype)
    fn(_ptr(x), x.size, _ptr(out))
    return out


def e2m1_encode_array(q) -> np.ndarray:
    return _encode_n(lib().orc_e2m1_encode_n, q, np.uint8)


def e4m3_encode_array(v) -> np.ndarray:
    return _encode_n(lib().orc_e4m3_encode_n, v, np.uint8)


def bf16_from_float_array(f) -> np.ndarray:
    return _encode_n(lib().orc_bf16_from_float_n, f, np.uint16)


def global_scale(amax: float) -> float:
    return lib().orc_global_scale(amax)


# ---- layouts ---------------------------------------------------------------------------------

def codes_pitch(cols: int) -> int:
    return lib().orc_codes_pitch(cols)


def sf_pitch(cols: int) -> int:
    return lib().orc_sf_pitch(cols)


def sf_mma_bytes(rows: int, cols: int) -> int:
    return lib().orc_sf_mma_bytes(rows, cols)


def sf_linear_to_mma(sf: np.ndarray, rows: int, cols: int) -> np.ndarray:
    sf = np.ascontiguousarray(sf, dtype=np.uint8)
    out = np.empty(sf_mma_bytes(rows, cols), dtype=np.uint8)
    lib().orc_sf_linear_to_mma(_ptr(sf), rows, cols, _ptr(out))
    return out


# ---- quantize / dequantize -------------------------------------------------------------------

class Quantized:
    """codes [rows, codes_pitch(cols)] u8, sf [rows, sf_pitch(cols)] u8 (linear), g float32."""

    def __init__(self, codes, sf, g, rows, cols):
        self.codes, self.sf, self.g, self.rows, self.cols = codes, sf, np.float32(g), rows, cols

    def sf_mma(self) -> np.ndarray:
        return sf_linear_to_mma(self.sf, self.rows, self.cols)


def amax(x) -> tuple[int, float]:
    xu = as_u16(x)
    rows, cols = xu.shape
    out = np.zeros(1, dtype=np.float32)
    st = lib().orc_amax(_ptr(xu), rows, cols, cols, _ptr(out))
    return st, float(out[0])


def quantize(x, colwise: bool = False, amax_in: float | None = None):
    """Row-wise (blocks along the contiguous dim) or column-wise (blocks along rows) NVFP4
    quantization of a BF16 [rows, cols] tensor.  Returns (status, Quantized)."""
    xu = as_u16(x)
    rows, cols = xu.shape
    orows, ocols = (cols, rows) if colwise else (rows, cols)
    codes = np.zeros((orows, codes_pitch(ocols)), dtype=np.uint8)
    sf = np.zeros((orows, sf_pitch(ocols)), dtype=np.uint8)
    g = np.zeros(1, dtype=np.float32)
    am = None if amax_in is None else np.array([amax_in], dtype=np.float32)
    fn = lib().orc_quantize_cols if colwise else lib().orc_quantize_rows
    st = fn(_ptr(xu), rows, cols, cols, None if am is None else _ptr(am), _ptr(codes), _ptr(sf), _ptr(g))
    return st, Quantized(codes, sf, g[0], orows, ocols)


def dequant(q: Quantized) -> np.ndarray:
    """BF16 bits (uint16) [rows, cols]."""
    y = np.empty((q.rows, q.cols), dtype=np.uint16)
    lib().orc_dequant(_ptr(q.codes), _ptr(q.sf), float(q.g), q.rows, q.cols, _ptr(y), q.cols)
    return y


def dequant_f64(q: Quantized) -> np.ndarray:
    y = np.empty((q.rows, q.cols), dtype=np.float64)
    lib().orc_dequant_f64(_ptr(q.codes), _ptr(q.sf), float(q.g), q.rows, q.cols, _ptr(y))
    return y


def bf16_bits_to_f32(u: np.ndarray) -> np.ndarray:
    return (np.asarray(u, dtype=np.uint32) << 16).view(np.float32)


# ---- GEMM ------------------------------------------------------------------------------------

def gemm_rows(A: Quantized, B: Quantized, rows=None, bias=None, resid=None, threads: int = 0):
    """fp64 reference Y[rows, N] = Adeq[rows] . Bdeq^T (+bias | +resid).  ``rows`` defaults to
    all rows of A.  Row chunks run on threads (ctypes releases the GIL); arithmetic per output
    element is the same plain sequential fp64 sum either way."""
    assert A.cols == B.cols
    M, N, K = A.rows, B.rows, A.cols
    rows = np.arange(M, dtype=np.int64) if rows is None else np.ascontiguousarray(rows, dtype=np.int64)
    bdeq = dequant_f64(B)
    b16 = None if bias is None else as_u16(bias)
    r16 = None if resid is None else as_u16(resid)
    y = np.empty((len(rows), N), dtype=np.float64)
    threads = threads or min(8, os.cpu_count() or 1)
    chunks = np.array_split(np.arange(len(rows)), max(1, min(threads, len(rows))))

    def run(idx):
        if len(idx) == 0:
            return
        sub = np.ascontiguousarray(rows[idx])
        out = np.empty((len(idx), N), dtype=np.float64)
        lib().orc_gemm_rows(_ptr(A.codes), _ptr(A.sf), float(A.g), _ptr(bdeq), N, K,
                            None if b16 is None else _ptr(b16),
                            None if r16 is None else _ptr(r16), N,
                            _ptr(sub), len(idx), _ptr(out))
        y[idx] = out

    with ThreadPoolExecutor(max_workers=len(chunks)) as ex:
        list(ex.map(run, chunks))
    return y


def gemm_full(A: Quantized, B: Quantized, bias=None, resid=None):
    """fp64 reference of every output, Y[M, N] = Adeq . Bdeq^T (+bias | +resid), for sizes where
    the per-row loop of gemm_rows would take hours on the host (K = 37440, 115 M outputs).

    Same definition as gemm_rows: the dequantized operands are exact in fp64 (dequant_f64), and
    the contraction is one library step, numpy's fp64 matmul.  Only the fp64 summation order
    differs from the plain sequential sum (relative differences ~1e-16 * sqrt(K), far below the
    1e-5 GEMM tolerance); tests/test_oracle_gemm.py checks the two against each other."""
    assert A.cols == B.cols
    y = dequant_f64(A) @ dequant_f64(B).T
    if bias is not None:
        y += bf16_bits_to_f32(as_u16(bias)).astype(np.float64)[None, :]
    if resid is not None:
        y += bf16_bits_to_f32(as_u16(resid)).astype(np.float64)
    return y


def bf16_from_f64(y) -> np.ndarray:
    """BF16 bits (uint16) of fp64 values rounded once, to nearest with ties to even (8 significant
    bits), without the detour through FP32 that would round twice.  Finite values in the BF16
    normal range; values beyond the BF16 range map to +-inf.  Used to compare a BF16 GEMM output
    with the rounding of the exact result."""
    y = np.asarray(y, dtype=np.float64)
    m, e = np.frexp(y)                                    # y = m * 2^e, 0.5 <= |m| < 1
    r = np.ldexp(np.rint(np.ldexp(m, 8)), e - 8)          # rint: ties to even
    with np.errstate(over="ignore"):
        f = r.astype(np.float32)                          # exact: 8 significant bits
    return (f.view(np.uint32) >> 16).astype(np.uint16)


# ---- KV cache model --------------------------------------------------------------------------

class KVCacheModel:
    """Chunk-slot NVFP4 KV cache: per (layer, slot) and for K and V separately, one row-wise
    quantized [tokens, heads*head_dim] chunk with its own per-tensor scale g."""

    def __init__(self, layers, heads, head_dim, slots, slot_tokens):
        self.layers, self.heads, self.head_dim = layers, heads, head_dim
        self.slots, self.slot_tokens = slots, slot_tokens
        self.store = {}

    def append(self, layer, slot, k, v):
        hd = self.heads * self.head_dim
        out = []
        for t in (k, v):
            st, q = quantize(as_u16(t).reshape(-1, hd))
            if st != ORC_OK:
                return st
            out.append(q)
        self.store[(layer, slot)] = tuple(out)
        return ORC_OK

    def dequant(self, layer, slots):
        ks, vs = [], []
        for s in slots:
            qk, qv = self.store[(layer, s)]
            ks.append(dequant(qk))
            vs.append(dequant(qv))
        shape = (-1, self.heads, self.head_dim)
        return np.concatenate(ks).reshape(shape), np.concatenate(vs).reshape(shape)

    def attention(self, layer, slots, q, scale, rows=None):
        """Attention of the queries q over the window of the listed slots: attention() over the
        BF16 K and V the window restores to."""
        k, v = self.dequant(layer, slots)
        return attention(q, k, v, scale, rows=rows)


# ---- attention over the restored KV window ---------------------------------------------------

def attention(q, k, v, scale, rows=None):
    """fp64 softmax attention over a restored KV window (LongLive-2.0 keeps the KV cache in NVFP4
    and restores it for attention: d9249.github.io review, section "핵심 아이디어 / 구조 / 동작
    방식"; arXiv abstract on fugumt.com).  For every head h and query row i:

        w_j      = exp(scale * <q[i, h, :], k[j, h, :]>)    over the window's tokens j
        O[i,h,:] = sum_j w_j v[j, h, :] / sum_j w_j

    q [Tq, H, D], k and v [Tk, H, D]: BF16 (torch CPU tensors or uint16 bit arrays), k and v as the
    window restores to (KVCacheModel.dequant); scale: the FP32 softmax scale (taken at its FP32
    value).  No mask: every query attends to every token of the window.  ``rows`` selects query
    rows (default all).  Returns fp64 [len(rows), H, D].  The per-row maximum of the exponent is
    subtracted before exp to keep it in range; it cancels in the ratio."""
    qf = bf16_bits_to_f32(as_u16(q)).astype(np.float64)
    kf = bf16_bits_to_f32(as_u16(k)).astype(np.float64)
    vf = bf16_bits_to_f32(as_u16(v)).astype(np.float64)
    if rows is not None:
        qf = qf[np.asarray(rows, dtype=np.int64)]
    tq, heads, d = qf.shape
    assert kf.shape[1:] == (heads, d) and vf.shape == kf.shape and kf.shape[0] > 0
    c = np.float64(np.float32(scale))
    out = np.empty((tq, heads, d), dtype=np.float64)
    for h in range(heads):
        e = (qf[:, h, :] @ kf[:, h, :].T) * c              # [tq, Tk] exponents
        e -= e.max(axis=1, keepdims=True)
        w = np.exp(e)
        out[:, h, :] = (w @ vf[:, h, :]) / w.sum(axis=1, keepdims=True)
    return out
