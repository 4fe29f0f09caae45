"""Python binding of the NVFP4 W4A4 / NVFP4 KV-cache library (libnvfp4.so, sm_100a).

Argument marshalling only: every step of the path runs in the CUDA kernels behind the C ABI of
``include/nvfp4.h``.  PyTorch provides device memory and the current stream.  There is no CPU
fallback: if ``libnvfp4.so`` cannot be loaded, every call raises.

Entry points (same names as the C ABI):
  nvfp4_amax(x)                               -> float32 device tensor [1]
  nvfp4_quantize(x, dir=ROWWISE, ...)         -> QTensor (codes, sf, g on the device)
  nvfp4_gemm(A, B, bias=None, resid=None, ...) -> BF16 (or FP32) [M, N]
  kv_quant_append(cache, layer, slot, k, v)   in place into a KVCache
  kv_dequant(cache, layer, slots)             -> (K, V) BF16 [tokens, heads, head_dim]
  kv_attention(cache, layer, slots, q, scale) -> O BF16 [tq, heads, head_dim] (restore fused)
"""
from __future__ import annotations

import ctypes
import os
import re

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
# NVFP4_LIB selects another build of the same library (e.g. the bounds-checked debug build,
# libnvfp4_checked.so); the default is the in-tree release build.
LIB_PATH = os.environ.get("NVFP4_LIB") or os.path.join(HERE, "libnvfp4.so")
HEADER = os.path.join(os.path.dirname(HERE), "include", "nvfp4.h")

NVFP4_OK, NVFP4_ERR_INVALID_ARG, NVFP4_ERR_UNSUPPORTED = 0, 1, 2
NVFP4_ERR_NONFINITE, NVFP4_ERR_TIMEOUT, NVFP4_ERR_CUDA, NVFP4_ERR_OUT_OF_BOUNDS = 3, 4, 5, 6
ROWWISE, COLWISE, ROWCOL = 0, 1, 2
SF_LINEAR, SF_MMA = 0, 1
OUT_BF16, OUT_F32 = 0, 1

_P = ctypes.c_void_p
_I32, _I64, _SZ = ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t


class NVFP4Error(RuntimeError):
    def __init__(self, fn, status, detail=""):
        self.status = status
        msg = f"{fn} failed: status {status}"
        if _lib is not None:
            msg += f" ({_lib.nvfp4_status_string(status).decode()})"
        if detail:
            msg += f": {detail}"
        super().__init__(msg)


class _Tensor(ctypes.Structure):
    _fields_ = [("codes", _P), ("sf", _P), ("g", _P), ("rows", _I64), ("cols", _I64), ("sf_layout", _I32)]


class _KVCache(ctypes.Structure):
    _fields_ = [("layers", _I32), ("heads", _I32), ("head_dim", _I32), ("slots", _I32), ("slot_tokens", _I32),
                ("codes_k", _P), ("codes_v", _P), ("sf_k", _P), ("sf_v", _P), ("g_k", _P), ("g_v", _P),
                ("len", ctypes.POINTER(_I32))]


_lib = None


def lib():
    """Load libnvfp4.so (raises if it is missing: there is no fallback path)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is not built; run `python -m bit_kv_cache_24_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        sig = {
            "nvfp4_version": (_I32, []),
            "nvfp4_checked_build": (_I32, []),
            "nvfp4_status_string": (ctypes.c_char_p, [_I32]),
            "nvfp4_last_error": (ctypes.c_char_p, []),
            "nvfp4_codes_pitch": (_I64, [_I64]),
            "nvfp4_sf_bytes": (_I64, [_I64, _I64, _I32]),
            "nvfp4_quantize_workspace": (_SZ, [_I64, _I64]),
            "nvfp4_kv_append_workspace": (_SZ, [_I64, _I32, _I32]),
            "nvfp4_amax": (_I32, [_P, _I64, _I64, _I64, _P, _P, _SZ, _P, _P]),
            "nvfp4_quantize": (_I32, [_P, _I64, _I64, _I64, _I32, _P, ctypes.POINTER(_Tensor), _P, _SZ, _P, _P]),
            "nvfp4_quantize_noalloc": (_I32, [_P, _I64, _I64, _I64, _I32, ctypes.POINTER(_Tensor), _P, _P]),
            "nvfp4_gemm": (_I32, [ctypes.POINTER(_Tensor), ctypes.POINTER(_Tensor), _P, _P, _P, _I64, _I32, _P, _P]),
            "nvfp4_gemm_quant_out": (_I32, [ctypes.POINTER(_Tensor), ctypes.POINTER(_Tensor), _P, _P, _P, _I64, _P,
                                            ctypes.POINTER(_Tensor), _P, _SZ, _P, _P]),
            "nvfp4_gemm_colamax_workspace": (_SZ, [_I64, _I64]),
            "nvfp4_gemm_colamax": (_I32, [ctypes.POINTER(_Tensor), ctypes.POINTER(_Tensor), _P, _P, _P, _I64, _I64, _P,
                                          _P, _SZ, _P, _P]),
            "nvfp4_kv_cache_bytes": (_I64, [_I32, _I32, _I32, _I32, _I32, _I32]),
            "kv_quant_append": (_I32, [ctypes.POINTER(_KVCache), _I32, _I32, _P, _P, _I64, _I64, _P, _SZ, _P, _P]),
            "kv_quant_append_amax": (_I32, [ctypes.POINTER(_KVCache), _I32, _I32, _P, _P, _I64, _I64, _P, _P, _SZ, _P,
                                            _P]),
            "kv_dequant": (_I32, [ctypes.POINTER(_KVCache), _I32, ctypes.POINTER(_I32), _I32, _P, _P, _P, _P]),
            "nvfp4_sf_to_linear": (_I32, [_P, _I64, _I64, _P]),
            "nvfp4_sf_to_mma": (_I32, [_P, _I64, _I64, _P]),
            "kv_attention": (_I32, [ctypes.POINTER(_KVCache), _I32, ctypes.POINTER(_I32), _I32, _P, _I64, _I64,
                                    ctypes.c_float, _P, _I64, _P, _P]),
            "nvfp4_encode_elements": (_I32, [_P, _I64, _P, _P, _P]),
            "nvfp4_selftest_wait_timeout": (_I32, [_P, _I64, _P]),
            "nvfp4_selftest_bounds": (_I32, [_P, _I64, _I64, _P, _P]),
        }
        for name, (res, args) in sig.items():
            f = getattr(L, name)
            f.restype, f.argtypes = res, args
        _lib = L
    return _lib


def header_functions() -> list[str]:
    """Names of the functions include/nvfp4.h declares."""
    src = open(HEADER).read()
    return re.findall(r"^NVFP4_API\s+[\w\s\*]*?\b(\w+)\s*\(", src, flags=re.M)


def _check(fn, status):
    if status != NVFP4_OK:
        detail = lib().nvfp4_last_error().decode() if status == NVFP4_ERR_CUDA else ""
        raise NVFP4Error(fn, status, detail)


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


_checked = None
_checked_status = {}      # device index -> int32 status word of the binding (checked build only)


def checked_build() -> bool:
    """True when the loaded library is the bounds-checked debug build (NVFP4_LIB selects it)."""
    global _checked
    if _checked is None:
        _checked = bool(lib().nvfp4_checked_build())
    return _checked


def _status(status):
    """The caller's status word; in the checked build, when the caller passes none, a per-device
    word of the binding's own, which checked_status() reads back."""
    if status is not None or not checked_build():
        return _ptr(status)
    dev = torch.cuda.current_device()
    t = _checked_status.get(dev)
    if t is None:
        t = _checked_status[dev] = torch.zeros(1, dtype=torch.int32, device=torch.device("cuda", dev))
    return _ptr(t)


def checked_status(reset: bool = True) -> int:
    """Checked build: the first nonzero code the kernels wrote to the binding's own status words
    (calls made without a status argument), 0 if none; synchronizes each device first."""
    code = 0
    for dev, t in _checked_status.items():
        with torch.cuda.device(dev):
            torch.cuda.synchronize()
            v = int(t.item())
            if reset:
                t.zero_()
        code = code or v
    return code


def _ws(nbytes, device):
    # workspace: a plain device buffer; the library never allocates
    return torch.empty(int(nbytes), dtype=torch.uint8, device=device)


def _bf16_2d(x, name):
    if not (isinstance(x, torch.Tensor) and x.is_cuda and x.dtype == torch.bfloat16 and x.dim() == 2):
        raise TypeError(f"{name} must be a 2-D bfloat16 CUDA tensor")
    if x.stride(1) != 1:
        raise ValueError(f"{name} must be contiguous along its last dimension")
    return x


class QTensor:
    """An NVFP4 matrix on the device: codes [rows, pitch] u8, sf (layout-dependent) u8, g [1] f32."""

    def __init__(self, rows, cols, sf_layout=SF_MMA, device="cuda"):
        L = lib()
        self.rows, self.cols, self.sf_layout = int(rows), int(cols), int(sf_layout)
        self.codes = torch.empty((self.rows, L.nvfp4_codes_pitch(self.cols)), dtype=torch.uint8, device=device)
        self.sf = torch.empty(L.nvfp4_sf_bytes(self.rows, self.cols, self.sf_layout), dtype=torch.uint8, device=device)
        self.g = torch.empty(1, dtype=torch.float32, device=device)

    def struct(self):
        return _Tensor(self.codes.data_ptr(), self.sf.data_ptr(), self.g.data_ptr(), self.rows, self.cols,
                       self.sf_layout)

    def nbytes(self):
        return self.codes.numel() + self.sf.numel() + 4


def nvfp4_amax(x, out=None, ws=None, status=None, stream=None):
    x = _bf16_2d(x, "x")
    L = lib()
    M, K = x.shape
    out = torch.empty(1, dtype=torch.float32, device=x.device) if out is None else out
    nws = L.nvfp4_quantize_workspace(M, K)
    ws = _ws(nws, x.device) if ws is None else ws
    _check("nvfp4_amax", L.nvfp4_amax(_ptr(x), M, K, x.stride(0), _ptr(out), _ptr(ws), ws.numel(), _status(status),
                                      _stream(stream)))
    return out


def nvfp4_quantize(x, dir=ROWWISE, amax_in=None, out=None, sf_layout=SF_MMA, ws=None, status=None, stream=None):
    """BF16 [M, K] -> NVFP4.  Row-wise: out is [M, K]; column-wise: out is [K, M] (blocks along M);
    ROWCOL: both from one read, out = (row-wise [M, K], column-wise [K, M])."""
    x = _bf16_2d(x, "x")
    L = lib()
    M, K = x.shape
    if out is None:
        if dir == ROWWISE:
            out = QTensor(M, K, sf_layout, x.device)
        elif dir == COLWISE:
            out = QTensor(K, M, sf_layout, x.device)
        else:
            out = (QTensor(M, K, sf_layout, x.device), QTensor(K, M, sf_layout, x.device))
    if ws is None:
        ws = _ws(L.nvfp4_quantize_workspace(M, K), x.device)
    outs = out if isinstance(out, tuple) else (out,)
    st = (_Tensor * len(outs))(*[o.struct() for o in outs])
    _check("nvfp4_quantize", L.nvfp4_quantize(_ptr(x), M, K, x.stride(0), dir, _ptr(amax_in), st,
                                              _ptr(ws), 0 if ws is None else ws.numel(), _status(status),
                                              _stream(stream)))
    return out


def nvfp4_gemm(A: QTensor, B: QTensor, bias=None, resid=None, out=None, out_dtype=OUT_BF16, status=None,
               stream=None):
    """Y = gA*gB * A . B^T (+bias | +resid); returns Y [M, N] (BF16, or FP32 with OUT_F32)."""
    L = lib()
    M, N = A.rows, B.rows
    if out is None:
        out = torch.empty((M, N), dtype=torch.float32 if out_dtype == OUT_F32 else torch.bfloat16,
                          device=A.codes.device)
    sa, sb = A.struct(), B.struct()
    _check("nvfp4_gemm", L.nvfp4_gemm(ctypes.byref(sa), ctypes.byref(sb), _ptr(bias), _ptr(resid), _ptr(out),
                                      out.stride(0), out_dtype, _status(status), _stream(stream)))
    return out


def nvfp4_gemm_quant_out(A: QTensor, B: QTensor, amax_in, bias=None, resid=None, out=None, q_out=None,
                         sf_layout=SF_MMA, write_y=True, ws=None, status=None, stream=None):
    """Y = gA*gB * A . B^T (+bias | +resid) in BF16 and, from the same epilogue, its row-wise NVFP4
    quantization with the scale of amax_in (a device float).  Returns (Y or None, q_out)."""
    L = lib()
    M, N = A.rows, B.rows
    if out is None and write_y:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=A.codes.device)
    if q_out is None:
        q_out = QTensor(M, N, sf_layout, A.codes.device)
    if ws is None:
        ws = _ws(L.nvfp4_quantize_workspace(M, N), A.codes.device)
    ldy = out.stride(0) if out is not None else (resid.stride(0) if resid is not None else N)
    sa, sb, sq = A.struct(), B.struct(), q_out.struct()
    _check("nvfp4_gemm_quant_out", L.nvfp4_gemm_quant_out(ctypes.byref(sa), ctypes.byref(sb), _ptr(bias), _ptr(resid),
                                                          _ptr(out), ldy, _ptr(amax_in), ctypes.byref(sq), _ptr(ws),
                                                          ws.numel(), _status(status), _stream(stream)))
    return out, q_out


def nvfp4_gemm_colamax(A: QTensor, B: QTensor, group_cols, bias=None, resid=None, out=None, amax_out=None,
                       ws=None, status=None, stream=None):
    """Y = gA*gB * A . B^T (+bias | +resid) in BF16 and max |Y| per group of group_cols columns
    (reduced in the epilogue).  Returns (Y, amax_out [N / group_cols] float32 on the device)."""
    L = lib()
    M, N = A.rows, B.rows
    dev = A.codes.device
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    if amax_out is None:
        amax_out = torch.empty(N // group_cols, dtype=torch.float32, device=dev)
    if ws is None:
        ws = _ws(L.nvfp4_gemm_colamax_workspace(M, N), dev)
    sa, sb = A.struct(), B.struct()
    _check("nvfp4_gemm_colamax", L.nvfp4_gemm_colamax(ctypes.byref(sa), ctypes.byref(sb), _ptr(bias), _ptr(resid),
                                                      _ptr(out), out.stride(0), group_cols, _ptr(amax_out), _ptr(ws),
                                                      ws.numel(), _status(status), _stream(stream)))
    return out, amax_out


class KVCache:
    """Caller-owned chunk-slot NVFP4 KV cache storage (device arrays + host slot lengths)."""

    def __init__(self, layers, heads, head_dim, slots, slot_tokens, device="cuda"):
        L = lib()
        self.layers, self.heads, self.head_dim = layers, heads, head_dim
        self.slots, self.slot_tokens = slots, slot_tokens
        nb = [L.nvfp4_kv_cache_bytes(layers, heads, head_dim, slots, slot_tokens, w) for w in range(3)]
        if min(nb) < 0:
            raise ValueError("bad KV cache geometry")
        self.codes_k = torch.empty(nb[0], dtype=torch.uint8, device=device)
        self.codes_v = torch.empty(nb[0], dtype=torch.uint8, device=device)
        self.sf_k = torch.empty(nb[1], dtype=torch.uint8, device=device)
        self.sf_v = torch.empty(nb[1], dtype=torch.uint8, device=device)
        self.g_k = torch.empty(layers * slots, dtype=torch.float32, device=device)
        self.g_v = torch.empty(layers * slots, dtype=torch.float32, device=device)
        self.len = (_I32 * (layers * slots))()
        self._c = _KVCache(layers, heads, head_dim, slots, slot_tokens, self.codes_k.data_ptr(),
                           self.codes_v.data_ptr(), self.sf_k.data_ptr(), self.sf_v.data_ptr(),
                           self.g_k.data_ptr(), self.g_v.data_ptr(), ctypes.cast(self.len, ctypes.POINTER(_I32)))
        self.ws = _ws(L.nvfp4_kv_append_workspace(slot_tokens, heads, head_dim), device)

    def nbytes(self):
        return 2 * (self.codes_k.numel() + self.sf_k.numel() + self.g_k.numel() * 4)

    def slot_len(self, layer, slot):
        return self.len[layer * self.slots + slot]


def kv_quant_append(cache: KVCache, layer, slot, k, v, status=None, stream=None, amax_kv=None):
    """Quantize one chunk's K and V ([ntok, heads, head_dim] or [ntok, heads*head_dim] BF16, rows
    possibly strided) into slot `slot` of `layer` in place.  amax_kv: optional device float[2]
    (amax of K, of V), e.g. from nvfp4_gemm_colamax; then no amax pass runs."""
    row = cache.heads * cache.head_dim
    k2 = k.reshape(k.shape[0], row) if k.dim() == 3 else k
    v2 = v.reshape(v.shape[0], row) if v.dim() == 3 else v
    _bf16_2d(k2, "k")
    _bf16_2d(v2, "v")
    if k2.stride(0) != v2.stride(0) or k2.shape != v2.shape:
        raise ValueError("k and v must have the same shape and row stride")
    if amax_kv is None:
        _check("kv_quant_append", lib().kv_quant_append(ctypes.byref(cache._c), layer, slot, _ptr(k2), _ptr(v2),
                                                        k2.shape[0], k2.stride(0), _ptr(cache.ws), cache.ws.numel(),
                                                        _status(status), _stream(stream)))
    else:
        _check("kv_quant_append_amax", lib().kv_quant_append_amax(ctypes.byref(cache._c), layer, slot, _ptr(k2),
                                                                  _ptr(v2), k2.shape[0], k2.stride(0), _ptr(amax_kv),
                                                                  _ptr(cache.ws), cache.ws.numel(), _status(status),
                                                                  _stream(stream)))


def kv_dequant(cache: KVCache, layer, slots, k_out=None, v_out=None, status=None, stream=None):
    """Restore the listed slots of `layer` to BF16 [tokens, heads, head_dim] (K, V)."""
    slots = [int(s) for s in slots]
    tokens = sum(cache.slot_len(layer, s) for s in slots)
    shape = (tokens, cache.heads, cache.head_dim)
    dev = cache.codes_k.device
    k_out = torch.empty(shape, dtype=torch.bfloat16, device=dev) if k_out is None else k_out
    v_out = torch.empty(shape, dtype=torch.bfloat16, device=dev) if v_out is None else v_out
    arr = (_I32 * len(slots))(*slots)
    _check("kv_dequant", lib().kv_dequant(ctypes.byref(cache._c), layer, arr, len(slots), _ptr(k_out), _ptr(v_out),
                                          _status(status), _stream(stream)))
    return k_out, v_out


def kv_attention(cache: KVCache, layer, slots, q, scale, out=None, status=None, stream=None):
    """Softmax attention of q over the listed slots of `layer`, the restore fused into the kernel.

    q: BF16 CUDA tensor [tq, heads, head_dim], or a 2-D [tq, >= heads * head_dim] view with unit
    column stride (e.g. the Q columns of a fused QKV output). Returns O, BF16 [tq, heads, head_dim]
    (or `out`, with the same shape rules)."""
    def rows(t, name):
        if not (isinstance(t, torch.Tensor) and t.is_cuda and t.dtype == torch.bfloat16):
            raise TypeError(f"{name} must be a bfloat16 CUDA tensor")
        if t.dim() == 3 and tuple(t.shape[1:]) == (cache.heads, cache.head_dim) and \
                t.stride(2) == 1 and t.stride(1) == cache.head_dim:
            return t.shape[0], t.stride(0)
        if t.dim() == 2 and t.shape[1] == cache.heads * cache.head_dim and t.stride(1) == 1:
            return t.shape[0], t.stride(0)
        raise ValueError(f"{name} must be [tq, heads, head_dim] with contiguous rows")
    tq, ldq = rows(q, "q")
    if out is None:
        out = torch.empty(tq, cache.heads, cache.head_dim, dtype=torch.bfloat16, device=q.device)
    to, ldo = rows(out, "out")
    if to != tq:
        raise ValueError("out must have q's row count")
    slots = [int(s) for s in slots]
    arr = (_I32 * len(slots))(*slots)
    _check("kv_attention", lib().kv_attention(ctypes.byref(cache._c), layer, arr, len(slots), _ptr(q), tq, ldq,
                                              float(scale), _ptr(out), ldo, _status(status), _stream(stream)))
    return out


def sf_to_linear(q: QTensor) -> torch.Tensor:
    """The scales of q as a host [rows, ceil(cols/16)] uint8 table (linear layout)."""
    sf = q.sf.cpu().contiguous()
    if q.sf_layout == SF_LINEAR:
        return sf.view(q.rows, -1)
    out = torch.empty(q.rows, (q.cols + 15) // 16, dtype=torch.uint8)
    _check("nvfp4_sf_to_linear", lib().nvfp4_sf_to_linear(_ptr(sf), q.rows, q.cols, _ptr(out)))
    return out


def encode_elements(x, stream=None):
    """Test support: the CUDA path's E2M1 code of each FP32 x and E4M3 byte of |x|."""
    assert x.is_cuda and x.dtype == torch.float32
    x = x.contiguous().view(-1)
    e2 = torch.empty(x.numel(), dtype=torch.uint8, device=x.device)
    e4 = torch.empty(x.numel(), dtype=torch.uint8, device=x.device)
    _check("nvfp4_encode_elements", lib().nvfp4_encode_elements(_ptr(x), x.numel(), _ptr(e2), _ptr(e4),
                                                                _stream(stream)))
    return e2, e4


def selftest_wait_timeout(limit_ns=1_000_000, device="cuda"):
    """Test support: a bounded wait that must give up; returns the device status word."""
    st = torch.zeros(1, dtype=torch.int32, device=device)
    _check("nvfp4_selftest_wait_timeout", lib().nvfp4_selftest_wait_timeout(_ptr(st), limit_ns, _stream(None)))
    torch.cuda.synchronize()
    return int(st.item())
