"""CPU oracle for the Mix-Quant NVFP4 prefill linear and the BF16 decode linear.

TEST INFRASTRUCTURE ONLY: only ``tests/``, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline / reference leg may import this package.  The product
library never imports it, and it imports nothing from the product package.

The arithmetic lives in ``mq_oracle.c`` (plain scalar C, binary32/binary64
steps written out, compiled with ``-ffp-contract=off``); this module only
builds it with gcc and marshals numpy arrays through ctypes.  Each wrapper
names the step of the method it follows; the citations are in the C source.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "mq_oracle.c")
_LIB = os.path.join(_HERE, "libmq_oracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (OpenMP over independent rows only)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp",
               "-ffp-contract=off", "-fno-fast-math", "-o", _LIB, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(_LIB)
            P = ctypes.c_void_p
            I64 = ctypes.c_int64
            lib.mqo_e2m1_decode.restype = ctypes.c_double
            lib.mqo_e2m1_decode.argtypes = [ctypes.c_int]
            lib.mqo_e4m3_decode.restype = ctypes.c_double
            lib.mqo_e4m3_decode.argtypes = [ctypes.c_int]
            lib.mqo_bf16_to_float.restype = ctypes.c_float
            lib.mqo_bf16_to_float.argtypes = [ctypes.c_uint16]
            lib.mqo_float_to_bf16_rne.restype = ctypes.c_uint16
            lib.mqo_float_to_bf16_rne.argtypes = [ctypes.c_float]
            lib.mqo_e4m3_encode_satfinite.restype = ctypes.c_int
            lib.mqo_e4m3_encode_satfinite.argtypes = [ctypes.c_float]
            lib.mqo_e2m1_encode_satfinite.restype = ctypes.c_int
            lib.mqo_e2m1_encode_satfinite.argtypes = [ctypes.c_float]
            lib.mqo_tensor_amax.restype = ctypes.c_float
            lib.mqo_tensor_amax.argtypes = [P, I64, I64, I64]
            lib.mqo_tensor_scale.restype = ctypes.c_float
            lib.mqo_tensor_scale.argtypes = [ctypes.c_float]
            lib.mqo_quantize.restype = None
            lib.mqo_quantize.argtypes = [P, I64, I64, I64, ctypes.c_float, P, P]
            lib.mqo_sf_swizzled_bytes.restype = I64
            lib.mqo_sf_swizzled_bytes.argtypes = [I64, I64]
            lib.mqo_sf_swizzled_offset.restype = I64
            lib.mqo_sf_swizzled_offset.argtypes = [I64, I64, I64]
            lib.mqo_sf_swizzle.restype = None
            lib.mqo_sf_swizzle.argtypes = [P, I64, I64, P]
            lib.mqo_sf_unswizzle.restype = None
            lib.mqo_sf_unswizzle.argtypes = [P, I64, I64, P]
            lib.mqo_gemm_nvfp4.restype = None
            lib.mqo_gemm_nvfp4.argtypes = [P, P, ctypes.c_float, P, I64, P, P, ctypes.c_float,
                                           I64, I64, P, P]
            lib.mqo_decode_linear.restype = None
            lib.mqo_decode_linear.argtypes = [P, I64, P, I64, I64, P, P]
            lib.mqo_swiglu.restype = None
            lib.mqo_swiglu.argtypes = [P, P, I64, P]
            lib.mqo_double_to_bf16_rne.restype = ctypes.c_uint16
            lib.mqo_double_to_bf16_rne.argtypes = [ctypes.c_double]
            lib.mqo_rmsnorm.restype = None
            lib.mqo_rmsnorm.argtypes = [P, I64, I64, I64, P, ctypes.c_double, P]
            lib.mqo_attention.restype = None
            lib.mqo_attention.argtypes = [P, I64, P, I64, I64, P, I64, I64, I64, I64, I64, I64,
                                          ctypes.c_double, P, I64, P, P]
            lib.mqo_set_threads.restype = None
            lib.mqo_set_threads.argtypes = [ctypes.c_int]
            lib.mqo_threads_used.restype = ctypes.c_int
            lib.mqo_threads_used.argtypes = []
            _lib = lib
    return _lib


def _ptr(a: np.ndarray) -> int:
    assert a.flags["C_CONTIGUOUS"], "oracle buffers must be C-contiguous"
    return a.ctypes.data


def _u16(x) -> np.ndarray:
    """Accept a numpy uint16 array or a CPU torch bfloat16 tensor (bit view)."""
    if isinstance(x, np.ndarray):
        assert x.dtype == np.uint16
        return np.ascontiguousarray(x)
    import torch  # local: the oracle itself needs only numpy
    assert x.dtype == torch.bfloat16 and x.device.type == "cpu"
    return np.ascontiguousarray(x.contiguous().view(torch.int16).numpy().view(np.uint16))


# -- thread control ---------------------------------------------------------

def set_threads(n: int) -> None:
    _load().mqo_set_threads(int(n))


def threads_used() -> int:
    return int(_load().mqo_threads_used())


# -- number formats -----------------------------------------------------------

def e2m1_decode(code: int) -> float:
    return float(_load().mqo_e2m1_decode(int(code)))


def e4m3_decode(byte: int) -> float:
    return float(_load().mqo_e4m3_decode(int(byte)))


def bf16_to_float(bits: int) -> float:
    return float(_load().mqo_bf16_to_float(int(bits)))


def float_to_bf16(v: float) -> int:
    return int(_load().mqo_float_to_bf16_rne(float(v)))


def e4m3_encode(v: float) -> int:
    return int(_load().mqo_e4m3_encode_satfinite(float(v)))


def e2m1_encode(v: float) -> int:
    return int(_load().mqo_e2m1_encode_satfinite(float(v)))


# -- tensor scale and quantization ---------------------------------------------

def tensor_amax(x) -> float:
    """max |x| over a 2-D BF16 matrix (tensor-level scale input)."""
    a = _u16(x)
    rows, cols = a.shape
    return float(_load().mqo_tensor_amax(_ptr(a), rows, cols, cols))


def tensor_scale(amax: float) -> float:
    """s_enc = fp32(2688 / amax), 1.0 for an all-zero tensor."""
    return float(_load().mqo_tensor_scale(float(amax)))


def quantize(x, s_enc: float):
    """NVFP4-quantize a BF16 matrix [rows, cols] with a given tensor scale.

    Returns (codes uint8 [rows, cols/2], sf uint8 [rows, cols/16] row-major).
    """
    a = _u16(x)
    rows, cols = a.shape
    assert cols % 16 == 0
    codes = np.zeros((rows, cols // 2), dtype=np.uint8)
    sf = np.zeros((rows, cols // 16), dtype=np.uint8)
    _load().mqo_quantize(_ptr(a), rows, cols, cols, float(s_enc), _ptr(codes), _ptr(sf))
    return codes, sf


def quantize_tensor(x):
    """amax -> s_enc -> quantize.  Returns (codes, sf_rowmajor, s_enc, amax)."""
    amax = tensor_amax(x)
    s = tensor_scale(amax)
    codes, sf = quantize(x, s)
    return codes, sf, s, amax


def sf_swizzled_bytes(rows: int, kblocks: int) -> int:
    return int(_load().mqo_sf_swizzled_bytes(rows, kblocks))


def sf_swizzled_offset(r: int, c: int, kblocks: int) -> int:
    return int(_load().mqo_sf_swizzled_offset(r, c, kblocks))


def sf_swizzle(sf: np.ndarray) -> np.ndarray:
    sf = np.ascontiguousarray(sf, dtype=np.uint8)
    rows, kb = sf.shape
    out = np.zeros(sf_swizzled_bytes(rows, kb), dtype=np.uint8)
    _load().mqo_sf_swizzle(_ptr(sf), rows, kb, _ptr(out))
    return out


def sf_unswizzle(swz: np.ndarray, rows: int, kblocks: int) -> np.ndarray:
    swz = np.ascontiguousarray(swz, dtype=np.uint8)
    assert swz.size >= sf_swizzled_bytes(rows, kblocks)
    out = np.zeros((rows, kblocks), dtype=np.uint8)
    _load().mqo_sf_unswizzle(_ptr(swz), rows, kblocks, _ptr(out))
    return out


# -- GEMM, decode, SwiGLU -------------------------------------------------------

def gemm_nvfp4(a_codes, a_sf, a_s_enc, b_codes, b_sf, b_s_enc, rows=None):
    """Exact block-scaled product Y = alpha * sum(deq products) for the given A
    rows (all rows if None).  Returns (y float64 [len(rows), N], p float64)."""
    a_codes = np.ascontiguousarray(a_codes, dtype=np.uint8)
    b_codes = np.ascontiguousarray(b_codes, dtype=np.uint8)
    a_sf = np.ascontiguousarray(a_sf, dtype=np.uint8)
    b_sf = np.ascontiguousarray(b_sf, dtype=np.uint8)
    M, K = a_codes.shape[0], a_codes.shape[1] * 2
    N = b_codes.shape[0]
    assert b_codes.shape[1] * 2 == K
    idx = np.arange(M, dtype=np.int64) if rows is None else np.ascontiguousarray(rows, dtype=np.int64)
    y = np.zeros((idx.size, N), dtype=np.float64)
    p = np.zeros((idx.size, N), dtype=np.float64)
    _load().mqo_gemm_nvfp4(_ptr(a_codes), _ptr(a_sf), float(a_s_enc), _ptr(idx), idx.size,
                           _ptr(b_codes), _ptr(b_sf), float(b_s_enc), N, K, _ptr(y), _ptr(p))
    return y, p


def decode_linear(x, w):
    """BF16 decode linear in float64: returns (y [M, N], p [M, N])."""
    xa = _u16(x)
    wa = _u16(w)
    M, K = xa.shape
    N = wa.shape[0]
    y = np.zeros((M, N), dtype=np.float64)
    p = np.zeros((M, N), dtype=np.float64)
    _load().mqo_decode_linear(_ptr(xa), M, _ptr(wa), N, K, _ptr(y), _ptr(p))
    return y, p


def swiglu(g, u) -> np.ndarray:
    """h = bf16(SiLU(g) * u) in binary32; returns uint16 bf16 bits."""
    ga = _u16(g)
    ua = _u16(u)
    assert ga.shape == ua.shape
    h = np.zeros(ga.shape, dtype=np.uint16)
    _load().mqo_swiglu(_ptr(ga), _ptr(ua), ga.size, _ptr(h))
    return h


def double_to_bf16(v: float) -> int:
    """One binary64 -> BF16 round-to-nearest-even; returns the bit pattern."""
    return int(_load().mqo_double_to_bf16_rne(float(v)))


def rmsnorm(x, gamma, eps: float) -> np.ndarray:
    """y = bf16(gamma * bf16(x / sqrt(mean(x^2) + eps))) per row, binary64
    (the RMSNorm in front of a prefill linear); returns uint16 bf16 bits."""
    xa = _u16(x)
    ga = _u16(gamma)
    rows, cols = xa.shape
    assert ga.shape == (cols,)
    y = np.zeros((rows, cols), dtype=np.uint16)
    _load().mqo_rmsnorm(_ptr(xa), rows, cols, cols, _ptr(ga), float(eps), _ptr(y))
    return y


# -- attention of the prefill layer / decode step ------------------------------

def attention(q, k, v, H: int, Hkv: int, D: int, pos0: int = 0, rows=None, scale=None):
    """Causal grouped-query softmax attention in binary64 (mqo_attention).

    q: BF16 [n_q, H*D] (query i at absolute position pos0 + i); k, v: BF16
    [n_k, Hkv*D] with n_k >= pos0 + n_q (key j at position j).  Returns
    (o float64 [len(rows), H, D], a float64 [len(rows), H, D]) for the query
    rows (all if None); a = the softmax-weighted |v|."""
    qa, ka, va = _u16(q), _u16(k), _u16(v)
    n_q = qa.shape[0]
    assert qa.shape[1] == H * D and ka.shape[1] == Hkv * D and va.shape[1] == Hkv * D
    assert ka.shape[0] >= pos0 + n_q and va.shape[0] >= pos0 + n_q and H % Hkv == 0
    idx = np.arange(n_q, dtype=np.int64) if rows is None else np.ascontiguousarray(rows, dtype=np.int64)
    out = np.zeros((idx.size, H, D), dtype=np.float64)
    a = np.zeros((idx.size, H, D), dtype=np.float64)
    sc = (1.0 / np.sqrt(D)) if scale is None else float(scale)
    _load().mqo_attention(_ptr(qa), H * D, _ptr(ka), Hkv * D, D, _ptr(va), Hkv * D, D, pos0, H, Hkv,
                          D, sc, _ptr(idx), idx.size, _ptr(out), _ptr(a))
    return out, a
