"""ctypes binding for libmq (include/mq.h): same entry-point names, argument
marshalling only.  Every step of the path runs in libmq's CUDA kernels; if the
library is missing this module raises -- there is no fallback.

Tensors are torch CUDA tensors (only their data pointers are passed); the
stream defaults to torch's current stream on the current device.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libmq.so")

MQ_AMAX_PARTIALS_MAX = 4096
STATUS = {0: "MQ_OK", 1: "MQ_ERR_INVALID_ARG", 2: "MQ_ERR_SHAPE", 3: "MQ_ERR_ALIGNMENT",
          4: "MQ_ERR_UNSUPPORTED_DEVICE", 5: "MQ_ERR_OOM", 6: "MQ_ERR_CUDA", 7: "MQ_ERR_TIMEOUT"}

# (name, restype, argtypes) for every symbol declared in include/mq.h
_P, _I64, _SZ, _I, _U8P = ctypes.c_void_p, ctypes.c_int64, ctypes.c_size_t, ctypes.c_int, ctypes.c_void_p
SIGNATURES = [
    ("mq_status_string", ctypes.c_char_p, [_I]),
    ("mq_check", _I, [_P]),
    ("mq_selftest_bounded_wait", _I, [ctypes.c_uint32, _P]),
    ("mq_weight_pack", _I, [_P, _I64, _I64, _P, ctypes.POINTER(_P)]),
    ("mq_weight_free", _I, [_P]),
    ("mq_weight_views", _I, [_P, ctypes.POINTER(_I64), ctypes.POINTER(_I64), ctypes.POINTER(_P),
                             ctypes.POINTER(_P), ctypes.POINTER(_P), ctypes.POINTER(_P)]),
    ("mq_sf_bytes", _SZ, [_I64, _I64]),
    ("mq_tensor_amax", _I, [_P, _I64, _I64, _I64, _P, ctypes.POINTER(_I), _P]),
    ("mq_amax_combine", _I, [_P, _I, _P, _P]),
    ("mq_quantize_nvfp4", _I, [_P, _I64, _I64, _I64, _U8P, _U8P, _P, _P, _I, _P, _SZ, _P]),
    ("mq_gemm_nvfp4", _I, [_U8P, _U8P, _P, _I64, _P, _P, _I64, _P]),
    ("mq_gemm_nvfp4_swiglu", _I, [_U8P, _U8P, _P, _I64, _P, _P, _P, ctypes.POINTER(_I), _P]),
    ("mq_workspace_bytes", _SZ, [_I64, _I64]),
    ("mq_prefill_linear_nvfp4", _I, [_P, _P, _I64, _P, _P, _SZ, _P]),
    ("mq_mlp_workspace_bytes", _SZ, [_I64, _I64, _I64]),
    ("mq_prefill_mlp_swiglu_nvfp4", _I, [_P, _P, _P, _I64, _P, _P, _P, _SZ, _P]),
    ("mq_prefill_linear_nvfp4_noalloc", _I, [_P, _P, _I64, _P, _P]),
    ("mq_decode_linear_bf16", _I, [_P, _P, _I64, _P, _P]),
    ("mq_decode_linear_nvfp4", _I, [_P, _P, _I64, _P, _P, _SZ, _P]),
    ("mq_rmsnorm_amax", _I, [_P, _P, ctypes.c_float, _I64, _I64, _I64, _P, _P, ctypes.POINTER(_I), _P]),
    ("mq_prefill_linear_rmsnorm_nvfp4", _I, [_P, _P, _P, ctypes.c_float, _I64, _P, _P, _P, _SZ, _P]),
    ("mq_attention_prefill_bf16", _I, [_P, _I64, _I64, _I64, _I64, _P, _P, _I64, _P, _P,
                                       ctypes.POINTER(_I), _P]),
    ("mq_attention_decode_workspace_bytes", _SZ, [_I64, _I64, _I64, _I64, _I64]),
    ("mq_attention_decode_bf16", _I, [_P, _I64, _I64, _I64, _I64, _I64, _P, _P, _I64, _P, _P, _SZ,
                                      _P]),
]

_lib = None


class MqError(RuntimeError):
    def __init__(self, fn: str, code: int):
        super().__init__(f"{fn} failed: {STATUS.get(code, code)}")
        self.code = code


def lib():
    """Loads libmq.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"libmq.so is not built ({LIB_PATH}); run __graft_entry__.build()")
        l = ctypes.CDLL(LIB_PATH)
        for name, res, args in SIGNATURES:
            f = getattr(l, name)
            f.restype = res
            f.argtypes = args
        _lib = l
    return _lib


def _ptr(t) -> Optional[int]:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _ok(fn: str, code: int) -> None:
    if code != 0:
        raise MqError(fn, code)


def mq_status_string(code: int) -> str:
    return lib().mq_status_string(code).decode()


def mq_check(stream=None) -> int:
    """Synchronizes the stream; returns the status (0 or MQ_ERR_*), does not raise."""
    return lib().mq_check(_stream(stream))


def mq_selftest_bounded_wait(limit_us: int, stream=None) -> None:
    _ok("mq_selftest_bounded_wait", lib().mq_selftest_bounded_wait(limit_us, _stream(stream)))


def mq_weight_pack(w_bf16, N: int, K: int, stream=None) -> int:
    h = ctypes.c_void_p()
    _ok("mq_weight_pack", lib().mq_weight_pack(_ptr(w_bf16), N, K, _stream(stream), ctypes.byref(h)))
    return h.value


def mq_weight_free(handle: int) -> None:
    _ok("mq_weight_free", lib().mq_weight_free(handle))


def mq_weight_views(handle: int) -> dict:
    n, k = ctypes.c_int64(), ctypes.c_int64()
    b, c, s, e = ctypes.c_void_p(), ctypes.c_void_p(), ctypes.c_void_p(), ctypes.c_void_p()
    _ok("mq_weight_views", lib().mq_weight_views(handle, ctypes.byref(n), ctypes.byref(k),
                                                 ctypes.byref(b), ctypes.byref(c),
                                                 ctypes.byref(s), ctypes.byref(e)))
    return {"N": n.value, "K": k.value, "bf16": b.value, "codes": c.value, "sf": s.value,
            "s_enc": e.value}


def mq_sf_bytes(rows: int, K: int) -> int:
    return int(lib().mq_sf_bytes(rows, K))


def mq_workspace_bytes(M: int, K: int) -> int:
    return int(lib().mq_workspace_bytes(M, K))


def mq_mlp_workspace_bytes(M: int, K: int, I: int) -> int:
    return int(lib().mq_mlp_workspace_bytes(M, K, I))


def mq_tensor_amax(x, M: int, K: int, ldx: int, amax_partials, stream=None) -> int:
    n = ctypes.c_int()
    _ok("mq_tensor_amax", lib().mq_tensor_amax(_ptr(x), M, K, ldx, _ptr(amax_partials),
                                               ctypes.byref(n), _stream(stream)))
    return n.value


def mq_amax_combine(amax_partials, n_partials: int, amax_out, stream=None) -> None:
    _ok("mq_amax_combine", lib().mq_amax_combine(_ptr(amax_partials), n_partials, _ptr(amax_out),
                                                 _stream(stream)))


def mq_quantize_nvfp4(x, M: int, K: int, ldx: int, codes, sf_swizzled, s_enc, amax_partials=None,
                      n_partials: int = 0, workspace=None, ws_bytes: int = 0, stream=None) -> None:
    _ok("mq_quantize_nvfp4", lib().mq_quantize_nvfp4(
        _ptr(x), M, K, ldx, _ptr(codes), _ptr(sf_swizzled), _ptr(s_enc), _ptr(amax_partials),
        n_partials, _ptr(workspace), ws_bytes, _stream(stream)))


def mq_gemm_nvfp4(a_codes, a_sf, a_s_enc, M: int, weight: int, y, ldy: int, stream=None) -> None:
    _ok("mq_gemm_nvfp4", lib().mq_gemm_nvfp4(_ptr(a_codes), _ptr(a_sf), _ptr(a_s_enc), M, weight,
                                             _ptr(y), ldy, _stream(stream)))


def mq_gemm_nvfp4_swiglu(a_codes, a_sf, a_s_enc, M: int, weight: int, h, h_amax_partials,
                         stream=None) -> int:
    n = ctypes.c_int()
    _ok("mq_gemm_nvfp4_swiglu", lib().mq_gemm_nvfp4_swiglu(
        _ptr(a_codes), _ptr(a_sf), _ptr(a_s_enc), M, weight, _ptr(h), _ptr(h_amax_partials),
        ctypes.byref(n), _stream(stream)))
    return n.value


def mq_prefill_linear_nvfp4(weight: int, x, M: int, y, workspace, ws_bytes: int, stream=None) -> None:
    _ok("mq_prefill_linear_nvfp4", lib().mq_prefill_linear_nvfp4(
        weight, _ptr(x), M, _ptr(y), _ptr(workspace), ws_bytes, _stream(stream)))


def mq_prefill_mlp_swiglu_nvfp4(w_gate_up: int, w_down: int, x, M: int, y, h, workspace,
                                ws_bytes: int, stream=None) -> None:
    _ok("mq_prefill_mlp_swiglu_nvfp4", lib().mq_prefill_mlp_swiglu_nvfp4(
        w_gate_up, w_down, _ptr(x), M, _ptr(y), _ptr(h), _ptr(workspace), ws_bytes,
        _stream(stream)))


def mq_prefill_linear_nvfp4_noalloc(weight: int, x, M: int, y, stream=None) -> None:
    _ok("mq_prefill_linear_nvfp4_noalloc", lib().mq_prefill_linear_nvfp4_noalloc(
        weight, _ptr(x), M, _ptr(y), _stream(stream)))


def mq_decode_linear_bf16(weight: int, x, M: int, y, stream=None) -> None:
    _ok("mq_decode_linear_bf16", lib().mq_decode_linear_bf16(weight, _ptr(x), M, _ptr(y),
                                                             _stream(stream)))


def mq_decode_linear_nvfp4(weight: int, x, M: int, y, workspace, ws_bytes: int,
                           stream=None) -> None:
    _ok("mq_decode_linear_nvfp4", lib().mq_decode_linear_nvfp4(
        weight, _ptr(x), M, _ptr(y), _ptr(workspace), ws_bytes, _stream(stream)))


def mq_rmsnorm_amax(x, gamma, eps: float, M: int, K: int, ldx: int, y, amax_partials,
                    stream=None) -> int:
    """Returns the number of partial maxima written."""
    n = ctypes.c_int()
    _ok("mq_rmsnorm_amax", lib().mq_rmsnorm_amax(
        _ptr(x), _ptr(gamma), float(eps), M, K, ldx, _ptr(y), _ptr(amax_partials),
        ctypes.byref(n), _stream(stream)))
    return n.value


def mq_prefill_linear_rmsnorm_nvfp4(weight: int, r, gamma, eps: float, M: int, xn, y, workspace,
                                    ws_bytes: int, stream=None) -> None:
    _ok("mq_prefill_linear_rmsnorm_nvfp4", lib().mq_prefill_linear_rmsnorm_nvfp4(
        weight, _ptr(r), _ptr(gamma), float(eps), M, _ptr(xn), _ptr(y), _ptr(workspace), ws_bytes,
        _stream(stream)))


class Weight:
    """Owns one mq_weight handle (BF16 + NVFP4 copies of a [N, K] matrix)."""

    def __init__(self, w_bf16, stream=None):
        assert w_bf16.is_cuda and w_bf16.is_contiguous()
        self.N, self.K = w_bf16.shape
        self.handle = mq_weight_pack(w_bf16, self.N, self.K, stream)

    def views(self) -> dict:
        return mq_weight_views(self.handle)

    def free(self) -> None:
        if self.handle:
            mq_weight_free(self.handle)
            self.handle = 0

    def __del__(self):
        try:
            self.free()
        except Exception:
            pass


def mq_attention_prefill_bf16(qkv, M: int, H: int, Hkv: int, D: int, k_cache, v_cache, S_max: int,
                              o, o_amax_partials, stream=None) -> int:
    """Returns the number of partial maxima written."""
    n = ctypes.c_int()
    _ok("mq_attention_prefill_bf16", lib().mq_attention_prefill_bf16(
        _ptr(qkv), M, H, Hkv, D, _ptr(k_cache), _ptr(v_cache), S_max, _ptr(o), _ptr(o_amax_partials),
        ctypes.byref(n), _stream(stream)))
    return n.value


def mq_attention_decode_workspace_bytes(m: int, pos0: int, H: int, Hkv: int, D: int) -> int:
    return lib().mq_attention_decode_workspace_bytes(m, pos0, H, Hkv, D)


def mq_attention_decode_bf16(qkv, m: int, pos0: int, H: int, Hkv: int, D: int, k_cache, v_cache,
                             S_max: int, o, workspace, ws_bytes: int, stream=None) -> None:
    _ok("mq_attention_decode_bf16", lib().mq_attention_decode_bf16(
        _ptr(qkv), m, pos0, H, Hkv, D, _ptr(k_cache), _ptr(v_cache), S_max, _ptr(o), _ptr(workspace),
        ws_bytes, _stream(stream)))
