"""Host-side checks of the C ABI: libmq.so builds, loads and exports every
symbol declared in include/mq.h; the binding declares the same set; argument
errors are reported before any device work.  No kernel runs here."""
import ctypes
import os
import re

import pytest

from nvfp4_quantized_prefill_b200 import binding, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def header_functions():
    src = open(os.path.join(ROOT, "include", "mq.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return set(re.findall(r"\b(mq_[a-z0-9_]+)\s*\(", src))


@pytest.fixture(scope="module")
def lib():
    build.build()
    return binding.lib()


def test_header_declares_expected_entry_points():
    names = header_functions()
    for n in ["mq_quantize_nvfp4", "mq_prefill_linear_nvfp4", "mq_decode_linear_bf16",
              "mq_weight_pack", "mq_weight_free", "mq_gemm_nvfp4", "mq_check"]:
        assert n in names


def debug_header_functions():
    src = open(os.path.join(ROOT, "include", "mq_debug.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return set(re.findall(r"\b(mq_[a-z0-9_]+)\s*\(", src))


def test_library_exports_every_header_symbol(lib):
    for name in header_functions() | debug_header_functions():
        assert hasattr(lib, name), name
        assert ctypes.cast(getattr(lib, name), ctypes.c_void_p).value


def test_debug_entry_point_checks_its_arguments_on_the_host(lib):
    f = lib.mq_debug_gemm_withhold_release
    f.restype = ctypes.c_int
    f.argtypes = [ctypes.c_void_p] * 3 + [ctypes.c_int64, ctypes.c_void_p, ctypes.c_void_p,
                                          ctypes.c_int64, ctypes.c_uint32, ctypes.c_void_p]
    assert debug_header_functions() == {"mq_debug_gemm_withhold_release"}
    assert not (debug_header_functions() & header_functions())   # not in the public header
    assert f(None, 16, 16, 8, 16, 16, 8, 20000, None) == 1       # null pointer
    assert f(16, 16, 16, 8, 16, 16, 8, 999, None) == 1           # wait limit below 1 ms
    assert f(16, 16, 16, 8, None, 16, 8, 20000, None) == 1       # no weight handle


def test_binding_covers_header(lib):
    assert {n for n, _, _ in binding.SIGNATURES} == header_functions()


def test_status_strings(lib):
    for code, name in binding.STATUS.items():
        assert binding.mq_status_string(code) == name


def test_size_queries(lib):
    # rows padded to 128, K/16 scales padded to a multiple of 4
    assert binding.mq_sf_bytes(128, 256) == 128 * 16
    assert binding.mq_sf_bytes(1, 64) == 128 * 4
    assert binding.mq_sf_bytes(200, 320) == 256 * 20
    assert binding.mq_sf_bytes(0, 64) == 0
    ws = binding.mq_workspace_bytes(8192, 4096)
    assert ws >= 8192 * 2048 + 8192 * 256 + 4 * binding.MQ_AMAX_PARTIALS_MAX
    assert binding.mq_workspace_bytes(0, 4096) == 0
    assert binding.mq_mlp_workspace_bytes(128, 256, 512) >= (
        binding.mq_workspace_bytes(128, 256) + 128 * 512 * 2 + binding.mq_workspace_bytes(128, 512))


def test_argument_errors_before_device_work(lib):
    L = lib
    # null pointers
    assert L.mq_prefill_linear_nvfp4(None, None, 8, None, None, 0, None) == 1
    assert L.mq_decode_linear_bf16(None, None, 1, None, None) == 1
    assert L.mq_gemm_nvfp4(None, None, None, 8, None, None, 8, None) == 1
    h = ctypes.c_void_p()
    assert L.mq_weight_pack(None, 64, 64, None, ctypes.byref(h)) == 1
    # shape errors: K not a multiple of 64, N < 1
    assert L.mq_weight_pack(16, 64, 100, None, ctypes.byref(h)) == 2
    assert L.mq_weight_pack(16, 0, 64, None, ctypes.byref(h)) == 2
    # misaligned weight pointer
    assert L.mq_weight_pack(17, 64, 64, None, ctypes.byref(h)) == 3
    n = ctypes.c_int()
    assert L.mq_tensor_amax(16, 0, 64, 64, 16, ctypes.byref(n), None) == 2
    assert L.mq_tensor_amax(24, 4, 64, 64, 16, ctypes.byref(n), None) == 3
    assert L.mq_quantize_nvfp4(16, 4, 96, 96, 16, 16, 16, None, 0, 16, 1 << 20, None) == 2
    assert L.mq_quantize_nvfp4(16, 4, 64, 64, 16, 16, 16, None, 0, None, 0, None) == 1
    assert L.mq_quantize_nvfp4(16, 4, 64, 64, 16, 16, 16, 16, 0, None, 0, None) == 1
    assert L.mq_weight_free(None) == 0
    assert L.mq_weight_views(None, None, None, None, None, None, None) == 1


def test_new_entry_points_reject_bad_arguments_on_the_host(lib):
    L = lib
    n = ctypes.c_int()
    # RMSNorm + amax: null pointers, negative eps, bad K, misaligned x
    assert L.mq_rmsnorm_amax(None, 16, ctypes.c_float(1e-5), 4, 64, 64, 16, 16, ctypes.byref(n), None) == 1
    assert L.mq_rmsnorm_amax(16, 16, ctypes.c_float(-1.0), 4, 64, 64, 16, 16, ctypes.byref(n), None) == 1
    assert L.mq_rmsnorm_amax(16, 16, ctypes.c_float(1e-5), 4, 60, 64, 16, 16, ctypes.byref(n), None) == 2
    assert L.mq_rmsnorm_amax(24, 16, ctypes.c_float(1e-5), 4, 64, 64, 16, 16, ctypes.byref(n), None) == 3
    assert L.mq_prefill_linear_rmsnorm_nvfp4(None, None, None, ctypes.c_float(1e-5), 4, None, None,
                                             None, 0, None) == 1
    # W4A4 decode and the failure-detection self-test
    assert L.mq_decode_linear_nvfp4(None, None, 1, None, None, 0, None) == 1
    assert L.mq_selftest_bounded_wait(0, None) == 1
    assert L.mq_selftest_bounded_wait(2000001, None) == 1
    # amax combine (token sharding): null pointers, count out of range, misalignment
    assert L.mq_amax_combine(None, 4, 16, None) == 1
    assert L.mq_amax_combine(16, 0, 16, None) == 1
    assert L.mq_amax_combine(16, 4097, 16, None) == 1
    assert L.mq_amax_combine(18, 4, 16, None) == 3


def test_amax_shape_bound_at_the_32_bit_edge(lib):
    """The amax kernel indexes the [M, K/8] vectors with 32-bit unsigned
    arithmetic, so the host accepts M * K / 8 < 2^32 - 1 and nothing larger.
    Just below the edge the call gets past the shape check and stops at the
    (deliberately misaligned) partials pointer; at the edge it is a shape
    error.  Neither reaches the device."""
    L = lib
    n = ctypes.c_int()
    below = (1 << 29) - 1          # M * 64 / 8 = 2^32 - 8
    assert below * 8 < (1 << 32) - 1
    assert L.mq_tensor_amax(16, below, 64, 64, 20, ctypes.byref(n), None) == 3
    assert L.mq_tensor_amax(16, 1 << 29, 64, 64, 20, ctypes.byref(n), None) == 2
    # the same edge with longer rows: K = 4096 -> 512 vectors a row
    rows = ((1 << 32) - 2) // 512  # largest M with M * 512 < 2^32 - 1
    assert L.mq_tensor_amax(16, rows, 4096, 4096, 20, ctypes.byref(n), None) == 3
    assert L.mq_tensor_amax(16, rows + 1, 4096, 4096, 20, ctypes.byref(n), None) == 2


def _dec_ws_expected(m, pos0, H, Hkv):
    """Workspace of the decode attention, written out from its definition:
    (max, sum, 128 partial outputs) in FP32 per query row and span, the
    spans being runs of 64-key blocks, as few blocks as keep spans x KV
    heads within 256."""
    n_keys = pos0 + m
    blocks = -(-n_keys // 64)
    span_blocks = max(1, -(-(blocks * Hkv) // 256))
    spans = -(-n_keys // (64 * span_blocks))
    return Hkv * spans * (H // Hkv * m) * (2 + 128) * 4


@pytest.mark.parametrize("m,pos0,H,Hkv", [(1, 0, 1, 1), (1, 63, 8, 2), (1, 64, 8, 2), (8, 8192, 32, 8),
                                          (1, 65535, 32, 8), (16, 200, 8, 2), (3, 6000, 16, 4)])
def test_decode_attention_workspace_bytes(lib, m, pos0, H, Hkv):
    assert binding.mq_attention_decode_workspace_bytes(m, pos0, H, Hkv, 128) == _dec_ws_expected(m, pos0, H, Hkv)


def test_attention_entry_points_reject_bad_arguments_on_the_host(lib):
    L = lib
    n = ctypes.c_int()
    ws = binding.mq_attention_decode_workspace_bytes
    # invalid sizes: no workspace at all
    assert ws(1, 8, 8, 2, 64) == 0 and ws(0, 8, 8, 2, 128) == 0 and ws(1, 8, 8, 3, 128) == 0
    assert ws(1, -1, 8, 2, 128) == 0
    # prefill: null pointers, one cache pointer without the other, shapes, alignment
    assert L.mq_attention_prefill_bf16(None, 16, 4, 2, 128, None, None, 0, 16, 16, ctypes.byref(n), None) == 1
    assert L.mq_attention_prefill_bf16(16, 16, 4, 2, 128, 16, None, 16, 16, 16, ctypes.byref(n), None) == 1
    assert L.mq_attention_prefill_bf16(16, 16, 4, 2, 64, None, None, 0, 16, 16, ctypes.byref(n), None) == 2
    assert L.mq_attention_prefill_bf16(16, 16, 4, 3, 128, None, None, 0, 16, 16, ctypes.byref(n), None) == 2
    assert L.mq_attention_prefill_bf16(16, 16, 4, 2, 128, 16, 16, 8, 16, 16, ctypes.byref(n), None) == 2
    assert L.mq_attention_prefill_bf16(24, 16, 4, 2, 128, None, None, 0, 16, 16, ctypes.byref(n), None) == 3
    # decode: rows per KV head above 64, the cache too short, workspace too small, alignment
    big = 1 << 30
    assert L.mq_attention_decode_bf16(None, 1, 8, 8, 2, 128, 16, 16, 16, 16, 16, big, None) == 1
    assert L.mq_attention_decode_bf16(16, 17, 8, 8, 2, 128, 16, 16, 64, 16, 16, big, None) == 2
    assert L.mq_attention_decode_bf16(16, 1, 8, 8, 2, 128, 16, 16, 8, 16, 16, big, None) == 2
    assert L.mq_attention_decode_bf16(16, 1, 8, 8, 2, 128, 16, 16, 16, 16, 16, 16, None) == 1
    assert L.mq_attention_decode_bf16(24, 1, 8, 8, 2, 128, 16, 16, 16, 16, 16, big, None) == 3
