"""Shared helpers for the GPU parity tests (not collected as tests).

The CUDA side is reached only through the C ABI (nvfp4_quantized_prefill_b200
.binding); the expected values come only from the CPU oracle."""
from __future__ import annotations

import numpy as np
import torch

import oracle
from nvfp4_quantized_prefill_b200 import binding as mq
from nvfp4_quantized_prefill_b200 import build as mqbuild

# Output tolerance: |gpu - ref| <= 2^-8 |ref| + 1e-5 * sum_k |products|.
REL = 2.0 ** -8
ABS_P = 1e-5


def ensure_built():
    mqbuild.build()
    oracle.build()
    mq.lib()


def u16(t: torch.Tensor) -> np.ndarray:
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


def bf16_from_u16(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16)


def gpu_quantize(x: torch.Tensor):
    """Quantize a CUDA BF16 matrix through mq_quantize_nvfp4 (amax inside)."""
    M, K = x.shape
    codes = torch.empty(M, K // 2, dtype=torch.uint8, device="cuda")
    sf = torch.empty(mq.mq_sf_bytes(M, K), dtype=torch.uint8, device="cuda")
    s = torch.empty(1, dtype=torch.float32, device="cuda")
    ws = torch.empty(mq.MQ_AMAX_PARTIALS_MAX, dtype=torch.float32, device="cuda")
    mq.mq_quantize_nvfp4(x, M, K, K, codes, sf, s, workspace=ws, ws_bytes=ws.numel() * 4)
    torch.cuda.synchronize()
    return codes.cpu().numpy(), sf.cpu().numpy(), float(s.item())


def assert_close(y_gpu: torch.Tensor, y_ref: np.ndarray, p_ref: np.ndarray, what: str):
    yg = y_gpu.detach().float().cpu().double().numpy()
    assert yg.shape == y_ref.shape, (yg.shape, y_ref.shape)
    bound = REL * np.abs(y_ref) + ABS_P * p_ref
    err = np.abs(yg - y_ref)
    bad = err > bound
    if bad.any():
        i = np.unravel_index(np.argmax(err - bound), err.shape)
        raise AssertionError(
            f"{what}: {int(bad.sum())}/{bad.size} outside |d| <= 2^-8|ref| + 1e-5 P; worst at {i}: "
            f"gpu {yg[i]!r} ref {y_ref[i]!r} P {p_ref[i]!r}")
    assert np.isfinite(yg).all()


def oracle_prefill_rows(x_cpu: torch.Tensor, w_cpu: torch.Tensor, rows, wrows=None):
    """Oracle output of the prefill linear for the given X rows (and optionally
    a subset of W rows), with the tensor scales taken over the FULL tensors."""
    sx = oracle.tensor_scale(oracle.tensor_amax(x_cpu))
    sw = oracle.tensor_scale(oracle.tensor_amax(w_cpu))
    rows = np.asarray(rows, dtype=np.int64)
    xc, xs = oracle.quantize(x_cpu[torch.from_numpy(rows)].contiguous(), sx)
    wsub = w_cpu if wrows is None else w_cpu[torch.from_numpy(np.asarray(wrows))].contiguous()
    wc, wsf = oracle.quantize(wsub, sw)
    return oracle.gemm_nvfp4(xc, xs, sx, wc, wsf, sw)


def sample_rows(M: int, n: int, seed: int):
    rng = np.random.default_rng(seed)
    fixed = [0, min(127, M - 1), min(128, M - 1), M - 1]
    extra = rng.choice(M, size=min(n, M), replace=False).tolist()
    return np.array(sorted(set(fixed + extra)), dtype=np.int64)


class _DevBuf:
    """__cuda_array_interface__ view of a raw device pointer (the caller only reads it)."""

    def __init__(self, ptr: int, nbytes: int):
        self.__cuda_array_interface__ = {"shape": (nbytes,), "typestr": "|u1",
                                         "data": (ptr, False), "version": 3}


def fetch_device(ptr: int, nbytes: int) -> np.ndarray:
    """Copies nbytes at a raw device pointer to a host uint8 array."""
    torch.cuda.synchronize()
    src = torch.as_tensor(_DevBuf(ptr, nbytes), device="cuda")
    return src.clone().cpu().numpy()


def check_h_from_gu(y, h, I, what):
    """h (BF16) against the oracle's SwiGLU of the GPU's own BF16 gate / up
    halves of y: within one BF16 ulp, and almost always identical."""
    g, u = y[:, :I].contiguous(), y[:, I:].contiguous()
    href = oracle.swiglu(g, u)
    hg = u16(h)
    # expf differs between the C library and CUDA by an ulp or so in FP32;
    # after rounding to BF16 that is at most one BF16 ulp, and rarely.
    a = bf16_from_u16(hg).double()
    b = bf16_from_u16(href).double()
    ulp = torch.clamp(b.abs(), min=2.0 ** -126) * 2.0 ** -7
    assert ((a - b).abs() <= ulp).all(), what
    assert (hg == href).mean() > 0.995, what
