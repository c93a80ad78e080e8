"""GPU parity of the uniform-NVFP4 (W4A4) decode linear against the oracle's
exact block-scaled GEMM on the same quantized operands."""
import numpy as np
import pytest
import torch

from mqtest import assert_close, ensure_built, oracle_prefill_rows
from nvfp4_quantized_prefill_b200 import binding as mq
from nvfp4_quantized_prefill_b200 import workloads

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    ensure_built()


def gpu_decode_nvfp4(x_cpu, W):
    M, K = x_cpu.shape
    y = torch.empty(M, W.N, dtype=torch.bfloat16, device="cuda")
    nb = mq.mq_workspace_bytes(M, K)
    ws = torch.empty(nb, dtype=torch.uint8, device="cuda")
    mq.mq_decode_linear_nvfp4(W.handle, x_cpu.cuda(), M, y, ws, nb)
    torch.cuda.synchronize()
    return y.cpu()


# (M, N, K): one token; 8 tokens with ragged N and a partial last 256-K step
# (FP16-MMA kernel); N < 16; 13 and 16 tokens (the tensor-core kernel's limit)
# and 17 (quantize kernels + FP16-MMA kernel, two launches); N = 1; few weight
# rows with a long K (tiles split across many CTAs); a long-K 8-token case;
# a partial last K step of three scale blocks; the Llama-3-8B QKV shape.
# Routing: 1-4 tokens on weights of up to 2^25 elements take the CUDA-core
# stream (partial last 1024-K step: K = 256, 64, 128, 2048 ...); larger weights
# with 1-4 tokens and 9-16 tokens (M K 9/16 <= 40 KB) the tensor-core kernel
# (the two shapes past 2^25 elements below, and 1 x 9000 x 4032 with a partial
# last K stage); 5-8 tokens the FP16-MMA kernel (also on weights past 2^25
# elements: 6 x 9000 x 4096, 8 x 8200 x 4096).
# The tensor-core kernel quantizes in each CTA only the K stages its units
# cover (a compact buffer: 13 x 1024 x 4096, 3 x 4100 x 8192, 1 x 9000 x 4032
# with a partial last stage), which lets 16 tokens with K = 14336 fit it.
SHAPES = [(1, 256, 256), (8, 300, 320), (3, 17, 64), (13, 1024, 4096), (1, 1, 128),
          (2, 64, 8192), (1, 16, 16384), (8, 4096, 14336), (5, 100, 448), (16, 520, 1024),
          (17, 200, 512), (1, 6144, 4096), (4, 1000, 2048), (1, 9000, 4096), (3, 4100, 8192),
          (1, 9000, 4032), (12, 300, 960), (6, 9000, 4096), (8, 8200, 4096), (16, 2048, 14336)]


@pytest.mark.parametrize("M,N,K", SHAPES)
def test_decode_nvfp4_all_elements(M, N, K):
    x = workloads.activation("outlier", M, K, 7, M)
    w = workloads.weight(N, K, 0.02, 7, N)
    W = mq.Weight(w.cuda())
    y = gpu_decode_nvfp4(x, W)
    yr, pr = oracle_prefill_rows(x, w, np.arange(M))
    assert_close(y, yr, pr, f"nvfp4 decode {M}x{N}x{K}")
    W.free()
    assert mq.mq_check() == 0


def test_decode_nvfp4_phase_switch_llama8b_qkv():
    """M = 1 and M = 8 on the handle the QKV prefill uses, all outputs."""
    wl = workloads.WORKLOADS["llama3_8b_qkv_o"]
    w = workloads.layer_weights(wl)[0]
    W = mq.Weight(w.cuda())
    for M in (1, 8):
        x = workloads.activation("channel_gain", M, w.shape[1], 30 + M, 0)
        y = gpu_decode_nvfp4(x, W)
        yr, pr = oracle_prefill_rows(x, w, np.arange(M))
        assert_close(y, yr, pr, f"nvfp4 decode qkv M={M}")
    W.free()


def test_decode_nvfp4_right_after_packing():
    """No operation between packing the weight and the decode: the
    tensor-core kernel streams the weight before waiting on the kernel before
    it, and packing ends with a memory set, so that kernel is never the one
    that writes the codes."""
    M, N, K = 1, 6144, 4096
    x = workloads.activation("outlier", M, K, 12, 0)
    w = workloads.weight(N, K, 0.02, 12, 1)
    xd, wd = x.cuda(), w.cuda()
    y = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    nb = mq.mq_workspace_bytes(M, K)
    ws = torch.empty(nb, dtype=torch.uint8, device="cuda")
    torch.cuda.synchronize()
    W = mq.Weight(wd)
    mq.mq_decode_linear_nvfp4(W.handle, xd, M, y, ws, nb)
    torch.cuda.synchronize()
    yr, pr = oracle_prefill_rows(x, w, np.arange(M))
    assert_close(y.cpu(), yr, pr, "nvfp4 decode right after packing")
    W.free()
    assert mq.mq_check() == 0


def test_decode_paths_share_scratch():
    """BF16 and NVFP4 decode on one split-K handle, alternating: each leaves
    the shared counters at zero for the other, and every round gives the same
    bits (the split-K partial sums are added in a fixed order)."""
    import oracle
    M, N, K = 2, 48, 8192
    x = workloads.activation("student_t3", M, K, 8, 0)
    w = workloads.weight(N, K, 0.02, 8, 1)
    W = mq.Weight(w.cuda())
    yr4, pr4 = oracle_prefill_rows(x, w, np.arange(M))
    yr16, pr16 = oracle.decode_linear(x, w)
    first = None
    for it in range(3):
        y16 = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
        mq.mq_decode_linear_bf16(W.handle, x.cuda(), M, y16)
        y4 = gpu_decode_nvfp4(x, W)
        assert_close(y16.cpu(), yr16, pr16, f"bf16 decode round {it}")
        assert_close(y4, yr4, pr4, f"nvfp4 decode round {it}")
        if first is None:
            first = (y16.cpu(), y4)
        assert torch.equal(y16.cpu().view(torch.int16), first[0].view(torch.int16)), it
        assert torch.equal(y4.view(torch.int16), first[1].view(torch.int16)), it
    W.free()
    assert mq.mq_check() == 0


def test_decode_nvfp4_matches_prefill():
    """The same tokens through the prefill linear and the W4A4 decode give the
    same rounded results up to FP32 summation order."""
    M, N, K = 8, 512, 1024
    x = workloads.activation("outlier", M, K, 9, 0)
    w = workloads.weight(N, K, 0.02, 9, 1)
    W = mq.Weight(w.cuda())
    y4 = gpu_decode_nvfp4(x, W)
    yp = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    nb = mq.mq_workspace_bytes(M, K)
    ws = torch.empty(nb, dtype=torch.uint8, device="cuda")
    mq.mq_prefill_linear_nvfp4(W.handle, x.cuda(), M, yp, ws, nb)
    torch.cuda.synchronize()
    yr, pr = oracle_prefill_rows(x, w, np.arange(M))
    assert_close(y4, yr, pr, "nvfp4 decode")
    assert_close(yp.cpu(), yr, pr, "prefill")
    W.free()
