"""The allocation-free prefill entry point, mq_prefill_linear_nvfp4_noalloc.

It exists for callers that cannot allocate device memory (a plugin handed
only its input and output buffers, or a latency-critical path that must not
pay the device synchronization of cudaMalloc / cudaFree): its scratch is a
fixed array inside the library's device image.  This file is collected last
so that a run stopping at the first failure has already run everything else.
"""
import numpy as np
import pytest
import torch

from mqtest import assert_close, ensure_built, oracle_prefill_rows
from nvfp4_quantized_prefill_b200 import binding as mq
from nvfp4_quantized_prefill_b200 import workloads

pytestmark = pytest.mark.gpu


def _existing(W, x, M):
    y = torch.empty(M, W.N, dtype=torch.bfloat16, device="cuda")
    nb = mq.mq_workspace_bytes(M, W.K)
    ws = torch.empty(nb, dtype=torch.uint8, device="cuda")
    mq.mq_prefill_linear_nvfp4(W.handle, x, M, y, ws, nb)
    return y


def test_noalloc_matches_workspace_entry_on_two_calls_in_a_row():
    ensure_built()
    # two different problems back to back through the shared scratch: the
    # second must not see anything the first left behind
    cases = [(300, 520, 512, 0), (1000, 768, 256, 1)]
    for M, N, K, seed in cases:
        x_cpu = workloads.activation("outlier", M, K, seed, 0)
        w_cpu = workloads.weight(N, K, 0.02, seed, 1)
        W = mq.Weight(w_cpu.cuda())
        x = x_cpu.cuda()
        y_ref = _existing(W, x, M)
        y_new = torch.full((M, N), 3.0, dtype=torch.bfloat16, device="cuda")
        mq.mq_prefill_linear_nvfp4_noalloc(W.handle, x, M, y_new)
        torch.cuda.synchronize()
        assert mq.mq_check() == 0
        # the same tolerance as every GEMM parity test, with the oracle's
        # sum of |products| for the bound
        _, p_ref = oracle_prefill_rows(x_cpu, w_cpu, np.arange(M))
        ref = y_ref.float().cpu().double().numpy()
        assert_close(y_new.cpu(), ref, p_ref, f"noalloc vs workspace entry {M}x{N}x{K}")
        W.free()


def test_noalloc_rejects_requests_larger_than_its_scratch():
    ensure_built()
    w_cpu = workloads.weight(256, 4096, 0.02, 2, 0)
    W = mq.Weight(w_cpu.cuda())
    M = 22016    # mq_workspace_bytes(M, 4096) > 48 MiB
    assert mq.mq_workspace_bytes(M, 4096) > (48 << 20)
    x = torch.zeros(M, 4096, dtype=torch.bfloat16, device="cuda")
    y = torch.empty(M, 256, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(mq.MqError) as e:
        mq.mq_prefill_linear_nvfp4_noalloc(W.handle, x, M, y)
    assert e.value.code == 2     # MQ_ERR_SHAPE, before any work is queued
    assert mq.mq_check() == 0
    W.free()
