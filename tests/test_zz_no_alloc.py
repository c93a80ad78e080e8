"""The allocation-free prefill entry point, mq_prefill_linear_nvfp4_noalloc.

It exists for callers that cannot allocate device memory (a plugin handed
only its input and output buffers, or a latency-critical path that must not
pay the device synchronization of cudaMalloc / cudaFree): its scratch is a
fixed array inside the library's device image, shared by every call.  This
file is collected last so that a run stopping at the first failure has
already run everything else.
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


def _check_sequence(cases):
    """Runs the cases back to back through the one shared scratch array.
    Each output must equal the workspace entry point's bit for bit (same
    kernels, same inputs) and be within the GEMM tolerance of the oracle."""
    for M, N, K, seed, recipe in cases:
        x_cpu = workloads.activation(recipe, M, K, seed, 0)
        w_cpu = workloads.weight(N, K, 0.02, seed, 1)
        W = mq.Weight(w_cpu.cuda())
        x = x_cpu.cuda()
        y_new = torch.full((M, N), 3.0, dtype=torch.bfloat16, device="cuda")
        mq.mq_prefill_linear_nvfp4_noalloc(W.handle, x, M, y_new)
        y_ref = _existing(W, x, M)
        torch.cuda.synchronize()
        assert mq.mq_check() == 0
        assert torch.equal(y_new.view(torch.int16), y_ref.view(torch.int16)), (
            f"noalloc differs from the workspace entry point at {M}x{N}x{K}")
        y_or, p_or = oracle_prefill_rows(x_cpu, w_cpu, np.arange(M))
        assert_close(y_new.cpu(), y_or, p_or, f"noalloc vs oracle {M}x{N}x{K}")
        W.free()


def test_noalloc_matches_workspace_entry_and_oracle_on_two_calls_in_a_row():
    ensure_built()
    # two different problems back to back: the second must not see anything
    # the first left behind
    _check_sequence([(300, 520, 512, 0, "outlier"), (1000, 768, 256, 1, "outlier")])


def test_noalloc_small_ragged_call_after_a_large_one():
    ensure_built()
    # the large call fills far more of the array (codes, scale tiles with
    # their padding rows, partial maxima, tensor scale) than the ragged call
    # after it writes, with a different scale, so stale bytes from the first
    # sit right after and inside the second call's region
    _check_sequence([(1500, 384, 1024, 3, "student_t3"), (77, 200, 320, 4, "outlier"),
                     (129, 256, 64, 5, "channel_gain")])


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
