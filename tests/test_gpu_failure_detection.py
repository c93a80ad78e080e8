"""Failure detection on the GPU without a fault: a bounded wait that runs out
latches the timeout bit, mq_check reports MQ_ERR_TIMEOUT once and clears it,
and the device keeps computing correctly afterwards."""
import numpy as np
import pytest
import torch

from mqtest import assert_close, ensure_built, oracle_prefill_rows
from nvfp4_quantized_prefill_b200 import binding as mq
from nvfp4_quantized_prefill_b200 import workloads

pytestmark = pytest.mark.gpu
MQ_ERR_TIMEOUT = 7


@pytest.fixture(scope="module", autouse=True)
def _built():
    ensure_built()


def test_bounded_wait_timeout_is_reported_and_cleared():
    assert mq.mq_check() == 0
    mq.mq_selftest_bounded_wait(20000)          # 20 ms on a phase nothing completes
    assert mq.mq_check() == MQ_ERR_TIMEOUT
    assert mq.mq_check() == 0                   # reported once, then cleared
    # the context is intact: a prefill linear still matches the oracle
    M, N, K = 64, 256, 512
    x = workloads.activation("outlier", M, K, 31, 0)
    w = workloads.weight(N, K, 0.02, 31, 1)
    W = mq.Weight(w.cuda())
    y = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    nb = mq.mq_workspace_bytes(M, K)
    ws = torch.empty(nb, dtype=torch.uint8, device="cuda")
    mq.mq_prefill_linear_nvfp4(W.handle, x.cuda(), M, y, ws, nb)
    assert mq.mq_check() == 0
    yr, pr = oracle_prefill_rows(x, w, np.arange(M))
    assert_close(y.cpu(), yr, pr, "prefill after a timeout")
    W.free()


def test_timeout_on_a_side_stream_is_seen_by_mq_check_on_that_stream():
    s = torch.cuda.Stream()
    mq.mq_selftest_bounded_wait(5000, s)
    assert mq.mq_check(s) == MQ_ERR_TIMEOUT
    assert mq.mq_check(s) == 0


def _debug_gemm():
    import ctypes
    L = mq.lib()
    f = L.mq_debug_gemm_withhold_release
    f.restype = ctypes.c_int
    f.argtypes = [ctypes.c_void_p] * 3 + [ctypes.c_int64, ctypes.c_void_p, ctypes.c_void_p,
                                          ctypes.c_int64, ctypes.c_uint32, ctypes.c_void_p]
    return f


@pytest.mark.parametrize("M,N,K", [(256, 256, 2048), (600, 768, 4096)])
def test_gemm_abort_path_latches_the_timeout_and_exits(M, N, K):
    """The GEMM's own abort path, driven without a fault: the test-only entry
    point withholds the release of the first K stage (20 ms wait limit), so
    the producers' waits for it run out.  The kernel must latch the timeout,
    stop every role, drain what it issued and exit in well under a second;
    mq_check reports it once; a prefill afterwards matches the oracle."""
    import time
    from mqtest import gpu_quantize
    x = workloads.activation("outlier", M, K, 33, 0)
    w = workloads.weight(N, K, 0.02, 33, 1)
    W = mq.Weight(w.cuda())
    codes, sf, s = gpu_quantize(x.cuda())
    c, f = torch.from_numpy(codes).cuda(), torch.from_numpy(sf).cuda()
    sd = torch.tensor([s], dtype=torch.float32, device="cuda")
    y = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    torch.cuda.synchronize()
    assert mq.mq_check() == 0
    t0 = time.perf_counter()
    rc = _debug_gemm()(c.data_ptr(), f.data_ptr(), sd.data_ptr(), M, W.handle, y.data_ptr(), N,
                       20000, torch.cuda.current_stream().cuda_stream)
    assert rc == 0
    torch.cuda.synchronize()
    assert time.perf_counter() - t0 < 1.0       # several 20 ms waits, no more
    assert mq.mq_check() == MQ_ERR_TIMEOUT
    assert mq.mq_check() == 0
    # the same handle, a normal prefill: the device keeps computing
    y2 = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    nb = mq.mq_workspace_bytes(M, K)
    ws = torch.empty(nb, dtype=torch.uint8, device="cuda")
    mq.mq_prefill_linear_nvfp4(W.handle, x.cuda(), M, y2, ws, nb)
    assert mq.mq_check() == 0
    yr, pr = oracle_prefill_rows(x, w, np.arange(M))
    assert_close(y2.cpu(), yr, pr, "prefill after the GEMM's abort")
    W.free()
