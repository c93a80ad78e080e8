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
