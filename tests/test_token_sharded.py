"""Token-sharded prefill (a batch split by rows across ranks, one float
exchanged): with the batch's tensor scale on every shard, each shard's codes,
scales and outputs are the single-GPU ones bit for bit.

CPU (gloo, 2 ranks): the exchange of nvfp4_quantized_prefill_b200.sharded
(all-reduce max of one float) with the oracle doing each rank's amax and
quantization.  GPU: the library's shard halves run for several shards in one
process (the exchange being the max of the shards' floats); each shard's
outputs are compared with the oracle's prefill of the whole batch, and all of
them together with the single-call prefill linear."""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


# uneven row split of a 37 x 320 batch
ROWS = [(0, 20), (20, 37)]


def _worker(rank, world, port, out):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import oracle
    from nvfp4_quantized_prefill_b200 import sharded, workloads
    x = workloads.activation("outlier", 37, 320, 11, 0)
    r0, r1 = ROWS[rank]
    mine = x[r0:r1].contiguous()
    amax = torch.tensor([oracle.tensor_amax(mine)], dtype=torch.float32)
    sharded.exchange_amax(amax)
    s = oracle.tensor_scale(float(amax.item()))
    codes, sf = oracle.quantize(mine, s)
    out[rank] = (float(amax.item()), s, codes.tobytes(), sf.tobytes())
    dist.barrier()
    dist.destroy_process_group()


def test_two_rank_amax_exchange_gloo():
    import oracle
    from nvfp4_quantized_prefill_b200 import workloads
    world = 2
    port = _free_port()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, port, out), nprocs=world, join=True,
                       start_method="spawn")
    x = workloads.activation("outlier", 37, 320, 11, 0)
    # the shards' own maxima differ, so a shard quantized with its own scale
    # (no exchange) would not match
    assert len({oracle.tensor_amax(x[a:b].contiguous()) for a, b in ROWS}) == 2
    full_amax = oracle.tensor_amax(x)
    s_full = oracle.tensor_scale(full_amax)
    codes_full, sf_full = oracle.quantize(x, s_full)
    for r in range(world):
        amax, s, codes, sf = out[r]
        assert amax == full_amax and s == s_full
        r0, r1 = ROWS[r]
        assert codes == codes_full[r0:r1].tobytes()
        assert sf == sf_full[r0:r1].tobytes()


def test_shard_workspace_sizes():
    """A shard's buffers: codes [M, K/2], the swizzled scales of M rows (rows
    padded to 128), the partial maxima and the one float that is exchanged."""
    from nvfp4_quantized_prefill_b200 import binding as mq
    from nvfp4_quantized_prefill_b200 import sharded
    ws = sharded.ShardWorkspace.create(37, 320, device="cpu")
    assert ws.codes.shape == (37, 160)
    assert ws.sf.numel() == mq.mq_sf_bytes(37, 320) == 128 * 20
    assert ws.partials.numel() == mq.MQ_AMAX_PARTIALS_MAX
    assert ws.amax.numel() == 1 and ws.s_enc.numel() == 1


@pytest.mark.gpu
def test_token_shards_on_one_gpu_bit_identical():
    from mqtest import ensure_built
    ensure_built()
    import oracle
    from nvfp4_quantized_prefill_b200 import binding as mq
    from nvfp4_quantized_prefill_b200 import sharded, workloads
    M, N, K = 1000, 520, 512
    bounds = [0, 333, 700, 1000]   # uneven, across 128-row tiles
    x = workloads.activation("outlier", M, K, 9, 0)
    W = mq.Weight(workloads.weight(N, K, 0.02, 9, 1).cuda())
    xd = x.cuda()
    y_full = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    nb = mq.mq_workspace_bytes(M, K)
    ws = torch.empty(nb, dtype=torch.uint8, device="cuda")
    mq.mq_prefill_linear_nvfp4(W.handle, xd, M, y_full, ws, nb)
    xs = [xd[a:b].contiguous() for a, b in zip(bounds, bounds[1:])]
    wss = [sharded.ShardWorkspace.create(t.shape[0], K) for t in xs]
    ys = [torch.empty(t.shape[0], N, dtype=torch.bfloat16, device="cuda") for t in xs]
    for t, w in zip(xs, wss):
        sharded.shard_amax(t, w)
    amax = torch.stack([w.amax for w in wss]).max()   # the exchange, in one process
    for w in wss:
        w.amax.copy_(amax)
    for t, y, w in zip(xs, ys, wss):
        sharded.shard_finish(W, t, y, w)
    torch.cuda.synchronize()
    assert float(amax) == oracle.tensor_amax(x)
    # every shard's rows against the oracle's prefill of the whole batch (the
    # batch's tensor scales), at the GEMM tolerance
    from mqtest import assert_close, oracle_prefill_rows
    w_cpu = workloads.weight(N, K, 0.02, 9, 1)
    for (a, b), y in zip(zip(bounds, bounds[1:]), ys):
        y_or, p_or = oracle_prefill_rows(x, w_cpu, np.arange(a, b))
        assert_close(y.cpu(), y_or, p_or, f"token shard rows {a}..{b}")
    # and the shards together reproduce the single-call prefill bit for bit
    assert torch.equal(torch.cat(ys).view(torch.int16), y_full.view(torch.int16))
    W.free()
    assert mq.mq_check() == 0
