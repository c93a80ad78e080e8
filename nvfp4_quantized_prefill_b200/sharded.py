"""Token-sharded NVFP4 prefill linear across GPUs (one process per GPU).

Each rank holds a contiguous block of the batch's rows (tokens) and a replica
of the weight handle.  Quantizing every shard with the tensor scale of the
whole batch makes each rank's rows of Y the single-GPU result bit for bit;
that scale comes from the batch's max |x| (gist.science technical summary,
section 2 "Hybrid Precision Strategy": one tensor-level scale per tensor), so
the ranks exchange one float -- the max of their shards' maxima -- with one
all-reduce over torch.distributed (NCCL on GPUs).  That is the only
collective; every other step runs in this library's kernels:

  mq_tensor_amax (shard partial maxima) -> mq_amax_combine (one float)
  -> all-reduce(max) -> mq_quantize_nvfp4 (n_partials = 1) -> mq_gemm_nvfp4

`shard_amax` and `shard_finish` are the two halves around the exchange, so
that shards can also be run one after another in one process (the exchange
then being a max over the shards' floats).
"""
from __future__ import annotations

from dataclasses import dataclass

import torch

from . import binding as mq


@dataclass
class ShardWorkspace:
    """Device buffers of one shard: NVFP4 codes and swizzled scales of the
    shard's rows, its tensor scale, the partial maxima and the one-float amax
    that is exchanged."""
    codes: torch.Tensor
    sf: torch.Tensor
    s_enc: torch.Tensor
    partials: torch.Tensor
    amax: torch.Tensor

    @staticmethod
    def create(M: int, K: int, device="cuda") -> "ShardWorkspace":
        return ShardWorkspace(
            codes=torch.empty(M, K // 2, dtype=torch.uint8, device=device),
            sf=torch.empty(mq.mq_sf_bytes(M, K), dtype=torch.uint8, device=device),
            s_enc=torch.empty(1, dtype=torch.float32, device=device),
            partials=torch.empty(mq.MQ_AMAX_PARTIALS_MAX, dtype=torch.float32, device=device),
            amax=torch.empty(1, dtype=torch.float32, device=device))


def exchange_amax(amax: torch.Tensor, group=None, stream=None) -> None:
    """In place: amax <- max over the ranks of `group` (all-reduce MAX of one
    float).  Runs after the work already queued on `stream` (default: the
    current stream)."""
    import torch.distributed as dist
    if stream is not None and amax.is_cuda:
        with torch.cuda.stream(stream):
            dist.all_reduce(amax, op=dist.ReduceOp.MAX, group=group)
    else:
        dist.all_reduce(amax, op=dist.ReduceOp.MAX, group=group)


def shard_amax(x_local: torch.Tensor, ws: ShardWorkspace, stream=None) -> torch.Tensor:
    """This shard's max |x| as one float in ws.amax (two kernels)."""
    M, K = x_local.shape
    n = mq.mq_tensor_amax(x_local, M, K, K, ws.partials, stream)
    mq.mq_amax_combine(ws.partials, n, ws.amax, stream)
    return ws.amax


def shard_finish(weight: "mq.Weight", x_local: torch.Tensor, y_local: torch.Tensor,
                 ws: ShardWorkspace, stream=None) -> None:
    """Quantizes the shard with the batch amax now in ws.amax and multiplies it
    by the weight: y_local = the shard's rows of the single-GPU result."""
    M, K = x_local.shape
    mq.mq_quantize_nvfp4(x_local, M, K, K, ws.codes, ws.sf, ws.s_enc, amax_partials=ws.amax,
                         n_partials=1, stream=stream)
    mq.mq_gemm_nvfp4(ws.codes, ws.sf, ws.s_enc, M, weight.handle, y_local, weight.N, stream)


def prefill_linear_token_sharded(weight: "mq.Weight", x_local: torch.Tensor,
                                 y_local: torch.Tensor, ws: ShardWorkspace, group=None,
                                 stream=None) -> None:
    """One rank's part of Y = X W^T for a batch split by rows across the ranks
    of `group`: x_local [M_r, K] BF16, y_local [M_r, N] BF16 (device,
    contiguous).  Every rank must call it, in the same order as its other
    collectives."""
    shard_amax(x_local, ws, stream)
    exchange_amax(ws.amax, group, stream)
    shard_finish(weight, x_local, y_local, ws, stream)
