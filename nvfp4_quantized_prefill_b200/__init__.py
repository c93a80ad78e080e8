"""B200-native NVFP4 quantized prefill linear layer (Mix-Quant hot path).

The compute lives in ``libmq.so`` (hand-written CUDA for sm_100a behind a C
ABI declared in ``include/mq.h``); :mod:`.binding` marshals arguments to it.
Importing the package loads nothing; the library is loaded on first use and
the binding raises if it is missing -- there is no CPU fallback.
"""
__all__ = ["binding", "workloads"]
