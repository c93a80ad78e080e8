"""Benchmark of the prefill-phase NVFP4 linear layer (Mix-Quant hot path).

One step = one pass of the hot path over one batch of synthetic input: the
prefill phase of the workload's projections -- per activation: tensor amax ->
NVFP4 quantize -> block-scaled tcgen05 GEMM (with the SwiGLU epilogue and the
quantize of h between gate/up and down for MLP workloads) -- then the BF16
decode linear at M = 1 on the same weight handles (the phase switch).

Metric: prefill linear TFLOP/s including activation quantization,
sum(2 M N K) / (t_amax + t_quant + t_gemm [+ t_quant(h)]), and its fraction of
the dense FP4 peak.  Timed with CUDA events on the launching stream; between
steps, outside the timed intervals, the L2 is flushed by writing one 256 MiB
buffer and then reading another, so no dirty lines are left for the next
kernel to write back.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
  python bench.py --impl reference ...   (the CPU oracle, bounded sample)
  python bench.py --sharded ...          (the batch split by tokens across ranks)
  python bench.py --profile-case NAME    (one small case for an ncu capture)

Multi-GPU: one process per GPU (torchrun), independent replicas (the layer
needs no exchange); value = work of all ranks / max-over-ranks time.  With
--sharded the batch is split by tokens and the ranks all-reduce one float per
activation (the tensor scale); value = the batch's work / max-over-ranks time.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from nvfp4_quantized_prefill_b200 import workloads  # noqa: E402

FP4_OVER_BF16 = 4.0   # nominal dense ratio (9 PF fp4 / 2.25 PF bf16)
RMS_EPS = 1e-5
METRIC = "prefill linear TFLOPS (NVFP4 incl. act-quant) and % of B200 dense FP4 peak"
CLOCK_QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
               "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
               "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
GEMM_SOURCES = ["nvfp4_quantized_prefill_b200/csrc/mq_gemm.cu",
                "nvfp4_quantized_prefill_b200/csrc/mq_ptx.cuh"]
COUNTERS = os.path.join(ROOT, "profiles", "counters.json")


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": d["hbm_gbs"], "bf16": d["bf16_tflops"],
                "bf16_sustained": d.get("bf16_tflops_sustained", d["bf16_tflops"]),
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16": 1590.0, "bf16_sustained": 1400.0, "source": "fallback"}


def gemm_source_hash() -> str:
    h = hashlib.sha256()
    for f in GEMM_SOURCES:
        h.update(open(os.path.join(ROOT, f), "rb").read())
    return h.hexdigest()[:16]


def recorded_traffic(workload_key: str):
    """DRAM bytes (read + write) per GEMM launch from the committed ncu summary,
    only if it was taken on the GEMM source as it is now.  Returns
    (mean bytes over the captured launches, their names) or (None, None)."""
    try:
        d = json.load(open(COUNTERS))
    except Exception:
        return None, None
    if d.get("gemm_source_hash") != gemm_source_hash():
        return None, None
    per = d.get("gemm_dram_bytes_per_launch", {}).get(workload_key)
    if not per:
        return None, None
    return sum(per.values()) / len(per), sorted(per)


def recorded_tensor_pipe(workload_key: str):
    """ncu's tensor-pipe activity (% of elapsed cycles) per GEMM launch from
    the same committed capture as the traffic, only if it was taken on the
    GEMM source as it is now; None otherwise."""
    try:
        d = json.load(open(COUNTERS))
    except Exception:
        return None
    if d.get("gemm_source_hash") != gemm_source_hash():
        return None
    return d.get("gemm_tensor_pipe_active_pct", {}).get(workload_key)


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples during the timed region."""

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = None   # a temporary file, made when sampling starts

    def __enter__(self):
        try:
            fd, self.path = tempfile.mkstemp(prefix=f"mq_clocks_rank{self.index}_", suffix=".csv")
            self.fh = os.fdopen(fd, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={CLOCK_QUERY}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=self.fh, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            self.fh.close()

    def summary(self):
        try:
            rows = [l.split(",") for l in open(self.path) if l.strip()]
        except Exception:
            return None
        finally:
            try:
                os.remove(self.path)
            except OSError:
                pass
        if not rows:
            return None
        num = lambda v: v.strip().replace(".", "", 1).isdigit()
        sm = [float(r[1]) for r in rows if num(r[1])]
        mx = [float(r[2]) for r in rows if num(r[2])]
        reasons = set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            for i, n in enumerate(names):
                if len(r) > 5 + i and "Active" in r[5 + i] and "Not" not in r[5 + i]:
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": sorted(reasons),
                "samples": len(rows)}


def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        torch.cuda.set_device(local)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                             device_id=torch.device("cuda", local))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    if world > 1:
        torch.distributed.barrier()


def reduce_over_ranks(v: float, world: int, op: str) -> float:
    """MAX or SUM of a host float over the ranks (NCCL: via the GPU; gloo: CPU)."""
    if world == 1:
        return v
    dev = "cuda" if torch.distributed.get_backend() == "nccl" else "cpu"
    t = torch.tensor([v], dtype=torch.float64, device=dev)
    torch.distributed.all_reduce(t, op=getattr(torch.distributed.ReduceOp, op))
    return float(t.item())


def aggregate_sharded(batch_flops: float, ms_local: float, world: int):
    """Whole-job throughput of a batch split by tokens across the ranks: the
    batch's work (counted once) over the slowest rank's time (strong
    scaling).  Returns (tflops, max_ms)."""
    max_ms = reduce_over_ranks(ms_local, world, "MAX")
    return batch_flops / (max_ms * 1e-3) / 1e12, max_ms


def aggregate(flops_local: float, prefill_ms_local: float, world: int):
    """Whole-job throughput of independent replicas: the work of all ranks over
    the slowest rank's time.  Returns (tflops, max_ms, total_flops)."""
    max_ms = reduce_over_ranks(prefill_ms_local, world, "MAX")
    total = reduce_over_ranks(flops_local, world, "SUM")
    return total / (max_ms * 1e-3) / 1e12, max_ms, total


# ---------------------------------------------------------------------------
# CPU oracle leg (reference arm and cpu_baseline)
# ---------------------------------------------------------------------------

def oracle_prepare(ws_cpu):
    """Weight packing on the oracle side (offline in the method, untimed)."""
    import oracle
    oracle.build()
    out = []
    for w in ws_cpu:
        s = oracle.tensor_scale(oracle.tensor_amax(w))
        c, f = oracle.quantize(w, s)
        out.append((c, f, s))
    return out


def oracle_sample(xs, wq, rows_per_linear: int):
    """Times the oracle on a bounded sample: per projection, the full-tensor
    amax, quantization of `rows_per_linear` activation rows and their exact
    block-scaled GEMM against the packed weight.  Returns (flops, seconds)."""
    import oracle
    flops = 0.0
    t0 = time.perf_counter()
    for x, (wc, wf, sw) in zip(xs, wq):
        sx = oracle.tensor_scale(oracle.tensor_amax(x))
        xc, xf = oracle.quantize(x[:rows_per_linear].contiguous(), sx)
        oracle.gemm_nvfp4(xc, xf, sx, wc, wf, sw)
        flops += 2.0 * rows_per_linear * wc.shape[0] * x.shape[1]
    return flops, time.perf_counter() - t0


# ---------------------------------------------------------------------------
# GPU leg
# ---------------------------------------------------------------------------

class Prefill:
    """Device buffers and the launch sequence of one workload's prefill."""

    def __init__(self, wl, mq, dev):
        self.wl, self.mq, self.dev = wl, mq, dev
        ws = workloads.layer_weights(wl, device=str(dev))
        self.ws = ws
        self.W = [mq.Weight(w) for w in ws]
        M = wl.M
        self.M = M
        u8, f32, bf = torch.uint8, torch.float32, torch.bfloat16

        def qbuf(K):
            return dict(codes=torch.empty(M, K // 2, dtype=u8, device=dev),
                        sf=torch.empty(mq.mq_sf_bytes(M, K), dtype=u8, device=dev),
                        s=torch.empty(1, dtype=f32, device=dev),
                        part=torch.empty(mq.MQ_AMAX_PARTIALS_MAX, dtype=f32, device=dev))

        self.ops = []    # list of (name, callable) kernel launches, in order
        self.flops = 0.0
        if wl.swiglu:
            # gate_up followed by down is one SwiGLU MLP (the GEMM epilogue
            # writes h and its amax); every other projection is a plain linear
            # with its own activation
            self.xs = []
            self.plan = []   # ("mlp", gate_up index, down index, x index) / ("linear", index, x index)
            lin = list(wl.linears)
            i = 0
            while i < len(lin):
                W = self.W[i]
                if lin[i].name == "gate_up" and i + 1 < len(lin) and lin[i + 1].name == "down":
                    Wgu, Wd = self.W[i], self.W[i + 1]
                    I = Wgu.N // 2
                    assert Wd.K == I, "down projection K must equal the SwiGLU width"
                    x = workloads.layer_activation(wl, Wgu.K, i, device=str(dev))
                    self.plan.append(("mlp", i, i + 1, len(self.xs)))
                    self.xs.append(x)
                    qx, qh = qbuf(Wgu.K), qbuf(I)
                    h = torch.empty(M, I, dtype=bf, device=dev)
                    y = torch.empty(M, Wd.N, dtype=bf, device=dev)
                    self._add_quant(f"amax+quant x{i}", x, Wgu.K, qx)
                    self.ops.append((f"gemm {lin[i].name}+swiglu", "gemm",
                                     lambda st, qx=qx, Wgu=Wgu, h=h, qh=qh: qh.__setitem__(
                                         "n", mq.mq_gemm_nvfp4_swiglu(qx["codes"], qx["sf"], qx["s"], M,
                                                                      Wgu.handle, h, qh["part"], st))))
                    self.ops.append((f"quant h{i}", "quant",
                                     lambda st, h=h, qh=qh, I=I: mq.mq_quantize_nvfp4(
                                         h, M, I, I, qh["codes"], qh["sf"], qh["s"],
                                         amax_partials=qh["part"], n_partials=qh["n"], stream=st)))
                    self.ops.append((f"gemm {lin[i + 1].name}", "gemm",
                                     lambda st, qh=qh, Wd=Wd, y=y: mq.mq_gemm_nvfp4(
                                         qh["codes"], qh["sf"], qh["s"], M, Wd.handle, y, Wd.N, st)))
                    self.flops += 2.0 * M * Wgu.N * Wgu.K + 2.0 * M * Wd.N * Wd.K
                    i += 2
                else:
                    x = workloads.layer_activation(wl, W.K, i, device=str(dev))
                    self.plan.append(("linear", i, len(self.xs)))
                    self.xs.append(x)
                    q = qbuf(W.K)
                    y = torch.empty(M, W.N, dtype=bf, device=dev)
                    self._add_quant(f"amax+quant x{i}", x, W.K, q)
                    self.ops.append((f"gemm {lin[i].name}", "gemm",
                                     lambda st, q=q, W=W, y=y: mq.mq_gemm_nvfp4(
                                         q["codes"], q["sf"], q["s"], M, W.handle, y, W.N, st)))
                    self.flops += 2.0 * M * W.N * W.K
                    i += 1
        elif wl.chunks > 1:
            # each chunk quantized once and used by every projection
            K = self.W[0].K
            self.xs = [workloads.layer_activation(wl, K, c, device=str(dev)) for c in range(wl.chunks)]
            q = qbuf(K)
            ys = [torch.empty(M, W.N, dtype=bf, device=dev) for W in self.W]
            for c, x in enumerate(self.xs):
                self._add_quant(f"amax+quant chunk{c}", x, K, q)
                for W, y, lin in zip(self.W, ys, wl.linears):
                    self.ops.append((f"gemm {lin.name} chunk{c}", "gemm",
                                     lambda st, q=q, W=W, y=y: mq.mq_gemm_nvfp4(
                                         q["codes"], q["sf"], q["s"], M, W.handle, y, W.N, st)))
                    self.flops += 2.0 * M * W.N * W.K
        else:
            self.xs = []
            self.rs = []
            for i, (W, lin) in enumerate(zip(self.W, wl.linears)):
                q = qbuf(W.K)
                y = torch.empty(M, W.N, dtype=bf, device=dev)
                if wl.rmsnorm and i == 0:
                    # RMSNorm of the residual stream writes x and its amax
                    r = workloads.layer_activation(wl, W.K, i, device=str(dev))
                    gain = workloads.rmsnorm_gain(W.K, wl.seed, 50, device=str(dev))
                    x = torch.empty(M, W.K, dtype=bf, device=dev)
                    self.rs.append((r, gain))
                    self.xs.append(x)

                    def rms(st, r=r, gain=gain, x=x, q=q, K=W.K):
                        q["n"] = mq.mq_rmsnorm_amax(r, gain, RMS_EPS, M, K, K, x, q["part"], st)

                    self.ops.append((f"rmsnorm+amax x{i}", "amax", rms))
                    self.ops.append((f"quant x{i}", "quant",
                                     lambda st, x=x, q=q, K=W.K: mq.mq_quantize_nvfp4(
                                         x, M, K, K, q["codes"], q["sf"], q["s"],
                                         amax_partials=q["part"], n_partials=q["n"], stream=st)))
                else:
                    x = workloads.layer_activation(wl, W.K, i, device=str(dev))
                    self.xs.append(x)
                    self._add_quant(f"amax+quant x{i}", x, W.K, q)
                self.ops.append((f"gemm {lin.name}", "gemm",
                                 lambda st, q=q, W=W, y=y: mq.mq_gemm_nvfp4(
                                     q["codes"], q["sf"], q["s"], M, W.handle, y, W.N, st)))
                self.flops += 2.0 * M * W.N * W.K
        # decode (phase switch) on every weight handle at M = 1: BF16, and
        # uniform NVFP4 (W4A4, tokens quantized inside the call) for comparison
        self.dec, self.decode_bytes = self.decode_calls(1, "bf16")
        self.dec4, self.decode4_bytes = self.decode_calls(1, "nvfp4")
        self.launches = len(self.ops) + len(self.dec)   # one kernel per op / decode call

    def decode_calls(self, Md: int, kind: str):
        """Decode of Md tokens on every weight handle (the first activation's
        first rows where K matches, zeros otherwise).  Returns (launch
        closures, bytes moved per pass: the weight at 2 (BF16) or 0.5625
        (NVFP4 codes + E4M3 scales) bytes per parameter, plus x and y)."""
        mq, dev, bf = self.mq, self.dev, torch.bfloat16
        calls, nbytes = [], 0.0
        x0 = self.xs[0][:Md].contiguous()
        for W in self.W:
            xd = x0 if W.K == x0.shape[1] else torch.zeros(Md, W.K, dtype=bf, device=dev)
            yd = torch.empty(Md, W.N, dtype=bf, device=dev)
            if kind == "bf16":
                calls.append(lambda st, W=W, xd=xd, yd=yd: mq.mq_decode_linear_bf16(
                    W.handle, xd, Md, yd, st))
                nbytes += 2.0 * W.N * W.K
            else:
                nb = mq.mq_workspace_bytes(Md, W.K)
                ws4 = torch.empty(nb, dtype=torch.uint8, device=dev)
                calls.append(lambda st, W=W, xd=xd, yd=yd, ws4=ws4, nb=nb:
                             mq.mq_decode_linear_nvfp4(W.handle, xd, Md, yd, ws4, nb, st))
                nbytes += 0.5625 * W.N * W.K
            nbytes += 2.0 * Md * W.K + 2.0 * Md * W.N
        return calls, nbytes

    def run_bf16(self):
        """The same-shape BF16 path (cuBLAS through torch.matmul; SiLU * up in
        torch for MLPs): the comparator of the speedup, not part of the library."""
        wl, P = self.wl, self
        if wl.swiglu:
            for item in P.plan:
                if item[0] == "mlp":
                    _, i, j, xi = item
                    gu = torch.matmul(P.xs[xi], P.ws[i].t())
                    I = gu.shape[1] // 2
                    h = torch.nn.functional.silu(gu[:, :I]) * gu[:, I:]
                    torch.matmul(h, P.ws[j].t())
                else:
                    _, i, xi = item
                    torch.matmul(P.xs[xi], P.ws[i].t())
        elif wl.chunks > 1:
            for x in P.xs:
                for w in P.ws:
                    torch.matmul(x, w.t())
        else:
            for i, (x, w) in enumerate(zip(P.xs, P.ws)):
                if wl.rmsnorm and i == 0:
                    r, gain = P.rs[0]
                    x = torch.nn.functional.rms_norm(r, (r.shape[1],), weight=gain, eps=RMS_EPS)
                torch.matmul(x, w.t())

    def _add_quant(self, name, x, K, q):
        mq, M = self.mq, self.M

        def amax(st):
            q["n"] = mq.mq_tensor_amax(x, M, K, K, q["part"], st)

        self.ops.append((name.replace("amax+quant", "amax"), "amax", amax))
        self.ops.append((name.replace("amax+quant", "quant"), "quant",
                         lambda st: mq.mq_quantize_nvfp4(x, M, K, K, q["codes"], q["sf"], q["s"],
                                                         amax_partials=q["part"],
                                                         n_partials=q["n"], stream=st)))

    def run_prefill(self, st):
        for _, _, f in self.ops:
            f(st)

    def run_decode(self, st):
        for f in self.dec:
            f(st)

    def free(self):
        for W in self.W:
            W.free()


# workloads measured next to the headline one (each in its own Prefill, freed
# before the next): the 8B SwiGLU MLP with decode at 1 and 8 tokens, the
# chunked 131072-token prefill and the 70B layer's linears
PER_CONFIG = ("llama3_8b_mlp", "chunked_131k", "llama3_70b_layer")


def measure_light(key, args, mq, dev, stream, flush, capture, replay_ms, pk):
    """One workload's prefill timed like the headline (CUDA events at the step
    boundaries, L2 flushed between steps, kernels chained by programmatic
    dependent launch), the GEMM-only rate from a pass with an event after
    every launch, the cuBLAS BF16 comparator, and decode device times from
    CUDA-graph replays.  Returns a dict for the bench line's per_config."""
    wl = workloads.WORKLOADS[key]
    P = Prefill(wl, mq, dev)
    ev = lambda: torch.cuda.Event(enable_timing=True)
    steps, warm = args.config_steps, max(3, args.warmup)
    for _ in range(warm):
        flush()
        P.run_prefill(stream)
    torch.cuda.synchronize()
    if mq.mq_check(stream) != 0:
        raise RuntimeError(f"device error in {key}")
    pairs = [(ev(), ev()) for _ in range(steps)]
    for a, b in pairs:
        flush()
        a.record(stream)
        P.run_prefill(stream)
        b.record(stream)
    torch.cuda.synchronize()
    t_ms = sum(a.elapsed_time(b) for a, b in pairs) / steps
    # GEMM launches alone (events between launches)
    gemm_ms = 0.0
    for _ in range(2):
        flush()
        evs = [ev() for _ in range(len(P.ops) + 1)]
        evs[0].record(stream)
        for i, (_, _, f) in enumerate(P.ops):
            f(stream)
            evs[i + 1].record(stream)
        torch.cuda.synchronize()
        gemm_ms += sum(evs[i].elapsed_time(evs[i + 1]) for i, o in enumerate(P.ops)
                       if o[1] == "gemm") / 2
    bts = []
    P.run_bf16()
    for _ in range(3):
        flush()
        a, b = ev(), ev()
        a.record(stream)
        P.run_bf16()
        b.record(stream)
        torch.cuda.synchronize()
        bts.append(a.elapsed_time(b))
    bf16_ms = statistics.median(bts)
    fp4_peak = pk["bf16"] * FP4_OVER_BF16
    tokens = wl.M * max(1, wl.chunks)
    tf = P.flops / (t_ms * 1e-3) / 1e12
    r = {"workload": wl.name, "tokens": tokens,
         "linears": [{"name": l.name, "N": l.N, "K": l.K} for l in wl.linears],
         "activations": wl.act, "seed": wl.seed, "steps": steps, "warmup": warm,
         "prefill_ms": round(t_ms, 4), "tflops": round(tf, 2),
         "fp4_peak_frac": round(tf / fp4_peak, 4),
         "gemm_only_tflops": round(P.flops / (gemm_ms * 1e-3) / 1e12, 2),
         "bf16_cublas_ms": round(bf16_ms, 4), "speedup_vs_bf16": round(bf16_ms / t_ms, 3),
         "tokens_per_s": round(tokens / (t_ms * 1e-3), 1)}
    if wl.chunks > 1:
        r["chunks"] = wl.chunks
        r["per_chunk_ms"] = round(t_ms / wl.chunks, 4)
        r["total_ms"] = round(t_ms, 4)
    # decode at the workload's token counts: device time per pass from graph
    # replays of R x (flush, decode of every handle) minus R flushes
    if len(wl.decode_M) > 1:
        R = 16
        t_flush = replay_ms(capture([]))
        dec = {}
        for Md in wl.decode_M:
            for kind in ("bf16", "nvfp4"):
                calls, nbytes = P.decode_calls(Md, kind)
                for f in calls:      # first calls outside the capture
                    f(stream)
                torch.cuda.synchronize()
                g = capture(calls)
                d_ms = (replay_ms(g) - t_flush) / R
                del g
                dec[f"{kind}_m{Md}_ms"] = round(d_ms, 4)
                dec[f"{kind}_m{Md}_gbs"] = round(nbytes / (d_ms * 1e-3) / 1e9, 1)
        r["decode"] = dec
        r["decode_note"] = ("device time per pass over every handle (graph replays, L2 flushed "
                            "before each pass); GB/s over the weight bytes (2 or 0.5625 B/param) "
                            "+ x + y; nvfp4 = W4A4 with the tokens quantized inside the call")
    P.free()
    del P
    return r


def measure_layer(args, mq, dev, stream, flush, capture, replay_ms, pk):
    """A whole Llama-3-8B-shaped layer at 8192 tokens, NVFP4 prefill against
    the same layer in BF16: RMSNorm -> QKV -> causal attention (32 query
    heads, 8 KV heads, head dim 128; writes the BF16 KV cache) -> O ->
    RMSNorm -> gate/up -> SwiGLU -> down.  NVFP4 path: this library's kernels
    only (the RMSNorms and the attention emit the next quantizer's amax).
    BF16 path: torch's rms_norm, cuBLAS matmuls, torch's scaled-dot-product
    attention (flash / cuDNN) and a copy of K, V into the cache.  Also: each
    attention alone, and the decode step's attention block (BF16 QKV ->
    attention over the cache -> BF16 O) for 1 and 8 new tokens."""
    M, H, Hkv, Dh, E, I = 8192, 32, 8, 128, 4096, 14336
    Nqkv = (H + 2 * Hkv) * Dh
    seed = 6
    bf, u8, f32 = torch.bfloat16, torch.uint8, torch.float32
    d = str(dev)
    x = workloads.activation("channel_gain", M, E, seed, 0, device=d)
    g1 = workloads.rmsnorm_gain(E, seed, 1, device=d)
    g2 = workloads.rmsnorm_gain(E, seed, 2, device=d)
    ws_ = [workloads.weight(n, k, 0.02, seed, 100 + i, device=d)
           for i, (n, k) in enumerate([(Nqkv, E), (E, E), (2 * I, E), (E, I)])]
    Wqkv, Wo, Wgu, Wd = [mq.Weight(w) for w in ws_]
    S_max = M + 16
    kc = torch.zeros(Hkv, S_max, Dh, dtype=bf, device=dev)
    vc = torch.zeros_like(kc)
    xn = torch.empty(M, E, dtype=bf, device=dev)
    qkv = torch.empty(M, Nqkv, dtype=bf, device=dev)
    o = torch.empty(M, E, dtype=bf, device=dev)
    yo = torch.empty(M, E, dtype=bf, device=dev)
    xn2 = torch.empty(M, E, dtype=bf, device=dev)
    h = torch.empty(M, I, dtype=bf, device=dev)
    y = torch.empty(M, E, dtype=bf, device=dev)

    def qb(K):
        return dict(codes=torch.empty(M, K // 2, dtype=u8, device=dev),
                    sf=torch.empty(mq.mq_sf_bytes(M, K), dtype=u8, device=dev),
                    s=torch.empty(1, dtype=f32, device=dev),
                    part=torch.empty(mq.MQ_AMAX_PARTIALS_MAX, dtype=f32, device=dev))
    q1, q2, q3, q4 = qb(E), qb(E), qb(E), qb(I)
    st = {}

    def attn():
        st["n2"] = mq.mq_attention_prefill_bf16(qkv, M, H, Hkv, Dh, kc, vc, S_max, o, q2["part"], stream)

    def nvfp4_layer():
        st["n1"] = mq.mq_rmsnorm_amax(x, g1, RMS_EPS, M, E, E, xn, q1["part"], stream)
        mq.mq_quantize_nvfp4(xn, M, E, E, q1["codes"], q1["sf"], q1["s"], amax_partials=q1["part"],
                             n_partials=st["n1"], stream=stream)
        mq.mq_gemm_nvfp4(q1["codes"], q1["sf"], q1["s"], M, Wqkv.handle, qkv, Nqkv, stream)
        attn()
        mq.mq_quantize_nvfp4(o, M, E, E, q2["codes"], q2["sf"], q2["s"], amax_partials=q2["part"],
                             n_partials=st["n2"], stream=stream)
        mq.mq_gemm_nvfp4(q2["codes"], q2["sf"], q2["s"], M, Wo.handle, yo, E, stream)
        st["n3"] = mq.mq_rmsnorm_amax(yo, g2, RMS_EPS, M, E, E, xn2, q3["part"], stream)
        mq.mq_quantize_nvfp4(xn2, M, E, E, q3["codes"], q3["sf"], q3["s"], amax_partials=q3["part"],
                             n_partials=st["n3"], stream=stream)
        st["n4"] = mq.mq_gemm_nvfp4_swiglu(q3["codes"], q3["sf"], q3["s"], M, Wgu.handle, h,
                                           q4["part"], stream)
        mq.mq_quantize_nvfp4(h, M, I, I, q4["codes"], q4["sf"], q4["s"], amax_partials=q4["part"],
                             n_partials=st["n4"], stream=stream)
        mq.mq_gemm_nvfp4(q4["codes"], q4["sf"], q4["s"], M, Wd.handle, y, E, stream)

    def sdpa(t=None):
        t = qkv if t is None else t
        q = t[:, :H * Dh].view(M, H, Dh).transpose(0, 1)
        k = t[:, H * Dh:(H + Hkv) * Dh].view(M, Hkv, Dh).transpose(0, 1)
        v = t[:, (H + Hkv) * Dh:].view(M, Hkv, Dh).transpose(0, 1)
        kc[:, :M].copy_(k)
        vc[:, :M].copy_(v)
        return torch.nn.functional.scaled_dot_product_attention(
            q.unsqueeze(0), k.unsqueeze(0), v.unsqueeze(0), is_causal=True,
            enable_gqa=True)[0].transpose(0, 1).reshape(M, H * Dh)

    def bf16_layer():
        a = torch.nn.functional.rms_norm(x, (E,), weight=g1, eps=RMS_EPS)
        ob = sdpa(torch.matmul(a, ws_[0].t()))
        yb = torch.matmul(ob, ws_[1].t())
        a2 = torch.nn.functional.rms_norm(yb, (E,), weight=g2, eps=RMS_EPS)
        gu = torch.matmul(a2, ws_[2].t())
        hb = torch.nn.functional.silu(gu[:, :I]) * gu[:, I:]
        torch.matmul(hb, ws_[3].t())

    ev = lambda: torch.cuda.Event(enable_timing=True)

    def timed_interleaved(fns, n):
        """Median event time of each function, the functions taking turns
        (each after an L2 flush) so that all of them see the same clock and
        power state; this measurement follows seconds of dense GEMMs."""
        for fn in fns:
            fn()
        torch.cuda.synchronize()
        ts = [[] for _ in fns]
        for _ in range(n):
            for i, fn in enumerate(fns):
                flush()
                a, b = ev(), ev()
                a.record(stream)
                fn()
                b.record(stream)
                torch.cuda.synchronize()
                ts[i].append(a.elapsed_time(b))
        return [statistics.median(t) for t in ts]

    n = max(3, args.config_steps)
    nvfp4_layer()
    torch.cuda.synchronize()
    if mq.mq_check(stream) != 0:
        raise RuntimeError("device error in the layer")
    t_nv, t_attn, t_sdpa, t_bf = timed_interleaved([nvfp4_layer, attn, sdpa, bf16_layer], n)
    if mq.mq_check(stream) != 0:
        raise RuntimeError("device error in the layer")
    attn_flops = 4.0 * Dh * H * M * (M + 1) / 2
    lin_flops = 2.0 * M * E * (Nqkv + E + 2 * I) + 2.0 * M * I * E
    r = {"workload": "llama3-8b layer (rmsnorm, qkv, causal gqa attention + kv cache, o, rmsnorm, "
                     "swiglu mlp), 8192 tokens", "tokens": M, "heads": H, "kv_heads": Hkv,
         "head_dim": Dh, "steps": n, "warmup": 1,
         "prefill_layer_ms": round(t_nv, 4), "bf16_layer_ms": round(t_bf, 4),
         "layer_speedup_vs_bf16": round(t_bf / t_nv, 3),
         "layer_tflops": round((attn_flops + lin_flops) / (t_nv * 1e-3) / 1e12, 1),
         "attention_ms": round(t_attn, 4),
         "attention_tflops": round(attn_flops / (t_attn * 1e-3) / 1e12, 1),
         "sdpa_ms": round(t_sdpa, 4),
         "sdpa_tflops": round(attn_flops / (t_sdpa * 1e-3) / 1e12, 1),
         "attention_flops": attn_flops, "linear_flops": lin_flops,
         "note": "NVFP4 layer: this library's kernels only; BF16 layer: torch rms_norm, cuBLAS, "
                 "torch SDPA (flash/cuDNN) + cache copy; sdpa_ms includes the K/V cache copy; "
                 "L2 flushed before each timed layer; medians of event-timed runs, the four functions taking turns"}
    # decode step's attention block on the cache the prefill wrote: BF16 QKV
    # -> attention over 8192 + m positions -> BF16 O (device time, graph replays)
    R = 16
    t_flush = replay_ms(capture([]))
    dec = {}
    for m in (1, 8):
        xt = x[:m].contiguous()
        qkv_t = torch.empty(m, Nqkv, dtype=bf, device=dev)
        ot = torch.empty(m, E, dtype=bf, device=dev)
        yt = torch.empty(m, E, dtype=bf, device=dev)
        nbd = mq.mq_attention_decode_workspace_bytes(m, M, H, Hkv, Dh)
        wsd = torch.empty(nbd, dtype=u8, device=dev)
        body = [lambda s2, xt=xt, qkv_t=qkv_t, m=m: mq.mq_decode_linear_bf16(Wqkv.handle, xt, m, qkv_t, s2),
                lambda s2, qkv_t=qkv_t, ot=ot, wsd=wsd, nbd=nbd, m=m: mq.mq_attention_decode_bf16(
                    qkv_t, m, M, H, Hkv, Dh, kc, vc, S_max, ot, wsd, nbd, s2),
                lambda s2, ot=ot, yt=yt, m=m: mq.mq_decode_linear_bf16(Wo.handle, ot, m, yt, s2)]
        for f in body:
            f(stream)
        torch.cuda.synchronize()
        g = capture(body)
        dec[f"m{m}_ms"] = round((replay_ms(g) - t_flush) / R, 4)
        del g
    r["decode_attention_block"] = dec
    r["decode_note"] = ("BF16 QKV decode linear -> decode attention over the 8192-token cache "
                        "(appending the new tokens) -> BF16 O decode linear; device time per step "
                        "from graph replays after an L2 flush")
    if mq.mq_check(stream) != 0:
        raise RuntimeError("device error in the layer decode")
    for W in (Wqkv, Wo, Wgu, Wd):
        W.free()
    return r


def run_gpu(args, wl, world, rank):
    from nvfp4_quantized_prefill_b200 import binding as mq
    mq.lib()
    dev = torch.device("cuda", torch.cuda.current_device())
    stream = torch.cuda.current_stream()
    pk = peaks()
    P = Prefill(wl, mq, dev)
    flush_w = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    flush_r = torch.ones(256 << 20, dtype=torch.uint8, device=dev)
    sink = torch.empty((), dtype=torch.int64, device=dev)

    def flush():
        flush_w.zero_()
        torch.sum(flush_r, dim=0, dtype=torch.int64, out=sink)

    nop = len(P.ops)
    ev = lambda: torch.cuda.Event(enable_timing=True)

    def step(evs):
        # the timed step: events only around the prefill and the decode, so
        # consecutive kernels may overlap through programmatic dependent launch
        evs[0].record(stream)
        P.run_prefill(stream)
        evs[1].record(stream)
        P.run_decode(stream)
        evs[2].record(stream)

    def step_breakdown(evs):
        # an event after every launch: per-kernel durations
        evs[0].record(stream)
        for i, (_, _, f) in enumerate(P.ops):
            f(stream)
            evs[i + 1].record(stream)

    for _ in range(args.warmup):
        flush()
        step([ev() for _ in range(3)])
    torch.cuda.synchronize()
    if mq.mq_check(stream) != 0:
        raise RuntimeError("device error during warm-up")

    all_evs = [[ev() for _ in range(3)] for _ in range(args.steps)]
    clocks = ClockSampler(int(os.environ.get("LOCAL_RANK", "0")))
    barrier(world)
    torch.cuda.synchronize()
    with clocks:
        time.sleep(0.3)
        for k in range(args.steps):
            flush()
            step(all_evs[k])
        torch.cuda.synchronize()
    barrier(world)
    if mq.mq_check(stream) != 0:
        raise RuntimeError("device error during timing")
    t_prefill = sum(e[0].elapsed_time(e[1]) for e in all_evs)
    t_dec = sum(e[1].elapsed_time(e[2]) for e in all_evs)
    t_step = sum(e[0].elapsed_time(e[2]) for e in all_evs)

    # per-launch breakdown: the same steps again with an event after each launch
    bd_evs = [[ev() for _ in range(nop + 1)] for _ in range(args.steps)]
    for k in range(args.steps):
        flush()
        step_breakdown(bd_evs[k])
    torch.cuda.synchronize()
    # Decode (M = 1) on the same handles, each pass on a cold L2, as device
    # time: CUDA-graph replays of R x (L2 flush, QKV decode, O decode) minus
    # R x (L2 flush).  One host launch per replay, so no host gaps between
    # these short kernels, and R passes per event pair, so the event clock's
    # granularity does not matter.  BF16 (the phase-switch path, isolated
    # from the prefill) and uniform NVFP4 (W4A4).
    for f in P.dec4:   # first calls outside the capture
        f(stream)
    torch.cuda.synchronize()
    R = 16

    def capture(body):
        g = torch.cuda.CUDAGraph()
        s2 = torch.cuda.Stream()
        s2.wait_stream(stream)
        with torch.cuda.stream(s2):
            with torch.cuda.graph(g, stream=s2):
                for _ in range(R):
                    flush()
                    for f in body:
                        f(s2)
        torch.cuda.synchronize()
        return g

    def replay_ms(g):
        ts = []
        for _ in range(3):
            a, b = ev(), ev()
            a.record()
            g.replay()
            b.record()
            torch.cuda.synchronize()
            ts.append(a.elapsed_time(b))
        return statistics.median(ts)

    def eager_ms(body):   # without graphs (if capture fails): host gaps included
        ts = []
        for _ in range(max(3, min(args.steps, 10))):
            flush()
            a, b = ev(), ev()
            a.record(stream)
            for f in body:
                f(stream)
            b.record(stream)
            torch.cuda.synchronize()
            ts.append(a.elapsed_time(b))
        return statistics.mean(ts)

    decode_timing = "cuda-graph replay"
    op_device_us = {}
    try:
        g_flush, g_dec, g_dec4 = capture([]), capture(P.dec), capture(P.dec4)
        t_flush = replay_ms(g_flush)
        t_dec_iso = (replay_ms(g_dec) - t_flush) / R
        t_dec4 = (replay_ms(g_dec4) - t_flush) / R
        del g_flush, g_dec, g_dec4
        # every prefill launch alone on a cold L2, same method (device time;
        # inside the step a quantize finds X partly in L2 after its amax)
        for name, _, f in P.ops:
            g = capture([f])
            op_device_us[name] = round((replay_ms(g) - t_flush) / R * 1e3, 2)
            del g
    except Exception as e:  # report, do not hide
        decode_timing = f"eager (graph capture failed: {type(e).__name__})"
        torch.cuda.synchronize()
        t_dec_iso, t_dec4 = eager_ms(P.dec), eager_ms(P.dec4)
    if mq.mq_check(stream) != 0:
        raise RuntimeError("device error during the decode passes")
    per_kind = {"amax": 0.0, "quant": 0.0, "gemm": 0.0}
    per_op = [0.0] * nop
    for evs in bd_evs:
        for i, (_, kind, _) in enumerate(P.ops):
            d = evs[i].elapsed_time(evs[i + 1])
            per_kind[kind] += d
            per_op[i] += d
    K_ = args.steps
    t_prefill_ms = t_prefill / K_
    value, t_prefill_max, total_flops = aggregate(P.flops, t_prefill_ms, world)
    t_step_max = reduce_over_ranks(t_step / K_, world, "MAX")
    gemm_ms = per_kind["gemm"] / K_
    n_gemm = sum(1 for o in P.ops if o[1] == "gemm")
    fp4_peak = pk["bf16"] * FP4_OVER_BF16
    achieved = P.flops / (gemm_ms * 1e-3) / 1e12

    # ---- CUDA-graph replay of the same prefill: a launch-overhead cross-check
    graph_ms = None
    try:
        g = torch.cuda.CUDAGraph()
        s2 = torch.cuda.Stream()
        s2.wait_stream(stream)
        with torch.cuda.stream(s2):
            with torch.cuda.graph(g, stream=s2):
                P.run_prefill(s2)
        torch.cuda.synchronize()
        gt = []
        for _ in range(max(3, min(args.steps, 10))):
            flush()
            a, b = ev(), ev()
            a.record(stream)
            g.replay()
            b.record(stream)
            torch.cuda.synchronize()
            gt.append(a.elapsed_time(b))
        graph_ms = statistics.median(gt)
        del g
    except Exception as e:  # report, do not hide
        graph_ms = f"unavailable: {type(e).__name__}: {e}"[:200]
    if mq.mq_check(stream) != 0:
        raise RuntimeError("device error during graph replay")

    # ---- the same-shape BF16 path (cuBLAS through torch.matmul): comparator only
    bf16_ms = None
    try:
        bf16_prefill = P.run_bf16
        bf16_prefill()
        bt = []
        for _ in range(max(3, min(args.steps, 10))):
            flush()
            a, b = ev(), ev()
            a.record(stream)
            bf16_prefill()
            b.record(stream)
            torch.cuda.synchronize()
            bt.append(a.elapsed_time(b))
        bf16_ms = statistics.median(bt)
    except Exception as e:
        bf16_ms = None

    # ---- RMSNorm-fed linear: the same chain with torch's RMSNorm and a
    # separate amax pass (what the fused RMSNorm + amax replaces)
    unfused_ms = None
    if wl.rmsnorm:
        r, gain = P.rs[0]
        W0 = P.W[0]
        qu = dict(codes=torch.empty(wl.M, W0.K // 2, dtype=torch.uint8, device=dev),
                  sf=torch.empty(mq.mq_sf_bytes(wl.M, W0.K), dtype=torch.uint8, device=dev),
                  s=torch.empty(1, dtype=torch.float32, device=dev),
                  part=torch.empty(mq.MQ_AMAX_PARTIALS_MAX, dtype=torch.float32, device=dev))
        yu = torch.empty(wl.M, W0.N, dtype=torch.bfloat16, device=dev)

        def unfused():
            xu = torch.nn.functional.rms_norm(r, (W0.K,), weight=gain, eps=RMS_EPS)
            n = mq.mq_tensor_amax(xu, wl.M, W0.K, W0.K, qu["part"], stream)
            mq.mq_quantize_nvfp4(xu, wl.M, W0.K, W0.K, qu["codes"], qu["sf"], qu["s"],
                                 amax_partials=qu["part"], n_partials=n, stream=stream)
            mq.mq_gemm_nvfp4(qu["codes"], qu["sf"], qu["s"], wl.M, W0.handle, yu, W0.N, stream)
        unfused()
        ut = []
        for _ in range(max(3, min(args.steps, 10))):
            flush()
            a, b = ev(), ev()
            a.record(stream)
            unfused()
            b.record(stream)
            torch.cuda.synchronize()
            ut.append(a.elapsed_time(b))
        unfused_ms = statistics.median(ut)

    # ---- end to end through the public call: pinned host X -> device, prefill
    # linear (amax + quantize + GEMM inside), result back to pinned host memory
    e2e = None
    if not wl.swiglu and wl.chunks == 1 and not wl.rmsnorm:
        M = wl.M
        xs_h = [x.cpu().pin_memory() for x in P.xs]
        ys_h = [torch.empty(M, W.N, dtype=torch.bfloat16).pin_memory() for W in P.W]
        xs_d = [torch.empty_like(x) for x in P.xs]
        ys_d = [torch.empty(M, W.N, dtype=torch.bfloat16, device=dev) for W in P.W]
        wsb = max(mq.mq_workspace_bytes(M, W.K) for W in P.W)
        wsp = torch.empty(wsb, dtype=torch.uint8, device=dev)

        # host->device copies, the prefill and device->host copies on three
        # streams, so PCIe carries X in and Y out at the same time while the
        # GPU computes; events keep each buffer's reuse ordered
        h2d, d2h = torch.cuda.Stream(), torch.cuda.Stream()
        n_proj = len(P.W)
        x_ready = [ev() for _ in range(n_proj)]
        x_free = [ev() for _ in range(n_proj)]
        y_ready = [ev() for _ in range(n_proj)]
        y_free = [ev() for _ in range(n_proj)]
        for e in x_free + y_free:
            e.record(stream)

        def e2e_step():
            for i, (W, xh, xd, yd, yh) in enumerate(zip(P.W, xs_h, xs_d, ys_d, ys_h)):
                h2d.wait_event(x_free[i])
                with torch.cuda.stream(h2d):
                    xd.copy_(xh, non_blocking=True)
                x_ready[i].record(h2d)
                stream.wait_event(x_ready[i])
                stream.wait_event(y_free[i])
                mq.mq_prefill_linear_nvfp4(W.handle, xd, M, yd, wsp, wsb, stream)
                x_free[i].record(stream)
                y_ready[i].record(stream)
                d2h.wait_event(y_ready[i])
                with torch.cuda.stream(d2h):
                    yh.copy_(yd, non_blocking=True)
                y_free[i].record(d2h)

        for _ in range(2):
            e2e_step()
        torch.cuda.synchronize()
        e0, e1 = ev(), ev()
        n_e2e = max(2, min(args.steps, 10))
        barrier(world)
        torch.cuda.synchronize()
        e0.record(stream)
        h2d.wait_event(e0)
        for _ in range(n_e2e):
            e2e_step()
        for e in y_free:
            stream.wait_event(e)
        e1.record(stream)
        torch.cuda.synchronize()
        e2e_ms = reduce_over_ranks(e0.elapsed_time(e1) / n_e2e, world, "MAX")
        e2e = {"value": round(total_flops / (e2e_ms * 1e-3) / 1e12, 3), "unit": "TFLOP/s",
               "h2d_bytes_per_step": sum(x.numel() * 2 for x in P.xs),
               "d2h_bytes_per_step": sum(M * W.N * 2 for W in P.W),
               "path": "mq_prefill_linear_nvfp4 per projection; pinned-host X in and Y out "
                       "on their own streams, overlapping each other and the compute"}

    # ---- the other workloads, lighter: prefill TFLOP/s incl. quantization,
    # GEMM-only TFLOP/s, the BF16 comparator, tokens/s, and decode at the
    # workload's token counts (BF16 and W4A4)
    per_config = None
    if args.per_config and world == 1:
        per_config = {}
        for key in PER_CONFIG:
            if key == args.workload:
                continue
            per_config[key] = measure_light(key, args, mq, dev, stream, flush, capture,
                                            replay_ms, pk)
            torch.cuda.empty_cache()
        per_config["llama3_8b_layer"] = measure_layer(args, mq, dev, stream, flush, capture,
                                                      replay_ms, pk)
        torch.cuda.empty_cache()
        if mq.mq_check(stream) != 0:
            raise RuntimeError("device error during the per-workload measurements")

    traffic, traffic_launches = recorded_traffic(args.workload)
    clk = clocks.summary()
    out = {
        "metric": METRIC,
        "value": round(value, 2),
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(t_step_max, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "nvfp4 (e2m1 codes, e4m3 per-16 scales, fp32 tensor scale) -> fp32 acc -> bf16",
        "data": "synthetic (seeded recipe, random-init weights of the named shapes)",
        "config": {
            "workload": wl.name,
            "workload_key": args.workload,
            "tokens": wl.M * max(1, wl.chunks),
            "linears": [{"name": l.name, "N": l.N, "K": l.K} for l in wl.linears],
            "activations": wl.act,
            "seed": wl.seed,
            "step": "prefill (amax -> NVFP4 quantize -> tcgen05 block-scaled GEMM per "
                    "activation) then BF16 decode M=1 on the same weight handles",
            "l2": "flushed between steps: write 256 MiB, then read another 256 MiB "
                  "(outside the timed intervals)",
            "parallelism": f"replicas x{world} (no exchange)",
        },
        "prefill_ms": round(t_prefill_max, 4),
        "breakdown_ms": {k: round(v / K_, 4) for k, v in per_kind.items()},
        "breakdown_note": "separate pass after the timed steps, one event after every launch "
                          "(events between kernels stop them from overlapping)",
        "per_launch_ms": {P.ops[i][0]: round(per_op[i] / K_, 4) for i in range(nop)},
        "decode_m1_ms": round(t_dec / K_, 4),
        "decode_gbs": round(P.decode_bytes / (t_dec / K_ * 1e-3) / 1e9, 1),
        "decode_m1_isolated_ms": round(t_dec_iso, 4),
        "decode_isolated_gbs": round(P.decode_bytes / (t_dec_iso * 1e-3) / 1e9, 1),
        "decode_nvfp4_m1_ms": round(t_dec4, 4),
        "decode_nvfp4_gbs": round(P.decode4_bytes / (t_dec4 * 1e-3) / 1e9, 1),
        "decode_note": "decode_m1_ms: the BF16 decode of every handle inside the timed step, "
                       "right after the prefill (whose dirty output lines L2 writes back "
                       "meanwhile); *_isolated_ms / decode_nvfp4_m1_ms: device time per pass "
                       "from CUDA-graph replays of (L2 flush, decode of every handle) minus "
                       "the flush alone; NVFP4 = W4A4, tokens quantized inside the kernel; "
                       "GB/s over the weight bytes (2 or 0.5625 B/param) + x + y",
        "decode_timing": decode_timing,
        "op_device_us": op_device_us,
        "op_device_note": "each prefill launch alone after an L2 flush, device time from "
                          "CUDA-graph replays (16 x (flush, launch) minus 16 flushes); "
                          "per_launch_ms, from events between launches, also holds the "
                          "launch gaps",
        "graph_prefill_ms": round(graph_ms, 4) if isinstance(graph_ms, float) else graph_ms,
        "tokens_per_s": round(world * wl.M * max(1, wl.chunks) / (t_prefill_max * 1e-3), 1),
        "fp4_peak_frac": round(value / fp4_peak, 4),
        "gemm_only_tflops": round(achieved, 2),
        "bf16_cublas_ms": round(bf16_ms, 4) if bf16_ms else None,
        "speedup_vs_bf16": round(bf16_ms / t_prefill_ms, 3) if bf16_ms else None,
        **({"unfused_rmsnorm_ms": round(unfused_ms, 4),
            "unfused_note": "torch RMSNorm, then amax, quantize, GEMM (the separate amax pass "
                            "that the fused RMSNorm + amax removes)"} if unfused_ms else {}),
        "roofline": {
            "kernel": "gemm_nvf4_kernel (tcgen05.mma.cta_group::2 kind::mxf4nvf4 block16)",
            "bound": "tensor",
            "achieved": round(achieved, 2),
            "peak": round(fp4_peak, 1),
            "peak_source": f"{pk['source']} bf16 burst {pk['bf16']} TF/s x {FP4_OVER_BF16} "
                           "(nominal dense fp4/bf16 ratio), of measured",
            "unit": "TFLOP/s",
            "frac": round(achieved / fp4_peak, 4),
            "traffic": traffic,
            "traffic_launches": traffic_launches,
            # read beside frac: frac is against 4x the measured BF16 burst,
            # this is the tensor pipe's own busy fraction under ncu
            "tensor_pipe_active_pct_ncu": recorded_tensor_pipe(args.workload),
            "launches_per_step": n_gemm,
        },
        "e2e": e2e,
        "gpu_launches": P.launches * args.steps,
        "clocks": clk,
        **({"per_config": per_config} if per_config is not None else {}),
    }
    return out, P


def run_sharded(args, wl, world, rank):
    """The workload's prefill with the batch split by tokens across the ranks
    (row blocks of every activation; weights replicated): per activation and
    rank, shard amax -> one float all-reduced (max) over NCCL -> quantize with
    the batch's tensor scale -> GEMM, so every rank's rows are the single-GPU
    result.  Timed like the replica leg: CUDA events at the step boundaries,
    L2 flushed between steps, max over ranks; value = the batch's FLOPs over
    the slowest rank's time."""
    from nvfp4_quantized_prefill_b200 import binding as mq
    from nvfp4_quantized_prefill_b200 import sharded
    mq.lib()
    if wl.swiglu or wl.chunks > 1 or wl.rmsnorm:
        raise SystemExit("--sharded runs plain projection workloads (e.g. llama3_8b_qkv_o)")
    dev = torch.device("cuda", torch.cuda.current_device())
    stream = torch.cuda.current_stream()
    M = wl.M
    lo, hi = M * rank // world, M * (rank + 1) // world
    Ml = hi - lo
    ws_full = workloads.layer_weights(wl, device=str(dev))
    W = [mq.Weight(w) for w in ws_full]
    # every rank draws the same batch (same seed) and keeps its rows
    xs = [workloads.layer_activation(wl, w.shape[1], i, device=str(dev))[lo:hi].contiguous()
          for i, w in enumerate(ws_full)]
    ys = [torch.empty(Ml, Wi.N, dtype=torch.bfloat16, device=dev) for Wi in W]
    shard_ws = [sharded.ShardWorkspace.create(Ml, Wi.K, device=dev) for Wi in W]
    flush_w = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    flush_r = torch.ones(256 << 20, dtype=torch.uint8, device=dev)
    sink = torch.empty((), dtype=torch.int64, device=dev)

    def step():
        for Wi, x, y, sw in zip(W, xs, ys, shard_ws):
            sharded.shard_amax(x, sw, stream)
            if world > 1:
                sharded.exchange_amax(sw.amax)
            sharded.shard_finish(Wi, x, y, sw, stream)

    for _ in range(args.warmup):
        flush_w.zero_()
        torch.sum(flush_r, dim=0, dtype=torch.int64, out=sink)
        step()
    torch.cuda.synchronize()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.steps)]
    clocks = ClockSampler(int(os.environ.get("LOCAL_RANK", "0")))
    barrier(world)
    torch.cuda.synchronize()
    with clocks:
        time.sleep(0.3)
        for a, b in evs:
            flush_w.zero_()
            torch.sum(flush_r, dim=0, dtype=torch.int64, out=sink)
            a.record(stream)
            step()
            b.record(stream)
        torch.cuda.synchronize()
    barrier(world)
    if mq.mq_check(stream) != 0:
        raise RuntimeError("device error during the sharded steps")
    ms = sum(a.elapsed_time(b) for a, b in evs) / args.steps
    batch_flops = sum(2.0 * M * w.shape[0] * w.shape[1] for w in ws_full)
    value, max_ms = aggregate_sharded(batch_flops, ms, world)
    pk = peaks()
    out = {
        "metric": METRIC, "value": round(value, 2), "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(max_ms, 4),
        "higher_is_better": True, "scaling": "strong", "vs_baseline": None,
        "dtype": "nvfp4 (e2m1 codes, e4m3 per-16 scales, fp32 tensor scale) -> fp32 acc -> bf16",
        "data": "synthetic (seeded recipe, random-init weights of the named shapes)",
        "config": {"workload": wl.name, "workload_key": args.workload, "tokens": M,
                   "tokens_per_rank": Ml,
                   "linears": [{"name": l.name, "N": l.N, "K": l.K} for l in wl.linears],
                   "parallelism": f"token-sharded x{world}: rows split across ranks, weights "
                                  "replicated, one float all-reduced (max) per activation",
                   "l2": "flushed between steps (outside the timed intervals)"},
        "fp4_peak_frac": round(value / (world * pk["bf16"] * FP4_OVER_BF16), 4),
        "e2e": None,
        "e2e_note": "the sharded leg times the device path only; e2e is reported by the "
                    "default (replica) leg",
        "gpu_launches": args.steps * len(W) * 4,
        "clocks": clocks.summary(),
    }
    for Wi in W:
        Wi.free()
    return out


def profile_case(name: str):
    """Runs one small case a few times for a kernel capture (ncu -k ... -c 1):
    attention_prefill (4096 tokens, 8 query / 2 KV heads, head dim 128),
    attention_decode (1 token over a 32768-position cache, 32 query / 8 KV
    heads), decode_nvfp4 (one token through the Llama-3-8B QKV weight, W4A4)."""
    from nvfp4_quantized_prefill_b200 import binding as mq
    mq.lib()
    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    g = torch.Generator(device="cuda")
    g.manual_seed(9)
    if name == "attention_prefill":
        M, H, Hkv, D = 4096, 8, 2, 128
        qkv = torch.randn(M, (H + 2 * Hkv) * D, device=dev, generator=g).to(torch.bfloat16)
        kc = torch.zeros(Hkv, M + 8, D, dtype=torch.bfloat16, device=dev)
        vc = torch.zeros_like(kc)
        o = torch.empty(M, H * D, dtype=torch.bfloat16, device=dev)
        part = torch.empty(mq.MQ_AMAX_PARTIALS_MAX, dtype=torch.float32, device=dev)
        for _ in range(3):
            mq.mq_attention_prefill_bf16(qkv, M, H, Hkv, D, kc, vc, M + 8, o, part)
    elif name == "attention_decode":
        # one token over a 32768-position cache at the Llama-3-8B head counts
        # (134 MB of K and V, above the L2)
        S, H, Hkv, D = 32768, 32, 8, 128
        kc = torch.randn(Hkv, S + 8, D, device=dev, generator=g).to(torch.bfloat16)
        vc = torch.randn(Hkv, S + 8, D, device=dev, generator=g).to(torch.bfloat16)
        qkv = torch.randn(1, (H + 2 * Hkv) * D, device=dev, generator=g).to(torch.bfloat16)
        ot = torch.empty(1, H * D, dtype=torch.bfloat16, device=dev)
        nb = mq.mq_attention_decode_workspace_bytes(1, S, H, Hkv, D)
        ws = torch.empty(nb, dtype=torch.uint8, device=dev)
        for _ in range(3):
            mq.mq_attention_decode_bf16(qkv, 1, S, H, Hkv, D, kc, vc, S + 8, ot, ws, nb)
    elif name == "decode_nvfp4":
        w = (torch.randn(6144, 4096, device=dev, generator=g) * 0.02).to(torch.bfloat16)
        W = mq.Weight(w)
        x = torch.randn(1, 4096, device=dev, generator=g).to(torch.bfloat16)
        y = torch.empty(1, 6144, dtype=torch.bfloat16, device=dev)
        nb = mq.mq_workspace_bytes(1, 4096)
        ws = torch.empty(nb, dtype=torch.uint8, device=dev)
        for _ in range(3):
            mq.mq_decode_linear_nvfp4(W.handle, x, 1, y, ws, nb)
    else:
        raise SystemExit(f"unknown profile case {name}")
    torch.cuda.synchronize()
    if mq.mq_check() != 0:
        raise RuntimeError("device error in the profile case")
    print(json.dumps({"profile_case": name, "ok": True}))


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="mq", choices=["mq", "reference"])
    ap.add_argument("--workload", default="llama3_8b_qkv_o", choices=sorted(workloads.WORKLOADS))
    ap.add_argument("--cpu-rows", type=int, default=32,
                    help="activation rows per projection in the CPU oracle sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-per-config", dest="per_config", action="store_false",
                    help="skip the lighter measurement of the other workloads")
    ap.add_argument("--config-steps", type=int, default=5,
                    help="timed steps per workload in per_config")
    ap.add_argument("--profile-case", default=None,
                    choices=["attention_prefill", "attention_decode", "decode_nvfp4"],
                    help="run one small case for a kernel capture and exit")
    ap.add_argument("--sharded", action="store_true",
                    help="split the batch by tokens across the ranks (one float all-reduced "
                         "per activation) instead of running replicas")
    args = ap.parse_args()
    wl = workloads.WORKLOADS[args.workload]
    if args.profile_case:
        profile_case(args.profile_case)
        return

    if args.impl == "reference":
        rank = int(os.environ.get("RANK", "0"))
        if rank != 0:
            return
        import oracle
        ws_cpu = workloads.layer_weights(wl)
        xs_cpu = [workloads.layer_activation(wl, w.shape[1], i) for i, w in enumerate(ws_cpu)]
        wq = oracle_prepare(ws_cpu)
        times, fl = [], 0.0
        for _ in range(args.warmup):
            oracle_sample(xs_cpu, wq, 1)
        for _ in range(args.steps):
            fl, t = oracle_sample(xs_cpu, wq, args.cpu_rows)
            times.append(t)
        v = fl * len(times) / sum(times) / 1e12
        print(json.dumps({
            "impl": "reference", "metric": METRIC, "value": v, "unit": "TFLOP/s", "n_gpus": 1,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": sum(times) / len(times) * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "int64 exact sum / fp64",
            "data": "synthetic", "config": {"workload": wl.name, "tokens": wl.M},
            "cpu_baseline": {"value": v, "unit": "TFLOP/s", "cores": oracle.threads_used(),
                             "kind": "oracle",
                             "sample": f"{args.cpu_rows} activation rows per projection "
                                       "(full-tensor amax, row quantize, exact GEMM)"},
            "e2e": {"value": v, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}))
        return

    world, rank, local = dist_setup()
    if args.sharded:
        out = run_sharded(args, wl, world, rank)
        if rank == 0:
            print(json.dumps(out))
        if world > 1:
            torch.distributed.destroy_process_group()
        return
    out, P = run_gpu(args, wl, world, rank)
    if rank == 0 and world == 1 and not args.no_cpu_baseline and not wl.swiglu and wl.chunks == 1 and not wl.rmsnorm:
        import oracle
        xs_cpu = [x.cpu() for x in P.xs]
        ws_cpu = [w.cpu() for w in P.ws]
        fl, t = oracle_sample(xs_cpu, oracle_prepare(ws_cpu), args.cpu_rows)
        out["cpu_baseline"] = {"value": fl / t / 1e12, "unit": "TFLOP/s",
                               "cores": oracle.threads_used(), "kind": "oracle",
                               "sample": f"{args.cpu_rows} activation rows per projection "
                                         "(full-tensor amax, row quantize, exact GEMM); "
                                         f"{t:.1f} s"}
    P.free()
    if rank == 0:
        print(json.dumps(out))
    if world > 1:
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
