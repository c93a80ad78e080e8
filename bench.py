"""Benchmark of the prefill-phase NVFP4 linear layer (Mix-Quant hot path).

One step = one pass of the hot path over one batch of synthetic input: for
each projection of the workload, tensor amax -> NVFP4 quantize -> block-scaled
GEMM (the prefill phase), then the BF16 decode linear at M = 1 on the same
weight handles (the phase switch).

Reported metric: prefill linear TFLOP/s including activation quantization,
2*M*N*K summed over projections / (t_amax + t_quant + t_gemm), plus its
fraction of the dense FP4 peak.  Timed with CUDA events on the launching
stream, L2 flushed (256 MiB write) between steps outside the timed intervals.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
  python bench.py --impl reference ...   (the CPU oracle, bounded sample)

Multi-GPU: one process per GPU (torchrun), independent replicas (the layer
needs no exchange); value = work of all ranks / max-over-ranks time.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from nvfp4_quantized_prefill_b200 import workloads  # noqa: E402

FP4_OVER_BF16 = 4.0   # nominal dense ratio (9 PF fp4 / 2.25 PF bf16)
METRIC = "prefill linear TFLOPS (NVFP4 incl. act-quant) and % of B200 dense FP4 peak"
CLOCK_QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
               "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
               "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": d["hbm_gbs"], "bf16": d["bf16_tflops"],
                "bf16_sustained": d.get("bf16_tflops_sustained", d["bf16_tflops"]),
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16": 1590.0, "bf16_sustained": 1400.0, "source": "fallback"}


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples during the timed region."""

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = os.path.join(ROOT, "gpurun_out", f"clocks_rank{index}.csv")

    def __enter__(self):
        try:
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
            self.fh = open(self.path, "w")
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
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].strip().replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].strip().replace(".", "").isdigit()]
        reasons = set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            for i, n in enumerate(names):
                if len(r) > 5 + i and "Active" in r[5 + i] and "Not" not in r[5 + i]:
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": sorted(reasons),
                "samples": len(rows)}


def dist_setup(n_gpus: int):
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


def max_over_ranks(v: float, world: int) -> float:
    if world == 1:
        return v
    t = torch.tensor([v], dtype=torch.float64, device="cuda")
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(v: float, world: int) -> float:
    if world == 1:
        return v
    t = torch.tensor([v], dtype=torch.float64, device="cuda")
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.SUM)
    return float(t.item())


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

def run_gpu(args, wl, world, rank):
    from nvfp4_quantized_prefill_b200 import binding as mq
    mq.lib()
    dev = torch.device("cuda", torch.cuda.current_device())
    stream = torch.cuda.current_stream()
    pk = peaks()

    ws_cpu = workloads.layer_weights(wl)
    xs_cpu = [workloads.layer_activation(wl, w.shape[1], i) for i, w in enumerate(ws_cpu)]
    Ws = [mq.Weight(w.to(dev)) for w in ws_cpu]
    xs = [x.to(dev) for x in xs_cpu]
    M = wl.M
    bufs = []
    for W in Ws:
        K = W.K
        bufs.append(dict(
            codes=torch.empty(M, K // 2, dtype=torch.uint8, device=dev),
            sf=torch.empty(mq.mq_sf_bytes(M, K), dtype=torch.uint8, device=dev),
            s=torch.empty(1, dtype=torch.float32, device=dev),
            part=torch.empty(mq.MQ_AMAX_PARTIALS_MAX, dtype=torch.float32, device=dev),
            y=torch.empty(M, W.N, dtype=torch.bfloat16, device=dev),
            yd=torch.empty(1, W.N, dtype=torch.bfloat16, device=dev)))
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    flops = sum(2.0 * M * W.N * W.K for W in Ws)
    gemm_flops = flops
    decode_bytes = sum(2.0 * W.N * W.K + 2.0 * W.K + 2.0 * W.N for W in Ws)
    launches_per_step = 3 * len(Ws) + len(Ws)

    def step(evs):
        """evs: list of events, 4 per projection (start, after amax, after
        quantize, after gemm) + 2 for decode (start, end)."""
        i = 0
        for W, x, b in zip(Ws, xs, bufs):
            evs[i].record(stream)
            n = mq.mq_tensor_amax(x, M, W.K, W.K, b["part"], stream)
            evs[i + 1].record(stream)
            mq.mq_quantize_nvfp4(x, M, W.K, W.K, b["codes"], b["sf"], b["s"],
                                 amax_partials=b["part"], n_partials=n, stream=stream)
            evs[i + 2].record(stream)
            mq.mq_gemm_nvfp4(b["codes"], b["sf"], b["s"], M, W.handle, b["y"], W.N, stream)
            evs[i + 3].record(stream)
            i += 4
        evs[i].record(stream)
        for W, x, b in zip(Ws, xs, bufs):
            mq.mq_decode_linear_bf16(W.handle, x[:1], 1, b["yd"], stream)
        evs[i + 1].record(stream)

    nev = 4 * len(Ws) + 2
    for _ in range(args.warmup):
        flush.zero_()
        step([torch.cuda.Event(enable_timing=True) for _ in range(nev)])
    torch.cuda.synchronize()
    st = mq.mq_check(stream)
    if st != 0:
        raise RuntimeError(f"device error during warm-up: {mq.STATUS.get(st)}")

    all_evs = [[torch.cuda.Event(enable_timing=True) for _ in range(nev)] for _ in range(args.steps)]
    clocks = ClockSampler(int(os.environ.get("LOCAL_RANK", "0")))
    barrier(world)
    torch.cuda.synchronize()
    with clocks:
        time.sleep(0.3)
        for k in range(args.steps):
            flush.zero_()
            step(all_evs[k])
        torch.cuda.synchronize()
    barrier(world)
    st = mq.mq_check(stream)
    if st != 0:
        raise RuntimeError(f"device error during timing: {mq.STATUS.get(st)}")

    t_amax = t_quant = t_gemm = t_dec = t_step = 0.0
    for evs in all_evs:
        i = 0
        for _ in Ws:
            t_amax += evs[i].elapsed_time(evs[i + 1])
            t_quant += evs[i + 1].elapsed_time(evs[i + 2])
            t_gemm += evs[i + 2].elapsed_time(evs[i + 3])
            i += 4
        t_dec += evs[i].elapsed_time(evs[i + 1])
        t_step += evs[0].elapsed_time(evs[i + 1])
    K_ = args.steps
    t_prefill_ms = (t_amax + t_quant + t_gemm) / K_
    t_prefill_max = max_over_ranks(t_prefill_ms, world)
    t_step_max = max_over_ranks(t_step / K_, world)
    total_flops = sum_over_ranks(flops, world)
    value = total_flops / (t_prefill_max * 1e-3) / 1e12
    gemm_ms = t_gemm / K_
    fp4_peak = pk["bf16"] * FP4_OVER_BF16
    achieved = gemm_flops / (gemm_ms * 1e-3) / 1e12

    # ---- end to end through the public call: pinned host X -> device, prefill
    # linear (amax + quantize + GEMM inside), result back to pinned host memory
    xs_h = [x.pin_memory() for x in xs_cpu]
    ys_h = [torch.empty(M, W.N, dtype=torch.bfloat16).pin_memory() for W in Ws]
    xs_d = [torch.empty_like(x) for x in xs]
    wsb = max(mq.mq_workspace_bytes(M, W.K) for W in Ws)
    wsp = torch.empty(wsb, dtype=torch.uint8, device=dev)

    def e2e_step():
        for W, xh, xd, b, yh in zip(Ws, xs_h, xs_d, bufs, ys_h):
            xd.copy_(xh, non_blocking=True)
            mq.mq_prefill_linear_nvfp4(W.handle, xd, M, b["y"], wsp, wsb, stream)
            yh.copy_(b["y"], non_blocking=True)

    for _ in range(2):
        e2e_step()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e2e_steps = max(2, min(args.steps, 10))
    barrier(world)
    torch.cuda.synchronize()
    e0.record(stream)
    for _ in range(e2e_steps):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / e2e_steps, world)
    h2d = sum(x.numel() * 2 for x in xs_cpu)
    d2h = sum(M * W.N * 2 for W in Ws)

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
        "dtype": "nvfp4 (e2m1 + e4m3 block scales) x nvfp4 -> fp32 acc -> bf16",
        "data": "synthetic (seeded, Llama-3-8B-shaped projections; random-init weights)",
        "config": {
            "workload": wl.name,
            "tokens": M,
            "linears": [{"name": l.name, "N": l.N, "K": l.K} for l in wl.linears],
            "activations": wl.act,
            "seed": wl.seed,
            "step": "per projection: tensor amax -> NVFP4 quantize -> block-scaled GEMM; "
                    "then BF16 decode M=1 on the same weights",
            "l2": "flushed between steps (256 MiB write, outside timed intervals)",
            "parallelism": f"replicas x{world} (no exchange)",
        },
        "prefill_ms": round(t_prefill_max, 4),
        "breakdown_ms": {"amax": round(t_amax / K_, 4), "quantize": round(t_quant / K_, 4),
                         "gemm": round(gemm_ms, 4), "decode_m1": round(t_dec / K_, 4)},
        "tokens_per_s": round(world * M / (t_prefill_max * 1e-3), 1),
        "fp4_peak_frac": round(value / fp4_peak, 4),
        "gemm_only_tflops": round(achieved, 2),
        "decode_gbs": round(decode_bytes / (t_dec / K_ * 1e-3) / 1e9, 1),
        "roofline": {
            "kernel": "gemm_nvf4_kernel (tcgen05 mxf4nvf4 block16)",
            "bound": "tensor",
            "achieved": round(achieved, 2),
            "peak": round(fp4_peak, 1),
            "peak_source": f"{pk['source']} bf16 burst {pk['bf16']} TF/s x {FP4_OVER_BF16} "
                           "(nominal dense fp4/bf16 ratio)",
            "unit": "TFLOP/s",
            "frac": round(achieved / fp4_peak, 4),
            "traffic": None,
        },
        "e2e": {"value": round(total_flops / (e2e_ms * 1e-3) / 1e12, 3),
                "unit": "TFLOP/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "path": "mq_prefill_linear_nvfp4 with pinned-host X in / Y out"},
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clk,
    }
    for W in Ws:
        W.free()
    return out, xs_cpu, ws_cpu


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
    args = ap.parse_args()
    wl = workloads.WORKLOADS[args.workload]

    if args.impl == "reference":
        world = int(os.environ.get("WORLD_SIZE", "1"))
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
            "scaling": "weak", "vs_baseline": None, "dtype": "int64 exact / fp64",
            "data": "synthetic", "config": {"workload": wl.name, "tokens": wl.M},
            "cpu_baseline": {"value": v, "unit": "TFLOP/s", "cores": oracle.threads_used(),
                             "kind": "oracle",
                             "sample": f"{args.cpu_rows} activation rows per projection "
                                       "(full-tensor amax, row quantize, exact GEMM)"},
            "e2e": {"value": v, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}))
        return

    world, rank, local = dist_setup(args.gpus)
    out, xs_cpu, ws_cpu = run_gpu(args, wl, world, rank)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import oracle
        fl, t = oracle_sample(xs_cpu, oracle_prepare(ws_cpu), args.cpu_rows)
        out["cpu_baseline"] = {"value": fl / t / 1e12, "unit": "TFLOP/s",
                               "cores": oracle.threads_used(), "kind": "oracle",
                               "sample": f"{args.cpu_rows} activation rows per projection "
                                         "(full-tensor amax, row quantize, exact GEMM); "
                                         f"{t:.1f} s"}
    if rank == 0:
        print(json.dumps(out))
    if world > 1:
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
