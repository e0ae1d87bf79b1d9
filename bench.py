"""Benchmark of the NVFP4 attention hot path on B200.

A step is one pass of the path over one batch: the NVFP4 pre-pass of Q, K
(smoothed) and V, then the FP4 attention forward.  Default workload: LLM
prefill B2 H16 N4096 D128 causal, max-scaling (seeded synthetic inputs).
Metric: FP4 attention TOPS = 4*B*H*N^2*D / t (causal halved), t = step time.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload llm]
                  [--mode max|search] [--impl ours|reference]

With N > 1 (torchrun) every rank runs an independent replica (the path has no
cross-GPU exchange), timing is the max over ranks, value is the job total.
--impl reference times the CPU oracle on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import bit_quantized_attention_channel_b200 as sa  # noqa: E402
from bit_quantized_attention_channel_b200 import workloads as wl  # noqa: E402

METRIC = "FP4 attention TOPS (4*B*H*N^2*d, causal halved)"
L2_FLUSH_BYTES = 256 << 20


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            m = json.load(f)
        return m["hbm_gbs"], m["bf16_tflops"], "measured"
    except Exception:
        return 6650.0, 1590.0, "fallback"


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled during the timed region."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "20"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except Exception:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *a):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], 0.0, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            p = [x.strip() for x in ln.split(",")]
            if len(p) < 7:
                continue
            try:
                sm.append(float(p[0]))
                mx = max(mx, float(p[1]))
            except ValueError:
                continue
            for n, v in zip(names, p[3:7]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx or None,
                "reasons": sorted(reasons), "samples": len(sm)}


def make_step(w, mode, q, k, v, stream):
    """Returns step() running the whole path on device-resident inputs, and
    the buffers it writes into (allocated once)."""
    st = {}

    def step(attn_events=None):
        qq = sa.sa_quant_nvfp4(q, "q", mode=mode, out=st.get("q"), stream=stream)
        kq = sa.sa_quant_nvfp4(k, "k", mode=mode, out=st.get("k"), stream=stream)
        vq = sa.sa_quant_nvfp4(v, "v", mode=mode, out=st.get("v"), stream=stream)
        st["q"], st["k"], st["v"] = qq, kq, vq
        if attn_events:
            attn_events[0].record(stream)
        out = sa.sa_attn_fwd(qq, kq, vq, w.causal, out=st.get("o"), stream=stream)
        if attn_events:
            attn_events[1].record(stream)
        st["o"] = out
        return out

    return step


def kernels_per_step(mode):
    # q: amax + quant; k: stats + final + quant; v: amax + quant; attention: 1
    return 2 + 3 + 2 + 1


def cpu_baseline(w, mode, budget_s=20.0):
    """Oracle (plain C, OpenMP) on a bounded sample: full pre-pass of Q, K, V
    plus attention for whole query tiles of every head, timed separately;
    throughput = sampled FLOPs / (attention time + pre-pass time scaled to the
    sampled share)."""
    import numpy as np

    import oracle as orc

    q, k, v = wl.prefill_inputs(w)
    ss = mode == "search"
    t0 = time.perf_counter()
    qo, ko, vo = orc.quantize(q, "q", search=ss), orc.quantize(k, "k", search=ss), orc.quantize(v, "v", search=ss)
    t_quant = time.perf_counter() - t0
    B, H, N, D = w.B, w.H, w.N, w.D
    T = (N + 127) // 128
    qd, kd, vd = qo.dequant(), ko.dequant(), vo.dequant()
    rows_done, flops, t_attn = [], 0.0, 0.0
    order = [T - 1, 0, T // 2, T // 4, 3 * T // 4] + list(range(T))
    seen = set()
    for t in order:
        if t in seen:
            continue
        seen.add(t)
        rows = np.arange(t * 128, min(N, t * 128 + 128), dtype=np.int32)
        t1 = time.perf_counter()
        orc.attn_f64(qd, kd, vd, w.causal, 1 / math.sqrt(D), True, rows=rows)
        t_attn += time.perf_counter() - t1
        keys = (rows + 1).sum() if w.causal else len(rows) * N
        flops += 4.0 * B * H * keys * D
        rows_done.append(t)
        if t_attn + t_quant > budget_s:
            break
    share = flops / w.flops()
    t_total = t_attn + t_quant * share
    return {"value": flops / t_total / 1e12, "unit": "TOPS", "cores": orc.num_threads(), "kind": "oracle",
            "sample": f"pre-pass of full Q,K,V ({t_quant:.1f} s, scaled by {share:.4f}) + FP64 attention of "
                      f"{len(rows_done)}/{T} query tiles of all {B * H} heads ({t_attn:.1f} s)"}


def run_reference(args, w, rank, world):
    if rank != 0:
        return
    cb = cpu_baseline(w, args.mode, budget_s=max(5.0, 60.0 / max(1, args.steps + args.warmup)))
    line = {"metric": METRIC, "value": cb["value"], "unit": "TOPS", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": w.flops() / (cb["value"] * 1e12) * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
            "config": config_of(w, args.mode), "cpu_baseline": cb,
            "e2e": {"value": cb["value"], "unit": "TOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def config_of(w, mode):
    return {"workload": w.description, "B": w.B, "H": w.H, "N": w.N, "D": w.D, "causal": w.causal,
            "scale_mode": mode, "l2": "flushed between steps (256 MiB write)", "parallelism": "replicas"}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="llm")
    ap.add_argument("--mode", default="max", choices=["max", "search"])
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    w = wl.WORKLOADS[args.workload]

    if args.impl == "reference":
        run_reference(args, w, rank, world)
        return

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    pg = None
    if world > 1:
        import datetime

        import torch.distributed as dist

        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
        pg = dist

    q, k, v = (t.to(dev) for t in wl.prefill_inputs(w))
    stream = torch.cuda.current_stream(dev)
    step = make_step(w, args.mode, q, k, v, stream)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    assert sa.sa_device_status() == 0

    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    aevs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    if pg:
        pg.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        t_wall = time.perf_counter()
        for i in range(args.steps):
            flush.fill_(i & 0xFF)  # evict L2 between steps (outside the step events)
            evs[i][0].record(stream)
            step(aevs[i])
            evs[i][1].record(stream)
        torch.cuda.synchronize()
        t_wall = time.perf_counter() - t_wall
    if pg:
        pg.barrier()
    st = sa.sa_device_status()
    assert st == 0, sa.STATUS[st]
    ms = sum(a.elapsed_time(b) for a, b in evs) / args.steps
    ms_attn = sum(a.elapsed_time(b) for a, b in aevs) / args.steps
    if pg:
        t = torch.tensor([ms, ms_attn], device=dev)
        pg.all_reduce(t, op=pg.ReduceOp.MAX)
        ms, ms_attn = t.tolist()

    # end to end through the C ABI from pinned host buffers
    hq, hk, hv = (t.cpu().pin_memory() for t in (q, k, v))
    hout = torch.empty(w.B, w.H, w.N, w.D, dtype=torch.float32).pin_memory()
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    step_e2e = make_step(w, args.mode, dq, dk, dv, stream)
    e2e_ms = []
    for i in range(args.warmup + args.steps):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        flush.fill_(i & 0xFF)
        a.record(stream)
        dq.copy_(hq, non_blocking=True)
        dk.copy_(hk, non_blocking=True)
        dv.copy_(hv, non_blocking=True)
        out = step_e2e()
        hout.copy_(out, non_blocking=True)
        b.record(stream)
        b.synchronize()
        if i >= args.warmup:
            e2e_ms.append(a.elapsed_time(b))
    e2e = statistics.mean(e2e_ms)
    if pg:
        t = torch.tensor([e2e], device=dev)
        pg.all_reduce(t, op=pg.ReduceOp.MAX)
        e2e = t.item()

    if rank == 0:
        hbm, bf16, src = peaks()
        fp4_peak = bf16 * 4.0  # dense FP4 = 4x dense bf16 (nominal ratio 9 / 2.25)
        flops = w.flops()
        achieved = flops / (ms_attn * 1e-3) / 1e12
        line = {
            "metric": METRIC, "value": world * flops / (ms * 1e-3) / 1e12, "unit": "TOPS", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "nvfp4", "data": "synthetic",
            "config": config_of(w, args.mode),
            "roofline": {"bound": "tensor", "kernel": "attn_fwd_kernel<128>", "achieved": achieved,
                         "peak": fp4_peak, "unit": "TFLOP/s", "frac": achieved / fp4_peak,
                         "peak_source": f"{src} bf16 {bf16} TFLOP/s x 4 (FP4/bf16 nominal ratio)",
                         "traffic": None, "ms_per_launch": ms_attn},
            "e2e": {"value": world * flops / (e2e * 1e-3) / 1e12, "unit": "TOPS",
                    "h2d_bytes_per_step": 3 * q.numel() * 2, "d2h_bytes_per_step": hout.numel() * 4},
            "gpu_launches": kernels_per_step(args.mode) * args.steps,
            "clocks": clk.summary(),
            "wall_s": t_wall,
        }
        if world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline(w, args.mode)
        print(json.dumps(line), flush=True)
    if pg:
        pg.barrier()
        pg.destroy_process_group()


if __name__ == "__main__":
    main()
