"""Benchmark of the NVFP4 attention hot path on B200.

A step is one pass of the path over one batch of seeded synthetic input: the
NVFP4 pre-pass of Q, K (smoothed) and V (plus the bf16-block selector when the
workload has one), then the attention forward (or, for decode, the split-KV
decode over a cache quantised once before timing).
Metric: FP4 attention TOPS = 4*B*H*N^2*D / t (causal halved), t = step time.

The headline workload is the long-context mixed-precision prefill (B1 H32
N65536 D128 causal, top 5% of blocks in bf16), the largest configuration that
fits one GPU; the LLM prefill (max-scaling, ScaleSearch on Q, K and V, and
ScaleSearch on Q, K, V and P, and incoherence processing of Q and K before
max-scaling), the video-shaped
prefill and the NVFP4-KV decode (plain, and with the cache's first and last
128-key tile at full precision) are measured in the same run and nested in the
line under "workloads".

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME [--only]]
                  [--mode max|search|psearch|ip|sink] [--impl ours|reference]

With N > 1 (torchrun) every rank runs an independent replica (the path has no
cross-GPU exchange), timing is the max over ranks, value is the job total.
--impl reference times the CPU oracle on bounded samples of the same workload.
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


# DRAM bytes per launch of the dominant kernel, from one ncu capture
# (dram__bytes_read.sum + dram__bytes_write.sum) on a batch slice of the same
# workload, scaled by the units of the full launch.  Keyed by workload, scale
# mode and kernel; any other key (or a kernel changed since its capture)
# reports null.
MEASURED_TRAFFIC = {
    # decode_kernel<128>, batch-4 slice x 8 (154.8 MB read + write per slice launch)
    ("decode", "max", "decode_kernel<128> + combine"): 1238.2e6,
    # attn_fwd_pp_kernel<128>, video 3-head slice x 8 (25.73 MB per slice launch)
    ("video", "search", "attn_fwd_pp_kernel<128>"): 205.8e6,
    # attn_fwd_pp_kernel<128>, batch-1 slice x 2 (14.36 MB per slice launch)
    ("llm", "max", "attn_fwd_pp_kernel<128>"): 28.73e6,
    ("llm", "search", "attn_fwd_pp_kernel<128>"): 28.73e6,
    # attn_fwd_pp_kernel<128, mixed>, 4-head slice x 8 (836.6 MB per slice launch)
    ("longctx", "max", "attn_fwd_pp_kernel<128, mixed>"): 6692.4e6,
}


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            m = json.load(f)
        return m["hbm_gbs"], m["bf16_tflops"], "measured"
    except Exception:
        return 6650.0, 1590.0, "fallback"


class ClockSampler:
    """SM clock and clock-event (throttle) reasons sampled during the timed
    region: an NVML polling thread (about one sample per millisecond), else
    nvidia-smi at its fastest rate."""

    REASONS = (("hw_slowdown", 0x8), ("hw_thermal_slowdown", 0x40), ("sw_thermal_slowdown", 0x20),
               ("sw_power_cap", 0x4))

    def __init__(self, cuda_index):
        self.cuda_index = cuda_index
        self.samples = []  # (sm_mhz, reason bits)
        self.max_mhz = None
        self.stop = threading.Event()
        self.ready = threading.Event()
        self.thread = None
        self.source = None

    def _handle(self, nv):
        try:
            uuid = str(torch.cuda.get_device_properties(self.cuda_index).uuid)
            return nv.nvmlDeviceGetHandleByUUID(uuid if uuid.startswith("GPU-") else "GPU-" + uuid)
        except Exception:
            return nv.nvmlDeviceGetHandleByIndex(self.cuda_index)

    def _poll_nvml(self, nv, h):
        get_reasons = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            nv.nvmlDeviceGetCurrentClocksThrottleReasons
        while not self.stop.is_set():
            try:
                self.samples.append((float(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)), int(get_reasons(h))))
            except Exception:
                pass
            self.ready.set()
            time.sleep(0.001)

    def _poll_smi(self):
        q = "clocks.sm,clocks.max.sm," + ",".join("clocks_event_reasons." + n for n, _ in self.REASONS)
        proc = subprocess.Popen(["nvidia-smi", "-i", str(self.cuda_index), f"--query-gpu={q}",
                                 "--format=csv,noheader,nounits", "-lms", "10"], stdout=subprocess.PIPE,
                                stderr=subprocess.DEVNULL, text=True)
        self.ready.set()
        for line in proc.stdout:
            p = [x.strip() for x in line.split(",")]
            if self.stop.is_set():
                break
            try:
                bits = sum(bit for (_, bit), v in zip(self.REASONS, p[2:]) if v.lower() == "active")
                self.samples.append((float(p[0]), bits))
                self.max_mhz = float(p[1])
            except (ValueError, IndexError):
                continue
        proc.terminate()

    def __enter__(self):
        try:
            import pynvml as nv

            nv.nvmlInit()
            h = self._handle(nv)
            self.max_mhz = float(nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM))
            self.thread = threading.Thread(target=self._poll_nvml, args=(nv, h), daemon=True)
            self.source = "nvml"
        except Exception:
            self.thread = threading.Thread(target=self._poll_smi, daemon=True)
            self.source = "nvidia-smi"
        self.thread.start()
        self.ready.wait(timeout=5)
        self.samples.clear()  # keep only samples taken inside the region
        return self

    def __exit__(self, *a):
        self.stop.set()
        self.thread.join(timeout=5)

    def summary(self):
        sm = [c for c, _ in self.samples]
        bits = 0
        for _, b in self.samples:
            bits |= b
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": self.max_mhz,
                "reasons": [n for n, bit in self.REASONS if bits & bit], "samples": len(sm), "source": self.source}


class Path:
    """The hot path of one workload as two device-side phases (pre-pass,
    attention), each captured once in a CUDA graph and replayed per step.
    Inputs stay resident; outputs are written into the same buffers."""

    def __init__(self, w, mode, q, k, v):
        self.w, self.mode, self.q, self.k, self.v = w, mode, q, k, v
        self.st = {}

    def prepass(self):
        w, st = self.w, self.st
        if w.kind == "decode":
            return  # the KV cache is quantised once, before timing (it is a cache)
        if self.mode == "ip":  # Q and K through incoherence processing, V as usual
            st["q"], st["k"], st["r"] = sa.sa_quant_nvfp4_ip(self.q, self.k, st["signs"])
            st["v"] = sa.sa_quant_nvfp4(self.v, "v", out=st.get("v"))
            return
        # Q, K (smoothed) and V in two launches: statistics, then quantisation
        st["qkv"] = sa.sa_quant_nvfp4_qkv(self.q, self.k, self.v, smooth=True, mode=prepass_mode(self.mode),
                                          out=st.get("qkv"))
        st["q"], st["k"], st["v"] = st["qkv"]
        if w.thrift_bp:
            st["mask"], _ = sa.sa_thrift_select(self.q, self.k, w.causal, w.thrift_bp)

    def attention(self):
        w, st = self.w, self.st
        if w.kind == "decode":
            st["o"] = sa.sa_attn_decode_kvfp4(self.q, st["kc"], st["vc"], out=st.get("o"),
                                              sink_tiles=sink_tiles(self.mode), k_sink=st.get("ks"),
                                              v_sink=st.get("vs"))
        elif w.thrift_bp:
            st["o"] = sa.sa_attn_fwd(st["q"], st["k"], st["v"], w.causal, mask=st["mask"], q_bf16=self.q,
                                     k_bf16=self.k, v_bf16=self.v, out=st.get("o"))
        else:
            st["o"] = sa.sa_attn_fwd(st["q"], st["k"], st["v"], w.causal, out=st.get("o"), p_mode=p_mode(self.mode))
        return st["o"]

    def setup(self):
        if self.mode == "ip":
            self.st["signs"] = torch.from_numpy(ip_signs(self.w.D)).to(self.q.device)
        if self.w.kind == "decode":
            self.st["kc"] = sa.sa_quant_nvfp4(self.k, "k")
            self.st["vc"] = sa.sa_quant_nvfp4(self.v, "v")
            if any(sink_tiles(self.mode)):  # the cache's full-precision first and last tiles
                self.st["ks"] = sa.sink_tiles_of(self.k, *sink_tiles(self.mode))
                self.st["vs"] = sa.sink_tiles_of(self.v, *sink_tiles(self.mode))

    def capture(self):
        """Warm up eagerly, then capture both phases as CUDA graphs."""
        self.setup()
        for _ in range(2):
            self.prepass()
            self.attention()
        torch.cuda.synchronize()
        self.g_pre, self.g_attn = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.g_pre):
            self.prepass()
        with torch.cuda.graph(self.g_attn):
            self.attention()
        torch.cuda.synchronize()

    def step(self, attn_events=None):
        self.g_pre.replay()
        if attn_events:
            attn_events[0].record()
        self.g_attn.replay()
        if attn_events:
            attn_events[1].record()
        return self.st["o"]


def prepass_mode(mode):
    """Block rule of the pre-pass: "search" and "psearch" use ScaleSearch."""
    return "search" if mode in ("search", "psearch") else "max"


def p_mode(mode):
    """Block rule of the requantised P: ScaleSearch only in mode "psearch"
    (Q, K, V and P all ScaleSearch)."""
    return "search" if mode == "psearch" else "max"


def ip_signs(D, seed=7):
    """Random signs of the incoherence rotation (mode "ip")."""
    import numpy as np

    return np.where(np.random.default_rng(seed).random(D) < 0.5, -1, 1).astype(np.int8)


def sink_tiles(mode):
    """Decode mode "sink": the first and the last 128-key tile of the cache
    at full precision (the attention-sink-aware mixed-precision cache)."""
    return (1, 1) if mode == "sink" else (0, 0)


def kernels_per_step(w, mode="max"):
    if w.kind == "decode":
        return 3  # q amax, split kernel, combine
    if mode == "ip":
        return 6 + 2 + 1  # K mean (2) + rotation sums, r, amax, quantisation; V amax + quantisation; attention
    n = 2 + 1  # fused pre-pass: statistics + quantisation of Q, K, V; attention
    if w.thrift_bp:
        n += 3  # pool, score, top-k
    return n


def flops_of(w):
    if w.kind == "decode":
        return 4.0 * w.B * w.H * w.N * w.D
    return w.flops()


def hbm_bytes_decode(w, mode="max"):
    """Algorithmic bytes of one decode: K and V codes + scales, q, out; with
    full-precision tiles, their bf16 K and V in place of their NVFP4 bytes."""
    nsink = 128 * sum(sink_tiles(mode))
    kv = 2 * w.B * w.Hkv * ((w.N - nsink) * w.D * 0.5625 + nsink * w.D * 2)
    return int(kv) + w.B * w.H * w.D * (2 + 4)


def prepass_bytes(w):
    """Algorithmic bytes of one pre-pass call: one bf16 read of Q, K and V
    plus their NVFP4 codes and scales written (2 + 0.5 + 0.0625 B per element)."""
    return 3 * w.B * w.H * w.N * w.D * 2.5625


def attn_algorithmic_bytes(w):
    """HBM bytes one attention launch must move: NVFP4 Q, K, V once (codes +
    scales) and the FP32 output (plus, with bf16 blocks, nothing more is
    counted: their raw tiles are re-reads of inputs already counted)."""
    el = w.B * w.H * w.N * w.D
    return 3 * el * 0.5625 + el * 4


# ---------------------------------------------------------------- CPU oracle
def cpu_sample_step(w, mode, q, k, v, tiles):
    """One bounded sample of the hot path on the CPU oracle over the
    single-head inputs (q, k, v): pre-pass of that head, the selector when the
    workload has bf16 blocks, then FP64 attention of the given query tiles.
    Returns (sampled FLOPs, seconds charged to them, wall seconds)."""
    import numpy as np

    import oracle as orc

    ss = prepass_mode(mode) == "search"
    N, D = w.N, w.D
    t0 = time.perf_counter()
    if mode == "ip":
        qi, ki, _ = orc.incoherence(q, k, ip_signs(D), orc.quantize(k, "k").k_mean)
        qo, ko, vo = orc.quantize_rows_f32(qi), orc.quantize_rows_f32(ki), orc.quantize(v, "v")
    else:
        qo, ko, vo = (orc.quantize(q, "q", search=ss), orc.quantize(k, "k", search=ss),
                      orc.quantize(v, "v", search=ss))
    mask = None
    if w.thrift_bp:
        mask, _ = orc.thrift_select(q, k, w.causal, w.thrift_bp)
    t_pre = time.perf_counter() - t0
    rows = np.concatenate([np.arange(t * 128, min(N, t * 128 + 128), dtype=np.int32) for t in tiles])
    t1 = time.perf_counter()
    if mask is not None:
        orc.attention(qo, ko, vo, w.causal, rows=rows, mask=mask, q_bf16=q, k_bf16=k, v_bf16=v)
    else:
        orc.attention(qo, ko, vo, w.causal, rows=rows, p_search=p_mode(mode) == "search")
    t_attn = time.perf_counter() - t1
    keys = float((rows + 1).sum()) if w.causal else float(len(rows)) * N
    flops = 4.0 * keys * D
    head_flops = w.flops() / (w.B * w.H)
    return flops, t_attn + t_pre * flops / head_flops, t_pre + t_attn


def cpu_sample_tiles(w, step, ntiles=8):
    """Query tiles of sample `step`: ntiles spread over the head, rotating."""
    T = (w.N + 127) // 128
    return sorted({(step * 7 + i * max(1, T // ntiles)) % T for i in range(ntiles)})


def cpu_baseline(w, mode, budget_s=20.0):
    """Oracle (plain C, OpenMP) timed on bounded samples of the workload: each
    sample is one head's pre-pass (plus selector) and FP64 attention of 8 of
    its query tiles; throughput = sampled FLOPs / (attention time + the share
    of the head's pre-pass those FLOPs account for)."""
    import oracle as orc

    if w.kind == "decode":
        return None
    q, k, v = wl.prefill_inputs(w, B=1, H=1)
    flops = secs = 0.0
    n = 0
    t_start = time.perf_counter()
    while time.perf_counter() - t_start < budget_s or n == 0:
        f, s, _ = cpu_sample_step(w, mode, q, k, v, cpu_sample_tiles(w, n))
        flops += f
        secs += s
        n += 1
    return {"value": flops / secs / 1e12, "unit": "TOPS", "cores": orc.num_threads(), "kind": "oracle",
            "sample": f"{n} samples of one head (B1 H1 N{w.N} D{w.D}, same recipe): its pre-pass"
                      f"{' and selector' if w.thrift_bp else ''} plus FP64 attention of 8 query tiles each; "
                      f"pre-pass time charged in proportion to the sampled FLOPs"}


def max_over_ranks(values, pg, device):
    """Element-wise max over all ranks of a list of floats (per-rank device
    timings); the values themselves on a single rank."""
    if pg is None:
        return [float(v) for v in values]
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    pg.all_reduce(t, op=pg.ReduceOp.MAX)
    return t.tolist()


def whole_job_tops(world, flops_per_rank, ms_max):
    """Weak scaling: every rank runs the full workload, so the job's work is
    world x the per-rank FLOPs, over the slowest rank's time."""
    return world * flops_per_rank / (ms_max * 1e-3) / 1e12


def run_reference(args, w, rank, world):
    """The oracle as the reference arm: W untimed and K timed steps, each one
    bounded sample of the workload on the host cores."""
    if rank != 0:
        return
    import oracle as orc

    if w.kind == "decode":
        print(json.dumps({"impl": "reference", "unavailable": "the decode workload has no CPU sample step"}))
        return
    q, k, v = wl.prefill_inputs(w, B=1, H=1)
    for i in range(args.warmup):
        cpu_sample_step(w, args.mode, q, k, v, cpu_sample_tiles(w, i))
    flops = charged = wall = 0.0
    for i in range(args.steps):
        f, s, wsec = cpu_sample_step(w, args.mode, q, k, v, cpu_sample_tiles(w, args.warmup + i))
        flops += f
        charged += s
        wall += wsec
    value = flops / charged / 1e12
    cb = {"value": value, "unit": "TOPS", "cores": orc.num_threads(), "kind": "oracle",
          "sample": f"each step: one head (B1 H1 N{w.N} D{w.D}) pre-pass{' + selector' if w.thrift_bp else ''} "
                    f"and FP64 attention of 8 query tiles; pre-pass charged in proportion to the sampled FLOPs"}
    line = {"metric": METRIC, "value": value, "unit": "TOPS", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": wall / args.steps * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
            "config": config_of(w, args.mode), "cpu_baseline": cb,
            "e2e": {"value": value, "unit": "TOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def traffic_of(w, mode, kname, args):
    """Measured DRAM bytes per launch for the full workload, else None."""
    if args.batch is not None or args.heads is not None:
        return None
    return MEASURED_TRAFFIC.get((w.name, mode, kname))


def config_of(w, mode):
    c = {"workload": w.description, "B": w.B, "H": w.H, "N": w.N, "D": w.D, "causal": w.causal,
         "scale_mode": prepass_mode(mode), "p_scale_mode": p_mode(mode),
         "incoherence_processing": mode == "ip", "l2": "flushed between steps (256 MiB write)", "parallelism": "replicas",
         "launch": "CUDA graphs (pre-pass graph + attention graph per step)"}
    if w.kind == "decode":
        c["Hkv"] = w.Hkv
        c["scale_mode"] = "max"
        c["sink_tiles"] = list(sink_tiles(mode))
    if w.thrift_bp:
        c["bf16_block_budget_bp"] = w.thrift_bp
    return c


def kernel_name(w, mode="max"):
    if w.kind == "decode":
        return "decode_kernel<128, sink> + combine" if any(sink_tiles(mode)) else "decode_kernel<128> + combine"
    if p_mode(mode) == "search":
        return "attn_fwd_pp_kernel<128, P ScaleSearch>"
    return "attn_fwd_pp_kernel<128, mixed>" if w.thrift_bp else "attn_fwd_pp_kernel<128>"


def measure(w, mode, args, dev, pg, world, flush, want_e2e=True):
    """Time one workload: W warm-up and K timed steps of the device-resident
    path (L2 flushed between steps), then the same steps end to end from
    pinned host memory.  Returns the fields of a bench line (rank 0 uses them)."""
    if w.kind == "decode":
        q, k, v = (t.to(dev) for t in wl.decode_inputs(w))
    else:
        q, k, v = (t.to(dev) for t in wl.prefill_inputs(w))
    path = Path(w, mode, q, k, v)
    path.capture()

    for _ in range(args.warmup):
        flush.fill_(1)
        path.step()
    torch.cuda.synchronize()
    st = sa.sa_device_status()
    assert st == 0, sa.STATUS[st]

    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    aevs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    if pg:
        pg.barrier()
    torch.cuda.synchronize()
    with ClockSampler(dev.index) as clk:
        t_wall = time.perf_counter()
        for i in range(args.steps):
            flush.fill_(i & 0xFF)  # evict L2 between steps (outside the step events)
            evs[i][0].record()
            path.step(aevs[i])
            evs[i][1].record()
        torch.cuda.synchronize()
        t_wall = time.perf_counter() - t_wall
    if pg:
        pg.barrier()
    st = sa.sa_device_status()
    assert st == 0, sa.STATUS[st]
    ms = sum(a.elapsed_time(b) for a, b in evs) / args.steps
    ms_attn = sum(a.elapsed_time(b) for a, b in aevs) / args.steps
    ms, ms_attn = max_over_ranks([ms, ms_attn], pg, dev)

    e2e = None
    if want_e2e:
        e2e = measure_e2e(w, mode, args, dev, pg, flush, path, q, k, v)

    hbm, bf16, src = peaks()
    fp4_peak = bf16 * 4.0  # dense FP4 = 4x dense bf16 (nominal ratio 9 / 2.25)
    flops = flops_of(w)
    kname = kernel_name(w, mode)
    if w.kind == "decode":
        gbs = hbm_bytes_decode(w, mode) / (ms_attn * 1e-3) / 1e9
        roof = {"bound": "hbm", "kernel": kname, "achieved": gbs, "peak": hbm, "unit": "GB/s", "frac": gbs / hbm,
                "peak_source": f"{src} copy bandwidth", "traffic": traffic_of(w, mode, kname, args),
                "traffic_unit": "DRAM bytes per launch (ncu, batch slice scaled)", "ms_per_launch": ms_attn,
                "algorithmic_bytes": hbm_bytes_decode(w, mode)}
        value = whole_job_tops(world, flops, ms)
    else:
        achieved = flops / (ms_attn * 1e-3) / 1e12
        roof = {"bound": "tensor", "kernel": kname, "achieved": achieved, "peak": fp4_peak, "unit": "TFLOP/s",
                "frac": achieved / fp4_peak,
                "peak_source": f"{src} bf16 {bf16} TFLOP/s x 4 (FP4/bf16 nominal ratio)",
                "traffic": traffic_of(w, mode, kname, args),
                "traffic_unit": "DRAM bytes per launch (ncu, batch slice scaled; the FP32 output's write-back "
                                "that leaves L2 after the kernel ends is not in the kernel's count)",
                "algorithmic_bytes": attn_algorithmic_bytes(w), "ms_per_launch": ms_attn}
        value = whole_job_tops(world, flops, ms)
    out = {"value": value, "ms_per_step": ms, "config": config_of(w, mode), "roofline": roof,
           "gpu_launches": kernels_per_step(w, mode) * args.steps, "clocks": clk.summary(), "wall_s": t_wall}
    if w.kind != "decode":
        ms_pre = ms - ms_attn  # the pre-pass (and selector) share of the step, between the graphs
        pb = prepass_bytes(w)
        out["prepass"] = {"ms": ms_pre, "algorithmic_bytes": pb, "achieved_gbs": pb / (ms_pre * 1e-3) / 1e9,
                          "frac_of_hbm": pb / (ms_pre * 1e-3) / 1e9 / hbm,
                          "note": "step time minus attention time (includes the selector when the workload has "
                                  "bf16 blocks, and the L2 flush's write-backs)"}
    if e2e is not None:
        out["e2e"] = {"value": whole_job_tops(world, flops, e2e["ms"]), "unit": "TOPS",
                      "h2d_bytes_per_step": e2e["h2d"], "d2h_bytes_per_step": e2e["d2h"]}
    del path
    torch.cuda.empty_cache()
    return out


def measure_e2e(w, mode, args, dev, pg, flush, path, q, k, v):
    """End to end through the C ABI from pinned host buffers, as a stream of
    steps: every step copies its inputs in, runs the path and copies its
    output back.  Two buffer sets and three streams let step i + 1's
    host->device copy overlap step i's compute and device->host copy (PCIe
    is full duplex); the L2 flush runs on the compute stream before each step."""
    hq, hk, hv = (t.cpu().pin_memory() for t in (q, k, v))
    e2e_paths, houts = [], []
    for _ in range(2):
        pth = Path(w, mode, torch.empty_like(q), torch.empty_like(k), torch.empty_like(v))
        pth.st.update({kk: path.st[kk] for kk in ("kc", "vc", "ks", "vs", "signs") if kk in path.st})
        e2e_paths.append(pth)
        houts.append(torch.empty(path.st["o"].shape, dtype=torch.float32).pin_memory())

    def inputs_of(pth):
        if w.kind == "decode":
            return [(pth.q, hq)]
        return [(pth.q, hq), (pth.k, hk), (pth.v, hv)]

    s_in, s_cmp, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev_in, ev_cmp, ev_out = ([torch.cuda.Event() for _ in range(2)] for _ in range(3))

    def e2e_step(i):
        bsel = i % 2
        pth = e2e_paths[bsel]
        with torch.cuda.stream(s_in):
            if i >= 2:
                s_in.wait_event(ev_cmp[bsel])  # the previous step on these inputs has run
            for dst, src in inputs_of(pth):
                dst.copy_(src, non_blocking=True)
            ev_in[bsel].record(s_in)
        with torch.cuda.stream(s_cmp):
            s_cmp.wait_event(ev_in[bsel])
            if i >= 2:
                s_cmp.wait_event(ev_out[bsel])  # this output buffer has been copied out
            flush.fill_(i & 0xFF)
            pth.prepass()
            out = pth.attention()
            ev_cmp[bsel].record(s_cmp)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev_cmp[bsel])
            houts[bsel].copy_(out, non_blocking=True)
            ev_out[bsel].record(s_out)

    for i in range(args.warmup):
        e2e_step(i)
    torch.cuda.synchronize()
    e_start, e_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e_start.record(s_in)
    for i in range(args.warmup, args.warmup + args.steps):
        e2e_step(i)
    s_out.wait_stream(s_in)
    s_out.wait_stream(s_cmp)
    e_end.record(s_out)
    torch.cuda.synchronize()
    # the last streamed step computed the same inputs as the device-timed path
    last = houts[(args.warmup + args.steps - 1) % 2]
    if not torch.equal(last, path.st["o"].cpu()):
        raise RuntimeError("end-to-end stream produced a different output than the resident path")
    (ms,) = max_over_ranks([e_start.elapsed_time(e_end) / args.steps], pg, dev)
    h2d = sum(src.numel() * src.element_size() for _, src in inputs_of(e2e_paths[0]))
    return {"ms": ms, "h2d": h2d, "d2h": houts[0].numel() * 4}


# The headline workload: the largest configuration that fits one GPU (the
# long-context mixed prefill); the others are measured in the same run and
# nested in the line.
HEADLINE = ("longctx", "max")
OTHERS = [("llm", "max"), ("llm", "search"), ("llm", "psearch"), ("llm", "ip"), ("video", "search"),
          ("decode", "max"), ("decode", "sink")]


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=HEADLINE[0])
    ap.add_argument("--mode", default=None, choices=["max", "search", "psearch", "ip", "sink"])
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--only", action="store_true", help="measure the named workload alone (no nested workloads)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--batch", type=int, default=None,
                    help="override the workload's batch (a smaller slice for ncu captures; not a bench line)")
    ap.add_argument("--heads", type=int, default=None,
                    help="override the workload's head count (a smaller slice for ncu captures; not a bench line)")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    w = wl.WORKLOADS[args.workload]
    if args.mode is None:
        args.mode = "search" if w.scale_modes == ("search",) else "max"
    if args.batch is not None or args.heads is not None:
        import dataclasses

        B = w.B if args.batch is None else args.batch
        H = w.H if args.heads is None else args.heads
        if w.kind == "decode" and H % w.Hkv:
            raise SystemExit("--heads must be a multiple of the workload's kv heads")
        w = dataclasses.replace(w, B=B, H=H, description=w.description + f" (slice B{B} H{H})")
        args.only = True

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
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)

    head = measure(w, args.mode, args, dev, pg, world, flush, want_e2e=not args.no_e2e)
    nested = []
    if not args.only and args.workload == HEADLINE[0]:
        for name, mode in OTHERS:
            r = measure(wl.WORKLOADS[name], mode, args, dev, pg, world, flush, want_e2e=not args.no_e2e)
            if rank == 0 and world == 1 and not args.no_cpu_baseline and wl.WORKLOADS[name].kind != "decode":
                r["cpu_baseline"] = cpu_baseline(wl.WORKLOADS[name], mode, budget_s=6.0)
            nested.append(r)

    if rank == 0:
        line = {"metric": METRIC, "value": head["value"], "unit": "TOPS", "n_gpus": world, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": head["ms_per_step"], "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "nvfp4", "data": "synthetic",
                "config": head["config"], "roofline": head["roofline"]}
        for key in ("prepass", "e2e", "gpu_launches", "clocks", "wall_s"):
            if key in head:
                line[key] = head[key]
        line["gpu_launches"] = head["gpu_launches"] + sum(r["gpu_launches"] for r in nested)
        if world == 1 and not args.no_cpu_baseline and w.kind != "decode":
            line["cpu_baseline"] = cpu_baseline(w, args.mode)
        if nested:
            line["workloads"] = nested
        print(json.dumps(line), flush=True)
    if pg:
        pg.barrier()
        pg.destroy_process_group()


if __name__ == "__main__":
    main()
