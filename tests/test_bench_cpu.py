"""The bench's bookkeeping on CPU: the work and byte counts its roofline and
throughput figures divide by, the modes' meaning and the measured-traffic
lookup.  No GPU is touched."""
import argparse
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from bit_quantized_attention_channel_b200 import workloads as wl  # noqa: E402


def args(**kw):
    a = argparse.Namespace(batch=None, heads=None, mode="max")
    a.__dict__.update(kw)
    return a


def test_flops_count_causal_pairs_once():
    w = wl.WORKLOADS["llm"]  # B2 H16 N4096 D128 causal
    assert bench.flops_of(w) == 4.0 * 2 * 16 * 4096 * 4096 * 128 / 2
    v = wl.WORKLOADS["video"]  # non-causal
    assert bench.flops_of(v) == 4.0 * 1 * 24 * 32768 * 32768 * 128
    d = wl.WORKLOADS["decode"]  # one query token: 4 D FLOP per (head, key)
    assert bench.flops_of(d) == 4.0 * 32 * 32 * 32768 * 128


def test_decode_bytes_are_the_nvfp4_cache_plus_q_and_out():
    d = wl.WORKLOADS["decode"]
    kv = 2 * 32 * 8 * 32768 * 128 * (0.5 + 1 / 16)
    assert bench.hbm_bytes_decode(d) == int(kv) + 32 * 32 * 128 * (2 + 4)
    # with the first and last tile at full precision, those 256 keys move 2 B per element instead
    sink = 2 * 32 * 8 * ((32768 - 256) * 128 * 0.5625 + 256 * 128 * 2)
    assert bench.hbm_bytes_decode(d, "sink") == int(sink) + 32 * 32 * 128 * 6


def test_attention_and_prepass_bytes():
    w = wl.WORKLOADS["llm"]
    el = 2 * 16 * 4096 * 128
    assert bench.attn_algorithmic_bytes(w) == 3 * el * 0.5625 + el * 4
    assert bench.prepass_bytes(w) == 3 * el * 2.5625


def test_modes():
    assert bench.prepass_mode("psearch") == "search" and bench.p_mode("psearch") == "search"
    assert bench.prepass_mode("search") == "search" and bench.p_mode("search") == "max"
    assert bench.prepass_mode("ip") == "max" and bench.p_mode("ip") == "max"
    assert bench.sink_tiles("sink") == (1, 1) and bench.sink_tiles("max") == (0, 0)
    c = bench.config_of(wl.WORKLOADS["llm"], "psearch")
    assert c["scale_mode"] == "search" and c["p_scale_mode"] == "search" and not c["incoherence_processing"]
    c = bench.config_of(wl.WORKLOADS["decode"], "sink")
    assert c["sink_tiles"] == [1, 1] and c["Hkv"] == 8


def test_kernel_counts_per_step():
    assert bench.kernels_per_step(wl.WORKLOADS["decode"]) == 3
    assert bench.kernels_per_step(wl.WORKLOADS["llm"]) == 3
    assert bench.kernels_per_step(wl.WORKLOADS["longctx"]) == 6  # + pool, score, top-k
    assert bench.kernels_per_step(wl.WORKLOADS["llm"], "ip") == 9


def test_measured_traffic_only_for_full_launches_of_the_captured_kernel():
    w = wl.WORKLOADS["llm"]
    name = bench.kernel_name(w, "max")
    assert bench.traffic_of(w, "max", name, args()) is not None
    assert bench.traffic_of(w, "max", name, args(batch=1)) is None     # a slice: not the bench launch
    assert bench.traffic_of(w, "psearch", bench.kernel_name(w, "psearch"), args()) is None  # not captured
    d = wl.WORKLOADS["decode"]
    assert bench.traffic_of(d, "sink", bench.kernel_name(d, "sink"), args()) is None
    # every stored figure is at least the algorithmic NVFP4 operand bytes of its launch
    for (wname, mode, kname), t in bench.MEASURED_TRAFFIC.items():
        wk = wl.WORKLOADS[wname]
        floor = bench.hbm_bytes_decode(wk) if wk.kind == "decode" else 3 * wk.B * wk.H * wk.N * wk.D * 0.5625
        assert t >= 0.95 * floor, (wname, mode, kname)


def test_headline_is_the_largest_workload():
    sizes = {n: w.B * w.H * w.N * w.N * w.D for n, w in wl.WORKLOADS.items() if w.kind == "prefill"}
    assert bench.HEADLINE[0] == max(sizes, key=sizes.get)
