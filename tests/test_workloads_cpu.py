"""The seeded synthetic inputs follow their stated recipe: shapes, value
distributions, per-channel K offsets, heavy tails and attention-sink rows,
and the same seed gives the same tensors.  Small slices of each workload
keep this on the CPU."""
import math

import numpy as np
import pytest

from bit_quantized_attention_channel_b200 import workloads as wl


def test_workload_shapes_and_flags():
    W = wl.WORKLOADS
    assert (W["tiny"].B, W["tiny"].H, W["tiny"].N, W["tiny"].D, W["tiny"].causal) == (1, 2, 256, 64, False)
    assert (W["llm"].B, W["llm"].H, W["llm"].N, W["llm"].D, W["llm"].causal) == (2, 16, 4096, 128, True)
    assert (W["video"].B, W["video"].H, W["video"].N, W["video"].D, W["video"].causal) == (1, 24, 32768, 128, False)
    assert (W["decode"].B, W["decode"].H, W["decode"].Hkv, W["decode"].N, W["decode"].D) == (32, 32, 8, 32768, 128)
    assert (W["longctx"].B, W["longctx"].H, W["longctx"].N, W["longctx"].D) == (1, 32, 65536, 128)
    assert W["longctx"].causal and W["longctx"].thrift_bp == 500


def _np(t):
    return t.float().numpy().astype(np.float64)


def test_llm_inputs_are_gaussian_with_a_k_channel_offset():
    q, k, v = (_np(t) for t in wl.prefill_inputs("llm", B=1, H=16, N=2048, D=128))
    assert q.shape == (1, 16, 2048, 128)
    for x in (q, v):
        assert abs(x.mean()) < 0.01 and abs(x.std() - 1.0) < 0.01
    # K = N(0,1) + an offset per (head, channel) drawn from N(0, 3^2)
    off = k.mean(axis=2)[0]                      # [H, D], token mean ~ offset
    assert abs(off.std() - 3.0) < 0.2
    assert abs((k - k.mean(axis=2, keepdims=True)).std() - 1.0) < 0.01


def test_video_inputs_are_student_t4_with_unit_variance():
    q, k, v = (_np(t) for t in wl.prefill_inputs("video", H=2, N=8192))
    for x in (q, v):
        assert abs(x.std() - 1.0) < 0.05          # t(4) has variance 2; / sqrt(2) gives 1
        # heavy tails: |x| > 4 is ~1e-3 for t(4)/sqrt(2) against 6e-5 for N(0, 1)
        assert (np.abs(x) > 4).mean() > 5e-4
    assert abs(k.mean(axis=2)[0].std() - 2.0) < 0.3  # K channel offsets N(0, 2^2)


def test_longctx_inputs_have_scaled_sink_key_rows():
    N = 4096
    _, k, _ = (_np(t) for t in wl.prefill_inputs("longctx", H=2, N=N))
    norms = np.linalg.norm(k[0, 0], axis=1)
    sinks = np.flatnonzero(norms > 4 * np.median(norms))
    assert len(sinks) == math.ceil(0.01 * N)
    assert abs(np.median(norms[sinks]) / np.median(norms) - 8.0) < 0.5
    # the same positions in every head
    norms1 = np.linalg.norm(k[0, 1], axis=1)
    assert np.array_equal(sinks, np.flatnonzero(norms1 > 4 * np.median(norms1)))


def test_decode_inputs_shapes():
    q, k, v = wl.decode_inputs("decode", B=2, L=1024)
    assert tuple(q.shape) == (2, 32, 128) and tuple(k.shape) == (2, 8, 1024, 128) and k.shape == v.shape


@pytest.mark.parametrize("name", ["tiny", "llm"])
def test_inputs_are_seeded(name):
    a = wl.prefill_inputs(name, B=1, H=2, N=256)
    b = wl.prefill_inputs(name, B=1, H=2, N=256)
    c = wl.prefill_inputs(name, seed=1, B=1, H=2, N=256)
    assert all(x.equal(y) for x, y in zip(a, b))
    assert not a[0].equal(c[0])
