"""GPU path (through the C ABI) vs the CPU oracle on the same seeded inputs.

Bar (from the method's definition of what is exact):
  * bit-exact: E2M1 codes, E4M3 scales, per-tensor g, K channel means,
    ScaleSearch offsets, selector masks and counts;
  * attention / decode outputs: max |O_gpu - O_oracle| <= 2e-3 * max |O_oracle|
    and cosine >= 0.9999 (P is requantised from FP32 scores on the GPU and
    from FP64 scores in the oracle, so individual P codes may differ where a
    score sits on a rounding boundary; the output tolerance covers that).
The oracle always quantises the raw inputs itself; nothing it consumes comes
from the GPU.
"""
import math

import numpy as np
import pytest
import torch

import bit_quantized_attention_channel_b200 as sa
import oracle as orc
from bit_quantized_attention_channel_b200 import workloads as wl

pytestmark = pytest.mark.gpu

ATOL_REL = 2e-3
COS_MIN = 0.9999


# ------------------------------------------------------------------ helpers
def status_ok():
    st = sa.sa_device_status(reset=True)
    assert st == 0, sa.STATUS[st]


def gpu_quant(x_cpu, role, smooth=True, mode="max"):
    r = sa.sa_quant_nvfp4(x_cpu.cuda(), role, smooth=smooth, mode=mode, ss_offsets=True)
    status_ok()
    return r


def assert_quant_equal(rg, ro, tag=""):
    B, H, N, D = rg.shape
    codes = sa.codes_to_logical(rg.codes.cpu(), B, H, N, D, rg.role).numpy()
    bad = codes != ro.codes
    assert not bad.any(), f"{tag}: {bad.sum()} code bytes differ, first at {np.argwhere(bad)[:3].tolist()}: " \
                          f"gpu {codes[bad][:8]} oracle {ro.codes[bad][:8]}"
    sc = sa.scales_to_logical(rg.scales.cpu(), B, H, N, D, rg.role).numpy()
    bad = sc != ro.scales
    assert not bad.any(), f"{tag}: {bad.sum()} scales differ: gpu {sc[bad][:8]} oracle {ro.scales[bad][:8]}"
    g = rg.g.cpu().numpy()
    assert g[0] == np.float32(ro.g) and g[1] == np.float32(ro.inv_g), (tag, g, ro.g, ro.inv_g)
    if ro.k_mean is not None:
        assert np.array_equal(rg.k_mean.cpu().numpy(), ro.k_mean), tag
    off = rg.ss_off.cpu().numpy()[: ro.ss_off.size].reshape(ro.ss_off.shape)
    assert np.array_equal(off, ro.ss_off), f"{tag}: {np.sum(off != ro.ss_off)} ScaleSearch offsets differ"
    # padding of the scale atoms is zero
    total = int(rg.scales.numel())
    R, C = (D, N) if rg.role == "v" else (N, D)
    if total > B * H * R * (C // 16):
        logical_sum = int(sc.astype(np.int64).sum())
        assert int(rg.scales.cpu().numpy().astype(np.int64).sum()) == logical_sum, f"{tag}: padding not zero"


def check_close(got, ref, tag=""):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    err = float(np.max(np.abs(got - ref)))
    scale = float(np.max(np.abs(ref)))
    cos = float(np.sum(got * ref) / (np.linalg.norm(got) * np.linalg.norm(ref)))
    print(f"{tag}: max|d|/max|O| = {err / scale:.2e}  cos = {cos:.7f}")
    assert err <= ATOL_REL * scale, (tag, err, scale)
    assert cos >= COS_MIN, (tag, cos)


def exact_rows(q, k, v, causal, rows, sm):
    """FP64 exact softmax attention on raw bf16 inputs for selected rows."""
    qd, kd, vd = (t.double().numpy() for t in (q, k, v))
    B, H, N, D = qd.shape
    out = np.zeros((B, H, len(rows), D))
    for i, r in enumerate(rows):
        s = np.einsum("bhd,bhjd->bhj", qd[:, :, r], kd) * sm
        if causal:
            s[:, :, r + 1:] = -np.inf
        s -= s.max(-1, keepdims=True)
        p = np.exp(s)
        out[:, :, i] = np.einsum("bhj,bhjd->bhd", p, vd) / p.sum(-1)[..., None]
    return out


def quality(got, ref):
    cos = float(np.sum(got * ref) / (np.linalg.norm(got) * np.linalg.norm(ref)))
    rl1 = float(np.abs(got - ref).sum() / np.abs(ref).sum())
    return cos, rl1


def sample_rows(N):
    """Rows compared at full size: edge query tiles {0, 1, T/2, T-2, T-1} at
    offsets {0, 1, 63, 64, 127}, plus 4 seeded random tiles at 8 offsets
    (the rows are the same for every head)."""
    T = (N + 127) // 128
    rows = set()
    for t in sorted({0, 1, T // 2, T - 2, T - 1}):
        if t < 0:
            continue
        for o in (0, 1, 63, 64, 127):
            r = t * 128 + o
            if r < N:
                rows.add(r)
    rng = np.random.default_rng(N)
    for t in rng.choice(T, size=min(4, T), replace=False):
        for o in (0, 17, 31, 32, 64, 95, 100, 127):
            r = int(t) * 128 + o
            if r < N:
                rows.add(r)
    return np.array(sorted(rows), np.int32)


# ------------------------------------------------------------------ inputs
_cache = {}


def inputs(name, **shape):
    key = (name, tuple(sorted(shape.items())))
    if key not in _cache:
        _cache[key] = wl.prefill_inputs(name, **shape)
    return _cache[key]


# ------------------------------------------------------------------ quant
QUANT_CASES = [
    ("tiny", {}, "max"),
    ("tiny", {"N": 400}, "search"),         # ragged: N not a multiple of 128 or 64
    ("llm", {}, "max"),
    ("llm", {}, "search"),
    ("video", {"H": 2}, "search"),
    ("longctx", {"H": 2, "N": 8192}, "max"),
]


@pytest.mark.parametrize("name,shape,mode", QUANT_CASES)
def test_quant_bit_exact(name, shape, mode):
    q, k, v = inputs(name, **shape)
    for role, x in (("q", q), ("k", k), ("v", v)):
        rg = gpu_quant(x, role, smooth=True, mode=mode)
        ro = orc.quantize(x, role, smooth=True, search=mode == "search")
        assert_quant_equal(rg, ro, f"{name}{shape}/{role}/{mode}")


def test_quant_k_unsmoothed_and_zero_tensor():
    _, k, _ = inputs("tiny")
    assert_quant_equal(gpu_quant(k, "k", smooth=False), orc.quantize(k, "k", smooth=False), "k unsmoothed")
    z = torch.zeros(1, 2, 128, 64, dtype=torch.bfloat16)
    for role in ("q", "k", "v"):
        assert_quant_equal(gpu_quant(z, role, mode="search"), orc.quantize(z, role, search=True), f"zero/{role}")


def test_quant_nonfinite_is_reported():
    x = torch.randn(1, 1, 128, 64).to(torch.bfloat16)
    x[0, 0, 5, 7] = float("nan")
    sa.sa_quant_nvfp4(x.cuda(), "q")
    assert sa.sa_device_status(reset=True) == 4  # SA_ERR_NONFINITE
    status_ok()


@pytest.mark.parametrize("name", ["video", "longctx"])
def test_quant_bit_exact_full_size(name):
    """Full-size pre-pass of the long workloads (every element compared)."""
    q, k, v = inputs(name)
    w = wl.WORKLOADS[name]
    mode = "search" if "search" in w.scale_modes else "max"
    for role, x in (("q", q), ("k", k), ("v", v)):
        assert_quant_equal(gpu_quant(x, role, mode=mode), orc.quantize(x, role, search=mode == "search"),
                           f"{name}/{role}")


# ------------------------------------------------------------------ selector
@pytest.mark.parametrize("causal,frac", [(False, 500), (True, 500), (True, 1000), (False, 0), (True, 10000)])
def test_select_bit_exact_small(causal, frac):
    q, k, _ = inputs("longctx", H=3, N=1024 + 256)
    mg, ng = sa.sa_thrift_select(q.cuda(), k.cuda(), causal, frac)
    status_ok()
    mo, no = orc.thrift_select(q, k, causal, frac)
    assert np.array_equal(ng.cpu().numpy(), no)
    assert np.array_equal(mg.cpu().numpy(), mo)


def test_select_ties_break_to_lower_index():
    q = torch.ones(1, 1, 1024, 64, dtype=torch.bfloat16)
    mg, ng = sa.sa_thrift_select(q.cuda(), q.cuda(), True, 1000)
    status_ok()
    mo, no = orc.thrift_select(q, q, True, 1000)
    assert np.array_equal(mg.cpu().numpy(), mo) and np.array_equal(ng.cpu().numpy(), no)


def test_select_bit_exact_full_size():
    """Selector on the full long-context workload (B1 H32 N65536, 5 %)."""
    q, k, _ = inputs("longctx")
    mg, ng = sa.sa_thrift_select(q.cuda(), k.cuda(), True, 500)
    status_ok()
    mo, no = orc.thrift_select(q, k, True, 500)
    assert np.array_equal(ng.cpu().numpy(), no)
    assert (no == 6567).all()
    assert np.array_equal(mg.cpu().numpy(), mo)


@pytest.mark.parametrize("per_row,smoothed,causal,frac", [(True, False, True, 500), (True, False, False, 500),
                                                          (False, True, True, 500), (True, True, True, 1500),
                                                          (True, False, True, 0), (True, True, False, 10000)])
def test_select_ex_bit_exact(per_row, smoothed, causal, frac):
    """Per-query-tile budgets and smoothed-K pooling: masks and counts equal
    the oracle's bit for bit (ragged N, several heads)."""
    q, k, _ = inputs("longctx", H=3, N=1024 + 256 + 64)
    # each side pools with its own channel means (bit-identical, checked by the quant tests)
    km_gpu = gpu_quant(k, "k").k_mean if smoothed else None
    km_orc = orc.quantize(k, "k").k_mean if smoothed else None
    mg, ng = sa.sa_thrift_select_ex(q.cuda(), k.cuda(), causal, frac, per_row=per_row, k_mean=km_gpu)
    status_ok()
    mo, no = orc.thrift_select(q, k, causal, frac, per_row=per_row, k_mean=km_orc)
    assert np.array_equal(ng.cpu().numpy(), no)
    assert np.array_equal(mg.cpu().numpy(), mo)


def test_select_ex_per_row_full_size():
    """Per-row budget on the full long-context workload (B1 H32 N65536)."""
    q, k, _ = inputs("longctx")
    mg, ng = sa.sa_thrift_select_ex(q.cuda(), k.cuda(), True, 500, per_row=True)
    status_ok()
    mo, no = orc.thrift_select(q, k, True, 500, per_row=True)
    assert np.array_equal(ng.cpu().numpy(), no)
    assert np.array_equal(mg.cpu().numpy(), mo)


@pytest.mark.parametrize("shape,smooth,mode", [({"N": 4096, "D": 128, "B": 2, "H": 16}, True, "max"),
                                               ({"N": 416, "D": 64}, True, "search"),
                                               ({"N": 352, "D": 128}, False, "max"),
                                               ({"N": 1040, "D": 64, "H": 3}, True, "max")])
def test_fused_prepass_equals_per_tensor(shape, smooth, mode):
    """sa_quant_nvfp4_qkv writes the same bytes as three sa_quant_nvfp4 calls."""
    q, k, v = (t.cuda() for t in inputs("tiny", **shape))
    ref = (sa.sa_quant_nvfp4(q, "q", mode=mode), sa.sa_quant_nvfp4(k, "k", smooth=smooth, mode=mode),
           sa.sa_quant_nvfp4(v, "v", mode=mode))
    got = sa.sa_quant_nvfp4_qkv(q, k, v, smooth=smooth, mode=mode)
    status_ok()
    B, H, N, D = q.shape
    for a, b in zip(got, ref):
        # V bytes past token N in the last 128-token tile are unspecified
        assert torch.equal(sa.codes_to_logical(a.codes, B, H, N, D, a.role),
                           sa.codes_to_logical(b.codes, B, H, N, D, b.role)), a.role
        assert torch.equal(a.scales, b.scales), a.role
        assert torch.equal(a.g, b.g), a.role
    if smooth:
        assert torch.equal(got[1].k_mean, ref[1].k_mean)


# ------------------------------------------------------------------ attention
ATTN_CASES = [
    ("tiny", {}, False, "max", None),                  # every row compared
    ("tiny", {}, True, "max", None),
    ("tiny", {"N": 416, "D": 128}, True, "max", None),  # ragged last tile (416 = 3*128 + 32)
    ("tiny", {"N": 352}, False, "search", None),       # ragged, D = 64
    ("tiny", {"N": 128, "H": 1}, True, "max", None),   # a single tile
    ("tiny", {"N": 640, "D": 128}, True, "max", None),  # odd tile count: last CTA has one query tile
    ("llm", {}, True, "max", "sample"),
    ("llm", {}, True, "search", "sample"),
    ("video", {}, False, "search", "sample"),         # full video size: non-causal, ~21 items per CTA
]


def run_attention(q, k, v, causal, mode):
    qg, kg, vg = (gpu_quant(x, r, mode=mode) for x, r in ((q, "q"), (k, "k"), (v, "v")))
    out, lse = sa.sa_attn_fwd(qg, kg, vg, causal, want_lse=True)
    status_ok()
    return out.cpu().numpy(), lse.cpu().numpy()


@pytest.mark.parametrize("name,shape,causal,mode,rows", ATTN_CASES)
def test_attention_matches_oracle(name, shape, causal, mode, rows):
    q, k, v = inputs(name, **shape)
    B, H, N, D = q.shape
    og, lg = run_attention(q, k, v, causal, mode)
    ss = mode == "search"
    qo, ko, vo = orc.quantize(q, "q", search=ss), orc.quantize(k, "k", search=ss), orc.quantize(v, "v", search=ss)
    rr = sample_rows(N) if rows == "sample" else None
    ref, lse_ref = orc.attention(qo, ko, vo, causal, rows=rr, want_lse=True)
    got = og if rr is None else og[:, :, rr]
    lse_got = lg if rr is None else lg[:, :, rr]
    check_close(got, ref, f"attn {name}{shape} causal={causal} {mode}")
    assert np.max(np.abs(lse_got - lse_ref)) < 1e-3
    # quality against exact FP64 attention on the raw inputs (reported)
    rq = rr if rr is not None else np.arange(N)
    ex = exact_rows(q, k, v, causal, rq[:64], 1 / math.sqrt(D))
    print("  quality vs exact (gpu): cos %.6f relL1 %.4f" % quality(got[:, :, :64], ex))
    print("  quality vs exact (oracle): cos %.6f relL1 %.4f" % quality(ref[:, :, :64], ex))


# ------------------------------------------------------------------ ScaleSearch on P
P_SEARCH_CASES = [
    ("tiny", {}, True, "max", None),                   # every row compared
    ("tiny", {"N": 416, "D": 128}, False, "search", None),  # ragged last tile, D = 128
    ("tiny", {"N": 352}, True, "search", None),        # ragged, causal, D = 64
    ("llm", {"B": 1, "H": 4}, True, "search", None),   # LLM shape, every row of 4 heads
    ("llm", {}, True, "search", "sample"),             # the full LLM workload: Q, K, P, V all ScaleSearch
]


@pytest.mark.parametrize("name,shape,causal,mode,rows", P_SEARCH_CASES)
def test_attention_p_search_matches_oracle(name, shape, causal, mode, rows):
    """ScaleSearch on the requantised P (sa_attn_fwd_ex) against the oracle's
    attention with P searched the same way."""
    q, k, v = inputs(name, **shape)
    B, H, N, D = q.shape
    qg, kg, vg = (gpu_quant(x, r, mode=mode) for x, r in ((q, "q"), (k, "k"), (v, "v")))
    og, lg = sa.sa_attn_fwd(qg, kg, vg, causal, want_lse=True, p_mode="search")
    status_ok()
    og, lg = og.cpu().numpy(), lg.cpu().numpy()
    ss = mode == "search"
    qo, ko, vo = orc.quantize(q, "q", search=ss), orc.quantize(k, "k", search=ss), orc.quantize(v, "v", search=ss)
    rr = sample_rows(N) if rows == "sample" else None
    ref, lse_ref = orc.attention(qo, ko, vo, causal, rows=rr, want_lse=True, p_search=True)
    got = og if rr is None else og[:, :, rr]
    lse_got = lg if rr is None else lg[:, :, rr]
    check_close(got, ref, f"attn P-search {name}{shape} causal={causal} {mode}")
    assert np.max(np.abs(lse_got - lse_ref)) < 1e-3
    if rr is None:
        # the searched P is a different requantisation: the max-scaled oracle is further away
        ref_max = orc.attention(qo, ko, vo, causal)
        d_search = np.abs(og - ref).mean()
        d_max = np.abs(og - ref_max).mean()
        print("  mean |gpu - oracle(P search)| %.3e, |gpu - oracle(P max)| %.3e" % (d_search, d_max))
        assert d_search < d_max


def test_attention_p_search_with_mask_is_unsupported():
    q, k, v = inputs("tiny")
    B, H, N, D = q.shape
    qg, kg, vg = (gpu_quant(x, r) for x, r in ((q, "q"), (k, "k"), (v, "v")))
    T = (N + 127) // 128
    mask = torch.zeros(B, H, T, T, dtype=torch.uint8, device="cuda")
    with pytest.raises(RuntimeError, match="UNSUPPORTED"):
        sa.sa_attn_fwd(qg, kg, vg, True, mask=mask, q_bf16=q.cuda(), k_bf16=k.cuda(), v_bf16=v.cuda(),
                       p_mode="search")
    status_ok()


# ------------------------------------------------------------------ incoherence processing
IP_CASES = [
    ("tiny", {}, True, "max", True),                         # B1 H2 N256 D64, causal
    # ragged last tile, ScaleSearch.  Causal: on 1056-key non-causal rows one P code flip at the top of
    # the E2M1 grid (FP32 exp2 here, FP64 exp in the oracle, a rounding-boundary case) moved one output
    # element by 6.5e-3 max|O| (cosine 0.9999999) while the Q' and K' bytes were identical
    ("tiny", {"N": 1056, "D": 128, "H": 3}, True, "search", True),
    ("tiny", {"N": 512}, False, "max", True),                # K not smoothed
    ("llm", {"B": 1, "H": 4, "N": 2048}, True, "max", True),  # LLM head shape
]


def ip_signs(D, seed=7):
    return np.where(np.random.default_rng(seed).random(D) < 0.5, -1, 1).astype(np.int8)


@pytest.mark.parametrize("name,shape,smooth,mode,causal", IP_CASES)
def test_incoherence_prepass_bit_exact(name, shape, smooth, mode, causal):
    """Q' and K' after the Hadamard rotation and the balancing pair: codes,
    scales, tensor scales, ScaleSearch offsets, r and the K mean bit-exact
    against the oracle; then attention on them against the oracle's."""
    q, k, v = inputs(name, **shape)
    B, H, N, D = q.shape
    signs = ip_signs(D)
    if name == "tiny" and N == 1056:  # the rotation pass alone also takes a tail of 16 rows
        q16, k16 = q[:, :, :1040].contiguous(), k[:, :, :1040].contiguous()
        a, b, r16 = sa.sa_quant_nvfp4_ip(q16.cuda(), k16.cuda(), torch.from_numpy(signs).cuda(), mode=mode,
                                         ss_offsets=True)
        status_ok()
        qo16, ko16, ro16 = orc.incoherence(q16, k16, signs, orc.quantize(k16, "k").k_mean)
        assert np.array_equal(r16.cpu().numpy(), ro16)
        assert_quant_equal(a, orc.quantize_rows_f32(qo16, search=mode == "search"), "Q' N=1040")
        assert_quant_equal(b, orc.quantize_rows_f32(ko16, search=mode == "search"), "K' N=1040")
    oq, ok, r = sa.sa_quant_nvfp4_ip(q.cuda(), k.cuda(), torch.from_numpy(signs).cuda(), smooth=smooth, mode=mode,
                                     ss_offsets=True)
    status_ok()
    ss = mode == "search"
    mu = orc.quantize(k, "k").k_mean if smooth else None
    qo, ko, ro = orc.incoherence(q, k, signs, mu)
    assert np.array_equal(r.cpu().numpy(), ro)
    if smooth:
        assert np.array_equal(ok.k_mean.cpu().numpy(), mu)
    rq, rk = orc.quantize_rows_f32(qo, search=ss), orc.quantize_rows_f32(ko, search=ss)
    assert_quant_equal(oq, rq, "Q'")
    assert_quant_equal(ok, rk, "K'")
    vg = gpu_quant(v, "v", mode=mode)
    og = sa.sa_attn_fwd(oq, ok, vg, causal).cpu().numpy()
    status_ok()
    ref = orc.attention(rq, rk, orc.quantize(v, "v", search=ss), causal)
    check_close(og, ref, f"attn after IP {name}{shape}")


def test_incoherence_keeps_the_scores():
    """Scores of the rotated, balanced operands (dequantised GPU codes)
    approximate Q (K - mu)^T as the plain NVFP4 operands do (the rotation and
    R cancel in the product): their error is of the same order (on these
    Gaussian inputs somewhat larger, as the oracle pins record)."""
    q, k, _ = inputs("tiny")
    B, H, N, D = q.shape
    oq, ok, _ = sa.sa_quant_nvfp4_ip(q.cuda(), k.cuda(), torch.from_numpy(ip_signs(D)).cuda())
    status_ok()

    def deq(t):
        c = sa.codes_to_logical(t.codes.cpu(), B, H, N, D, t.role).numpy()
        sc = sa.scales_to_logical(t.scales.cpu(), B, H, N, D, t.role).numpy()
        return orc.Quantized(c, sc, float(t.g[0]), float(t.g[1]), None, None, "q", (B, H, N, D)).dequant()

    S_ip = np.einsum("bhid,bhjd->bhij", deq(oq), deq(ok))
    ko = orc.quantize(k, "k")
    mu = ko.k_mean.astype(np.float64)
    S = np.einsum("bhid,bhjd->bhij", q.double().numpy(), k.double().numpy() - mu[:, :, None, :])
    S_plain = np.einsum("bhid,bhjd->bhij", orc.quantize(q, "q").dequant(), ko.dequant())
    rel = np.abs(S_ip - S).mean() / np.abs(S).mean()
    rel_plain = np.abs(S_plain - S).mean() / np.abs(S).mean()
    print("  mean |S - S_exact| / mean |S_exact|: IP %.4f, plain %.4f" % (rel, rel_plain))
    assert rel < 2.0 * rel_plain


# ------------------------------------------------------------------ decode
def run_decode(q, k, v):
    B, Hkv, L, D = k.shape
    kg = gpu_quant(k, "k")
    vg = gpu_quant(v, "v")
    out = sa.sa_attn_decode_kvfp4(q.cuda(), kg, vg)
    status_ok()
    return out.cpu().numpy()


@pytest.mark.parametrize("shape", [dict(B=2, Hq=8, Hkv=2, L=8192, D=128), dict(B=1, Hq=4, Hkv=4, L=4096 + 384, D=64),
                                   dict(B=3, Hq=8, Hkv=1, L=256, D=128)])
def test_decode_matches_oracle(shape):
    q, k, v = wl.decode_inputs(**shape)
    og = run_decode(q, k, v)
    ko, vo = orc.quantize(k, "k"), orc.quantize(v, "v")
    ref = orc.decode(q, ko, vo).reshape(og.shape)
    check_close(og, ref, f"decode {shape}")


def test_decode_full_size_sampled():
    """Full decode workload (B32 Hq32 Hkv8 L32768 D128); all outputs from the
    GPU, sampled (b, head) pairs from the oracle."""
    q, k, v = wl.decode_inputs("decode")
    og = run_decode(q, k, v)
    ko, vo = orc.quantize(k, "k"), orc.quantize(v, "v")
    fixed = [0, 1, 5, 31, 32 * 7 + 3, 32 * 16 + 17, 32 * 31 + 30, 32 * 32 - 1]
    extra = np.random.default_rng(4).choice(32 * 32, size=24, replace=False)
    pairs = np.array(sorted(set(fixed) | {int(e) for e in extra}), np.int32)
    ref = orc.decode(q, ko, vo, pairs=pairs)
    check_close(og.reshape(-1, 128)[pairs], ref, "decode full")


# ------------------------------------------------------------------ sink-aware decode cache
def sink_cache(shape, seed=0):
    """Decode inputs whose first and last keys carry extra score mass (the
    attention-sink pattern): the first and last 8 keys of every head x3."""
    q, k, v = wl.decode_inputs(seed=seed, **shape) if shape else wl.decode_inputs("decode", seed=seed)
    k = k.float()
    k[:, :, :8] *= 3.0
    k[:, :, -8:] *= 3.0
    return q, k.bfloat16(), v


def run_decode_sink(q, k, v, tiles, smooth=True):
    kg = gpu_quant(k, "k", smooth=smooth)
    vg = gpu_quant(v, "v")
    kd, vd = k.cuda(), v.cuda()
    out = sa.sa_attn_decode_kvfp4(q.cuda(), kg, vg, sink_tiles=tiles, k_sink=sa.sink_tiles_of(kd, *tiles),
                                  v_sink=sa.sink_tiles_of(vd, *tiles))
    status_ok()
    return out.cpu().numpy()


@pytest.mark.parametrize("shape,tiles,smooth", [
    (dict(B=2, Hq=8, Hkv=2, L=8192, D=128), (1, 1), True),
    (dict(B=2, Hq=8, Hkv=2, L=8192, D=128), (4, 36), True),   # the last tiles span two splits
    (dict(B=1, Hq=4, Hkv=4, L=4096 + 384, D=64), (2, 3), True),
    (dict(B=1, Hq=4, Hkv=4, L=4096 + 384, D=64), (1, 0), False),  # K not smoothed
    (dict(B=3, Hq=8, Hkv=1, L=256, D=128), (1, 1), True),   # every tile at full precision
    (dict(B=2, Hq=6, Hkv=2, L=1024, D=128), (0, 2), True),  # G = 3
])
def test_decode_sink_matches_oracle(shape, tiles, smooth):
    q, k, v = sink_cache(shape)
    og = run_decode_sink(q, k, v, tiles, smooth)
    ko, vo = orc.quantize(k, "k", smooth=smooth), orc.quantize(v, "v")
    ref = orc.decode(q, ko, vo, sink_tiles=tiles, k_bf16=k, v_bf16=v).reshape(og.shape)
    check_close(og, ref, f"decode sink {shape} {tiles}")
    # the full-precision tiles matter: the plain NVFP4 decode is measurably further away
    plain = orc.decode(q, ko, vo).reshape(og.shape)
    print("  |sink - plain| / max|O| = %.2e" % (np.max(np.abs(ref - plain)) / np.max(np.abs(ref))))


def test_decode_sink_full_size_sampled():
    """Decode workload (B32 Hq32 Hkv8 L32768 D128) with the first and last
    tile at full precision; all outputs from the GPU, sampled (b, head)
    pairs from the oracle."""
    q, k, v = sink_cache(None)
    tiles = (1, 1)
    og = run_decode_sink(q, k, v, tiles)
    ko, vo = orc.quantize(k, "k"), orc.quantize(v, "v")
    pairs = np.array(sorted({0, 7, 32 * 9 + 4, 32 * 31 + 31} |
                            {int(e) for e in np.random.default_rng(5).choice(32 * 32, size=20, replace=False)}),
                     np.int32)
    ref = orc.decode(q, ko, vo, pairs=pairs, sink_tiles=tiles, k_bf16=k, v_bf16=v)
    check_close(og.reshape(-1, 128)[pairs], ref, "decode sink full")


def test_decode_sink_none_is_plain_decode():
    """sink_tiles = (0, 0) runs the plain NVFP4 decode (bit-identical)."""
    q, k, v = wl.decode_inputs(B=2, Hq=8, Hkv=2, L=8192, D=128)
    kg, vg = gpu_quant(k, "k"), gpu_quant(v, "v")
    a = sa.sa_attn_decode_kvfp4(q.cuda(), kg, vg)
    b = sa.sa_attn_decode_kvfp4(q.cuda(), kg, vg, sink_tiles=(0, 0))
    status_ok()
    assert torch.equal(a, b)


# ------------------------------------------------------------------ mixed precision
def run_mixed(q, k, v, causal, mask_cpu):
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    qg, kg, vg = gpu_quant(q, "q"), gpu_quant(k, "k"), gpu_quant(v, "v")
    out, lse = sa.sa_attn_fwd(qg, kg, vg, causal, mask=torch.from_numpy(mask_cpu).cuda(), q_bf16=qd, k_bf16=kd,
                              v_bf16=vd, want_lse=True)
    status_ok()
    return out.cpu().numpy(), lse.cpu().numpy()


@pytest.mark.parametrize("mask_kind,causal,N,D", [("select", True, 1024, 128), ("select", False, 1024 + 256, 64),
                                                  ("all", True, 512, 128), ("random", True, 640, 128),
                                                  ("random", False, 416, 64)])
def test_mixed_attention_matches_oracle(mask_kind, causal, N, D):
    q, k, v = inputs("longctx", H=2, N=N, D=D)
    T = (N + 127) // 128
    if mask_kind == "select":
        mask, _ = orc.thrift_select(q, k, causal, 1500)
    elif mask_kind == "all":
        mask = np.ones((1, 2, T, T), np.uint8)
    else:
        mask = (np.random.default_rng(3).random((1, 2, T, T)) < 0.3).astype(np.uint8)
    og, lg = run_mixed(q, k, v, causal, mask)
    qo, ko, vo = orc.quantize(q, "q"), orc.quantize(k, "k"), orc.quantize(v, "v")
    ref, lse_ref = orc.attention(qo, ko, vo, causal, mask=mask, q_bf16=q, k_bf16=k, v_bf16=v, want_lse=True)
    check_close(og, ref, f"mixed {mask_kind} causal={causal} N={N} D={D}")
    # a bf16 block's P is rounded to bf16 as the method states, then scaled into
    # the NVFP4 accumulator's units and rounded again: the denominator can
    # differ by up to 2^-8 relative where bf16 blocks dominate a row
    assert np.max(np.abs(lg - lse_ref)) < 4e-3
    # with no block selected the mixed kernel computes the NVFP4 result
    if mask_kind == "select":
        og0, _ = run_mixed(q, k, v, causal, np.zeros_like(mask))
        of, _ = run_attention(q, k, v, causal, "max")
        check_close(og0, of, "mixed kernel, empty mask vs NVFP4 kernel")


def test_mixed_full_size_sampled():
    """Long-context mixed workload (B1 H32 N65536 causal, 5 % bf16 blocks
    chosen by the GPU selector, checked bit-exact against the oracle's)."""
    q, k, v = inputs("longctx")
    mg, _ = sa.sa_thrift_select(q.cuda(), k.cuda(), True, 500)
    mask = mg.cpu().numpy()
    mo, _ = orc.thrift_select(q, k, True, 500)
    assert np.array_equal(mask, mo)
    og, _ = run_mixed(q, k, v, True, mask)
    qo, ko, vo = orc.quantize(q, "q"), orc.quantize(k, "k"), orc.quantize(v, "v")
    rows = sample_rows(q.shape[2])
    ref = orc.attention(qo, ko, vo, True, rows=rows, mask=mo, q_bf16=q, k_bf16=k, v_bf16=v)
    check_close(og[:, :, rows], ref, "mixed full size")
    # report the ThriftAttention-style gap recovery on these rows
    fp4 = orc.attention(qo, ko, vo, True, rows=rows)
    ex = exact_rows(q, k, v, True, rows, 1 / math.sqrt(q.shape[3]))
    e4 = np.linalg.norm(fp4 - ex)
    emx = np.linalg.norm(ref - ex)
    print(f"  FP4->exact gap recovered by 5% bf16 blocks: {100 * (1 - emx / e4):.1f}%")


# ------------------------------------------------------------------ bounded waits
def test_wait_limit_gives_up_cleanly_and_the_next_call_is_normal():
    """A wait limit far below one copy's latency makes the attention kernel's
    first pipeline wait give up: the call reports SA_ERR_TIMEOUT through the
    status word (every warp unwinds, issued copies and MMAs are drained), and
    with the default limit restored the next call runs and matches the oracle.
    Nothing is broken on purpose: every arrive still happens."""
    q, k, v = inputs("tiny")
    qg, kg, vg = (gpu_quant(x, r) for x, r in ((q, "q"), (k, "k"), (v, "v")))
    try:
        sa.sa_set_wait_cycles(200)
        sa.sa_attn_fwd(qg, kg, vg, False)
        assert sa.sa_device_status(reset=True) == 6  # SA_ERR_TIMEOUT
    finally:
        sa.sa_set_wait_cycles(0)
    out = sa.sa_attn_fwd(qg, kg, vg, False)
    status_ok()
    qo, ko, vo = orc.quantize(q, "q"), orc.quantize(k, "k"), orc.quantize(v, "v")
    check_close(out.cpu().numpy(), orc.attention(qo, ko, vo, False), "attention after a timed-out call")
