"""CPU oracle for the NVFP4 attention hot path -- TEST INFRASTRUCTURE ONLY.

Only the test-suite, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product library
(``bit_quantized_attention_channel_b200``) never imports, links or calls it,
and it shares no code with the CUDA path.

The arithmetic lives in ``oracle.c`` (plain C, FP64 where the method is not
integer-deciding); this module only marshals numpy arrays through ctypes.
Functions and the passages they follow are documented in ``oracle.c``.

Parity status: every entry point here is pinned by ``tests/test_oracle_pins.py``
(closed forms, library routines, brute force, invariants, hand-worked examples
under ``tests/golden/``).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

CFLAGS = ["-O2", "-fopenmp", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared", "-std=c11"]


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so next to it (gcc, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", *CFLAGS, "-o", _LIB, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
    return _LIB


_lib = None


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB)
        P = ctypes.c_void_p
        i, f, d = ctypes.c_int, ctypes.c_float, ctypes.c_double
        L.orc_e2m1_value.argtypes, L.orc_e2m1_value.restype = [i], d
        L.orc_e4m3_value.argtypes, L.orc_e4m3_value.restype = [i], d
        L.orc_e2m1_code.argtypes, L.orc_e2m1_code.restype = [f], i
        L.orc_e4m3_code.argtypes, L.orc_e4m3_code.restype = [f], i
        L.orc_f32_to_bf16.argtypes, L.orc_f32_to_bf16.restype = [f], ctypes.c_uint16
        L.orc_tensor_scale.argtypes = [f, P, P]
        L.orc_quant_nvfp4.argtypes = [P, i, i, i, i, i, i, i, i, i, P, P, P, P, P]
        L.orc_quant_nvfp4.restype = i
        L.orc_dequant.argtypes = [P, P, f, ctypes.c_size_t, i, P]
        L.orc_attn_f64.argtypes = [P, P, P, ctypes.c_long, i, i, i, d, i, P, P, P, P, P, i, P, P]
        L.orc_attn_f64.restype = i
        L.orc_decode_f64.argtypes = [P, P, P, i, i, i, i, i, d, i, i, P, i, P]
        L.orc_decode_f64.restype = i
        L.orc_decode_sink_f64.argtypes = [P, P, P, i, i, i, i, i, d, i, i, i, i, P, P, P, P, i, P]
        L.orc_decode_sink_f64.restype = i
        L.orc_thrift_select.argtypes = [P, P, i, i, i, i, i, i, P, P, P]
        L.orc_thrift_select.restype = i
        L.orc_thrift_select_ex.argtypes = [P, P, P, i, i, i, i, i, i, i, P, P, P]
        L.orc_thrift_select_ex.restype = i
        L.orc_num_threads.restype = i
        L.orc_quant_block.argtypes = [P, i, i, i, P, P, P, P]
        L.orc_block_err.argtypes, L.orc_block_err.restype = [P, i], f
        L.orc_requant_p.argtypes = [P, i, P]
        L.orc_requant_p_mode.argtypes, L.orc_requant_p_mode.restype = [P, i, P, i], i
        L.orc_quant_rows_f32.argtypes = [P, ctypes.c_long, i, i, i, i, P, P, P, P]
        L.orc_quant_rows_f32.restype = i
        L.orc_incoherence.argtypes = [P, P, P, i, i, i, i, P, P, P, P]
        L.orc_incoherence.restype = i
        _lib = L
    return _lib


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def num_threads() -> int:
    return lib().orc_num_threads()


# ---------------------------------------------------------------- formats
def e2m1_value(code: int) -> float:
    return lib().orc_e2m1_value(int(code))


def e4m3_value(code: int) -> float:
    return lib().orc_e4m3_value(int(code))


def e2m1_code(x: float) -> int:
    return lib().orc_e2m1_code(float(x))


def e4m3_code(x: float) -> int:
    return lib().orc_e4m3_code(float(x))


def f32_to_bf16_bits(x: float) -> int:
    return lib().orc_f32_to_bf16(float(x))


def quant_block(xt, search: bool = False, f_lo: int = -2, f_hi: int = 6):
    """One 16-value block in the g-normalised domain -> (codes[16], scale
    code, chosen offset, error of the chosen scale)."""
    x = np.ascontiguousarray(xt, dtype=np.float32)
    assert x.shape == (16,)
    c16 = np.zeros(16, np.uint8)
    sc = np.zeros(1, np.uint8)
    off = np.zeros(1, np.int8)
    err = np.zeros(1, np.float32)
    lib().orc_quant_block(_p(x), int(search), f_lo, f_hi, _p(c16), _p(sc), _p(off), _p(err))
    return c16, int(sc[0]), int(off[0]), float(err[0])


def block_err(xt, scale_code: int) -> float:
    x = np.ascontiguousarray(xt, dtype=np.float32)
    return float(lib().orc_block_err(_p(x), int(scale_code)))


def requant_p(pt):
    p = np.ascontiguousarray(pt, dtype=np.float64)
    out = np.zeros_like(p)
    lib().orc_requant_p(_p(p), len(p), _p(out))
    return out


def requant_p_search(pt, search: bool = True):
    """One block of P~ (at most 16 values) requantised with ScaleSearch (or
    max-scaling): (dequantised P^, chosen E4M3 scale code)."""
    p = np.ascontiguousarray(pt, dtype=np.float64)
    out = np.zeros_like(p)
    c = lib().orc_requant_p_mode(_p(p), len(p), _p(out), int(search))
    return out, c


def _quant_p_mode(quant_p, p_search: bool) -> int:
    """0: P~ kept unquantised, 1: max-scaling, 2: ScaleSearch on P."""
    if not quant_p:
        return 0
    return 2 if p_search else 1


def tensor_scale(amax: float):
    g = ctypes.c_float()
    ig = ctypes.c_float()
    lib().orc_tensor_scale(float(amax), ctypes.byref(g), ctypes.byref(ig))
    return g.value, ig.value


def bf16_bits(x) -> np.ndarray:
    """uint16 view of a bf16 tensor/array (torch bf16 tensor or uint16 array)."""
    if isinstance(x, np.ndarray):
        assert x.dtype == np.uint16
        return np.ascontiguousarray(x)
    import torch

    return np.ascontiguousarray(x.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16))


def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


# ---------------------------------------------------------------- quantisation
ROLE = {"q": 0, "k": 1, "v": 2}


class Quantized:
    """Result of quantize(): logical (row-major) codes and scales."""

    def __init__(self, codes, scales, g, inv_g, k_mean, ss_off, role, shape):
        self.codes, self.scales, self.g, self.inv_g = codes, scales, g, inv_g
        self.k_mean, self.ss_off, self.role, self.shape = k_mean, ss_off, role, shape

    def dequant(self) -> np.ndarray:
        """FP64 values in token-major [B,H,N,D] order (V is transposed back)."""
        B, H, N, D = self.shape
        if self.role == "v":
            rows, cols = B * H * D, N
        else:
            rows, cols = B * H * N, D
        out = np.empty(rows * cols, dtype=np.float64)
        lib().orc_dequant(_p(self.codes), _p(self.scales), self.g, rows, cols, _p(out))
        if self.role == "v":
            return out.reshape(B, H, D, N).transpose(0, 1, 3, 2).copy()
        return out.reshape(B, H, N, D)


def quantize(x, role: str, smooth: bool = True, search: bool = False, f_lo: int = -2, f_hi: int = 6) -> Quantized:
    """Quantise a bf16 [B,H,N,D] tensor (torch bf16 or uint16 bits)."""
    bits = bf16_bits(x)
    B, H, N, D = bits.shape
    r = ROLE[role]
    if r == 2:
        codes = np.zeros((B, H, D, N // 2), np.uint8)
        scales = np.zeros((B, H, D, N // 16), np.uint8)
    else:
        codes = np.zeros((B, H, N, D // 2), np.uint8)
        scales = np.zeros((B, H, N, D // 16), np.uint8)
    off = np.zeros(scales.shape, np.int8)
    g2 = np.zeros(2, np.float32)
    kmean = np.zeros((B, H, D), np.float32) if (r == 1 and smooth) else None
    rc = lib().orc_quant_nvfp4(_p(bits), B, H, N, D, r, int(smooth), int(search), f_lo, f_hi, _p(codes), _p(scales),
                               _p(g2), _p(kmean), _p(off))
    if rc != 0:
        raise ValueError(f"orc_quant_nvfp4 failed: {rc}")
    return Quantized(codes, scales, float(g2[0]), float(g2[1]), kmean, off, role, (B, H, N, D))


def quantize_rows_f32(x, search: bool = False, f_lo: int = -2, f_hi: int = 6) -> Quantized:
    """Quantise FP32 [B,H,N,D] rows (Q/K block layout) to NVFP4 with the same
    tensor scale and block rule as quantize(); no smoothing."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    B, H, N, D = x.shape
    codes = np.zeros((B, H, N, D // 2), np.uint8)
    scales = np.zeros((B, H, N, D // 16), np.uint8)
    off = np.zeros(scales.shape, np.int8)
    g2 = np.zeros(2, np.float32)
    rc = lib().orc_quant_rows_f32(_p(x), B * H * N, D, int(search), f_lo, f_hi, _p(codes), _p(scales), _p(g2),
                                  _p(off))
    if rc != 0:
        raise ValueError(f"orc_quant_rows_f32 failed: {rc}")
    return Quantized(codes, scales, float(g2[0]), float(g2[1]), None, off, "q", (B, H, N, D))


def incoherence(q_bf16, k_bf16, signs, k_mean=None):
    """Incoherence processing of Q and K ("ScaleSearchAttention"): signed
    Hadamard rotation and the per-(b,h,channel) balancing scale r.
    Returns (Q' FP32, K' FP32, r FP32 [B,H,D])."""
    qb, kb = bf16_bits(q_bf16), bf16_bits(k_bf16)
    B, H, N, D = qb.shape
    sg = np.ascontiguousarray(signs, dtype=np.int8)
    km = None if k_mean is None else np.ascontiguousarray(k_mean, dtype=np.float32)
    qo = np.zeros((B, H, N, D), np.float32)
    ko = np.zeros((B, H, N, D), np.float32)
    r = np.zeros((B, H, D), np.float32)
    rc = lib().orc_incoherence(_p(qb), _p(kb), _p(km), B, H, N, D, _p(sg), _p(qo), _p(ko), _p(r))
    if rc != 0:
        raise ValueError(f"orc_incoherence failed: {rc}")
    return qo, ko, r


# ---------------------------------------------------------------- attention
def attn_f64(q, k, v, causal: bool, sm_scale: float, quant_p: bool = True, mask=None, q_raw=None,
             k_raw_smoothed=None, v_raw=None, rows=None, want_lse: bool = False, p_search: bool = False):
    """Run the attention schedule on FP64 [B,H,N,D] operands.  rows: optional
    array of query-row indices (same for every head).  p_search: requantise
    P with ScaleSearch instead of max-scaling."""
    q, k, v = (np.ascontiguousarray(a, dtype=np.float64) for a in (q, k, v))
    B, H, N, D = q.shape
    rr = None if rows is None else np.ascontiguousarray(rows, dtype=np.int32)
    nr = N if rr is None else len(rr)
    out = np.zeros((B, H, nr, D), np.float64)
    lse = np.zeros((B, H, nr), np.float64) if want_lse else None
    if mask is not None:
        mask = np.ascontiguousarray(mask, dtype=np.uint8)
        q_raw, k_raw_smoothed, v_raw = (np.ascontiguousarray(a, dtype=np.float64) for a in
                                        (q_raw, k_raw_smoothed, v_raw))
    rc = lib().orc_attn_f64(_p(q), _p(k), _p(v), B * H, N, D, int(causal), float(sm_scale),
                            _quant_p_mode(quant_p, p_search), _p(mask),
                            _p(q_raw), _p(k_raw_smoothed), _p(v_raw), _p(rr), nr, _p(out), _p(lse))
    if rc != 0:
        raise ValueError(f"orc_attn_f64 failed: {rc}")
    return (out, lse) if want_lse else out


def attention(qq: Quantized, kq: Quantized, vq: Quantized, causal: bool, sm_scale: float | None = None, rows=None,
              mask=None, q_bf16=None, k_bf16=None, v_bf16=None, want_lse: bool = False, p_search: bool = False):
    """NVFP4 attention forward on quantised operands (optionally with
    high-precision blocks from `mask`, which then needs the raw bf16 inputs).
    p_search: ScaleSearch on the requantised P blocks."""
    B, H, N, D = qq.shape
    if sm_scale is None:
        sm_scale = 1.0 / np.sqrt(D)
    q, k, v = qq.dequant(), kq.dequant(), vq.dequant()
    q_raw = k_s = v_raw = None
    if mask is not None:
        q_raw = bf16_to_f64(bf16_bits(q_bf16))
        k_s = bf16_to_f64(bf16_bits(k_bf16))
        if kq.k_mean is not None:
            k_s = k_s - kq.k_mean.astype(np.float64)[:, :, None, :]
        v_raw = bf16_to_f64(bf16_bits(v_bf16))
    return attn_f64(q, k, v, causal, sm_scale, True, mask, q_raw, k_s, v_raw, rows, want_lse, p_search)


def decode_f64(q, k, v, sm_scale: float, quant_p: bool = True, split: int = 4096, pairs=None,
               sink_tiles=(0, 0), q_raw=None, k_raw_smoothed=None, v_raw=None, p_search: bool = False):
    """Split-KV decode on FP64 operands: q [B,Hq,D], k/v [B,Hkv,L,D].
    sink_tiles = (first, last): that many 128-key tiles at each end of the
    cache use the raw operands (q_raw [B,Hq,D], k_raw_smoothed and v_raw
    [B,Hkv,L,D]) with bf16-rounded P."""
    q, k, v = (np.ascontiguousarray(a, dtype=np.float64) for a in (q, k, v))
    B, Hq, D = q.shape
    _, Hkv, L, _ = k.shape
    pp = None if pairs is None else np.ascontiguousarray(pairs, dtype=np.int32)
    npairs = B * Hq if pp is None else len(pp)
    out = np.zeros((npairs, D), np.float64)
    first, last = (int(t) for t in sink_tiles)
    if first or last:
        q_raw, k_raw_smoothed, v_raw = (np.ascontiguousarray(a, dtype=np.float64) for a in
                                        (q_raw, k_raw_smoothed, v_raw))
        assert q_raw.shape == q.shape and k_raw_smoothed.shape == k.shape and v_raw.shape == v.shape
    else:
        q_raw = k_raw_smoothed = v_raw = None
    rc = lib().orc_decode_sink_f64(_p(q), _p(k), _p(v), B, Hq, Hkv, L, D, float(sm_scale),
                                   _quant_p_mode(quant_p, p_search), int(split),
                                   first, last, _p(q_raw), _p(k_raw_smoothed), _p(v_raw), _p(pp), npairs, _p(out))
    if rc != 0:
        raise ValueError(f"orc_decode_sink_f64 failed: {rc}")
    return out


def decode(q_bf16, kq: Quantized, vq: Quantized, sm_scale: float | None = None, split: int = 4096, pairs=None,
           sink_tiles=(0, 0), k_bf16=None, v_bf16=None):
    """NVFP4-KV decode: q [B,Hq,D] bf16 is quantised like a Q tensor (its own
    per-tensor scale, blocks along D, max-scaling).  sink_tiles = (first,
    last) keeps that many 128-key tiles at each end of the cache at full
    precision ("ScaleSearchAttention", attention-sink-aware mixed-precision
    caching); they need the raw bf16 cache k_bf16, v_bf16 [B,Hkv,L,D], and
    the smoothed K mean of kq offsets their keys like the NVFP4 ones."""
    qb = bf16_bits(q_bf16)
    B, Hq, D = qb.shape
    qq = quantize(qb.reshape(1, B, Hq, D), "q", smooth=False, search=False)
    qd = qq.dequant().reshape(B, Hq, D)
    if sm_scale is None:
        sm_scale = 1.0 / np.sqrt(D)
    q_raw = k_s = v_raw = None
    if sink_tiles[0] or sink_tiles[1]:
        q_raw = bf16_to_f64(qb)
        k_s = bf16_to_f64(bf16_bits(k_bf16))
        if kq.k_mean is not None:
            k_s = k_s - kq.k_mean.astype(np.float64)[:, :, None, :]
        v_raw = bf16_to_f64(bf16_bits(v_bf16))
    return decode_f64(qd, kq.dequant(), vq.dequant(), sm_scale, True, split, pairs, sink_tiles, q_raw, k_s, v_raw)


# ---------------------------------------------------------------- selector
def thrift_select(q_bf16, k_bf16, causal: bool, frac_bp: int = 500, want_scores: bool = False,
                  per_row: bool = False, k_mean=None):
    """Block selector.  Default: raw keys, one budget per (b, h).  per_row:
    one budget per query tile; k_mean [B,H,D]: pool the smoothed keys."""
    qb, kb = bf16_bits(q_bf16), bf16_bits(k_bf16)
    B, H, N, D = qb.shape
    T = (N + 127) // 128
    mask = np.zeros((B, H, T, T), np.uint8)
    nsel = np.zeros((B, H), np.int32)
    scores = np.zeros((B, H, T, T), np.float32) if want_scores else None
    km = None if k_mean is None else np.ascontiguousarray(k_mean, dtype=np.float32)
    rc = lib().orc_thrift_select_ex(_p(qb), _p(kb), _p(km), B, H, N, D, int(causal), int(frac_bp), int(per_row),
                                    _p(mask), _p(nsel), _p(scores))
    if rc != 0:
        raise ValueError(f"orc_thrift_select failed: {rc}")
    return (mask, nsel, scores) if want_scores else (mask, nsel)
