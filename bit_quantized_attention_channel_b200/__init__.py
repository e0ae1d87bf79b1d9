"""B200-native NVFP4 attention: Python binding of libsa (include/sa.h).

This module only marshals arguments: it allocates result tensors with torch
(device memory and streams are torch's plumbing) and passes raw pointers to the
C ABI, whose CUDA kernels do every step of the computation.  There is no CPU or
PyTorch fallback: if libsa.so is missing or a call fails, an exception is
raised.

Entry points keep the C names:
  sa_quant_nvfp4        smoothing + NVFP4 pre-pass (max-scaling or ScaleSearch)
  sa_quant_nvfp4_qkv    the same for Q, K and V of one shape in two launches
  sa_thrift_select      high-precision block selector
  sa_thrift_select_ex   the selector with per-row budgets / smoothed-K pooling
  sa_attn_fwd           NVFP4 attention forward (optionally with bf16 blocks)
  sa_attn_decode_kvfp4  decode over an NVFP4 KV cache (optionally with
                        full-precision first/last tiles)
"""
from __future__ import annotations

import ctypes
import math
import os
from dataclasses import dataclass

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libsa.so")

SA_ROLE = {"q": 0, "k": 1, "v": 2}
SA_SCALE = {"max": 0, "search": 1}
STATUS = ["SA_OK", "SA_ERR_INVALID_ARG", "SA_ERR_UNSUPPORTED", "SA_ERR_WORKSPACE", "SA_ERR_NONFINITE", "SA_ERR_CUDA",
          "SA_ERR_TIMEOUT", "SA_ERR_DEVICE_ASSERT"]


class SAError(RuntimeError):
    def __init__(self, fn, code):
        name = STATUS[code] if 0 <= code < len(STATUS) else str(code)
        super().__init__(f"{fn} returned {name}")
        self.code = code


_lib = None


def lib():
    """Load libsa.so (built in-tree by build.py); raises if it is absent."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"libsa.so not found at {LIB_PATH}; run `python -m bit_quantized_attention_channel_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        P, I, F, Z = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
        L.sa_status_string.argtypes, L.sa_status_string.restype = [I], ctypes.c_char_p
        L.sa_device_status.argtypes, L.sa_device_status.restype = [P, I], I
        L.sa_set_wait_cycles.argtypes, L.sa_set_wait_cycles.restype = [ctypes.c_longlong], None
        for n in ("sa_codes_bytes", "sa_scales_bytes"):
            getattr(L, n).argtypes, getattr(L, n).restype = [I, I, I, I, I], Z
        L.sa_quant_workspace_size.argtypes, L.sa_quant_workspace_size.restype = [I, I, I, I, I], Z
        L.sa_quant_nvfp4.argtypes = [P, I, I, I, I, I, I, I, I, I, P, P, P, P, P, P, Z, P]
        L.sa_quant_nvfp4.restype = I
        L.sa_quant_nvfp4_noalloc.argtypes = [P, I, I, I, I, I, I, I, I, I, P, P, P, P, P, P]
        L.sa_quant_nvfp4_noalloc.restype = I
        L.sa_quant_qkv_workspace_size.argtypes, L.sa_quant_qkv_workspace_size.restype = [I, I, I, I], Z
        L.sa_quant_nvfp4_qkv.argtypes = [P, P, P, I, I, I, I, I, I, I, I, P, P, P, P, P, P, P, P, P, P, P, Z, P]
        L.sa_quant_nvfp4_qkv.restype = I
        L.sa_select_workspace_size.argtypes, L.sa_select_workspace_size.restype = [I, I, I, I], Z
        L.sa_thrift_select.argtypes = [P, P, I, I, I, I, I, I, P, P, P, Z, P]
        L.sa_thrift_select.restype = I
        L.sa_thrift_select_ex.argtypes = [P, P, P, I, I, I, I, I, I, I, P, P, P, Z, P]
        L.sa_thrift_select_ex.restype = I
        L.sa_attn_fwd.argtypes = [P, P, P, P, P, P, P, P, P, I, I, I, I, I, F, P, P, P, P, P, P, P, P]
        L.sa_attn_fwd.restype = I
        L.sa_decode_workspace_size.argtypes, L.sa_decode_workspace_size.restype = [I, I, I, I, I], Z
        L.sa_attn_decode_kvfp4.argtypes = [P, P, P, P, P, P, P, I, I, I, I, I, F, P, P, Z, P]
        L.sa_attn_decode_kvfp4.restype = I
        L.sa_attn_decode_kvfp4_sink.argtypes = [P, P, P, P, P, P, P, I, I, I, I, I, F, I, I, P, P, P, P, P, Z, P]
        L.sa_attn_decode_kvfp4_sink.restype = I
        L.sa_attn_fwd_ex.argtypes = [P, P, P, P, P, P, P, P, P, I, I, I, I, I, F, I, P, P, P, P, P, P, P, P]
        L.sa_attn_fwd_ex.restype = I
        L.sa_quant_ip_workspace_size.argtypes, L.sa_quant_ip_workspace_size.restype = [I, I, I, I], Z
        L.sa_quant_nvfp4_ip.argtypes = [P, P, I, I, I, I, P, I, I, I, I, P, P, P, P, P, P, P, P, P, P, P, Z, P]
        L.sa_quant_nvfp4_ip.restype = I
        _lib = L
    return _lib


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    import torch

    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _check(fn, code):
    if code != 0:
        raise SAError(fn, code)


def _tensor(name, t, dtype, ndim, shape=None):
    """Raise unless t is a contiguous CUDA tensor of dtype with ndim dims
    (and the given shape)."""
    import torch

    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name}: expected a torch.Tensor, got {type(t).__name__}")
    if t.dtype != dtype:
        raise ValueError(f"{name}: dtype {t.dtype}, expected {dtype}")
    if not t.is_cuda:
        raise ValueError(f"{name}: must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name}: must be contiguous")
    if t.dim() != ndim or (shape is not None and tuple(t.shape) != tuple(shape)):
        want = tuple(shape) if shape is not None else f"{ndim} dims"
        raise ValueError(f"{name}: shape {tuple(t.shape)}, expected {want}")


def _bf16(name, t, ndim, shape=None):
    import torch

    _tensor(name, t, torch.bfloat16, ndim, shape)


def _nvfp4(name, t, shape=None, v_layout=None):
    """Raise unless t is an NVFP4Tensor of the shape (V layout or not)."""
    if not isinstance(t, NVFP4Tensor):
        raise TypeError(f"{name}: expected an NVFP4Tensor, got {type(t).__name__}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: shape {tuple(t.shape)}, expected {tuple(shape)}")
    if v_layout is not None and (t.role == "v") != v_layout:
        raise ValueError(f"{name}: role {t.role!r} has the wrong layout here")


def _on_device(name, t):
    """Raise unless an NVFP4Tensor's buffers are in device memory."""
    for part in ("codes", "scales", "g"):
        if not getattr(t, part).is_cuda:
            raise ValueError(f"{name}.{part}: must be in device memory")


def _mode(mode):
    if mode not in SA_SCALE:
        raise ValueError(f"mode {mode!r}: expected one of {sorted(SA_SCALE)}")
    return SA_SCALE[mode]


def _role(role):
    if role not in SA_ROLE:
        raise ValueError(f"role {role!r}: expected one of {sorted(SA_ROLE)}")
    return SA_ROLE[role]


def _empty(nbytes, device, dtype=None):
    import torch

    return torch.empty(max(int(nbytes), 1), dtype=dtype or torch.uint8, device=device)


@dataclass
class NVFP4Tensor:
    """NVFP4 encoding of one [B,H,N,D] tensor (device memory).  codes and
    scales use the layouts documented in include/sa.h."""
    codes: "torch.Tensor"
    scales: "torch.Tensor"
    g: "torch.Tensor"  # float32[2] = {g, 1/g}
    role: str
    shape: tuple
    k_mean: "torch.Tensor | None" = None
    ss_off: "torch.Tensor | None" = None


def sa_device_status(reset: bool = True, stream=None) -> int:
    """Synchronise and return the library's device status word."""
    return lib().sa_device_status(_stream(stream), int(reset))


def sa_set_wait_cycles(cycles: int = 0) -> None:
    """Limit of every pipeline wait of the attention kernel in later calls,
    in SM clock cycles (0: the default, about 2 s); see include/sa.h."""
    lib().sa_set_wait_cycles(int(cycles))


def sa_quant_nvfp4(x, role: str, smooth: bool = True, mode: str = "max", f_lo: int = -2, f_hi: int = 6,
                   ss_offsets: bool = False, out: NVFP4Tensor | None = None, stream=None) -> NVFP4Tensor:
    """Quantise bf16 x [B,H,N,D] (CUDA) to NVFP4 (see include/sa.h)."""
    import torch

    _bf16("x", x, 4)
    B, H, N, D = x.shape
    r, m = _role(role), _mode(mode)
    if out is not None:
        _nvfp4("out", out, (B, H, N, D))
        if out.role != role:
            raise ValueError(f"out: role {out.role!r}, expected {role!r}")
        _on_device("out", out)
    L = lib()
    if out is None:
        codes = _empty(L.sa_codes_bytes(B, H, N, D, r), x.device)
        scales = _empty(L.sa_scales_bytes(B, H, N, D, r), x.device)
        g = torch.empty(2, dtype=torch.float32, device=x.device)
        km = torch.empty(B, H, D, dtype=torch.float32, device=x.device) if (r == 1 and smooth) else None
        nblk = B * H * N * D // 16
        off = torch.empty(max(nblk, 1), dtype=torch.int8, device=x.device) if ss_offsets else None
        out = NVFP4Tensor(codes, scales, g, role, (B, H, N, D), km, off)
    ws_bytes = L.sa_quant_workspace_size(B, H, N, D, r)
    ws = _empty(ws_bytes, x.device)
    _check("sa_quant_nvfp4",
           L.sa_quant_nvfp4(_ptr(x), B, H, N, D, r, int(smooth), m, f_lo, f_hi, _ptr(out.codes),
                            _ptr(out.scales), _ptr(out.g), _ptr(out.k_mean), _ptr(out.ss_off), _ptr(ws), ws_bytes,
                            _stream(stream)))
    return out


def sa_quant_nvfp4_qkv(q, k, v, smooth: bool = True, mode: str = "max", f_lo: int = -2, f_hi: int = 6,
                       out=None, stream=None):
    """Pre-pass of Q, K (smoothed when `smooth`) and V of one shape in two
    launches; same results as three sa_quant_nvfp4 calls.  Returns
    (NVFP4Tensor q, k, v); `out` may pass the three to reuse."""
    import torch

    _bf16("q", q, 4)
    B, H, N, D = q.shape
    _bf16("k", k, 4, (B, H, N, D))
    _bf16("v", v, 4, (B, H, N, D))
    m = _mode(mode)
    if out is not None:
        if len(out) != 3:
            raise ValueError("out: expected the (q, k, v) NVFP4Tensors of an earlier call")
        for name, t, role in (("out[0]", out[0], "q"), ("out[1]", out[1], "k"), ("out[2]", out[2], "v")):
            _nvfp4(name, t, (B, H, N, D))
            if t.role != role:
                raise ValueError(f"{name}: role {t.role!r}, expected {role!r}")
            _on_device(name, t)
        if smooth and out[1].k_mean is None:
            raise ValueError("out[1]: smoothing needs a k_mean buffer")
    L = lib()
    if out is None:
        out = []
        for role, r in (("q", 0), ("k", 1), ("v", 2)):
            codes = _empty(L.sa_codes_bytes(B, H, N, D, r), q.device)
            scales = _empty(L.sa_scales_bytes(B, H, N, D, r), q.device)
            g = torch.empty(2, dtype=torch.float32, device=q.device)
            km = torch.empty(B, H, D, dtype=torch.float32, device=q.device) if (role == "k" and smooth) else None
            out.append(NVFP4Tensor(codes, scales, g, role, (B, H, N, D), km, None))
    qt, kt, vt = out
    ws_bytes = L.sa_quant_qkv_workspace_size(B, H, N, D)
    ws = _empty(ws_bytes, q.device)
    _check("sa_quant_nvfp4_qkv",
           L.sa_quant_nvfp4_qkv(_ptr(q), _ptr(k), _ptr(v), B, H, N, D, int(smooth), m, f_lo, f_hi,
                                _ptr(qt.codes), _ptr(qt.scales), _ptr(qt.g), _ptr(kt.codes), _ptr(kt.scales),
                                _ptr(kt.g), _ptr(kt.k_mean), _ptr(vt.codes), _ptr(vt.scales), _ptr(vt.g), _ptr(ws),
                                ws_bytes, _stream(stream)))
    return qt, kt, vt


def sa_thrift_select(q, k, causal: bool, frac_bp: int = 500, stream=None):
    """(mask uint8 [B,H,T,T], nsel int32 [B,H]) on the device."""
    import torch

    _bf16("q", q, 4)
    B, H, N, D = q.shape
    _bf16("k", k, 4, (B, H, N, D))
    T = (N + 127) // 128
    L = lib()
    mask = torch.empty(B, H, T, T, dtype=torch.uint8, device=q.device)
    nsel = torch.empty(B, H, dtype=torch.int32, device=q.device)
    ws_bytes = L.sa_select_workspace_size(B, H, N, D)
    ws = _empty(ws_bytes, q.device)
    _check("sa_thrift_select", L.sa_thrift_select(_ptr(q), _ptr(k), B, H, N, D, int(causal), int(frac_bp), _ptr(mask),
                                                  _ptr(nsel), _ptr(ws), ws_bytes, _stream(stream)))
    return mask, nsel


def sa_thrift_select_ex(q, k, causal: bool, frac_bp: int = 500, per_row: bool = False, k_mean=None,
                        stream=None):
    """sa_thrift_select with a per-query-tile budget (per_row) and/or keys
    pooled after subtracting k_mean (float32 [B,H,D], device).  Returns
    (mask uint8 [B,H,T,T], nsel int32 [B,H]) on the device."""
    import torch

    _bf16("q", q, 4)
    B, H, N, D = q.shape
    _bf16("k", k, 4, (B, H, N, D))
    if k_mean is not None:
        _tensor("k_mean", k_mean, torch.float32, 3, (B, H, D))
    T = (N + 127) // 128
    L = lib()
    mask = torch.empty(B, H, T, T, dtype=torch.uint8, device=q.device)
    nsel = torch.empty(B, H, dtype=torch.int32, device=q.device)
    ws_bytes = L.sa_select_workspace_size(B, H, N, D)
    ws = _empty(ws_bytes, q.device)
    _check("sa_thrift_select_ex",
           L.sa_thrift_select_ex(_ptr(q), _ptr(k), _ptr(k_mean), B, H, N, D, int(causal), int(frac_bp),
                                 int(per_row), _ptr(mask), _ptr(nsel), _ptr(ws), ws_bytes, _stream(stream)))
    return mask, nsel


def sa_quant_nvfp4_ip(q, k, signs, smooth: bool = True, mode: str = "max", f_lo: int = -2, f_hi: int = 6,
                      ss_offsets: bool = False, stream=None):
    """Incoherence processing of bf16 q, k [B,H,N,D] (CUDA) and the NVFP4
    pre-pass of the results (include/sa.h, sa_quant_nvfp4_ip).  signs: int8
    [D] of +-1 on the same device.  Returns (Q' NVFP4Tensor, K' NVFP4Tensor,
    r FP32 [B,H,D]); both tensors use the Q/K layout (role "q" for Q', "k"
    for K', whose k_mean is the smoothing mean or None)."""
    import torch

    _bf16("q", q, 4)
    B, H, N, D = q.shape
    _bf16("k", k, 4, (B, H, N, D))
    _tensor("signs", signs, torch.int8, 1, (D,))
    m = _mode(mode)
    L = lib()
    outs = []
    for role in ("q", "k"):
        codes = _empty(L.sa_codes_bytes(B, H, N, D, 0), q.device)
        scales = _empty(L.sa_scales_bytes(B, H, N, D, 0), q.device)
        g = torch.empty(2, dtype=torch.float32, device=q.device)
        km = torch.empty(B, H, D, dtype=torch.float32, device=q.device) if (role == "k" and smooth) else None
        off = torch.empty(max(B * H * N * D // 16, 1), dtype=torch.int8, device=q.device) if ss_offsets else None
        outs.append(NVFP4Tensor(codes, scales, g, role, (B, H, N, D), km, off))
    r = torch.empty(B, H, D, dtype=torch.float32, device=q.device)
    ws_bytes = L.sa_quant_ip_workspace_size(B, H, N, D)
    ws = _empty(ws_bytes, q.device)
    oq, ok = outs
    _check("sa_quant_nvfp4_ip",
           L.sa_quant_nvfp4_ip(_ptr(q), _ptr(k), B, H, N, D, _ptr(signs), int(smooth), m, f_lo, f_hi,
                               _ptr(oq.codes), _ptr(oq.scales), _ptr(oq.g), _ptr(ok.codes), _ptr(ok.scales),
                               _ptr(ok.g), _ptr(ok.k_mean), _ptr(r), _ptr(oq.ss_off), _ptr(ok.ss_off), _ptr(ws),
                               ws_bytes, _stream(stream)))
    return oq, ok, r


def sa_attn_fwd(q: NVFP4Tensor, k: NVFP4Tensor, v: NVFP4Tensor, causal: bool, sm_scale: float = 0.0, mask=None,
                q_bf16=None, k_bf16=None, v_bf16=None, want_lse: bool = False, out=None, stream=None,
                p_mode: str = "max"):
    """FP32 attention output [B,H,N,D] (and lse [B,H,N] if asked).
    p_mode: block rule of the requantised P, "max" (max-scaling) or
    "search" (ScaleSearch; sa_attn_fwd_ex)."""
    import torch

    _nvfp4("q", q, v_layout=False)
    B, H, N, D = q.shape
    _nvfp4("k", k, (B, H, N, D), v_layout=False)
    _nvfp4("v", v, (B, H, N, D), v_layout=True)
    if mask is not None:
        T = (N + 127) // 128
        _tensor("mask", mask, torch.uint8, 4, (B, H, T, T))
        for name, t in (("q_bf16", q_bf16), ("k_bf16", k_bf16), ("v_bf16", v_bf16)):
            if t is None:
                raise ValueError(f"{name}: the bf16 blocks of a mask need the raw inputs")
            _bf16(name, t, 4, (B, H, N, D))
    if out is not None:
        _tensor("out", out, torch.float32, 4, (B, H, N, D))
    for name, t in (("q", q), ("k", k), ("v", v)):
        _on_device(name, t)
    dev = q.codes.device
    if out is None:
        out = torch.empty(B, H, N, D, dtype=torch.float32, device=dev)
    lse = torch.empty(B, H, N, dtype=torch.float32, device=dev) if want_lse else None
    km = k.k_mean if mask is not None else None
    pm = _mode(p_mode)
    if pm == 0:
        _check("sa_attn_fwd",
               lib().sa_attn_fwd(_ptr(q.codes), _ptr(q.scales), _ptr(q.g), _ptr(k.codes), _ptr(k.scales),
                                 _ptr(k.g), _ptr(v.codes), _ptr(v.scales), _ptr(v.g), B, H, N, D, int(causal),
                                 float(sm_scale), _ptr(mask), _ptr(q_bf16), _ptr(k_bf16), _ptr(v_bf16), _ptr(km),
                                 _ptr(out), _ptr(lse), _stream(stream)))
    else:
        _check("sa_attn_fwd_ex",
               lib().sa_attn_fwd_ex(_ptr(q.codes), _ptr(q.scales), _ptr(q.g), _ptr(k.codes), _ptr(k.scales),
                                    _ptr(k.g), _ptr(v.codes), _ptr(v.scales), _ptr(v.g), B, H, N, D, int(causal),
                                    float(sm_scale), pm, _ptr(mask), _ptr(q_bf16), _ptr(k_bf16), _ptr(v_bf16),
                                    _ptr(km), _ptr(out), _ptr(lse), _stream(stream)))
    return (out, lse) if want_lse else out


def sa_attn_decode_kvfp4(q, k: NVFP4Tensor, v: NVFP4Tensor, sm_scale: float = 0.0, out=None, stream=None,
                         sink_tiles=(0, 0), k_sink=None, v_sink=None):
    """q bf16 [B,Hq,D]; caches quantised as [B,Hkv,L,D]; returns FP32 [B,Hq,D].
    sink_tiles = (first, last) keeps that many 128-key tiles at each end of
    the cache at full precision (sa_attn_decode_kvfp4_sink); k_sink, v_sink
    are then bf16 [B,Hkv,128 (first + last),D] holding those tiles, and the
    channel means of k (k.k_mean) offset their keys."""
    import torch

    _bf16("q", q, 3)
    B, Hq, D = q.shape
    _nvfp4("k", k, v_layout=False)
    _, Hkv, Lk, _ = k.shape
    if k.shape[0] != B or k.shape[3] != D:
        raise ValueError(f"k: shape {tuple(k.shape)} does not match q {tuple(q.shape)}")
    _nvfp4("v", v, tuple(k.shape), v_layout=True)
    if out is not None:
        _tensor("out", out, torch.float32, 3, (B, Hq, D))
    _on_device("k", k)
    _on_device("v", v)
    first, last = (int(t) for t in sink_tiles)
    if first < 0 or last < 0:
        raise ValueError(f"sink_tiles: {sink_tiles}")
    if first or last:
        ns = 128 * (first + last)
        _bf16("k_sink", k_sink, 4, (B, Hkv, ns, D))
        _bf16("v_sink", v_sink, 4, (B, Hkv, ns, D))
    L = lib()
    if out is None:
        out = torch.empty(B, Hq, D, dtype=torch.float32, device=q.device)
    ws_bytes = L.sa_decode_workspace_size(B, Hq, Hkv, Lk, D)
    ws = _empty(ws_bytes, q.device)
    if first or last:
        _check("sa_attn_decode_kvfp4_sink",
               L.sa_attn_decode_kvfp4_sink(_ptr(q), _ptr(k.codes), _ptr(k.scales), _ptr(k.g), _ptr(v.codes),
                                           _ptr(v.scales), _ptr(v.g), B, Hq, Hkv, Lk, D, float(sm_scale), first, last,
                                           _ptr(k_sink), _ptr(v_sink), _ptr(k.k_mean), _ptr(out), _ptr(ws), ws_bytes,
                                           _stream(stream)))
    else:
        _check("sa_attn_decode_kvfp4",
               L.sa_attn_decode_kvfp4(_ptr(q), _ptr(k.codes), _ptr(k.scales), _ptr(k.g), _ptr(v.codes),
                                      _ptr(v.scales), _ptr(v.g), B, Hq, Hkv, Lk, D, float(sm_scale), _ptr(out),
                                      _ptr(ws), ws_bytes, _stream(stream)))
    return out


def sink_tiles_of(x, first: int, last: int):
    """The compact full-precision copy that sa_attn_decode_kvfp4 takes for
    sink_tiles = (first, last): the first `first` and the last `last`
    128-key tiles of a [B,Hkv,L,D] cache, concatenated along the keys."""
    import torch

    L = x.shape[2]
    parts = [x[:, :, : 128 * first]] if first else []
    if last:
        parts.append(x[:, :, L - 128 * last:])
    return torch.cat(parts, dim=2).contiguous()


# --------------------------------------------------------------------- layouts
def codes_to_logical(codes, B: int, H: int, N: int, D: int, role: str):
    """Codes in the logical row-major layout: [B,H,N,D/2] for Q/K (already
    so stored) and [B,H,D,N/2] for V, whose storage is 128-token tiles
    [B,H,ceil(N/128),D,64] (include/sa.h).  Pure index permutation."""
    if role != "v":
        return codes.reshape(B, H, N, D // 2)
    NT = (N + 127) // 128
    a = codes.reshape(B, H, NT, D, 64).permute(0, 1, 3, 2, 4) if hasattr(codes, "permute") else \
        codes.reshape(B, H, NT, D, 64).transpose(0, 1, 3, 2, 4)
    a = a.reshape(B, H, D, NT * 64)[:, :, :, : N // 2]
    return a.contiguous() if hasattr(a, "contiguous") else a


def scales_to_logical(scales, B: int, H: int, N: int, D: int, role: str):
    """Unpack the tensor-core atom layout of scale bytes (include/sa.h) into
    the logical row-major [B,H,R,C/16] layout (R, C = N, D for Q/K and D, N for
    V).  Pure index permutation, host or device tensors."""
    import torch

    R, C = (D, N) if role == "v" else (N, D)
    RT, CK = math.ceil(R / 128), math.ceil(C / 64)
    a = scales.reshape(B * H, RT, CK, 32, 4, 4)  # [bh, rt, ck, r%32, r/32, j]
    a = a.permute(0, 1, 4, 3, 2, 5)  # [bh, rt, r/32, r%32, ck, j]
    a = a.reshape(B * H, RT * 128, CK * 4)[:, :R, : C // 16]
    return a.reshape(B, H, R, C // 16).contiguous() if isinstance(a, torch.Tensor) else a
