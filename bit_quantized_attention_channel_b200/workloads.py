"""Seeded synthetic inputs shaped like the pages' workloads.

This module holds no arithmetic of the method; it only draws random tensors.
Both the CUDA path (tests, bench) and the CPU oracle (tests) are fed from it.

Recipe (NumPy ``default_rng(seed)``, PCG64, seed 0 unless stated):
  * draw order Q, K, per-channel K offset, V, then (long-context case) the
    attention-sink key positions;
  * Gaussian draws are float32 ``standard_normal``; Student-t draws are
    ``standard_t(4)`` divided by sqrt(2) (unit variance), cast to float32;
  * the K offset has shape [H, D] (shared by batch and tokens) and is added
    before the bf16 cast; the sink case multiplies whole K rows at
    ceil(0.01 N) distinct positions (shared by all heads) by 8;
  * every tensor is cast to bf16 with round-to-nearest-even (torch).
Large tensors are drawn in row chunks; NumPy's generators consume the stream
element by element, so chunking does not change the values.

Stand-ins for the pages' workloads (none of which is in this container):
  tiny       -- the small parity case;
  llm        -- LLM prefill (Llama/Qwen-style shapes) with K channel outliers;
  video      -- video-DiT-shaped 32K non-causal attention (Mochi/CogVideoX);
  decode     -- 4-bit KV-cache decode with grouped-query heads;
  longctx    -- long-context causal prefill with attention-sink keys
                (ThriftAttention's long-context setting).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np

CHUNK = 1 << 24  # elements per draw


@dataclass(frozen=True)
class Workload:
    name: str
    kind: str  # "prefill" or "decode"
    B: int
    H: int
    N: int
    D: int
    causal: bool = False
    dist: str = "normal"  # or "student_t4"
    k_offset_std: float = 0.0
    sink_frac: float = 0.0
    sink_scale: float = 1.0
    Hkv: int = 0  # decode only
    scale_modes: tuple = ("max",)
    thrift_bp: int = 0  # selector budget in basis points (0 = off)
    description: str = ""
    extra: dict = field(default_factory=dict)

    def flops(self) -> float:
        """4 * B * H * N^2 * D, halved when causal (prefill only)."""
        f = 4.0 * self.B * self.H * self.N * self.N * self.D
        return f / 2 if self.causal else f


WORKLOADS = {
    "tiny": Workload("tiny", "prefill", B=1, H=2, N=256, D=64, causal=False, k_offset_std=3.0,
                     description="Tiny NVFP4 attention forward B1 H2 N256 D64, non-causal, max-scaling"),
    "llm": Workload("llm", "prefill", B=2, H=16, N=4096, D=128, causal=True, k_offset_std=3.0,
                    scale_modes=("max", "search"),
                    description="LLM prefill B2 H16 N4096 D128 causal, K offset N(0,3^2), smoothing on"),
    "video": Workload("video", "prefill", B=1, H=24, N=32768, D=128, causal=False, dist="student_t4",
                      k_offset_std=2.0, scale_modes=("search",),
                      description="Video-DiT long non-causal B1 H24 N32768 D128, Student-t(4), ScaleSearch"),
    "decode": Workload("decode", "decode", B=32, H=32, N=32768, D=128, Hkv=8, k_offset_std=3.0,
                       description="Decode over NVFP4 KV cache B32 Hq32 Hkv8 L32768 D128, 1 query token"),
    "longctx": Workload("longctx", "prefill", B=1, H=32, N=65536, D=128, causal=True, sink_frac=0.01,
                        sink_scale=8.0, thrift_bp=500,
                        description="Mixed-precision long-context B1 H32 N65536 D128 causal, 1% sink keys x8, "
                                    "top 5% blocks in bf16"),
}


def _draw(rng: np.random.Generator, shape, dist: str) -> np.ndarray:
    n = int(np.prod(shape))
    out = np.empty(n, dtype=np.float32)
    for s in range(0, n, CHUNK):
        e = min(n, s + CHUNK)
        if dist == "normal":
            out[s:e] = rng.standard_normal(e - s, dtype=np.float32)
        elif dist == "student_t4":
            out[s:e] = (rng.standard_t(4, e - s) / math.sqrt(2.0)).astype(np.float32)
        else:
            raise ValueError(dist)
    return out.reshape(shape)


def _to_bf16(a: np.ndarray):
    import torch

    return torch.from_numpy(a).to(torch.bfloat16)


def prefill_inputs(w: Workload | str, seed: int = 0, B=None, H=None, N=None, D=None):
    """(q, k, v) bf16 CPU tensors [B,H,N,D] for a prefill workload.  Shape
    overrides give smaller cases with the same distribution."""
    if isinstance(w, str):
        w = WORKLOADS[w]
    B = w.B if B is None else B
    H = w.H if H is None else H
    N = w.N if N is None else N
    D = w.D if D is None else D
    rng = np.random.default_rng(seed)
    q = _draw(rng, (B, H, N, D), w.dist)
    k = _draw(rng, (B, H, N, D), w.dist)
    if w.k_offset_std:
        off = (rng.standard_normal((H, D), dtype=np.float32) * np.float32(w.k_offset_std)).astype(np.float32)
        k += off[None, :, None, :]
    v = _draw(rng, (B, H, N, D), w.dist)
    if w.sink_frac:
        pos = rng.choice(N, int(math.ceil(w.sink_frac * N)), replace=False)
        k[:, :, pos, :] *= np.float32(w.sink_scale)
    return _to_bf16(q), _to_bf16(k), _to_bf16(v)


def decode_inputs(w: Workload | str = "decode", seed: int = 0, B=None, Hq=None, Hkv=None, L=None, D=None):
    """(q [B,Hq,D], k_cache [B,Hkv,L,D], v_cache [B,Hkv,L,D]) bf16 CPU tensors."""
    if isinstance(w, str):
        w = WORKLOADS[w]
    B = w.B if B is None else B
    Hq = w.H if Hq is None else Hq
    Hkv = w.Hkv if Hkv is None else Hkv
    L = w.N if L is None else L
    D = w.D if D is None else D
    rng = np.random.default_rng(seed)
    q = _draw(rng, (B, Hq, D), w.dist)
    k = _draw(rng, (B, Hkv, L, D), w.dist)
    if w.k_offset_std:
        off = (rng.standard_normal((Hkv, D), dtype=np.float32) * np.float32(w.k_offset_std)).astype(np.float32)
        k += off[None, :, None, :]
    v = _draw(rng, (B, Hkv, L, D), w.dist)
    return _to_bf16(q), _to_bf16(k), _to_bf16(v)
