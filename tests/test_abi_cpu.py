"""C-ABI checks that need no GPU: libsa.so builds, loads, exports every
function that include/sa.h declares, sizes its buffers as documented, and
rejects bad arguments before launching anything."""
import ctypes
import os
import re

import pytest

import bit_quantized_attention_channel_b200 as sa
from bit_quantized_attention_channel_b200 import build as sabuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    sabuild.build()
    return sa.lib()


def declared_functions():
    hdr = open(os.path.join(ROOT, "include", "sa.h")).read()
    hdr = re.sub(r"/\*.*?\*/", "", hdr, flags=re.S)
    return sorted(set(re.findall(r"\b(sa_[a-z0-9_]+)\s*\(", hdr)))


def test_exports_every_declared_symbol(L):
    names = declared_functions()
    assert len(names) >= 10
    for n in names:
        assert hasattr(L, n), n


def test_status_strings(L):
    for i, name in enumerate(sa.STATUS):
        assert L.sa_status_string(i).decode() == name


def test_buffer_sizes(L):
    # Q/K: codes B*H*N*D/2; scales: 512-byte atoms per (128 rows, 64 columns)
    assert L.sa_codes_bytes(2, 16, 4096, 128, 0) == 2 * 16 * 4096 * 64
    # V codes are stored in whole 128-token tiles
    assert L.sa_codes_bytes(2, 16, 4096, 128, 2) == 2 * 16 * 32 * 128 * 64
    assert L.sa_codes_bytes(1, 1, 416, 64, 2) == 4 * 64 * 64
    assert L.sa_scales_bytes(2, 16, 4096, 128, 0) == 2 * 16 * 32 * 2 * 512
    # ragged N rounds the row tiles up
    assert L.sa_scales_bytes(1, 1, 400, 64, 1) == 4 * 1 * 512
    # V: rows are channels (one 128-row tile for D <= 128), chunks along tokens
    assert L.sa_scales_bytes(1, 2, 4096, 128, 2) == 2 * 1 * 64 * 512
    assert L.sa_scales_bytes(1, 1, 400, 64, 2) == 1 * 1 * 7 * 512
    assert L.sa_quant_workspace_size(1, 1, 256, 64, 0) == 256
    assert L.sa_quant_workspace_size(1, 1, 256, 64, 1) > 256


def test_rejects_bad_arguments_before_launch(L):
    n = None
    # unsupported head dim
    assert L.sa_quant_nvfp4(n, 1, 1, 128, 96, 0, 0, 0, -2, 6, n, n, n, n, n, n, 0, n) == 2
    # N not a multiple of 16
    assert L.sa_quant_nvfp4(n, 1, 1, 100, 64, 0, 0, 0, -2, 6, n, n, n, n, n, n, 0, n) == 1
    # bad ScaleSearch range
    assert L.sa_quant_nvfp4(n, 1, 1, 128, 64, 0, 0, 1, 1, 6, n, n, n, n, n, n, 0, n) == 1
    # empty tensor: valid, nothing launched
    assert L.sa_quant_nvfp4(n, 0, 1, 128, 64, 0, 0, 0, -2, 6, n, n, n, n, n, n, 0, n) == 0
    # null buffers
    assert L.sa_quant_nvfp4(n, 1, 1, 128, 64, 0, 0, 0, -2, 6, n, n, n, n, n, n, 0, n) == 1
    # attention: N % 32, unsupported D, null pointers
    assert L.sa_attn_fwd(*([n] * 9), 1, 1, 48, 64, 0, 0.0, *([n] * 8)) == 1
    assert L.sa_attn_fwd(*([n] * 9), 1, 1, 64, 80, 0, 0.0, *([n] * 8)) == 2
    assert L.sa_attn_fwd(*([n] * 9), 1, 1, 64, 64, 0, 0.0, *([n] * 8)) == 1
    # decode: Hq % Hkv, L % 128
    assert L.sa_attn_decode_kvfp4(*([n] * 7), 1, 6, 4, 256, 128, 0.0, n, n, 0, n) == 1
    assert L.sa_attn_decode_kvfp4(*([n] * 7), 1, 8, 2, 200, 128, 0.0, n, n, 0, n) == 1
    # selector: budget out of range
    assert L.sa_thrift_select(n, n, 1, 1, 256, 64, 1, 20000, n, n, n, 0, n) == 1


def test_new_entry_points_reject_bad_arguments_before_launch(L):
    n = None
    # attention with a P block rule: unknown mode; ScaleSearch on P with a bf16 block mask
    assert L.sa_attn_fwd_ex(*([n] * 9), 1, 1, 64, 64, 0, 0.0, 7, *([n] * 8)) == 1
    mask = ctypes.c_void_p(16)  # never dereferenced: the call returns first
    assert L.sa_attn_fwd_ex(*([n] * 9), 1, 1, 64, 64, 0, 0.0, 1, mask, *([n] * 7)) == 2
    # sink decode: negative counts, more sink tiles than the cache holds, missing sink buffers
    dec = [n] * 7
    assert L.sa_attn_decode_kvfp4_sink(*dec, 1, 8, 2, 256, 128, 0.0, -1, 0, n, n, n, n, n, 0, n) == 1
    assert L.sa_attn_decode_kvfp4_sink(*dec, 1, 8, 2, 256, 128, 0.0, 2, 1, n, n, n, n, n, 0, n) == 1
    assert L.sa_attn_decode_kvfp4_sink(*dec, 1, 8, 2, 256, 128, 0.0, 1, 1, n, n, n, n, n, 0, n) == 1
    # sink decode with (0, 0) and no work is the plain call's empty case
    assert L.sa_attn_decode_kvfp4_sink(*dec, 0, 8, 2, 256, 128, 0.0, 0, 0, n, n, n, n, n, 0, n) == 0
    # incoherence pre-pass: unsupported D, N % 16, bad ScaleSearch range, null signs
    assert L.sa_quant_nvfp4_ip(n, n, 1, 1, 128, 96, n, 1, 0, -2, 6, *([n] * 11), 0, n) == 2
    assert L.sa_quant_nvfp4_ip(n, n, 1, 1, 100, 64, n, 1, 0, -2, 6, *([n] * 11), 0, n) == 1
    assert L.sa_quant_nvfp4_ip(n, n, 1, 1, 128, 64, n, 1, 1, 1, 6, *([n] * 11), 0, n) == 1
    assert L.sa_quant_nvfp4_ip(n, n, 1, 1, 128, 64, n, 1, 0, -2, 6, *([n] * 11), 0, n) == 1
    assert L.sa_quant_ip_workspace_size(1, 2, 256, 128) > L.sa_quant_workspace_size(1, 2, 256, 128, 1)
    # selector variants: per-row budget out of range
    assert L.sa_thrift_select_ex(n, n, n, 1, 1, 256, 64, 1, -1, 1, n, n, n, 0, n) == 1


def test_scales_to_logical_roundtrip():
    import numpy as np
    import torch

    B, H, N, D = 1, 2, 400, 64
    R, C = N, D
    logical = torch.randint(0, 127, (B, H, R, C // 16), dtype=torch.uint8)
    RT, CK = (R + 127) // 128, (C + 63) // 64
    atoms = torch.zeros(B * H * RT * CK * 512, dtype=torch.uint8)
    for bh in range(B * H):
        for r in range(R):
            for j in range(C // 16):
                a = (bh * RT + r // 128) * CK + j // 4
                atoms[a * 512 + (r % 32) * 16 + ((r % 128) // 32) * 4 + j % 4] = logical.view(B * H, R, -1)[bh, r, j]
    back = sa.scales_to_logical(atoms, B, H, N, D, "q")
    assert torch.equal(back, logical)


def test_v_codes_to_logical_roundtrip():
    """V codes are stored as 128-token tiles [B,H,ceil(N/128),D,64]; the
    logical view is [B,H,D,N/2] (channel rows, token pairs)."""
    import torch

    B, H, N, D = 2, 3, 416, 64
    NT = (N + 127) // 128
    logical = torch.randint(0, 256, (B, H, D, N // 2), dtype=torch.uint8)
    tiled = torch.full((B, H, NT, D, 64), 0xEE, dtype=torch.uint8)  # padding is never read back
    for t in range(NT):
        w = min(64, N // 2 - 64 * t)
        tiled[:, :, t, :, :w] = logical[:, :, :, 64 * t: 64 * t + w]
    back = sa.codes_to_logical(tiled.reshape(-1), B, H, N, D, "v")
    assert torch.equal(back, logical)
    # byte address of (channel d, token n) in the stored layout
    d, n = 37, 300
    flat = tiled.reshape(-1)
    assert flat[((1 * H + 2) * NT + n // 128) * D * 64 + d * 64 + (n % 128) // 2] == logical[1, 2, d, n // 2]


def test_fused_prepass_rejects_bad_arguments(L):
    n = None
    ws = L.sa_quant_qkv_workspace_size(1, 2, 256, 128)
    assert ws >= 256 + 2 * 2 * 128 * (8 + 4 + 4) + 2 * 128 * 4
    # D unsupported, N not a multiple of 16, bad mode, null pointers: before any launch
    assert L.sa_quant_nvfp4_qkv(n, n, n, 1, 1, 256, 96, 1, 0, -2, 6, *([n] * 10), n, 0, n) == 2
    assert L.sa_quant_nvfp4_qkv(n, n, n, 1, 1, 250, 128, 1, 0, -2, 6, *([n] * 10), n, 0, n) == 1
    assert L.sa_quant_nvfp4_qkv(n, n, n, 1, 1, 256, 128, 1, 7, -2, 6, *([n] * 10), n, 0, n) == 1
    assert L.sa_quant_nvfp4_qkv(n, n, n, 1, 1, 256, 128, 1, 0, -2, 6, *([n] * 10), n, 0, n) == 1
    # empty call
    assert L.sa_quant_nvfp4_qkv(n, n, n, 0, 1, 256, 128, 1, 0, -2, 6, *([n] * 10), n, 0, n) == 0


def test_binding_validates_arguments_before_any_launch():
    """The Python binding rejects host tensors, wrong dtypes, shapes, roles,
    modes and masks with ValueError/TypeError before it loads a stream or
    calls the library, so no host pointer ever reaches a kernel."""
    import torch

    x = torch.zeros(1, 2, 128, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="CUDA"):
        sa.sa_quant_nvfp4(x, "q")
    with pytest.raises(ValueError, match="dtype"):
        sa.sa_quant_nvfp4(x.float(), "q")
    with pytest.raises(TypeError):
        sa.sa_quant_nvfp4(x.numpy(), "q")
    with pytest.raises(ValueError, match="CUDA"):
        sa.sa_quant_nvfp4_qkv(x, x, x)
    with pytest.raises(ValueError, match="CUDA"):
        sa.sa_thrift_select(x, x, True)
    with pytest.raises(ValueError, match="CUDA"):
        sa.sa_attn_decode_kvfp4(x[0], None, None)
    with pytest.raises(ValueError, match="mode"):
        sa._mode("maximum")
    with pytest.raises(ValueError, match="role"):
        sa._role("o")
    with pytest.raises(ValueError, match="CUDA"):
        sa._bf16("k", x, 4, (1, 2, 128, 128))      # device before shape

    def fake(role, shape=(1, 2, 128, 64)):
        b = torch.zeros(16, dtype=torch.uint8)
        return sa.NVFP4Tensor(b, b, torch.ones(2), role, shape)

    q, k, v = fake("q"), fake("k"), fake("v")
    with pytest.raises(ValueError, match="layout"):
        sa.sa_attn_fwd(q, k, fake("q"), True)        # V must carry the V layout
    with pytest.raises(ValueError, match="layout"):
        sa.sa_attn_fwd(fake("v"), k, v, True)
    with pytest.raises(ValueError, match="shape"):
        sa.sa_attn_fwd(q, fake("k", (1, 2, 256, 64)), v, True)
    with pytest.raises(TypeError):
        sa.sa_attn_fwd(q, k, "v", True)
    with pytest.raises(ValueError, match="device memory"):
        sa.sa_attn_fwd(q, k, v, True)                # host buffers never reach the library
    with pytest.raises(ValueError, match="mask"):
        sa.sa_attn_fwd(q, k, v, True, mask=torch.zeros(1, 2, 2, 2, dtype=torch.int32))


def test_empty_calls_are_valid_and_launch_nothing(L):
    """B = 0 or H = 0 is a valid empty call for every entry point: SA_OK, with
    null buffers and no CUDA work (this host has no GPU)."""
    n = None
    assert L.sa_quant_nvfp4(n, 0, 1, 128, 64, 0, 0, 0, -2, 6, n, n, n, n, n, n, 0, n) == 0
    assert L.sa_quant_nvfp4_qkv(n, n, n, 0, 1, 256, 128, 1, 0, -2, 6, *([n] * 10), n, 0, n) == 0
    assert L.sa_attn_fwd(*([n] * 9), 0, 1, 128, 64, 0, 0.0, *([n] * 8)) == 0
    assert L.sa_attn_fwd(*([n] * 9), 1, 0, 128, 64, 1, 0.0, *([n] * 8)) == 0
    assert L.sa_attn_decode_kvfp4(*([n] * 7), 0, 8, 2, 256, 128, 0.0, n, n, 0, n) == 0
    assert L.sa_thrift_select(n, n, 0, 1, 256, 64, 1, 500, n, n, n, 0, n) == 0
