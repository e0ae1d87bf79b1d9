"""sa_quant_nvfp4_noalloc through the C ABI: for callers that cannot allocate
device memory (pool-owned memory, plug-ins without an allocator, loops that
must not synchronise the device), the pre-pass runs on scratch that lives
inside the library.  Its results must equal those of sa_quant_nvfp4 (which
takes a caller workspace) bit for bit, on two calls in a row (the scratch keeps
the previous call's contents, so the second call checks that the call clears
what must start at zero).  Kept in a file of its own, collected last."""
import ctypes

import pytest
import torch

import bit_quantized_attention_channel_b200 as sa
from bit_quantized_attention_channel_b200 import workloads as wl

pytestmark = pytest.mark.gpu


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _noalloc(x, role, smooth, mode):
    L = sa.lib()
    B, H, N, D = x.shape
    r = sa.SA_ROLE[role]
    codes = torch.empty(L.sa_codes_bytes(B, H, N, D, r), dtype=torch.uint8, device=x.device)
    scales = torch.empty(L.sa_scales_bytes(B, H, N, D, r), dtype=torch.uint8, device=x.device)
    g = torch.empty(2, dtype=torch.float32, device=x.device)
    km = torch.empty(B, H, D, dtype=torch.float32, device=x.device) if (role == "k" and smooth) else None
    off = torch.empty(B * H * N * D // 16, dtype=torch.int8, device=x.device)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    rc = L.sa_quant_nvfp4_noalloc(_p(x), B, H, N, D, r, int(smooth), sa.SA_SCALE[mode], -2, 6, _p(codes), _p(scales),
                                  _p(g), _p(km), _p(off), stream)
    assert rc == 0, sa.STATUS[rc]
    assert sa.sa_device_status(reset=True) == 0
    return codes, scales, g, km, off


def _same(a, b):
    return torch.equal(a.cpu(), b.cpu())


def test_noalloc_matches_workspace_entry_point_on_two_calls():
    q, k, _ = wl.prefill_inputs("llm", H=4)
    small = (q[:, :2] * 0.25).contiguous()  # smaller amax than the first call's tensor
    cases = [(k.cuda(), "k", True, "search"), (small.cuda(), "q", True, "max")]
    for x, role, smooth, mode in cases:
        codes, scales, g, km, off = _noalloc(x, role, smooth, mode)
        ref = sa.sa_quant_nvfp4(x, role, smooth=smooth, mode=mode, ss_offsets=True)
        assert sa.sa_device_status(reset=True) == 0
        assert _same(codes, ref.codes) and _same(scales, ref.scales) and _same(g, ref.g)
        assert _same(off, ref.ss_off)
        if km is not None:
            assert _same(km, ref.k_mean)


def test_noalloc_rejects_sizes_beyond_its_scratch():
    """A K pre-pass whose statistics do not fit the 8 MiB scratch is refused
    before anything is launched (null pointers are never touched)."""
    L = sa.lib()
    n = None
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    rc = L.sa_quant_nvfp4_noalloc(n, 1, 32, 65536, 128, 1, 1, 0, -2, 6, n, n, n, n, n, stream)
    assert rc == 3  # SA_ERR_WORKSPACE
