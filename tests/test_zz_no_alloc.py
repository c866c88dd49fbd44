"""GPU test of octo_decode_attn_static, the decode step for callers that
cannot allocate device memory (their host framework owns every device
allocation, or their allocator is out of reach of the code that issues the
decode). The entry point uses a fixed scratch array inside the library
instead of a caller-provided workspace; its results must match
octo_decode_attn's, call after call.

This file is collected last on purpose, and passes both alone and after the
other GPU tests (the shared scratch keeps the previous call's contents, so
each call clears what must start at zero).
"""

import ctypes
import math

import numpy as np
import pytest
import torch

from oracle import tables
from rotation_preconditioned_quantization_b200 import _lib, api, inputs

from . import parity

pytestmark = pytest.mark.gpu


def _static_call(lay, dev, q, cache, V, Hkv, out, logits):
    B, Hq, Lq, d = q.shape
    return _lib.lib().octo_decode_attn_static(
        lay.ref, dev.ref, q.data_ptr(), _lib.BF16, B, Hq, Hkv, Lq, cache.length, cache.cap,
        cache.packed.data_ptr(), cache.gamma.data_ptr(), None, None, V.data_ptr(), ctypes.c_float(1.0 / math.sqrt(d)),
        out.data_ptr(), logits.data_ptr(), torch.cuda.current_stream().cuda_stream)


@pytest.mark.parametrize("B,Hq,Hkv,N", [(1, 8, 2, 5000), (2, 32, 8, 20000)])
def test_static_scratch_matches_workspace_entry_point(cuda_ok, B, Hq, Hkv, N):
    d, b = 128, 3
    lay = api.Layout(d, b)
    dev = api.DeviceTables(*parity.oracle_tables(d, b), tables.rotation_signs(0, d, Hkv))
    keys = torch.from_numpy(inputs.to_bf16(inputs.llm_keys(1, B * Hkv, N, d))).to(torch.bfloat16).cuda()
    V = torch.from_numpy(inputs.to_bf16(inputs.normal(2, (B * Hkv, N, d)))).to(torch.bfloat16).cuda()
    q = torch.from_numpy(inputs.to_bf16(inputs.normal(3, (B, Hq, 1, d)))).to(torch.bfloat16).cuda()
    cache = api.Cache.empty(lay, B * Hkv, N)
    api.encode(lay, dev, keys, cache)
    ref, ref_lg = api.decode_attn(lay, dev, q, cache, V, Hkv, logits=True)
    torch.cuda.synchronize()
    ref = ref.cpu().numpy()
    tol = 2e-3 * np.max(np.abs(ref), axis=-1, keepdims=True)
    for call in range(2):  # the scratch keeps the previous call's contents
        out = torch.full((B, Hq, 1, d), float("nan"), device="cuda")
        lg = torch.full((B, Hq, 1, N), float("nan"), device="cuda")
        assert _static_call(lay, dev, q, cache, V, Hkv, out, lg) == _lib.OCTO_OK
        torch.cuda.synchronize()
        assert _status() == 0  # no bounded on-chip wait expired
        got = out.cpu().numpy()
        assert np.all(np.abs(got - ref) <= tol), f"call {call}: max err {np.max(np.abs(got - ref))}"
        assert torch.allclose(lg, ref_lg, rtol=0, atol=1e-4 * float(ref_lg.abs().max()))


def _status():
    st = ctypes.c_int(-1)
    assert _lib.lib().octo_decode_attn_static_status(ctypes.byref(st), torch.cuda.current_stream().cuda_stream) == 0
    return st.value


def test_static_scratch_cleared_after_garbage_and_a_wider_call(cuda_ok):
    """Each call must clear the status word and arrival counters itself: the
    array is filled with 0xff bytes (what an interrupted call could leave:
    a set status bit, counters far from zero) before the first call, and a
    call over more cache heads precedes one over fewer, so the narrower
    call's counters sit where the wider call's were. Without the clearing
    the ticket never reaches the last split and the outputs stay NaN, or the
    status word reads nonzero."""
    d, b = 128, 3
    lay = api.Layout(d, b)
    shapes = [(2, 32, 8, 24000), (1, 8, 2, 9000)]  # wider first, then narrower
    Hkv_max = 8
    dev = api.DeviceTables(*parity.oracle_tables(d, b), tables.rotation_signs(0, d, Hkv_max))
    assert _lib.lib().octo_decode_attn_static_fill(0xFF, torch.cuda.current_stream().cuda_stream) == 0
    torch.cuda.synchronize()
    assert _status() == -1  # every byte 0xff
    for B, Hq, Hkv, N in shapes:
        keys = torch.from_numpy(inputs.to_bf16(inputs.llm_keys(5, B * Hkv, N, d))).to(torch.bfloat16).cuda()
        V = torch.from_numpy(inputs.to_bf16(inputs.normal(6, (B * Hkv, N, d)))).to(torch.bfloat16).cuda()
        q = torch.from_numpy(inputs.to_bf16(inputs.normal(7, (B, Hq, 1, d)))).to(torch.bfloat16).cuda()
        cache = api.Cache.empty(lay, B * Hkv, N)
        api.encode(lay, dev, keys, cache)
        ref, ref_lg = api.decode_attn(lay, dev, q, cache, V, Hkv, logits=True)
        torch.cuda.synchronize()
        ref = ref.cpu().numpy()
        out = torch.full((B, Hq, 1, d), float("nan"), device="cuda")
        lg = torch.full((B, Hq, 1, N), float("nan"), device="cuda")
        assert _static_call(lay, dev, q, cache, V, Hkv, out, lg) == _lib.OCTO_OK
        torch.cuda.synchronize()
        assert _status() == 0
        got = out.cpu().numpy()
        tol = 2e-3 * np.max(np.abs(ref), axis=-1, keepdims=True)
        assert np.all(np.abs(got - ref) <= tol), f"{(B, Hq, Hkv, N)}: max err {np.nanmax(np.abs(got - ref))}"
        assert torch.allclose(lg, ref_lg, rtol=0, atol=1e-4 * float(ref_lg.abs().max()))


def test_static_scratch_rejects_sizes_beyond_its_maximum(cuda_ok):
    lay = api.Layout(128, 3)
    # the smallest batch (of 8 KV heads, 8 query rows each, 131072 tokens) whose workspace is over the limit
    B = next(b for b in (8, 64, 512, 4096) if api.decode_attn_workspace_bytes(lay, b, 64, 8, 1, 131072) > 8 << 20)
    t = _lib.OctoTables(256, 256, 256, 256, 256, None, 8)
    st = _lib.lib().octo_decode_attn_static(lay.ref, ctypes.byref(t), 256, _lib.BF16, B, 64, 8, 1, 131072, 131072,
                                            256, 256, None, None, 256, ctypes.c_float(0.1), 256, None, None)
    assert st == _lib.OCTO_EWORKSPACE
