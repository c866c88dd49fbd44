"""CPU tests of the Python binding's argument checks: shapes and devices that
the C ABI cannot see through plain pointers are refused with ValueError
before any library call (a wrong V row count or a cache with fewer heads
would otherwise make the kernels read past the end of a buffer)."""

import numpy as np
import pytest
import torch

from oracle import tables
from rotation_preconditioned_quantization_b200 import api


def _tabs(lay, n_heads, device="cpu", qjl=False):
    tb = tables.as_f32(*tables.codebooks(lay.d, lay.b))
    S = tables.qjl_matrix(1, lay.d, n_heads) if qjl else None
    return api.DeviceTables(*tb, tables.rotation_signs(0, lay.d, n_heads), S, device=device)


def test_encode_refuses_more_heads_than_the_cache():
    lay = api.Layout(64, 3)
    cache = api.Cache.empty(lay, 2, 16, device="cpu")
    keys = torch.zeros((3, 8, 64))
    with pytest.raises(ValueError, match="heads"):
        api.encode(lay, _tabs(lay, 2), keys, cache, 0)


def test_encode_refuses_a_cache_of_another_layout():
    cache = api.Cache.empty(api.Layout(128, 2), 1, 16, device="cpu")   # 9 words per key
    lay = api.Layout(128, 4)                                           # 17 words per key
    with pytest.raises(ValueError, match="packed"):
        api.encode(lay, _tabs(lay, 1), torch.zeros((1, 8, 128)), cache, 0)


def test_qjl_layout_needs_sketch_planes_and_projections():
    lay = api.Layout(128, 4, qjl=True)
    plain = api.Cache.empty(api.Layout(128, 4), 1, 16, device="cpu")
    with pytest.raises(ValueError, match="sketch"):
        api.encode(lay, _tabs(lay, 1, qjl=True), torch.zeros((1, 8, 128)), plain, 0)
    full = api.Cache.empty(lay, 1, 16, device="cpu")
    with pytest.raises(ValueError, match="qjl_S"):
        api.encode(lay, _tabs(lay, 1, qjl=False), torch.zeros((1, 8, 128)), full, 0)


def test_tables_on_another_device_are_refused():
    lay = api.Layout(64, 2)
    cache = api.Cache.empty(lay, 1, 16, device="cpu")
    cache.length = 16
    with pytest.raises(ValueError, match="device"):
        api.dequant(lay, _tabs(lay, 1, device="meta"), cache)
    with pytest.raises(ValueError, match="device"):
        api.encode(lay, _tabs(lay, 1), torch.zeros((1, 8, 64), device="meta"), cache, 0)


def _decode_args(B=1, Hq=4, Hkv=2, N=30, d=64):
    lay = api.Layout(d, 2)
    cache = api.Cache.empty(lay, B * Hkv, N, device="cpu")             # capacity rounds up to 32
    cache.length = N
    q = torch.zeros((B, Hq, 1, d), dtype=torch.bfloat16)
    V = torch.zeros((B * Hkv, cache.cap, d), dtype=torch.bfloat16)
    return lay, _tabs(lay, Hkv), q, cache, V, Hkv


def test_decode_refuses_v_rows_other_than_the_capacity():
    lay, tabs, q, cache, V, Hkv = _decode_args()
    assert cache.cap == 32
    short = torch.zeros((V.shape[0], 30, 64), dtype=torch.bfloat16)  # the token count, not the capacity
    with pytest.raises(ValueError, match="V must be"):
        api.decode_attn(lay, tabs, q, cache, short, Hkv)
    with pytest.raises(ValueError, match="V must be"):
        api.decode_attn(lay, tabs, q, cache, V[:1], Hkv)              # fewer heads than B*Hkv
    with pytest.raises(ValueError, match="V must be"):
        api.decode_attn(lay, tabs, q, cache, V.float(), Hkv)


def test_decode_refuses_a_cache_with_fewer_heads():
    lay, tabs, q, cache, V, Hkv = _decode_args()
    small = api.Cache(cache.packed[:1].contiguous(), cache.gamma[:1].contiguous(), length=cache.length)
    with pytest.raises(ValueError, match="heads"):
        api.decode_attn(lay, tabs, q, small, None, Hkv, logits=True)


def test_decode_refuses_wrong_out_and_logits():
    lay, tabs, q, cache, V, Hkv = _decode_args()
    with pytest.raises(ValueError, match="out must be"):
        api.decode_attn(lay, tabs, q, cache, V, Hkv, out=torch.zeros((1, 4, 1, 64), dtype=torch.bfloat16))
    with pytest.raises(ValueError, match="out must be"):
        api.decode_attn(lay, tabs, q, cache, V, Hkv, out=torch.zeros((1, 4, 1, 32)))
    with pytest.raises(ValueError, match="logits must be"):
        api.decode_attn(lay, tabs, q, cache, None, Hkv, logits=torch.zeros((1, 4, 1, 29)))
    with pytest.raises(ValueError, match="device"):
        api.decode_attn(lay, tabs, q.to("meta"), cache, None, Hkv, logits=True)


def test_dequant_refuses_a_non_contiguous_cache():
    lay = api.Layout(64, 3)
    big = api.Cache.empty(lay, 2, 64, device="cpu")
    view = api.Cache(big.packed[:, :, :32], big.gamma[:, :32], length=32)  # strided planes
    with pytest.raises(ValueError, match="packed"):
        api.dequant(lay, _tabs(lay, 2), view)
    assert np.all(big.gamma.numpy() == 0)


def test_static_entry_point_refuses_like_the_workspace_one():
    """octo_decode_attn_static runs octo_decode_attn's own checks first: for every
    rejected argument set both return the same status, and the static one does so
    before it looks up or clears its scratch array (nothing here reaches CUDA)."""
    import ctypes

    from rotation_preconditioned_quantization_b200 import _lib

    lib = _lib.lib()
    good = api.Layout(128, 3)
    d96 = _lib.OctoLayout()
    ctypes.memmove(ctypes.byref(d96), good.ref, ctypes.sizeof(d96))
    d96.d = 96
    T = _lib.OctoTables(256, 256, 256, 256, 256, None, 8)
    nan = float("nan")
    cases = {  # name: (layout, q, B, Hq, Hkv, Lq, kv, cap, scale)
        "d=96": (ctypes.byref(d96), 256, 1, 4, 1, 1, 8, 8, 0.1),
        "B*Hkv > 65535": (good.ref, 256, 65536, 4, 1, 1, 8, 8, 0.1),
        "B*Hkv > 65535, many tokens": (good.ref, 256, 8192, 64, 8, 1, 131072, 131072, 0.1),
        "9 query rows": (good.ref, 256, 1, 9, 1, 1, 8, 8, 0.1),
        "q NULL": (good.ref, None, 1, 4, 1, 1, 8, 8, 0.1),
        "kv_len > cap": (good.ref, 256, 1, 4, 1, 1, 12, 8, 0.1),
        "NaN scale": (good.ref, 256, 1, 4, 1, 1, 8, 8, nan),
    }
    want = {"d=96": _lib.OCTO_EUNSUPPORTED, "B*Hkv > 65535": _lib.OCTO_EUNSUPPORTED,
            "B*Hkv > 65535, many tokens": _lib.OCTO_EUNSUPPORTED, "9 query rows": _lib.OCTO_EUNSUPPORTED,
            "q NULL": _lib.OCTO_EINVAL, "kv_len > cap": _lib.OCTO_EINVAL, "NaN scale": _lib.OCTO_EINVAL}
    for name, (L, q, B, Hq, Hkv, Lq, kv, cap, sc) in cases.items():
        ws = lib.octo_decode_attn(L, ctypes.byref(T), q, _lib.BF16, B, Hq, Hkv, Lq, kv, cap, 256, 256, None, None,
                                  256, ctypes.c_float(sc), 256, None, 256, 1 << 40, None)
        st = lib.octo_decode_attn_static(L, ctypes.byref(T), q, _lib.BF16, B, Hq, Hkv, Lq, kv, cap, 256, 256, None,
                                         None, 256, ctypes.c_float(sc), 256, None, None)
        assert ws == st == want[name], (name, ws, st)
    assert lib.octo_decode_attn_static_status(None, None) == _lib.OCTO_EINVAL
