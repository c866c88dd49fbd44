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
