"""CPU tests of the C ABI: the library loads, exports every declared symbol,
its host table builders agree with the oracle, and argument validation
returns a status before anything is launched."""

import ctypes
import os
import re

import numpy as np
import pytest

from oracle import tables
from rotation_preconditioned_quantization_b200 import _lib, api

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "octopus.h")


def _declared():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(octo_[a-z0-9_]+)\s*\(", src)))


def test_library_exports_every_declared_symbol():
    L = _lib.lib()
    names = _declared()
    assert len(names) >= 9
    for n in names:
        assert hasattr(L, n), n
    assert set(names) == set(_lib.exported_symbols())
    assert L.octo_abi_version() == 102


@pytest.mark.parametrize("d,b", [(64, 2), (64, 4), (128, 3), (128, 4), (256, 2), (256, 4)])
def test_layout_init(d, b):
    lay = api.Layout(d, b, qjl=True)
    T = -(-d // 3)
    assert (lay.T, lay.b_dir, lay.b_rho, lay.code_bits) == (T, b + 1, b - 1, 3 * b + 1)
    assert lay.words == -(-T * (3 * b + 1) // 32)
    assert (lay.n_dir, lay.n_rho, lay.qjl_words) == (2 ** (b + 1), 2 ** (b - 1), d // 32)


def test_layout_words_of_the_workloads():
    # 43 triplets x 10 bits = 14 words (d=128, b=3); 22 x 7 = 5 (d=64, b=2); 43 x 13 = 18 (d=128, b=4)
    assert api.Layout(128, 3).words == 14
    assert api.Layout(64, 2).words == 5
    assert api.Layout(128, 4).words == 18


def test_layout_rejects_unsupported():
    L = _lib.OctoLayout()
    f = _lib.lib().octo_layout_init
    assert f(ctypes.byref(L), 96, 3, 0, 1) == _lib.OCTO_EUNSUPPORTED
    assert f(ctypes.byref(L), 128, 5, 0, 1) == _lib.OCTO_EUNSUPPORTED
    assert f(ctypes.byref(L), 128, 1, 0, 1) == _lib.OCTO_EUNSUPPORTED
    assert f(ctypes.byref(L), 128, 3, 2, 1) == _lib.OCTO_EINVAL
    assert f(ctypes.byref(L), 128, 3, 0, 7) == _lib.OCTO_EINVAL
    assert f(None, 128, 3, 0, 1) == _lib.OCTO_EINVAL


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("b", [2, 3, 4])
def test_host_codebooks_match_oracle(d, b):
    lay = api.Layout(d, b)
    dc, dt, rc, rt = api.codebook_build(lay)
    odc, odt, orc, ort = tables.codebooks(d, b)
    # independent constructions (closed-form marginal + own quadrature vs nested quadrature)
    assert np.max(np.abs(dc - odc)) < 1e-7 and np.max(np.abs(rc - orc)) < 1e-7
    assert np.max(np.abs(dt - odt)) < 1e-7
    if len(ort):
        assert np.max(np.abs(rt - ort)) < 1e-7
    # and after rounding to float32 they are the same tables
    f = lambda x: np.asarray(x, dtype=np.float32)
    assert np.array_equal(dc, f(odc)) and np.array_equal(rc, f(orc)) and np.array_equal(dt, f(odt))


def test_host_signs_and_qjl_match_oracle():
    s = api.rotation_build(7, 128, 3)
    assert np.array_equal(s, tables.rotation_signs(7, 128, 3).astype(np.float32))
    S = api.qjl_build(3, 64, 2)
    oS = tables.qjl_matrix(3, 64, 2).astype(np.float32)
    # libm vs numpy transcendental functions may differ in the last bit of the double
    ulp = np.spacing(np.abs(oS))
    assert np.all(np.abs(S - oS) <= ulp)
    assert np.mean(S == oS) > 0.999


def test_encode_and_decode_validate_before_launch():
    L = api.Layout(128, 3)
    lib = _lib.lib()
    T = _lib.OctoTables()
    null = None
    # NULL tables / keys
    assert lib.octo_encode(L.ref, None, null, 0, 1, 1, 128, 128, 4, 0, null, null, null, null, null) == _lib.OCTO_EINVAL
    assert lib.octo_encode(L.ref, ctypes.byref(T), null, 0, 1, 1, 128, 128, 4, 0, null, null, null, null, null) == _lib.OCTO_EINVAL
    # range checks: offset + n > cap, negative sizes, bad dtype
    assert lib.octo_encode(L.ref, ctypes.byref(T), 16, 0, 1, 5, 128, 128, 4, 0, 16, 16, null, null, null) == _lib.OCTO_EINVAL
    assert lib.octo_encode(L.ref, ctypes.byref(T), 16, 0, -1, 1, 128, 128, 4, 0, 16, 16, null, null, null) == _lib.OCTO_EINVAL
    assert lib.octo_encode(L.ref, ctypes.byref(T), 16, 9, 1, 1, 128, 128, 4, 0, 16, 16, null, null, null) == _lib.OCTO_EINVAL
    # zero tokens is a no-op
    assert lib.octo_encode(L.ref, ctypes.byref(T), null, 0, 1, 0, 128, 128, 4, 0, null, null, null, null, null) == _lib.OCTO_OK
    # decode: kv_len > cap, Hq % Hkv, both outputs NULL, too many query rows
    args = lambda **k: dict(dict(q=16, qd=0, B=1, Hq=4, Hkv=1, Lq=1, kv=8, cap=8, V=16, out=16, lg=null), **k)

    def dec(a):
        return lib.octo_decode_attn(L.ref, ctypes.byref(T), a["q"], a["qd"], a["B"], a["Hq"], a["Hkv"], a["Lq"],
                                    a["kv"], a["cap"], 16, 16, null, null, a["V"], ctypes.c_float(0.1), a["out"], a["lg"],
                                    null, 0, null)
    assert dec(args()) == _lib.OCTO_EINVAL                    # tables hold NULL pointers
    Tf = _lib.OctoTables(16, 16, 16, 16, 16, None, 1)
    assert lib.octo_decode_attn(L.ref, ctypes.byref(Tf), 16, 0, 1, 4, 1, 1, 9, 8, 16, 16, null, null, 16,
                                ctypes.c_float(0.1), 16, null, null, 0, null) == _lib.OCTO_EINVAL
    assert lib.octo_decode_attn(L.ref, ctypes.byref(Tf), 16, 0, 1, 3, 2, 1, 8, 8, 16, 16, null, null, 16,
                                ctypes.c_float(0.1), 16, null, null, 0, null) == _lib.OCTO_EINVAL
    assert lib.octo_decode_attn(L.ref, ctypes.byref(Tf), 16, 0, 1, 4, 1, 1, 8, 8, 16, 16, null, null, null,
                                ctypes.c_float(0.1), null, null, null, 0, null) == _lib.OCTO_EINVAL
    # the workspace is always required (status word), 256-byte aligned
    assert lib.octo_decode_attn(L.ref, ctypes.byref(Tf), 16, 0, 1, 4, 1, 1, 8, 8, 16, 16, null, null, 16,
                                ctypes.c_float(0.1), 16, null, null, 0, null) == _lib.OCTO_EINVAL
    assert lib.octo_decode_attn(L.ref, ctypes.byref(Tf), 16, 0, 1, 4, 1, 1, 8, 8, 16, 16, null, null, 16,
                                ctypes.c_float(0.1), 16, null, 272, 1 << 20, null) == _lib.OCTO_EINVAL
    # cache rows are staged with 16-byte copies: capacity % 4 and aligned cache pointers
    assert lib.octo_decode_attn(L.ref, ctypes.byref(Tf), 16, 0, 1, 4, 1, 1, 6, 6, 16, 16, null, null, 16,
                                ctypes.c_float(0.1), 16, null, 256, 1 << 20, null) == _lib.OCTO_EINVAL
    assert lib.octo_decode_attn(L.ref, ctypes.byref(Tf), 16, 0, 1, 4, 1, 1, 8, 8, 20, 16, null, null, 16,
                                ctypes.c_float(0.1), 16, null, 256, 1 << 20, null) == _lib.OCTO_EINVAL
    # too many query rows per KV head
    assert lib.octo_decode_attn(L.ref, ctypes.byref(Tf), 16, 0, 1, 16, 1, 1, 8, 8, 16, 16, null, null, 16,
                                ctypes.c_float(0.1), 16, null, 256, 1 << 20, null) == _lib.OCTO_EUNSUPPORTED
    # QJL layout without sketch buffers
    Lq = api.Layout(128, 4, qjl=True)
    assert lib.octo_decode_attn(Lq.ref, ctypes.byref(Tf), 16, 0, 1, 4, 1, 1, 8, 8, 16, 16, null, null, 16,
                                ctypes.c_float(0.1), 16, null, null, 0, null) == _lib.OCTO_EINVAL
    assert lib.octo_decode_attn_workspace(L.ref, 1, 16, 1, 1, 8) == 0
    assert lib.octo_decode_attn_workspace(L.ref, 1, 4, 1, 1, 0) >= 256


def test_decode_size_limits_return_unsupported_before_launch():
    """B*Hkv is the grid's y extent (at most 65535) and token coordinates of the tensor copies
    are 32-bit: larger requests are refused before anything touches the GPU."""
    L = api.Layout(128, 3)
    lib = _lib.lib()
    Tf = _lib.OctoTables(16, 16, 16, 16, 16, None, 1)

    def dec(B, Hkv, kv, cap, scale=0.1):
        return lib.octo_decode_attn(L.ref, ctypes.byref(Tf), 256, 0, B, 4 * Hkv, Hkv, 1, kv, cap, 256, 256, None,
                                    None, 256, ctypes.c_float(scale), 256, None, 256, 1 << 30, None)
    assert dec(65536, 1, 8, 8) == _lib.OCTO_EUNSUPPORTED
    assert dec(4096, 16, 8, 8) == _lib.OCTO_EUNSUPPORTED
    assert dec(1, 1, 1 << 31, 1 << 31) == _lib.OCTO_EUNSUPPORTED
    assert dec(1, 1, 8, 8, scale=float("nan")) == _lib.OCTO_EINVAL


def test_dequant_validates_before_launch():
    L = api.Layout(128, 3)
    lib = _lib.lib()
    null = None
    Tf = _lib.OctoTables(16, 16, 16, 16, 16, None, 1)

    def dq(tab=ctypes.byref(Tf), heads=1, n=4, cap=8, off=0, packed=16, gamma=16, out=16, dt=_lib.F32, lay=L):
        return lib.octo_dequant(lay.ref, tab, heads, n, cap, off, packed, gamma, out, dt, null)
    assert dq(tab=None) == _lib.OCTO_EINVAL
    assert dq(tab=ctypes.byref(_lib.OctoTables())) == _lib.OCTO_EINVAL   # tables hold NULL pointers
    assert dq(off=5) == _lib.OCTO_EINVAL                                  # token_offset + n_tokens > cache_cap
    assert dq(n=-1) == _lib.OCTO_EINVAL and dq(heads=-1) == _lib.OCTO_EINVAL
    assert dq(dt=7) == _lib.OCTO_EINVAL                                   # output dtype
    assert dq(out=24) == _lib.OCTO_EINVAL                                 # out not 16-byte aligned
    assert dq(packed=null) == _lib.OCTO_EINVAL and dq(gamma=null) == _lib.OCTO_EINVAL and dq(out=null) == _lib.OCTO_EINVAL
    bad = _lib.OctoLayout()
    ctypes.memmove(ctypes.byref(bad), L.ref, ctypes.sizeof(bad))
    bad.words += 1                                                        # a layout that init would not produce
    assert lib.octo_dequant(ctypes.byref(bad), ctypes.byref(Tf), 1, 4, 8, 0, 16, 16, 16, _lib.F32, null) == _lib.OCTO_EINVAL
    # nothing to do: no launch, even with NULL buffers
    assert dq(n=0, packed=null, gamma=null, out=null) == _lib.OCTO_OK
    assert dq(heads=0, packed=null, gamma=null, out=null) == _lib.OCTO_OK


def test_status_strings():
    for s in (0, -1, -2, -3, -4):
        assert _lib.status_string(s).startswith("OCTO_")
    with pytest.raises(_lib.OctoError):
        _lib.check(-1, "x")


def _planned_workspace(heads, kv_len, d, words, qjl, G, sms=148):
    """Workspace bytes for the split count the planner documents: minimise
    waves(s) * (8 us + keys per slice * unit bytes / 30 GB/s per SM) over
    s <= min(1024, ceil(kv/64)); slices are rounded up to 16 keys. Then, when
    the CTAs span several waves and the last is partly empty, as many heads
    as fill it take one slice more (if that adds a slice), and the partials
    take that larger count of slots per head."""
    unit = 4 * words + 4 + 2 * d + (4 * (d // 32) + 4 if qjl else 0)
    kv = max(kv_len, 1)
    best, best_s = None, 1
    for s in range(1, max(1, min(1024, (kv + 63) // 64)) + 1):
        waves = (heads * s + sms - 1) // sms
        cost = waves * (8.0 + ((kv + s - 1) // s) * unit / 30.0e3)
        if best is None or cost < best * (1.0 - 1e-9):
            best, best_s = cost, s
    per = -(-kv // best_s)
    per = -(-per // 16) * 16
    n_splits = max(1, -(-kv // per))
    ctas, rem = heads * n_splits, heads * n_splits % sms
    if kv_len > 0 and ctas > sms and rem and sms - rem < heads:
        per_hi = -(-(-(-kv // (n_splits + 1))) // 16) * 16
        if -(-kv // per_hi) == n_splits + 1:
            n_splits += 1
    up = lambda x: (x + 255) // 256 * 256  # noqa: E731
    total = 256 + up(4 * heads) + 2 * up(4 * heads * n_splits * G) + up(4 * heads * n_splits * G * d)
    if qjl and d <= 128:
        # the sketch's query preparation: per head G rotated rows of whole 12-float k-steps (at least d + 4
        # floats), then G rows of p = S q_rot
        t = (d + 2) // 3
        qrow = max(12 * ((t + 3) // 4), d + 4)
        total += up(4 * heads * G * (qrow + d))
    return n_splits, total


@pytest.mark.parametrize("B,Hq,Hkv,Lq,d,b,qjl,kv,G", [
    (1, 32, 8, 1, 128, 3, False, 32768, 4),    # the LLM decode workload
    (1, 16, 16, 8, 64, 2, False, 65536, 8),    # video/audio: 8 query tokens per head
    (8, 32, 8, 1, 128, 4, True, 131072, 4),    # long context with the QJL sketch
    (8, 32, 8, 1, 128, 3, False, 131072, 4),
    (1, 4, 1, 1, 256, 2, False, 5, 4),         # fewer keys than one chunk
    (2, 2, 2, 1, 64, 4, False, 100000, 1),
])
def test_split_planner_workspace(B, Hq, Hkv, Lq, d, b, qjl, kv, G):
    """The host's split plan, seen through the workspace size it asks for
    (on a machine without a GPU the planner assumes 148 SMs)."""
    L = api.Layout(d, b, qjl=qjl)
    n_splits, total = _planned_workspace(B * Hkv, kv, d, L.words, qjl, G)
    assert _lib.lib().octo_decode_attn_workspace(L.ref, B, Hq, Hkv, Lq, kv) == total
    if (B, kv) == (1, 32768):
        assert n_splits == 18  # 8 heads x 18 slices: 144 CTAs, one wave on 148 SMs
    if (B, kv, b) == (8, 131072, 4):
        # 64 heads x 9 slices = 576 CTAs leave the fourth wave 16 short: 16 heads take 10 slices (592 = 4 x 148)
        assert n_splits == 10


@pytest.mark.parametrize("b,delta", [(3, -1), (3, 0), (3, 1), (3, 2), (4, -1), (4, 0), (4, 1), (2, 0), (2, 1)])
def test_layout_init_delta_matches_the_oracle_layout(b, delta):
    """The split of the bit budget ([EXPL] "non-uniform bit allocation": b + delta bits per direction
    coordinate, b - delta for the norm) gives the oracle's sizes; delta = +1 is octo_layout_init."""
    from oracle import codec
    lay = api.Layout(128, b, delta=delta)
    ol = codec.Layout(128, b, delta)
    assert (lay.b_dir, lay.b_rho, lay.code_bits, lay.words, lay.n_dir, lay.n_rho, lay.T) == (
        ol.b_dir, ol.b_rho, ol.code_bits, ol.words, ol.n_dir, ol.n_rho, ol.T)
    assert lay.code_bits == 3 * b + delta
    if delta == 1:
        ref = api.Layout(128, b)
        assert bytes(lay.c) == bytes(ref.c)


def test_layout_init_delta_refusals_and_decode_split():
    L = _lib.OctoLayout()
    f = _lib.lib().octo_layout_init_delta
    assert f(ctypes.byref(L), 128, 4, 2, 0, 1) == _lib.OCTO_EUNSUPPORTED   # 6 direction bits
    assert f(ctypes.byref(L), 128, 2, 1, 0, 1) == _lib.OCTO_OK
    assert f(ctypes.byref(L), 128, 2, 2, 0, 1) == _lib.OCTO_EUNSUPPORTED   # no norm bits
    assert f(ctypes.byref(L), 128, 3, 0, 1, 1) == _lib.OCTO_EUNSUPPORTED   # the sketch: OCTOPUS split only
    assert f(None, 128, 3, 0, 0, 1) == _lib.OCTO_EINVAL
    lib = _lib.lib()
    T = _lib.OctoTables(256, 256, 256, 256, 256, None, 1)
    sweep = api.Layout(128, 3, delta=0)
    # the fused decode runs the OCTOPUS split only; refused before anything is launched
    assert lib.octo_decode_attn(sweep.ref, ctypes.byref(T), 256, 0, 1, 4, 1, 1, 8, 8, 256, 256, None, None, 256,
                                ctypes.c_float(0.1), 256, None, 256, 1 << 20, None) == _lib.OCTO_EUNSUPPORTED
    assert lib.octo_decode_attn_workspace(sweep.ref, 1, 4, 1, 1, 8) == 0
    # encode / reconstruction of a sweep split exist at d = 128 only
    off = api.Layout(64, 3, delta=0)
    assert lib.octo_encode(off.ref, ctypes.byref(T), 256, 0, 1, 4, 64, 64, 4, 0, 256, 256, None, None,
                           None) == _lib.OCTO_EUNSUPPORTED
    assert lib.octo_dequant(off.ref, ctypes.byref(T), 1, 4, 4, 0, 256, 256, 256, 0, None) == _lib.OCTO_EUNSUPPORTED
