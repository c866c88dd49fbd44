"""Thin PyTorch binding of the OCTOPUS C ABI (argument marshalling only).

PyTorch supplies device memory and the current CUDA stream; every step of
the codec runs in the library's CUDA kernels (``octo_encode``,
``octo_decode_attn``) or its host table builders. Names follow the C ABI:

* :class:`Layout`          - ``octo_layout_init``
* :func:`codebook_build`   - ``octo_codebook_build`` (host)
* :func:`rotation_build`   - ``octo_rotation_build`` (host)
* :func:`qjl_build`        - ``octo_qjl_build`` (host)
* :class:`DeviceTables`    - device copies + the ``octo_tables`` struct
* :class:`Cache`           - the compressed cache buffers (word-planar layout)
* :func:`encode`           - ``octo_encode``
* :func:`decode_attn`      - ``octo_decode_attn`` (+ ``octo_decode_attn_workspace``)
"""

from __future__ import annotations

import ctypes
import math
from dataclasses import dataclass, field

import numpy as np
import torch

from . import _lib

ROUND_SCALAR = _lib.ROUND_SCALAR
ROUND_JOINT = _lib.ROUND_JOINT


def _stream_ptr(stream=None) -> int:
    s = stream if stream is not None else torch.cuda.current_stream()
    return int(s.cuda_stream)


def _ptr(t) -> int | None:
    return None if t is None else int(t.data_ptr())


class Layout:
    """Sizes of the code for head dimension d and bit budget b (``octo_layout``)."""

    def __init__(self, d: int, b: int, qjl: bool = False, rounding: int = ROUND_JOINT, delta: int = 1):
        """delta: the split of the bit budget, b + delta bits per direction coordinate and
        b - delta for the norm (``octo_layout_init_delta``); +1 is the OCTOPUS allocation."""
        self.c = _lib.OctoLayout()
        _lib.check(_lib.lib().octo_layout_init_delta(ctypes.byref(self.c), int(d), int(b), int(delta), int(bool(qjl)),
                                                     int(rounding)), "octo_layout_init_delta")

    def __getattr__(self, name):
        return getattr(self.__dict__["c"], name)

    @property
    def ref(self):
        return ctypes.byref(self.c)

    def __repr__(self):
        c = self.c
        return (f"Layout(d={c.d}, b={c.b}, T={c.T}, words={c.words}, code_bits={c.code_bits}, "
                f"qjl={c.qjl}, rounding={'joint' if c.rounding else 'scalar'})")


def codebook_build(layout: Layout):
    """Host Lloyd-Max codebooks: (dir_c, dir_t, rho_c, rho_t) float32 numpy arrays."""
    dc = np.zeros(layout.n_dir, np.float32)
    dt = np.zeros(layout.n_dir - 1, np.float32)
    rc = np.zeros(layout.n_rho, np.float32)
    rt = np.zeros(max(layout.n_rho - 1, 1), np.float32)
    _lib.check(_lib.lib().octo_codebook_build(layout.ref, dc.ctypes.data, dt.ctypes.data, rc.ctypes.data,
                                              rt.ctypes.data), "octo_codebook_build")
    return dc, dt, rc, rt[: layout.n_rho - 1]


def rotation_build(seed: int, d: int, n_heads: int) -> np.ndarray:
    """Host rotation signs [n_heads][d] float32 (+1/-1)."""
    s = np.zeros((n_heads, d), np.float32)
    _lib.check(_lib.lib().octo_rotation_build(seed & (2 ** 64 - 1), d, n_heads, s.ctypes.data), "octo_rotation_build")
    return s


def qjl_build(seed: int, d: int, n_heads: int) -> np.ndarray:
    """Host QJL projections [n_heads][d][d] float32."""
    S = np.zeros((n_heads, d, d), np.float32)
    _lib.check(_lib.lib().octo_qjl_build(seed & (2 ** 64 - 1), d, n_heads, S.ctypes.data), "octo_qjl_build")
    return S


class DeviceTables:
    """Device copies of the codec tables plus the ``octo_tables`` struct pointing at them."""

    def __init__(self, dir_c, dir_t, rho_c, rho_t, signs, qjl_S=None, device="cuda"):
        f = lambda x: torch.as_tensor(np.ascontiguousarray(x, dtype=np.float32)).to(device)
        self.dir_c, self.dir_t = f(dir_c), f(dir_t)
        self.rho_c = f(rho_c)
        rt = np.asarray(rho_t, dtype=np.float32)
        self.rho_t = f(rt if rt.size else np.zeros(1, np.float32))
        self.signs = f(signs)
        self.qjl_S = None if qjl_S is None else f(qjl_S)
        self.c = _lib.OctoTables(_ptr(self.dir_c), _ptr(self.dir_t), _ptr(self.rho_c), _ptr(self.rho_t),
                                 _ptr(self.signs), _ptr(self.qjl_S), int(self.signs.shape[0]))

    @classmethod
    def build(cls, layout: Layout, seed: int, n_heads: int, qjl_seed: int | None = None, device="cuda"):
        """Codebooks, signs (and QJL projections) from the library's host builders."""
        dc, dt, rc, rt = codebook_build(layout)
        S = qjl_build(qjl_seed if qjl_seed is not None else seed + 0x517CC1, layout.d, n_heads) if layout.qjl else None
        return cls(dc, dt, rc, rt, rotation_build(seed, layout.d, n_heads), S, device)

    @property
    def ref(self):
        return ctypes.byref(self.c)


@dataclass
class Cache:
    """Compressed key cache of ``n_heads`` heads x ``cap`` tokens (word-planar layout)."""
    packed: torch.Tensor             # uint32 viewed as int32 [n_heads][W][cap]
    gamma: torch.Tensor              # float32 [n_heads][cap]
    qjl_bits: torch.Tensor | None = None   # int32 [n_heads][d/32][cap]
    qjl_norm: torch.Tensor | None = None   # float32 [n_heads][cap]
    length: int = 0                  # tokens written so far (host bookkeeping)
    extra: dict = field(default_factory=dict)

    @classmethod
    def empty(cls, layout: Layout, n_heads: int, cap: int, device="cuda"):
        """Zeroed cache; the capacity is rounded up to a multiple of 4 tokens
        (decode stages code rows with 16-byte copies)."""
        cap = (int(cap) + 3) // 4 * 4
        packed = torch.zeros((n_heads, layout.words, cap), dtype=torch.int32, device=device)
        gamma = torch.zeros((n_heads, cap), dtype=torch.float32, device=device)
        qb = qn = None
        if layout.qjl:
            qb = torch.zeros((n_heads, layout.qjl_words, cap), dtype=torch.int32, device=device)
            qn = torch.zeros((n_heads, cap), dtype=torch.float32, device=device)
        return cls(packed, gamma, qb, qn)

    @property
    def cap(self) -> int:
        return int(self.gamma.shape[1])

    @property
    def n_heads(self) -> int:
        return int(self.gamma.shape[0])


def _check_cache(layout: Layout, tables: DeviceTables, cache: Cache, heads: int, *others):
    """The C ABI takes plain pointers, so the shapes and devices it cannot see
    are checked here: the cache must hold at least ``heads`` heads in the
    layout's word count (and sketch planes for a QJL layout), contiguous, and
    the tables and every other tensor must live on the cache's device."""
    cap = cache.cap
    if cache.packed.dtype != torch.int32 or cache.gamma.dtype != torch.float32:
        raise ValueError("cache.packed must be int32 and cache.gamma float32")
    H = int(cache.gamma.shape[0])
    if tuple(cache.packed.shape) != (H, layout.words, cap) or not cache.packed.is_contiguous():
        raise ValueError(f"cache.packed must be a contiguous [{H}][{layout.words}][{cap}] tensor for {layout!r}")
    if cache.gamma.dim() != 2 or not cache.gamma.is_contiguous():
        raise ValueError("cache.gamma must be a contiguous [n_heads][cap] tensor")
    if layout.qjl:
        qb, qn = cache.qjl_bits, cache.qjl_norm
        if qb is None or qn is None:
            raise ValueError("a QJL layout needs a cache with sketch planes (qjl_bits, qjl_norm)")
        if (qb.dtype != torch.int32 or tuple(qb.shape) != (H, layout.qjl_words, cap) or not qb.is_contiguous()
                or qn.dtype != torch.float32 or tuple(qn.shape) != (H, cap) or not qn.is_contiguous()):
            raise ValueError(f"cache sketch planes must be contiguous [{H}][{layout.qjl_words}][{cap}] int32 "
                             f"and [{H}][{cap}] float32")
    if heads > H:
        raise ValueError(f"{heads} heads requested, the cache holds {H}")
    dev = cache.gamma.device
    for t in (cache.packed, cache.qjl_bits, cache.qjl_norm, tables.dir_c, tables.rho_c, tables.signs,
              tables.qjl_S) + others:
        if t is not None and t.device != dev:
            raise ValueError(f"a tensor is on device {t.device}, the cache on device {dev}")
    if layout.qjl and tables.qjl_S is None:
        raise ValueError("a QJL layout needs tables with the projection matrices (qjl_S)")


def encode(layout: Layout, tables: DeviceTables, keys: torch.Tensor, cache: Cache, token_offset: int | None = None,
           stream=None) -> Cache:
    """Encode keys [n_heads][n_tokens][d] (float32 or bfloat16, CUDA) into cache at token_offset.

    token_offset defaults to ``cache.length`` (append); cache.length is
    advanced to the end of the written range.
    """
    if keys.dim() != 3 or keys.shape[-1] != layout.d:
        raise ValueError(f"keys must be [n_heads][n_tokens][{layout.d}], got {tuple(keys.shape)}")
    if keys.stride(-1) != 1:
        raise ValueError("keys must be contiguous in the last dimension")
    dt = {torch.float32: _lib.F32, torch.bfloat16: _lib.BF16}.get(keys.dtype)
    if dt is None:
        raise ValueError(f"unsupported key dtype {keys.dtype}")
    off = cache.length if token_offset is None else int(token_offset)
    n_heads, n_tok = int(keys.shape[0]), int(keys.shape[1])
    _check_cache(layout, tables, cache, n_heads, keys)
    st = _lib.lib().octo_encode(layout.ref, tables.ref, _ptr(keys), dt, n_heads, n_tok, keys.stride(0), keys.stride(1),
                                cache.cap, off, _ptr(cache.packed), _ptr(cache.gamma), _ptr(cache.qjl_bits),
                                _ptr(cache.qjl_norm), _stream_ptr(stream))
    _lib.check(st, "octo_encode")
    cache.length = max(cache.length, off + n_tok)
    return cache


def dequant(layout: Layout, tables: DeviceTables, cache: Cache, n_tokens: int | None = None, token_offset: int = 0,
            n_heads: int | None = None, dtype=torch.float32, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Reconstructed keys k_hat = gamma R^T u_hat of tokens [token_offset, token_offset + n_tokens)
    of the first n_heads cache heads, as [n_heads][n_tokens][d] (float32 or bfloat16).

    n_tokens defaults to ``cache.length - token_offset``, n_heads to all cache heads.
    """
    dt = {torch.float32: _lib.F32, torch.bfloat16: _lib.BF16}.get(dtype if out is None else out.dtype)
    if dt is None:
        raise ValueError(f"unsupported output dtype {dtype if out is None else out.dtype}")
    n = cache.length - int(token_offset) if n_tokens is None else int(n_tokens)
    h = cache.n_heads if n_heads is None else int(n_heads)
    if h > cache.n_heads:
        raise ValueError(f"n_heads {h} > cache heads {cache.n_heads}")
    shape = (h, max(n, 0), layout.d)
    if out is None:
        out = torch.empty(shape, dtype=dtype, device=cache.gamma.device)
    elif tuple(out.shape) != shape or not out.is_contiguous():
        raise ValueError(f"out must be a contiguous {shape} tensor")
    _check_cache(layout, tables, cache, h, out)
    st = _lib.lib().octo_dequant(layout.ref, tables.ref, h, n, cache.cap, int(token_offset), _ptr(cache.packed),
                                 _ptr(cache.gamma), _ptr(out), dt, _stream_ptr(stream))
    _lib.check(st, "octo_dequant")
    return out


def decode_attn_workspace_bytes(layout: Layout, B: int, Hq: int, Hkv: int, Lq: int, kv_len: int) -> int:
    return int(_lib.lib().octo_decode_attn_workspace(layout.ref, B, Hq, Hkv, Lq, kv_len))


class Workspace:
    """Device workspace for decode_attn: status word, ticket counters (zeroed
    here, left zero by every completed call) and split partials."""

    def __init__(self, nbytes: int, device="cuda"):
        n = max(512, (int(nbytes) + 255) // 256 * 256)
        self.buf = torch.zeros(n // 4, dtype=torch.int32, device=device)

    @property
    def nbytes(self) -> int:
        return self.buf.numel() * 4

    def status(self) -> int:
        """Device status word (synchronises): nonzero if a bounded on-chip wait expired."""
        return int(self.buf[0].item())

    def counters(self, n_heads: int) -> torch.Tensor:
        return self.buf[64:64 + n_heads]

    def ensure(self, nbytes: int):
        if nbytes > self.nbytes:
            self.__init__(nbytes, self.buf.device)
        return self


def decode_attn(layout: Layout, tables: DeviceTables, q: torch.Tensor, cache: Cache, V: torch.Tensor | None,
                Hkv: int, kv_len: int | None = None, scale: float | None = None, out: torch.Tensor | None = None,
                logits: torch.Tensor | None = None, workspace: Workspace | None = None, stream=None):
    """One fused decode-attention step.

    q [B][Hq][Lq][d] (float32 or bfloat16), cache heads = B*Hkv,
    V [B*Hkv][cap][d] bfloat16 or None (logits only). Returns (out, logits):
    out [B][Hq][Lq][d] float32 (None without V), logits [B][Hq][Lq][kv_len]
    float32 raw logits when requested (pass ``logits=True`` to allocate).
    """
    if q.dim() != 4 or q.shape[-1] != layout.d or not q.is_contiguous():
        raise ValueError("q must be contiguous [B][Hq][Lq][d]")
    B, Hq, Lq = int(q.shape[0]), int(q.shape[1]), int(q.shape[2])
    qdt = {torch.float32: _lib.F32, torch.bfloat16: _lib.BF16}.get(q.dtype)
    if qdt is None:
        raise ValueError(f"unsupported query dtype {q.dtype}")
    kv = cache.length if kv_len is None else int(kv_len)
    if scale is None:
        scale = 1.0 / math.sqrt(layout.d)
    if V is not None:
        # the kernel steps from head to head by cap rows of V
        if (V.dtype != torch.bfloat16 or not V.is_contiguous() or V.dim() != 3 or V.shape[0] < B * Hkv
                or tuple(V.shape[1:]) != (cache.cap, layout.d)):
            raise ValueError(f"V must be contiguous bfloat16 [B*Hkv][{cache.cap}][{layout.d}] (the cache's capacity)")
        if out is None:
            out = torch.empty((B, Hq, Lq, layout.d), dtype=torch.float32, device=q.device)
        elif out.dtype != torch.float32 or tuple(out.shape) != (B, Hq, Lq, layout.d) or not out.is_contiguous():
            raise ValueError(f"out must be a contiguous float32 {(B, Hq, Lq, layout.d)} tensor")
    if logits is True:
        logits = torch.empty((B, Hq, Lq, kv), dtype=torch.float32, device=q.device)
    elif logits is False:
        logits = None
    elif logits is not None and (logits.dtype != torch.float32 or tuple(logits.shape) != (B, Hq, Lq, kv)
                                 or not logits.is_contiguous()):
        raise ValueError(f"logits must be a contiguous float32 {(B, Hq, Lq, kv)} tensor")
    _check_cache(layout, tables, cache, B * Hkv, q, V, out, logits)
    need = decode_attn_workspace_bytes(layout, B, Hq, Hkv, Lq, kv)
    if workspace is None:
        workspace = Workspace(need, q.device)
    workspace.ensure(need)
    ws_ptr, ws_n = _ptr(workspace.buf), workspace.nbytes
    st = _lib.lib().octo_decode_attn(layout.ref, tables.ref, _ptr(q), qdt, B, Hq, Hkv, Lq, kv, cache.cap,
                                     _ptr(cache.packed), _ptr(cache.gamma), _ptr(cache.qjl_bits), _ptr(cache.qjl_norm),
                                     _ptr(V), ctypes.c_float(scale), _ptr(out), _ptr(logits), ws_ptr, ws_n,
                                     _stream_ptr(stream))
    _lib.check(st, "octo_decode_attn")
    return out, logits
