"""GPU parity of octo_dequant (key reconstruction, k_hat = gamma R^T u_hat)
against the oracle, called through the C ABI.

Small cases decode the ORACLE's encoding of seeded keys (packed by the
oracle, copied into the word-planar cache), so no oracle input comes from
the GPU. The full-size case fills the cache with seeded random words (every
bit pattern is a valid code) and checks sampled tokens.

Tolerances (the kernel computes in fp32, the oracle in fp64 from the same
fp32 codebooks and the fp32 gamma the cache stores):
* fp32 output: |k_gpu - k_ref| <= 1e-5 * ||k_ref|| per element;
* bf16 output: the same plus 2^-7 |k_ref| (one bf16 step at most).
"""

import numpy as np
import pytest
import torch

from oracle import codec, tables
from rotation_preconditioned_quantization_b200 import api, inputs

from . import parity

pytestmark = pytest.mark.gpu


def _oracle_cache(keys, d, b, signs_rows, tb, cap, qjl=False):
    H, N, _ = keys.shape
    olay = codec.Layout(d, b)
    encs = [codec.encode(keys[h].astype(np.float64), signs_rows[h], tb, olay) for h in range(H)]
    cache = api.Cache.empty(api.Layout(d, b, qjl=qjl), H, cap)
    cache.packed[:, :, :N] = torch.from_numpy(parity.to_planar(np.stack([e.words for e in encs])).view(np.int32)).cuda()
    cache.gamma[:, :N] = torch.from_numpy(np.stack([e.gamma for e in encs]).astype(np.float32)).cuda()
    cache.length = N
    return encs, cache


def _reference(gamma32, i_xi, i_eta, i_rho, signs, tb, d, b):
    return codec.decode_keys(np.asarray(gamma32, np.float64), i_xi, i_eta, i_rho, signs, tb, codec.Layout(d, b))


def _check(got, ref, bf16=False):
    got = np.asarray(got, dtype=np.float64)
    tol = 1e-5 * np.linalg.norm(ref, axis=-1, keepdims=True)
    if bf16:
        tol = tol + 2.0 ** -7 * np.abs(ref)
    err = np.abs(got - ref)
    tol = np.broadcast_to(tol, err.shape)
    assert np.all(err <= tol), f"max err {err.max():.3e} (tol at argmax {tol.flat[np.argmax(err - tol)]:.3e})"


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("b", [2, 3, 4])
def test_dequant_matches_oracle(cuda_ok, d, b):
    H, N, cap, off, n = 3, 300, 320, 5, 290  # several 64-key tiles, a ragged tail, an offset start
    tb = parity.oracle_tables(d, b)
    signs = tables.rotation_signs(11, d, 2)    # 2 sign rows for 3 cache heads: head 2 uses row 0
    rows = [signs[h % 2] for h in range(H)]
    keys = inputs.to_bf16(inputs.llm_keys(12 + d + b, H, N, d))
    encs, cache = _oracle_cache(keys, d, b, rows, tb, cap)
    lay = api.Layout(d, b)
    dev = api.DeviceTables(*tb, signs)
    out = api.dequant(lay, dev, cache, n_tokens=n, token_offset=off)
    torch.cuda.synchronize()
    got = out.cpu().numpy()
    assert got.shape == (H, n, d)
    for h, e in enumerate(encs):
        sl = slice(off, off + n)
        ref = _reference(np.float32(e.gamma[sl]), e.i_xi[sl], e.i_eta[sl], e.i_rho[sl], rows[h], tb, d, b)
        _check(got[h], ref)


def test_dequant_bf16_output_and_head_subset(cuda_ok):
    d, b, H, N = 128, 3, 4, 200
    tb = parity.oracle_tables(d, b)
    signs = tables.rotation_signs(13, d, H)
    keys = inputs.to_bf16(inputs.llm_keys(14, H, N, d))
    encs, cache = _oracle_cache(keys, d, b, list(signs), tb, N)
    lay = api.Layout(d, b)
    dev = api.DeviceTables(*tb, signs)
    out = api.dequant(lay, dev, cache, n_heads=2, dtype=torch.bfloat16)
    torch.cuda.synchronize()
    assert out.shape == (2, N, d) and out.dtype == torch.bfloat16
    got = out.float().cpu().numpy()
    for h in range(2):
        e = encs[h]
        _check(got[h], _reference(np.float32(e.gamma), e.i_xi, e.i_eta, e.i_rho, signs[h], tb, d, b), bf16=True)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_dequant_output_only_16_byte_aligned(cuda_ok, dtype):
    """An output that is 16- but not 32-byte aligned takes the 16-byte store path."""
    d, b, H, N = 128, 3, 2, 150
    tb = parity.oracle_tables(d, b)
    signs = tables.rotation_signs(19, d, H)
    keys = inputs.to_bf16(inputs.llm_keys(20, H, N, d))
    encs, cache = _oracle_cache(keys, d, b, list(signs), tb, N)
    esz = 4 if dtype == torch.float32 else 2
    buf = torch.empty(H * N * d + 32, dtype=dtype, device="cuda")
    shift = 16 // esz
    out = buf[shift:shift + H * N * d].view(H, N, d)
    assert out.data_ptr() % 32 == 16
    api.dequant(api.Layout(d, b), api.DeviceTables(*tb, signs), cache, out=out)
    torch.cuda.synchronize()
    got = out.float().cpu().numpy()
    for h in range(H):
        e = encs[h]
        _check(got[h], _reference(np.float32(e.gamma), e.i_xi, e.i_eta, e.i_rho, signs[h], tb, d, b),
               bf16=dtype == torch.bfloat16)


def test_dequant_ignores_the_qjl_sketch(cuda_ok):
    """A QJL layout reconstructs from the base codes alone: the result equals
    the plain layout's on the same words, whatever the sketch holds."""
    d, b, H, N = 128, 4, 2, 130
    tb = parity.oracle_tables(d, b)
    signs = tables.rotation_signs(15, d, H)
    keys = inputs.to_bf16(inputs.llm_keys(16, H, N, d))
    _, cache = _oracle_cache(keys, d, b, list(signs), tb, N, qjl=True)
    cache.qjl_bits.random_()
    cache.qjl_norm.uniform_(0.0, 1.0)
    dev = api.DeviceTables(*tb, signs, tables.qjl_matrix(3, d, H))
    a = api.dequant(api.Layout(d, b, qjl=True), dev, cache)
    plain = api.Cache(cache.packed, cache.gamma, length=N)
    c = api.dequant(api.Layout(d, b), dev, plain)
    torch.cuda.synchronize()
    assert torch.equal(a, c)


def test_dequant_empty_ranges(cuda_ok):
    d, b = 64, 2
    tb = parity.oracle_tables(d, b)
    dev = api.DeviceTables(*tb, tables.rotation_signs(0, d, 1))
    cache = api.Cache.empty(api.Layout(d, b), 2, 16)
    cache.length = 16
    assert api.dequant(api.Layout(d, b), dev, cache, n_tokens=0).shape == (2, 0, d)
    assert api.dequant(api.Layout(d, b), dev, cache, n_heads=0).shape == (0, 16, d)


def test_dequant_full_size_sampled(cuda_ok):
    """The LLM prefill cache (8 KV heads x 32768 tokens, d=128, b=3) filled
    with seeded random code words and gammas; sampled tokens of every head
    against the oracle."""
    d, b, H, N = 128, 3, 8, 32768
    lay = api.Layout(d, b)
    tb = parity.oracle_tables(d, b)
    signs = tables.rotation_signs(17, d, H)
    rng = np.random.default_rng(18)
    words = rng.integers(0, 2 ** 32, (H, N, lay.words), dtype=np.uint64).astype(np.uint32)
    gam = rng.uniform(0.25, 4.0, (H, N)).astype(np.float32)
    cache = api.Cache.empty(lay, H, N)
    cache.packed.copy_(torch.from_numpy(parity.to_planar(words).view(np.int32)))
    cache.gamma.copy_(torch.from_numpy(gam))
    cache.length = N
    dev = api.DeviceTables(*tb, signs)
    for dt in (torch.float32, torch.bfloat16):
        out = api.dequant(lay, dev, cache, dtype=dt)
        torch.cuda.synchronize()
        idx = np.sort(rng.choice(N, 64, replace=False))
        idx = np.concatenate([[0, N - 1], idx])
        got = out[:, torch.from_numpy(idx).cuda()].float().cpu().numpy()
        olay = codec.Layout(d, b)
        for h in range(H):
            ix, iy, ir = codec.unpack(words[h, idx], olay)
            _check(got[h], _reference(gam[h, idx], ix, iy, ir, signs[h], tb, d, b), bf16=dt == torch.bfloat16)
