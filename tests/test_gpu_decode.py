"""GPU parity of octo_decode_attn against the oracle (called through the C ABI).

The cache the GPU decodes is the ORACLE's encoding of the keys (packed by
the oracle and copied into the word-planar layout), so encode boundary flips
cannot leak into these checks and no oracle input comes from the GPU.
The oracle takes the materialised route (k_hat = gamma R^T u_hat, q . k_hat);
the kernel the rotated-query route.
"""

import math

import numpy as np
import pytest
import torch

from oracle import attention, codec, tables
from rotation_preconditioned_quantization_b200 import api, inputs

from . import parity

pytestmark = pytest.mark.gpu


def _oracle_cache(keys, d, b, signs_rows, tb, qjl_S=None, cap=None):
    """Oracle-encode keys [H][N][d]; return (encodings, device Cache)."""
    H, N, _ = keys.shape
    cap = N if cap is None else cap
    olay = codec.Layout(d, b)
    lay = api.Layout(d, b, qjl=qjl_S is not None)
    encs, words, gam, qb, qn = [], [], [], [], []
    for h in range(H):
        e = codec.encode(keys[h].astype(np.float64), signs_rows[h], tb, olay)
        encs.append(e)
        words.append(e.words)
        gam.append(e.gamma)
        if qjl_S is not None:
            uh = codec.decode_rotated(e.i_xi, e.i_eta, e.i_rho, tb, olay)
            bits, nu, _ = codec.qjl_encode(e.u_rot, uh, qjl_S[h])
            e.qbits, e.nu = bits, nu
            qb.append(codec.qjl_pack(bits))
            qn.append(nu)
    cache = api.Cache.empty(lay, H, cap)
    planar = parity.to_planar(np.stack(words)).view(np.int32)
    cache.packed[:, :, :N] = torch.from_numpy(planar).cuda()
    cache.gamma[:, :N] = torch.from_numpy(np.stack(gam).astype(np.float32)).cuda()
    if qjl_S is not None:
        cache.qjl_bits[:, :, :N] = torch.from_numpy(parity.to_planar(np.stack(qb)).view(np.int32)).cuda()
        cache.qjl_norm[:, :N] = torch.from_numpy(np.stack(qn).astype(np.float32)).cuda()
    cache.length = N
    return encs, cache


def _run_case(B, Hq, Hkv, Lq, d, b, N, qjl=False, q_dtype=torch.bfloat16, cap=None, seed=0, logits_only=False,
              kv_len=None, check_logits=True, key_ramp=0.0):
    tb = parity.oracle_tables(d, b)
    H = B * Hkv
    signs = tables.rotation_signs(seed, d, Hkv)
    S = tables.qjl_matrix(seed + 7, d, Hkv) if qjl else None
    keys = inputs.llm_keys(seed + 1, H, N, d)
    if key_ramp:
        # key norms grow along the sequence, so the running maximum of the logits keeps moving
        keys = keys * (1.0 + key_ramp * np.arange(N, dtype=np.float32) / N)[None, :, None]
    keys = inputs.to_bf16(keys)
    rows = [signs[h % Hkv] for h in range(H)]
    Srows = [S[h % Hkv] for h in range(H)] if qjl else None
    encs, cache = _oracle_cache(keys, d, b, rows, tb, Srows, cap)
    cap = cache.cap
    kv = N if kv_len is None else kv_len
    q = inputs.normal(seed + 2, (B, Hq, Lq, d))
    if q_dtype == torch.bfloat16:
        q = inputs.to_bf16(q)
    Vn = inputs.to_bf16(inputs.normal(seed + 3, (H, cap, d)))
    lay = api.Layout(d, b, qjl=qjl)
    dev = api.DeviceTables(*tb, signs, S)
    qt = torch.from_numpy(q).to(q_dtype).cuda()
    Vt = None if logits_only else torch.from_numpy(Vn).to(torch.bfloat16).cuda()
    ws = api.Workspace(api.decode_attn_workspace_bytes(lay, B, Hq, Hkv, Lq, kv))
    out, lg = api.decode_attn(lay, dev, qt, cache, Vt, Hkv, kv_len=kv, logits=check_logits, workspace=ws)
    torch.cuda.synchronize()
    assert ws.status() == 0, "a bounded device wait expired"
    olay = codec.Layout(d, b)
    g = Hq // Hkv
    if kv == 0:
        assert torch.count_nonzero(out) == 0
        return
    worst_l, worst_o = 0.0, 0.0
    for bi in range(B):
        for hk in range(Hkv):
            h = bi * Hkv + hk
            e = encs[h]
            qq = q[bi, hk * g:(hk + 1) * g].reshape(g * Lq, d).astype(np.float64)
            sl = slice(0, kv)
            qjl_args = (e.qbits[sl], e.nu[sl], S[hk]) if qjl else None
            ref_o, ref_l = attention.decode_attention(qq, e.gamma[sl], e.i_xi[sl], e.i_eta[sl], e.i_rho[sl],
                                                      Vn[h, sl].astype(np.float64), signs[hk], tb, olay, qjl=qjl_args)
            if check_logits and kv > 0:
                got_l = lg[bi, hk * g:(hk + 1) * g].reshape(g * Lq, kv).cpu().numpy()
                tol = 1e-4 * e.gamma[sl][None, :] * np.linalg.norm(qq, axis=1)[:, None]
                err = np.abs(got_l - ref_l)
                assert np.all(err <= tol), f"logit error {np.max(err / np.maximum(tol, 1e-30))} x tol"
                worst_l = max(worst_l, float(np.max(err / np.maximum(tol, 1e-30))))
            if not logits_only:
                got_o = out[bi, hk * g:(hk + 1) * g].reshape(g * Lq, d).cpu().numpy()
                tol = 2e-3 * np.max(np.abs(ref_o), axis=1, keepdims=True)
                err = np.abs(got_o - ref_o)
                assert np.all(err <= tol), f"output error {np.max(err / tol)} x tol"
                worst_o = max(worst_o, float(np.max(err / tol)))
    print(f"\n[decode parity] B={B} Hq={Hq} Hkv={Hkv} Lq={Lq} d={d} b={b} N={N} kv={kv} qjl={qjl}: "
          f"worst logit err {worst_l:.3g} x tol, worst output err {worst_o:.3g} x tol")


def test_logits_single_head_4096(cuda_ok):
    """One head, d=128, 4096 keys, b=3, one fp32 query: raw logits only."""
    tb = parity.oracle_tables(128, 3)
    signs = tables.rotation_signs(0, 128, 1)
    keys = inputs.gaussian_keys(0, 1, 4096, 128)
    encs, cache = _oracle_cache(keys, 128, 3, signs, tb)
    q = inputs.normal(1, (1, 1, 1, 128))
    lay = api.Layout(128, 3)
    dev = api.DeviceTables(*tb, signs)
    _, lg = api.decode_attn(lay, dev, torch.from_numpy(q).cuda(), cache, None, 1, logits=True)
    torch.cuda.synchronize()
    ref = attention.logits(q[0, 0].astype(np.float64), encs[0].gamma, encs[0].i_xi, encs[0].i_eta, encs[0].i_rho,
                           signs[0], tb, codec.Layout(128, 3))[0]
    got = lg.cpu().numpy()[0, 0, 0]
    tol = 1e-4 * encs[0].gamma * np.linalg.norm(q)
    assert np.all(np.abs(got - ref) <= tol)


@pytest.mark.parametrize("case", [
    dict(B=1, Hq=8, Hkv=2, Lq=1, d=128, b=3, N=3000),                      # GQA 4, ragged tail
    dict(B=1, Hq=2, Hkv=2, Lq=8, d=64, b=2, N=5000),                       # 8 query tokens per head
    dict(B=2, Hq=8, Hkv=2, Lq=1, d=128, b=4, N=2000, qjl=True),            # OCTOPUS-QJL
    dict(B=1, Hq=4, Hkv=4, Lq=1, d=128, b=3, N=1000, q_dtype=torch.float32),  # MHA (1 row)
    dict(B=1, Hq=4, Hkv=2, Lq=1, d=256, b=2, N=777),                       # 2 rows, d=256
    dict(B=1, Hq=2, Hkv=1, Lq=3, d=64, b=4, N=100),                        # 6 rows
    dict(B=1, Hq=4, Hkv=1, Lq=1, d=256, b=4, N=1500, qjl=True),            # QJL, d=256
    dict(B=1, Hq=8, Hkv=1, Lq=1, d=64, b=3, N=640, qjl=True),              # QJL, 8 rows
    dict(B=1, Hq=4, Hkv=1, Lq=1, d=128, b=3, N=300, cap=1000),             # cache larger than kv_len
    dict(B=1, Hq=4, Hkv=1, Lq=1, d=128, b=3, N=1),                         # a single key
    dict(B=3, Hq=4, Hkv=1, Lq=1, d=128, b=2, N=64, kv_len=0),              # empty context
    dict(B=1, Hq=8, Hkv=1, Lq=1, d=128, b=3, N=2000),                      # 8 rows at d=128 (three products)
    dict(B=1, Hq=16, Hkv=2, Lq=1, d=128, b=4, N=1500, qjl=True),           # 8 rows, b=4, QJL
    dict(B=2, Hq=4, Hkv=2, Lq=1, d=128, b=2, N=900),                       # 2 rows in the 4-row layout
    dict(B=1, Hq=4, Hkv=1, Lq=1, d=128, b=3, N=40000),                     # one head: > 32 slices to merge
    dict(B=1, Hq=4, Hkv=1, Lq=1, d=128, b=3, N=6000, key_ramp=20.0),       # logits growing along the cache
])
def test_decode_attention_cases(cuda_ok, case):
    _run_case(**case)


def test_decode_many_heads_mixed_slice_counts(cuda_ok):
    """160 KV heads of 300 keys, OCTOPUS-QJL at d=128, b=4. On 148 SMs one slice per head would leave the second
    wave 136 CTAs short, so the planner gives 136 heads two slices and keeps one for the other 24 (296 CTAs, two
    whole waves): both kinds of head, and the query preparation of every head, against the oracle."""
    _run_case(B=2, Hq=320, Hkv=80, Lq=1, d=128, b=4, N=300, qjl=True)


def test_decode_rescale_when_the_maximum_jumps(cuda_ok):
    """Keys along the query direction: the first 400 give scaled logits near 0, the rest near 9 (base 2),
    so the running maximum jumps past the slack once; the earlier keys keep a share of about
    400 * 2^-9 / 600 of the weight, which a missed or misapplied rescale would multiply by 2^9."""
    d, b, N, G = 128, 3, 1000, 4
    tb = parity.oracle_tables(d, b)
    signs = tables.rotation_signs(21, d, 1)
    q = inputs.normal(22, (1, 1, 1, d))
    q = np.repeat(q, G, axis=1)                                   # 4 equal query rows of one KV head
    qn = q[0, 0, 0] / np.linalg.norm(q[0, 0, 0])
    noise = inputs.normal(23, (N, d)) * 0.05
    target = np.where(np.arange(N) < 400, 0.0, 9.0) / (math.log2(math.e) / math.sqrt(d))  # raw logit per key
    keys = ((target / np.linalg.norm(q[0, 0, 0]))[:, None] * qn[None, :] + noise)[None].astype(np.float32)
    encs, cache = _oracle_cache(keys, d, b, list(signs), tb)
    V = inputs.to_bf16(inputs.normal(24, (1, cache.cap, d)))
    lay = api.Layout(d, b)
    out, _ = api.decode_attn(lay, api.DeviceTables(*tb, signs), torch.from_numpy(q).cuda(), cache,
                             torch.from_numpy(V).to(torch.bfloat16).cuda(), 1)
    torch.cuda.synchronize()
    e = encs[0]
    ref, lg = attention.decode_attention(q[0, :, 0].astype(np.float64), e.gamma, e.i_xi, e.i_eta, e.i_rho,
                                         V[0, :N].astype(np.float64), signs[0], tb, codec.Layout(d, b))
    w = np.exp((lg[0] - lg[0].max()) / math.sqrt(d))
    assert 1e-4 < w[:400].sum() / w.sum() < 0.2               # small, but a missed rescale would weigh it 2^9 times
    got = out[0, :, 0].cpu().numpy()
    assert np.all(np.abs(got - ref) <= 2e-3 * np.max(np.abs(ref), axis=1, keepdims=True))


def test_decode_identical_keys_give_the_mean_of_v(cuda_ok):
    """Every key the same: all logits are equal, so the attention output is the plain mean of the
    V rows (a closed form, checked against numpy's mean as well as the oracle)."""
    d, b, N = 128, 3, 777
    tb = parity.oracle_tables(d, b)
    signs = tables.rotation_signs(25, d, 1)
    key = inputs.llm_keys(26, 1, 1, d)
    keys = np.repeat(key, N, axis=1)
    encs, cache = _oracle_cache(keys, d, b, list(signs), tb)
    V = inputs.to_bf16(inputs.normal(27, (1, cache.cap, d)))
    q = inputs.normal(28, (1, 4, 1, d))
    out, lg = api.decode_attn(api.Layout(d, b), api.DeviceTables(*tb, signs), torch.from_numpy(q).cuda(), cache,
                              torch.from_numpy(V).to(torch.bfloat16).cuda(), 1, logits=True)
    torch.cuda.synchronize()
    mean_v = V[0, :N].astype(np.float64).mean(axis=0)
    got = out[0, :, 0].cpu().numpy()
    assert np.all(np.abs(got - mean_v[None, :]) <= 2e-3 * np.max(np.abs(mean_v)))
    l = lg[0, :, 0].cpu().numpy()
    assert np.all(l == l[:, :1])  # the same code words give the same logit, bit for bit
    e = encs[0]
    ref, _ = attention.decode_attention(q[0, :, 0].astype(np.float64), e.gamma, e.i_xi, e.i_eta, e.i_rho,
                                        V[0, :N].astype(np.float64), signs[0], tb, codec.Layout(d, b))
    assert np.allclose(ref, mean_v[None, :], rtol=0, atol=1e-12)


def test_decode_llm_shaped_full_size(cuda_ok):
    """B=1, 32 query / 8 KV heads, d=128, 32768 tokens, b=3: every output and logit."""
    _run_case(1, 32, 8, 1, 128, 3, 32768)


def test_decode_workspace_reuse_and_counters(cuda_ok):
    """Repeated calls with one workspace give identical results (tickets reset)."""
    tb = parity.oracle_tables(128, 3)
    signs = tables.rotation_signs(0, 128, 2)
    keys = inputs.to_bf16(inputs.llm_keys(3, 2, 20000, 128))
    encs, cache = _oracle_cache(keys, 128, 3, signs, tb)
    lay = api.Layout(128, 3)
    dev = api.DeviceTables(*tb, signs)
    q = torch.from_numpy(inputs.to_bf16(inputs.normal(4, (1, 8, 1, 128)))).to(torch.bfloat16).cuda()
    V = torch.from_numpy(inputs.to_bf16(inputs.normal(5, (2, 20000, 128)))).to(torch.bfloat16).cuda()
    ws = api.Workspace(api.decode_attn_workspace_bytes(lay, 1, 8, 2, 1, 20000))
    o1, _ = api.decode_attn(lay, dev, q, cache, V, 2, workspace=ws)
    o2, _ = api.decode_attn(lay, dev, q, cache, V, 2, workspace=ws)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2)
    assert int(ws.counters(2).abs().sum()) == 0
    assert ws.status() == 0


def test_decode_rejects_small_workspace(cuda_ok):
    lay = api.Layout(128, 3)
    tb = parity.oracle_tables(128, 3)
    dev = api.DeviceTables(*tb, tables.rotation_signs(0, 128, 1))
    cache = api.Cache.empty(lay, 1, 100000)
    cache.length = 100000
    q = torch.zeros((1, 4, 1, 128), dtype=torch.bfloat16, device="cuda")
    V = torch.zeros((1, 100000, 128), dtype=torch.bfloat16, device="cuda")
    ws = api.Workspace(256)
    from rotation_preconditioned_quantization_b200 import _lib
    need = api.decode_attn_workspace_bytes(lay, 1, 4, 1, 1, 100000)
    assert need > 256
    st = _lib.lib().octo_decode_attn(lay.ref, dev.ref, q.data_ptr(), _lib.BF16, 1, 4, 1, 1, 100000, 100000,
                                     cache.packed.data_ptr(), cache.gamma.data_ptr(), None, None, V.data_ptr(),
                                     0.1, torch.empty((1, 4, 1, 128), device="cuda").data_ptr(), None,
                                     ws.buf.data_ptr(), 256, None)
    assert st == _lib.OCTO_EWORKSPACE


def _run_sampled_full_size(B, Hq, Hkv, Lq, d, b, N, qjl, sample, keys_fn, seed=11):
    """Full-size decode; every output and logit of the sampled KV heads is checked.

    The sampled heads hold the oracle's encoding of seeded keys and seeded V.
    The other heads hold arbitrary code words and V, drawn on the device,
    since decode attention is independent per (batch, KV head).
    """
    tb = parity.oracle_tables(d, b)
    H = B * Hkv
    lay = api.Layout(d, b, qjl=qjl)
    olay = codec.Layout(d, b)
    signs = tables.rotation_signs(seed, d, Hkv)
    S = tables.qjl_matrix(seed + 7, d, Hkv) if qjl else None
    cache = api.Cache.empty(lay, H, N)
    g = torch.Generator(device="cuda").manual_seed(seed)
    cache.packed.random_(generator=g)
    cache.gamma.uniform_(0.5, 2.0, generator=g)
    if qjl:
        cache.qjl_bits.random_(generator=g)
        cache.qjl_norm.uniform_(0.0, 0.3, generator=g)
    V = torch.randn((H, N, d), device="cuda", generator=g).to(torch.bfloat16)
    cache.length = N
    refs = {}
    for h in sample:
        keys = keys_fn(seed + 100 + h, N, d)
        e = codec.encode(keys.astype(np.float64), signs[h % Hkv], tb, olay)
        cache.packed[h, :, :N] = torch.from_numpy(parity.to_planar(e.words[None])[0].view(np.int32)).cuda()
        cache.gamma[h, :N] = torch.from_numpy(e.gamma.astype(np.float32)).cuda()
        if qjl:
            uh = codec.decode_rotated(e.i_xi, e.i_eta, e.i_rho, tb, olay)
            bits, nu, _ = codec.qjl_encode(e.u_rot, uh, S[h % Hkv])
            e.qbits, e.nu = bits, nu
            cache.qjl_bits[h, :, :N] = torch.from_numpy(parity.to_planar(codec.qjl_pack(bits)[None])[0].view(np.int32)).cuda()
            cache.qjl_norm[h, :N] = torch.from_numpy(nu.astype(np.float32)).cuda()
        vh = inputs.to_bf16(inputs.normal(seed + 200 + h, (N, d)))
        V[h] = torch.from_numpy(vh).to(torch.bfloat16).cuda()
        refs[h] = (e, vh)
    q = inputs.to_bf16(inputs.normal(seed + 2, (B, Hq, Lq, d)))
    dev = api.DeviceTables(*tb, signs, S)
    ws = api.Workspace(api.decode_attn_workspace_bytes(lay, B, Hq, Hkv, Lq, N))
    out, lg = api.decode_attn(lay, dev, torch.from_numpy(q).to(torch.bfloat16).cuda(), cache, V, Hkv,
                              logits=True, workspace=ws)
    torch.cuda.synchronize()
    assert ws.status() == 0, "a bounded device wait expired"
    grp = Hq // Hkv
    for h, (e, vh) in refs.items():
        bi, hk = divmod(h, Hkv)
        qq = q[bi, hk * grp:(hk + 1) * grp].reshape(grp * Lq, d).astype(np.float64)
        qjl_args = (e.qbits, e.nu, S[hk]) if qjl else None
        ref_o, ref_l = attention.decode_attention(qq, e.gamma, e.i_xi, e.i_eta, e.i_rho, vh.astype(np.float64),
                                                  signs[hk], tb, olay, qjl=qjl_args)
        got_l = lg[bi, hk * grp:(hk + 1) * grp].reshape(grp * Lq, N).cpu().numpy()
        tol_l = 1e-4 * e.gamma[None, :] * np.linalg.norm(qq, axis=1)[:, None]
        assert np.all(np.abs(got_l - ref_l) <= tol_l), f"head {h}: logit error"
        got_o = out[bi, hk * grp:(hk + 1) * grp].reshape(grp * Lq, d).cpu().numpy()
        tol_o = 2e-3 * np.max(np.abs(ref_o), axis=1, keepdims=True)
        assert np.all(np.abs(got_o - ref_o) <= tol_o), f"head {h}: output error {np.max(np.abs(got_o - ref_o) / tol_o)} x tol"


def test_decode_video_audio_shaped_full_size(cuda_ok):
    """16 heads, d=64 (22 triplets, last padded), 65536 tokens, b=2, 8 query tokens per head;
    bf16 keys ~ N(0,1). Heads 0 and 9 are checked in full."""
    _run_sampled_full_size(1, 16, 16, 8, 64, 2, 65536, False, (0, 9),
                           lambda s, n, d: inputs.to_bf16(inputs.gaussian_keys(s, 1, n, d)[0]))


def test_decode_qjl_long_context_full_size(cuda_ok):
    """Batch 8, 32 query / 8 KV heads, d=128, 131072 tokens, b=4 + OCTOPUS-QJL sketch;
    LLM-shaped bf16 keys. KV heads 0 and 43 (batch 5) are checked in full."""
    _run_sampled_full_size(8, 32, 8, 1, 128, 4, 131072, True, (0, 43),
                           lambda s, n, d: inputs.to_bf16(inputs.llm_keys(s, 1, n, d)[0]))
