"""Pins of the oracle's decode attention over an FP8 KV cache.

An FP8 KV cache and FP8 attention are the step from the linear layers' speedup
to the recipe's full one (section "Real-world performance gains" of "NVIDIA
NeMo RL Achieves 48% Speedup With End-to-End FP8 Precision Training").  The
pins are properties of attention, not the formula retyped: a single cached
token returns its value vector; equal value vectors are returned unchanged; a
zero query averages the values; the result does not depend on token order;
grouped-query heads read their own key/value head; tokens past a sequence's
length are ignored; and a brute-force case matches scipy's softmax with
torch's float8 decode.
"""
import numpy as np
import pytest
import torch
from scipy.special import softmax

import oracle


def _bits(x):
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def _dec(codes):
    return torch.from_numpy(np.ascontiguousarray(codes)).view(torch.float8_e4m3fn).float().numpy().astype(np.float64)


def _cache(rng, B, S, Hkv, D=128, mode=oracle.SCALE_FP32):
    k = rng.standard_normal((B, S, Hkv, D)).astype(np.float32)
    v = rng.standard_normal((B, S, Hkv, D)).astype(np.float32)
    kq, ks = oracle.quant_kv(_bits(k), mode)
    vq, vs = oracle.quant_kv(_bits(v), mode)
    return kq, ks, vq, vs


def test_quant_kv_one_scale_per_head_vector():
    rng = np.random.default_rng(0)
    kq, ks, vq, vs = _cache(rng, 2, 5, 3)
    assert kq.shape == (2, 5, 3, 128) and ks.shape == (2, 5, 3)
    # every head vector's amax lands on +-448 (0x7E / 0xFE)
    assert np.all(np.any((kq & 0x7F) == 0x7E, axis=3))


def test_single_token_returns_its_value_vector():
    rng = np.random.default_rng(1)
    B, Hq, Hkv = 2, 4, 2
    kq, ks, vq, vs = _cache(rng, B, 3, Hkv)
    q = _bits(rng.standard_normal((B, Hq, 128)))
    o = oracle.decode_attention(q, kq, ks, vq, vs, [1, 1], 0.1)
    for b in range(B):
        for h in range(Hq):
            g = h // (Hq // Hkv)
            assert np.allclose(o[b, h], _dec(vq[b, 0, g]) * vs[b, 0, g], rtol=1e-15, atol=0)


def test_equal_values_are_returned_and_zero_query_averages():
    rng = np.random.default_rng(2)
    B, S, Hq, Hkv = 1, 37, 2, 1
    kq, ks, vq, vs = _cache(rng, B, S, Hkv)
    vq2 = np.repeat(vq[:, :1], S, axis=1)
    vs2 = np.repeat(vs[:, :1], S, axis=1)
    q = _bits(rng.standard_normal((B, Hq, 128)))
    o = oracle.decode_attention(q, kq, ks, vq2, vs2, [S], 0.2)
    ref = _dec(vq2[0, 0, 0]) * vs2[0, 0, 0]
    assert np.allclose(o[0, 0], ref, rtol=1e-13, atol=1e-15)
    z = np.zeros((B, Hq, 128), np.uint16)
    o = oracle.decode_attention(z, kq, ks, vq, vs, [S], 0.2)
    mean = np.mean(_dec(vq[0, :, 0]) * vs[0, :, 0, None], axis=0)
    assert np.allclose(o[0, 1], mean, rtol=1e-12, atol=1e-14)


def test_token_order_does_not_matter():
    rng = np.random.default_rng(3)
    B, S, Hq, Hkv = 1, 50, 4, 2
    kq, ks, vq, vs = _cache(rng, B, S, Hkv)
    q = _bits(rng.standard_normal((B, Hq, 128)))
    perm = rng.permutation(S)
    a = oracle.decode_attention(q, kq, ks, vq, vs, [S], 0.09)
    b = oracle.decode_attention(q, kq[:, perm], ks[:, perm], vq[:, perm], vs[:, perm], [S], 0.09)
    assert np.allclose(a, b, rtol=1e-12, atol=1e-14)


def test_grouped_query_heads_read_their_own_kv_head():
    # value vectors of head g are all equal to g + 1 (exact in E4M3), so every
    # query head of group g must return g + 1 whatever its weights
    rng = np.random.default_rng(4)
    B, S, Hq, Hkv = 1, 9, 8, 4
    kq, ks, _, _ = _cache(rng, B, S, Hkv)
    v = np.zeros((B, S, Hkv, 128), np.float32)
    for g in range(Hkv):
        v[:, :, g, :] = g + 1
    vq, vs = oracle.quant_kv(_bits(v), oracle.SCALE_POW2)
    q = _bits(rng.standard_normal((B, Hq, 128)))
    o = oracle.decode_attention(q, kq, ks, vq, vs, [S], 0.1)
    for h in range(Hq):
        assert np.allclose(o[0, h], h // (Hq // Hkv) + 1, rtol=1e-14, atol=0)


def test_tokens_past_the_length_are_ignored_and_empty_is_zero():
    rng = np.random.default_rng(5)
    B, S, Hq, Hkv = 3, 20, 2, 1
    kq, ks, vq, vs = _cache(rng, B, S, Hkv)
    q = _bits(rng.standard_normal((B, Hq, 128)))
    a = oracle.decode_attention(q, kq, ks, vq, vs, [7, 0, 20], 0.1)
    kq2, vq2, ks2, vs2 = kq.copy(), vq.copy(), ks.copy(), vs.copy()
    kq2[0, 7:] = 0x7E
    vq2[0, 7:] = 0x7E
    ks2[0, 7:] = 1e6
    vs2[0, 7:] = 1e6
    b = oracle.decode_attention(q, kq2, ks2, vq2, vs2, [7, 0, 20], 0.1)
    assert np.array_equal(a, b)
    assert not a[1].any()


def test_brute_force_against_scipy_softmax():
    rng = np.random.default_rng(6)
    B, S, Hq, Hkv = 2, 33, 4, 2
    kq, ks, vq, vs = _cache(rng, B, S, Hkv, mode=oracle.SCALE_POW2)
    qf = rng.standard_normal((B, Hq, 128))
    q = _bits(qf)
    lens = [33, 12]
    scale = 1.0 / np.sqrt(128.0)
    o = oracle.decode_attention(q, kq, ks, vq, vs, lens, scale)
    qd = torch.from_numpy(q.view(np.int16)).view(torch.bfloat16).double().numpy()
    for b in range(B):
        L = lens[b]
        for h in range(Hq):
            g = h // (Hq // Hkv)
            kk = _dec(kq[b, :L, g]) * ks[b, :L, g, None]
            vv = _dec(vq[b, :L, g]) * vs[b, :L, g, None]
            p = softmax(scale * (kk @ qd[b, h]))
            assert np.allclose(o[b, h], p @ vv, rtol=1e-12, atol=1e-14)


# --- causal (prefill) attention over FP8 queries, keys and values -------------

def _qkv(rng, B, S, Hq, Hkv, mode=oracle.SCALE_FP32):
    q = rng.standard_normal((B, S, Hq, 128)).astype(np.float32)
    qq, qs = oracle.quant_kv(_bits(q), mode)
    kq, ks, vq, vs = _cache(rng, B, S, Hkv, mode=mode)
    return qq, qs, kq, ks, vq, vs


def test_prefill_brute_force_against_scipy_softmax():
    # the definition evaluated independently: torch's E4M3 decode, numpy
    # products, a causal mask and scipy's softmax, row by row
    rng = np.random.default_rng(10)
    B, S, Hq, Hkv = 2, 45, 4, 2
    qq, qs, kq, ks, vq, vs = _qkv(rng, B, S, Hq, Hkv)
    lens = [45, 17]
    scale = 1.0 / np.sqrt(128.0)
    o, mag = oracle.prefill_attention(qq, qs, kq, ks, vq, vs, lens, scale, want_mag=True)
    o = o.reshape(B, S, Hq, 128)
    mag = mag.reshape(B, S, Hq, 128)
    for b in range(B):
        L = lens[b]
        for h in range(Hq):
            g = h // (Hq // Hkv)
            qd = _dec(qq[b, :L, h]) * qs[b, :L, h, None]
            kd = _dec(kq[b, :L, g]) * ks[b, :L, g, None]
            vd = _dec(vq[b, :L, g]) * vs[b, :L, g, None]
            s = scale * (qd @ kd.T)
            s[np.triu_indices(L, 1)] = -np.inf
            p = softmax(s, axis=1)
            assert np.allclose(o[b, :L, h], p @ vd, rtol=1e-12, atol=1e-14)
            assert np.allclose(mag[b, :L, h], p @ np.abs(vd), rtol=1e-12, atol=1e-14)
        assert not o[b, L:].any() and not mag[b, L:].any()


def test_prefill_first_row_is_its_own_value_and_future_keys_do_not_matter():
    rng = np.random.default_rng(11)
    B, S, Hq, Hkv = 1, 30, 4, 1
    qq, qs, kq, ks, vq, vs = _qkv(rng, B, S, Hq, Hkv)
    a = oracle.prefill_attention(qq, qs, kq, ks, vq, vs, [S], 0.1).reshape(B, S, Hq, 128)
    for h in range(Hq):
        assert np.array_equal(a[0, 0, h], _dec(vq[0, 0, 0]) * np.float64(vs[0, 0, 0]))
    # rewriting keys and values at positions > 12 leaves rows 0..12 unchanged
    kq2, vq2, ks2, vs2 = kq.copy(), vq.copy(), ks.copy(), vs.copy()
    kq2[0, 13:] = 0x7E
    vq2[0, 13:] = 0xFE
    ks2[0, 13:] = 3.0
    b = oracle.prefill_attention(qq, qs, kq2, ks2, vq2, vs2, [S], 0.1).reshape(B, S, Hq, 128)
    assert np.array_equal(a[0, :13], b[0, :13])
    assert not np.allclose(a[0, 13:], b[0, 13:])


def test_prefill_zero_query_averages_the_visible_values():
    rng = np.random.default_rng(12)
    B, S, Hq, Hkv = 1, 21, 2, 2
    qq, qs, kq, ks, vq, vs = _qkv(rng, B, S, Hq, Hkv)
    qq[:] = 0
    o = oracle.prefill_attention(qq, qs, kq, ks, vq, vs, [S], 0.3).reshape(B, S, Hq, 128)
    for i in range(S):
        for h in range(Hq):
            mean = np.mean(_dec(vq[0, :i + 1, h]) * vs[0, :i + 1, h, None], axis=0)
            assert np.allclose(o[0, i, h], mean, rtol=1e-12, atol=1e-15)


def test_prefill_last_row_equals_decode_attention():
    # with power-of-two scales a dequantized query is exactly a bf16 vector, so
    # the last prefill row must equal the (separately pinned) decode attention
    # of that query over the same cache
    rng = np.random.default_rng(13)
    B, S, Hq, Hkv = 2, 40, 8, 2
    qq, qs, kq, ks, vq, vs = _qkv(rng, B, S, Hq, Hkv, mode=oracle.SCALE_POW2)
    lens = [40, 23]
    o = oracle.prefill_attention(qq, qs, kq, ks, vq, vs, lens, 0.088).reshape(B, S, Hq, 128)
    qlast = np.stack([_dec(qq[b, lens[b] - 1]) * qs[b, lens[b] - 1, :, None] for b in range(B)])
    qb = _bits(qlast)
    assert np.array_equal(torch.from_numpy(qb.view(np.int16)).view(torch.bfloat16).double().numpy(), qlast)
    d = oracle.decode_attention(qb, kq, ks, vq, vs, lens, 0.088)
    for b in range(B):
        assert np.allclose(o[b, lens[b] - 1], d[b], rtol=1e-12, atol=1e-15)


def test_prefill_row_subset_and_grouped_heads():
    rng = np.random.default_rng(14)
    B, S, Hq, Hkv = 2, 19, 8, 4
    qq, qs, kq, ks, vq, vs = _qkv(rng, B, S, Hq, Hkv)
    full = oracle.prefill_attention(qq, qs, kq, ks, vq, vs, [19, 19], 0.1)
    rows = np.array([0, 5, 18, 19, 37])
    sub = oracle.prefill_attention(qq, qs, kq, ks, vq, vs, [19, 19], 0.1, rows=rows)
    assert np.array_equal(full[rows], sub)
    # value vectors of key/value head g all equal g + 1 (exact): every query head
    # of group g returns g + 1
    v = np.zeros((B, S, Hkv, 128), np.float32)
    for g in range(Hkv):
        v[:, :, g, :] = g + 1
    vq2, vs2 = oracle.quant_kv(_bits(v), oracle.SCALE_POW2)
    o = oracle.prefill_attention(qq, qs, kq, ks, vq2, vs2, [19, 19], 0.1).reshape(B, S, Hq, 128)
    for h in range(Hq):
        assert np.allclose(o[:, :, h], h // (Hq // Hkv) + 1, rtol=1e-14, atol=0)
