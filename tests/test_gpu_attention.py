"""GPU parity of the FP8 KV cache (append: bit-exact codes and scales) and of
decode attention over it (within the GEMM tolerance against the oracle's
double-precision attention of the same cached codes).
"""
import math

import numpy as np
import pytest
import torch

import fp8_block_scaled_fp8bq_b200 as fq
import oracle
from helpers import assert_gemm_close, bf16_bits, bf16_to_f64, f32, need_gpu, u8

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _gpu_and_clean_error_word():
    need_gpu()
    yield
    st, word = fq.device_error()
    assert st == 0 and word == 0, "device error word 0x%x" % word


def _bf16(shape, seed, scale=1.0):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(shape, generator=g) * scale).to(torch.bfloat16)


def _cache(B, S, Hkv, seed, mode=fq.SCALE_FP32):
    """Seeded bf16 keys/values [B, S, Hkv, 128] quantized by the oracle."""
    k = _bf16((B, S, Hkv, 128), seed)
    v = _bf16((B, S, Hkv, 128), seed + 1)
    kq, ks = oracle.quant_kv(bf16_bits(k), mode)
    vq, vs = oracle.quant_kv(bf16_bits(v), mode)
    return kq, ks, vq, vs


def _run(q, kq, ks, vq, vs, lens, scale):
    dev = [torch.from_numpy(np.ascontiguousarray(a)).cuda() for a in (kq, ks, vq, vs)]
    ln = torch.tensor(lens, dtype=torch.int32).cuda()
    o = fq.decode_attention(q.cuda(), *dev, ln, scale)
    torch.cuda.synchronize()
    return bf16_to_f64(o)


@pytest.mark.parametrize("G", [1, 2, 4, 8])
def test_decode_attention_against_oracle(G):
    B, Hkv, S = 3, 2, 300
    Hq = G * Hkv
    kq, ks, vq, vs = _cache(B, S, Hkv, seed=G)
    q = _bf16((B, Hq, 128), seed=100 + G)
    lens = [300, 1, 173]
    scale = 1.0 / math.sqrt(128.0)
    got = _run(q, kq, ks, vq, vs, lens, scale)
    ref = oracle.decode_attention(bf16_bits(q), kq, ks, vq, vs, lens, scale)
    assert_gemm_close(got, ref, "decode attention G=%d" % G)


def test_empty_and_overlong_sequences():
    B, Hkv, Hq, S = 3, 1, 4, 64
    kq, ks, vq, vs = _cache(B, S, Hkv, seed=7)
    q = _bf16((B, Hq, 128), seed=8)
    got = _run(q, kq, ks, vq, vs, [0, 1000, 64], 0.1)
    assert not got[0].any()
    ref = oracle.decode_attention(bf16_bits(q), kq, ks, vq, vs, [0, 64, 64], 0.1)
    assert_gemm_close(got[1:], ref[1:], "clamped length")


def test_peaked_scores_pick_one_token():
    # one key equals the query direction with a large scale: softmax ~ one-hot
    B, Hkv, Hq, S = 1, 1, 1, 500
    k = torch.zeros((B, S, Hkv, 128))
    q = torch.ones((B, Hq, 128)).to(torch.bfloat16)
    k[0, 321, 0, :] = 1.0
    v = _bf16((B, S, Hkv, 128), seed=9)
    kq, ks = oracle.quant_kv(bf16_bits(k.to(torch.bfloat16)), fq.SCALE_POW2)
    vq, vs = oracle.quant_kv(bf16_bits(v), fq.SCALE_POW2)
    got = _run(q, kq, ks, vq, vs, [S], 1.0)
    ref = oracle.decode_attention(bf16_bits(q), kq, ks, vq, vs, [S], 1.0)
    assert_gemm_close(got, ref, "one-hot")


def test_value_scales_spanning_decades():
    # value vectors whose magnitudes grow and shrink over 2^-12 .. 2^12 along
    # the sequence: the largest value scale seen so far changes many times
    B, Hkv, Hq, S = 2, 2, 8, 700
    k = _bf16((B, S, Hkv, 128), seed=31)
    v = _bf16((B, S, Hkv, 128), seed=32).float()
    t = torch.arange(S, dtype=torch.float32)
    mag = torch.exp2(12.0 * torch.sin(t / 37.0))[None, :, None, None]
    v = (v * mag).to(torch.bfloat16)
    kq, ks = oracle.quant_kv(bf16_bits(k), fq.SCALE_FP32)
    vq, vs = oracle.quant_kv(bf16_bits(v), fq.SCALE_FP32)
    q = _bf16((B, Hq, 128), seed=33, scale=0.3)
    got = _run(q, kq, ks, vq, vs, [S, 517], 0.125)
    ref = oracle.decode_attention(bf16_bits(q), kq, ks, vq, vs, [S, 517], 0.125)
    assert_gemm_close(got, ref, "value scales over decades")


@pytest.mark.parametrize("qscale", [0.0, 1e-30, 1e-6, 1e3, 1e20])
def test_query_magnitudes(qscale):
    # the per-head power-of-two scaling of the query keeps tiny and huge
    # queries exact; a zero query averages the values
    B, Hkv, Hq, S = 2, 2, 4, 200
    kq, ks, vq, vs = _cache(B, S, Hkv, seed=41)
    q = (_bf16((B, Hq, 128), seed=42).float() * qscale).to(torch.bfloat16)
    q[1, 3] = _bf16((128,), seed=43)  # one head of ordinary size beside them
    got = _run(q, kq, ks, vq, vs, [S, 150], 0.09)
    ref = oracle.decode_attention(bf16_bits(q), kq, ks, vq, vs, [S, 150], 0.09)
    assert_gemm_close(got, ref, "query scale %g" % qscale)


@pytest.mark.parametrize("mode", [fq.SCALE_FP32, fq.SCALE_POW2])
def test_kv_append_bit_exact(mode):
    B, Hkv, S = 4, 8, 40
    kq = torch.full((B, S, Hkv, 128), 0x55, dtype=torch.uint8, device="cuda")
    vq = torch.full((B, S, Hkv, 128), 0x55, dtype=torch.uint8, device="cuda")
    ks = torch.full((B, S, Hkv), 7.0, dtype=torch.float32, device="cuda")
    vs = torch.full((B, S, Hkv), 7.0, dtype=torch.float32, device="cuda")
    k_new = _bf16((B, Hkv, 128), seed=11, scale=3.0)
    v_new = _bf16((B, Hkv, 128), seed=12)
    pos = [0, 17, 39, 40]                          # the last one is outside the cache
    fq.kv_cache_append(k_new.cuda(), v_new.cuda(), torch.tensor(pos, dtype=torch.int32).cuda(), kq, ks, vq, vs, mode)
    torch.cuda.synchronize()
    ok_, oks = oracle.quant_act(bf16_bits(k_new.reshape(B * Hkv, 128)), mode)
    ov_, ovs = oracle.quant_act(bf16_bits(v_new.reshape(B * Hkv, 128)), mode)
    ok_, ov_ = ok_.reshape(B, Hkv, 128), ov_.reshape(B, Hkv, 128)
    oks, ovs = oks[0, :B * Hkv].reshape(B, Hkv), ovs[0, :B * Hkv].reshape(B, Hkv)
    gk, gv, gks, gvs = u8(kq), u8(vq), f32(ks), f32(vs)
    for b, t in enumerate(pos):
        if t < S:
            assert np.array_equal(gk[b, t], ok_[b]) and np.array_equal(gv[b, t], ov_[b])
            assert np.array_equal(gks[b, t].view(np.uint32), oks[b].view(np.uint32))
            assert np.array_equal(gvs[b, t].view(np.uint32), ovs[b].view(np.uint32))
    untouched = np.ones((B, S), bool)
    for b, t in enumerate(pos):
        if t < S:
            untouched[b, t] = False
    assert np.all(gk[untouched] == 0x55) and np.all(gks[untouched] == 7.0)


def test_llama8b_decode_batch16_context8192():
    """Llama-3.1-8B attention shape (32 query heads, 8 key/value heads, D = 128)
    over an 8192-token FP8 cache for 16 sequences; the oracle recomputes two
    sequences in full."""
    B, S, Hkv, Hq = 16, 8192, 8, 32
    kq, ks, vq, vs = _cache(B, S, Hkv, seed=21)
    q = _bf16((B, Hq, 128), seed=22)
    lens = [S - 37 * b for b in range(B)]
    scale = 1.0 / math.sqrt(128.0)
    got = _run(q, kq, ks, vq, vs, lens, scale)
    for b in (0, 13):
        ref = oracle.decode_attention(bf16_bits(q[b:b + 1]), kq[b:b + 1], ks[b:b + 1], vq[b:b + 1], vs[b:b + 1],
                                      [lens[b]], scale)
        assert_gemm_close(got[b:b + 1], ref, "llama decode b=%d" % b)


@pytest.mark.parametrize("B,Hkv,Hq,S", [(1, 1, 8, 20000),     # one head: many splits of one sequence
                                         (40, 4, 16, 900)])     # more heads than SMs: whole or few splits
def test_split_regimes(B, Hkv, Hq, S):
    kq, ks, vq, vs = _cache(B, S, Hkv, seed=51)
    q = _bf16((B, Hq, 128), seed=52)
    lens = [S - (97 * b) % S for b in range(B)]
    scale = 1.0 / math.sqrt(128.0)
    got = _run(q, kq, ks, vq, vs, lens, scale)
    for b in sorted({0, B // 2, B - 1}):
        ref = oracle.decode_attention(bf16_bits(q[b:b + 1]), kq[b:b + 1], ks[b:b + 1], vq[b:b + 1], vs[b:b + 1],
                                      [lens[b]], scale)
        assert_gemm_close(got[b:b + 1], ref, "b=%d" % b)


def test_workspace_too_small():
    B, Hkv, Hq, S = 2, 2, 4, 512
    kq = torch.zeros((B, S, Hkv, 128), dtype=torch.uint8, device="cuda")
    ks = torch.ones((B, S, Hkv), dtype=torch.float32, device="cuda")
    q = torch.zeros((B, Hq, 128), dtype=torch.bfloat16, device="cuda")
    lens = torch.tensor([S, S], dtype=torch.int32, device="cuda")
    need = int(fq.lib().fp8bq_decode_attention_workspace_size(B, Hq, Hkv, S))
    small = torch.empty(max(16, need - 16), dtype=torch.uint8, device="cuda")
    with pytest.raises(fq.Fp8bqError) as e:
        fq.decode_attention(q, kq, ks, kq, ks, lens, 0.1, ws=small)
    assert e.value.status == 4
