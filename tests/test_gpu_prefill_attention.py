"""GPU parity of the causal (prefill) FP8 attention against the oracle's
double-precision attention of the same E4M3 codes and scales.

The kernel feeds the softmax weights to the value product as E4M3 codes (the
FP8 attention of section "Real-world performance gains": both contractions on
FP8 operands), so the comparison bound is derived from that arithmetic,
element by element:
  |o_gpu - o| <= sum_j e_j (vmax_j / 256) |v_jd| / l      (E4M3 rounding of each weight)
               + 2^-11 sum_j p_j |v_jd|                    (FP32 scores and sums, exp2)
               + 2^-8 |o|                                  (bf16 output)
where the weight of key j in the kernel's units is w_j = 2^(s_j - max s) * 256
vs_j / vmax_j (vmax_j: the largest value scale among the valid keys of j's
128-key block), e_j = max(2^-4 w_j, 2^-10) is the largest E4M3 rounding error
at w_j (half a step: 2^-4 of the value in the normal range, 2^-10 below it),
and l = sum_j 2^(s_j - max s).  A case with exactly representable weights and
values is compared bit for bit.
"""
import math

import numpy as np
import pytest
import torch

import fp8_block_scaled_fp8bq_b200 as fq
import oracle
from helpers import bf16_bits, bf16_to_f64, need_gpu

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _gpu_and_clean_error_word():
    need_gpu()
    yield
    st, word = fq.device_error()
    assert st == 0 and word == 0, "device error word 0x%x" % word


def _dec(codes):
    return torch.from_numpy(np.ascontiguousarray(codes)).view(torch.float8_e4m3fn).double().numpy()


def _inputs(B, S, Hq, Hkv, seed, mode=fq.SCALE_FP32, qscale=1.0):
    g = torch.Generator().manual_seed(seed)
    q = (torch.randn((B, S, Hq, 128), generator=g) * qscale).to(torch.bfloat16)
    k = torch.randn((B, S, Hkv, 128), generator=g).to(torch.bfloat16)
    v = torch.randn((B, S, Hkv, 128), generator=g).to(torch.bfloat16)
    qq, qs = oracle.quant_kv(bf16_bits(q), mode)
    kq, ks = oracle.quant_kv(bf16_bits(k), mode)
    vq, vs = oracle.quant_kv(bf16_bits(v), mode)
    return qq, qs, kq, ks, vq, vs


def _run(qq, qs, kq, ks, vq, vs, lens, scale):
    dev = [torch.from_numpy(np.ascontiguousarray(a)).cuda() for a in (qq, qs, kq, ks, vq, vs)]
    ln = torch.tensor(lens, dtype=torch.int32).cuda()
    o = fq.prefill_attention(*dev, ln, scale)
    torch.cuda.synchronize()
    return o


def _bound(qq, qs, kq, ks, vq, vs, lens, scale, rows, ref, mag):
    """The per-element bound above for the flat query rows `rows` (b * S + i)."""
    B, S, Hq, _ = qq.shape
    Hkv = kq.shape[2]
    out = np.zeros((len(rows), Hq, 128))
    for n, bi in enumerate(rows):
        b, i = divmod(int(bi), S)
        L = min(max(lens[b], 0), S)
        if i >= L:
            continue
        kd = _dec(kq[b, :i + 1])                      # [i+1, Hkv, 128]
        vd = np.abs(_dec(vq[b, :i + 1]))
        vmax = np.zeros((i + 1, Hkv))
        for kb in range(0, i + 1, 128):
            hi = min(kb + 128, L)
            vmax[kb:min(kb + 128, i + 1)] = vs[b, kb:hi].max(axis=0)
        for h in range(Hq):
            g = h // (Hq // Hkv)
            qd = _dec(qq[b, i, h])
            s = scale * float(qs[b, i, h]) * ks[b, :i + 1, g].astype(np.float64) * (kd[:, g] @ qd)
            pt = np.exp(s - s.max())
            l = pt.sum()
            w = pt * 256.0 * vs[b, :i + 1, g] / vmax[:, g]
            e = np.maximum(2.0 ** -4 * w, 2.0 ** -10)
            out[n, h] = (e * vmax[:, g] / 256.0) @ vd[:, g] / l
    return out + 2.0 ** -11 * mag + 2.0 ** -8 * np.abs(ref) + 1e-30


def _check(got, ref, bound, what):
    """Every element within its bound; and the errors are not all pushed to
    the bound (a systematic bias, e.g. a misplaced scale that happens to stay
    inside it, would be): their mean is at most 0.6 of the bound's mean."""
    err = np.abs(got - ref)
    worst = float(np.max(err / bound)) if err.size else 0.0
    assert worst <= 1.0, "%s: error %.3g x the derived bound" % (what, worst)
    live = np.abs(ref) > 0
    assert err[live].mean() <= 0.6 * bound[live].mean(), "%s: mean error %.3g vs mean bound %.3g" % (
        what, err[live].mean(), bound[live].mean())
    fro = np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-300)
    print("%s: relative Frobenius error %.4f, worst %.3f of the bound" % (what, fro, worst))


@pytest.mark.parametrize("G,S,lens", [(1, 300, [300, 137]), (4, 300, [300, 1]), (8, 257, [129, 257]),
                                      (2, 128, [128, 127])])
def test_prefill_attention_against_oracle(G, S, lens):
    B, Hkv = 2, 2
    Hq = G * Hkv
    qq, qs, kq, ks, vq, vs = _inputs(B, S, Hq, Hkv, seed=G + S)
    scale = 1.0 / math.sqrt(128.0)
    o = _run(qq, qs, kq, ks, vq, vs, lens, scale)
    got = bf16_to_f64(o).reshape(B * S, Hq, 128)
    ref, mag = oracle.prefill_attention(qq, qs, kq, ks, vq, vs, lens, scale, want_mag=True)
    rows = np.arange(B * S)
    _check(got, ref, _bound(qq, qs, kq, ks, vq, vs, lens, scale, rows, ref, mag), "G=%d S=%d" % (G, S))
    # rows at or past a sequence's length are zero
    for b in range(B):
        assert not got[b * S + lens[b]:(b + 1) * S].any()


def test_prefill_attention_sharp_and_power_of_two_scales():
    # larger query magnitudes make the softmax peaked (most weights far below
    # the E4M3 normal range); power-of-two scales
    B, S, Hq, Hkv = 1, 384, 4, 1
    qq, qs, kq, ks, vq, vs = _inputs(B, S, Hq, Hkv, seed=7, mode=fq.SCALE_POW2, qscale=4.0)
    scale = 1.0 / math.sqrt(128.0)
    lens = [S]
    got = bf16_to_f64(_run(qq, qs, kq, ks, vq, vs, lens, scale)).reshape(S, Hq, 128)
    ref, mag = oracle.prefill_attention(qq, qs, kq, ks, vq, vs, lens, scale, want_mag=True)
    _check(got, ref, _bound(qq, qs, kq, ks, vq, vs, lens, scale, np.arange(S), ref, mag), "sharp")


def test_prefill_attention_exact_uniform_rows():
    # zero queries: every visible key has weight 2^0 = 1, so each P' code is
    # exactly 256 when all value scales are equal; small integer value codes
    # keep every FP32 sum exact; rows with a power-of-two key count divide
    # exactly.  Those rows must equal the oracle's bf16 result bit for bit.
    B, S, Hq, Hkv = 1, 512, 2, 1
    qq = np.zeros((B, S, Hq, 128), np.uint8)
    qs = np.ones((B, S, Hq), np.float32)
    rng = np.random.default_rng(3)
    kq = rng.integers(0, 0x70, size=(B, S, Hkv, 128), dtype=np.uint8)
    ks = np.full((B, S, Hkv), 0.5, np.float32)
    vals = rng.integers(-8, 9, size=(B, S, Hkv, 128)).astype(np.float32)
    vq = torch.from_numpy(vals).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(_dec(vq), vals)
    vs = np.full((B, S, Hkv), 0.25, np.float32)
    got = _run(qq, qs, kq, ks, vq, vs, [S], 0.1)
    ref = oracle.prefill_attention(qq, qs, kq, ks, vq, vs, [S], 0.1)
    ref_bits = oracle.f64_to_bf16(ref)
    got_bits = bf16_bits(got).reshape(S, Hq, 128)
    for i in (0, 1, 3, 7, 15, 31, 63, 127, 255, 511):
        assert np.array_equal(got_bits[i], ref_bits[i]), "row %d" % i


def test_prefill_attention_llama8b_heads_full_size_sampled_rows():
    # Llama-3.1-8B attention (32 query heads, 8 key/value heads, D = 128) over
    # 4 sequences of 2048 tokens: two rows of every 128-row tile of each
    # sequence (its first and last), all heads, against the oracle
    B, S, Hq, Hkv = 4, 2048, 32, 8
    qq, qs, kq, ks, vq, vs = _inputs(B, S, Hq, Hkv, seed=11)
    lens = [2048, 2048, 1500, 700]
    scale = 1.0 / math.sqrt(128.0)
    got = bf16_to_f64(_run(qq, qs, kq, ks, vq, vs, lens, scale)).reshape(B * S, Hq, 128)
    rows = np.array(sorted({b * S + min(t * 128 + o, S - 1) for b in range(B) for t in range(S // 128)
                            for o in (0, 127)} | {2 * S + 1499, 3 * S + 699, 3 * S + 700}))
    ref, mag = oracle.prefill_attention(qq, qs, kq, ks, vq, vs, lens, scale, rows=rows, want_mag=True)
    _check(got[rows], ref, _bound(qq, qs, kq, ks, vq, vs, lens, scale, rows, ref, mag), "llama8b")
    for b in range(B):
        assert not got[b * S + lens[b]:(b + 1) * S].any()
