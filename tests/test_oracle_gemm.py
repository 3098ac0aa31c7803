"""Pins of the oracle's block-scaled GEMM and grouped GEMM.

- integer-valued codes with unit scales: the result is an integer matmul
  (numpy int64), exact;
- distinct power-of-two scales per (row, K-block) and per (N-block, K-block)
  on codes of a narrow exponent range: every double sum is exact, so numpy's
  float64 matmul of operands dequantized through torch's float8 cast must agree
  bit for bit; non-square shapes catch a transposed operand or scale table;
- the two oracle formulations (per-element double, per-block integer) agree;
- the grouped GEMM equals the dense oracle on each expert's row range,
  including empty and single-row experts.
"""
import numpy as np
import pytest
import torch

import oracle
import fp8bq_workloads as wl


def torch_decode(codes):
    t = torch.from_numpy(np.ascontiguousarray(codes, dtype=np.uint8))
    return t.view(torch.float8_e4m3fn).to(torch.float64).numpy()


def int_codes(rng, shape, vmax):
    """Codes of integers in [-vmax, vmax] (exact in E4M3 for vmax <= 16), from torch's cast."""
    v = rng.integers(-vmax, vmax + 1, size=shape).astype(np.float32)
    return torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy(), v


def test_gemm_integer_exact():
    rng = np.random.default_rng(0)
    M, N, K = 70, 200, 384
    qa, va = int_codes(rng, (M, K), 16)
    qw, vw = int_codes(rng, (N, K), 16)
    sa = np.ones((K // 128, M), dtype=np.float32)
    sw = np.ones((2, K // 128), dtype=np.float32)
    ref = va.astype(np.int64) @ vw.astype(np.int64).T
    for blockint in (False, True):
        y = oracle.gemm(qa, sa, qw, sw, blockint=blockint)
        assert np.array_equal(y, ref.astype(np.float64))


def narrow_codes(rng, shape):
    """Random codes with exponent field in [4, 11] (values in [2^-3, 2^5)), random signs."""
    E = rng.integers(4, 12, size=shape)
    m = rng.integers(0, 8, size=shape)
    s = rng.integers(0, 2, size=shape)
    return ((s << 7) | (E << 3) | m).astype(np.uint8)


def test_gemm_pow2_block_scales_exact_and_indexed():
    rng = np.random.default_rng(1)
    M, N, K = 136, 384, 512                                   # NB=3, KB=4, ragged M
    KB, NB = K // 128, N // 128
    qa = narrow_codes(rng, (M, K))
    qw = narrow_codes(rng, (N, K))
    m_idx = np.arange(M)[None, :]
    kb_idx = np.arange(KB)[:, None]
    sa = (2.0 ** ((m_idx + kb_idx) % 5)).astype(np.float32)  # [KB, M]
    nb_idx = np.arange(NB)[:, None]
    sw = (2.0 ** (nb_idx - 2 * np.arange(KB)[None, :])).astype(np.float32)  # [NB, KB]
    da = torch_decode(qa) * np.repeat(sa.T.astype(np.float64), 128, axis=1)
    dw = torch_decode(qw) * np.repeat(np.repeat(sw.astype(np.float64), 128, axis=0), 128, axis=1)
    ref = da @ dw.T                                          # exact: spread < 2^53
    for blockint in (False, True):
        y = oracle.gemm(qa, sa, qw, sw, blockint=blockint)
        assert np.array_equal(y, ref)
    # swapping the roles of the two scale tables must change the answer
    sw_t = sw[::-1].copy()
    assert not np.array_equal(oracle.gemm(qa, sa, qw, sw_t), ref)


def test_gemm_formulations_agree_on_random_data():
    x = wl.activations(48, 512, seed=2, n_out=4)
    w = wl.weights(256, 512, seed=3)
    xb = x.view(torch.int16).numpy().view(np.uint16)
    wb = w.view(torch.int16).numpy().view(np.uint16)
    qa, sa = oracle.quant_act(xb, oracle.SCALE_FP32)
    qw, sw = oracle.quant_weight(wb, oracle.SCALE_FP32)
    y1 = oracle.gemm(qa, sa, qw, sw)
    y2 = oracle.gemm(qa, sa, qw, sw, blockint=True)
    assert np.max(np.abs(y1 - y2)) <= 1e-12 * np.max(np.abs(y1))
    # and both equal numpy's matmul of the oracle's dequantized operands to rounding
    ref = oracle.dequant_act(qa, sa) @ oracle.dequant_weight(qw, sw).T
    assert np.max(np.abs(y1 - ref)) <= 1e-12 * np.max(np.abs(ref))
    # row subsets give the same rows
    rows = np.array([47, 0, 13])
    assert np.array_equal(oracle.gemm(qa, sa, qw, sw, rows=rows), y1[rows])


def test_dequant_uses_torch_values():
    rng = np.random.default_rng(4)
    q = narrow_codes(rng, (3, 256))
    sa = np.array([[0.5, 2.0, 4.0], [8.0, 0.25, 1.0]], dtype=np.float32)
    d = oracle.dequant_act(q, sa)
    ref = torch_decode(q) * np.repeat(sa.T.astype(np.float64), 128, axis=1)
    assert np.array_equal(d, ref)


def test_grouped_matches_dense_per_expert():
    rng = np.random.default_rng(5)
    E, N, K = 5, 256, 256
    counts = np.array([0, 1, 130, 0, 7])
    offsets = np.concatenate([[0], np.cumsum(counts)])
    R = int(offsets[-1])
    qa = narrow_codes(rng, (R, K))
    sa = (2.0 ** rng.integers(-3, 3, size=(K // 128, R))).astype(np.float32)
    qw = narrow_codes(rng, (E, N, K))
    sw = (2.0 ** rng.integers(-3, 3, size=(E, N // 128, K // 128))).astype(np.float32)
    y = oracle.grouped_gemm(qa, sa, qw, sw, offsets)
    for e in range(E):
        r0, r1 = offsets[e], offsets[e + 1]
        if r1 == r0:
            continue
        ref = oracle.gemm(qa[r0:r1], np.ascontiguousarray(sa[:, r0:r1]), qw[e], sw[e])
        assert np.array_equal(y[r0:r1], ref), e
    rows = np.array([0, R - 1, 5])
    assert np.array_equal(oracle.grouped_gemm(qa, sa, qw, sw, offsets, rows=rows), y[rows])


@pytest.mark.parametrize("vals", [
    [1.0, -2.5, 0.0, -0.0, 3.140625, 1e-40, 65504.0, 3.0e38],
])
def test_f64_to_bf16_against_torch(vals):
    rng = np.random.default_rng(6)
    v = np.concatenate([np.array(vals, dtype=np.float32),
                        rng.standard_normal(100000).astype(np.float32) * 1e3,
                        (rng.integers(0, 1 << 32, 100000, dtype=np.uint64)
                         .astype(np.uint32).view(np.float32))])
    v = v[np.isfinite(v)]
    # float32 inputs: double -> bf16 is a single rounding, as is torch's float -> bf16
    mine = oracle.f64_to_bf16(v.astype(np.float64))
    ref = torch.from_numpy(v.copy()).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(mine, ref)


def test_f64_to_bf16_ties():
    one = 1.0
    ulp = 2.0 ** -7
    assert oracle.f64_to_bf16(one + ulp / 2) == 0x3F80                # tie -> even (1.0)
    assert oracle.f64_to_bf16(one + 3 * ulp / 2) == 0x3F82            # tie -> even (1+2ulp)
    assert oracle.f64_to_bf16(one + ulp / 2 + 2.0 ** -40) == 0x3F81   # just above the tie
