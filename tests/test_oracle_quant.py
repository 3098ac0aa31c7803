"""Pins of the oracle's scales and quantizers.

Expected values here come from library routines and invariants, never from the
oracle's own encoder or scale code: numpy float32 division (IEEE binary32),
torch's float8_e4m3fn cast, exact rational arithmetic (fractions), and the
error bound of a round-to-nearest 3-bit-mantissa format.
"""
import math
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
import fp8bq_workloads as wl

FP32, POW2 = oracle.SCALE_FP32, oracle.SCALE_POW2


def all_positive_bf16():
    bits = np.arange(1, 0x7F80, dtype=np.uint16)          # +denormals .. max finite
    return bits, oracle.bf16_to_f32(bits)


def torch_encode(q32):
    """E4M3 code of float32 values via torch (defined the same way for |v| <= 464)."""
    q32 = np.asarray(q32, dtype=np.float32)
    assert np.all(np.abs(q32[np.isfinite(q32)]) <= 464.0)
    return torch.from_numpy(q32.copy()).to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def pow2_exponent_exact(amax):
    """Smallest integer e with amax <= 448 * 2^e, by exact rational arithmetic."""
    f = Fraction(float(amax)) / 448
    e = f.numerator.bit_length() - f.denominator.bit_length()
    while Fraction(2) ** e < f:
        e += 1
    while Fraction(2) ** (e - 1) >= f:
        e -= 1
    return max(-127, min(127, e))


def test_fp32_scale_is_ieee_division_for_every_bf16_amax():
    _, a = all_positive_bf16()
    s = np.array([oracle.scale(v, FP32) for v in a[::7]], dtype=np.float32)
    ref = a[::7] / np.float32(448.0)                      # numpy binary32 division
    assert np.array_equal(s.view(np.uint32), ref.view(np.uint32))
    assert oracle.scale(0.0, FP32) == 1.0


def test_fp32_scale_maps_amax_to_top_code():
    _, a = all_positive_bf16()
    s = a / np.float32(448.0)
    q = a / s                                             # float32 quotient
    normal = s >= np.float32(2.0 ** -126)
    assert np.all(q[normal] <= np.float32(448.0) * np.float32(1 + 2 ** -22))
    # a denormal scale loses relative precision, but the quotient stays in
    # (432, 464], all of which encodes to 448
    assert np.all(q > 432.0) and np.all(q <= 464.0)
    assert np.all(torch_encode(q) == 0x7E)


def test_pow2_scale_invariants_every_bf16_amax():
    _, a = all_positive_bf16()
    for v in a[::3]:
        s = oracle.scale(v, POW2)
        m, e = math.frexp(s)
        assert m == 0.5, "scale must be a power of two"
        e = e - 1
        assert e == pow2_exponent_exact(v)
        if -127 < e:
            # unique exponent: amax/s in (224, 448]
            r = Fraction(float(v)) / Fraction(s)
            assert 224 < r <= 448
    assert oracle.scale(0.0, POW2) == 1.0


def test_pow2_scale_clamps_at_minus_127():
    tiny = np.float32(1e-40)                               # below 448 * 2^-127
    assert oracle.scale(tiny, POW2) == 2.0 ** -127


def _tile_reference(x32, mode):
    """Codes and scale of one tile from library routines only."""
    amax = np.float32(np.max(np.abs(x32))) if x32.size else np.float32(0)
    if amax == 0:
        s = np.float32(1.0)
    elif mode == FP32:
        s = np.float32(amax / np.float32(448.0))
    else:
        s = np.float32(2.0 ** pow2_exponent_exact(amax))
    q = x32 / s                                            # numpy float32 division
    return torch_encode(q), s


@pytest.mark.parametrize("mode", [FP32, POW2])
def test_quant_act_against_library_routines(mode):
    x = wl.activations(37, 300, seed=5, n_out=3)           # ragged last 1x128 tile (44 wide)
    xb = x.view(torch.int16).numpy().view(np.uint16)
    q, sa = oracle.quant_act(xb, mode)
    x32 = oracle.bf16_to_f32(xb)
    for m in range(37):
        for kb in range(3):
            k0, k1 = 128 * kb, min(128 * kb + 128, 300)
            rq, rs = _tile_reference(x32[m, k0:k1], mode)
            assert sa[kb, m] == rs
            assert np.array_equal(q[m, k0:k1], rq), (m, kb)


@pytest.mark.parametrize("mode", [FP32, POW2])
def test_quant_weight_against_library_routines(mode):
    w = wl.weights(200, 300, seed=6)                       # 2x3 tiles, both edges ragged
    wb = w.view(torch.int16).numpy().view(np.uint16)
    q, sw = oracle.quant_weight(wb, mode)
    w32 = oracle.bf16_to_f32(wb)
    assert sw.shape == (2, 3)
    for nb in range(2):
        for kb in range(3):
            n0, n1 = 128 * nb, min(128 * nb + 128, 200)
            k0, k1 = 128 * kb, min(128 * kb + 128, 300)
            rq, rs = _tile_reference(w32[n0:n1, k0:k1].ravel(), mode)
            assert sw[nb, kb] == rs
            assert np.array_equal(q[n0:n1, k0:k1].ravel(), rq), (nb, kb)


@pytest.mark.parametrize("mode", [FP32, POW2])
def test_quant_error_bound(mode):
    x = wl.activations(64, 512, seed=9, n_out=4)
    xb = x.view(torch.int16).numpy().view(np.uint16)
    q, sa = oracle.quant_act(xb, mode)
    x64 = oracle.bf16_to_f32(xb).astype(np.float64)
    d = oracle.dequant_act(q, sa)
    s = np.repeat(sa.T.astype(np.float64), 128, axis=1)     # [M, K] per-element scale
    bound = np.maximum(2.0 ** -4 * np.abs(x64), 2.0 ** -10 * s) * (1 + 2.0 ** -20)
    assert np.all(np.abs(x64 - d) <= bound)
    # the element holding each tile's amax lands on +-448 (fp32) or in [224, 448] (pow2)
    x3 = np.abs(x64).reshape(64, 4, 128)
    idx = np.argmax(x3, axis=2)
    top = q.reshape(64, 4, 128)[np.arange(64)[:, None], np.arange(4)[None, :], idx] & 0x7F
    if mode == FP32:
        assert np.all(top == 0x7E)
    else:
        assert np.all(top >= 0x76) and np.all(top <= 0x7E)   # 224 = 0x76


def test_zero_tile_and_signed_zero():
    x = np.zeros((2, 128), dtype=np.uint16)
    x[1, 5] = 0x8000                                      # -0.0
    for mode in (FP32, POW2):
        q, sa = oracle.quant_act(x, mode)
        assert np.all(sa == 1.0)
        assert q[1, 5] == 0x80 and q[0, 5] == 0x00
        assert np.count_nonzero(q) == 1


def test_negative_underflow_keeps_sign():
    x = np.zeros((1, 128), dtype=np.uint16)
    x[0, 0] = np.float32(448.0).view(np.uint32) >> 16     # amax 448 -> s = 1 (fp32)
    x[0, 1] = np.float32(-1e-4).view(np.uint32) >> 16     # |q| < 2^-10 -> signed zero
    q, sa = oracle.quant_act(x, FP32)
    assert sa[0, 0] == 1.0
    assert q[0, 0] == 0x7E and q[0, 1] == 0x80


def test_recalibration_is_pure_function_of_weights():
    w = wl.weights(256, 256, seed=3)
    w2 = wl.weight_step(w, seed=4)
    wb = w.view(torch.int16).numpy().view(np.uint16)
    wb2 = w2.view(torch.int16).numpy().view(np.uint16)
    q1, s1 = oracle.quant_weight(wb2, POW2)
    oracle.quant_weight(wb, POW2)
    q2, s2 = oracle.quant_weight(wb2, POW2)
    assert np.array_equal(q1, q2) and np.array_equal(s1, s2)
    assert not np.array_equal(wb, wb2)
