"""Pins of the oracle's gate/up activation (SwiGLU) and of the composition the
fused gate+up epilogue is compared with.

SwiGLU is the feed-forward activation of the Llama 3.1 8B model named in
section "Technical breakthrough" of "NVIDIA NeMo RL Achieves 48% Speedup With
End-to-End FP8 Precision Training"; the same section keeps non-linear
functions in BF16.  silu(g) = g * sigmoid(g) (N. Shazeer, "GLU Variants
Improve Transformer", 2020).  The pins are facts of the mathematics, not the
formula retyped: an odd-part identity, the closed-form minimum, an exact
sigmoid value, the limits, and exact scaling and sign laws of the product.
"""
import math

import numpy as np
import pytest
from scipy.special import lambertw

import oracle


def bf16_bits(x):
    """float64 values -> bf16 bit patterns (the oracle's single RNE rounding)."""
    return oracle.f64_to_bf16(np.asarray(x, dtype=np.float64))


def bf16_to_f64(bits):
    return oracle.bf16_to_f32(bits).astype(np.float64)


pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


def test_silu_odd_part_identity():
    # g*s(g) - (-g)*s(-g) = g (s(g) + s(-g)) = g, since s(g) + s(-g) = 1.
    # A sign slip in the exponent gives -g instead.
    for g in np.linspace(-30.0, 30.0, 601):
        d = oracle.silu(g) - oracle.silu(-g)
        assert abs(d - g) <= 4e-16 * max(1.0, abs(g)), g


def test_silu_minimum_is_minus_lambert_w_of_1_over_e():
    # silu'(x) = 0 at x* = -(1 + W(1/e)) where silu(x*) = -W(1/e).
    w = float(lambertw(1.0 / math.e).real)
    x_star = -(1.0 + w)
    assert abs(oracle.silu(x_star) - (-w)) <= 1e-15
    grid = np.linspace(-3.0, 1.0, 40001)
    vals = np.array([oracle.silu(x) for x in grid])
    i = int(np.argmin(vals))
    assert abs(grid[i] - x_star) <= 2e-4
    assert vals[i] >= -w - 1e-15


def test_silu_exact_sigmoid_value():
    # sigmoid(ln 3) = 3/4 exactly.
    x = math.log(3.0)
    assert abs(oracle.silu(x) - 0.75 * x) <= 2e-16


def test_silu_limits_and_zero():
    assert oracle.silu(0.0) == 0.0
    assert oracle.silu(40.0) == 40.0                    # 1 + e^-40 rounds to 1 in double
    assert abs(oracle.silu(-40.0) - (-40.0 * math.exp(-40.0))) <= 1e-15 * 40.0 * math.exp(-40.0)
    assert oracle.silu(-1e6) == 0.0 or oracle.silu(-1e6) == -0.0
    assert oracle.silu(1.0) > 0.73 and oracle.silu(1.0) < 0.74


def _bf16_grid(seed, n):
    rng = np.random.default_rng(seed)
    return bf16_bits(rng.standard_normal(n) * 3.0)


def test_swiglu_bf16_power_of_two_scaling_and_sign():
    # h(g, 2u) = 2 h(g, u) and h(g, -u) = -h(g, u) exactly: scaling by a power of
    # two and negation commute with round-to-nearest-even (no overflow here).
    g = _bf16_grid(1, 4096)
    u = _bf16_grid(2, 4096)
    h = oracle.swiglu_bf16(g, u)
    u2 = bf16_bits(bf16_to_f64(u) * 2.0)
    un = u ^ np.uint16(0x8000)
    h2 = oracle.swiglu_bf16(g, u2)
    hn = oracle.swiglu_bf16(g, un)
    assert np.array_equal(bf16_to_f64(h2), 2.0 * bf16_to_f64(h))
    assert np.array_equal(bf16_to_f64(hn), -bf16_to_f64(h))


def test_swiglu_bf16_is_one_rounding_of_the_exact_product():
    # The result is the bf16 nearest to silu(g) u: within half a bf16 step of it
    # (at most 2^-8 relative for 8 significant bits), and no other bf16 is nearer.
    g = _bf16_grid(3, 2048)
    u = _bf16_grid(4, 2048)
    h = bf16_to_f64(oracle.swiglu_bf16(g, u))
    exact = np.array([oracle.silu(a) * b for a, b in zip(bf16_to_f64(g), bf16_to_f64(u))])
    nz = exact != 0
    rel = np.abs(h[nz] - exact[nz]) / np.abs(exact[nz])
    assert rel.max() <= 2.0 ** -8
    # neighbours of h are no nearer
    hb = bf16_bits(h)
    up = bf16_to_f64((hb.astype(np.int32) + 1).astype(np.uint16))
    dn = bf16_to_f64((hb.astype(np.int32) - 1).astype(np.uint16))
    sel = (hb & 0x7FFF) != 0
    assert np.all(np.abs(h - exact)[sel] <= np.abs(up - exact)[sel])
    assert np.all(np.abs(h - exact)[sel] <= np.abs(dn - exact)[sel])


def test_swiglu_bf16_special_cases():
    g = bf16_bits(np.array([0.0, 1.0, -1.0, 2.0, 100.0]))
    u = bf16_bits(np.array([5.0, 0.0, 0.0, 1.0, 1.0]))
    h = bf16_to_f64(oracle.swiglu_bf16(g, u))
    assert h[0] == 0.0 and h[1] == 0.0 and h[2] == 0.0
    assert h[4] == 100.0                                 # silu(100) = 100 (1 - 3.7e-44)
    assert abs(h[3] - 2.0 / (1.0 + math.exp(-2.0))) <= 2.0 ** -8 * 2.0


def test_split_gate_up_layout():
    # 128-column blocks alternate gate block j, up block j.
    R, I = 3, 384
    y = np.zeros((R, 2 * I), dtype=np.int32)
    for j in range(I // 128):
        y[:, 256 * j:256 * j + 128] = j
        y[:, 256 * j + 128:256 * j + 256] = 1000 + j
    g, u = oracle.split_gate_up(y)
    assert g.shape == (R, I) and u.shape == (R, I)
    for j in range(I // 128):
        assert np.all(g[:, 128 * j:128 * j + 128] == j)
        assert np.all(u[:, 128 * j:128 * j + 128] == 1000 + j)
    with pytest.raises(ValueError):
        oracle.split_gate_up(np.zeros((1, 384)))


def test_swiglu_quant_from_y_structure():
    # gate 0 -> h = 0 -> every code 0x00 and scale 1; a tile whose gate is large
    # (silu(g) = g) has h = bf16(g u), and its amax maps to 448.
    R, I = 2, 256
    y = np.zeros((R, 2 * I))
    y[:, 256:384] = 64.0                        # gate block 1
    y[:, 384:512] = np.linspace(-2.0, 2.0, 128)  # up block 1
    q, s, h = oracle.swiglu_quant_from_y(y, oracle.SCALE_FP32)
    assert q.shape == (R, I) and s.shape == (2, R) and h.shape == (R, I)
    assert np.all(q[:, :128] == 0) and np.all(s[0] == 1.0)
    hv = bf16_to_f64(h[:, 128:])
    u = bf16_to_f64(bf16_bits(np.linspace(-2.0, 2.0, 128)))
    assert np.array_equal(hv, np.repeat((64.0 * u)[None, :], R, 0))
    assert np.all(s[1] == np.float32(128.0) / np.float32(448.0))
    assert q[0, 255] == 0x7E and q[0, 128] == 0xFE
