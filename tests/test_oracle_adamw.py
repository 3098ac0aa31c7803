"""Pins of the oracle's optimizer step (AdamW on binary32 state) and of the
fused step + recalibration composition.

The scales are recalibrated after every training step (section "Real-world
performance gains" of "NVIDIA NeMo RL Achieves 48% Speedup With End-to-End FP8
Precision Training"); the step is AdamW (Loshchilov & Hutter 2019, Adam's
bias-corrected moments of Kingma & Ba 2015).  The pins are closed forms of the
algorithm, not the update retyped: the first step from zero moments moves every
weight by lr * g / (|g| + eps); with a constant gradient the bias-corrected
moments equal g and g^2 at every step; the weight decay alone scales the weight
by (1 - lr wd); the moment recursions have closed forms; zero gradient and
zero state leave everything unchanged.
"""
import numpy as np
import pytest
import torch

import oracle

# The hyperparameters are binary32 values (the optimizer's arithmetic is binary32).
LR, B1, B2, EPS = (float(np.float32(x)) for x in (1e-3, 0.9, 0.999, 1e-8))


def _rng_arrays(seed, shape):
    rng = np.random.default_rng(seed)
    p = rng.standard_normal(shape).astype(np.float32) * 0.02
    g = rng.standard_normal(shape).astype(np.float32) * 1e-3
    return p, g


def _ulp(x):
    return np.spacing(np.abs(x).astype(np.float32)).astype(np.float64)


def _step_tol(p, expect, update):
    """Binary32 rounding of p - lr u: a few ulps of the operands and the result,
    plus the relative rounding (a few 2^-24) of the update term itself."""
    return 3 * np.maximum(_ulp(p), _ulp(expect)) + 8 * 2.0 ** -24 * np.abs(update)


def test_first_step_moves_by_lr_times_sign():
    p, g = _rng_arrays(1, (64, 96))
    z = np.zeros_like(p)
    p1, m1, v1 = oracle.adamw_step(p, g, z, z, LR, B1, B2, EPS, 0.0, 1)
    update = LR * g / (np.abs(g) + EPS)
    expect = p.astype(np.float64) - update
    assert np.all(np.abs(p1 - expect) <= _step_tol(p, expect, update))
    # m1 = (1 - b1) g, v1 = (1 - b2) g^2 (to binary32 rounding)
    assert np.allclose(m1, (1 - B1) * g.astype(np.float64), rtol=3e-7, atol=0)
    assert np.allclose(v1, (1 - B2) * g.astype(np.float64) ** 2, rtol=5e-7, atol=0)


def test_decoupled_weight_decay_alone():
    p, _ = _rng_arrays(2, (32, 32))
    z = np.zeros_like(p)
    wd = 0.1
    p1, m1, v1 = oracle.adamw_step(p, z, z, z, LR, B1, B2, EPS, wd, 5)
    assert np.all(np.abs(p1 - p.astype(np.float64) * (1 - LR * wd)) <= 2 * _ulp(p))
    assert not m1.any() and not v1.any()


def test_zero_gradient_and_state_leave_everything_unchanged():
    p, _ = _rng_arrays(3, (16, 16))
    z = np.zeros_like(p)
    p1, m1, v1 = oracle.adamw_step(p, z, z, z, LR, B1, B2, EPS, 0.0, 7)
    assert np.array_equal(p1, p) and not m1.any() and not v1.any()


def test_constant_gradient_bias_corrected_moments_are_exact():
    # m_t = g (1 - b1^t), v_t = g^2 (1 - b2^t): after bias correction every step
    # is lr g / (|g| + eps), so T steps move the weight by T times that.
    shape = (8, 40)
    rng = np.random.default_rng(4)
    g = (rng.standard_normal(shape) * 1e-2).astype(np.float32)
    p = np.zeros(shape, dtype=np.float32) + np.float32(0.5)
    m = np.zeros(shape, dtype=np.float32)
    v = np.zeros(shape, dtype=np.float32)
    T = 50
    for t in range(1, T + 1):
        p, m, v = oracle.adamw_step(p, g, m, v, LR, B1, B2, EPS, 0.0, t)
    g64 = g.astype(np.float64)
    assert np.allclose(m, g64 * (1 - B1 ** T), rtol=T * 2e-7, atol=0)
    assert np.allclose(v, g64 ** 2 * (1 - B2 ** T), rtol=T * 3e-7, atol=0)
    expect = 0.5 - T * LR * g64 / (np.abs(g64) + EPS)
    assert np.all(np.abs(p - expect) <= T * 4 * _ulp(np.float32(0.5)))


def test_step_number_enters_only_through_the_bias_correction():
    p, g = _rng_arrays(5, (16, 64))
    rng = np.random.default_rng(6)
    m = (rng.standard_normal(p.shape) * 1e-3).astype(np.float32)
    v = (rng.random(p.shape) * 1e-6).astype(np.float32)
    a = oracle.adamw_step(p, g, m, v, LR, B1, B2, EPS, 0.0, 3)
    b = oracle.adamw_step(p, g, m, v, LR, B1, B2, EPS, 0.0, 4)
    assert np.array_equal(a[1], b[1]) and np.array_equal(a[2], b[2])   # moments do not depend on t
    assert not np.array_equal(a[0], b[0])
    # at a very large step the corrections are 1: p' = p - lr m' / (sqrt(v') + eps)
    c = oracle.adamw_step(p, g, m, v, LR, B1, B2, EPS, 0.0, 10 ** 9)
    m1, v1 = c[1].astype(np.float64), c[2].astype(np.float64)
    update = LR * m1 / (np.sqrt(v1) + EPS)
    expect = p - update
    assert np.all(np.abs(c[0] - expect) <= _step_tol(p, expect, update))


def test_f32_to_bf16_matches_torch_cast():
    rng = np.random.default_rng(7)
    x = np.concatenate([rng.standard_normal(100000).astype(np.float32),
                        np.array([0.0, -0.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, 1e-40, -3e38], np.float32)])
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(oracle.f32_to_bf16(x), ref)


@pytest.mark.parametrize("mode", [oracle.SCALE_FP32, oracle.SCALE_POW2])
def test_adamw_recalibrate_composition(mode):
    p, g = _rng_arrays(8, (200, 264))      # ragged: 2 x 3 tiles, the last ones partial
    z = np.zeros_like(p)
    p1, m1, v1, w, q, s = oracle.adamw_recalibrate(p, g, z, z, LR, B1, B2, EPS, 0.01, 1, mode)
    assert w.shape == p.shape and q.shape == p.shape and s.shape == (2, 3)
    assert np.array_equal(w, torch.from_numpy(p1).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16))
    q2, s2 = oracle.quant_weight(w, mode)
    assert np.array_equal(q, q2) and np.array_equal(s, s2)
