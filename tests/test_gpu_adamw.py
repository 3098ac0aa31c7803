"""GPU parity of the fused optimizer step + recalibration (fp8bq_adamw_recalibrate)
against the oracle's binary32 AdamW and 128x128 quantizer: every output (master
weight, both moments, the bf16 copy, codes and scales) bit for bit, since both
sides perform the same correctly rounded binary32 operations in the same order.
"""
import numpy as np
import pytest
import torch

import fp8_block_scaled_fp8bq_b200 as fq
import fp8bq_workloads as wl
import oracle
from helpers import bf16_bits, f32, need_gpu, u8

pytestmark = pytest.mark.gpu

HP = dict(lr=3e-4, beta1=0.9, beta2=0.95, eps=1e-8, weight_decay=0.1)


@pytest.fixture(autouse=True)
def _gpu_and_clean_error_word():
    need_gpu()
    yield
    st, word = fq.device_error()
    assert st == 0 and word == 0, "device error word 0x%x" % word


def state(N, K, seed):
    """fp32 master weight ~ N(0, 0.02), gradient ~ N(0, 1e-3), moments from a
    few earlier steps' worth of magnitude (seeded, host)."""
    g = torch.Generator().manual_seed(seed)
    p = torch.randn((N, K), generator=g) * 0.02
    gr = torch.randn((N, K), generator=g) * 1e-3
    m = torch.randn((N, K), generator=g) * 1e-4
    v = torch.rand((N, K), generator=g) * 1e-6
    return [t.float().contiguous() for t in (p, gr, m, v)]


def run_gpu(tensors, step, mode, with_w=True):
    dev = []
    for p, g, m, v in tensors:
        N, K = p.shape
        d = [t.cuda() for t in (p, g, m, v)]
        w = torch.empty((N, K), dtype=torch.bfloat16, device="cuda") if with_w else None
        q = torch.empty((N, K), dtype=torch.uint8, device="cuda")
        s = torch.empty(((N + 127) // 128, (K + 127) // 128), dtype=torch.float32, device="cuda")
        dev.append((*d, w, q, s))
    fq.adamw_recalibrate(dev, step=step, mode=mode, **HP)
    torch.cuda.synchronize()
    return dev


def check(tensors, dev, step, mode, with_w=True):
    for (p, g, m, v), (dp, dg, dm, dv, dw, dq, ds) in zip(tensors, dev):
        hp = dict(HP)
        p1, m1, v1, w, q, s = oracle.adamw_recalibrate(p.numpy(), g.numpy(), m.numpy(), v.numpy(),
                                                       hp["lr"], hp["beta1"], hp["beta2"], hp["eps"],
                                                       hp["weight_decay"], step, mode)
        assert np.array_equal(f32(dp).view(np.uint32), p1.view(np.uint32)), "param"
        assert np.array_equal(f32(dm).view(np.uint32), m1.view(np.uint32)), "exp_avg"
        assert np.array_equal(f32(dv).view(np.uint32), v1.view(np.uint32)), "exp_avg_sq"
        assert np.array_equal(f32(dg), g.numpy()), "gradient untouched"
        if with_w:
            assert np.array_equal(bf16_bits(dw), w), "bf16 weight"
        assert np.array_equal(u8(dq), q), "codes"
        assert np.array_equal(f32(ds).view(np.uint32), s.view(np.uint32)), "scales"


@pytest.mark.parametrize("mode", [fq.SCALE_FP32, fq.SCALE_POW2])
@pytest.mark.parametrize("shape", [(200, 264), (128, 128), (1, 4), (300, 1000), (257, 132)])
def test_single_tensor_bit_exact(mode, shape):
    t = [state(*shape, seed=shape[0] * 7 + shape[1])]
    check(t, run_gpu(t, 3, mode), 3, mode)


@pytest.mark.parametrize("mode", [fq.SCALE_FP32, fq.SCALE_POW2])
def test_many_tensors_one_launch_and_two_steps(mode):
    shapes = [(384, 256), (130, 516), (64, 128), (512, 4)]
    t = [state(N, K, seed=i + 50) for i, (N, K) in enumerate(shapes)]
    dev = run_gpu(t, 1, mode)
    check(t, dev, 1, mode)
    # a second step from the first step's state (the oracle recomputes from its own)
    t2 = []
    for (p, g, m, v) in t:
        p1, m1, v1 = oracle.adamw_step(p.numpy(), g.numpy(), m.numpy(), v.numpy(), HP["lr"], HP["beta1"],
                                       HP["beta2"], HP["eps"], HP["weight_decay"], 1)
        t2.append([torch.from_numpy(p1), g, torch.from_numpy(m1), torch.from_numpy(v1)])
    dev2 = []
    for (dp, dg, dm, dv, dw, dq, ds) in dev:
        dev2.append((dp, dg, dm, dv, dw, dq, ds))
    fq.adamw_recalibrate(dev2, step=2, mode=mode, **HP)
    torch.cuda.synchronize()
    check(t2, dev2, 2, mode)


def test_without_bf16_copy():
    t = [state(256, 384, seed=9)]
    check(t, run_gpu(t, 5, fq.SCALE_POW2, with_w=False), 5, fq.SCALE_POW2, with_w=False)


def test_llama_o_projection_full_size():
    """The 4096 x 4096 output projection of the Llama-3.1-8B-shaped layer."""
    N, K = wl.LLAMA8B_SHAPES["o"]
    t = [state(N, K, seed=77)]
    check(t, run_gpu(t, 10, fq.SCALE_POW2), 10, fq.SCALE_POW2)


def test_validation():
    p, g, m, v = [x.cuda() for x in state(128, 128, seed=1)]
    q = torch.empty((128, 128), dtype=torch.uint8, device="cuda")
    s = torch.empty((1, 1), dtype=torch.float32, device="cuda")
    with pytest.raises(fq.Fp8bqError):
        fq.adamw_recalibrate([(p, g, m, v, None, q, s)], lr=1e-3, step=0)
    with pytest.raises(fq.Fp8bqError):
        fq.adamw_recalibrate([(p, g, m, v, None, q, s)], lr=1e-3, beta1=1.0)
    p6 = torch.zeros((128, 6), dtype=torch.float32, device="cuda")
    with pytest.raises(fq.Fp8bqError) as e:
        fq.adamw_recalibrate([(p6, p6, p6, p6, None, torch.empty((128, 6), dtype=torch.uint8, device="cuda"), s)],
                             lr=1e-3)
    assert e.value.status == 2
