"""GPU parity of the backward-pass operations of the FP8 linear layer:
token-axis 1x128 quantization (bit-exact codes and scales), the weight
transpose (bit-exact), the data-gradient GEMM dX = dY W and the
weight-gradient GEMM dW = dY^T X (within the GEMM tolerance against the
oracle's FP64 sums; bit-exact on exact integer / power-of-two cases).
The oracle quantizes the same seeded bf16 inputs itself.
"""
import numpy as np
import pytest
import torch

import fp8_block_scaled_fp8bq_b200 as fq
import fp8bq_workloads as wl
import oracle
from helpers import assert_gemm_close, bf16_bits, bf16_to_f64, f32, need_gpu, oracle_weight, u8

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _gpu_and_clean_error_word():
    need_gpu()
    yield
    st, word = fq.device_error()
    assert st == 0 and word == 0, "device error word 0x%x" % word


@pytest.mark.parametrize("mode", [fq.SCALE_FP32, fq.SCALE_POW2])
@pytest.mark.parametrize("M,K", [(300, 40), (128, 64), (1, 8), (1000, 520), (8192, 4096)])
def test_quant_act_t_bit_exact(mode, M, K):
    x = wl.activations(M, K, seed=M + K, device="cuda")
    qt, st = fq.quant_act_t(x, mode)
    torch.cuda.synchronize()
    oq, os_ = oracle.quant_act_t(bf16_bits(x), mode)
    assert np.array_equal(u8(qt)[:, :M], oq)
    assert np.array_equal(f32(st)[:, :K].view(np.uint32), os_.view(np.uint32))


@pytest.mark.parametrize("N,K", [(128, 128), (384, 640), (48, 80), (4096, 14336)])
def test_transpose_weight_bit_exact(N, K):
    w = wl.weights(N, K, seed=N + 3 * K, device="cuda")
    q, s = fq.quant_weight(w)
    qt, st = fq.transpose_weight(q, s)
    torch.cuda.synchronize()
    assert torch.equal(qt, q.t()) and torch.equal(st, s.t())


def _int_codes(rng, shape, vmax):
    v = rng.integers(-vmax, vmax + 1, size=shape).astype(np.float32)
    return torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()


@pytest.mark.parametrize("mode", [fq.SCALE_FP32, fq.SCALE_POW2])   # FP32 promotion / native block-scaled MMA
def test_wgrad_exact_integer_pow2_case_bit_exact(mode):
    rng = np.random.default_rng(4)
    N, K, M = 200, 264, 384                          # ragged tiles on both output axes
    qa = _int_codes(rng, (N, M), 4)
    qb = _int_codes(rng, (K, M), 4)
    MB = M // 128
    sa = np.array([[2.0 ** ((n + mb) % 3 - 1) for n in range(N)] for mb in range(MB)], np.float32)
    sb = np.array([[2.0 ** (-((k + mb) % 2)) for k in range(K)] for mb in range(MB)], np.float32)
    ref = oracle.f64_to_bf16(oracle.gemm_wgrad(qa, sa, qb, sb))
    sa_d = torch.zeros((MB, 200), dtype=torch.float32)
    sa_d[:, :N] = torch.from_numpy(sa)
    sb_d = torch.zeros((MB, 264), dtype=torch.float32)
    sb_d[:, :K] = torch.from_numpy(sb)
    y = fq.gemm_wgrad(torch.from_numpy(qa).cuda(), sa_d.cuda(), torch.from_numpy(qb).cuda(), sb_d.cuda(), M, mode)
    torch.cuda.synchronize()
    assert np.array_equal(bf16_bits(y), ref)


@pytest.mark.parametrize("mode", [fq.SCALE_FP32, fq.SCALE_POW2])
def test_wgrad_within_tolerance(mode):
    M, N, K = 1024, 768, 520
    dy = wl.activations(M, N, seed=41, device="cuda")
    x = wl.activations(M, K, seed=42, device="cuda")
    qa, sa = fq.quant_act_t(dy, mode)
    qb, sb = fq.quant_act_t(x, mode)
    y = fq.gemm_wgrad(qa, sa, qb, sb, M, mode)
    torch.cuda.synchronize()
    oa, osa = oracle.quant_act_t(bf16_bits(dy), mode)
    ob, osb = oracle.quant_act_t(bf16_bits(x), mode)
    assert_gemm_close(bf16_to_f64(y), oracle.gemm_wgrad(oa, osa, ob, osb), "wgrad")


@pytest.mark.parametrize("mode", [fq.SCALE_FP32, fq.SCALE_POW2])
@pytest.mark.parametrize("name", ["qkv", "down"])
def test_wgrad_llama_full_size_sampled_rows(name, mode):
    """dW of a Llama-8B-shaped projection at M = 8192 tokens; the oracle
    quantizes dY and X itself and computes one row of dW in every 128-row tile
    (power-of-two scales: the native block-scaled MMA path)."""
    N, K = wl.LLAMA8B_SHAPES[name]
    M = wl.PREFILL_TOKENS
    dy = wl.activations(M, N, seed=51, device="cuda")
    x = wl.activations(M, K, seed=52, device="cuda")
    qa, sa = fq.quant_act_t(dy, mode)
    qb, sb = fq.quant_act_t(x, mode)
    y = fq.gemm_wgrad(qa, sa, qb, sb, M, mode)
    torch.cuda.synchronize()
    rng = np.random.default_rng(N)
    rows = np.array(sorted({0, N - 1} | {int(rng.integers(t, min(t + 128, N))) for t in range(0, N, 128)}))
    oa, osa = oracle.quant_act_t(bf16_bits(dy[:, torch.from_numpy(rows).cuda()]), mode)
    ob, osb = oracle.quant_act_t(bf16_bits(x), mode)
    ref = oracle.gemm_wgrad(oa, osa, ob, osb)
    assert_gemm_close(bf16_to_f64(y[torch.from_numpy(rows).cuda()]), ref, "wgrad " + name)


@pytest.mark.parametrize("mode", [fq.SCALE_FP32, fq.SCALE_POW2])
def test_dgrad_within_tolerance(mode):
    M, N, K = 640, 512, 768                          # dY [M, N], W [N, K]
    dy = wl.activations(M, N, seed=61, device="cuda")
    w = wl.weights(N, K, seed=62, device="cuda")
    q_dy, s_dy = fq.quant_act(dy, mode)
    qw, sw = fq.quant_weight(w, mode)
    qwt, swt = fq.transpose_weight(qw, sw)
    dx = fq.gemm_dgrad(q_dy, s_dy, qwt, swt, mode)
    torch.cuda.synchronize()
    oq, os_ = oracle.quant_act(bf16_bits(dy), mode)
    oqw, osw = oracle_weight(w, mode)
    assert_gemm_close(bf16_to_f64(dx), oracle.gemm_dgrad(oq, os_, oqw, osw), "dgrad")


def test_dgrad_llama_down_full_size_sampled_rows():
    """dX of the down projection (W [4096, 14336]) at M = 8192 tokens."""
    N, K = wl.LLAMA8B_SHAPES["down"]
    M = wl.PREFILL_TOKENS
    dy = wl.activations(M, N, seed=71, device="cuda")
    w = wl.weights(N, K, seed=72, device="cuda")
    q_dy, s_dy = fq.quant_act(dy)
    qw, sw = fq.quant_weight(w)
    qwt, swt = fq.transpose_weight(qw, sw)
    dx = fq.gemm_dgrad(q_dy, s_dy, qwt, swt)
    torch.cuda.synchronize()
    rng = np.random.default_rng(M)
    rows = np.array(sorted({0, M - 1} | {int(rng.integers(t, t + 128)) for t in range(0, M, 128)}))
    oq, os_ = oracle.quant_act(bf16_bits(dy[torch.from_numpy(rows).cuda()]), fq.SCALE_FP32)
    oqw, osw = oracle_weight(w, fq.SCALE_FP32)
    ref = oracle.gemm_dgrad(oq, os_, oqw, osw)
    assert_gemm_close(bf16_to_f64(dx[torch.from_numpy(rows).cuda()]), ref, "dgrad down")
