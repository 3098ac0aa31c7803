"""GPU parity of the decode-shaped linear (on-the-fly 1x128 activation
quantization + block-scaled GEMM against pre-quantized 128x128 weights).

The activation codes are recomputed by the oracle from X (bit-exact codes are
the quantizer's contract), the GEMM is compared with the oracle's FP64 sum on
every row, for every decode M of the Llama-8B-shaped workload and every
projection shape (split-K and unsplit paths), plus ragged M and the argument
checks (workspace, M limit)."""
import numpy as np
import pytest
import torch

import fp8_block_scaled_fp8bq_b200 as fq
import fp8bq_workloads as wl
import oracle
from helpers import oracle_weight, assert_gemm_close, bf16_bits, bf16_to_f64, f32, need_gpu, u8

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _gpu_and_clean_error_word():
    need_gpu()
    yield
    st, word = fq.device_error()
    assert st == 0 and word == 0, "device error word 0x%x" % word


_W = {}
_OW = {}


def qweights(name, mode):
    """GPU-quantized weight (codes, scales); the oracle's own quantization of
    the same bf16 weight is kept beside it for check_decode."""
    key = (name, mode)
    if key not in _W:
        N, K = wl.LLAMA8B_SHAPES[name]
        w = wl.weights(N, K, seed=N * 3 + K, device="cuda")
        _W[key] = fq.quant_weight(w, mode)
        _OW[_W[key][0].data_ptr()] = oracle_weight(w, mode)
    return _W[key]


def check_decode(x, qw, sw, mode, ws=None):
    M, K = x.shape
    y = fq.gemm_decode(x, qw, sw, mode, ws=ws)
    torch.cuda.synchronize()
    qa, sa = oracle.quant_act(bf16_bits(x), mode)
    oqw, osw = _OW[qw.data_ptr()]
    ref = oracle.gemm(qa, sa, oqw, osw, blockint=True)
    assert_gemm_close(bf16_to_f64(y), ref, "decode M=%d" % M)
    return y


@pytest.mark.parametrize("M", wl.DECODE_TOKENS)
@pytest.mark.parametrize("name", list(wl.LLAMA8B_SHAPES))
def test_llama_decode_shapes(M, name):
    N, K = wl.LLAMA8B_SHAPES[name]
    qw, sw = qweights(name, fq.SCALE_FP32)
    x = wl.activations(M, K, seed=M + K, device="cuda")
    check_decode(x, qw, sw, fq.SCALE_FP32)


@pytest.mark.parametrize("M", [2, 3, 17, 33, 100, 129, 200])
def test_ragged_m_both_modes(M):
    for mode in (fq.SCALE_FP32, fq.SCALE_POW2):
        qw, sw = qweights("o", mode)
        x = wl.activations(M, 4096, seed=M, device="cuda")
        check_decode(x, qw, sw, mode)


def test_decode_matches_quant_then_gemm():
    qw, sw = qweights("qkv", fq.SCALE_FP32)
    x = wl.activations(64, 4096, seed=7, device="cuda")
    y = fq.gemm_decode(x, qw, sw)
    qa, sa = fq.quant_act(x)
    y2 = fq.gemm(qa, sa, qw, sw)
    torch.cuda.synchronize()
    # same codes and scales, FP32 summation order differs (split K)
    assert_gemm_close(bf16_to_f64(y), bf16_to_f64(y2), "decode vs gemm")


def test_rerun_bit_identical():
    qw, sw = qweights("down", fq.SCALE_FP32)
    x = wl.activations(16, 14336, seed=8, device="cuda")
    y1 = fq.gemm_decode(x, qw, sw)
    y2 = fq.gemm_decode(x, qw, sw)
    torch.cuda.synchronize()
    assert torch.equal(y1.view(torch.int16), y2.view(torch.int16))


def test_workspace_and_limits():
    qw, sw = qweights("o", fq.SCALE_FP32)
    x = wl.activations(16, 4096, seed=9, device="cuda")
    need = fq.gemm_decode_workspace_size(16, 4096, 4096)
    assert need > 0
    small = torch.empty(need - 256, dtype=torch.uint8, device="cuda")
    with pytest.raises(fq.Fp8bqError) as e:
        fq.gemm_decode(x, qw, sw, ws=small)
    assert e.value.status == 4
    big = wl.activations(257, 4096, seed=9, device="cuda")
    with pytest.raises(fq.Fp8bqError) as e:
        fq.gemm_decode(big, qw, sw)
    assert e.value.status == 2


def test_one_workspace_reused_across_shapes():
    # one workspace for every shape, its contents left from the previous call:
    # the single-launch path (M <= 16), the two-launch one above it, and
    # unaligned activations (through the prologue), every row against the oracle
    need = max(fq.gemm_decode_workspace_size(M, N, K) for N, K in wl.LLAMA8B_SHAPES.values() for M in (1, 16, 40))
    ws = torch.full((need,), 0xAB, dtype=torch.uint8, device="cuda")
    for name, (N, K) in wl.LLAMA8B_SHAPES.items():
        qw, sw = qweights(name, fq.SCALE_FP32)
        for M in (1, 16, 40):
            x = wl.activations(M, K, seed=3 * M + K, device="cuda")
            check_decode(x, qw, sw, fq.SCALE_FP32, ws=ws)
        # a row view whose leading dimension is odd: not 16-byte loadable
        xb = wl.activations(4, K + 1, seed=K, device="cuda")[:, :K]
        check_decode(xb, qw, sw, fq.SCALE_FP32, ws=ws)


@pytest.mark.parametrize("M", [1, 5, 16])
def test_single_launch_pow2(M):
    qw, sw = qweights("gate_up", fq.SCALE_POW2)
    x = wl.activations(M, 4096, seed=40 + M, device="cuda")
    check_decode(x, qw, sw, fq.SCALE_POW2)
