"""GPU parity of each kernel behind fp8bq_gemm_decode, forced one at a time
through FP8BQ_DECODE_KERNEL (narrow: 128 weight rows x the tokens per MMA;
wide: the tokens x 256 weight rows per MMA, K split over clusters of up to 16
CTAs with the cross-CTA sum spread over the cluster; gemm: the prefill GEMM
after the prologue quantization).

Every output row is compared with the oracle's FP64 sum of the oracle's own
quantization of the same X and W: the Llama-8B projections at the decode
token counts, ragged N (a half-empty last 256-row tile, a last tile shorter
than 128 rows, N below one tile), K from one block to the down projection's
112, unaligned activations (prologue path), both scale modes, and
bit-identical reruns (the split sums run in rank order)."""
import pytest
import torch

import fp8_block_scaled_fp8bq_b200 as fq
import fp8bq_workloads as wl
import oracle
from helpers import oracle_weight, assert_gemm_close, bf16_bits, bf16_to_f64, need_gpu

pytestmark = pytest.mark.gpu

KERNELS = ("narrow", "wide", "gemm")


@pytest.fixture(autouse=True)
def _gpu_and_clean_error_word():
    need_gpu()
    yield
    st, word = fq.device_error()
    assert st == 0 and word == 0, "device error word 0x%x" % word


_W = {}


def qweights(N, K, mode):
    """GPU-quantized weight and the oracle's quantization of the same bf16 weight."""
    key = (N, K, mode)
    if key not in _W:
        w = wl.weights(N, K, seed=N * 7 + K, device="cuda")
        qw, sw = fq.quant_weight(w, mode)
        _W[key] = (qw, sw, oracle_weight(w, mode))
    return _W[key]


def check(kernel, monkeypatch, M, N, K, mode, x=None):
    monkeypatch.setenv("FP8BQ_DECODE_KERNEL", kernel)
    qw, sw, (oqw, osw) = qweights(N, K, mode)
    if x is None:
        x = wl.activations(M, K, seed=M * 5 + N + K, device="cuda")
    y = fq.gemm_decode(x, qw, sw, mode)
    torch.cuda.synchronize()
    qa, sa = oracle.quant_act(bf16_bits(x), mode)
    ref = oracle.gemm(qa, sa, oqw, osw, blockint=True)
    assert_gemm_close(bf16_to_f64(y), ref, "%s M=%d N=%d K=%d mode=%d" % (kernel, M, N, K, mode))
    return y


@pytest.mark.parametrize("kernel", KERNELS)
@pytest.mark.parametrize("M", [1, 16, 64])
@pytest.mark.parametrize("name", list(wl.LLAMA8B_SHAPES))
def test_llama_shapes(kernel, M, name, monkeypatch):
    N, K = wl.LLAMA8B_SHAPES[name]
    check(kernel, monkeypatch, M, N, K, fq.SCALE_FP32)


@pytest.mark.parametrize("kernel", KERNELS)
@pytest.mark.parametrize("M,N,K", [
    (1, 4096 + 128, 4096),    # last 256-row tile half empty
    (3, 1000, 2048),          # last tile 232 rows: a 128-row block of 104 rows
    (16, 200, 1024),          # N below one tile
    (7, 72, 128),             # one K-block, N below one 128-row block
    (20, 3072 + 40, 14336),   # NT = 32, deep K, ragged N
    (64, 640, 512),           # NT = 64, few K-blocks
    (33, 6144, 4096),         # NT = 64 at M = 33
])
def test_ragged(kernel, M, N, K, monkeypatch):
    for mode in (fq.SCALE_FP32, fq.SCALE_POW2):
        check(kernel, monkeypatch, M, N, K, mode)


@pytest.mark.parametrize("kernel", ("narrow", "wide"))
@pytest.mark.parametrize("M", [1, 9, 40])
def test_unaligned_activations(kernel, M, monkeypatch):
    # a leading dimension of K + 1 elements: rows are not 16-byte aligned, so
    # the activation goes through the prologue (no in-kernel quantization)
    K = 4096
    x = wl.activations(M, K + 1, seed=M, device="cuda")[:, :K]
    check(kernel, monkeypatch, M, 6144, K, fq.SCALE_FP32, x=x)


@pytest.mark.parametrize("kernel", ("narrow", "wide"))
@pytest.mark.parametrize("M,N,K", [(1, 4096, 14336), (16, 6144, 4096), (48, 4096, 4096)])
def test_rerun_bit_identical(kernel, M, N, K, monkeypatch):
    monkeypatch.setenv("FP8BQ_DECODE_KERNEL", kernel)
    qw, sw, _ = qweights(N, K, fq.SCALE_FP32)
    x = wl.activations(M, K, seed=11 + M, device="cuda")
    y1 = fq.gemm_decode(x, qw, sw)
    y2 = fq.gemm_decode(x, qw, sw)
    torch.cuda.synchronize()
    assert torch.equal(y1.view(torch.int16), y2.view(torch.int16))


def test_wide_many_tiles_per_cluster(monkeypatch):
    # N = 28672 (112 tiles of 256 rows) in the wide form: clusters take
    # several tiles each, so the partial buffer is reused across tiles
    check("wide", monkeypatch, 5, 28672, 4096, fq.SCALE_FP32)
    check("wide", monkeypatch, 40, 28672, 1024, fq.SCALE_POW2)


@pytest.mark.parametrize("M", [65, 100, 129, 200, 256])
@pytest.mark.parametrize("N,K", [(6144, 4096), (4096, 14336), (1000, 2048)])
def test_wide_token_groups(M, N, K, monkeypatch):
    # M > 64 in the wide form: one block per (weight tile, group of 64
    # tokens), the last group ragged
    check("wide", monkeypatch, M, N, K, fq.SCALE_FP32)
    if N == 1000:
        check("wide", monkeypatch, M, N, K, fq.SCALE_POW2)
