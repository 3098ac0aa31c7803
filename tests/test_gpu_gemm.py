"""GPU parity of the block-scaled FP8 GEMM against the CPU oracle.

Exact cases (bit-exact bf16 output): integer-valued codes with unit scales, and
distinct power-of-two scales per (row, K-block) and (N-block, K-block), where
the FP32 sums are exact, so any misplaced scale, operand or tile shows.
Tolerance cases: the single-linear workload and the Llama-8B-shaped prefill
GEMMs at full size (sampled rows), both scale modes.  Edge cases: ragged M and
N, K = 128, K = 0, a single row.  Metamorphic: reruns are bit-identical and
doubling power-of-two activation scales doubles the output exactly.
"""
import numpy as np
import pytest
import torch

import fp8_block_scaled_fp8bq_b200 as fq
import fp8bq_workloads as wl
import oracle
from helpers import oracle_act, oracle_weight, assert_gemm_close, bf16_bits, bf16_to_f64, f32, need_gpu, u8

pytestmark = pytest.mark.gpu
VARIANTS = [fq.GEMM_PROMOTE, fq.GEMM_PROMOTE_PAIR, fq.GEMM_PROMOTE_PAIR_N128]


@pytest.fixture(autouse=True)
def _gpu_and_clean_error_word():
    need_gpu()
    yield
    st, word = fq.device_error()
    assert st == 0 and word == 0, "device error word 0x%x" % word


def int_codes(rng, shape, vmax):
    v = rng.integers(-vmax, vmax + 1, size=shape).astype(np.float32)
    return torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def tile_rows(M, seed, per_tile=1):
    """`per_tile` seeded rows of every 128-row tile (the first and last rows of
    the matrix always among them), so every persistent CTA's tiles are checked."""
    rng = np.random.default_rng(seed)
    rows = {0, M - 1}
    for t in range(0, M, 128):
        rows.update(int(r) for r in rng.integers(t, min(t + 128, M), size=per_tile))
    return np.array(sorted(rows))


def run_gemm(qa, sa, qw, sw, mode=fq.SCALE_FP32, variant=fq.GEMM_PROMOTE):
    """numpy operands -> GPU bf16 output as numpy uint16 bits and float64 values."""
    M, K = qa.shape
    ldsa = fq.act_scale_shape(M, K)[1]
    sa_d = torch.zeros((K // 128, ldsa), dtype=torch.float32)
    sa_d[:, :M] = torch.from_numpy(np.ascontiguousarray(sa))
    y = fq.gemm(torch.from_numpy(qa).cuda(), sa_d.cuda(), torch.from_numpy(qw).cuda(),
                torch.from_numpy(np.ascontiguousarray(sw)).cuda(), mode=mode, variant=variant)
    torch.cuda.synchronize()
    return bf16_bits(y), bf16_to_f64(y)


@pytest.mark.parametrize("variant", VARIANTS)
@pytest.mark.parametrize("M,N,K", [(256, 512, 512), (200, 384, 256), (1, 256, 128), (129, 136, 384)])
def test_integer_codes_unit_scales_bit_exact(variant, M, N, K):
    rng = np.random.default_rng(M + N + K)
    qa = int_codes(rng, (M, K), 8)
    qw = int_codes(rng, (N, K), 8)
    sa = np.ones((K // 128, M), dtype=np.float32)
    sw = np.ones(((N + 127) // 128, K // 128), dtype=np.float32)
    bits, _ = run_gemm(qa, sa, qw, sw, fq.SCALE_POW2, variant)
    ref = oracle.f64_to_bf16(oracle.gemm(qa, sa, qw, sw))
    assert np.array_equal(bits, ref), np.argwhere(bits != ref)[:5]


@pytest.mark.parametrize("variant", VARIANTS)
def test_distinct_pow2_block_scales_bit_exact(variant):
    rng = np.random.default_rng(11)
    M, N, K = 384, 768, 1024                                  # 3 x 3 tiles, 8 K-blocks, NB = 6
    KB, NB = K // 128, N // 128
    qa = int_codes(rng, (M, K), 4)
    qw = int_codes(rng, (N, K), 4)
    sa = (2.0 ** (((np.arange(M)[None, :] + np.arange(KB)[:, None]) % 5) - 2)).astype(np.float32)
    sw = (2.0 ** (((np.arange(NB)[:, None] * 3 + np.arange(KB)[None, :]) % 7) - 3)).astype(np.float32)
    bits, _ = run_gemm(qa, sa, qw, sw, fq.SCALE_POW2, variant)
    y64 = oracle.gemm(qa, sa, qw, sw)
    ref = oracle.f64_to_bf16(y64)
    assert np.array_equal(bits, ref), np.argwhere(bits != ref)[:5]


@pytest.mark.parametrize("mode", [fq.SCALE_FP32, fq.SCALE_POW2])
def test_single_linear_within_tolerance(mode):
    x, w = wl.single_linear(seed=0)
    qa, sa = oracle.quant_act(bf16_bits(x), mode)
    qw, sw = oracle.quant_weight(bf16_bits(w), mode)
    _, y = run_gemm(qa, sa, qw, sw, mode)
    assert_gemm_close(y, oracle.gemm(qa, sa, qw, sw), "single linear")


@pytest.mark.parametrize("mode", [fq.SCALE_FP32, fq.SCALE_POW2])
@pytest.mark.parametrize("name", list(wl.LLAMA8B_SHAPES))
def test_llama_prefill_full_size_sampled_rows(mode, name):
    """The bench's launch configuration (M = 8192) end to end on the GPU: quantize
    X and W, GEMM; the oracle quantizes the same bf16 inputs itself (one row of
    every 128-row tile of X, all of W) and computes those rows, every column."""
    N, K = wl.LLAMA8B_SHAPES[name]
    M = wl.PREFILL_TOKENS
    x = wl.activations(M, K, seed=N, device="cuda")
    w = wl.weights(N, K, seed=N + 1, device="cuda")
    qa, sa = fq.quant_act(x, mode)
    qw, sw = fq.quant_weight(w, mode)
    y = fq.gemm(qa, sa, qw, sw, mode)
    torch.cuda.synchronize()
    rows = tile_rows(M, seed=N)
    oqa, osa = oracle_act(x, mode, rows)
    oqw, osw = oracle_weight(w, mode)
    ref = oracle.gemm(oqa, osa, oqw, osw, blockint=True)
    got = bf16_to_f64(y[torch.from_numpy(rows).cuda()])
    assert_gemm_close(got, ref, name)


def test_k_zero_writes_zeros():
    y = torch.full((4, 64), 7.0, dtype=torch.bfloat16, device="cuda")
    qa = torch.empty((4, 0), dtype=torch.uint8, device="cuda")
    qw = torch.empty((64, 0), dtype=torch.uint8, device="cuda")
    sa = torch.empty((1, 4), dtype=torch.float32, device="cuda")
    sw = torch.empty((1, 1), dtype=torch.float32, device="cuda")
    fq.gemm(qa, sa, qw, sw, out=y)
    torch.cuda.synchronize()
    assert torch.count_nonzero(y).item() == 0


def test_rerun_bit_identical_and_pow2_scaling():
    x = wl.activations(300, 1024, seed=1, device="cuda")
    w = wl.weights(640, 1024, seed=2, device="cuda")
    qa, sa = fq.quant_act(x, fq.SCALE_POW2)
    qw, sw = fq.quant_weight(w, fq.SCALE_POW2)
    y1 = fq.gemm(qa, sa, qw, sw, fq.SCALE_POW2)
    y2 = fq.gemm(qa, sa, qw, sw, fq.SCALE_POW2)
    y3 = fq.gemm(qa, sa * 2, qw, sw, fq.SCALE_POW2)
    torch.cuda.synchronize()
    assert torch.equal(y1.view(torch.int16), y2.view(torch.int16))
    assert torch.equal((y1.float() * 2).to(torch.bfloat16).view(torch.int16), y3.view(torch.int16))


def test_row_subset_gives_identical_rows():
    x = wl.activations(512, 512, seed=4, device="cuda")
    w = wl.weights(512, 512, seed=5, device="cuda")
    qa, sa = fq.quant_act(x)
    qw, sw = fq.quant_weight(w)
    y = fq.gemm(qa, sa, qw, sw)
    qa2, sa2 = fq.quant_act(x[128:256].contiguous())
    y2 = fq.gemm(qa2, sa2, qw, sw)
    torch.cuda.synchronize()
    assert torch.equal(y[128:256].view(torch.int16), y2.view(torch.int16))


@pytest.mark.parametrize("pair_variant", [fq.GEMM_PROMOTE_PAIR, fq.GEMM_PROMOTE_PAIR_N128])
def test_pair_kernel_equals_one_sm_kernel(pair_variant):
    """The CTA-pair kernels (256x256 or 256x128 tiles, paired MMA) and the
    one-SM kernel compute every output from the same K-block partials in the
    same order."""
    x = wl.activations(640, 1024, seed=21, device="cuda")
    w = wl.weights(768, 1024, seed=22, device="cuda")
    qa, sa = fq.quant_act(x)
    qw, sw = fq.quant_weight(w)
    y_pair = fq.gemm(qa, sa, qw, sw, variant=pair_variant)
    y_one = fq.gemm(qa, sa, qw, sw, variant=fq.GEMM_PROMOTE)
    torch.cuda.synchronize()
    assert_gemm_close(bf16_to_f64(y_pair), bf16_to_f64(y_one), "pair vs one-SM")
    assert torch.equal(y_pair.view(torch.int16), y_one.view(torch.int16))


@pytest.mark.parametrize("variant", VARIANTS + [fq.GEMM_NATIVE_POW2])
def test_distinct_pow2_scales_more_tiles_than_sms_bit_exact(variant):
    """Integer codes with distinct power-of-two scales per (row, K-block) and
    (N-block, K-block) at M = 2048, N = 28672 (the gate+up shape's N): 1792
    tiles of 128x256, about 12 per persistent CTA, so every CTA carries its
    TMEM phase and its tile order across many tiles.  The FP32 sums are exact,
    so the bf16 result equals the oracle's bit for bit; one row of every
    128-row tile, every column, is compared."""
    rng = np.random.default_rng(29)
    M, N, K = 2048, 28672, 512
    KB, NB = K // 128, N // 128
    qa = int_codes(rng, (M, K), 4)
    qw = int_codes(rng, (N, K), 4)
    sa = (2.0 ** (((np.arange(M)[None, :] * 7 + np.arange(KB)[:, None]) % 5) - 2)).astype(np.float32)
    sw = (2.0 ** (((np.arange(NB)[:, None] * 3 + np.arange(KB)[None, :]) % 7) - 3)).astype(np.float32)
    bits, _ = run_gemm(qa, sa, qw, sw, fq.SCALE_POW2, variant)
    rows = tile_rows(M, seed=5, per_tile=1)
    ref = oracle.f64_to_bf16(oracle.gemm(qa, sa, qw, sw, rows=rows))
    got = bits[rows]
    assert np.array_equal(got, ref), np.argwhere(got != ref)[:5]
