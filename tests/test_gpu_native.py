"""The native block-scaled MMA path for power-of-two scales
(fp8bq_gemm_ex variant FP8BQ_GEMM_NATIVE_POW2): UE8M0 scale factors in TMEM,
one accumulator over the whole K loop.

Exact cases (distinct power-of-two scales per row and per weight block,
integer codes) must be bit-exact against the oracle; random Llama-shaped
cases within the GEMM tolerance, and within the tolerance of the promotion
path (they differ only in FP32 summation order)."""
import numpy as np
import pytest
import torch

import fp8_block_scaled_fp8bq_b200 as fq
import fp8bq_workloads as wl
import oracle
from helpers import oracle_act, oracle_weight, assert_gemm_close, bf16_bits, bf16_to_f64, f32, need_gpu, u8

pytestmark = pytest.mark.gpu
NATIVE = fq.GEMM_NATIVE_POW2


@pytest.fixture(autouse=True)
def _gpu_and_clean_error_word():
    need_gpu()
    yield
    st, word = fq.device_error()
    assert st == 0 and word == 0, "device error word 0x%x" % word


def int_codes(rng, shape, vmax):
    v = rng.integers(-vmax, vmax + 1, size=shape).astype(np.float32)
    return torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def run(qa, sa, qw, sw):
    M, K = qa.shape
    ldsa = fq.act_scale_shape(M, K)[1]
    sa_d = torch.zeros((K // 128, ldsa), dtype=torch.float32)
    sa_d[:, :M] = torch.from_numpy(np.ascontiguousarray(sa))
    y = fq.gemm(torch.from_numpy(qa).cuda(), sa_d.cuda(), torch.from_numpy(qw).cuda(),
                torch.from_numpy(np.ascontiguousarray(sw)).cuda(), mode=fq.SCALE_POW2, variant=NATIVE)
    torch.cuda.synchronize()
    return bf16_bits(y), bf16_to_f64(y)


@pytest.mark.parametrize("M,N,K", [(128, 256, 128), (256, 512, 512), (200, 384, 1024), (1, 256, 256)])
def test_exact_distinct_pow2_scales(M, N, K):
    rng = np.random.default_rng(M * 7 + N + K)
    KB, NB = K // 128, (N + 127) // 128
    qa = int_codes(rng, (M, K), 4)
    qw = int_codes(rng, (N, K), 4)
    sa = (2.0 ** (((np.arange(M)[None, :] + np.arange(KB)[:, None]) % 5) - 2)).astype(np.float32)
    sw = (2.0 ** (((np.arange(NB)[:, None] * 3 + np.arange(KB)[None, :]) % 7) - 3)).astype(np.float32)
    bits, _ = run(qa, sa, qw, sw)
    ref = oracle.f64_to_bf16(oracle.gemm(qa, sa, qw, sw))
    assert np.array_equal(bits, ref), np.argwhere(bits != ref)[:5]


@pytest.mark.parametrize("name", list(wl.LLAMA8B_SHAPES))
def test_llama_shapes_against_oracle_and_promotion(name):
    N, K = wl.LLAMA8B_SHAPES[name]
    M = 1024
    x = wl.activations(M, K, seed=N, device="cuda")
    w = wl.weights(N, K, seed=N + 1, device="cuda")
    qa, sa = fq.quant_act(x, fq.SCALE_POW2)
    qw, sw = fq.quant_weight(w, fq.SCALE_POW2)
    yn = fq.gemm(qa, sa, qw, sw, fq.SCALE_POW2, variant=NATIVE)
    yp = fq.gemm(qa, sa, qw, sw, fq.SCALE_POW2, variant=fq.GEMM_PROMOTE)
    torch.cuda.synchronize()
    rng = np.random.default_rng(N)
    rows = np.array(sorted({0, 1, 127, 128, M - 1} | {int(rng.integers(t, t + 128)) for t in range(0, M, 128)}))
    oqa, osa = oracle_act(x, fq.SCALE_POW2, rows)
    oqw, osw = oracle_weight(w, fq.SCALE_POW2)
    ref = oracle.gemm(oqa, osa, oqw, osw, blockint=True)
    assert_gemm_close(bf16_to_f64(yn[torch.from_numpy(rows).cuda()]), ref, "native " + name)
    assert_gemm_close(bf16_to_f64(yn), bf16_to_f64(yp), "native vs promotion " + name)
