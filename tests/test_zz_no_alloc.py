"""The allocation-free decode entry point (fp8bq_gemm_decode_noalloc).

It is for callers that cannot allocate device memory when they call (a C or
Fortran host program without a framework's memory pool, a serving loop with a
fixed memory budget): the scratch lives in a fixed device array inside the
library.  This test calls it through the C ABI and checks its output against
fp8bq_gemm_decode with a caller workspace and against the oracle (its own
quantization of the same bf16 activations and weights, FP64 sums; every row up
to M = 64, one row of every 16 above), within the GEMM tolerance of the other
tests, on two calls in a row (the array keeps the previous call's contents,
which must not leak into the next result).  It sits in its own file, collected
last, and passes both alone in a fresh process and after the others.
"""
import ctypes

import numpy as np
import pytest
import torch

import fp8_block_scaled_fp8bq_b200 as fq
import fp8bq_workloads as wl
import oracle
from helpers import assert_gemm_close, bf16_to_f64, need_gpu, oracle_act, oracle_weight

pytestmark = pytest.mark.gpu

WORKSPACE_ERR = 4


def call_noalloc(x, qw, sw, mode, y):
    M, K = x.shape
    N = qw.shape[0]
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return fq.lib().fp8bq_gemm_decode_noalloc(
        ctypes.c_void_p(x.data_ptr()), x.stride(0), ctypes.c_void_p(qw.data_ptr()), qw.stride(0),
        ctypes.c_void_p(sw.data_ptr()), ctypes.c_void_p(y.data_ptr()), y.stride(0), M, N, K, mode, stream)


@pytest.mark.parametrize("name,M,mode", [("qkv", 1, fq.SCALE_FP32), ("down", 16, fq.SCALE_FP32),
                                         ("o", 64, fq.SCALE_POW2), ("gate_up", 256, fq.SCALE_FP32)])
def test_noalloc_matches_workspace_entry_point(name, M, mode):
    need_gpu()
    N, K = wl.LLAMA8B_SHAPES[name]
    w = wl.weights(N, K, seed=N + K, device="cuda")
    qw, sw = fq.quant_weight(w, mode)
    oqw, osw = oracle_weight(w, mode)
    rows = np.arange(M) if M <= 64 else np.arange(0, M, 16)
    for call in range(2):                      # two calls in a row, different inputs
        x = wl.activations(M, K, seed=1000 * call + M, device="cuda")
        ref = fq.gemm_decode(x, qw, sw, mode)
        y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
        st = call_noalloc(x, qw, sw, mode, y)
        assert st == 0, "status %d" % st
        torch.cuda.synchronize()
        assert_gemm_close(bf16_to_f64(y), bf16_to_f64(ref), "%s M=%d call %d" % (name, M, call))
        oqa, osa = oracle_act(x, mode, rows)
        y64 = oracle.gemm(oqa, osa, oqw, osw, blockint=True)
        got = bf16_to_f64(y[torch.from_numpy(rows).cuda()])
        assert_gemm_close(got, y64, "%s M=%d call %d vs oracle" % (name, M, call))
    st, word = fq.device_error()
    assert st == 0 and word == 0


def test_noalloc_refuses_shapes_beyond_its_scratch():
    need_gpu()
    M, N, K = 256, 65536, 131072 * 2           # workspace far beyond 32 MiB; nothing is touched
    assert fq.gemm_decode_workspace_size(M, N, K) > (32 << 20)
    x = torch.empty((1, 1), dtype=torch.bfloat16, device="cuda")
    y = torch.empty((1, 8), dtype=torch.bfloat16, device="cuda")
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    st = fq.lib().fp8bq_gemm_decode_noalloc(ctypes.c_void_p(x.data_ptr()), K, ctypes.c_void_p(x.data_ptr()), K,
                                            ctypes.c_void_p(x.data_ptr()), ctypes.c_void_p(y.data_ptr()), N,
                                            M, N, K, 0, stream)
    assert st == WORKSPACE_ERR
    _ = np
