"""Failure detection without a GPU fault: every on-chip barrier wait in the
tensor-core kernels is bounded.  The self-test variant runs the promotion GEMM
with its TMA producer disabled, so the MMA issuer's wait for the first stage
never completes; after about a second the kernel records the wait site in the
device error word, the other roles stop, TMEM is freed and the kernel returns.
The host reads FP8BQ_ERR_TIMEOUT, and the context stays usable."""
import numpy as np
import pytest
import torch

import fp8_block_scaled_fp8bq_b200 as fq
import fp8bq_workloads as wl
from helpers import assert_gemm_close, bf16_to_f64, need_gpu

pytestmark = pytest.mark.gpu

TIMEOUT = 5
SITE_MMA_FULL = 2         # the MMA issuer's wait for a filled stage
SITE_EPI_TMEM_FULL = 4    # an epilogue warp's wait for a TMEM partial (may time out first)


def test_bounded_wait_reports_timeout_and_context_survives():
    need_gpu()
    assert fq.device_error() == (0, 0)
    x = wl.activations(256, 256, seed=1, device="cuda")
    w = wl.weights(256, 256, seed=2, device="cuda")
    qa, sa = fq.quant_act(x)
    qw, sw = fq.quant_weight(w)
    y = torch.zeros((256, 256), dtype=torch.bfloat16, device="cuda")
    fq.gemm(qa, sa, qw, sw, out=y, variant=fq.GEMM_SELFTEST_TIMEOUT)
    torch.cuda.synchronize()
    st, word = fq.device_error()
    assert st == TIMEOUT
    assert (word >> 16) in (SITE_MMA_FULL, SITE_EPI_TMEM_FULL)
    assert fq.device_error() == (0, 0)                  # reading cleared it
    # the context still works: a normal GEMM gives the right answer
    y2 = fq.gemm(qa, sa, qw, sw)
    y3 = fq.gemm(qa, sa, qw, sw, variant=fq.GEMM_PROMOTE)
    torch.cuda.synchronize()
    assert torch.equal(y2.view(torch.int16), y3.view(torch.int16))
    assert_gemm_close(bf16_to_f64(y2), bf16_to_f64(y3))
    assert fq.device_error() == (0, 0)
    _ = np
