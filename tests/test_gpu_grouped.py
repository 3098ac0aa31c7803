"""GPU parity of the grouped (mixture-of-experts) block-scaled GEMM.

Exact cases (bit-exact bf16): integer codes and distinct power-of-two scales
per expert block, with empty, single-row and multi-tile experts.  The
Qwen3-30B-A3B-shaped MoE layer (4096 tokens, top-8 of 128 experts with Zipf
popularity; gate+up 2048->1536 and down 768->2048) at full size against the
oracle on sampled rows of every expert.  Invariants: each expert's rows equal
the dense GEMM of that expert bit for bit; E = 1 equals the dense GEMM;
offsets that break the contract give no fault.
"""
import numpy as np
import pytest
import torch

import fp8_block_scaled_fp8bq_b200 as fq
import fp8bq_workloads as wl
import oracle
from helpers import oracle_act, oracle_weight, assert_gemm_close, bf16_bits, bf16_to_f64, f32, need_gpu, u8

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _gpu_and_clean_error_word():
    need_gpu()
    yield
    st, word = fq.device_error()
    assert st == 0 and word == 0, "device error word 0x%x" % word


def int_codes(rng, shape, vmax):
    v = rng.integers(-vmax, vmax + 1, size=shape).astype(np.float32)
    return torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def run_grouped(qa, sa, qw, sw, offsets, mode=fq.SCALE_POW2):
    R, K = qa.shape
    ldsa = fq.act_scale_shape(max(R, 1), K)[1]
    sa_d = torch.zeros((K // 128, ldsa), dtype=torch.float32)
    sa_d[:, :R] = torch.from_numpy(np.ascontiguousarray(sa))
    off = torch.tensor(np.asarray(offsets), dtype=torch.int32).cuda()
    y = fq.grouped_gemm(torch.from_numpy(qa).cuda(), sa_d.cuda(), torch.from_numpy(qw).cuda(),
                        torch.from_numpy(np.ascontiguousarray(sw)).cuda(), off, mode)
    torch.cuda.synchronize()
    return bf16_bits(y), bf16_to_f64(y)


@pytest.mark.parametrize("counts,N,K", [
    ([0, 1, 130, 0, 7], 256, 256),
    ([300, 5, 0, 129, 128, 1], 384, 512),
    ([0, 0, 0, 17], 256, 128),
])
def test_exact_integer_and_pow2_scales(counts, N, K):
    rng = np.random.default_rng(sum(counts) + N + K)
    E = len(counts)
    off = np.concatenate([[0], np.cumsum(counts)]).astype(np.int64)
    R = int(off[-1])
    KB, NB = K // 128, N // 128
    qa = int_codes(rng, (R, K), 4)
    qw = int_codes(rng, (E, N, K), 4)
    sa = (2.0 ** rng.integers(-2, 3, size=(KB, R))).astype(np.float32)
    sw = (2.0 ** rng.integers(-3, 2, size=(E, NB, KB))).astype(np.float32)
    bits, _ = run_grouped(qa, sa, qw, sw, off)
    ref = oracle.f64_to_bf16(oracle.grouped_gemm(qa, sa, qw, sw, off))
    assert np.array_equal(bits, ref), np.argwhere(bits != ref)[:5]


def test_each_expert_equals_dense_gemm_bitwise():
    rng = np.random.default_rng(3)
    counts = [200, 0, 1, 77, 256]
    E, N, K = len(counts), 512, 384
    off = np.concatenate([[0], np.cumsum(counts)])
    R = int(off[-1])
    x = wl.activations(R, K, seed=9, device="cuda")
    w = wl.weights(E * N, K, seed=10, device="cuda")
    qa, sa = fq.quant_act(x)
    qw, sw = fq.quant_weight(w)                          # [E*N, K]: N % 128 == 0, tiles align with experts
    y = fq.grouped_gemm(qa, sa, qw.view(E, N, K), sw.view(E, N // 128, K // 128),
                        torch.tensor(off, dtype=torch.int32, device="cuda"))
    for e in range(E):
        r0, r1 = int(off[e]), int(off[e + 1])
        if r1 == r0:
            continue
        qa_e, sa_e = fq.quant_act(x[r0:r1].contiguous())
        y_e = fq.gemm(qa_e, sa_e, qw[e * N:(e + 1) * N], sw[e * (N // 128):(e + 1) * (N // 128)])
        torch.cuda.synchronize()
        assert torch.equal(y[r0:r1].view(torch.int16), y_e.view(torch.int16)), e
    _ = rng


def test_single_expert_equals_dense():
    x = wl.activations(333, 512, seed=1, device="cuda")
    w = wl.weights(256, 512, seed=2, device="cuda")
    qa, sa = fq.quant_act(x)
    qw, sw = fq.quant_weight(w)
    y = fq.gemm(qa, sa, qw, sw)
    yg = fq.grouped_gemm(qa, sa, qw.view(1, 256, 512), sw.view(1, 2, 4),
                         torch.tensor([0, 333], dtype=torch.int32, device="cuda"))
    torch.cuda.synchronize()
    assert torch.equal(y.view(torch.int16), yg.view(torch.int16))


def _quant_experts(w, mode):
    E, N, K = w.shape
    qw, sw = fq.quant_weight(w.reshape(E * N, K), mode)
    return qw.view(E, N, K), sw.view(E, N // 128, K // 128)


@pytest.mark.parametrize("which", ["up", "down"])
def test_moe_layer_full_size(which):
    moe = wl.moe_layer(seed=0, device="cuda")
    off = moe["offsets"]
    x = moe["x_" + which]
    w = moe["w_" + which]
    mode = fq.SCALE_FP32
    qa, sa = fq.quant_act(x, mode)
    qw, sw = _quant_experts(w, mode)
    y = fq.grouped_gemm(qa, sa, qw, sw, off.to(torch.int32).cuda(), mode)
    torch.cuda.synchronize()
    offn = off.numpy()
    R = int(offn[-1])
    rows = set()
    rng = np.random.default_rng(5)
    for e in range(len(offn) - 1):
        r0, r1 = int(offn[e]), int(offn[e + 1])
        if r1 > r0:
            rows.update({r0, r1 - 1, int(rng.integers(r0, r1))})
    rows = np.array(sorted(rows), dtype=np.int64)
    oqa, osa = oracle_act(x, mode)
    oqw, osw = oracle_weight(w, mode)
    ref = oracle.grouped_gemm(oqa, osa, oqw, osw, offn, rows=rows)
    got = bf16_to_f64(y[torch.from_numpy(rows).cuda()])
    assert_gemm_close(got, ref, "moe " + which)


def test_contract_breaking_offsets_do_not_fault():
    x = wl.activations(300, 256, seed=3, device="cuda")
    w = wl.weights(3 * 256, 256, seed=4, device="cuda")
    qa, sa = fq.quant_act(x)
    qw, sw = fq.quant_weight(w)
    for bad in ([5, 400, 100, 300], [-7, 10, 9, 1000], [0, 0, 0, 0]):
        fq.grouped_gemm(qa, sa, qw.view(3, 256, 256), sw.view(3, 2, 2),
                        torch.tensor(bad, dtype=torch.int32, device="cuda"))
    torch.cuda.synchronize()


def test_empty_rows_no_op():
    qa = torch.empty((0, 256), dtype=torch.uint8, device="cuda")
    sa = torch.empty((2, 4), dtype=torch.float32, device="cuda")
    qw = torch.zeros((2, 256, 256), dtype=torch.uint8, device="cuda")
    sw = torch.ones((2, 2, 2), dtype=torch.float32, device="cuda")
    fq.grouped_gemm(qa, sa, qw, sw, torch.zeros(3, dtype=torch.int32, device="cuda"))
    torch.cuda.synchronize()
