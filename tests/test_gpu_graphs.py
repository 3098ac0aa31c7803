"""Every entry point can be captured in a CUDA graph: the calls make no host
synchronisation and allocate nothing, so a captured sequence replays with new
inputs copied into its static buffers and gives, bit for bit, what the same
calls give when launched one by one (the kernels are deterministic).
"""
import pytest
import torch

import fp8_block_scaled_fp8bq_b200 as fq
import fp8bq_workloads as wl
from helpers import need_gpu

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _gpu_and_clean_error_word():
    need_gpu()
    yield
    st, word = fq.device_error()
    assert st == 0 and word == 0, "device error word 0x%x" % word


def _same(a, b):
    return torch.equal(a.view(torch.uint8) if a.dtype != torch.uint8 else a,
                       b.view(torch.uint8) if b.dtype != torch.uint8 else b)


def _replay_matches(static_inputs, make_inputs, run):
    """Capture run() on the static inputs, then for two fresh input sets copy
    them in, replay, and compare every output with an eager run on the same
    values."""
    torch.cuda.synchronize()
    run()  # warm-up outside the capture (lazy kernel attributes, workspaces)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        outs = run()
    for seed in (1, 2):
        fresh = make_inputs(seed)
        for dst, src in zip(static_inputs, fresh):
            dst.copy_(src)
        g.replay()
        torch.cuda.synchronize()
        got = [o.clone() for o in outs]
        want = run()
        torch.cuda.synchronize()
        for a, b in zip(got, want):
            assert _same(a, b)
    del g


@pytest.mark.parametrize("mode", [fq.SCALE_FP32, fq.SCALE_POW2])
def test_quantize_and_gemm_in_a_graph(mode):
    M, N, K = 512, 1024, 1024

    def make(seed):
        return [wl.activations(M, K, seed=seed, device="cuda"), wl.weights(N, K, seed=seed + 50, device="cuda")]
    x, w = make(0)
    qa = torch.empty((M, K), dtype=torch.uint8, device="cuda")
    sa = torch.empty(fq.act_scale_shape(M, K), dtype=torch.float32, device="cuda")
    qw = torch.empty((N, K), dtype=torch.uint8, device="cuda")
    sw = torch.empty((N // 128, K // 128), dtype=torch.float32, device="cuda")
    y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")

    def run():
        fq.quant_act(x, mode, q=qa, sa=sa)
        fq.recalibrate([(w, qw, sw)], mode)
        fq.gemm(qa, sa, qw, sw, mode, out=y)
        return [qa, sa, qw, sw, y]
    _replay_matches([x, w], make, run)


def test_decode_gemm_in_a_graph():
    M, N, K = 16, 4096, 4096
    qw, sw = fq.quant_weight(wl.weights(N, K, seed=7, device="cuda"), fq.SCALE_FP32)

    def make(seed):
        return [wl.activations(M, K, seed=seed, device="cuda")]
    (x,) = make(0)
    y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    ws = torch.zeros(max(fq.gemm_decode_workspace_size(M, N, K), 256), dtype=torch.uint8, device="cuda")

    def run():
        fq.gemm_decode(x, qw, sw, fq.SCALE_FP32, out=y, ws=ws)
        return [y]
    _replay_matches([x], make, run)


def test_decode_attention_in_a_graph():
    B, Hkv, Hq, S = 4, 2, 8, 1000
    g0 = torch.Generator(device="cuda").manual_seed(3)
    k = (torch.randn((B, S, Hkv, 128), generator=g0, device="cuda")).to(torch.bfloat16)
    v = (torch.randn((B, S, Hkv, 128), generator=g0, device="cuda")).to(torch.bfloat16)
    kq = torch.empty((B, S, Hkv, 128), dtype=torch.uint8, device="cuda")
    vq = torch.empty_like(kq)
    ks = torch.empty((B, S, Hkv), dtype=torch.float32, device="cuda")
    vs = torch.empty_like(ks)
    qk, sk = fq.quant_act(k.reshape(-1, 128), fq.SCALE_FP32)
    qv, sv = fq.quant_act(v.reshape(-1, 128), fq.SCALE_FP32)
    kq.copy_(qk.reshape(B, S, Hkv, 128))
    vq.copy_(qv.reshape(B, S, Hkv, 128))
    ks.copy_(sk[0, :B * S * Hkv].reshape(B, S, Hkv))
    vs.copy_(sv[0, :B * S * Hkv].reshape(B, S, Hkv))
    lens = torch.tensor([1000, 1, 517, 999], dtype=torch.int32, device="cuda")

    def make(seed):
        g = torch.Generator(device="cuda").manual_seed(seed)
        return [torch.randn((B, Hq, 128), generator=g, device="cuda").to(torch.bfloat16)]
    (q,) = make(0)
    o = torch.empty((B, Hq, 128), dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(max(int(fq.lib().fp8bq_decode_attention_workspace_size(B, Hq, Hkv, S)), 16), dtype=torch.uint8,
                     device="cuda")

    def run():
        fq.decode_attention(q, kq, ks, vq, vs, lens, 0.09, out=o, ws=ws)
        return [o]
    _replay_matches([q], make, run)


def test_grouped_gemm_in_a_graph():
    E, N, K = 8, 512, 512
    counts = [0, 200, 3, 128, 0, 77, 300, 1]
    R = sum(counts)
    offs = torch.tensor([0] + list(torch.tensor(counts).cumsum(0)), dtype=torch.int32, device="cuda")
    w = torch.stack([wl.weights(N, K, seed=100 + e, device="cuda") for e in range(E)])
    qw = torch.empty((E, N, K), dtype=torch.uint8, device="cuda")
    sw = torch.empty((E, N // 128, K // 128), dtype=torch.float32, device="cuda")
    for e in range(E):
        fq.quant_weight(w[e], fq.SCALE_FP32, q=qw[e], sw=sw[e])

    def make(seed):
        return [wl.activations(R, K, seed=seed, device="cuda")]
    (x,) = make(0)
    qa = torch.empty((R, K), dtype=torch.uint8, device="cuda")
    sa = torch.empty(fq.act_scale_shape(R, K), dtype=torch.float32, device="cuda")
    y = torch.empty((R, N), dtype=torch.bfloat16, device="cuda")

    def run():
        fq.quant_act(x, fq.SCALE_FP32, q=qa, sa=sa)
        fq.grouped_gemm(qa, sa, qw, sw, offs, fq.SCALE_FP32, out=y)
        return [y]
    _replay_matches([x], make, run)
