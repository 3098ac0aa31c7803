"""GPU parity of the fused gate+up epilogue (fp8bq_gemm_swiglu_quant and its
grouped form): H = bf16(silu(g) * u) of the gate+up GEMM and the 1x128
quantization of H, against the oracle (GEMM in FP64, SwiGLU in double, the
1x128 quantizer).

What is unique and what is compared:
  * H: the GPU evaluates silu(g) * u in FP32 and the oracle in double, and the
    GPU's g and u come from an FP32 promotion where the oracle's come from an
    FP64 sum, so a bf16 H may differ by a rounding step where the exact value
    lies next to a bf16 rounding boundary.  H is compared elementwise within
    two bf16 steps, and such differences must be rare.
  * codes and scales: a 1x128 tile whose 128 H values equal the oracle's bit
    for bit must have the oracle's codes and scale bit for bit (both sides then
    quantize the same bf16 values with the same FP32 arithmetic).  Every tile,
    equal or not, must dequantize to within the quantization error bound of
    the oracle's H.
  * the epilogue's quantization equals the library's own 1x128 quantizer run
    on the epilogue's H output, bit for bit (GPU against GPU).
"""
import numpy as np
import pytest
import torch

import fp8_block_scaled_fp8bq_b200 as fq
import fp8bq_workloads as wl
import oracle
from helpers import assert_gemm_close, bf16_bits, bf16_to_f64, f32, need_gpu, oracle_act, oracle_weight, u8

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _gpu_and_clean_error_word():
    need_gpu()
    yield
    st, word = fq.device_error()
    assert st == 0 and word == 0, "device error word 0x%x" % word


def _h_f64(bits):
    return oracle.bf16_to_f32(bits).astype(np.float64)


def _dequant_tiles(q, s):
    """q [R, I] codes, s [I/128, >=R] scales -> float64 [R, I]."""
    R, I = q.shape
    table = oracle.e4m3_decode_table()
    return table[q] * np.repeat(s[:, :R].T.astype(np.float64), 128, axis=1)[:, :I]


def check_against_oracle(qh, sh, h, y64, mode, what, max_diff_frac=2e-3):
    """qh/sh/h: the GPU's outputs for R rows (numpy); y64: the oracle's FP64
    gate+up GEMM of the same rows."""
    oq, osh, oh = oracle.swiglu_quant_from_y(y64, mode)
    R, I = oq.shape
    gh = _h_f64(h)
    rh = _h_f64(oh)
    # Tolerance from the arithmetic.  The GPU's g and u come from an FP32
    # promotion: each may sit one bf16 step (<= 2^-7 relative) from the
    # oracle's, plus the FP32 accumulation error, which is absolute (about
    # 2^-24 per K-block of the partial sums' size; 2^-18 rms(Y) bounds it with
    # margin) and dominates where the sum cancels to a tiny g or u.  Each side
    # rounds H once (2^-8 relative each).  To first order
    #   |dH| <= |silu'(g) u| dg + |silu(g)| du + 2^-8 (|H_gpu| + |H_oracle|),
    #   dg = 2^-7 |g| + a,  du = 2^-7 |u| + a,  a = 2^-18 rms(Y),
    # with silu'(g) = s (1 + g (1 - s)), s = sigmoid(g).
    g, u = oracle.split_gate_up(oracle.f64_to_bf16(y64))
    g, u = _h_f64(g), _h_f64(u)
    a = 2.0 ** -18 * np.sqrt(np.mean(y64 * y64))
    sg = 1.0 / (1.0 + np.exp(-g))
    dsilu = sg * (1.0 + g * (1.0 - sg))
    tol = (np.abs(dsilu * u) * (2.0 ** -7 * np.abs(g) + a) + np.abs(g * sg) * (2.0 ** -7 * np.abs(u) + a)
           + 2.0 ** -8 * (np.abs(gh) + np.abs(rh))) * 1.05
    tol += 1e-30
    diff = np.abs(gh - rh)
    if not np.all(diff <= tol):
        i = np.unravel_index(int(np.argmax(diff / tol)), diff.shape)
        raise AssertionError("%s: H off by %.3g x the bound at %s (g %r, u %r, H gpu %r, H oracle %r)"
                             % (what, float(diff[i] / tol[i]), i, g[i], u[i], gh[i], rh[i]))
    differs = h != oh
    assert differs.mean() <= max_diff_frac, "%s: %.2e of H differ" % (what, differs.mean())
    # tiles with identical H: bit-exact codes and scales
    same_tile = ~differs.reshape(R, I // 128, 128).any(axis=2)          # [R, I/128]
    min_same = 0.9 if same_tile.size >= 50 else 0.5
    assert same_tile.mean() >= min_same, "%s: only %.3f of tiles have identical H" % (what, same_tile.mean())
    qt = qh.reshape(R, I // 128, 128)
    oqt = oq.reshape(R, I // 128, 128)
    bad = same_tile & (qt != oqt).any(axis=2)
    assert not bad.any(), "%s: codes differ in %d tiles with identical H" % (what, int(bad.sum()))
    gs = sh[:, :R].T                                                    # [R, I/128]
    os_ = osh[:, :R].T
    assert np.array_equal(gs.view(np.uint32)[same_tile], os_.view(np.uint32)[same_tile]), what + ": scales"
    # every tile: dequantized codes within the quantization bound of the oracle's H
    deq = _dequant_tiles(qh, sh)
    s_el = np.repeat(gs.astype(np.float64), 128, axis=1)
    bound = np.maximum(2.0 ** -4 * np.abs(gh), 2.0 ** -10 * s_el) * (1 + 2 ** -20) + tol
    assert np.all(np.abs(deq - rh) <= bound), what + ": dequantized H outside the bound"


def run_dense(qa, sa, qw, sw, mode):
    """GPU call on the oracle's codes (host numpy) -> numpy outputs."""
    M, K = qa.shape
    ldsa = fq.act_scale_shape(M, K)[1]
    sa_d = torch.zeros((K // 128, ldsa), dtype=torch.float32)
    sa_d[:, :M] = torch.from_numpy(np.ascontiguousarray(sa[:, :M]))
    qh, sh, h = fq.gemm_swiglu_quant(torch.from_numpy(qa).cuda(), sa_d.cuda(), torch.from_numpy(qw).cuda(),
                                     torch.from_numpy(sw).cuda(), mode, want_h=True)
    torch.cuda.synchronize()
    return u8(qh), f32(sh), bf16_bits(h)


def gate_up(I, K, seed):
    return fq.interleave_gate_up(wl.weights(I, K, seed=seed), wl.weights(I, K, seed=seed + 1))


@pytest.mark.parametrize("mode", [fq.SCALE_FP32, fq.SCALE_POW2])
@pytest.mark.parametrize("M,I,K", [(300, 384, 512), (128, 128, 128), (1, 256, 256), (129, 256, 1024)])
def test_dense_against_oracle(mode, M, I, K):
    x = wl.activations(M, K, seed=M + I)
    w = gate_up(I, K, seed=K)
    qa, sa = oracle.quant_act(bf16_bits(x), mode)
    qw, sw = oracle.quant_weight(bf16_bits(w), mode)
    qh, sh, h = run_dense(qa, sa, qw, sw, mode)
    check_against_oracle(qh, sh, h, oracle.gemm(qa, sa, qw, sw), mode, "dense %dx%dx%d" % (M, I, K),
                         max_diff_frac=1e-2 if M * I < 4096 else 2e-3)


@pytest.mark.parametrize("mode", [fq.SCALE_FP32, fq.SCALE_POW2])
def test_llama_gate_up_full_size(mode):
    """M = 8192 tokens, I = 14336, K = 4096 (the Llama-3.1-8B feed-forward),
    quantized and run on the GPU; the oracle quantizes the same bf16 inputs
    itself and computes 12 sampled rows."""
    M, K = wl.PREFILL_TOKENS, 4096
    N2, _ = wl.LLAMA8B_SHAPES["gate_up"]
    I = N2 // 2
    x = wl.activations(M, K, seed=11, device="cuda")
    w = wl.weights(N2, K, seed=12, device="cuda")   # taken as the interleaved gate+up weight
    qa, sa = fq.quant_act(x, mode)
    qw, sw = fq.quant_weight(w, mode)
    qh, sh, h = fq.gemm_swiglu_quant(qa, sa, qw, sw, mode, want_h=True)
    torch.cuda.synchronize()
    rows = np.sort(np.random.default_rng(3).choice(M, 12, replace=False))
    rows[0], rows[-1] = 0, M - 1
    oqa, osa = oracle_act(x, mode, rows)
    oqw, osw = oracle_weight(w, mode)
    y64 = oracle.gemm(oqa, osa, oqw, osw, blockint=True)
    ri = torch.from_numpy(rows).cuda()
    check_against_oracle(u8(qh[ri]), f32(sh)[:, rows], bf16_bits(h[ri]), y64, mode, "llama gate+up")
    # the epilogue's quantization is the 1x128 quantizer on its own H, bit for bit
    q2, s2 = fq.quant_act(h, mode)
    torch.cuda.synchronize()
    assert torch.equal(q2, qh)
    assert torch.equal(s2[:, :M].contiguous().view(torch.int32), sh[:, :M].contiguous().view(torch.int32))


def test_without_h_output_same_codes():
    M, I, K = 256, 256, 512
    x = wl.activations(M, K, seed=5, device="cuda")
    w = gate_up(I, K, seed=6).cuda()
    qa, sa = fq.quant_act(x)
    qw, sw = fq.quant_weight(w)
    q1, s1, h1 = fq.gemm_swiglu_quant(qa, sa, qw, sw, want_h=True)
    q2, s2, h2 = fq.gemm_swiglu_quant(qa, sa, qw, sw)
    torch.cuda.synchronize()
    assert h2 is None
    assert torch.equal(q1, q2) and torch.equal(s1.view(torch.int32), s2.view(torch.int32))


def test_k_zero_gives_zero_codes_unit_scales():
    M, I = 70, 256
    qa = torch.empty((M, 0), dtype=torch.uint8, device="cuda")
    sa = torch.empty((1, 72), dtype=torch.float32, device="cuda")
    qw = torch.empty((2 * I, 0), dtype=torch.uint8, device="cuda")
    sw = torch.empty((4, 1), dtype=torch.float32, device="cuda")
    qh = torch.full((M, I), 0x55, dtype=torch.uint8, device="cuda")
    sh = torch.full(fq.act_scale_shape(M, I), 7.0, dtype=torch.float32, device="cuda")
    h = torch.full((M, I), 3.0, dtype=torch.bfloat16, device="cuda")
    fq.gemm_swiglu_quant(qa, sa, qw, sw, qh=qh, sh=sh, h=h)
    torch.cuda.synchronize()
    assert torch.all(qh == 0) and torch.all(h == 0) and torch.all(sh[:, :M] == 1.0)


def test_rerun_bit_identical_and_outputs_usable_by_down_gemm():
    """A whole feed-forward block: fused gate+up, then the down GEMM on (qh, sh)
    as they are.  The oracle runs the same chain from the bf16 inputs; rows whose
    H codes and scales equal the oracle's must give the down output within the
    GEMM tolerance."""
    M, I, K = 512, 512, 1024
    mode = fq.SCALE_FP32
    x = wl.activations(M, K, seed=7, device="cuda")
    w = gate_up(I, K, seed=8).cuda()
    wd = wl.weights(K, I, seed=9, device="cuda")   # down projection: I -> K
    qa, sa = fq.quant_act(x, mode)
    qw, sw = fq.quant_weight(w, mode)
    qd, sd = fq.quant_weight(wd, mode)
    q1, s1, _ = fq.gemm_swiglu_quant(qa, sa, qw, sw, mode)
    q2, s2, _ = fq.gemm_swiglu_quant(qa, sa, qw, sw, mode)
    y = fq.gemm(q1, s1, qd, sd, mode)
    torch.cuda.synchronize()
    assert torch.equal(q1, q2) and torch.equal(s1.view(torch.int32), s2.view(torch.int32))
    oq, osc, _ = oracle.swiglu_quant_from_y(oracle.gemm(*oracle_act(x, mode), *oracle_weight(w, mode)), mode)
    yd = oracle.gemm(oq, osc, *oracle_weight(wd, mode))
    rows_ok = np.all(u8(q1) == oq, axis=1) & np.all(f32(s1)[:, :M] == osc, axis=0)
    assert rows_ok.mean() >= 0.5, rows_ok.mean()
    assert_gemm_close(bf16_to_f64(y)[rows_ok], yd[rows_ok], "down after fused gate+up")


# --------------------------------------------------------------------------- grouped

def run_grouped(qa, sa, qw, sw, offsets, mode):
    R, K = qa.shape
    ldsa = fq.act_scale_shape(max(R, 1), K)[1]
    sa_d = torch.zeros((K // 128, ldsa), dtype=torch.float32)
    sa_d[:, :R] = torch.from_numpy(np.ascontiguousarray(sa[:, :R]))
    off = torch.tensor(offsets, dtype=torch.int32).cuda()
    qh, sh, h = fq.grouped_gemm_swiglu_quant(torch.from_numpy(qa).cuda(), sa_d.cuda(), torch.from_numpy(qw).cuda(),
                                             torch.from_numpy(sw).cuda(), off, mode, want_h=True)
    torch.cuda.synchronize()
    return u8(qh), f32(sh), bf16_bits(h)


@pytest.mark.parametrize("mode", [fq.SCALE_FP32, fq.SCALE_POW2])
def test_grouped_against_oracle(mode):
    # experts: empty, one row, a partial tile, several tiles with a ragged tail, empty at the end
    sizes = [0, 1, 77, 300, 128, 0]
    offsets = np.concatenate([[0], np.cumsum(sizes)]).astype(np.int64)
    R, I, K, E = int(offsets[-1]), 256, 384, len(sizes)
    x = wl.activations(R, K, seed=21)
    w = torch.stack([gate_up(I, K, seed=100 + 2 * e) for e in range(E)])
    qa, sa = oracle.quant_act(bf16_bits(x), mode)
    qw, sw = oracle_weight(w, mode)
    qh, sh, h = run_grouped(qa, sa, qw, sw, offsets, mode)
    y64 = oracle.grouped_gemm(qa, sa, qw, sw, offsets)
    check_against_oracle(qh, sh, h, y64, mode, "grouped", max_diff_frac=1e-2)


def test_grouped_equals_dense_per_expert():
    """Each expert's rows of the grouped call equal the dense call on those rows
    with that expert's weight, bit for bit (same tiles, same arithmetic)."""
    sizes = [130, 0, 5, 256]
    offsets = np.concatenate([[0], np.cumsum(sizes)]).astype(np.int64)
    R, I, K, E = int(offsets[-1]), 384, 256, len(sizes)
    x = wl.activations(R, K, seed=31, device="cuda")
    w = torch.stack([gate_up(I, K, seed=200 + 2 * e) for e in range(E)]).cuda()
    qa, sa = fq.quant_act(x)
    qw, sw = fq.quant_weight(w.reshape(E * 2 * I, K))
    qw, sw = qw.view(E, 2 * I, K), sw.view(E, 2 * I // 128, K // 128)
    off = torch.tensor(offsets, dtype=torch.int32).cuda()
    gq, gs, gh = fq.grouped_gemm_swiglu_quant(qa, sa, qw, sw, off, want_h=True)
    for e in range(E):
        r0, r1 = int(offsets[e]), int(offsets[e + 1])
        if r1 == r0:
            continue
        q_e, s_e = fq.quant_act(x[r0:r1])
        dq, ds, dh = fq.gemm_swiglu_quant(q_e, s_e, qw[e].contiguous(), sw[e].contiguous(), want_h=True)
        torch.cuda.synchronize()
        assert torch.equal(gq[r0:r1], dq), e
        assert torch.equal(gh[r0:r1].view(torch.int16), dh.view(torch.int16)), e
        assert torch.equal(gs[:, r0:r1].contiguous().view(torch.int32), ds[:, :r1 - r0].contiguous().view(torch.int32))


def test_moe_up_full_size():
    """The Qwen3-30B-A3B-shaped MoE gate+up (4096 tokens x top-8 = 32768 routed
    rows, 128 experts, K = 2048, I = 768) on the GPU; the oracle quantizes the
    same bf16 inputs and computes sampled rows of every non-empty expert."""
    moe = wl.moe_layer(seed=0, device="cuda")
    off = moe["offsets"]
    x, w = moe["x_up"], moe["w_up"]
    mode = fq.SCALE_FP32
    E, N2, K = w.shape
    qa, sa = fq.quant_act(x, mode)
    qw, sw = fq.quant_weight(w.reshape(E * N2, K), mode)
    qw, sw = qw.view(E, N2, K), sw.view(E, N2 // 128, K // 128)
    qh, sh, h = fq.grouped_gemm_swiglu_quant(qa, sa, qw, sw, off.to(torch.int32).cuda(), mode, want_h=True)
    torch.cuda.synchronize()
    offn = off.numpy()
    rows = set()
    rng = np.random.default_rng(9)
    for e in range(E):
        r0, r1 = int(offn[e]), int(offn[e + 1])
        if r1 > r0:
            rows.update({r0, r1 - 1, int(rng.integers(r0, r1))})
    rows = np.array(sorted(rows), dtype=np.int64)
    oqa, osa = oracle_act(x, mode)
    oqw, osw = oracle_weight(w, mode)
    y64 = oracle.grouped_gemm(oqa, osa, oqw, osw, offn, rows=rows)
    ri = torch.from_numpy(rows).cuda()
    check_against_oracle(u8(qh[ri]), f32(sh)[:, rows], bf16_bits(h[ri]), y64, mode, "moe gate+up")
