"""GPU parity of the quantizers against the CPU oracle: codes and scales bit-exact.

Covers the element encoder over all 2^32 float32 patterns, the division over a
sweep of (tile amax, element) pairs, the single-linear and Llama-8B-shaped
activations at full size, ragged and unaligned shapes (vector and scalar
paths), weight tiles of every Llama-8B projection, and the multi-tensor
recalibration.
"""
import numpy as np
import pytest
import torch

import fp8_block_scaled_fp8bq_b200 as fq
import fp8bq_workloads as wl
import oracle
from helpers import bf16_bits, f32, need_gpu, u8

pytestmark = pytest.mark.gpu
MODES = [fq.SCALE_FP32, fq.SCALE_POW2]


@pytest.fixture(autouse=True)
def _gpu_and_clean_error_word():
    need_gpu()
    yield
    st, word = fq.device_error()
    assert st == 0 and word == 0, "device error word 0x%x" % word


def check_act(x, mode, q=None, sa=None, ldsa=None):
    """Quantize x on the GPU and compare codes and scales with the oracle."""
    M, K = x.shape
    q, sa = fq.quant_act(x, mode, q=q, sa=sa)
    torch.cuda.synchronize()
    oq, osa = oracle.quant_act(bf16_bits(x), mode, ldsa=sa.shape[1])
    gq = u8(q)[:, :K] if q.dim() == 2 else u8(q)
    assert np.array_equal(gq, oq), "codes differ at %s" % (np.argwhere(gq != oq)[:5],)
    g = f32(sa)[:, :M]
    assert np.array_equal(g.view(np.uint32), osa[:, :M].view(np.uint32)), "scales differ"


def test_e4m3_encoder_all_fp32_patterns():
    step = 1 << 26
    for start in range(-(1 << 31), 1 << 31, step):
        x = torch.arange(start, start + step, dtype=torch.int32, device="cuda").view(torch.float32)
        q = u8(fq.e4m3_encode(x))
        first = start & 0xFFFFFFFF
        ref = oracle.encode_patterns(first, step)
        pats = np.arange(first, first + step, dtype=np.uint32)
        nan = ((pats & 0x7F800000) == 0x7F800000) & ((pats & 0x7FFFFF) != 0)  # outside the contract
        ok = (q == ref) | nan
        assert ok.all(), "first mismatch at pattern 0x%08x" % int(pats[np.argmin(ok)])


def _rows_for_amax(amaxes):
    """1x128 tiles whose element 0 is the amax a and whose other 127 elements run,
    across consecutive rows, over every bf16 pattern x with |x| <= a (both signs)."""
    a = np.asarray(amaxes, dtype=np.int64)
    R = -(-2 * (a + 1) // 127)                              # rows needed per amax
    row_a = np.repeat(a, R)
    row_i = np.arange(int(R.sum()), dtype=np.int64) - np.repeat(np.cumsum(R) - R, R)
    t = row_i[:, None] * 127 + np.arange(127, dtype=np.int64)[None, :]
    A = row_a[:, None]
    x = np.where(t <= A, t, np.where(t < 2 * (A + 1), (t - (A + 1)) | 0x8000, 0))
    return np.concatenate([row_a[:, None], x], axis=1).astype(np.uint16)


@pytest.mark.slow
def test_quotient_every_amax_element_pair():
    """Exhaustive over the quantizer's arithmetic domain: for every finite positive
    bf16 tile amax a and every finite bf16 element x with |x| <= a, the code of
    x / s(a) equals the oracle's.  (The scale depends only on a, so this covers
    every quotient the quantizers can ever form.)"""
    all_a = np.arange(1, 0x7F80, dtype=np.uint32)
    # chunks of about 2^25 elements
    cuts = [0]
    acc = 0
    for i, a in enumerate(all_a):
        acc += 2 * (int(a) + 1)
        if acc >= (1 << 25):
            cuts.append(i + 1)
            acc = 0
    cuts.append(all_a.size)
    for c0, c1 in zip(cuts[:-1], cuts[1:]):
        if c1 <= c0:
            continue
        xb = _rows_for_amax(all_a[c0:c1])
        x = torch.from_numpy(xb.view(np.int16)).view(torch.bfloat16).cuda()
        for mode in MODES:
            check_act(x, mode)


@pytest.mark.parametrize("mode", MODES)
def test_single_linear_activation(mode):
    x, _ = wl.single_linear(seed=0)
    check_act(x.cuda(), mode)


@pytest.mark.parametrize("K", [4096, 14336])
def test_llama_prefill_activation_full(K):
    x = wl.activations(wl.PREFILL_TOKENS, K, seed=K, device="cuda")
    check_act(x, fq.SCALE_FP32)


@pytest.mark.parametrize("mode", MODES)
@pytest.mark.parametrize("M,K", [(1, 128), (3, 8), (129, 136), (37, 300), (5, 1), (64, 4096), (17, 1000)])
def test_activation_ragged_shapes(mode, M, K):
    x = wl.activations(M, K, seed=M * 1000 + K, n_out=min(4, K))
    check_act(x.cuda(), mode)


@pytest.mark.parametrize("mode", MODES)
def test_activation_unaligned_views(mode):
    base = wl.activations(70, 520, seed=3, n_out=5).cuda()
    x = base[:, 3:259]                                    # ldx = 520, pointer off by 6 bytes
    q = torch.zeros((70, 300), dtype=torch.uint8, device="cuda")[:, 1:257]
    check_act(x, mode, q=q)


def test_activation_special_values():
    x = torch.zeros((4, 256), dtype=torch.bfloat16)
    x[1, 3] = -0.0
    x[2, :128] = torch.linspace(-448, 448, 128)
    x[2, 5] = -1e-30                                      # negative underflow keeps its sign
    x[3, 130] = 3.0e38                                    # huge amax
    x[3, 131] = 1e-38
    for mode in MODES:
        check_act(x.cuda(), mode)


def check_weight(w, mode):
    q, sw = fq.quant_weight(w, mode)
    torch.cuda.synchronize()
    oq, osw = oracle.quant_weight(bf16_bits(w), mode)
    assert np.array_equal(u8(q), oq)
    assert np.array_equal(f32(sw).view(np.uint32), osw.view(np.uint32))


@pytest.mark.parametrize("mode", MODES)
@pytest.mark.parametrize("name", list(wl.LLAMA8B_SHAPES))
def test_weight_llama_shapes(mode, name):
    N, K = wl.LLAMA8B_SHAPES[name]
    check_weight(wl.weights(N, K, seed=N + K, device="cuda"), mode)


@pytest.mark.parametrize("mode", MODES)
@pytest.mark.parametrize("N,K", [(1, 1), (200, 300), (128, 128), (129, 257), (300, 1000)])
def test_weight_ragged(mode, N, K):
    check_weight(wl.weights(N, K, seed=N * 7 + K).cuda(), mode)


@pytest.mark.parametrize("mode", MODES)
def test_recalibrate_layer_equals_oracle(mode):
    tensors = []
    for name, (N, K) in wl.LLAMA8B_SHAPES.items():
        w = wl.weights(N, K, seed=wl.layer_weight_seed(0, name), device="cuda")
        w = wl.weight_step(w, seed=wl.layer_weight_seed(0, name) + 1)
        q = torch.empty((N, K), dtype=torch.uint8, device="cuda")
        s = torch.empty((fq.ceil_div(N, 128), fq.ceil_div(K, 128)), dtype=torch.float32, device="cuda")
        tensors.append((w, q, s))
    odd = wl.weights(200, 300, seed=5).cuda()              # a ragged tensor in the same launch
    tensors.append((odd, torch.empty((200, 300), dtype=torch.uint8, device="cuda"),
                    torch.empty((2, 3), dtype=torch.float32, device="cuda")))
    fq.recalibrate(tensors, mode)
    torch.cuda.synchronize()
    for w, q, s in tensors:
        oq, osw = oracle.quant_weight(bf16_bits(w), mode)
        assert np.array_equal(u8(q), oq)
        assert np.array_equal(f32(s).view(np.uint32), osw.view(np.uint32))


def test_recalibrate_whole_model_full_size():
    """The recalibration step at full size: 32 layers x the four Llama-8B-shaped
    weights (6,979,321,856 parameters) after one synthetic update, requantized
    in one call with power-of-2 scales.  Every tile is checked for the scale
    rule (an exact power of two, the smallest with amax <= 448 s) and every
    element for the encode's error bound; the first, the last and two seeded
    tiles of every tensor are compared with the oracle bit for bit."""
    tensors = []
    for layer, name, w in wl.model_weights_after_step(device="cuda"):
        N, K = w.shape
        tensors.append((w, torch.empty((N, K), dtype=torch.uint8, device="cuda"),
                        torch.empty((N // 128, K // 128), dtype=torch.float32, device="cuda")))
    assert sum(w.numel() for w, _, _ in tensors) == 6_979_321_856
    fq.recalibrate(tensors, fq.SCALE_POW2)
    torch.cuda.synchronize()
    rng = np.random.default_rng(2024)
    for w, q, s in tensors:
        N, K = w.shape
        NB, KB = N // 128, K // 128
        # every tile: s = 2^e with amax <= 448 s < 2 amax (smallest such e; amax > 0 here)
        amax = w.float().abs().reshape(NB, 128, KB, 128).amax(dim=(1, 3))
        mant = s.view(torch.int32) & 0x7FFFFF
        assert bool((mant == 0).all()) and bool((amax <= 448.0 * s).all()) and bool((448.0 * s < 2 * amax).all())
        # every element: |dec(q) s - w| <= max(2^-4 |w|, 2^-10 s) (half an E4M3 step, normal or subnormal)
        for r0 in range(0, N, 4096):
            rows = slice(r0, min(N, r0 + 4096))
            se = s[r0 // 128:(rows.stop + 127) // 128].repeat_interleave(128, 0).repeat_interleave(128, 1)
            dec = q[rows].view(torch.float8_e4m3fn).float() * se
            wf = w[rows].float()
            assert bool(((dec - wf).abs() <= torch.maximum(wf.abs() / 16, se / 1024)).all())
        picks = {(0, 0), (NB - 1, KB - 1)} | {(int(rng.integers(NB)), int(rng.integers(KB))) for _ in range(2)}
        for nb, kb in sorted(picks):
            tile = (slice(nb * 128, nb * 128 + 128), slice(kb * 128, kb * 128 + 128))
            oq, osw = oracle.quant_weight(bf16_bits(w[tile]), fq.SCALE_POW2)
            assert np.array_equal(u8(q[tile]), oq)
            assert f32(s[nb, kb]).view(np.uint32) == osw.reshape(-1)[0].view(np.uint32)


def test_recalibrate_many_tensors_crosses_launch_chunks():
    tensors = []
    for i in range(300):                                  # > 128 descriptors: several launches
        N, K = 64 + (i % 5) * 40, 128 + (i % 3) * 72
        w = wl.weights(N, K, seed=i).cuda()
        tensors.append((w, torch.empty((N, K), dtype=torch.uint8, device="cuda"),
                        torch.empty((fq.ceil_div(N, 128), fq.ceil_div(K, 128)), dtype=torch.float32,
                                    device="cuda")))
    fq.recalibrate(tensors, fq.SCALE_POW2)
    torch.cuda.synchronize()
    for w, q, s in tensors[::7]:
        oq, osw = oracle.quant_weight(bf16_bits(w), fq.SCALE_POW2)
        assert np.array_equal(u8(q), oq)
        assert np.array_equal(f32(s), osw)
