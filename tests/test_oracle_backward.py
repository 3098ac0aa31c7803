"""Pins of the oracle's backward-pass operations of the FP8 linear layer: the
1x128 quantization along the token axis (transposed output), the data-gradient
GEMM dX = dY W and the weight-gradient GEMM dW = dY^T X.

Training runs the linear layers in FP8 as generation does (section "Technical
breakthrough" of "NVIDIA NeMo RL Achieves 48% Speedup With End-to-End FP8
Precision Training").  The pins use independent routines: numpy float32
division and torch's float8_e4m3fn cast for the quantizer, and exact integer or
exactly representable float64 matrix products (numpy) for the GEMMs, on
non-square shapes so that a transposed operand or scale table fails.
"""
import numpy as np
import torch

import oracle


def _e4m3_values(codes):
    """Decode with torch's float8_e4m3fn (independent of the oracle's decoder)."""
    return torch.from_numpy(np.ascontiguousarray(codes)).view(torch.float8_e4m3fn).float().numpy().astype(np.float64)


def _int_codes(rng, shape, vmax):
    v = rng.integers(-vmax, vmax + 1, size=shape).astype(np.float32)
    return torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def test_quant_act_t_tiles_run_along_the_token_axis():
    rng = np.random.default_rng(0)
    M, K = 300, 40                                   # 3 token blocks, the last one partial
    x = (rng.standard_normal((M, K)) * np.where(rng.random((M, K)) < 0.02, 30.0, 1.0)).astype(np.float32)
    xb = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    q, s = oracle.quant_act_t(xb, oracle.SCALE_FP32)
    assert q.shape == (K, M) and s.shape == (3, K)
    xf = torch.from_numpy(xb.view(np.int16)).view(torch.bfloat16).float().numpy()
    for k in range(K):
        for mb in range(3):
            seg = xf[128 * mb:min(128 * mb + 128, M), k]
            amax = np.float32(np.max(np.abs(seg)))
            scale = np.float32(amax) / np.float32(448.0) if amax > 0 else np.float32(1.0)
            assert s[mb, k] == scale
            ref = torch.from_numpy((seg / scale).astype(np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
            assert np.array_equal(q[k, 128 * mb:128 * mb + len(seg)], ref)


def test_wgrad_integer_codes_unit_scales_exact():
    rng = np.random.default_rng(1)
    N, K, M = 96, 160, 384
    a = _int_codes(rng, (N, M), 8)                    # dY^T codes
    b = _int_codes(rng, (K, M), 8)                    # X^T codes
    sa = np.ones((M // 128, N), np.float32)
    sb = np.ones((M // 128, K), np.float32)
    y = oracle.gemm_wgrad(a, sa, b, sb)
    ref = _e4m3_values(a).astype(np.int64) @ _e4m3_values(b).astype(np.int64).T
    assert np.array_equal(y, ref.astype(np.float64))


def test_wgrad_distinct_pow2_scales_per_row_and_token_block_exact():
    rng = np.random.default_rng(2)
    N, K, M = 72, 136, 512
    a = _int_codes(rng, (N, M), 6)
    b = _int_codes(rng, (K, M), 6)
    MB = M // 128
    sa = np.array([[2.0 ** ((n + mb) % 5 - 2) for n in range(N)] for mb in range(MB)], np.float32)
    sb = np.array([[2.0 ** (-((k + 2 * mb) % 4)) for k in range(K)] for mb in range(MB)], np.float32)
    da = _e4m3_values(a) * np.repeat(sa.T.astype(np.float64), 128, axis=1)
    db = _e4m3_values(b) * np.repeat(sb.T.astype(np.float64), 128, axis=1)
    ref = da @ db.T                                   # every product and sum exact in float64
    assert np.array_equal(oracle.gemm_wgrad(a, sa, b, sb), ref)
    rows = np.array([0, 5, N - 1])
    assert np.array_equal(oracle.gemm_wgrad(a, sa, b, sb, rows=rows), ref[rows])


def test_dgrad_uses_the_transposed_weight_with_the_same_tile_scales_exact():
    rng = np.random.default_rng(3)
    M, N, K = 64, 256, 384                            # dY [M, N], W [N, K]
    qdy = _int_codes(rng, (M, N), 6)
    qw = _int_codes(rng, (N, K), 6)
    sdy = np.array([[2.0 ** ((m + nb) % 3) for m in range(M)] for nb in range(N // 128)], np.float32)
    sw = np.array([[2.0 ** (nb - 2 * kb) for kb in range(K // 128)] for nb in range(N // 128)], np.float32)
    ddy = _e4m3_values(qdy) * np.repeat(sdy.T.astype(np.float64), 128, axis=1)
    dw = _e4m3_values(qw) * np.kron(sw.astype(np.float64), np.ones((128, 128)))
    ref = ddy @ dw                                    # dX = dY W, exact
    assert np.array_equal(oracle.gemm_dgrad(qdy, sdy, qw, sw), ref)
