"""Shared test helpers: tensor <-> numpy bit views, the GEMM tolerance, and the
GPU availability gate.  No method arithmetic lives here."""
import numpy as np
import torch


def bf16_bits(t):
    """bf16 torch tensor (any device) -> numpy uint16 bit patterns."""
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


def u8(t):
    return t.detach().contiguous().cpu().numpy()


def f32(t):
    return t.detach().contiguous().cpu().numpy()


def bf16_to_f64(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


# GEMM tolerance against the oracle's FP64 sum of the same dequantized operands:
# relative Frobenius error <= 2e-3 and per element |err| <= 1e-2 (|ref| + 1e-2 rms(ref)).
# The bf16 output rounding alone contributes <= 2^-9 relative per element
# (~1.1e-3 rms), FP32 accumulation of 128-deep blocks a few 1e-7.
REL_FROB = 2e-3
ELEM_REL = 1e-2
ELEM_FLOOR = 1e-2


def gemm_errors(y, ref):
    y = np.asarray(y, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    err = y - ref
    fro = np.linalg.norm(err) / max(np.linalg.norm(ref), 1e-300)
    rms = np.sqrt(np.mean(ref * ref)) if ref.size else 0.0
    bound = ELEM_REL * (np.abs(ref) + ELEM_FLOOR * rms)
    worst = np.max(np.abs(err) / np.maximum(bound, 1e-300)) if ref.size else 0.0
    return fro, worst


def assert_gemm_close(y, ref, what=""):
    fro, worst = gemm_errors(y, ref)
    assert fro <= REL_FROB, "%s: relative Frobenius error %.3g > %.1g" % (what, fro, REL_FROB)
    assert worst <= 1.0, "%s: per-element error %.3g x the bound" % (what, worst)


def need_gpu():
    """GPU tests fail (not skip) without a device: they must never pass vacuously."""
    assert torch.cuda.is_available(), "gpu-marked test run without a CUDA device"


def oracle_act(x, mode, rows=None):
    """The oracle's own 1x128 quantization of bf16 activations (only `rows`, if
    given: each row's tiles depend on that row alone).  Returns (codes, scales)."""
    import oracle
    if rows is not None:
        x = x[torch.as_tensor(rows, device=x.device)]
    return oracle.quant_act(bf16_bits(x), mode)


def oracle_weight(w, mode):
    """The oracle's own 128x128 quantization of a bf16 weight [N, K] (or
    [E, N, K], tile by tile per expert).  Returns (codes, scales)."""
    import oracle
    if w.dim() == 3:
        E, N, K = w.shape
        q, s = oracle.quant_weight(bf16_bits(w.reshape(E * N, K)), mode)
        return q.reshape(E, N, K), s.reshape(E, N // 128, -(-K // 128))
    return oracle.quant_weight(bf16_bits(w), mode)
