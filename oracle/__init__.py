"""fp8bq oracle: numpy/ctypes front end of the plain CPU library in fp8bq_oracle.c.

TEST INFRASTRUCTURE ONLY.  Only tests/, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference legs of ``bench.py`` may import this package.  It
imports nothing from the CUDA path and the CUDA path imports nothing from it.

Method source: "NVIDIA NeMo RL Achieves 48% Speedup With End-to-End FP8
Precision Training", section "Technical breakthrough" (block-wise E4M3, 128x128
weight tiles, 1x128 activation tiles), section "Real-world performance gains"
(per-step scale recalibration) and section "Why this matters for AI economics"
(power-of-2 scales).  Each wrapper below names the C function it calls; the C
file states every reading taken where the pages are silent.

Arrays: bf16 data travels as ``np.uint16`` bit patterns, codes as ``np.uint8``,
scales as ``np.float32``, GEMM results as ``np.float64``.
"""
import ctypes
import os

import numpy as np

from . import build as _build

SCALE_FP32 = 0
SCALE_POW2 = 1

_lib = None


def lib():
    """Load (building first if needed) liboracle.so."""
    global _lib
    if _lib is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        P = ctypes.c_void_p
        I64 = ctypes.c_int64
        L.o_e4m3_decode.restype = ctypes.c_double
        L.o_e4m3_decode.argtypes = [ctypes.c_uint8]
        L.o_e4m3_encode.restype = ctypes.c_uint8
        L.o_e4m3_encode.argtypes = [ctypes.c_float]
        L.o_e4m3_encode_nearest.restype = ctypes.c_uint8
        L.o_e4m3_encode_nearest.argtypes = [ctypes.c_float]
        L.o_sweep_encoders.restype = ctypes.c_uint64
        L.o_sweep_encoders.argtypes = [ctypes.c_uint64, ctypes.c_uint64, ctypes.POINTER(ctypes.c_uint32)]
        L.o_encode_patterns.restype = None
        L.o_encode_patterns.argtypes = [ctypes.c_uint64, ctypes.c_uint64, P]
        L.o_encode_array.restype = None
        L.o_encode_array.argtypes = [P, I64, P]
        L.o_bf16_to_f32.restype = ctypes.c_float
        L.o_bf16_to_f32.argtypes = [ctypes.c_uint16]
        L.o_scale.restype = ctypes.c_float
        L.o_scale.argtypes = [ctypes.c_float, ctypes.c_int]
        L.o_quant_act.restype = None
        L.o_quant_act.argtypes = [P, I64, I64, I64, P, I64, P, I64, ctypes.c_int]
        L.o_quant_weight.restype = None
        L.o_quant_weight.argtypes = [P, I64, I64, I64, P, I64, P, ctypes.c_int]
        L.o_dequant_act.restype = None
        L.o_dequant_act.argtypes = [P, I64, I64, I64, P, I64, P]
        L.o_dequant_weight.restype = None
        L.o_dequant_weight.argtypes = [P, I64, I64, I64, P, P]
        for name in ("o_gemm_rows", "o_gemm_blockint_rows"):
            f = getattr(L, name)
            f.restype = None
            f.argtypes = [P, I64, P, I64, P, I64, P, I64, I64, I64, P, I64, P]
        L.o_grouped_gemm_rows.restype = None
        L.o_grouped_gemm_rows.argtypes = [P, I64, P, I64, P, P, P, I64, I64, I64, P, I64, P]
        L.o_f64_to_bf16.restype = ctypes.c_uint16
        L.o_f64_to_bf16.argtypes = [ctypes.c_double]
        L.o_f64_to_bf16_array.restype = None
        L.o_f64_to_bf16_array.argtypes = [P, I64, P]
        L.o_silu.restype = ctypes.c_double
        L.o_silu.argtypes = [ctypes.c_double]
        L.o_swiglu_bf16.restype = None
        L.o_swiglu_bf16.argtypes = [P, P, I64, P]
        L.o_gemm_wgrad_rows.restype = None
        L.o_gemm_wgrad_rows.argtypes = [P, I64, P, I64, P, I64, P, I64, I64, I64, I64, P, I64, P]
        L.o_decode_attention.restype = None
        L.o_decode_attention.argtypes = [P, P, P, P, P, P, I64, I64, I64, I64, I64, ctypes.c_double, P]
        L.o_prefill_attention.restype = None
        L.o_prefill_attention.argtypes = [P, P, P, P, P, P, P, I64, I64, I64, I64, I64, ctypes.c_double, P, I64, P, P]
        L.o_adamw_step.restype = None
        L.o_adamw_step.argtypes = [P, P, P, P, I64, ctypes.c_float, ctypes.c_float, ctypes.c_float, ctypes.c_float,
                                   ctypes.c_float, I64]
        L.o_f32_to_bf16_array.restype = None
        L.o_f32_to_bf16_array.argtypes = [P, I64, P]
        L.o_num_threads.restype = ctypes.c_int
        L.o_num_threads.argtypes = []
        _lib = L
    return _lib


def _p(a):
    return a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    a = np.asarray(a)
    if a.dtype != dtype:
        raise TypeError("expected %s, got %s" % (np.dtype(dtype), a.dtype))
    return np.ascontiguousarray(a)


def num_threads():
    return lib().o_num_threads()


# --- E4M3 --------------------------------------------------------------------

def e4m3_decode(code):
    return lib().o_e4m3_decode(int(code))


def e4m3_decode_table():
    """float64[256]: the exact value of every code (NaN for 0x7F / 0xFF)."""
    return np.array([e4m3_decode(c) for c in range(256)], dtype=np.float64)


def e4m3_encode(v):
    """Encoder A (round to nearest even, saturate at 448) of one float."""
    return lib().o_e4m3_encode(float(np.float32(v)))


def e4m3_encode_nearest(v):
    """Encoder B (nearest value by brute force, ties to even code)."""
    return lib().o_e4m3_encode_nearest(float(np.float32(v)))


def e4m3_encode_array(v):
    v = _c(np.asarray(v, dtype=np.float32), np.float32)
    out = np.empty(v.shape, dtype=np.uint8)
    lib().o_encode_array(_p(v), v.size, _p(out))
    return out


def encode_patterns(start, count):
    """Encoder A over the fp32 bit patterns [start, start + count)."""
    out = np.empty(count, dtype=np.uint8)
    lib().o_encode_patterns(start, count, _p(out))
    return out


def sweep_encoders(start, count):
    """(mismatches, first mismatching pattern) of encoder A vs B over a pattern range."""
    first = ctypes.c_uint32(0)
    bad = lib().o_sweep_encoders(start, count, ctypes.byref(first))
    return int(bad), int(first.value)


# --- scales and quantizers ----------------------------------------------------

def scale(amax, mode):
    return lib().o_scale(float(np.float32(amax)), int(mode))


def bf16_to_f32(bits):
    """Exact widening of bf16 bit patterns (uint16) to float32."""
    bits = np.asarray(bits, dtype=np.uint16)
    return (bits.astype(np.uint32) << 16).view(np.float32)


def quant_act(x_bits, mode, ldsa=None):
    """1x128 activation quantization of bf16 bits [M, K] -> (codes [M, K], sa [KB, ldsa])."""
    x = _c(x_bits, np.uint16)
    M, K = x.shape
    KB = (K + 127) // 128
    ldsa = M if ldsa is None else ldsa
    q = np.empty((M, K), dtype=np.uint8)
    sa = np.zeros((KB, ldsa), dtype=np.float32)
    lib().o_quant_act(_p(x), M, K, K, _p(q), K, _p(sa), ldsa, int(mode))
    return q, sa


def quant_weight(w_bits, mode):
    """128x128 weight quantization of bf16 bits [N, K] -> (codes [N, K], sw [NB, KB])."""
    w = _c(w_bits, np.uint16)
    N, K = w.shape
    NB, KB = (N + 127) // 128, (K + 127) // 128
    q = np.empty((N, K), dtype=np.uint8)
    sw = np.empty((NB, KB), dtype=np.float32)
    lib().o_quant_weight(_p(w), N, K, K, _p(q), K, _p(sw), int(mode))
    return q, sw


def dequant_act(q, sa):
    q = _c(q, np.uint8)
    sa = _c(sa, np.float32)
    M, K = q.shape
    out = np.empty((M, K), dtype=np.float64)
    lib().o_dequant_act(_p(q), M, K, K, _p(sa), sa.shape[1], _p(out))
    return out


def dequant_weight(q, sw):
    q = _c(q, np.uint8)
    sw = _c(sw, np.float32)
    N, K = q.shape
    out = np.empty((N, K), dtype=np.float64)
    lib().o_dequant_weight(_p(q), N, K, K, _p(sw), _p(out))
    return out


def gemm(qa, sa, qw, sw, rows=None, blockint=False):
    """Y64 = deq(qa) . deq(qw)^T in double (rows: optional subset of output rows)."""
    qa = _c(qa, np.uint8)
    sa = _c(sa, np.float32)
    qw = _c(qw, np.uint8)
    sw = _c(sw, np.float32)
    M, K = qa.shape
    N = qw.shape[0]
    if rows is None:
        r = None
        R = M
    else:
        r = _c(np.asarray(rows, dtype=np.int64), np.int64)
        R = r.size
    y = np.empty((R, N), dtype=np.float64)
    f = lib().o_gemm_blockint_rows if blockint else lib().o_gemm_rows
    f(_p(qa), K, _p(sa), sa.shape[1], _p(qw), K, _p(sw), M, N, K,
      None if r is None else _p(r), R, _p(y))
    return y


def grouped_gemm(qa, sa, qw, sw, offsets, rows=None):
    """Per-expert Y64 for row-sorted activations; qw [E, N, K], sw [E, NB, KB]."""
    qa = _c(qa, np.uint8)
    sa = _c(sa, np.float32)
    qw = _c(qw, np.uint8)
    sw = _c(sw, np.float32)
    off = _c(np.asarray(offsets, dtype=np.int64), np.int64)
    E, N, K = qw.shape
    if rows is None:
        r = None
        R = int(off[-1])
    else:
        r = _c(np.asarray(rows, dtype=np.int64), np.int64)
        R = r.size
    y = np.empty((R, N), dtype=np.float64)
    lib().o_grouped_gemm_rows(_p(qa), K, _p(sa), sa.shape[1], _p(qw), _p(sw), _p(off), E, N, K,
                              None if r is None else _p(r), R, _p(y))
    return y


def f64_to_bf16(v):
    """Round doubles to bf16 (nearest even), returned as uint16 bit patterns."""
    v = _c(np.asarray(v, dtype=np.float64), np.float64)
    out = np.empty(v.shape, dtype=np.uint16)
    lib().o_f64_to_bf16_array(_p(v), v.size, _p(out))
    return out


# --- gate/up activation (SwiGLU) and the fused gate+up -> H codes composition

def silu(g):
    """silu(g) = g / (1 + e^-g) in double."""
    return lib().o_silu(float(g))


def swiglu_bf16(g_bits, u_bits):
    """h = bf16_RNE(silu(g) * u) elementwise on bf16 bit patterns (double arithmetic)."""
    g = _c(np.asarray(g_bits, dtype=np.uint16), np.uint16)
    u = _c(np.asarray(u_bits, dtype=np.uint16), np.uint16)
    if g.shape != u.shape:
        raise ValueError("gate and up shapes differ")
    h = np.empty(g.shape, dtype=np.uint16)
    lib().o_swiglu_bf16(_p(g), _p(u), g.size, _p(h))
    return h


def split_gate_up(y_bits):
    """De-interleave a gate+up output [R, 2I] whose 128-column blocks alternate
    gate block j, up block j (j = 0..I/128-1) into (g [R, I], u [R, I])."""
    y = np.asarray(y_bits)
    R, N2 = y.shape
    if N2 % 256:
        raise ValueError("the gate+up width must be a multiple of 256")
    blocks = y.reshape(R, N2 // 256, 2, 128)
    return (np.ascontiguousarray(blocks[:, :, 0, :].reshape(R, N2 // 2)),
            np.ascontiguousarray(blocks[:, :, 1, :].reshape(R, N2 // 2)))


def swiglu_quant_from_y(y64, mode):
    """The fused epilogue's definition, from the gate+up GEMM's FP64 result
    [R, 2I]: round to bf16 (the GEMM's output), h = swiglu_bf16(g, u), then the
    1x128 activation quantization of h.  Returns (codes [R, I], scales [I/128, R],
    h bits [R, I])."""
    g, u = split_gate_up(f64_to_bf16(y64))
    h = swiglu_bf16(g, u)
    q, s = quant_act(h, mode)
    return q, s, h


# --- optimizer step + recalibration -------------------------------------------

def adamw_step(p, g, m, v, lr, beta1, beta2, eps, weight_decay, step):
    """One binary32 AdamW step; returns new (p, m, v) (inputs are not modified)."""
    p = np.array(_c(p, np.float32), copy=True)
    m = np.array(_c(m, np.float32), copy=True)
    v = np.array(_c(v, np.float32), copy=True)
    g = _c(g, np.float32)
    if not (p.shape == g.shape == m.shape == v.shape):
        raise ValueError("shapes differ")
    lib().o_adamw_step(_p(p), _p(g), _p(m), _p(v), p.size, float(lr), float(beta1), float(beta2), float(eps),
                       float(weight_decay), int(step))
    return p, m, v


def f32_to_bf16(x):
    """binary32 -> bf16 bit patterns, round to nearest even."""
    x = _c(np.asarray(x, dtype=np.float32), np.float32)
    out = np.empty(x.shape, dtype=np.uint16)
    lib().o_f32_to_bf16_array(_p(x), x.size, _p(out))
    return out


def adamw_recalibrate(p, g, m, v, lr, beta1, beta2, eps, weight_decay, step, mode):
    """The fused optimizer step + recalibration, by composition: the AdamW step
    on the FP32 master weight [N, K], its bf16 copy, and the 128x128
    quantization of that copy.  Returns (p, m, v, w_bits, q, s)."""
    p1, m1, v1 = adamw_step(p, g, m, v, lr, beta1, beta2, eps, weight_decay, step)
    w = f32_to_bf16(p1)
    q, s = quant_weight(w, mode)
    return p1, m1, v1, w, q, s


# --- backward pass of the linear layer ----------------------------------------

def quant_act_t(x_bits, mode):
    """1x128 quantization along the token axis, transposed: bf16 X [M, K] ->
    (codes of X^T [K, M], scales [ceil(M/128), K]).  The quantization of X^T
    over 1x128 tiles of its rows (tokens are the contraction of the
    weight-gradient GEMM)."""
    x = _c(x_bits, np.uint16)
    return quant_act(np.ascontiguousarray(x.T), mode)


def gemm_dgrad(q_dy, s_dy, qw, sw, rows=None):
    """dX = dY . W in double from 1x128 codes of dY [M, N] and the 128x128 codes
    of W [N, K]: the forward GEMM's definition with W^T as the second operand
    (a square tile's scale applies to its transpose unchanged)."""
    return gemm(q_dy, s_dy, np.ascontiguousarray(np.asarray(qw).T), np.ascontiguousarray(np.asarray(sw).T),
                rows=rows)


def gemm_wgrad(qa, sa, qb, sb, rows=None):
    """dW[n, k] = sum_m deq(dY^T)[n, m] deq(X^T)[k, m] in double; qa [N, M], sa [MB, >=N],
    qb [K, M], sb [MB, >=K] (1x128 tiles along m on both operands)."""
    qa = _c(qa, np.uint8)
    sa = _c(sa, np.float32)
    qb = _c(qb, np.uint8)
    sb = _c(sb, np.float32)
    N, M = qa.shape
    K = qb.shape[0]
    if rows is None:
        r = None
        R = N
    else:
        r = _c(np.asarray(rows, dtype=np.int64), np.int64)
        R = r.size
    y = np.empty((R, K), dtype=np.float64)
    lib().o_gemm_wgrad_rows(_p(qa), M, _p(sa), sa.shape[1], _p(qb), M, _p(sb), sb.shape[1], N, K, M,
                            None if r is None else _p(r), R, _p(y))
    return y


# --- decode attention over an FP8 KV cache --------------------------------------

def quant_kv(x_bits, mode):
    """E4M3 codes of a key or value cache [B, S, Hkv, D=128] (bf16 bits) with one
    scale per head vector (one 1x128 tile): returns (codes [B, S, Hkv, D],
    scales [B, S, Hkv])."""
    x = np.asarray(x_bits, dtype=np.uint16)
    B, S, H, D = x.shape
    if D != 128:
        raise ValueError("head dimension must be 128 (one 1x128 tile)")
    q, s = quant_act(x.reshape(B * S * H, D), mode)
    return q.reshape(B, S, H, D), s[0, :B * S * H].reshape(B, S, H)


def decode_attention(q_bits, kq, ks, vq, vs, lens, scale):
    """Attention of one query token per batch entry over its cached tokens
    (see o_decode_attention); returns float64 [B, Hq, D]."""
    q = _c(q_bits, np.uint16)
    kq = _c(kq, np.uint8)
    vq = _c(vq, np.uint8)
    ks = _c(ks, np.float32)
    vs = _c(vs, np.float32)
    lens = _c(np.asarray(lens, dtype=np.int32), np.int32)
    B, Hq, D = q.shape
    _, S, Hkv, _ = kq.shape
    if Hq % Hkv:
        raise ValueError("Hq must be a multiple of Hkv")
    out = np.empty((B, Hq, D), dtype=np.float64)
    lib().o_decode_attention(_p(q), _p(kq), _p(ks), _p(vq), _p(vs), _p(lens), B, Hq, Hkv, S, D, float(scale),
                             _p(out))
    return out


def prefill_attention(qq, qs, kq, ks, vq, vs, lens, scale, rows=None, want_mag=False):
    """Causal attention of FP8 queries over FP8 keys/values of the same
    sequences (see o_prefill_attention).  qq [B, S, Hq, D] codes, qs [B, S, Hq];
    kq, vq [B, S, Hkv, D], ks, vs [B, S, Hkv]; lens [B].  rows: optional flat
    query indices b * S + i.  Returns float64 [R, Hq, D] (and the term
    magnitudes sum_j p_j |v_j| if want_mag)."""
    qq = _c(qq, np.uint8)
    kq = _c(kq, np.uint8)
    vq = _c(vq, np.uint8)
    qs = _c(qs, np.float32)
    ks = _c(ks, np.float32)
    vs = _c(vs, np.float32)
    lens = _c(np.asarray(lens, dtype=np.int32), np.int32)
    B, S, Hq, D = qq.shape
    Hkv = kq.shape[2]
    if Hq % Hkv:
        raise ValueError("Hq must be a multiple of Hkv")
    if rows is None:
        r, R = None, B * S
    else:
        r = _c(np.asarray(rows, dtype=np.int64), np.int64)
        R = r.size
    out = np.empty((R, Hq, D), dtype=np.float64)
    mag = np.empty((R, Hq, D), dtype=np.float64) if want_mag else None
    lib().o_prefill_attention(_p(qq), _p(qs), _p(kq), _p(ks), _p(vq), _p(vs), _p(lens), B, S, Hq, Hkv, D,
                              float(scale), None if r is None else _p(r), R, _p(out),
                              None if mag is None else _p(mag))
    return (out, mag) if want_mag else out
