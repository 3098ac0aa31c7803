"""Python binding of libfp8bq (the block-wise FP8 E4M3 linear layer for B200).

Argument marshalling only: every step of the path runs in the library's CUDA
kernels, called through its C ABI (include/fp8bq.h) with ctypes.  torch is
used for device memory and streams.  There is no fallback: if the library is
missing or fails to load, every call raises.

Method: "NVIDIA NeMo RL Achieves 48% Speedup With End-to-End FP8 Precision
Training", section "Technical breakthrough" (block-wise E4M3, 1x128 activation
tiles, 128x128 weight tiles, FP8 linear layers), section "Real-world
performance gains" (per-step scale recalibration; mixture-of-experts) and
section "Why this matters for AI economics" (power-of-2 scales).
"""
import ctypes
import math
import os

import torch

SCALE_FP32 = 0
SCALE_POW2 = 1

GEMM_AUTO = 0
GEMM_PROMOTE = 1
GEMM_NATIVE_POW2 = 2
GEMM_PROMOTE_PAIR = 3
GEMM_PROMOTE_PAIR_N128 = 4
GEMM_SELFTEST_TIMEOUT = 99

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libfp8bq.so")

_STATUS = {0: "FP8BQ_OK", 1: "FP8BQ_ERR_INVALID_ARG", 2: "FP8BQ_ERR_UNSUPPORTED", 3: "FP8BQ_ERR_CUDA",
           4: "FP8BQ_ERR_WORKSPACE", 5: "FP8BQ_ERR_TIMEOUT"}


class Fp8bqError(RuntimeError):
    def __init__(self, status, what, detail=""):
        self.status = status
        msg = "%s failed: %s" % (what, _STATUS.get(status, str(status)))
        if detail:
            msg += " (" + detail + ")"
        super().__init__(msg)


class WeightDesc(ctypes.Structure):
    _fields_ = [("w", ctypes.c_void_p), ("q", ctypes.c_void_p), ("s", ctypes.c_void_p),
                ("N", ctypes.c_int64), ("K", ctypes.c_int64), ("ldw", ctypes.c_int64), ("ldq", ctypes.c_int64)]


class AdamWDesc(ctypes.Structure):
    _fields_ = [("param", ctypes.c_void_p), ("grad", ctypes.c_void_p), ("exp_avg", ctypes.c_void_p),
                ("exp_avg_sq", ctypes.c_void_p), ("w", ctypes.c_void_p), ("q", ctypes.c_void_p),
                ("s", ctypes.c_void_p), ("N", ctypes.c_int64), ("K", ctypes.c_int64)]


class AdamWConfig(ctypes.Structure):
    _fields_ = [("lr", ctypes.c_float), ("beta1", ctypes.c_float), ("beta2", ctypes.c_float),
                ("eps", ctypes.c_float), ("weight_decay", ctypes.c_float), ("step", ctypes.c_int64)]


# name -> (restype, argtypes); the full list of the C ABI's entry points.
P, I64, I32, SZ = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_size_t
SIGNATURES = {
    "fp8bq_version": (ctypes.c_int, []),
    "fp8bq_status_string": (ctypes.c_char_p, [I32]),
    "fp8bq_last_cuda_error": (ctypes.c_char_p, []),
    "fp8bq_get_last_cuda_error": (I32, [ctypes.POINTER(ctypes.c_int)]),
    "fp8bq_recalibrate_workspace_size": (SZ, [I32]),
    "fp8bq_grouped_gemm_workspace_size": (SZ, [I32, I64, I64, I64]),
    "fp8bq_get_device_error": (I32, [ctypes.POINTER(ctypes.c_uint64)]),
    "fp8bq_e4m3_encode": (I32, [P, I64, P, P]),
    "fp8bq_quant_act": (I32, [P, I64, I64, I64, P, I64, P, I64, I32, P]),
    "fp8bq_quant_weight": (I32, [P, I64, I64, I64, P, I64, P, I32, P]),
    "fp8bq_recalibrate": (I32, [ctypes.POINTER(WeightDesc), I32, I32, P]),
    "fp8bq_gemm": (I32, [P, I64, P, I64, P, I64, P, P, I64, I64, I64, I64, I32, P]),
    "fp8bq_gemm_ex": (I32, [P, I64, P, I64, P, I64, P, P, I64, I64, I64, I64, I32, I32, P]),
    "fp8bq_gemm_decode_workspace_size": (SZ, [I64, I64, I64]),
    "fp8bq_gemm_decode": (I32, [P, I64, P, I64, P, P, I64, I64, I64, I64, I32, P, SZ, P]),
    "fp8bq_gemm_decode_noalloc": (I32, [P, I64, P, I64, P, P, I64, I64, I64, I64, I32, P]),
    "fp8bq_grouped_gemm": (I32, [P, I64, P, I64, P, P, P, I32, I64, I64, I64, P, I64, I32, P]),
    "fp8bq_quant_act_t": (I32, [P, I64, I64, I64, P, I64, P, I64, I32, P]),
    "fp8bq_transpose_weight": (I32, [P, I64, I64, I64, P, P, I64, P, P]),
    "fp8bq_gemm_wgrad": (I32, [P, I64, P, I64, P, I64, P, I64, P, I64, I64, I64, I64, I32, P]),
    "fp8bq_kv_cache_append": (I32, [P, P, P, P, P, P, P, I64, I64, I64, I32, P]),
    "fp8bq_decode_attention_workspace_size": (SZ, [I64, I64, I64, I64]),
    "fp8bq_decode_attention": (I32, [P, P, P, P, P, P, I64, I64, I64, I64, ctypes.c_float, P, P, SZ, P]),
    "fp8bq_prefill_attention": (I32, [P, P, P, P, P, P, P, I64, I64, I64, I64, ctypes.c_float, P, P]),
    "fp8bq_adamw_recalibrate": (I32, [ctypes.POINTER(AdamWDesc), I32, ctypes.POINTER(AdamWConfig), I32, P]),
    "fp8bq_gemm_swiglu_quant": (I32, [P, I64, P, I64, P, I64, P, P, I64, P, I64, P, I64, I64, I64, I64, I32, P]),
    "fp8bq_grouped_gemm_swiglu_quant": (I32, [P, I64, P, I64, P, P, P, I32, I64, I64, I64, P, I64, P, I64, P, I64,
                                              I32, P]),
}

_lib = None


def lib():
    """The loaded C library (raises if it is missing: there is no fallback)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError("libfp8bq.so is not built (run __graft_entry__.build() or "
                               "python fp8_block_scaled_fp8bq_b200/build.py)")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


def _check(status, what):
    if status != 0:
        detail = ""
        if status == 3:
            detail = lib().fp8bq_last_cuda_error().decode(errors="replace")
        raise Fp8bqError(status, what, detail)


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else None


def _ld(t):
    assert t.dim() == 2 and t.stride(1) == 1, "row-major 2-D tensor with unit column stride expected"
    return t.stride(0)


def ceil_div(a, b):
    return -(-a // b)


def act_scale_shape(M, K):
    """sa is [ceil(K/128), ldsa] with ldsa = M rounded up to a multiple of 4."""
    return ceil_div(K, 128), ceil_div(max(M, 1), 4) * 4


def e4m3_encode(x, q=None, stream=None):
    """Element-wise E4M3 code (round to nearest even, saturate at 448) of fp32 x."""
    if q is None:
        q = torch.empty(x.shape, dtype=torch.uint8, device=x.device)
    _check(lib().fp8bq_e4m3_encode(_ptr(x), x.numel(), _ptr(q), _stream(stream)), "fp8bq_e4m3_encode")
    return q


def quant_act(x, mode=SCALE_FP32, q=None, sa=None, stream=None):
    """1x128 E4M3 quantization of bf16 x [M, K] -> (codes uint8 [M, K], scales fp32 [KB, ldsa])."""
    M, K = x.shape
    if q is None:
        q = torch.empty((M, K), dtype=torch.uint8, device=x.device)
    if sa is None:
        sa = torch.empty(act_scale_shape(M, K), dtype=torch.float32, device=x.device)
    _check(lib().fp8bq_quant_act(_ptr(x), M, K, _ld(x), _ptr(q), _ld(q), _ptr(sa), sa.stride(0),
                                 mode, _stream(stream)), "fp8bq_quant_act")
    return q, sa


def quant_weight(w, mode=SCALE_FP32, q=None, sw=None, stream=None):
    """128x128 E4M3 quantization of bf16 w [N, K] -> (codes uint8 [N, K], scales fp32 [NB, KB])."""
    N, K = w.shape
    if q is None:
        q = torch.empty((N, K), dtype=torch.uint8, device=w.device)
    if sw is None:
        sw = torch.empty((ceil_div(N, 128), ceil_div(K, 128)), dtype=torch.float32, device=w.device)
    _check(lib().fp8bq_quant_weight(_ptr(w), N, K, _ld(w), _ptr(q), _ld(q), _ptr(sw), mode, _stream(stream)),
           "fp8bq_quant_weight")
    return q, sw


def recalibrate(tensors, mode=SCALE_POW2, stream=None):
    """Requantize every 128x128 tile of [(w, q, s), ...] in place (per-step recalibration)."""
    arr = (WeightDesc * len(tensors))()
    for i, (w, q, s) in enumerate(tensors):
        N, K = w.shape
        arr[i] = WeightDesc(w.data_ptr(), q.data_ptr(), s.data_ptr(), N, K, _ld(w), _ld(q))
    _check(lib().fp8bq_recalibrate(arr, len(tensors), mode, _stream(stream)), "fp8bq_recalibrate")


def quant_act_t(x, mode=SCALE_FP32, qt=None, st=None, stream=None):
    """Token-axis 1x128 quantization of bf16 x [M, K] with transposed output ->
    (codes of x^T uint8 [K, ldqt>=M], scales fp32 [ceil(M/128), ldst>=K])."""
    M, K = x.shape
    if qt is None:
        qt = torch.empty((K, ceil_div(max(M, 1), 16) * 16), dtype=torch.uint8, device=x.device)
    if st is None:
        st = torch.empty((ceil_div(M, 128), ceil_div(max(K, 1), 4) * 4), dtype=torch.float32, device=x.device)
    _check(lib().fp8bq_quant_act_t(_ptr(x), M, K, _ld(x), _ptr(qt), _ld(qt), _ptr(st), st.stride(0), mode,
                                   _stream(stream)), "fp8bq_quant_act_t")
    return qt, st


def transpose_weight(q, sw, qt=None, swt=None, stream=None):
    """Codes and tile scales of W^T from those of W [N, K] (no requantization)."""
    N, K = q.shape
    if qt is None:
        qt = torch.empty((K, N), dtype=torch.uint8, device=q.device)
    if swt is None:
        swt = torch.empty((sw.shape[1], sw.shape[0]), dtype=torch.float32, device=q.device)
    _check(lib().fp8bq_transpose_weight(_ptr(q), N, K, _ld(q), _ptr(sw), _ptr(qt), _ld(qt), _ptr(swt),
                                        _stream(stream)), "fp8bq_transpose_weight")
    return qt, swt


def gemm_dgrad(q_dy, s_dy, qwt, swt, mode=SCALE_FP32, out=None, stream=None):
    """dX = dY . W from dY's 1x128 codes and W^T's codes (transpose_weight)."""
    return gemm(q_dy, s_dy, qwt, swt, mode, out=out, stream=stream)


def gemm_wgrad(qa, sa, qb, sb, M, mode=SCALE_FP32, out=None, stream=None):
    """dW [N, K] = dY^T X from the token-axis codes of dY^T (qa [N, >=M], sa) and
    X^T (qb [K, >=M], sb); M = tokens."""
    N, K = qa.shape[0], qb.shape[0]
    if out is None:
        out = torch.empty((N, K), dtype=torch.bfloat16, device=qa.device)
    _check(lib().fp8bq_gemm_wgrad(_ptr(qa), _ld(qa), _ptr(sa), sa.stride(0), _ptr(qb), _ld(qb), _ptr(sb),
                                  sb.stride(0), _ptr(out), _ld(out), N, K, M, mode, _stream(stream)),
           "fp8bq_gemm_wgrad")
    return out


def kv_cache_append(k_new, v_new, positions, kq, ks, vq, vs, mode=SCALE_FP32, stream=None):
    """Quantize one new token per sequence into the FP8 cache at positions[b]."""
    B, S, Hkv, D = kq.shape
    _check(lib().fp8bq_kv_cache_append(_ptr(k_new), _ptr(v_new), _ptr(positions), _ptr(kq), _ptr(ks), _ptr(vq),
                                       _ptr(vs), B, Hkv, S, mode, _stream(stream)), "fp8bq_kv_cache_append")


def decode_attention(q, kq, ks, vq, vs, seq_lens, softmax_scale=None, out=None, ws=None, stream=None):
    """One query token per sequence over its FP8 KV cache; q bf16 [B, Hq, 128]."""
    B, Hq, D = q.shape
    _, S, Hkv, _ = kq.shape
    if softmax_scale is None:
        softmax_scale = 1.0 / float(D) ** 0.5
    if out is None:
        out = torch.empty((B, Hq, D), dtype=torch.bfloat16, device=q.device)
    need = int(lib().fp8bq_decode_attention_workspace_size(B, Hq, Hkv, S))
    if ws is None:
        ws = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    _check(lib().fp8bq_decode_attention(_ptr(q), _ptr(kq), _ptr(ks), _ptr(vq), _ptr(vs), _ptr(seq_lens), B, Hq, Hkv,
                                        S, softmax_scale, _ptr(out), _ptr(ws), ws.numel(), _stream(stream)),
           "fp8bq_decode_attention")
    return out


def prefill_attention(qq, qs, kq, ks, vq, vs, seq_lens, softmax_scale=None, out=None, stream=None):
    """Causal attention of FP8 queries over FP8 keys and values of the same
    sequences.  qq uint8 [B, S, Hq, 128], qs fp32 [B, S, Hq]; kq, vq uint8
    [B, S, Hkv, 128], ks, vs fp32 [B, S, Hkv]; seq_lens int32 [B] (device).
    Returns bf16 [B, S, Hq, 128]."""
    B, S, Hq, D = qq.shape
    Hkv = kq.shape[2]
    if softmax_scale is None:
        softmax_scale = 1.0 / math.sqrt(D)
    for t in (qq, qs, kq, ks, vq, vs, seq_lens):
        assert t.is_contiguous(), "contiguous tensors expected"
    if out is None:
        out = torch.empty((B, S, Hq, D), dtype=torch.bfloat16, device=qq.device)
    _check(lib().fp8bq_prefill_attention(_ptr(qq), _ptr(qs), _ptr(kq), _ptr(ks), _ptr(vq), _ptr(vs), _ptr(seq_lens),
                                         B, S, Hq, Hkv, float(softmax_scale), _ptr(out), _stream(stream)),
           "fp8bq_prefill_attention")
    return out


def adamw_recalibrate(tensors, lr, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=0.0, step=1, mode=SCALE_POW2,
                      stream=None):
    """One AdamW step on fp32 master weights fused with their 128x128 recalibration.

    tensors: [(param, grad, exp_avg, exp_avg_sq, w_bf16_or_None, q, s), ...], all
    dense [N, K] (s [ceil(N/128), ceil(K/128)]); updated in place."""
    arr = (AdamWDesc * len(tensors))()
    for i, (p, g, m, v, w, q, s) in enumerate(tensors):
        N, K = p.shape
        for t in (p, g, m, v, q) + ((w,) if w is not None else ()):
            if t.shape != (N, K) or not t.is_contiguous():
                raise ValueError("dense [N, K] tensors expected")
        arr[i] = AdamWDesc(p.data_ptr(), g.data_ptr(), m.data_ptr(), v.data_ptr(),
                           w.data_ptr() if w is not None else None, q.data_ptr(), s.data_ptr(), N, K)
    cfg = AdamWConfig(lr, beta1, beta2, eps, weight_decay, step)
    _check(lib().fp8bq_adamw_recalibrate(arr, len(tensors), ctypes.byref(cfg), mode, _stream(stream)),
           "fp8bq_adamw_recalibrate")


def gemm(qa, sa, qw, sw, mode=SCALE_FP32, out=None, variant=GEMM_AUTO, stream=None):
    """Block-scaled FP8 GEMM: bf16 [M, N] = deq(qa) . deq(qw)^T."""
    M, K = qa.shape
    N = qw.shape[0]
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=qa.device)
    _check(lib().fp8bq_gemm_ex(_ptr(qa), _ld(qa), _ptr(sa), sa.stride(0), _ptr(qw), _ld(qw), _ptr(sw),
                               _ptr(out), _ld(out), M, N, K, mode, variant, _stream(stream)), "fp8bq_gemm")
    return out


def gemm_decode_workspace_size(M, N, K):
    return int(lib().fp8bq_gemm_decode_workspace_size(M, N, K))


def gemm_decode(x, qw, sw, mode=SCALE_FP32, out=None, ws=None, stream=None):
    """Small-M linear with on-the-fly 1x128 activation quantization (`ws`: an
    optional uint8 workspace of gemm_decode_workspace_size bytes)."""
    M, K = x.shape
    N = qw.shape[0]
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=x.device)
    need = gemm_decode_workspace_size(M, N, K)
    if ws is None:
        ws = torch.empty(max(need, 256), dtype=torch.uint8, device=x.device)
    _check(lib().fp8bq_gemm_decode(_ptr(x), _ld(x), _ptr(qw), _ld(qw), _ptr(sw), _ptr(out), _ld(out), M, N, K,
                                   mode, _ptr(ws), ws.numel(), _stream(stream)), "fp8bq_gemm_decode")
    return out


def grouped_gemm(qa, sa, qw, sw, offsets, mode=SCALE_FP32, out=None, stream=None):
    """Per-expert block-scaled GEMM over expert-sorted rows (offsets int32 [E+1] on the device)."""
    R, K = qa.shape
    E, N, _ = qw.shape
    if out is None:
        out = torch.empty((R, N), dtype=torch.bfloat16, device=qa.device)
    _check(lib().fp8bq_grouped_gemm(_ptr(qa), _ld(qa), _ptr(sa), sa.stride(0), _ptr(qw), _ptr(sw), _ptr(offsets),
                                    E, R, N, K, _ptr(out), _ld(out), mode, _stream(stream)), "fp8bq_grouped_gemm")
    return out


def interleave_gate_up(w_gate, w_up):
    """Storage layout of a gated feed-forward block's gate+up weight for
    gemm_swiglu_quant: [..., 2I, K] with 128-row blocks alternating gate block j,
    up block j.  A one-time layout step when the weights are created; the
    recalibration then quantizes the interleaved tensor in place every step."""
    if w_gate.shape != w_up.shape or w_gate.shape[-2] % 128:
        raise ValueError("gate and up must have the same shape with a multiple of 128 rows")
    *lead, I, K = w_gate.shape
    g = w_gate.reshape(*lead, I // 128, 1, 128, K)
    u = w_up.reshape(*lead, I // 128, 1, 128, K)
    return torch.cat([g, u], dim=-3).reshape(*lead, 2 * I, K).contiguous()


def gemm_swiglu_quant(qa, sa, qw, sw, mode=SCALE_FP32, qh=None, sh=None, h=None, want_h=False, stream=None):
    """Gate+up GEMM with H = bf16(silu(g) * u) and its 1x128 quantization in the epilogue.

    qw/sw: the interleaved gate+up weight [2I, K] (see interleave_gate_up).
    Returns (qh uint8 [M, I], sh fp32 [I/128, ldsh], h bf16 [M, I] or None)."""
    M, K = qa.shape
    I = qw.shape[0] // 2
    if qh is None:
        qh = torch.empty((M, I), dtype=torch.uint8, device=qa.device)
    if sh is None:
        sh = torch.empty(act_scale_shape(M, I), dtype=torch.float32, device=qa.device)
    if h is None and want_h:
        h = torch.empty((M, I), dtype=torch.bfloat16, device=qa.device)
    _check(lib().fp8bq_gemm_swiglu_quant(_ptr(qa), _ld(qa), _ptr(sa), sa.stride(0), _ptr(qw), _ld(qw), _ptr(sw),
                                         _ptr(qh), _ld(qh), _ptr(sh), sh.stride(0), _ptr(h),
                                         _ld(h) if h is not None else 0, M, I, K, mode, _stream(stream)),
           "fp8bq_gemm_swiglu_quant")
    return qh, sh, h


def grouped_gemm_swiglu_quant(qa, sa, qw, sw, offsets, mode=SCALE_FP32, qh=None, sh=None, h=None, want_h=False,
                              stream=None):
    """Grouped (mixture-of-experts) form of gemm_swiglu_quant; qw [E, 2I, K] interleaved per expert."""
    R, K = qa.shape
    E, N2, _ = qw.shape
    I = N2 // 2
    if qh is None:
        qh = torch.empty((R, I), dtype=torch.uint8, device=qa.device)
    if sh is None:
        sh = torch.empty(act_scale_shape(R, I), dtype=torch.float32, device=qa.device)
    if h is None and want_h:
        h = torch.empty((R, I), dtype=torch.bfloat16, device=qa.device)
    _check(lib().fp8bq_grouped_gemm_swiglu_quant(_ptr(qa), _ld(qa), _ptr(sa), sa.stride(0), _ptr(qw), _ptr(sw),
                                                 _ptr(offsets), E, R, I, K, _ptr(qh), _ld(qh), _ptr(sh),
                                                 sh.stride(0), _ptr(h), _ld(h) if h is not None else 0, mode,
                                                 _stream(stream)),
           "fp8bq_grouped_gemm_swiglu_quant")
    return qh, sh, h


def device_error():
    """(status, raw word) of the device error word; reading clears it (synchronizes)."""
    v = ctypes.c_uint64(0)
    st = lib().fp8bq_get_device_error(ctypes.byref(v))
    return st, int(v.value)
