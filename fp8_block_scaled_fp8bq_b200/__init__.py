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
import os

import torch

SCALE_FP32 = 0
SCALE_POW2 = 1

GEMM_AUTO = 0
GEMM_PROMOTE = 1
GEMM_NATIVE_POW2 = 2
GEMM_PROMOTE_PAIR = 3
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


# name -> (restype, argtypes); the full list of the C ABI's entry points.
P, I64, I32, SZ = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_size_t
SIGNATURES = {
    "fp8bq_version": (ctypes.c_int, []),
    "fp8bq_status_string": (ctypes.c_char_p, [I32]),
    "fp8bq_last_cuda_error": (ctypes.c_char_p, []),
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
    """Small-M linear with on-the-fly 1x128 activation quantization."""
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


def device_error():
    """(status, raw word) of the device error word; reading clears it (synchronizes)."""
    v = ctypes.c_uint64(0)
    st = lib().fp8bq_get_device_error(ctypes.byref(v))
    return st, int(v.value)
