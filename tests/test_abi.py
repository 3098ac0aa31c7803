"""The C-ABI library builds, loads without a GPU, exports every entry point that
include/fp8bq.h declares, and rejects bad arguments before touching the GPU."""
import ctypes
import os
import re
import subprocess

import pytest

import fp8_block_scaled_fp8bq_b200 as fq
from fp8_block_scaled_fp8bq_b200 import build as fbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "fp8bq.h")

INVALID, UNSUPPORTED = 1, 2


def declared_functions():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"FP8BQ_API\s+[\w\s\*]+?\b(fp8bq_\w+)\s*\(", text)))


@pytest.fixture(scope="module")
def L():
    fbuild.build()
    return fq.lib()


def test_header_declares_the_boundary():
    names = declared_functions()
    # the hot path's entry points and their size queries and diagnostics
    for n in ("fp8bq_quant_act", "fp8bq_quant_weight", "fp8bq_recalibrate", "fp8bq_recalibrate_workspace_size",
              "fp8bq_gemm", "fp8bq_gemm_decode", "fp8bq_gemm_decode_workspace_size", "fp8bq_grouped_gemm",
              "fp8bq_grouped_gemm_workspace_size", "fp8bq_status_string", "fp8bq_get_last_cuda_error"):
        assert n in names


def test_workspace_queries_and_last_error(L):
    # recalibration and the grouped GEMM keep their tables in launch parameters
    # and shared memory: no workspace
    assert L.fp8bq_recalibrate_workspace_size(128) == 0
    assert L.fp8bq_grouped_gemm_workspace_size(128, 32768, 1536, 2048) == 0
    code = ctypes.c_int(-1)
    assert L.fp8bq_get_last_cuda_error(ctypes.byref(code)) in (0, 3)
    # reading clears it
    assert L.fp8bq_get_last_cuda_error(ctypes.byref(code)) == 0 and code.value == 0
    assert L.fp8bq_get_last_cuda_error(None) == 0


def test_every_declared_symbol_is_exported(L):
    out = subprocess.run(["nm", "-D", "--defined-only", fq.LIB_PATH], capture_output=True, text=True,
                         check=True).stdout
    exported = set(re.findall(r" T (fp8bq_\w+)", out))
    missing = [n for n in declared_functions() if n not in exported]
    assert not missing, missing
    # and nothing else from the library's internals leaks out
    extra = [n for n in exported if n not in declared_functions()]
    assert not extra, extra
    assert set(fq.SIGNATURES) == set(declared_functions())


def test_header_compiles_as_c():
    src = '#include "fp8bq.h"\nint main(void){return FP8BQ_OK;}\n'
    r = subprocess.run(["gcc", "-x", "c", "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"),
                        "-fsyntax-only", "-"], input=src, text=True, capture_output=True)
    assert r.returncode == 0, r.stderr


def test_status_strings(L):
    assert L.fp8bq_status_string(0) == b"FP8BQ_OK"
    assert L.fp8bq_status_string(5) == b"FP8BQ_ERR_TIMEOUT"
    assert L.fp8bq_version() >= 100


FAKE = ctypes.c_void_p(0x10000)      # a 64 KiB-aligned address: never dereferenced


def test_quant_act_validation(L):
    f = L.fp8bq_quant_act
    assert f(FAKE, -1, 128, 128, FAKE, 128, FAKE, 4, 0, None) == INVALID
    assert f(FAKE, 4, 128, 64, FAKE, 128, FAKE, 4, 0, None) == INVALID     # ldx < K
    assert f(FAKE, 4, 128, 128, FAKE, 128, FAKE, 3, 0, None) == INVALID    # ldsa < M
    assert f(None, 4, 128, 128, FAKE, 128, FAKE, 4, 0, None) == INVALID
    assert f(FAKE, 4, 128, 128, FAKE, 128, FAKE, 4, 7, None) == INVALID    # bad mode
    assert f(None, 0, 128, 128, None, 128, None, 4, 0, None) == 0          # empty: no-op


def test_gemm_validation(L):
    g = L.fp8bq_gemm

    def call(M=256, N=256, K=256, lda=256, ldw=256, ldy=256, ldsa=256, qa=FAKE, y=FAKE, mode=0):
        return g(qa, lda, FAKE, ldsa, FAKE, ldw, FAKE, y, ldy, M, N, K, mode, None)
    assert call(K=200, lda=256, ldw=256) == UNSUPPORTED                   # K % 128
    assert call(lda=128) == INVALID                                       # lda < K
    assert call(ldy=255) == INVALID                                       # ldy < N
    assert call(ldy=260) == INVALID                                       # ldy % 8
    assert call(ldsa=255) == INVALID                                      # ldsa < M
    assert call(ldsa=258) == INVALID                                      # ldsa % 4
    assert call(qa=ctypes.c_void_p(0x10008)) == INVALID                   # 16-byte alignment
    assert call(M=-1) == INVALID
    assert call(M=0) == 0 and call(N=0) == 0                              # empty: no-op
    assert call(mode=2) == INVALID
    assert L.fp8bq_gemm_ex(FAKE, 256, FAKE, 256, FAKE, 256, FAKE, FAKE, 256, 256, 256, 256, 0, 2, None) == INVALID


def test_recalibrate_validation(L):
    arr = (fq.WeightDesc * 2)()
    arr[0] = fq.WeightDesc(0x10000, 0x20000, 0x30000, 128, 128, 128, 128)
    arr[1] = fq.WeightDesc(0x10000, 0x20000, 0x30000, 128, 128, 64, 128)   # ldw < K
    assert L.fp8bq_recalibrate(arr, 2, 1, None) == INVALID
    assert L.fp8bq_recalibrate(arr, -1, 1, None) == INVALID
    assert L.fp8bq_recalibrate(arr, 0, 1, None) == 0


def test_grouped_validation(L):
    f = L.fp8bq_grouped_gemm

    def call(E=4, rows=256, N=256, K=256, lda=256, ldsa=256, ldy=256, off=FAKE):
        return f(FAKE, lda, FAKE, ldsa, FAKE, FAKE, off, E, rows, N, K, FAKE, ldy, 0, None)
    assert call(E=0) == INVALID
    assert call(E=1025) == UNSUPPORTED
    assert call(off=None) == INVALID
    assert call(N=260, ldy=264) == UNSUPPORTED                            # N % 8
    assert call(K=200, lda=208) == UNSUPPORTED                            # K % 128
    assert call(rows=0) == 0


def test_swiglu_validation(L):
    f = L.fp8bq_gemm_swiglu_quant

    def call(M=256, I=256, K=256, lda=256, ldsa=256, ldw=256, ldqh=256, ldsh=256, h=None, ldh=0, mode=0, qh=FAKE,
             sh=FAKE):
        return f(FAKE, lda, FAKE, ldsa, FAKE, ldw, FAKE, qh, ldqh, sh, ldsh, h, ldh, M, I, K, mode, None)
    assert call(I=192, ldqh=192) == UNSUPPORTED                          # I % 128
    assert call(K=200, lda=208, ldw=208) == UNSUPPORTED                  # K % 128
    assert call(ldqh=128) == INVALID                                     # ldqh < I
    assert call(ldqh=264) == INVALID                                     # ldqh % 16
    assert call(qh=None) == INVALID
    assert call(sh=None) == INVALID
    assert call(ldsh=255) == INVALID                                     # ldsh < M
    assert call(ldsh=258) == INVALID                                     # ldsh % 4
    assert call(h=FAKE, ldh=128) == INVALID                              # ldh < I
    assert call(h=FAKE, ldh=260) == INVALID                              # ldh % 8
    assert call(h=ctypes.c_void_p(0x10008), ldh=256) == INVALID          # h alignment
    assert call(lda=128) == INVALID                                      # lda < K
    assert call(M=-1) == INVALID
    assert call(mode=3) == INVALID
    assert call(M=0) == 0 and call(I=0) == 0

    g = L.fp8bq_grouped_gemm_swiglu_quant

    def gcall(E=4, rows=256, I=256, K=256, off=FAKE, ldqh=256):
        return g(FAKE, 256, FAKE, 256, FAKE, FAKE, off, E, rows, I, K, FAKE, ldqh, FAKE, 256, None, 0, 0, None)
    assert gcall(E=0) == INVALID
    assert gcall(E=1025) == UNSUPPORTED
    assert gcall(off=None) == INVALID
    assert gcall(I=192, ldqh=192) == UNSUPPORTED
    assert gcall(ldqh=100) == INVALID
    assert gcall(rows=0) == 0


def test_decode_attention_validation(L):
    f = L.fp8bq_decode_attention

    def call(B=2, Hq=8, Hkv=2, S=64, q=FAKE, kq=FAKE, vq=FAKE, ws=FAKE, o=FAKE):
        return f(q, kq, FAKE, vq, FAKE, FAKE, B, Hq, Hkv, S, 0.1, o, ws, 1 << 20, None)
    assert call(Hq=6, Hkv=4) == INVALID                                  # Hq % Hkv
    assert call(Hq=6, Hkv=2) == UNSUPPORTED                              # 3 query heads per key/value head
    assert call(Hq=32, Hkv=2) == UNSUPPORTED                             # 16 per key/value head
    assert call(kq=ctypes.c_void_p(0x10004)) == INVALID                  # kq 16-byte alignment
    assert call(vq=ctypes.c_void_p(0x10004)) == INVALID                  # vq 16-byte alignment
    assert call(ws=ctypes.c_void_p(0x10008)) == INVALID
    assert call(o=ctypes.c_void_p(0x10004)) == INVALID
    assert call(vq=None) == INVALID
    assert call(B=-1) == INVALID
    assert call(B=0) == 0 and call(Hq=0) == 0


def test_decode_gemm_validation(L):
    f = L.fp8bq_gemm_decode

    def call(M=16, N=256, K=256, ldx=256, ldw=256, ldy=256, mode=0, x=FAKE, qw=FAKE, y=FAKE):
        return f(x, ldx, qw, ldw, FAKE, y, ldy, M, N, K, mode, FAKE, 1 << 20, None)
    assert call(M=-1) == INVALID
    assert call(mode=3) == INVALID
    assert call(M=0) == 0 and call(N=0) == 0
    assert call(y=ctypes.c_void_p(0x10008)) == INVALID                 # y 16-byte alignment
    assert call(ldy=200) == INVALID                                    # ldy < N
    assert call(K=200, ldx=200, ldw=208) == UNSUPPORTED                # K % 128
    assert call(M=257) == UNSUPPORTED                                  # beyond the decode sizes
    assert call(x=None) == INVALID
    assert call(ldx=128) == INVALID                                    # ldx < K
    assert call(qw=ctypes.c_void_p(0x10004)) == INVALID
    g = L.fp8bq_gemm_decode_noalloc
    assert g(FAKE, 256, FAKE, 256, FAKE, FAKE, 256, -1, 256, 256, 0, None) == INVALID
    assert g(FAKE, 256, FAKE, 256, FAKE, FAKE, 256, 0, 256, 256, 0, None) == 0


def test_backward_validation(L):
    qt = L.fp8bq_quant_act_t

    def call_qt(M=256, K=256, ldx=256, ldqt=256, ldst=256, st=FAKE):
        return qt(FAKE, M, K, ldx, FAKE, ldqt, st, ldst, 0, None)
    assert call_qt(K=260, ldx=264, ldst=264) == UNSUPPORTED              # K % 8
    assert call_qt(ldqt=264) == INVALID                                 # ldqt % 16
    assert call_qt(ldx=128) == INVALID                                  # ldx < K
    assert call_qt(st=ctypes.c_void_p(0x10004)) == INVALID              # st 16-byte alignment
    assert call_qt(M=0) == 0 and call_qt(M=-1) == INVALID
    tw = L.fp8bq_transpose_weight

    def call_tw(N=256, K=256, ldq=256, ldqt=256):
        return tw(FAKE, N, K, ldq, FAKE, FAKE, ldqt, FAKE, None)
    assert call_tw(N=200) == UNSUPPORTED                                # N % 16
    assert call_tw(K=200, ldq=208) == UNSUPPORTED                       # K % 16
    assert call_tw(ldq=264) == INVALID and call_tw(ldqt=128) == INVALID
    assert call_tw(N=0) == 0
    wg = L.fp8bq_gemm_wgrad

    def call_wg(N=256, K=256, M=256, lda=256, ldb=256, ldsa=256, ldsb=256, ldy=256, y=FAKE):
        return wg(FAKE, lda, FAKE, ldsa, FAKE, ldb, FAKE, ldsb, y, ldy, N, K, M, 0, None)
    assert call_wg(M=200, lda=208, ldb=208) == UNSUPPORTED              # M % 128
    assert call_wg(ldy=260) == INVALID                                  # ldy % 8
    assert call_wg(lda=128) == INVALID                                  # lda < M
    assert call_wg(ldsb=200) == INVALID                                 # ldsb < K
    assert call_wg(y=None) == INVALID
    assert call_wg(N=0) == 0


def test_kv_append_and_adamw_validation(L):
    kv = L.fp8bq_kv_cache_append

    def call_kv(B=2, Hkv=2, S=16, mode=0, k=FAKE):
        return kv(k, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, B, Hkv, S, mode, None)
    assert call_kv(mode=5) == INVALID
    assert call_kv(k=ctypes.c_void_p(0x10004)) == INVALID              # k_new 8-byte alignment
    assert call_kv(B=-1) == INVALID
    assert call_kv(B=0) == 0 and call_kv(S=0) == 0
    ad = L.fp8bq_adamw_recalibrate

    def desc(K=256, grad=FAKE):
        return fq.AdamWDesc(FAKE, grad, FAKE, FAKE, None, FAKE, FAKE, 128, K)

    def cfg(beta1=0.9, step=1):
        return fq.AdamWConfig(1e-3, beta1, 0.999, 1e-8, 0.0, step)
    one = (fq.AdamWDesc * 1)(desc())
    assert ad(one, 1, ctypes.byref(cfg(beta1=1.0)), 0, None) == INVALID
    assert ad(one, 1, ctypes.byref(cfg(step=0)), 0, None) == INVALID
    assert ad(one, 1, None, 0, None) == INVALID
    assert ad((fq.AdamWDesc * 1)(desc(K=258)), 1, ctypes.byref(cfg()), 0, None) == UNSUPPORTED   # K % 4
    assert ad((fq.AdamWDesc * 1)(desc(grad=None)), 1, ctypes.byref(cfg()), 0, None) == INVALID
    assert ad(one, 0, ctypes.byref(cfg()), 0, None) == 0


def test_interleave_gate_up_layout():
    """Host-side layout helper of the fused gate+up call: 128-row blocks
    alternate gate block j, up block j (values exact in bf16)."""
    import torch
    import fp8_block_scaled_fp8bq_b200 as fq
    I, K = 256, 128
    g = torch.arange(I, dtype=torch.float32)[:, None].expand(I, K).to(torch.bfloat16)
    u = (-1 - torch.arange(I, dtype=torch.float32))[:, None].expand(I, K).to(torch.bfloat16)
    col = fq.interleave_gate_up(g, u)[:, 0].float()
    r = torch.arange(128, dtype=torch.float32)
    assert torch.equal(col[0:128], r) and torch.equal(col[128:256], -1 - r)
    assert torch.equal(col[256:384], 128 + r) and torch.equal(col[384:512], -129 - r)
    e = fq.interleave_gate_up(g.reshape(1, I, K).expand(3, I, K), u.reshape(1, I, K).expand(3, I, K))
    assert e.shape == (3, 2 * I, K) and torch.equal(e[2, :, 0].float(), col)


def test_prefill_attention_validation(L):
    f = L.fp8bq_prefill_attention
    P = FAKE
    assert f(P, P, P, P, P, P, P, 1, 128, 8, 3, 0.1, P, None) == INVALID           # Hq % Hkv
    assert f(P, P, P, P, P, P, P, 1, 128, 8, 2, 0.0, P, None) == INVALID           # scale <= 0
    assert f(P, P, P, P, P, P, P, 1, 128, 8, 2, float("inf"), P, None) == INVALID
    assert f(ctypes.c_void_p(0x10004), P, P, P, P, P, P, 1, 128, 8, 2, 0.1, P, None) == INVALID  # alignment
    assert f(P, P, P, P, P, P, None, 1, 128, 8, 2, 0.1, P, None) == INVALID        # no lengths
    assert f(None, None, None, None, None, None, None, 0, 128, 8, 2, 0.1, None, None) == 0   # empty: no-op
