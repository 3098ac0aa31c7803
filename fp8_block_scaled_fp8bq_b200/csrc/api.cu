// C ABI of libfp8bq: argument validation, status codes, device error word,
// TMA descriptor encoding.  Every entry point checks its arguments before it
// launches anything, and never throws.
#include <math.h>
#include <stdio.h>
#include <string.h>

#include <algorithm>
#include <mutex>

#include "device.cuh"
#include "internal.h"

namespace fp8bq {

namespace {

std::atomic<int> g_sms[kMaxDevices] = {};

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn g_encode = nullptr;
std::once_flag g_encode_once;

thread_local char g_last_cuda_error[256] = {0};
thread_local int g_last_cuda_code = 0;  // cudaError_t of this thread's last failing call, 0 once read

TensorMapCache g_maps;

TensorMapKey map_key(int rank, CUtensorMapDataType dtype, const void *base, const uint64_t *dims,
                     const uint64_t *strides, uint32_t box0, uint32_t box1, CUtensorMapSwizzle swizzle,
                     uint32_t box2 = 0) {
  TensorMapKey k;
  memset(&k, 0, sizeof(k));
  k.base = base;
  for (int i = 0; i < rank; ++i) k.dims[i] = dims[i];
  for (int i = 0; i + 1 < rank; ++i) k.strides[i] = strides[i];
  k.box[0] = box0;
  k.box[1] = box1;
  k.box[2] = box2;
  k.rank = rank;
  k.dtype = (int32_t)dtype;
  k.swizzle = (int32_t)swizzle;
  return k;
}

bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

int current_device() {
  int d = 0;
  if (cudaGetDevice(&d) != cudaSuccess) return 0;
  return d;
}

}  // namespace

int num_sms() {
  const int d = current_device();
  if (d < 0 || d >= kMaxDevices) {  // not cached: ask the runtime every time
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, d) != cudaSuccess || n <= 0) n = 148;
    return n;
  }
  int n = g_sms[d].load(std::memory_order_relaxed);
  if (n == 0) {
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, d) != cudaSuccess || n <= 0) n = 148;
    g_sms[d].store(n, std::memory_order_relaxed);  // every thread computes the same value
  }
  return n;
}

fp8bq_status cuda_fail(cudaError_t e, const char *what) {
  snprintf(g_last_cuda_error, sizeof(g_last_cuda_error), "%s: %s", what, cudaGetErrorString(e));
  g_last_cuda_code = (int)e;
  return FP8BQ_ERR_CUDA;
}

fp8bq_status check_launch(const char *what) {
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? FP8BQ_OK : cuda_fail(e, what);
}

bool make_tmap_2d(CUtensorMap *map, CUtensorMapDataType dtype, const void *base, uint64_t inner, uint64_t outer,
                  uint64_t row_stride_bytes, uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle swizzle) {
  std::call_once(g_encode_once, [] {
    void *fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<EncodeTiledFn>(fn);
  });
  if (g_encode == nullptr) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {row_stride_bytes};
  const TensorMapKey key = map_key(2, dtype, base, dims, strides, box_inner, box_outer, swizzle);
  if (g_maps.find(key, map)) return true;
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estride[2] = {1, 1};
  CUresult r = g_encode(map, dtype, 2, const_cast<void *>(base), dims, strides, box, estride,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return false;
  g_maps.insert(key, *map);
  return true;
}

bool make_tmap_3d(CUtensorMap *map, CUtensorMapDataType dtype, const void *base, uint64_t d0, uint64_t d1, uint64_t d2,
                  uint64_t stride1_bytes, uint64_t stride2_bytes, uint32_t box0, uint32_t box1,
                  CUtensorMapSwizzle swizzle, uint32_t box2) {
  cuuint64_t dims[3] = {d0, d1, d2};
  cuuint64_t strides[2] = {stride1_bytes, stride2_bytes};
  const TensorMapKey key = map_key(3, dtype, base, dims, strides, box0, box1, swizzle, box2);
  if (g_maps.find(key, map)) return true;
  CUtensorMap probe;
  if (!make_tmap_2d(&probe, dtype, base, d0, d1, stride1_bytes, box0, box1, swizzle)) return false;  // loads g_encode
  cuuint32_t box[3] = {box0, box1, box2};
  cuuint32_t estride[3] = {1, 1, 1};
  CUresult r = g_encode(map, dtype, 3, const_cast<void *>(base), dims, strides, box, estride,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return false;
  g_maps.insert(key, *map);
  return true;
}

fp8bq_status check_decode_args(const void *x, int64_t ldx, const uint8_t *qw, int64_t ldw, const float *sw,
                               const void *y, int64_t ldy, int64_t M, int64_t N, int64_t K, int mode, bool *work) {
  *work = false;
  if (M < 0 || N < 0 || K < 0 || (mode != FP8BQ_SCALE_FP32 && mode != FP8BQ_SCALE_POW2)) return FP8BQ_ERR_INVALID_ARG;
  if (M >= ((int64_t)1 << 31) || N >= ((int64_t)1 << 31) || K >= ((int64_t)1 << 31)) return FP8BQ_ERR_UNSUPPORTED;
  if (M == 0 || N == 0) return FP8BQ_OK;
  if (y == nullptr || ldy < N || !aligned(y, 16) || ldy % 8 != 0) return FP8BQ_ERR_INVALID_ARG;
  if (K != 0) {
    if (K % 128 != 0 || M > 256) return FP8BQ_ERR_UNSUPPORTED;
    if (!x || !qw || !sw || ldx < K || ldw < K) return FP8BQ_ERR_INVALID_ARG;
    if (!aligned(x, 2) || !aligned(qw, 16) || ldw % 16 != 0 || !aligned(sw, 4)) return FP8BQ_ERR_INVALID_ARG;
  }
  *work = true;
  return FP8BQ_OK;
}

}  // namespace fp8bq

using namespace fp8bq;

namespace {

bool bad_mode(int mode) { return mode != FP8BQ_SCALE_FP32 && mode != FP8BQ_SCALE_POW2; }

constexpr int64_t kMaxDim = (int64_t)1 << 31;

// The GEMM's inputs (M, N > 0): codes and scales of both operands.
fp8bq_status check_gemm_inputs(const uint8_t *qa, int64_t lda, const float *sa, int64_t ldsa, const uint8_t *qw,
                               int64_t ldw, const float *sw, int64_t M, int64_t K) {
  if (K == 0) return FP8BQ_OK;
  if (K % 128 != 0) return FP8BQ_ERR_UNSUPPORTED;
  if (!qa || !sa || !qw || !sw) return FP8BQ_ERR_INVALID_ARG;
  if (lda < K || ldw < K || ldsa < M) return FP8BQ_ERR_INVALID_ARG;
  if (!aligned(qa, 16) || !aligned(qw, 16) || lda % 16 != 0 || ldw % 16 != 0) return FP8BQ_ERR_INVALID_ARG;
  if (!aligned(sa, 16) || !aligned(sw, 4) || ldsa % 4 != 0) return FP8BQ_ERR_INVALID_ARG;
  return FP8BQ_OK;
}

fp8bq_status check_gemm_operands(const uint8_t *qa, int64_t lda, const float *sa, int64_t ldsa, const uint8_t *qw,
                                 int64_t ldw, const float *sw, const void *y, int64_t ldy, int64_t M, int64_t N,
                                 int64_t K, int mode) {
  if (M < 0 || N < 0 || K < 0 || bad_mode(mode)) return FP8BQ_ERR_INVALID_ARG;
  if (M >= kMaxDim || N >= kMaxDim || K >= kMaxDim) return FP8BQ_ERR_UNSUPPORTED;
  if (M == 0 || N == 0) return FP8BQ_OK;
  if (y == nullptr || ldy < N || !aligned(y, 16) || ldy % 8 != 0) return FP8BQ_ERR_INVALID_ARG;
  return check_gemm_inputs(qa, lda, sa, ldsa, qw, ldw, sw, M, K);
}

// The fused gate+up epilogue's operands: W_gu has 2I rows; the outputs are the
// H codes [M][ldqh], the H scales [I/128][ldsh] (the activation-scale layout the
// next GEMM reads) and the optional bf16 H [M][ldh].
fp8bq_status check_swiglu_operands(const uint8_t *qa, int64_t lda, const float *sa, int64_t ldsa, const uint8_t *qw,
                                   int64_t ldw, const float *sw, const uint8_t *qh, int64_t ldqh, const float *sh,
                                   int64_t ldsh, const void *h, int64_t ldh, int64_t M, int64_t I, int64_t K,
                                   int mode) {
  if (M < 0 || I < 0 || K < 0 || bad_mode(mode)) return FP8BQ_ERR_INVALID_ARG;
  if (M >= kMaxDim || 2 * I >= kMaxDim || K >= kMaxDim) return FP8BQ_ERR_UNSUPPORTED;
  if (M == 0 || I == 0) return FP8BQ_OK;
  if (I % 128 != 0) return FP8BQ_ERR_UNSUPPORTED;
  if (!qh || ldqh < I || ldqh % 16 != 0 || !aligned(qh, 16)) return FP8BQ_ERR_INVALID_ARG;
  if (!sh || ldsh < M || ldsh % 4 != 0 || !aligned(sh, 16)) return FP8BQ_ERR_INVALID_ARG;
  if (h != nullptr && (ldh < I || ldh % 8 != 0 || !aligned(h, 16))) return FP8BQ_ERR_INVALID_ARG;
  return check_gemm_inputs(qa, lda, sa, ldsa, qw, ldw, sw, M, K);
}

}  // namespace

extern "C" {

int fp8bq_version(void) { return 100; }

const char *fp8bq_status_string(fp8bq_status s) {
  switch (s) {
    case FP8BQ_OK: return "FP8BQ_OK";
    case FP8BQ_ERR_INVALID_ARG: return "FP8BQ_ERR_INVALID_ARG";
    case FP8BQ_ERR_UNSUPPORTED: return "FP8BQ_ERR_UNSUPPORTED";
    case FP8BQ_ERR_CUDA: return "FP8BQ_ERR_CUDA";
    case FP8BQ_ERR_WORKSPACE: return "FP8BQ_ERR_WORKSPACE";
    case FP8BQ_ERR_TIMEOUT: return "FP8BQ_ERR_TIMEOUT";
  }
  return "FP8BQ_ERR_UNKNOWN";
}

const char *fp8bq_last_cuda_error(void) { return g_last_cuda_error; }

fp8bq_status fp8bq_get_last_cuda_error(int *cuda_code) {
  const int c = g_last_cuda_code;
  g_last_cuda_code = 0;
  if (cuda_code) *cuda_code = c;
  return c != 0 ? FP8BQ_ERR_CUDA : FP8BQ_OK;
}

size_t fp8bq_recalibrate_workspace_size(int n) {
  (void)n;
  return 0;
}

size_t fp8bq_grouped_gemm_workspace_size(int E, int64_t max_rows, int64_t N, int64_t K) {
  (void)E;
  (void)max_rows;
  (void)N;
  (void)K;
  return 0;
}

fp8bq_status fp8bq_get_device_error(uint64_t *code) {
  unsigned long long v = 0, w = 0;
  cudaError_t e = cudaDeviceSynchronize();
  if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceSynchronize");
  cudaError_t (*takers[])(unsigned long long *) = {take_device_error_gemm, take_device_error_decode,
                                                    take_device_error_native, take_device_error_pair,
                                                    take_device_error_swiglu, take_device_error_wgrad,
                                                    take_device_error_prefill_attn, take_device_error_decode_wide};
  for (auto take : takers) {
    e = take(&w);
    if (e != cudaSuccess) return cuda_fail(e, "read device error word");
    if (v == 0) v = w;
  }
  if (code) *code = v;
  return v ? FP8BQ_ERR_TIMEOUT : FP8BQ_OK;
}

fp8bq_status fp8bq_e4m3_encode(const float *x, int64_t n, uint8_t *q, void *stream) {
  if (n < 0) return FP8BQ_ERR_INVALID_ARG;
  if (n == 0) return FP8BQ_OK;
  if (!x || !q || !aligned(x, 16) || !aligned(q, 4)) return FP8BQ_ERR_INVALID_ARG;
  return launch_encode(x, n, q, static_cast<cudaStream_t>(stream));
}

fp8bq_status fp8bq_quant_act(const void *x, int64_t M, int64_t K, int64_t ldx, uint8_t *q, int64_t ldq, float *sa,
                             int64_t ldsa, int mode, void *stream) {
  if (M < 0 || K < 0 || bad_mode(mode)) return FP8BQ_ERR_INVALID_ARG;
  if (M == 0 || K == 0) return FP8BQ_OK;
  if (!x || !q || !sa) return FP8BQ_ERR_INVALID_ARG;
  if (ldx < K || ldq < K || ldsa < M) return FP8BQ_ERR_INVALID_ARG;
  if (!aligned(x, 2) || !aligned(sa, 4)) return FP8BQ_ERR_INVALID_ARG;
  return launch_quant_act(x, M, K, ldx, q, ldq, sa, ldsa, mode, static_cast<cudaStream_t>(stream));
}

static fp8bq_status check_weight_desc(const fp8bq_weight_desc &d) {
  if (d.N < 0 || d.K < 0) return FP8BQ_ERR_INVALID_ARG;
  if (d.N == 0 || d.K == 0) return FP8BQ_OK;
  if (!d.w || !d.q || !d.s) return FP8BQ_ERR_INVALID_ARG;
  if (d.ldw < d.K || d.ldq < d.K) return FP8BQ_ERR_INVALID_ARG;
  if (!aligned(d.w, 2) || !aligned(d.s, 4)) return FP8BQ_ERR_INVALID_ARG;
  return FP8BQ_OK;
}

fp8bq_status fp8bq_quant_weight(const void *w, int64_t N, int64_t K, int64_t ldw, uint8_t *q, int64_t ldq, float *sw,
                                int mode, void *stream) {
  if (bad_mode(mode)) return FP8BQ_ERR_INVALID_ARG;
  fp8bq_weight_desc d;
  d.w = w;
  d.q = q;
  d.s = sw;
  d.N = N;
  d.K = K;
  d.ldw = ldw;
  d.ldq = ldq;
  fp8bq_status st = check_weight_desc(d);
  if (st != FP8BQ_OK || N == 0 || K == 0) return st;
  return launch_recalibrate(&d, 1, mode, static_cast<cudaStream_t>(stream));
}

fp8bq_status fp8bq_recalibrate(const fp8bq_weight_desc *descs, int n, int mode, void *stream) {
  if (n < 0 || bad_mode(mode)) return FP8BQ_ERR_INVALID_ARG;
  if (n == 0) return FP8BQ_OK;
  if (!descs) return FP8BQ_ERR_INVALID_ARG;
  for (int i = 0; i < n; ++i) {
    fp8bq_status st = check_weight_desc(descs[i]);
    if (st != FP8BQ_OK) return st;
  }
  return launch_recalibrate(descs, n, mode, static_cast<cudaStream_t>(stream));
}

fp8bq_status fp8bq_gemm_ex(const uint8_t *qa, int64_t lda, const float *sa, int64_t ldsa, const uint8_t *qw,
                           int64_t ldw, const float *sw, void *y, int64_t ldy, int64_t M, int64_t N, int64_t K,
                           int mode, int variant, void *stream) {
  if ((variant < FP8BQ_GEMM_AUTO || variant > FP8BQ_GEMM_PROMOTE_PAIR_N128) && variant != FP8BQ_GEMM_SELFTEST_TIMEOUT)
    return FP8BQ_ERR_INVALID_ARG;
  if (variant == FP8BQ_GEMM_NATIVE_POW2 && mode != FP8BQ_SCALE_POW2) return FP8BQ_ERR_INVALID_ARG;
  fp8bq_status st = check_gemm_operands(qa, lda, sa, ldsa, qw, ldw, sw, y, ldy, M, N, K, mode);
  if (st != FP8BQ_OK || M == 0 || N == 0) return st;
  return launch_gemm(qa, lda, sa, ldsa, qw, ldw, sw, y, ldy, M, N, K, mode, variant,
                     static_cast<cudaStream_t>(stream));
}

size_t fp8bq_gemm_decode_workspace_size(int64_t M, int64_t N, int64_t K) { return decode_workspace_size(M, N, K); }

fp8bq_status fp8bq_gemm_decode(const void *x, int64_t ldx, const uint8_t *qw, int64_t ldw, const float *sw, void *y,
                               int64_t ldy, int64_t M, int64_t N, int64_t K, int mode, void *ws, size_t ws_bytes,
                               void *stream) {
  bool work = false;
  const fp8bq_status st = check_decode_args(x, ldx, qw, ldw, sw, y, ldy, M, N, K, mode, &work);
  if (st != FP8BQ_OK || !work) return st;
  if (K == 0) {
    cudaError_t e = cudaMemset2DAsync(y, (size_t)ldy * 2, 0, (size_t)N * 2, (size_t)M, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? FP8BQ_OK : cuda_fail(e, "memset(y)");
  }
  return launch_gemm_decode(x, ldx, qw, ldw, sw, y, ldy, M, N, K, mode, ws, ws_bytes,
                            static_cast<cudaStream_t>(stream));
}

fp8bq_status fp8bq_grouped_gemm(const uint8_t *qa, int64_t lda, const float *sa, int64_t ldsa, const uint8_t *qw,
                                const float *sw, const int32_t *offsets, int E, int64_t total_rows, int64_t N,
                                int64_t K, void *y, int64_t ldy, int mode, void *stream) {
  if (E < 1 || E > kMaxExperts || total_rows < 0) return E > kMaxExperts ? FP8BQ_ERR_UNSUPPORTED : FP8BQ_ERR_INVALID_ARG;
  if (!offsets || !aligned(offsets, 4)) return FP8BQ_ERR_INVALID_ARG;
  if (N % 8 != 0) return FP8BQ_ERR_UNSUPPORTED;
  if ((int64_t)E * N >= kMaxDim) return FP8BQ_ERR_UNSUPPORTED;
  // the expert weights are dense [E][N][K]: lda-like checks apply with ldw = K
  fp8bq_status st = check_gemm_operands(qa, lda, sa, ldsa, qw, K, sw, y, ldy, total_rows, N, K, mode);
  if (st != FP8BQ_OK || total_rows == 0 || N == 0) return st;
  return launch_grouped_gemm(qa, lda, sa, ldsa, qw, sw, offsets, E, total_rows, N, K, y, ldy,
                             static_cast<cudaStream_t>(stream));
}

fp8bq_status fp8bq_gemm_swiglu_quant(const uint8_t *qa, int64_t lda, const float *sa, int64_t ldsa,
                                     const uint8_t *qw, int64_t ldw, const float *sw, uint8_t *qh, int64_t ldqh,
                                     float *sh, int64_t ldsh, void *h, int64_t ldh, int64_t M, int64_t I, int64_t K,
                                     int mode, void *stream) {
  fp8bq_status st = check_swiglu_operands(qa, lda, sa, ldsa, qw, ldw, sw, qh, ldqh, sh, ldsh, h, ldh, M, I, K, mode);
  if (st != FP8BQ_OK || M == 0 || I == 0) return st;
  return launch_gemm_swiglu(qa, lda, sa, ldsa, qw, ldw, sw, qh, ldqh, sh, ldsh, h, ldh, M, I, K, mode,
                            static_cast<cudaStream_t>(stream));
}

fp8bq_status fp8bq_grouped_gemm_swiglu_quant(const uint8_t *qa, int64_t lda, const float *sa, int64_t ldsa,
                                             const uint8_t *qw, const float *sw, const int32_t *offsets, int E,
                                             int64_t total_rows, int64_t I, int64_t K, uint8_t *qh, int64_t ldqh,
                                             float *sh, int64_t ldsh, void *h, int64_t ldh, int mode, void *stream) {
  if (E < 1 || E > kMaxExperts || total_rows < 0) return E > kMaxExperts ? FP8BQ_ERR_UNSUPPORTED : FP8BQ_ERR_INVALID_ARG;
  if (!offsets || !aligned(offsets, 4)) return FP8BQ_ERR_INVALID_ARG;
  if ((int64_t)E * 2 * I >= kMaxDim) return FP8BQ_ERR_UNSUPPORTED;
  fp8bq_status st =
      check_swiglu_operands(qa, lda, sa, ldsa, qw, K, sw, qh, ldqh, sh, ldsh, h, ldh, total_rows, I, K, mode);
  if (st != FP8BQ_OK || total_rows == 0 || I == 0) return st;
  return launch_grouped_gemm_swiglu(qa, lda, sa, ldsa, qw, sw, offsets, E, total_rows, I, K, qh, ldqh, sh, ldsh, h,
                                    ldh, mode, static_cast<cudaStream_t>(stream));
}

fp8bq_status fp8bq_quant_act_t(const void *x, int64_t M, int64_t K, int64_t ldx, uint8_t *qt, int64_t ldqt, float *st,
                               int64_t ldst, int mode, void *stream) {
  if (M < 0 || K < 0 || bad_mode(mode)) return FP8BQ_ERR_INVALID_ARG;
  if (M >= kMaxDim || K >= kMaxDim) return FP8BQ_ERR_UNSUPPORTED;
  if (M == 0 || K == 0) return FP8BQ_OK;
  if (K % 8 != 0) return FP8BQ_ERR_UNSUPPORTED;
  if (!x || !qt || !st) return FP8BQ_ERR_INVALID_ARG;
  if (ldx < K || ldx % 8 != 0 || !aligned(x, 16)) return FP8BQ_ERR_INVALID_ARG;
  if (ldqt < M || ldqt % 16 != 0 || !aligned(qt, 16)) return FP8BQ_ERR_INVALID_ARG;
  if (ldst < K || ldst % 4 != 0 || !aligned(st, 16)) return FP8BQ_ERR_INVALID_ARG;
  return launch_quant_act_t(x, M, K, ldx, qt, ldqt, st, ldst, mode, static_cast<cudaStream_t>(stream));
}

fp8bq_status fp8bq_transpose_weight(const uint8_t *q, int64_t N, int64_t K, int64_t ldq, const float *sw, uint8_t *qt,
                                    int64_t ldqt, float *swt, void *stream) {
  if (N < 0 || K < 0) return FP8BQ_ERR_INVALID_ARG;
  if (N >= kMaxDim || K >= kMaxDim) return FP8BQ_ERR_UNSUPPORTED;
  if (N == 0 || K == 0) return FP8BQ_OK;
  if (N % 16 != 0 || K % 16 != 0) return FP8BQ_ERR_UNSUPPORTED;
  if (!q || !sw || !qt || !swt) return FP8BQ_ERR_INVALID_ARG;
  if (ldq < K || ldq % 16 != 0 || !aligned(q, 16) || ldqt < N || ldqt % 16 != 0 || !aligned(qt, 16))
    return FP8BQ_ERR_INVALID_ARG;
  if (!aligned(sw, 4) || !aligned(swt, 4)) return FP8BQ_ERR_INVALID_ARG;
  return launch_transpose_weight(q, N, K, ldq, sw, qt, ldqt, swt, static_cast<cudaStream_t>(stream));
}

fp8bq_status fp8bq_gemm_wgrad(const uint8_t *qa, int64_t lda, const float *sa, int64_t ldsa, const uint8_t *qb,
                              int64_t ldb, const float *sb, int64_t ldsb, void *y, int64_t ldy, int64_t N, int64_t K,
                              int64_t M, int mode, void *stream) {
  if (N < 0 || K < 0 || M < 0 || bad_mode(mode)) return FP8BQ_ERR_INVALID_ARG;
  if (N >= kMaxDim || K >= kMaxDim || M >= kMaxDim) return FP8BQ_ERR_UNSUPPORTED;
  if (N == 0 || K == 0) return FP8BQ_OK;
  if (y == nullptr || ldy < K || !aligned(y, 16) || ldy % 8 != 0) return FP8BQ_ERR_INVALID_ARG;
  if (M == 0) return launch_gemm_wgrad(qa, lda, sa, ldsa, qb, ldb, sb, ldsb, y, ldy, N, K, M, static_cast<cudaStream_t>(stream));
  if (M % 128 != 0 || K % 4 != 0) return FP8BQ_ERR_UNSUPPORTED;
  if (!qa || !sa || !qb || !sb) return FP8BQ_ERR_INVALID_ARG;
  if (lda < M || ldb < M || lda % 16 != 0 || ldb % 16 != 0 || !aligned(qa, 16) || !aligned(qb, 16))
    return FP8BQ_ERR_INVALID_ARG;
  if (ldsa < N || ldsa % 4 != 0 || !aligned(sa, 16)) return FP8BQ_ERR_INVALID_ARG;
  if (ldsb < K || ldsb % 4 != 0 || !aligned(sb, 16)) return FP8BQ_ERR_INVALID_ARG;
  // power-of-two scales: the native block-scaled MMA applies both operands'
  // scales (exact, no promotion); FP32 scales: FP32 promotion per token block
  if (mode == FP8BQ_SCALE_POW2)
    return launch_gemm_native_wgrad(qa, lda, sa, ldsa, qb, ldb, sb, ldsb, y, ldy, N, K, M,
                                    static_cast<cudaStream_t>(stream));
  return launch_gemm_wgrad(qa, lda, sa, ldsa, qb, ldb, sb, ldsb, y, ldy, N, K, M, static_cast<cudaStream_t>(stream));
}

size_t fp8bq_decode_attention_workspace_size(int64_t B, int64_t Hq, int64_t Hkv, int64_t S) {
  return decode_attention_workspace_size(B, Hq, Hkv, S);
}

fp8bq_status fp8bq_decode_attention(const void *q, const uint8_t *kq, const float *ks, const uint8_t *vq,
                                    const float *vs, const int32_t *seq_lens, int64_t B, int64_t Hq, int64_t Hkv,
                                    int64_t S, float softmax_scale, void *o, void *ws, size_t ws_bytes,
                                    void *stream) {
  if (B < 0 || Hq < 0 || Hkv < 0 || S < 0) return FP8BQ_ERR_INVALID_ARG;
  if (B >= kMaxDim || Hq >= 65536 || Hkv >= 65536 || S >= kMaxDim) return FP8BQ_ERR_UNSUPPORTED;
  if (B == 0 || Hq == 0) return FP8BQ_OK;
  if (Hkv == 0 || Hq % Hkv != 0) return FP8BQ_ERR_INVALID_ARG;
  const int64_t G = Hq / Hkv;
  if (G != 1 && G != 2 && G != 4 && G != 8) return FP8BQ_ERR_UNSUPPORTED;
  if (B * Hq > 0x7fffffffLL) return FP8BQ_ERR_UNSUPPORTED;
  if (!q || !o || !aligned(q, 2) || !aligned(o, 8)) return FP8BQ_ERR_INVALID_ARG;
  if (S > 0) {
    if (!kq || !ks || !vq || !vs || !seq_lens || !ws) return FP8BQ_ERR_INVALID_ARG;
    if (!aligned(kq, 16) || !aligned(vq, 16) || !aligned(ks, 4) || !aligned(vs, 4) || !aligned(seq_lens, 4) ||
        !aligned(ws, 16))
      return FP8BQ_ERR_INVALID_ARG;
  }
  return launch_decode_attention(q, kq, ks, vq, vs, seq_lens, B, Hq, Hkv, S, softmax_scale, o, ws, ws_bytes,
                                 static_cast<cudaStream_t>(stream));
}

fp8bq_status fp8bq_prefill_attention(const uint8_t *qq, const float *qs, const uint8_t *kq, const float *ks,
                                     const uint8_t *vq, const float *vs, const int32_t *seq_lens, int64_t B, int64_t S,
                                     int64_t Hq, int64_t Hkv, float softmax_scale, void *o, void *stream) {
  if (B < 0 || S < 0 || Hq < 0 || Hkv < 0) return FP8BQ_ERR_INVALID_ARG;
  if (!(softmax_scale > 0.f) || !(softmax_scale < INFINITY)) return FP8BQ_ERR_INVALID_ARG;
  if (B == 0 || S == 0 || Hq == 0) return FP8BQ_OK;
  if (Hkv == 0 || Hq % Hkv != 0) return FP8BQ_ERR_INVALID_ARG;
  if (Hq >= 65536 || B * S >= kMaxDim || B * Hq * ((S + 127) / 128) >= kMaxDim) return FP8BQ_ERR_UNSUPPORTED;
  if (!qq || !qs || !kq || !ks || !vq || !vs || !seq_lens || !o) return FP8BQ_ERR_INVALID_ARG;
  if (!aligned(qq, 16) || !aligned(kq, 16) || !aligned(vq, 16) || !aligned(o, 16)) return FP8BQ_ERR_INVALID_ARG;
  if (!aligned(qs, 4) || !aligned(ks, 4) || !aligned(vs, 4) || !aligned(seq_lens, 4)) return FP8BQ_ERR_INVALID_ARG;
  return launch_prefill_attention(qq, qs, kq, ks, vq, vs, seq_lens, B, S, Hq, Hkv, softmax_scale, o,
                                  static_cast<cudaStream_t>(stream));
}

fp8bq_status fp8bq_kv_cache_append(const void *k_new, const void *v_new, const int32_t *positions, uint8_t *kq,
                                   float *ks, uint8_t *vq, float *vs, int64_t B, int64_t Hkv, int64_t S, int mode,
                                   void *stream) {
  if (B < 0 || Hkv < 0 || S < 0 || bad_mode(mode)) return FP8BQ_ERR_INVALID_ARG;
  if (2 * B * Hkv >= kMaxDim || S >= kMaxDim) return FP8BQ_ERR_UNSUPPORTED;
  if (B == 0 || Hkv == 0 || S == 0) return FP8BQ_OK;
  if (!k_new || !v_new || !positions || !kq || !ks || !vq || !vs) return FP8BQ_ERR_INVALID_ARG;
  if (!aligned(k_new, 8) || !aligned(v_new, 8) || !aligned(positions, 4) || !aligned(kq, 4) || !aligned(vq, 4) ||
      !aligned(ks, 4) || !aligned(vs, 4))
    return FP8BQ_ERR_INVALID_ARG;
  return launch_kv_append(k_new, v_new, positions, kq, ks, vq, vs, B, Hkv, S, mode, static_cast<cudaStream_t>(stream));
}

fp8bq_status fp8bq_adamw_recalibrate(const fp8bq_adamw_desc *descs, int n, const fp8bq_adamw_config *cfg, int mode,
                                     void *stream) {
  if (n < 0 || bad_mode(mode) || cfg == nullptr) return FP8BQ_ERR_INVALID_ARG;
  if (!(cfg->beta1 >= 0.f && cfg->beta1 < 1.f && cfg->beta2 >= 0.f && cfg->beta2 < 1.f && cfg->eps >= 0.f) ||
      cfg->step < 1)
    return FP8BQ_ERR_INVALID_ARG;
  if (n == 0) return FP8BQ_OK;
  if (!descs) return FP8BQ_ERR_INVALID_ARG;
  for (int i = 0; i < n; ++i) {
    const fp8bq_adamw_desc &d = descs[i];
    if (d.N < 0 || d.K < 0) return FP8BQ_ERR_INVALID_ARG;
    if (d.N >= kMaxDim || d.K >= kMaxDim) return FP8BQ_ERR_UNSUPPORTED;
    if (d.N == 0 || d.K == 0) continue;
    if (d.K % 4 != 0) return FP8BQ_ERR_UNSUPPORTED;
    if (!d.param || !d.grad || !d.exp_avg || !d.exp_avg_sq || !d.q || !d.s) return FP8BQ_ERR_INVALID_ARG;
    if (!aligned(d.param, 16) || !aligned(d.grad, 16) || !aligned(d.exp_avg, 16) || !aligned(d.exp_avg_sq, 16) ||
        !aligned(d.w, 8) || !aligned(d.q, 4) || !aligned(d.s, 4))
      return FP8BQ_ERR_INVALID_ARG;
  }
  return launch_adamw_recalibrate(descs, n, cfg, mode, static_cast<cudaStream_t>(stream));
}

fp8bq_status fp8bq_gemm(const uint8_t *qa, int64_t lda, const float *sa, int64_t ldsa, const uint8_t *qw, int64_t ldw,
                        const float *sw, void *y, int64_t ldy, int64_t M, int64_t N, int64_t K, int mode,
                        void *stream) {
  return fp8bq_gemm_ex(qa, lda, sa, ldsa, qw, ldw, sw, y, ldy, M, N, K, mode, FP8BQ_GEMM_AUTO, stream);
}

}  // extern "C"
