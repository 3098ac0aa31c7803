// Decode-shaped block-scaled GEMM (placeholder until the kernel lands).
#include "device.cuh"
#include "internal.h"

extern "C" {

size_t fp8bq_gemm_decode_workspace_size(int64_t M, int64_t N, int64_t K) {
  (void)M;
  (void)N;
  (void)K;
  return 0;
}

fp8bq_status fp8bq_gemm_decode(const void *x, int64_t ldx, const uint8_t *qw, int64_t ldw, const float *sw, void *y,
                               int64_t ldy, int64_t M, int64_t N, int64_t K, int mode, void *ws, size_t ws_bytes,
                               void *stream) {
  (void)x; (void)ldx; (void)qw; (void)ldw; (void)sw; (void)y; (void)ldy; (void)M; (void)N; (void)K;
  (void)mode; (void)ws; (void)ws_bytes; (void)stream;
  return FP8BQ_ERR_UNSUPPORTED;
}

fp8bq_status fp8bq_grouped_gemm(const uint8_t *qa, int64_t lda, const float *sa, int64_t ldsa, const uint8_t *qw,
                                const float *sw, const int32_t *offsets, int E, int64_t total_rows, int64_t N,
                                int64_t K, void *y, int64_t ldy, int mode, void *stream) {
  (void)qa; (void)lda; (void)sa; (void)ldsa; (void)qw; (void)sw; (void)offsets; (void)E; (void)total_rows;
  (void)N; (void)K; (void)y; (void)ldy; (void)mode; (void)stream;
  return FP8BQ_ERR_UNSUPPORTED;
}

}  // extern "C"
