// Host-side declarations shared by the library's translation units.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/fp8bq.h"

namespace fp8bq {

// Largest expert count of fp8bq_grouped_gemm (the device scheduler keeps the
// offsets and the tile prefix of all experts in shared memory).
constexpr int kMaxExperts = 1024;

// Number of SMs of the current device (cached per device).
int num_sms();

// Record the failing CUDA call for diagnostics and map it to FP8BQ_ERR_CUDA.
fp8bq_status cuda_fail(cudaError_t e, const char *what);

// Check the last launch.
fp8bq_status check_launch(const char *what);

// cuTensorMapEncodeTiled through the runtime's driver entry point (no -lcuda).
// Returns false if the driver rejects the map.
bool make_tmap_2d(CUtensorMap *map, CUtensorMapDataType dtype, const void *base, uint64_t inner, uint64_t outer,
                  uint64_t row_stride_bytes, uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle swizzle);

// 3-D variant: dims {d0 (innermost), d1, d2}, byte strides of dims 1 and 2, box {box0, box1, 1}.
bool make_tmap_3d(CUtensorMap *map, CUtensorMapDataType dtype, const void *base, uint64_t d0, uint64_t d1, uint64_t d2,
                  uint64_t stride1_bytes, uint64_t stride2_bytes, uint32_t box0, uint32_t box1,
                  CUtensorMapSwizzle swizzle);

// Tile order of a persistent GEMM over an M x N output in bm x bn tiles with
// depth K (bytes per operand row = K): picks the banded dimension and the band
// width (see raster_tile) that minimise the operand bytes read from DRAM when
// a band's panels of one operand stay in L2.
void choose_raster(int64_t M, int64_t N, int64_t K, int bm, int bn, int32_t *band, int32_t *n_major);

// Per translation unit: read and clear its device error word.
cudaError_t take_device_error_gemm(unsigned long long *v);
cudaError_t take_device_error_decode(unsigned long long *v);
cudaError_t take_device_error_native(unsigned long long *v);
cudaError_t take_device_error_pair(unsigned long long *v);
cudaError_t take_device_error_swiglu(unsigned long long *v);
cudaError_t take_device_error_wgrad(unsigned long long *v);

// Launchers (arguments already validated).
fp8bq_status launch_encode(const float *x, int64_t n, uint8_t *q, cudaStream_t stream);
fp8bq_status launch_quant_act(const void *x, int64_t M, int64_t K, int64_t ldx, uint8_t *q, int64_t ldq, float *sa,
                              int64_t ldsa, int mode, cudaStream_t stream);
fp8bq_status launch_recalibrate(const fp8bq_weight_desc *descs, int n, int mode, cudaStream_t stream);
fp8bq_status launch_gemm(const uint8_t *qa, int64_t lda, const float *sa, int64_t ldsa, const uint8_t *qw,
                         int64_t ldw, const float *sw, void *y, int64_t ldy, int64_t M, int64_t N, int64_t K, int mode,
                         int variant, cudaStream_t stream);
bool pair_gemm_available();
fp8bq_status launch_gemm_pair(const uint8_t *qa, int64_t lda, const float *sa, int64_t ldsa, const uint8_t *qw,
                              int64_t ldw, const float *sw, void *y, int64_t ldy, int64_t M, int64_t N, int64_t K,
                              int tile_n, cudaStream_t stream);
fp8bq_status launch_gemm_native(const uint8_t *qa, int64_t lda, const float *sa, int64_t ldsa, const uint8_t *qw,
                                int64_t ldw, const float *sw, void *y, int64_t ldy, int64_t M, int64_t N, int64_t K,
                                cudaStream_t stream);
size_t decode_workspace_size(int64_t M, int64_t N, int64_t K);
fp8bq_status launch_gemm_decode(const void *x, int64_t ldx, const uint8_t *qw, int64_t ldw, const float *sw, void *y,
                                int64_t ldy, int64_t M, int64_t N, int64_t K, int mode, void *ws, size_t ws_bytes,
                                cudaStream_t stream);
fp8bq_status launch_grouped_gemm(const uint8_t *qa, int64_t lda, const float *sa, int64_t ldsa, const uint8_t *qw,
                                 const float *sw, const int32_t *offsets, int E, int64_t rows, int64_t N, int64_t K,
                                 void *y, int64_t ldy, cudaStream_t stream);
fp8bq_status launch_gemm_swiglu(const uint8_t *qa, int64_t lda, const float *sa, int64_t ldsa, const uint8_t *qw,
                                int64_t ldw, const float *sw, uint8_t *qh, int64_t ldqh, float *sh, int64_t ldsh,
                                void *h, int64_t ldh, int64_t M, int64_t I, int64_t K, int mode, cudaStream_t stream);
fp8bq_status launch_grouped_gemm_swiglu(const uint8_t *qa, int64_t lda, const float *sa, int64_t ldsa,
                                        const uint8_t *qw, const float *sw, const int32_t *offsets, int E,
                                        int64_t rows, int64_t I, int64_t K, uint8_t *qh, int64_t ldqh, float *sh,
                                        int64_t ldsh, void *h, int64_t ldh, int mode, cudaStream_t stream);
fp8bq_status launch_adamw_recalibrate(const fp8bq_adamw_desc *descs, int n, const fp8bq_adamw_config *cfg, int mode,
                                      cudaStream_t stream);
fp8bq_status launch_quant_act_t(const void *x, int64_t M, int64_t K, int64_t ldx, uint8_t *qt, int64_t ldqt, float *st,
                                int64_t ldst, int mode, cudaStream_t stream);
fp8bq_status launch_transpose_weight(const uint8_t *q, int64_t N, int64_t K, int64_t ldq, const float *sw,
                                     uint8_t *qt, int64_t ldqt, float *swt, cudaStream_t stream);
fp8bq_status launch_gemm_wgrad(const uint8_t *qa, int64_t lda, const float *sa, int64_t ldsa, const uint8_t *qb,
                               int64_t ldb, const float *sb, int64_t ldsb, void *y, int64_t ldy, int64_t N, int64_t K,
                               int64_t M, cudaStream_t stream);
size_t decode_attention_workspace_size(int64_t B, int64_t Hq, int64_t Hkv, int64_t S);
fp8bq_status launch_decode_attention(const void *q, const uint8_t *kq, const float *ks, const uint8_t *vq,
                                     const float *vs, const int32_t *lens, int64_t B, int64_t Hq, int64_t Hkv,
                                     int64_t S, float scale, void *o, void *ws, size_t ws_bytes, cudaStream_t stream);
fp8bq_status launch_kv_append(const void *k_new, const void *v_new, const int32_t *pos, uint8_t *kq, float *ks,
                              uint8_t *vq, float *vs, int64_t B, int64_t Hkv, int64_t S, int mode,
                              cudaStream_t stream);

}  // namespace fp8bq
