// The gate+up projection of a gated feed-forward block with its activation
// and the next layer's input quantization fused into the GEMM epilogue:
//   G|U = X . W_gu^T  (block-scaled FP8, FP32 promotion, bf16-rounded),
//   H   = bf16(silu(G) * U),
//   (qh, sh) = 1x128 E4M3 quantization of H,
// dense and grouped (mixture-of-experts).  H is the down projection's input,
// so the down GEMM reads qh/sh directly and no bf16 G|U or H tensor (and no
// separate activation or quantization pass) touches HBM.
//
// Method: "NVIDIA NeMo RL Achieves 48% Speedup With End-to-End FP8 Precision
// Training", section "Technical breakthrough" (FP8 linear layers on 1x128 /
// 128x128 block-wise E4M3 operands; non-linear functions in BF16; the Llama
// 3.1 8B model, whose feed-forward block is SwiGLU) and section "Real-world
// performance gains" (the quantization kernels are part of what keeps the
// FP8 linear layers from their full speedup).
#include "gemm_promote.cuh"

namespace fp8bq {
namespace {

// K = 0: G = U = 0, so H = 0, every code is +0 and every scale is 1.
__global__ void swiglu_empty_k_kernel(uint8_t *qh, int64_t ldqh, float *sh, int64_t ldsh, uint16_t *h, int64_t ldh,
                                      int64_t M, int64_t I) {
  const int64_t n = M * I;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += stride) {
    const int64_t m = i / I, c = i - m * I;
    qh[m * ldqh + c] = 0;
    if (h != nullptr) h[m * ldh + c] = 0;
    if (c % 128 == 0) sh[(c / 128) * ldsh + m] = 1.f;
  }
}

fp8bq_status fill_empty_k(uint8_t *qh, int64_t ldqh, float *sh, int64_t ldsh, void *h, int64_t ldh, int64_t M,
                          int64_t I, cudaStream_t stream) {
  const int64_t n = M * I;
  const int grid = (int)std::min<int64_t>((n + 255) / 256, (int64_t)num_sms() * 8);
  swiglu_empty_k_kernel<<<grid, 256, 0, stream>>>(qh, ldqh, sh, ldsh, static_cast<uint16_t *>(h), ldh, M, I);
  return check_launch("swiglu(K=0)");
}

template <bool G>
fp8bq_status prepare_swiglu(int mode) {
  return mode == FP8BQ_SCALE_POW2 ? prepare_kernel<G, kEpiSwigluPow2>() : prepare_kernel<G, kEpiSwigluFp32>();
}

template <bool G>
void launch_swiglu_kernel(int grid, const CUtensorMap &tA, const CUtensorMap &tB, const CUtensorMap &tY,
                          const GemmArgs &a, int mode, cudaStream_t stream) {
  if (mode == FP8BQ_SCALE_POW2)
    gemm_promote_kernel<G, kEpiSwigluPow2><<<grid, kThreads, Cfg<G>::kSmemBytes, stream>>>(tA, tB, tY, a);
  else
    gemm_promote_kernel<G, kEpiSwigluFp32><<<grid, kThreads, Cfg<G>::kSmemBytes, stream>>>(tA, tB, tY, a);
}

void set_outputs(GemmArgs &a, uint8_t *qh, int64_t ldqh, float *sh, int64_t ldsh, void *h, int64_t ldh) {
  a.qh = qh;
  a.ldqh = ldqh;
  a.sh = sh;
  a.ldsh = ldsh;
  a.h = static_cast<uint16_t *>(h);
  a.ldh = ldh;
}

}  // namespace

cudaError_t take_device_error_swiglu(unsigned long long *v) { return take_tu_device_error(v); }

fp8bq_status launch_gemm_swiglu(const uint8_t *qa, int64_t lda, const float *sa, int64_t ldsa, const uint8_t *qw,
                                int64_t ldw, const float *sw, uint8_t *qh, int64_t ldqh, float *sh, int64_t ldsh,
                                void *h, int64_t ldh, int64_t M, int64_t I, int64_t K, int mode,
                                cudaStream_t stream) {
  if (M == 0 || I == 0) return FP8BQ_OK;
  if (K == 0) return fill_empty_k(qh, ldqh, sh, ldsh, h, ldh, M, I, stream);
  const int64_t N = 2 * I;
  CUtensorMap tA, tB, tY;
  memset(&tY, 0, sizeof(tY));
  if (!make_tmap_2d(&tA, CU_TENSOR_MAP_DATA_TYPE_UINT8, qa, (uint64_t)K, (uint64_t)M, (uint64_t)lda, BK, BM,
                    CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_tmap_2d(&tB, CU_TENSOR_MAP_DATA_TYPE_UINT8, qw, (uint64_t)K, (uint64_t)N, (uint64_t)ldw, BK, BN,
                    CU_TENSOR_MAP_SWIZZLE_128B))
    return FP8BQ_ERR_INVALID_ARG;
  fp8bq_status st = prepare_swiglu<false>(mode);
  if (st != FP8BQ_OK) return st;
  GemmArgs a = {};
  a.sa = sa;
  a.sw = sw;
  a.ldsa = ldsa;
  a.M = (int32_t)M;
  a.N = (int32_t)N;
  a.KB = (int32_t)(K / BK);
  a.NB = (int32_t)(N / 128);
  a.num_m = (int32_t)((M + BM - 1) / BM);
  a.num_n = (int32_t)(N / BN);
  choose_raster(M, N, K, BM, BN, &a.band, &a.n_major);
  set_outputs(a, qh, ldqh, sh, ldsh, h, ldh);
  const int64_t tiles = (int64_t)a.num_m * a.num_n;
  const int grid = (int)std::min<int64_t>(tiles, num_sms());
  launch_swiglu_kernel<false>(grid, tA, tB, tY, a, mode, stream);
  return check_launch("gemm_swiglu");
}

fp8bq_status launch_grouped_gemm_swiglu(const uint8_t *qa, int64_t lda, const float *sa, int64_t ldsa,
                                        const uint8_t *qw, const float *sw, const int32_t *offsets, int E,
                                        int64_t rows, int64_t I, int64_t K, uint8_t *qh, int64_t ldqh, float *sh,
                                        int64_t ldsh, void *h, int64_t ldh, int mode, cudaStream_t stream) {
  if (rows == 0 || I == 0) return FP8BQ_OK;
  if (K == 0) return fill_empty_k(qh, ldqh, sh, ldsh, h, ldh, rows, I, stream);
  const int64_t N = 2 * I;
  CUtensorMap tA, tB, tY;
  memset(&tY, 0, sizeof(tY));
  if (!make_tmap_2d(&tA, CU_TENSOR_MAP_DATA_TYPE_UINT8, qa, (uint64_t)K, (uint64_t)rows, (uint64_t)lda, BK, BM,
                    CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_tmap_3d(&tB, CU_TENSOR_MAP_DATA_TYPE_UINT8, qw, (uint64_t)K, (uint64_t)N, (uint64_t)E, (uint64_t)K,
                    (uint64_t)N * (uint64_t)K, BK, BN, CU_TENSOR_MAP_SWIZZLE_128B))
    return FP8BQ_ERR_INVALID_ARG;
  fp8bq_status st = prepare_swiglu<true>(mode);
  if (st != FP8BQ_OK) return st;
  GemmArgs a = {};
  a.sa = sa;
  a.sw = sw;
  a.ldsa = ldsa;
  a.M = (int32_t)rows;
  a.N = (int32_t)N;
  a.KB = (int32_t)(K / BK);
  a.NB = (int32_t)(N / 128);
  a.num_m = 0;
  a.num_n = (int32_t)(N / BN);
  a.offsets = offsets;
  a.E = E;
  set_outputs(a, qh, ldqh, sh, ldsh, h, ldh);
  launch_swiglu_kernel<true>(num_sms(), tA, tB, tY, a, mode, stream);
  return check_launch("grouped_gemm_swiglu");
}

}  // namespace fp8bq
