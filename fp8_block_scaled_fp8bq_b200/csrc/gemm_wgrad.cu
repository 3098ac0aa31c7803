// The weight-gradient GEMM of the FP8 linear layer's backward pass:
//   dW[N][K] = sum over tokens m of dY[m][n] X[m][k],
// from the token-axis 1x128 codes of dY^T [N][M] and X^T [K][M] (both
// token-contiguous, as fp8bq_quant_act_t writes them).  It runs on the
// promotion kernel of gemm_promote.cuh: A = dY^T with its row scales, and B =
// X^T whose 1x128 scales vary per B row (output column), so the epilogue forms
// the scale product per column pair (kEpiBf16RowB).
//
// Method: "NVIDIA NeMo RL Achieves 48% Speedup With End-to-End FP8 Precision
// Training", section "Technical breakthrough": FP8 in training as in
// generation, block-wise E4M3 with 1x128 tiles for activations (here both
// operands are activations or their gradients, tiled along the contraction).
#include "gemm_promote.cuh"

namespace fp8bq {

cudaError_t take_device_error_wgrad(unsigned long long *v) { return take_tu_device_error(v); }

fp8bq_status launch_gemm_wgrad(const uint8_t *qa, int64_t lda, const float *sa, int64_t ldsa, const uint8_t *qb,
                               int64_t ldb, const float *sb, int64_t ldsb, void *y, int64_t ldy, int64_t N, int64_t K,
                               int64_t M, cudaStream_t stream) {
  if (N == 0 || K == 0) return FP8BQ_OK;
  if (M == 0) {
    cudaError_t e = cudaMemset2DAsync(y, (size_t)ldy * 2, 0, (size_t)K * 2, (size_t)N, stream);
    return e == cudaSuccess ? FP8BQ_OK : cuda_fail(e, "memset(dW)");
  }
  CUtensorMap tA, tB, tY;
  if (!make_tmap_2d(&tA, CU_TENSOR_MAP_DATA_TYPE_UINT8, qa, (uint64_t)M, (uint64_t)N, (uint64_t)lda, BK, BM,
                    CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_tmap_2d(&tB, CU_TENSOR_MAP_DATA_TYPE_UINT8, qb, (uint64_t)M, (uint64_t)K, (uint64_t)ldb, BK, BN,
                    CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_tmap_2d(&tY, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, y, (uint64_t)K, (uint64_t)N, (uint64_t)ldy * 2, 64, 32,
                    CU_TENSOR_MAP_SWIZZLE_128B))
    return FP8BQ_ERR_INVALID_ARG;
  fp8bq_status st = prepare_kernel<false, kEpiBf16RowB>();
  if (st != FP8BQ_OK) return st;
  GemmArgs a = {};
  a.sa = sa;
  a.sw = sb;
  a.ldsa = ldsa;
  a.ldsw = ldsb;
  a.M = (int32_t)N;
  a.N = (int32_t)K;
  a.KB = (int32_t)(M / BK);
  a.NB = (int32_t)((K + 127) / 128);
  a.num_m = (int32_t)((N + BM - 1) / BM);
  a.num_n = (int32_t)((K + BN - 1) / BN);
  choose_raster(N, K, M, BM, BN, &a.band, &a.n_major);
  const int64_t tiles = (int64_t)a.num_m * a.num_n;
  const int grid = (int)std::min<int64_t>(tiles, num_sms());
  gemm_promote_kernel<false, kEpiBf16RowB><<<grid, kThreads, Cfg<false>::kSmemBytes, stream>>>(tA, tB, tY, a);
  return check_launch("gemm_wgrad");
}

}  // namespace fp8bq
