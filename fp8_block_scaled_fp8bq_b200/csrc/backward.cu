// Operand preparation for the backward pass of the FP8 linear layer:
//   * the 1x128 quantization along the token axis with transposed output (the
//     weight-gradient GEMM contracts over tokens, so both of its operands, dY
//     and X, are quantized in 128-token tiles and stored token-contiguous);
//   * the transpose of a weight's 128x128-tile codes and scales (the
//     data-gradient GEMM dX = dY W multiplies by W^T; a square tile's scale
//     applies to its transpose unchanged, so no requantization is needed).
//
// Method: "NVIDIA NeMo RL Achieves 48% Speedup With End-to-End FP8 Precision
// Training", section "Technical breakthrough": FP8 in both generation and
// training, block-wise E4M3 with 1x128 activation and 128x128 weight tiles.
//
// Both kernels are HBM-bound: 2 bytes read and 1 written per element for the
// quantizer, 1 and 1 for the transpose.  Each block stages its tile in shared
// memory so that the global reads and writes are both row-contiguous.
#include <algorithm>

#include "device.cuh"
#include "internal.h"
#include "quant.cuh"

namespace fp8bq {
namespace {

using namespace qdev;

// ---------------------------------------------------------------------------
// Token-axis 1x128 quantization, transposed output
// ---------------------------------------------------------------------------
// Block (bx, by): tokens [128 by, +128) x columns [128 bx, +128) of X.  The
// 128 x 128 bf16 tile is staged in shared memory (256-byte rows, 16-byte
// loads, 16 lanes per row).  Warp w owns tokens [32 (w & 3), +32) of column
// half w >> 2, and lane l the column pair (2 l, 2 l + 1) of that half: it reads
// one 4-byte word per token (a warp reads 128 contiguous bytes of one row:
// no bank conflicts).  The four token groups' partial amaxes meet in shared
// memory; each lane then writes 32 token-contiguous codes of each of its two
// columns into X^T, i.e. whole 32-byte sectors.
constexpr int kTTok = 128, kTCol = 128;

// The 32 tokens of two columns (low and high bf16 halves of w[]) -> codes.
template <int MODE, bool FAST>
__device__ __forceinline__ void encode_columns(const uint32_t (&w)[32], const TileScale &t0, const TileScale &t1,
                                               uint32_t (&ca)[8], uint32_t (&cb)[8]) {
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    // codes of -(x / s), sign bits flipped back (see neg_quotient2)
    const float2 qa0 = neg_quotient2<MODE, FAST>(make_float2(bf16_lo(w[4 * j]), bf16_lo(w[4 * j + 1])), t0);
    const float2 qa1 = neg_quotient2<MODE, FAST>(make_float2(bf16_lo(w[4 * j + 2]), bf16_lo(w[4 * j + 3])), t0);
    const float2 qb0 = neg_quotient2<MODE, FAST>(make_float2(bf16_hi(w[4 * j]), bf16_hi(w[4 * j + 1])), t1);
    const float2 qb1 = neg_quotient2<MODE, FAST>(make_float2(bf16_hi(w[4 * j + 2]), bf16_hi(w[4 * j + 3])), t1);
    ca[j] = (e4m3x2(qa0.x, qa0.y) | (e4m3x2(qa1.x, qa1.y) << 16)) ^ 0x80808080u;
    cb[j] = (e4m3x2(qb0.x, qb0.y) | (e4m3x2(qb1.x, qb1.y) << 16)) ^ 0x80808080u;
  }
}

template <int MODE>
__global__ void __launch_bounds__(256) quant_act_t_kernel(const uint16_t *__restrict__ x, int64_t M, int64_t K,
                                                          int64_t ldx, uint8_t *__restrict__ qt, int64_t ldqt,
                                                          float *__restrict__ st, int64_t ldst) {
  __shared__ __align__(16) uint32_t tile[kTTok][kTCol / 2];
  __shared__ uint32_t part[4][kTCol / 2];  // [token group][column pair]: packed |bf16| maxima
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t m0 = (int64_t)blockIdx.y * kTTok, k0 = (int64_t)blockIdx.x * kTCol;

#pragma unroll
  for (int it = 0; it < 8; ++it) {  // 128 rows x 16 chunks of 16 bytes
    const int idx = it * 256 + threadIdx.x;
    const int r = idx >> 4, c = idx & 15;
    const int64_t m = m0 + r, k = k0 + c * 8;
    const uint4 v = (m < M && k < K) ? ld_nc_v4(x + m * ldx + k) : make_uint4(0, 0, 0, 0);
    *reinterpret_cast<uint4 *>(&tile[r][c * 4]) = v;
  }
  __syncthreads();

  const int tg = warp & 3, ch = warp >> 2;
  const int pc = ch * 32 + lane;  // column pair within the tile
  uint32_t w[32];
  uint32_t am = 0;
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    w[i] = tile[tg * 32 + i][pc];
    am = __vmaxu2(am, w[i] & 0x7FFF7FFFu);
  }
  part[tg][pc] = am;
  __syncthreads();
  am = __vmaxu2(__vmaxu2(part[0][pc], part[1][pc]), __vmaxu2(part[2][pc], part[3][pc]));
  const TileScale t0 = tile_scale<MODE>(bits_to_amax(am & 0xFFFFu));
  const TileScale t1 = tile_scale<MODE>(bits_to_amax(am >> 16));

  const int64_t ka = k0 + 2 * pc, kb = ka + 1;
  const int64_t mt = m0 + tg * 32;  // first token of this lane's 32
  uint32_t ca[8], cb[8];            // 32 codes of column ka, 32 of column kb
  if (fast_tile<MODE>(t0) && fast_tile<MODE>(t1)) encode_columns<MODE, true>(w, t0, t1, ca, cb);
  else encode_columns<MODE, false>(w, t0, t1, ca, cb);
  if (mt < M) {
    const bool whole = mt + 32 <= M;
    if (ka < K) {
      uint8_t *d = qt + ka * ldqt + mt;
      if (whole) {
        *reinterpret_cast<uint4 *>(d) = make_uint4(ca[0], ca[1], ca[2], ca[3]);
        *reinterpret_cast<uint4 *>(d + 16) = make_uint4(ca[4], ca[5], ca[6], ca[7]);
      } else {
        for (int i = 0; i < 32 && mt + i < M; ++i) d[i] = (uint8_t)(ca[i >> 2] >> (8 * (i & 3)));
      }
    }
    if (kb < K) {
      uint8_t *d = qt + kb * ldqt + mt;
      if (whole) {
        *reinterpret_cast<uint4 *>(d) = make_uint4(cb[0], cb[1], cb[2], cb[3]);
        *reinterpret_cast<uint4 *>(d + 16) = make_uint4(cb[4], cb[5], cb[6], cb[7]);
      } else {
        for (int i = 0; i < 32 && mt + i < M; ++i) d[i] = (uint8_t)(cb[i >> 2] >> (8 * (i & 3)));
      }
    }
  }
  if (tg == 0) {
    float *srow = st + (int64_t)blockIdx.y * ldst;
    if (ka < K) srow[ka] = t0.s;
    if (kb < K) srow[kb] = t1.s;
  }
}

// ---------------------------------------------------------------------------
// Transpose of a weight's codes and tile scales
// ---------------------------------------------------------------------------
// Block (bx, by): rows [64 by, +64) x columns [64 bx, +64) of q.  Staged as
// 64 x 64 bytes (16-byte loads, 4 lanes per row), read back column-wise as
// 4-byte words gathered from 4 rows, written as 16-byte rows of q^T.
constexpr int kTB = 64;

__global__ void __launch_bounds__(256) transpose_codes_kernel(const uint8_t *__restrict__ q, int64_t R, int64_t C,
                                                              int64_t ldq, uint8_t *__restrict__ qt, int64_t ldqt) {
  __shared__ __align__(16) uint8_t tile[kTB][kTB + 4];
  const int64_t r0 = (int64_t)blockIdx.y * kTB, c0 = (int64_t)blockIdx.x * kTB;
  {
    const int r = threadIdx.x >> 2, c = (threadIdx.x & 3) * 16;  // 64 rows x 4 chunks
    const int64_t gr = r0 + r, gc = c0 + c;
    uint4 v = make_uint4(0, 0, 0, 0);
    if (gr < R && gc < C) v = *reinterpret_cast<const uint4 *>(q + gr * ldq + gc);
    const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) *reinterpret_cast<uint32_t *>(&tile[r][c + 4 * i]) = u[i];
  }
  __syncthreads();
  {
    const int oc = threadIdx.x >> 2, orr = (threadIdx.x & 3) * 16;  // output row = input column oc
    uint32_t u[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int rr = orr + 4 * i;
      u[i] = (uint32_t)tile[rr][oc] | ((uint32_t)tile[rr + 1][oc] << 8) | ((uint32_t)tile[rr + 2][oc] << 16) |
             ((uint32_t)tile[rr + 3][oc] << 24);
    }
    const int64_t gr = c0 + oc, gc = r0 + orr;
    if (gr < C && gc < R) *reinterpret_cast<uint4 *>(qt + gr * ldqt + gc) = make_uint4(u[0], u[1], u[2], u[3]);
  }
}

__global__ void transpose_scales_kernel(const float *__restrict__ s, int64_t NB, int64_t KB, float *__restrict__ st) {
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < NB * KB; i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t nb = i / KB, kb = i - nb * KB;
    st[kb * NB + nb] = s[i];
  }
}

}  // namespace

fp8bq_status launch_quant_act_t(const void *x, int64_t M, int64_t K, int64_t ldx, uint8_t *qt, int64_t ldqt, float *st,
                                int64_t ldst, int mode, cudaStream_t stream) {
  const int64_t gx = (K + kTCol - 1) / kTCol, gy = (M + kTTok - 1) / kTTok;
  if (gx > 0x7fffffff || gy > 65535) return FP8BQ_ERR_UNSUPPORTED;
  const dim3 grid((unsigned)gx, (unsigned)gy);
  const uint16_t *xs = static_cast<const uint16_t *>(x);
  if (mode == FP8BQ_SCALE_FP32)
    quant_act_t_kernel<FP8BQ_SCALE_FP32><<<grid, 256, 0, stream>>>(xs, M, K, ldx, qt, ldqt, st, ldst);
  else
    quant_act_t_kernel<FP8BQ_SCALE_POW2><<<grid, 256, 0, stream>>>(xs, M, K, ldx, qt, ldqt, st, ldst);
  return check_launch("quant_act_t");
}

fp8bq_status launch_transpose_weight(const uint8_t *q, int64_t N, int64_t K, int64_t ldq, const float *sw,
                                     uint8_t *qt, int64_t ldqt, float *swt, cudaStream_t stream) {
  const int64_t gx = (K + kTB - 1) / kTB, gy = (N + kTB - 1) / kTB;
  if (gx > 0x7fffffff || gy > 65535) return FP8BQ_ERR_UNSUPPORTED;
  transpose_codes_kernel<<<dim3((unsigned)gx, (unsigned)gy), 256, 0, stream>>>(q, N, K, ldq, qt, ldqt);
  fp8bq_status st = check_launch("transpose_weight(codes)");
  if (st != FP8BQ_OK) return st;
  const int64_t NB = (N + 127) / 128, KB = (K + 127) / 128;
  const int blocks = (int)std::min<int64_t>((NB * KB + 255) / 256, 1024);
  transpose_scales_kernel<<<blocks, 256, 0, stream>>>(sw, NB, KB, swt);
  return check_launch("transpose_weight(scales)");
}

}  // namespace fp8bq
