// E4M3 quantization device code shared by the quantizer kernels and the
// decode prologue: tile scales, the correctly rounded element quotient, the
// E4M3 conversion, and the 1x128 activation tile kernel.
//
// Method: "NVIDIA NeMo RL Achieves 48% Speedup With End-to-End FP8 Precision
// Training", section "Technical breakthrough" (block-wise E4M3; activations
// 1x128, weights 128x128); power-of-2 scales from section "Why this matters
// for AI economics".
#pragma once

#include <cuda_fp8.h>

#include "device.cuh"
#include "../../include/fp8bq.h"

namespace fp8bq {
namespace qdev {

// ---------------------------------------------------------------------------
// Scales
// ---------------------------------------------------------------------------
// Smallest e with amax <= 448 * 2^e, clamped to [-127, 127].  With
// amax = f * 2^E, f in [1, 2): 448 * 2^e = 1.75 * 2^(e+8), so e = E - 8 when
// f <= 1.75 and e = E - 7 otherwise.  amax > 0.
__device__ __forceinline__ int pow2_exponent(float amax) {
  uint32_t b = __float_as_uint(amax);
  int ef = (int)(b >> 23);
  uint32_t frac = b & 0x7FFFFFu;
  int E;
  if (ef == 0) {                        // denormal: normalize the fraction
    int p = 31 - __clz((int)frac);      // leading one, 0..22
    E = p - 149;
    frac = (frac << (23 - p)) & 0x7FFFFFu;
  } else {
    E = ef - 127;
  }
  int e = (frac <= 0x600000u) ? E - 8 : E - 7;
  return max(-127, min(127, e));
}

// 2^e for e in [-127, 127], exactly (2^-127 is a binary32 denormal).
__device__ __forceinline__ float exp2_exact(int e) {
  return e >= -126 ? __uint_as_float((uint32_t)(e + 127) << 23) : __uint_as_float(0x00400000u);
}

// Per-tile constants of the element quotient x / s.
//   FP32 scales: s = amax / 448; r = RN(1/s).  When s >= 2^-60 the quotient is
//     computed with Markstein's correction (P. Markstein, "Computation of
//     elementary functions on the IBM RISC System/6000 processor", IBM J. Res.
//     Dev. 34(1), 1990): q0 = RN(x r), the residual q0 s - x is formed
//     exactly by one fma, and q1 = RN(q0 - residual * r) is the correctly
//     rounded quotient (see quotient() for the sign of zero).  Below 2^-60 (tiles whose amax is under ~4e-16) the residual
//     could underflow, so those tiles use the IEEE division.  A GPU test
//     compares the codes this produces with the oracle's (an IEEE division)
//     for every pair (tile amax, element) of bf16 values.
//   POW2 scales: s = 2^e and r = 2^-e exactly; x * r is the single rounding of
//     the exact quotient, i.e. the same as the division.
struct TileScale {
  float s;     // the scale
  float r;     // reciprocal (exact for POW2, RN(1/s) for FP32)
  bool exact;  // FP32 only: use the IEEE division for this tile
};

template <int MODE>
__device__ __forceinline__ TileScale tile_scale(float amax) {
  TileScale t;
  if (!(amax > 0.f)) {
    t.s = 1.f;
    t.r = 1.f;
    t.exact = false;
  } else if (MODE == FP8BQ_SCALE_FP32) {
    t.s = __fdiv_rn(amax, 448.f);
    t.r = __frcp_rn(t.s);
    t.exact = !(t.s >= 8.673617379884035e-19f);  // 2^-60
  } else {
    const int e = pow2_exponent(amax);
    t.s = exp2_exact(e);
    t.r = exp2_exact(-e);
    t.exact = false;
  }
  return t;
}

// The binary32 quotient x / s, correctly rounded.  The residual is formed as
// q0 s - x (exact by one fma) and subtracted in the correcting fma, which keeps
// the sign of zero: x = -0 gives q0 = -0, residual +0 and q1 = -0 + -0 = -0,
// while x = +0 gives +0.
template <int MODE>
__device__ __forceinline__ float quotient(float x, const TileScale &t) {
  if (MODE == FP8BQ_SCALE_POW2) return __fmul_rn(x, t.r);
  if (t.exact) return __fdiv_rn(x, t.s);
  const float q0 = __fmul_rn(x, t.r);
  const float res = __fmaf_rn(q0, t.s, -x);
  return __fmaf_rn(-res, t.r, q0);
}

__device__ __forceinline__ uint32_t e4m3x2(float lo, float hi) {
  return (uint32_t)__nv_cvt_float2_to_fp8x2(make_float2(lo, hi), __NV_SATFINITE, __NV_E4M3);
}

// The negated quotient -(x / s), correctly rounded, two lanes per instruction.
// Negating the per-tile constant r instead of per-element values leaves the
// packed sequence with no sign flips:
//   -q0 = RN(x * -r),  e = x - q0 s = fma(-q0, s, x) (exact),
//   -q1 = RN(e * -r - q0) = fma(e, -r, -q0),
// which is -(q0 + e r), Markstein's correction of q0, negated (round to
// nearest is symmetric).  Zero keeps its sign: x = -0 gives +0 = -(-0) and
// x = +0 gives -0.  The E4M3 code of x / s is then the code of -(x / s) with
// its sign bit flipped (the conversion is sign-symmetric).
//
// FAST = true drops the per-call test of t.exact: the caller has tested the
// tile once (fast_tile) and takes this path only when it holds, so the test
// is not repeated for every pair of elements (for FP32 scales that test cost
// about a fifth of a quantizer's instructions).
template <int MODE>
__device__ __forceinline__ bool fast_tile(const TileScale &t) {
  return MODE == FP8BQ_SCALE_POW2 || !t.exact;
}

template <int MODE, bool FAST = false>
__device__ __forceinline__ float2 neg_quotient2(float2 x, const TileScale &t) {
  const float2 nr2 = make_float2(-t.r, -t.r);
  if (MODE == FP8BQ_SCALE_POW2) return __fmul2_rn(x, nr2);
  if (!FAST && t.exact) return make_float2(-__fdiv_rn(x.x, t.s), -__fdiv_rn(x.y, t.s));
  const float2 nq0 = __fmul2_rn(x, nr2);
  const float2 e = __ffma2_rn(nq0, make_float2(t.s, t.s), x);
  return __ffma2_rn(e, nr2, nq0);
}

// Codes of -(x / s) for two bf16 packed in a 32-bit word (lower address in the
// low half): the codes of x / s with both sign bits flipped.
template <int MODE, bool FAST = false>
__device__ __forceinline__ uint32_t encode2_neg(uint32_t w, const TileScale &t) {
  const float2 nq = neg_quotient2<MODE, FAST>(make_float2(bf16_lo(w), bf16_hi(w)), t);
  return e4m3x2(nq.x, nq.y);
}

// Four bf16 (two packed words) -> four E4M3 codes.
template <int MODE, bool FAST = false>
__device__ __forceinline__ uint32_t encode4(uint32_t w01, uint32_t w23, const TileScale &t) {
  return (encode2_neg<MODE, FAST>(w01, t) | (encode2_neg<MODE, FAST>(w23, t) << 16)) ^ 0x80808080u;
}

// Two bf16 packed in a 32-bit word -> E4M3x2.
template <int MODE, bool FAST = false>
__device__ __forceinline__ uint32_t encode2(uint32_t w, const TileScale &t) {
  return encode2_neg<MODE, FAST>(w, t) ^ 0x8080u;
}

// 8 bf16 (one 16-byte vector) -> 8 E4M3 codes (8 bytes).
template <int MODE, bool FAST = false>
__device__ __forceinline__ uint2 encode8(uint4 v, const TileScale &t) {
  uint2 r;
  r.x = encode4<MODE, FAST>(v.x, v.y, t);
  r.y = encode4<MODE, FAST>(v.z, v.w, t);
  return r;
}

// max |x| of 8 bf16 as a bf16 bit pattern (exact for finite values).
__device__ __forceinline__ uint32_t absmax_bits8(uint4 v) {
  uint32_t m = __vmaxu2(__vmaxu2(v.x & 0x7FFF7FFFu, v.y & 0x7FFF7FFFu), __vmaxu2(v.z & 0x7FFF7FFFu, v.w & 0x7FFF7FFFu));
  return max(m & 0xFFFFu, m >> 16);
}

__device__ __forceinline__ float bits_to_amax(uint32_t b16) { return __uint_as_float(b16 << 16); }

// One 1x128 tile of the activation (row m, K-block kb) quantized by a group of
// four lanes into a shared-memory tile of 128-byte rows in the MMA operand's
// 128-byte-swizzled layout (16-byte chunk c of row m at chunk position
// c ^ (m & 7)); lane qd of the group owns chunks qd, qd + 4,
// qd + 8, qd + 12 of the row, as fp8bq_quant_act's vector kernel does.
// Every lane of the warp calls it (the amax shuffles span the warp); lanes
// with have == false store nothing.  v: the lane's four 16-byte pieces of the
// row (pieces qd, qd + 4, qd + 8, qd + 12), loaded by the caller.
template <int MODE>
__device__ __forceinline__ void quant_row_tile_to_smem(bool have, const uint4 (&v)[4], int qd, uint8_t *tile, int m,
                                                       float *scale) {
  uint32_t am = max(max(absmax_bits8(v[0]), absmax_bits8(v[1])), max(absmax_bits8(v[2]), absmax_bits8(v[3])));
  am = max(am, __shfl_xor_sync(0xffffffffu, am, 1));
  am = max(am, __shfl_xor_sync(0xffffffffu, am, 2));
  if (!have) return;
  const TileScale ts = tile_scale<MODE>(bits_to_amax(am));
  uint8_t *row = tile + m * 128;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const int e8 = j * 4 + qd;  // 8-element piece of the row
    const uint2 c = fast_tile<MODE>(ts) ? encode8<MODE, true>(v[j], ts) : encode8<MODE>(v[j], ts);
    *reinterpret_cast<uint2 *>(row + (((e8 >> 1) ^ (m & 7)) << 4) + (e8 & 1) * 8) = c;
  }
  if (qd == 0) *scale = ts.s;
}

// ---------------------------------------------------------------------------
// Activation quantization, 1x128 tiles
// ---------------------------------------------------------------------------
// Block = 8 warps = 64 tiles: rows [bx * 64, +64) of K-block by.  Four lanes
// share a tile: lane qd holds the tile's 16-byte chunks qd, qd+4, qd+8, qd+12
// (32 elements), so each load instruction reads 64 contiguous bytes per row and
// each store writes 32; the tile amax takes two shuffles and every lane's
// scale computation is spread over 32 elements.
template <int MODE>
__device__ __forceinline__ void quant_act_vec_block(int64_t bx, int64_t by, const uint16_t *__restrict__ x,
                                                    int64_t M, int64_t K, int64_t ldx, uint8_t *__restrict__ q,
                                                    int64_t ldq, float *__restrict__ sa, int64_t ldsa) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int qd = lane & 3;
  const int64_t r = bx * 64 + warp * 8 + (lane >> 2);
  const int64_t kb = by;
  uint4 v[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const int64_t k = kb * 128 + (j * 4 + qd) * 8;  // K % 8 == 0 here: a vector is wholly in or out
    v[j] = (r < M && k < K) ? ld_nc_v4(x + r * ldx + k) : make_uint4(0, 0, 0, 0);
  }
  uint32_t m = max(max(absmax_bits8(v[0]), absmax_bits8(v[1])), max(absmax_bits8(v[2]), absmax_bits8(v[3])));
  m = max(m, __shfl_xor_sync(0xffffffffu, m, 1));
  m = max(m, __shfl_xor_sync(0xffffffffu, m, 2));
  const TileScale ts = tile_scale<MODE>(bits_to_amax(m));
  if (r < M) {
    if (fast_tile<MODE>(ts)) {
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int64_t k = kb * 128 + (j * 4 + qd) * 8;
        if (k < K) *reinterpret_cast<uint2 *>(q + r * ldq + k) = encode8<MODE, true>(v[j], ts);
      }
    } else {
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int64_t k = kb * 128 + (j * 4 + qd) * 8;
        if (k < K) *reinterpret_cast<uint2 *>(q + r * ldq + k) = encode8<MODE>(v[j], ts);
      }
    }
    if (qd == 0) sa[kb * ldsa + r] = ts.s;
  }
}

// Any alignment: one half-warp per tile, element j of lane hl is k0 + hl + 16 j.
// Block (bx, by) covers rows [bx * 16, +16) of K-block by.
template <int MODE>
__device__ __forceinline__ void quant_act_scalar_block(int64_t bx, int64_t by, const uint16_t *__restrict__ x,
                                                       int64_t M, int64_t K, int64_t ldx, uint8_t *__restrict__ q,
                                                       int64_t ldq, float *__restrict__ sa, int64_t ldsa) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int hl = lane & 15, half = lane >> 4;
  const int64_t kb = by;
  const int64_t r = bx * 16 + warp * 2 + half;
  uint16_t e[8];
  uint32_t m = 0;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const int64_t k = kb * 128 + hl + 16 * j;
    e[j] = (r < M && k < K) ? x[r * ldx + k] : (uint16_t)0;
    m = max(m, (uint32_t)(e[j] & 0x7FFFu));
  }
  m = max(m, __shfl_xor_sync(0xffffffffu, m, 8));
  m = max(m, __shfl_xor_sync(0xffffffffu, m, 4));
  m = max(m, __shfl_xor_sync(0xffffffffu, m, 2));
  m = max(m, __shfl_xor_sync(0xffffffffu, m, 1));
  const TileScale ts = tile_scale<MODE>(bits_to_amax(m));
  if (r >= M) return;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const int64_t k = kb * 128 + hl + 16 * j;
    if (k < K) {
      const float f = __uint_as_float((uint32_t)e[j] << 16);
      q[r * ldq + k] = (uint8_t)(e4m3x2(quotient<MODE>(f, ts), 0.f) & 0xFFu);
    }
  }
  if (hl == 0) sa[kb * ldsa + r] = ts.s;
}

template <int MODE>
__global__ void __launch_bounds__(256) quant_act_vec_kernel(const uint16_t *__restrict__ x, int64_t M, int64_t K,
                                                            int64_t ldx, uint8_t *__restrict__ q, int64_t ldq,
                                                            float *__restrict__ sa, int64_t ldsa) {
  quant_act_vec_block<MODE>(blockIdx.x, blockIdx.y, x, M, K, ldx, q, ldq, sa, ldsa);
}

template <int MODE>
__global__ void __launch_bounds__(256) quant_act_scalar_kernel(const uint16_t *__restrict__ x, int64_t M, int64_t K,
                                                               int64_t ldx, uint8_t *__restrict__ q, int64_t ldq,
                                                               float *__restrict__ sa, int64_t ldsa) {
  quant_act_scalar_block<MODE>(blockIdx.x, blockIdx.y, x, M, K, ldx, q, ldq, sa, ldsa);
}

}  // namespace qdev
}  // namespace fp8bq
