// The optimizer step fused with the recalibration that follows it: one pass
// over each weight's FP32 master copy, gradient and moments updates them
// (AdamW), rounds the new weight to bf16 and requantizes it over 128x128 tiles.
//
// Method: "NVIDIA NeMo RL Achieves 48% Speedup With End-to-End FP8 Precision
// Training", section "Real-world performance gains": the policy weights change
// with every training step, so the scales are recalibrated after each step
// (the pages put that overhead at a few percent); section "Technical
// breakthrough": 128x128 weight tiles in E4M3.  The optimizer is AdamW
// (Loshchilov & Hutter, "Decoupled Weight Decay Regularization", ICLR 2019,
// with the bias-corrected moments of Kingma & Ba, "Adam", ICLR 2015) on binary32
// state; every operation is one correctly rounded binary32 operation in the
// order the header states, so the result is bit for bit that definition.
//
// HBM-bound: per weight element 16 bytes are read (weight, gradient, two
// moments) and 12 + 1 (+ 2 with the bf16 copy) written.  One 128x128 tile per
// 256-thread block iteration: warp w owns rows 16 w .. 16 w + 15, lane l the
// 16-byte column chunk l, so every load and store instruction of a warp covers
// 512 contiguous bytes of one row (fp32) and the code stores 128.  The new bf16
// weights stay in registers (32 per thread) until the tile's amax is known.
#include <math.h>

#include <algorithm>

#include "device.cuh"
#include "internal.h"
#include "quant.cuh"

namespace fp8bq {
namespace {

using namespace qdev;

constexpr int kMaxOptDescs = 96;

struct OptTensor {
  float *p;
  const float *g;
  float *m;
  float *v;
  uint16_t *w;  // may be null
  uint8_t *q;
  float *s;
  int64_t N, K;
  int64_t tile_begin;
  int32_t KB;
};

struct OptParams {
  int32_t n;
  int64_t total;
  float lr, b1, b2, eps, wd;
  float c1, c2;    // 1 - b1, 1 - b2 (binary32)
  float bc1, bc2;  // 1 - b^t (double pow, rounded to binary32)
  OptTensor t[kMaxOptDescs];
};

// One AdamW element, each step one IEEE binary32 operation.
__device__ __forceinline__ void adamw_elem(float &p, float g, float &m, float &v, const OptParams &P) {
  const float mi = __fadd_rn(__fmul_rn(P.b1, m), __fmul_rn(P.c1, g));
  const float vi = __fadd_rn(__fmul_rn(P.b2, v), __fmul_rn(__fmul_rn(P.c2, g), g));
  const float mh = __fdiv_rn(mi, P.bc1);
  const float vh = __fdiv_rn(vi, P.bc2);
  const float d = __fadd_rn(__fsqrt_rn(vh), P.eps);
  const float u = __fadd_rn(__fdiv_rn(mh, d), __fmul_rn(P.wd, p));
  p = __fsub_rn(p, __fmul_rn(P.lr, u));
  m = mi;
  v = vi;
}

__device__ __forceinline__ uint32_t bf16x2_bits(float lo, float hi) {
  __nv_bfloat162 b = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t *>(&b);
}

__device__ __forceinline__ float4 ld4(const float *p) { return *reinterpret_cast<const float4 *>(p); }

__device__ __forceinline__ float4 ld4_nc(const float *p) {
  const uint4 u = ld_nc_v4(p);
  return make_float4(__uint_as_float(u.x), __uint_as_float(u.y), __uint_as_float(u.z), __uint_as_float(u.w));
}

template <int MODE>
__device__ __forceinline__ void adamw_tile(const OptTensor &T, const OptParams &P, int64_t nb, int64_t kb,
                                           uint32_t *red) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t k = kb * 128 + lane * 4;
  const bool kin = k < T.K;  // K % 4 == 0: a chunk is wholly in or out
  const int64_t r0 = nb * 128 + warp * 16;
  uint32_t wb[16][2];
  uint32_t amax = 0;
#pragma unroll
  for (int i0 = 0; i0 < 16; i0 += 4) {
    float4 pv[4], gv[4], mv[4], vv[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int64_t n = r0 + i0 + j;
      const bool in = kin && n < T.N;
      const int64_t o = n * T.K + k;
      const float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
      pv[j] = in ? ld4(T.p + o) : z;
      gv[j] = in ? ld4_nc(T.g + o) : z;
      mv[j] = in ? ld4(T.m + o) : z;
      vv[j] = in ? ld4(T.v + o) : z;
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int64_t n = r0 + i0 + j;
      const bool in = kin && n < T.N;
      adamw_elem(pv[j].x, gv[j].x, mv[j].x, vv[j].x, P);
      adamw_elem(pv[j].y, gv[j].y, mv[j].y, vv[j].y, P);
      adamw_elem(pv[j].z, gv[j].z, mv[j].z, vv[j].z, P);
      adamw_elem(pv[j].w, gv[j].w, mv[j].w, vv[j].w, P);
      wb[i0 + j][0] = in ? bf16x2_bits(pv[j].x, pv[j].y) : 0u;
      wb[i0 + j][1] = in ? bf16x2_bits(pv[j].z, pv[j].w) : 0u;
      if (in) {
        const int64_t o = n * T.K + k;
        *reinterpret_cast<float4 *>(T.p + o) = pv[j];
        *reinterpret_cast<float4 *>(T.m + o) = mv[j];
        *reinterpret_cast<float4 *>(T.v + o) = vv[j];
        if (T.w != nullptr) *reinterpret_cast<uint2 *>(T.w + o) = make_uint2(wb[i0 + j][0], wb[i0 + j][1]);
      }
      const uint32_t a = __vmaxu2(wb[i0 + j][0] & 0x7FFF7FFFu, wb[i0 + j][1] & 0x7FFF7FFFu);
      amax = max(amax, max(a & 0xFFFFu, a >> 16));
    }
  }
  amax = __reduce_max_sync(0xffffffffu, amax);
  if (lane == 0) red[warp] = amax;
  __syncthreads();
  amax = red[0];
#pragma unroll
  for (int w = 1; w < 8; ++w) amax = max(amax, red[w]);
  const TileScale ts = tile_scale<MODE>(bits_to_amax(amax));
  if (fast_tile<MODE>(ts)) {
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const int64_t n = r0 + i;
      if (kin && n < T.N)
        *reinterpret_cast<uint32_t *>(T.q + n * T.K + k) = encode4<MODE, true>(wb[i][0], wb[i][1], ts);
    }
  } else {
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const int64_t n = r0 + i;
      if (kin && n < T.N)
        *reinterpret_cast<uint32_t *>(T.q + n * T.K + k) = encode4<MODE>(wb[i][0], wb[i][1], ts);
    }
  }
  if (threadIdx.x == 0) T.s[nb * T.KB + kb] = ts.s;
  __syncthreads();  // red[] is reused by the next tile
}

template <int MODE>
__global__ void __launch_bounds__(256, 2) adamw_recal_kernel(const __grid_constant__ OptParams P) {
  __shared__ uint32_t red[8];
  for (int64_t tile = blockIdx.x; tile < P.total; tile += gridDim.x) {
    int lo = 0, hi = P.n - 1;  // last tensor whose first tile is <= tile
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (P.t[mid].tile_begin <= tile) lo = mid;
      else hi = mid - 1;
    }
    const OptTensor &T = P.t[lo];
    const int64_t local = tile - T.tile_begin;
    const int64_t nb = local / T.KB, kb = local - nb * T.KB;
    adamw_tile<MODE>(T, P, nb, kb, red);
  }
}

int g_opt_blocks_per_sm[2] = {0, 0};

}  // namespace

fp8bq_status launch_adamw_recalibrate(const fp8bq_adamw_desc *descs, int n, const fp8bq_adamw_config *cfg, int mode,
                                      cudaStream_t stream) {
  const int mi = mode == FP8BQ_SCALE_FP32 ? 0 : 1;
  if (g_opt_blocks_per_sm[mi] == 0) {
    int b = 0;
    cudaError_t e = mode == FP8BQ_SCALE_FP32
                        ? cudaOccupancyMaxActiveBlocksPerMultiprocessor(&b, adamw_recal_kernel<FP8BQ_SCALE_FP32>, 256, 0)
                        : cudaOccupancyMaxActiveBlocksPerMultiprocessor(&b, adamw_recal_kernel<FP8BQ_SCALE_POW2>, 256, 0);
    if (e != cudaSuccess) return cuda_fail(e, "occupancy(adamw_recalibrate)");
    g_opt_blocks_per_sm[mi] = std::max(1, b);
  }
  const int64_t resident = (int64_t)num_sms() * g_opt_blocks_per_sm[mi];
  OptParams P;
  P.lr = cfg->lr;
  P.b1 = cfg->beta1;
  P.b2 = cfg->beta2;
  P.eps = cfg->eps;
  P.wd = cfg->weight_decay;
  P.c1 = 1.0f - cfg->beta1;
  P.c2 = 1.0f - cfg->beta2;
  P.bc1 = (float)(1.0 - pow((double)cfg->beta1, (double)cfg->step));
  P.bc2 = (float)(1.0 - pow((double)cfg->beta2, (double)cfg->step));
  for (int base = 0; base < n; base += kMaxOptDescs) {
    P.n = 0;
    P.total = 0;
    for (int i = base; i < n && i < base + kMaxOptDescs; ++i) {
      const fp8bq_adamw_desc &d = descs[i];
      if (d.N == 0 || d.K == 0) continue;
      OptTensor &t = P.t[P.n++];
      t.p = d.param;
      t.g = d.grad;
      t.m = d.exp_avg;
      t.v = d.exp_avg_sq;
      t.w = static_cast<uint16_t *>(d.w);
      t.q = d.q;
      t.s = d.s;
      t.N = d.N;
      t.K = d.K;
      t.KB = (int32_t)((d.K + 127) / 128);
      t.tile_begin = P.total;
      P.total += ((d.N + 127) / 128) * t.KB;
    }
    if (P.n == 0) continue;
    const int grid = (int)std::min<int64_t>(P.total, resident);
    if (mode == FP8BQ_SCALE_FP32) adamw_recal_kernel<FP8BQ_SCALE_FP32><<<grid, 256, 0, stream>>>(P);
    else adamw_recal_kernel<FP8BQ_SCALE_POW2><<<grid, 256, 0, stream>>>(P);
    fp8bq_status st = check_launch("adamw_recalibrate");
    if (st != FP8BQ_OK) return st;
  }
  return FP8BQ_OK;
}

}  // namespace fp8bq
