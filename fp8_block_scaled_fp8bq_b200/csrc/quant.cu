// E4M3 quantization kernels: 1x128 activation tiles, 128x128 weight tiles and
// the multi-tensor per-step recalibration.
//
// Method: "NVIDIA NeMo RL Achieves 48% Speedup With End-to-End FP8 Precision
// Training", section "Technical breakthrough" (block-wise E4M3; weights
// 128x128, activations 1x128) and section "Real-world performance gains"
// (scales recalibrated after every training step); power-of-2 scales from
// section "Why this matters for AI economics".
//
// These kernels are HBM-bound (2 bytes read, 1 byte written per element):
// 16-byte vector loads of bf16, an integer max over |x| bit patterns (for
// non-negative bf16 the bit order is the value order, so the amax is exact),
// a correctly rounded quotient per element (one multiply and two fmas with FP32
// scales, one multiply by the exact reciprocal with POW2 scales; see
// tile_scale), and the hardware E4M3 conversion with
// round-to-nearest-even and saturation (cvt.rn.satfinite.e4m3x2.f32).
#include <algorithm>

#include "device.cuh"
#include "internal.h"
#include <cuda_bf16.h>

#include "quant.cuh"

namespace fp8bq {
namespace {

using namespace qdev;

// ---------------------------------------------------------------------------
// Weight quantization / recalibration, 128x128 tiles
// ---------------------------------------------------------------------------
constexpr int kMaxDescs = 128;

struct TileTensor {
  const uint16_t *w;
  uint8_t *q;
  float *s;
  int64_t N, K, ldw, ldq;
  int64_t tile_begin;  // global id of this tensor's first tile
  int32_t KB;          // tiles along K
  int32_t vec;         // 16-byte vector path allowed
};

struct RecalParams {
  int32_t n;
  int64_t total;  // tiles over all tensors
  TileTensor t[kMaxDescs];
};

// One 128x128 tile, 256 threads: thread t holds rows (t>>4) + 16 i, i = 0..7, of
// the 16-byte column chunk (t & 15).  The tile stays in registers between the
// amax and the encode, so it is read from HBM once.
template <int MODE>
__device__ __forceinline__ void quant_tile_vec(const TileTensor &T, int64_t nb, int64_t kb, uint32_t *red) {
  const int t = threadIdx.x;
  const int c = t & 15, r0 = t >> 4;
  const int64_t k = kb * 128 + c * 8;
  const bool kin = k < T.K;
  uint4 v[8];
  uint32_t m = 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int64_t n = nb * 128 + r0 + 16 * i;
    v[i] = (kin && n < T.N) ? ld_nc_v4(T.w + n * T.ldw + k) : make_uint4(0, 0, 0, 0);
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) m = max(m, absmax_bits8(v[i]));
  m = __reduce_max_sync(0xffffffffu, m);
  if ((t & 31) == 0) red[t >> 5] = m;
  __syncthreads();
  m = red[0];
#pragma unroll
  for (int w = 1; w < 8; ++w) m = max(m, red[w]);
  const TileScale ts = tile_scale<MODE>(bits_to_amax(m));
  if (fast_tile<MODE>(ts)) {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int64_t n = nb * 128 + r0 + 16 * i;
      if (kin && n < T.N) *reinterpret_cast<uint2 *>(T.q + n * T.ldq + k) = encode8<MODE, true>(v[i], ts);
    }
  } else {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int64_t n = nb * 128 + r0 + 16 * i;
      if (kin && n < T.N) *reinterpret_cast<uint2 *>(T.q + n * T.ldq + k) = encode8<MODE>(v[i], ts);
    }
  }
  if (t == 0) T.s[nb * T.KB + kb] = ts.s;
  __syncthreads();  // red[] is reused by the next tile
}

// Any alignment: two passes over the (cached) tile with scalar accesses.
template <int MODE>
__device__ __forceinline__ void quant_tile_scalar(const TileTensor &T, int64_t nb, int64_t kb, uint32_t *red) {
  const int t = threadIdx.x;
  uint32_t m = 0;
  for (int idx = t; idx < 128 * 128; idx += 256) {
    const int64_t n = nb * 128 + (idx >> 7), k = kb * 128 + (idx & 127);
    if (n < T.N && k < T.K) m = max(m, (uint32_t)(T.w[n * T.ldw + k] & 0x7FFFu));
  }
  m = __reduce_max_sync(0xffffffffu, m);
  if ((t & 31) == 0) red[t >> 5] = m;
  __syncthreads();
  m = red[0];
#pragma unroll
  for (int w = 1; w < 8; ++w) m = max(m, red[w]);
  const TileScale ts = tile_scale<MODE>(bits_to_amax(m));
  for (int idx = t; idx < 128 * 128; idx += 256) {
    const int64_t n = nb * 128 + (idx >> 7), k = kb * 128 + (idx & 127);
    if (n < T.N && k < T.K) {
      const float f = __uint_as_float((uint32_t)T.w[n * T.ldw + k] << 16);
      T.q[n * T.ldq + k] = (uint8_t)(e4m3x2(quotient<MODE>(f, ts), 0.f) & 0xFFu);
    }
  }
  if (t == 0) T.s[nb * T.KB + kb] = ts.s;
  __syncthreads();
}

// The tensor holding global tile `tile`: the last one whose first tile is <= tile.
__device__ __forceinline__ int tensor_of(const RecalParams &p, int64_t tile) {
  int lo = 0, hi = p.n - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (p.t[mid].tile_begin <= tile) lo = mid;
    else hi = mid - 1;
  }
  return lo;
}

// Vector path, software pipelined through shared memory: every thread copies
// its own eight 16-byte chunks of the next tile with cp.async while it encodes
// the current one, so a block always has a tile's loads in flight.  A thread
// reads back only the chunks it copied itself (no block barrier is needed for
// the data; the one per tile is for the amax).
__device__ __forceinline__ void issue_tile_copy(const TileTensor &T, int64_t nb, int64_t kb, uint4 *buf) {
  const int t = threadIdx.x;
  const int c = t & 15, r0 = t >> 4;
  const int64_t k = kb * 128 + c * 8;
  const bool kin = k < T.K;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int64_t n = nb * 128 + r0 + 16 * i;
    const bool in = kin && n < T.N;
    cp_async_16(buf + i * 256 + t, in ? static_cast<const void *>(T.w + n * T.ldw + k) : static_cast<const void *>(T.w),
                in ? 16u : 0u);
  }
}

// max |x| of 8 bf16 as a bf16 bit pattern, by packed bf16 maxima of the
// absolute values (exact for finite values).
__device__ __forceinline__ uint32_t absmax_bits8_bf16(uint4 v) {
  auto pair = [](uint32_t a, uint32_t b) {
    const __nv_bfloat162 m = __hmax2(__habs2(*reinterpret_cast<const __nv_bfloat162 *>(&a)),
                                     __habs2(*reinterpret_cast<const __nv_bfloat162 *>(&b)));
    return *reinterpret_cast<const uint32_t *>(&m);
  };
  const uint32_t m = pair(pair(v.x, v.y), pair(v.z, v.w));
  return max(m & 0xFFFFu, m >> 16);
}

template <int MODE>
__global__ void __launch_bounds__(256, 3) recalibrate_pipelined_kernel(const __grid_constant__ RecalParams p) {
  __shared__ uint32_t red[8];
  extern __shared__ uint4 stage_buf[];  // 2 x [8][256] 16-byte chunks (64 KB)
  int64_t tile = blockIdx.x;
  if (tile >= p.total) return;
  int ti = tensor_of(p, tile);
  int64_t local = tile - p.t[ti].tile_begin;
  int64_t nb = local / p.t[ti].KB, kb = local - nb * p.t[ti].KB;
  issue_tile_copy(p.t[ti], nb, kb, stage_buf);
  cp_async_commit();
  for (int it = 0;; ++it) {
    uint4 *cur = stage_buf + (it & 1) * 2048;
    const int64_t next = tile + gridDim.x;
    int tn = ti;
    int64_t nbn = 0, kbn = 0;
    if (next < p.total) {
      tn = tensor_of(p, next);
      const int64_t ln = next - p.t[tn].tile_begin;
      nbn = ln / p.t[tn].KB;
      kbn = ln - nbn * p.t[tn].KB;
      issue_tile_copy(p.t[tn], nbn, kbn, stage_buf + ((it + 1) & 1) * 2048);
    }
    cp_async_commit();
    cp_async_wait<1>();  // this thread's copies of the current tile have landed
    uint4 v[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = cur[i * 256 + threadIdx.x];
    uint32_t m = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) m = max(m, absmax_bits8_bf16(v[i]));
    m = __reduce_max_sync(0xffffffffu, m);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
    __syncthreads();
    m = red[0];
#pragma unroll
    for (int w = 1; w < 8; ++w) m = max(m, red[w]);
    const TileScale ts = tile_scale<MODE>(bits_to_amax(m));
    const TileTensor &T = p.t[ti];
    const int c = threadIdx.x & 15, r0 = threadIdx.x >> 4;
    const int64_t k = kb * 128 + c * 8;
    if (k < T.K) {
      if (fast_tile<MODE>(ts)) {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int64_t n = nb * 128 + r0 + 16 * i;
          if (n < T.N) *reinterpret_cast<uint2 *>(T.q + n * T.ldq + k) = encode8<MODE, true>(v[i], ts);
        }
      } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int64_t n = nb * 128 + r0 + 16 * i;
          if (n < T.N) *reinterpret_cast<uint2 *>(T.q + n * T.ldq + k) = encode8<MODE>(v[i], ts);
        }
      }
    }
    if (threadIdx.x == 0) T.s[nb * T.KB + kb] = ts.s;
    __syncthreads();  // red[] is reused by the next tile
    if (next >= p.total) break;
    tile = next;
    ti = tn;
    nb = nbn;
    kb = kbn;
  }
  cp_async_wait<0>();
}

template <int MODE>
__global__ void __launch_bounds__(256, 3) recalibrate_kernel(const __grid_constant__ RecalParams p) {
  __shared__ uint32_t red[8];
  for (int64_t tile = blockIdx.x; tile < p.total; tile += gridDim.x) {
    const TileTensor &T = p.t[tensor_of(p, tile)];
    const int64_t local = tile - T.tile_begin;
    const int64_t nb = local / T.KB, kb = local - nb * T.KB;
    if (T.vec) quant_tile_vec<MODE>(T, nb, kb, red);
    else quant_tile_scalar<MODE>(T, nb, kb, red);
  }
}

__global__ void __launch_bounds__(256) encode_kernel(const float *__restrict__ x, int64_t n, uint8_t *__restrict__ q) {
  const int64_t stride = (int64_t)gridDim.x * blockDim.x * 4;
  for (int64_t i = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) * 4; i < n; i += stride) {
    if (i + 4 <= n) {
      const float4 v = *reinterpret_cast<const float4 *>(x + i);
      *reinterpret_cast<uint32_t *>(q + i) = e4m3x2(v.x, v.y) | (e4m3x2(v.z, v.w) << 16);
    } else {
      for (int64_t j = i; j < n; ++j) q[j] = (uint8_t)(e4m3x2(x[j], 0.f) & 0xFFu);
    }
  }
}

bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

int g_recal_blocks_per_sm[2] = {0, 0};

constexpr int kPipeSmem = 2 * 8 * 256 * 16;  // two stages of a 128x128 bf16 tile
int g_pipe_blocks_per_sm = 0;

fp8bq_status prepare_pipelined() {
  if (g_pipe_blocks_per_sm > 0) return FP8BQ_OK;
  cudaError_t e = cudaFuncSetAttribute(recalibrate_pipelined_kernel<FP8BQ_SCALE_FP32>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, kPipeSmem);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(recalibrate_pipelined_kernel<FP8BQ_SCALE_POW2>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             kPipeSmem);
  if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(recalibrate)");
  int b = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&b, recalibrate_pipelined_kernel<FP8BQ_SCALE_FP32>, 256,
                                                    kPipeSmem);
  if (e != cudaSuccess) return cuda_fail(e, "occupancy(recalibrate)");
  g_pipe_blocks_per_sm = std::max(1, b);
  return FP8BQ_OK;
}

}  // namespace

fp8bq_status launch_encode(const float *x, int64_t n, uint8_t *q, cudaStream_t stream) {
  if (n == 0) return FP8BQ_OK;
  const int64_t blocks = std::min<int64_t>((n + 1023) / 1024, (int64_t)num_sms() * 16);
  encode_kernel<<<(unsigned)blocks, 256, 0, stream>>>(x, n, q);
  return check_launch("e4m3_encode");
}

fp8bq_status launch_quant_act(const void *x, int64_t M, int64_t K, int64_t ldx, uint8_t *q, int64_t ldq, float *sa,
                              int64_t ldsa, int mode, cudaStream_t stream) {
  const int64_t KB = (K + 127) / 128;
  if (M == 0 || K == 0) return FP8BQ_OK;
  if (KB > 65535) return FP8BQ_ERR_UNSUPPORTED;
  const uint16_t *xs = static_cast<const uint16_t *>(x);
  const bool vec = aligned(x, 16) && ldx % 8 == 0 && K % 8 == 0 && aligned(q, 8) && ldq % 8 == 0;
  if (vec) {
    dim3 grid((unsigned)((M + 63) / 64), (unsigned)KB);
    if (mode == FP8BQ_SCALE_FP32)
      quant_act_vec_kernel<FP8BQ_SCALE_FP32><<<grid, 256, 0, stream>>>(xs, M, K, ldx, q, ldq, sa, ldsa);
    else
      quant_act_vec_kernel<FP8BQ_SCALE_POW2><<<grid, 256, 0, stream>>>(xs, M, K, ldx, q, ldq, sa, ldsa);
  } else {
    dim3 grid((unsigned)((M + 15) / 16), (unsigned)KB);
    if (mode == FP8BQ_SCALE_FP32)
      quant_act_scalar_kernel<FP8BQ_SCALE_FP32><<<grid, 256, 0, stream>>>(xs, M, K, ldx, q, ldq, sa, ldsa);
    else
      quant_act_scalar_kernel<FP8BQ_SCALE_POW2><<<grid, 256, 0, stream>>>(xs, M, K, ldx, q, ldq, sa, ldsa);
  }
  return check_launch("quant_act");
}

fp8bq_status launch_recalibrate(const fp8bq_weight_desc *descs, int n, int mode, cudaStream_t stream) {
  const int mi = mode == FP8BQ_SCALE_FP32 ? 0 : 1;
  if (g_recal_blocks_per_sm[mi] == 0) {
    int b = 0;
    cudaError_t e = mode == FP8BQ_SCALE_FP32
                        ? cudaOccupancyMaxActiveBlocksPerMultiprocessor(&b, recalibrate_kernel<FP8BQ_SCALE_FP32>, 256, 0)
                        : cudaOccupancyMaxActiveBlocksPerMultiprocessor(&b, recalibrate_kernel<FP8BQ_SCALE_POW2>, 256, 0);
    if (e != cudaSuccess) return cuda_fail(e, "occupancy(recalibrate)");
    g_recal_blocks_per_sm[mi] = std::max(1, b);
  }
  const int64_t resident = (int64_t)num_sms() * g_recal_blocks_per_sm[mi];
  for (int base = 0; base < n; base += kMaxDescs) {
    RecalParams p;
    p.n = 0;
    p.total = 0;
    for (int i = base; i < n && i < base + kMaxDescs; ++i) {
      const fp8bq_weight_desc &d = descs[i];
      if (d.N == 0 || d.K == 0) continue;
      TileTensor &t = p.t[p.n++];
      t.w = static_cast<const uint16_t *>(d.w);
      t.q = d.q;
      t.s = d.s;
      t.N = d.N;
      t.K = d.K;
      t.ldw = d.ldw;
      t.ldq = d.ldq;
      t.KB = (int32_t)((d.K + 127) / 128);
      t.tile_begin = p.total;
      t.vec = aligned(d.w, 16) && d.ldw % 8 == 0 && d.K % 8 == 0 && aligned(d.q, 8) && d.ldq % 8 == 0;
      p.total += ((d.N + 127) / 128) * (int64_t)t.KB;
    }
    if (p.total == 0) continue;
    bool all_vec = true;
    for (int i = 0; i < p.n; ++i) all_vec = all_vec && p.t[i].vec;
    if (all_vec) {
      fp8bq_status st = prepare_pipelined();
      if (st != FP8BQ_OK) return st;
      const unsigned grid = (unsigned)std::min<int64_t>(p.total, (int64_t)num_sms() * g_pipe_blocks_per_sm);
      if (mode == FP8BQ_SCALE_FP32)
        recalibrate_pipelined_kernel<FP8BQ_SCALE_FP32><<<grid, 256, kPipeSmem, stream>>>(p);
      else
        recalibrate_pipelined_kernel<FP8BQ_SCALE_POW2><<<grid, 256, kPipeSmem, stream>>>(p);
    } else {
      const unsigned grid = (unsigned)std::min<int64_t>(p.total, resident);
      if (mode == FP8BQ_SCALE_FP32)
        recalibrate_kernel<FP8BQ_SCALE_FP32><<<grid, 256, 0, stream>>>(p);
      else
        recalibrate_kernel<FP8BQ_SCALE_POW2><<<grid, 256, 0, stream>>>(p);
    }
    fp8bq_status st = check_launch("recalibrate");
    if (st != FP8BQ_OK) return st;
  }
  return FP8BQ_OK;
}

}  // namespace fp8bq
