// Decode attention over an FP8 (E4M3) KV cache, and the append that fills it.
//
// Method: "NVIDIA NeMo RL Achieves 48% Speedup With End-to-End FP8 Precision
// Training", section "Real-world performance gains": an FP8 KV cache and FP8
// attention take the recipe's speedup from the linear layers' 15-25% to about
// 48%.  Every key and value head vector (D = 128) is one 1x128 tile of the
// activation quantization of section "Technical breakthrough": E4M3 codes and
// one scale per vector.
//
// Decode attention is HBM-bound: each query token reads its sequence's whole
// cache (2 x 128 code bytes + 2 x 4 scale bytes per token and key/value head).
// Split over the sequence (flash decoding): block (b, g, split) handles one
// key/value head g of batch entry b over one chunk of tokens, for all G query
// heads that share g (grouped-query attention), so each cached vector is read
// once.  Every warp streams its 32-token steps through two shared-memory
// stages with cp.async (16-byte pieces, each key and value row read as whole
// 128-byte lines), so the next step's bytes are in flight while the current
// one is computed.  Per warp and step:
//   scores   lane l takes token l: its key row from the stage, converted
//            pairwise (e4m3x2 -> f16x2 -> f32), dotted with the G queries
//            (shared memory, broadcast reads) with packed FP32 fma;
//   softmax  running max and sum per head across the warp (online softmax);
//   values   the probabilities go to shared memory; lane l then owns head
//            dimensions 4l .. 4l+3 and reads each token's 4 value bytes from
//            the stage and the token's G probabilities (one broadcast load)
//            and accumulates with packed fma.
// The four warps' partial (max, sum, output) meet in shared memory and the
// block writes one partial per query head; a second kernel merges the splits.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <math.h>

#include <algorithm>

#include "device.cuh"
#include "internal.h"
#include "quant.cuh"

namespace fp8bq {
namespace {

using namespace qdev;

constexpr int kD = 128;           // head dimension = one 1x128 tile
constexpr int kAttnWarps = 4;
constexpr int kTokPerIter = 32;   // tokens per warp iteration
constexpr int kChunkQuantum = kAttnWarps * kTokPerIter;
constexpr int kPart = kD + 4;     // floats per split partial: output [D], max, sum, 2 pad (16-byte rows)

// 4-byte asynchronous copy global -> shared (src_bytes = 0: zero-fill, nothing read).
__device__ __forceinline__ void cp_async_4(void *smem_dst, const void *src, uint32_t src_bytes) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(smem_addr(smem_dst)), "l"(src), "r"(src_bytes)
               : "memory");
}

// Two E4M3 codes (low byte first) -> two floats, exactly.
__device__ __forceinline__ float2 e4m3x2_to_float2(uint16_t c) {
  __half2_raw h = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)c, __NV_E4M3);
  return __half22float2(*reinterpret_cast<__half2 *>(&h));
}

struct AttnArgs {
  const uint16_t *q;    // [B][Hq][D] bf16
  const uint8_t *kq;    // [B][S][Hkv][D]
  const float *ks;      // [B][S][Hkv]
  const uint8_t *vq;
  const float *vs;
  const int32_t *lens;  // [B]
  float *ws;            // [B][Hq][nsplit][kPart]: output [D], max, sum
  int32_t B, Hq, Hkv, S, nsplit, chunk;
  float scale;
};

// Per-warp staging of one 32-token step in shared memory (two such stages per
// warp, double-buffered): key rows padded to 144 bytes so that each lane's
// eight 16-byte reads of its own row are conflict-free, value rows of 128
// bytes, and the 32 tokens' key and value scales.
constexpr int kKPitch = 144;
struct StepStage {
  uint8_t k[kTokPerIter][kKPitch];
  uint8_t v[kTokPerIter][kD];
  float ks[kTokPerIter];
  float vs[kTokPerIter];
};

// Issue the asynchronous copies of the step at token `base` (this lane's
// share: four 16-byte key pieces, four value pieces, one key and one value
// scale).  Tokens at or past t_end are zero-filled.
__device__ __forceinline__ void issue_step(StepStage &st, const uint8_t *kbase, const uint8_t *vbase,
                                           const float *ksb, const float *vsb, int64_t row_stride, int64_t Hkv,
                                           int base, int t_end, int lane) {
  const int c = lane & 7, r = lane >> 3;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int u = 4 * i + r;
    const bool in = base + u < t_end;
    const int64_t off = (int64_t)(in ? base + u : 0) * row_stride + 16 * c;
    cp_async_16(&st.k[u][16 * c], kbase + off, in ? 16u : 0u);
    cp_async_16(&st.v[u][16 * c], vbase + off, in ? 16u : 0u);
  }
  const bool in = base + lane < t_end;
  const int64_t so = (int64_t)(in ? base + lane : 0) * Hkv;
  cp_async_4(&st.ks[lane], ksb + so, in ? 4u : 0u);
  cp_async_4(&st.vs[lane], vsb + so, in ? 4u : 0u);
}

// Sum over the 8 lanes of a lane group (lanes 8k .. 8k+7) of v[0..7],
// reduce-scatter style: afterwards lane l holds the group sum of v[l & 7].
// Seven shuffles instead of the 24 of eight separate reductions.
__device__ __forceinline__ float group8_reduce_scatter(const float (&v)[8], int lane) {
  const bool b2 = lane & 4, b1 = lane & 2, b0 = lane & 1;
  float w[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const float send = b2 ? v[k] : v[k + 4];
    const float keep = b2 ? v[k + 4] : v[k];
    w[k] = keep + __shfl_xor_sync(0xffffffffu, send, 4);
  }
  float x[2];
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    const float send = b1 ? w[k] : w[k + 2];
    const float keep = b1 ? w[k + 2] : w[k];
    x[k] = keep + __shfl_xor_sync(0xffffffffu, send, 2);
  }
  const float send = b0 ? x[0] : x[1];
  const float keep = b0 ? x[1] : x[0];
  return keep + __shfl_xor_sync(0xffffffffu, send, 1);
}

template <int G>
__global__ void __launch_bounds__(kAttnWarps * 32) decode_attn_kernel(const AttnArgs a) {
  extern __shared__ __align__(16) uint8_t attn_smem[];
  StepStage *stages = reinterpret_cast<StepStage *>(attn_smem);  // [kAttnWarps][2]
  float(*qs)[kD] = reinterpret_cast<float(*)[kD]>(attn_smem + sizeof(StepStage) * 2 * kAttnWarps);
  float(*ps)[kTokPerIter][G] = reinterpret_cast<float(*)[kTokPerIter][G]>(qs + G);
  __shared__ float red_m[kAttnWarps][G], red_l[kAttnWarps][G];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int bg = blockIdx.x, split = blockIdx.y;
  const int b = bg / a.Hkv, g = bg - b * a.Hkv;
  const int h0 = g * G;
  const int L = min(max(a.lens[b], 0), a.S);
  const int t_begin = split * a.chunk, t_end = min(t_begin + a.chunk, L);

  for (int i = threadIdx.x; i < G * kD; i += blockDim.x) {
    const int j = i / kD, d = i - j * kD;
    qs[j][d] = __uint_as_float((uint32_t)a.q[((int64_t)b * a.Hq + h0 + j) * kD + d] << 16);
  }
  __syncthreads();

  // G <= 4: lane (grp = lane >> 3, dg = lane & 7) scores token 4 i + grp of
  // step i = 0..7 over head dimensions [16 dg, +16), with its 16 query
  // dimensions of each head held in registers; a reduce-scatter across each
  // 8-lane group then leaves lane l the score of token 4 (l & 7) + (l >> 3).
  // G = 8: lane l scores token l over all 128 dimensions, queries read from
  // shared memory.
  constexpr bool kQReg = G <= 4;
  const int dg = lane & 7, grp = lane >> 3;
  float2 qr[kQReg ? G : 1][8];
  if constexpr (kQReg) {
#pragma unroll
    for (int j = 0; j < G; ++j)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float4 qv = *reinterpret_cast<const float4 *>(&qs[j][dg * 16 + 4 * e]);
        qr[j][2 * e] = make_float2(qv.x, qv.y);
        qr[j][2 * e + 1] = make_float2(qv.z, qv.w);
      }
  }
  const int my_u = kQReg ? 4 * dg + grp : lane;  // the token whose score this lane ends up with

  float m[G], l[G];
  float2 o[G][2];  // dimensions 4 lane .. 4 lane + 3
#pragma unroll
  for (int j = 0; j < G; ++j) {
    m[j] = -INFINITY;
    l[j] = 0.f;
    o[j][0] = o[j][1] = make_float2(0.f, 0.f);
  }
  const int64_t row_stride = (int64_t)a.Hkv * kD;  // bytes between tokens
  const uint8_t *kbase = a.kq + ((int64_t)b * a.S * a.Hkv + g) * kD;
  const uint8_t *vbase = a.vq + ((int64_t)b * a.S * a.Hkv + g) * kD;
  const float *ksb = a.ks + (int64_t)b * a.S * a.Hkv + g;
  const float *vsb = a.vs + (int64_t)b * a.S * a.Hkv + g;
  StepStage *my = stages + 2 * warp;

  int base = t_begin + warp * kTokPerIter;
  if (base < t_end) issue_step(my[0], kbase, vbase, ksb, vsb, row_stride, a.Hkv, base, t_end, lane);
  cp_async_commit();
  for (int it = 0; base < t_end; ++it, base += kAttnWarps * kTokPerIter) {
    StepStage &st = my[it & 1];
    const int next = base + kAttnWarps * kTokPerIter;
    if (next < t_end) issue_step(my[(it + 1) & 1], kbase, vbase, ksb, vsb, row_stride, a.Hkv, next, t_end, lane);
    cp_async_commit();
    cp_async_wait<1>();  // this lane's copies of the current step have landed
    __syncwarp();        // ... and every other lane's
    // ---- scores
    const bool valid = base + my_u < t_end;
    float sc[G];
    if constexpr (kQReg) {
      float part[G][8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const uint4 kv = *reinterpret_cast<const uint4 *>(&st.k[4 * i + grp][16 * dg]);
        const uint32_t w4[4] = {kv.x, kv.y, kv.z, kv.w};
        float2 kf[8];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          kf[2 * c] = e4m3x2_to_float2((uint16_t)(w4[c] & 0xFFFFu));
          kf[2 * c + 1] = e4m3x2_to_float2((uint16_t)(w4[c] >> 16));
        }
#pragma unroll
        for (int j = 0; j < G; ++j) {
          float2 acc = __fmul2_rn(kf[0], qr[j][0]);
#pragma unroll
          for (int e = 1; e < 8; ++e) acc = __ffma2_rn(kf[e], qr[j][e], acc);
          part[j][i] = acc.x + acc.y;
        }
      }
#pragma unroll
      for (int j = 0; j < G; ++j) sc[j] = group8_reduce_scatter(part[j], lane);
    } else {
      float2 acc[G];
#pragma unroll
      for (int j = 0; j < G; ++j) acc[j] = make_float2(0.f, 0.f);
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        const uint4 kv = *reinterpret_cast<const uint4 *>(&st.k[lane][16 * c]);
        const uint32_t w4[4] = {kv.x, kv.y, kv.z, kv.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float2 k01 = e4m3x2_to_float2((uint16_t)(w4[i] & 0xFFFFu));
          const float2 k23 = e4m3x2_to_float2((uint16_t)(w4[i] >> 16));
          const int d = c * 16 + i * 4;
#pragma unroll
          for (int j = 0; j < G; ++j) {
            const float4 qv = *reinterpret_cast<const float4 *>(&qs[j][d]);
            acc[j] = __ffma2_rn(k01, make_float2(qv.x, qv.y), acc[j]);
            acc[j] = __ffma2_rn(k23, make_float2(qv.z, qv.w), acc[j]);
          }
        }
      }
#pragma unroll
      for (int j = 0; j < G; ++j) sc[j] = acc[j].x + acc[j].y;
    }
    const float kscale = st.ks[my_u], vscale = st.vs[my_u];
    // ---- online softmax across the warp's 32 tokens
    float p[G];
#pragma unroll
    for (int j = 0; j < G; ++j) {
      const float s = valid ? sc[j] * kscale * a.scale : -INFINITY;
      float mt = s;
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, off));
      const float mn = fmaxf(m[j], mt);  // finite: token base is valid
      const float alpha = expf(m[j] - mn);
      const float e = valid ? expf(s - mn) : 0.f;
      float sum = e;
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
      l[j] = l[j] * alpha + sum;
      m[j] = mn;
      o[j][0] = make_float2(o[j][0].x * alpha, o[j][0].y * alpha);
      o[j][1] = make_float2(o[j][1].x * alpha, o[j][1].y * alpha);
      p[j] = e * vscale;  // the value scale rides with the probability
    }
#pragma unroll
    for (int j = 0; j < G; ++j) ps[warp][my_u][j] = p[j];
    __syncwarp();
    // ---- values: lane = 4 head dimensions
    const int n = min(kTokPerIter, t_end - base);
    for (int u = 0; u < n; ++u) {
      const uint32_t vw = *reinterpret_cast<const uint32_t *>(&st.v[u][4 * lane]);
      const float2 v01 = e4m3x2_to_float2((uint16_t)(vw & 0xFFFFu));
      const float2 v23 = e4m3x2_to_float2((uint16_t)(vw >> 16));
#pragma unroll
      for (int j = 0; j < G; ++j) {
        const float pj = ps[warp][u][j];
        o[j][0] = __ffma2_rn(v01, make_float2(pj, pj), o[j][0]);
        o[j][1] = __ffma2_rn(v23, make_float2(pj, pj), o[j][1]);
      }
    }
    __syncwarp();  // the stage and ps are rewritten by later steps
  }
  cp_async_wait<0>();

  // ---- merge the four warps (the stage buffers are free now: reuse them for
  // the partial outputs), write this split's partial per query head
  __syncthreads();
  float(*red_o)[G][kD] = reinterpret_cast<float(*)[G][kD]>(attn_smem);
#pragma unroll
  for (int j = 0; j < G; ++j) {
    if (lane == 0) {
      red_m[warp][j] = m[j];
      red_l[warp][j] = l[j];
    }
    *reinterpret_cast<float4 *>(&red_o[warp][j][4 * lane]) = make_float4(o[j][0].x, o[j][0].y, o[j][1].x, o[j][1].y);
  }
  __syncthreads();
  for (int i = threadIdx.x; i < G * (kD + 2); i += blockDim.x) {
    const int j = i / (kD + 2), c = i - j * (kD + 2);
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kAttnWarps; ++w) M = fmaxf(M, red_m[w][j]);
    float val = 0.f;
    if (c < kD) {
      if (M != -INFINITY)
#pragma unroll
        for (int w = 0; w < kAttnWarps; ++w)
          if (red_m[w][j] != -INFINITY) val += red_o[w][j][c] * expf(red_m[w][j] - M);
    } else if (c == kD) {
      val = M;
    } else if (M != -INFINITY) {
#pragma unroll
      for (int w = 0; w < kAttnWarps; ++w)
        if (red_m[w][j] != -INFINITY) val += red_l[w][j] * expf(red_m[w][j] - M);
    }
    a.ws[(((int64_t)b * a.Hq + h0 + j) * a.nsplit + split) * kPart + c] = val;
  }
}

template <int G>
constexpr int attn_smem_bytes() {
  return (int)(sizeof(StepStage) * 2 * kAttnWarps + sizeof(float) * G * kD + sizeof(float) * kAttnWarps * kTokPerIter * G);
}
static_assert(sizeof(StepStage) * 2 * kAttnWarps >= sizeof(float) * kAttnWarps * 8 * kD, "partial outputs fit the stages");

// One warp per (b, query head): merge the splits and round to bf16.  The
// split maxima are read by the lanes in parallel; the weighted sum over the
// splits keeps eight 16-byte loads in flight per lane.
__global__ void __launch_bounds__(128) decode_attn_combine_kernel(const float *__restrict__ ws, int32_t BH,
                                                                  int32_t nsplit, uint16_t *__restrict__ out) {
  const int bh = blockIdx.x * 4 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (bh >= BH) return;
  const float *p = ws + (int64_t)bh * nsplit * kPart;
  float M = -INFINITY;
  for (int s = lane; s < nsplit; s += 32) M = fmaxf(M, p[s * kPart + kD]);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  float den = 0.f;
  if (M != -INFINITY) {
    for (int s0 = 0; s0 < nsplit; s0 += 8) {
      float4 v[8];
      float ms[8], ls[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const int s = s0 + k;
        const bool in = s < nsplit;
        v[k] = in ? *reinterpret_cast<const float4 *>(p + s * kPart + 4 * lane) : make_float4(0.f, 0.f, 0.f, 0.f);
        ms[k] = in ? p[s * kPart + kD] : -INFINITY;
        ls[k] = in ? p[s * kPart + kD + 1] : 0.f;
      }
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        if (ms[k] == -INFINITY) continue;
        const float w = expf(ms[k] - M);
        acc.x += w * v[k].x;
        acc.y += w * v[k].y;
        acc.z += w * v[k].z;
        acc.w += w * v[k].w;
        den += w * ls[k];
      }
    }
  }
  const float r = den > 0.f ? 1.f / den : 0.f;
  __nv_bfloat162 lo = __floats2bfloat162_rn(acc.x * r, acc.y * r);
  __nv_bfloat162 hi = __floats2bfloat162_rn(acc.z * r, acc.w * r);
  uint2 pk;
  pk.x = *reinterpret_cast<uint32_t *>(&lo);
  pk.y = *reinterpret_cast<uint32_t *>(&hi);
  *reinterpret_cast<uint2 *>(out + (int64_t)bh * kD + 4 * lane) = pk;
}

// ---------------------------------------------------------------------------
// KV append: one warp quantizes one new key or value head vector (one 1x128
// tile: 4 elements per lane, warp-wide amax) and writes it at its position.
// ---------------------------------------------------------------------------
template <int MODE>
__global__ void __launch_bounds__(256) kv_append_kernel(const uint16_t *__restrict__ k_new,
                                                        const uint16_t *__restrict__ v_new,
                                                        const int32_t *__restrict__ pos, uint8_t *kq, float *ks,
                                                        uint8_t *vq, float *vs, int32_t B, int32_t Hkv, int32_t S) {
  const int row = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (row >= 2 * B * Hkv) return;
  const int which = row / (B * Hkv), bg = row - which * B * Hkv;  // 0: key, 1: value
  const int b = bg / Hkv, g = bg - b * Hkv;
  const int t = pos[b];
  if (t < 0 || t >= S) return;  // outside the cache: nothing is written
  const uint16_t *src = (which ? v_new : k_new) + (int64_t)bg * kD;
  const uint2 x = *reinterpret_cast<const uint2 *>(src + 4 * lane);
  uint32_t am = max(max(x.x & 0x7FFFu, (x.x >> 16) & 0x7FFFu), max(x.y & 0x7FFFu, (x.y >> 16) & 0x7FFFu));
  am = __reduce_max_sync(0xffffffffu, am);
  const TileScale ts = tile_scale<MODE>(bits_to_amax(am));
  const int64_t slot = ((int64_t)b * S + t) * Hkv + g;
  uint8_t *dst = (which ? vq : kq) + slot * kD;
  *reinterpret_cast<uint32_t *>(dst + 4 * lane) = encode4<MODE>(x.x, x.y, ts);
  if (lane == 0) (which ? vs : ks)[slot] = ts.s;
}

int g_attn_ready = 0;

// The stages need more than the default 48 KB of dynamic shared memory.
fp8bq_status prepare_attention() {
  if (g_attn_ready) return FP8BQ_OK;
  cudaError_t e = cudaFuncSetAttribute(decode_attn_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       attn_smem_bytes<1>());
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(decode_attn_kernel<2>, cudaFuncAttributeMaxDynamicSharedMemorySize, attn_smem_bytes<2>());
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(decode_attn_kernel<4>, cudaFuncAttributeMaxDynamicSharedMemorySize, attn_smem_bytes<4>());
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(decode_attn_kernel<8>, cudaFuncAttributeMaxDynamicSharedMemorySize, attn_smem_bytes<8>());
  if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(decode_attention)");
  g_attn_ready = 1;
  return FP8BQ_OK;
}

// Splits of the sequence: about eight blocks per SM in all, never chunks
// shorter than four passes of a block (a block's fixed costs -- the queries,
// the pipeline fill, the merge -- stay small against its streaming).
int attn_splits(int64_t B, int64_t Hkv, int64_t S) {
  const int64_t max_splits = std::max<int64_t>(1, (S + 4 * kChunkQuantum - 1) / (4 * kChunkQuantum));
  const int64_t want = std::max<int64_t>(1, (8 * (int64_t)num_sms() + B * Hkv - 1) / std::max<int64_t>(B * Hkv, 1));
  return (int)std::min(max_splits, want);
}

}  // namespace

size_t decode_attention_workspace_size(int64_t B, int64_t Hq, int64_t Hkv, int64_t S) {
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || S <= 0) return 0;
  return (size_t)B * Hq * attn_splits(B, Hkv, S) * kPart * sizeof(float);
}

fp8bq_status launch_decode_attention(const void *q, const uint8_t *kq, const float *ks, const uint8_t *vq,
                                     const float *vs, const int32_t *lens, int64_t B, int64_t Hq, int64_t Hkv,
                                     int64_t S, float scale, void *o, void *ws, size_t ws_bytes,
                                     cudaStream_t stream) {
  if (S == 0) {  // nothing cached: every output is 0
    cudaError_t e = cudaMemsetAsync(o, 0, (size_t)B * Hq * kD * 2, stream);
    return e == cudaSuccess ? FP8BQ_OK : cuda_fail(e, "memset(o)");
  }
  if (decode_attention_workspace_size(B, Hq, Hkv, S) > ws_bytes) return FP8BQ_ERR_WORKSPACE;
  AttnArgs a;
  a.q = static_cast<const uint16_t *>(q);
  a.kq = kq;
  a.ks = ks;
  a.vq = vq;
  a.vs = vs;
  a.lens = lens;
  a.ws = static_cast<float *>(ws);
  a.B = (int32_t)B;
  a.Hq = (int32_t)Hq;
  a.Hkv = (int32_t)Hkv;
  a.S = (int32_t)S;
  a.nsplit = attn_splits(B, Hkv, S);
  const int64_t chunk = (S + a.nsplit - 1) / a.nsplit;
  a.chunk = (int32_t)((chunk + kChunkQuantum - 1) / kChunkQuantum * kChunkQuantum);
  a.scale = scale;
  const dim3 grid((unsigned)(B * Hkv), (unsigned)a.nsplit);
  fp8bq_status st = prepare_attention();
  if (st != FP8BQ_OK) return st;
  switch (Hq / Hkv) {
    case 1: decode_attn_kernel<1><<<grid, kAttnWarps * 32, attn_smem_bytes<1>(), stream>>>(a); break;
    case 2: decode_attn_kernel<2><<<grid, kAttnWarps * 32, attn_smem_bytes<2>(), stream>>>(a); break;
    case 4: decode_attn_kernel<4><<<grid, kAttnWarps * 32, attn_smem_bytes<4>(), stream>>>(a); break;
    case 8: decode_attn_kernel<8><<<grid, kAttnWarps * 32, attn_smem_bytes<8>(), stream>>>(a); break;
    default: return FP8BQ_ERR_UNSUPPORTED;
  }
  st = check_launch("decode_attention");
  if (st != FP8BQ_OK) return st;
  const int32_t BH = (int32_t)(B * Hq);
  decode_attn_combine_kernel<<<(unsigned)((BH + 3) / 4), 128, 0, stream>>>(a.ws, BH, a.nsplit,
                                                                           static_cast<uint16_t *>(o));
  return check_launch("decode_attention(combine)");
}

fp8bq_status launch_kv_append(const void *k_new, const void *v_new, const int32_t *pos, uint8_t *kq, float *ks,
                              uint8_t *vq, float *vs, int64_t B, int64_t Hkv, int64_t S, int mode,
                              cudaStream_t stream) {
  const int64_t rows = 2 * B * Hkv;
  const unsigned grid = (unsigned)((rows + 7) / 8);
  const uint16_t *k = static_cast<const uint16_t *>(k_new), *v = static_cast<const uint16_t *>(v_new);
  if (mode == FP8BQ_SCALE_FP32)
    kv_append_kernel<FP8BQ_SCALE_FP32><<<grid, 256, 0, stream>>>(k, v, pos, kq, ks, vq, vs, (int32_t)B, (int32_t)Hkv,
                                                                  (int32_t)S);
  else
    kv_append_kernel<FP8BQ_SCALE_POW2><<<grid, 256, 0, stream>>>(k, v, pos, kq, ks, vq, vs, (int32_t)B, (int32_t)Hkv,
                                                                  (int32_t)S);
  return check_launch("kv_append");
}

}  // namespace fp8bq
