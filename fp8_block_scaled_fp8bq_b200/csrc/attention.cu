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
// stages with cp.async (16-byte pieces, whole 128-byte key and value rows), so
// the next step's bytes are in flight while the current one is computed.
//
// Both contractions of a step run on the tensor cores (warp-level
// m16n8k16 f16 MMA with FP32 accumulators), so the per-element work left on
// the CUDA cores is the exact E4M3 -> f16 conversion (two codes per
// instruction):
//   scores   S[t][h] = K[t][:] . Q[h][:], tokens as M (two 16-token tiles),
//            the G <= 8 query heads as N (padded to 8), D = 128 as K.  The
//            queries are loaded once as f16 B fragments, each head scaled by
//            a power of two 2^E that puts its largest |q| in [2^14, 2^15)
//            (every bf16 element at most 2^28 below it converts exactly);
//            the key codes of a thread's two token rows are A fragments.
//            The head dimension is permuted inside each MMA (a sum over D
//            does not depend on its order): thread (row group r, column
//            pair c) of k-step s takes head dimensions 32 c + 4 s .. + 3, so
//            it reads 32 contiguous bytes of each of its key rows.
//   softmax  per head, in base 2 (log2 e is folded into the score factor):
//            a running max over all tokens so far, partial sums per thread.
//   values   O^T[d][h] = V^T[d][:] . P^T[:][h], head dimensions as M (8
//            tiles), heads as N, 16 tokens per k-step.  The probability tile
//            of the score accumulators is exactly the transpose of the B
//            fragment the value MMA needs: movmatrix.trans moves it.  The
//            value scale of each token rides on its probability, relative to
//            the largest value scale seen so far (so the weight stays in
//            [0, 1]; the accumulator is rescaled when that largest scale
//            grows, together with the softmax rescale).  Each weight is split
//            into two f16 values (high part + rounded remainder) and the MMA
//            runs on both, so the weights keep about 22 bits.  A thread's
//            value A fragments pair two tokens' codes at one head dimension
//            (byte permutes of its two rows' 16-byte pieces).
// The four warps' partial (max, sum, output) meet in shared memory and the
// block writes one partial per query head; a second kernel merges the splits.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <math.h>
#include <stdint.h>

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
constexpr int kStages = 2;        // per-warp ring of staged steps (kStages - 1 in flight)
constexpr int kPart = kD + 4;     // floats per split partial: output [D], max (log2 units), sum, 2 pad
constexpr float kLog2e = 1.4426950408889634f;

// 4-byte asynchronous copy global -> shared (src_bytes = 0: zero-fill, nothing read).
__device__ __forceinline__ void cp_async_4(void *smem_dst, const void *src, uint32_t src_bytes) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(smem_addr(smem_dst)), "l"(src), "r"(src_bytes)
               : "memory");
}

// Four E4M3 codes (bytes 0..3 of w) -> two f16x2, exactly: lo = (byte 0,
// byte 1), hi = (byte 2, byte 3), the lower byte in the lower half.  The
// 16-bit halves of w are read in place.
__device__ __forceinline__ void e4m3x4_f16(uint32_t w, uint32_t &lo, uint32_t &hi) {
  asm("{\n\t.reg .b16 l, h;\n\tmov.b32 {l, h}, %2;\n\tcvt.rn.f16x2.e4m3x2 %0, l;\n\t"
      "cvt.rn.f16x2.e4m3x2 %1, h;\n\t}"
      : "=r"(lo), "=r"(hi)
      : "r"(w));
}

__device__ __forceinline__ uint32_t f16x2_bits(float lo, float hi) {
  const __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<const uint32_t *>(&h);
}

// D += A . B, m16n8k16, f16 operands, FP32 accumulators.
__device__ __forceinline__ void mma_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                          uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// 2^x (the hardware's approximate base-2 exponential, relative error about
// 2^-22; 2^-inf = +0).
__device__ __forceinline__ float exp2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Transpose of an 8x8 b16 matrix held one row pair per thread.
__device__ __forceinline__ uint32_t movmatrix_trans(uint32_t x) {
  uint32_t r;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(r) : "r"(x));
  return r;
}

struct AttnArgs {
  const uint16_t *q;    // [B][Hq][D] bf16
  const uint8_t *kq;    // [B][S][Hkv][D]
  const float *ks;      // [B][S][Hkv]
  const uint8_t *vq;
  const float *vs;
  const int32_t *lens;  // [B]
  float *ws;            // [B][Hq][nsplit][kPart]: output [D], max (log2 units), sum
  int32_t B, Hq, Hkv, S, nsplit, chunk;
  float scale;
};

// Per-warp staging of one 32-token step in shared memory (two such stages per
// warp, double-buffered).  Rows are padded to 144 bytes: the key reads (row
// group r, 32-byte piece c) and the value reads (rows 2 c .. of a 16-token
// tile, 16-byte piece r) of a quarter warp then fall on distinct banks.
constexpr int kRowPitch = 144;
struct StepStage {
  uint8_t k[kTokPerIter][kRowPitch];
  uint8_t v[kTokPerIter][kRowPitch];
  float ks[kTokPerIter];
  float vs[kTokPerIter];
};

// Issue the asynchronous copies of the step at token `base` (this lane's
// share: four 16-byte key pieces, four value pieces, one key and one value
// scale).  Tokens at or past t_end are zero-filled; a step wholly before
// t_end takes the branch without per-row checks.
__device__ __forceinline__ void issue_step(StepStage &st, const uint8_t *kbase, const uint8_t *vbase,
                                           const float *ksb, const float *vsb, int64_t row_stride, int64_t Hkv,
                                           int base, int t_end, int lane) {
  const int c = lane & 7, r = lane >> 3;
  if (base + kTokPerIter <= t_end) {
    const int64_t off = (int64_t)(base + r) * row_stride + 16 * c;
    const uint8_t *kp = kbase + off, *vp = vbase + off;
    const int64_t step4 = 4 * row_stride;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      cp_async_16(&st.k[4 * i + r][16 * c], kp + i * step4, 16u);
      cp_async_16(&st.v[4 * i + r][16 * c], vp + i * step4, 16u);
    }
    const int64_t so = (int64_t)(base + lane) * Hkv;
    cp_async_4(&st.ks[lane], ksb + so, 4u);
    cp_async_4(&st.vs[lane], vsb + so, 4u);
    return;
  }
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

__device__ __forceinline__ float max_over_row_groups(float x) {
  x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, 4));
  x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, 8));
  return fmaxf(x, __shfl_xor_sync(0xffffffffu, x, 16));
}

__device__ __forceinline__ float sum_over_row_groups(float x) {
  x += __shfl_xor_sync(0xffffffffu, x, 4);
  x += __shfl_xor_sync(0xffffffffu, x, 8);
  return x + __shfl_xor_sync(0xffffffffu, x, 16);
}

// Fragment roles (m16n8k16): lane = 4 r + c, r = row group 0..7, c = column
// pair 0..3.  Score accumulators sc[i][*]: token 16 i + r (elements 0, 1) and
// 16 i + r + 8 (elements 2, 3), heads 2 c and 2 c + 1.  Value accumulators
// o[m][*]: head dimension 16 r + 2 m (elements 0, 1) and 16 r + 2 m + 1
// (elements 2, 3), heads 2 c and 2 c + 1.
template <int G>
__global__ void __launch_bounds__(kAttnWarps * 32) decode_attn_kernel(const AttnArgs a) {
  extern __shared__ __align__(16) uint8_t attn_smem[];
  StepStage *stages = reinterpret_cast<StepStage *>(attn_smem);  // [kAttnWarps][kStages]
  __shared__ float red_m[kAttnWarps][G], red_l[kAttnWarps][G];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int r = lane >> 2, c = lane & 3;
  const int bg = blockIdx.x, split = blockIdx.y;
  const int b = bg / a.Hkv, g = bg - b * a.Hkv;
  const int h0 = g * G;
  const int L = min(max(a.lens[b], 0), a.S);
  const int t_begin = split * a.chunk, t_end = min(t_begin + a.chunk, L);

  const int64_t row_stride = (int64_t)a.Hkv * kD;  // bytes between tokens
  const uint8_t *kbase = a.kq + ((int64_t)b * a.S * a.Hkv + g) * kD;
  const uint8_t *vbase = a.vq + ((int64_t)b * a.S * a.Hkv + g) * kD;
  const float *ksb = a.ks + (int64_t)b * a.S * a.Hkv + g;
  const float *vsb = a.vs + (int64_t)b * a.S * a.Hkv + g;
  StepStage *my = stages + kStages * warp;

  // the first steps' copies are in flight while the queries are prepared
  constexpr int kPass = kAttnWarps * kTokPerIter;  // tokens between a warp's steps
  int base = t_begin + warp * kTokPerIter;
#pragma unroll
  for (int i = 0; i < kStages - 1; ++i) {
    if (base + i * kPass < t_end)
      issue_step(my[i], kbase, vbase, ksb, vsb, row_stride, a.Hkv, base + i * kPass, t_end, lane);
    cp_async_commit();
  }

  // ---- queries: B fragments of head r (zero for r >= G), dimensions
  // [32 c, 32 c + 32), scaled by 2^E of the head
  uint32_t qb[16];
  float hf[2];  // score factor of heads 2 c, 2 c + 1: log2(e) * scale * 2^-E
  {
    float qf[32];
    float amax = 0.f;
    const uint16_t *qrow = a.q + ((int64_t)b * a.Hq + h0 + r) * kD + 32 * c;
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      qf[i] = r < G ? __uint_as_float((uint32_t)qrow[i] << 16) : 0.f;
      amax = fmaxf(amax, fabsf(qf[i]));
    }
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
    const int E = amax > 0.f ? 14 - ilogbf(amax) : 0;
#pragma unroll
    for (int s = 0; s < 8; ++s) {
      qb[2 * s] = f16x2_bits(scalbnf(qf[4 * s], E), scalbnf(qf[4 * s + 1], E));
      qb[2 * s + 1] = f16x2_bits(scalbnf(qf[4 * s + 2], E), scalbnf(qf[4 * s + 3], E));
    }
    const int E0 = __shfl_sync(0xffffffffu, E, 8 * c), E1 = __shfl_sync(0xffffffffu, E, 8 * c + 4);
    hf[0] = scalbnf(a.scale * kLog2e, -E0);
    hf[1] = scalbnf(a.scale * kLog2e, -E1);
  }

  float m2[2] = {-INFINITY, -INFINITY};  // running max per head (log2 units)
  float lsum[2] = {0.f, 0.f};           // this thread's share of the softmax sum
  float vref = 0.f;                     // largest value scale so far
  float o[8][4];
#pragma unroll
  for (int m = 0; m < 8; ++m) o[m][0] = o[m][1] = o[m][2] = o[m][3] = 0.f;

  int slot = 0;  // stage of the current step; the ring's next free stage is the one before it
  for (; base < t_end; base += kPass) {
    StepStage &st = my[slot];
    const int ahead = base + (kStages - 1) * kPass;
    const int free_slot = slot == 0 ? kStages - 1 : slot - 1;
    if (ahead < t_end) issue_step(my[free_slot], kbase, vbase, ksb, vsb, row_stride, a.Hkv, ahead, t_end, lane);
    cp_async_commit();  // one group per step, empty or not, so the count below holds
    cp_async_wait<kStages - 1>();  // this lane's copies of the current step have landed
    __syncwarp();        // ... and every other lane's

    // ---- scores: two 16-token tiles x 8 k-steps
    float sc[2][4], sd[2][4];  // even and odd k-steps: two independent MMA chains per tile
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      sc[i][0] = sc[i][1] = sc[i][2] = sc[i][3] = 0.f;
      sd[i][0] = sd[i][1] = sd[i][2] = sd[i][3] = 0.f;
      const uint4 ka = *reinterpret_cast<const uint4 *>(&st.k[16 * i + r][32 * c]);
      const uint4 kb = *reinterpret_cast<const uint4 *>(&st.k[16 * i + r][32 * c + 16]);
      const uint4 la = *reinterpret_cast<const uint4 *>(&st.k[16 * i + r + 8][32 * c]);
      const uint4 lb = *reinterpret_cast<const uint4 *>(&st.k[16 * i + r + 8][32 * c + 16]);
      const uint32_t w0[8] = {ka.x, ka.y, ka.z, ka.w, kb.x, kb.y, kb.z, kb.w};
      const uint32_t w1[8] = {la.x, la.y, la.z, la.w, lb.x, lb.y, lb.z, lb.w};
#pragma unroll
      for (int s = 0; s < 8; ++s) {
        uint32_t a0, a1, a2, a3;
        e4m3x4_f16(w0[s], a0, a2);
        e4m3x4_f16(w1[s], a1, a3);
        mma_16816((s & 1) ? sd[i] : sc[i], a0, a1, a2, a3, qb[2 * s], qb[2 * s + 1]);
      }
#pragma unroll
      for (int e = 0; e < 4; ++e) sc[i][e] += sd[i][e];
    }

    // ---- online softmax (base 2)
    float s2[4][2], vsv[4];
    float mx[2] = {-INFINITY, -INFINITY}, vm = 0.f;
#pragma unroll
    for (int j = 0; j < 4; ++j) {  // token 16 (j >> 1) + r + 8 (j & 1)
      const int u = 16 * (j >> 1) + r + 8 * (j & 1);
      const bool valid = base + u < t_end;
      const float kscale = st.ks[u];
      vsv[j] = st.vs[u];  // 0 for zero-filled tokens
      vm = fmaxf(vm, vsv[j]);
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        s2[j][h] = valid ? sc[j >> 1][2 * (j & 1) + h] * kscale * hf[h] : -INFINITY;
        mx[h] = fmaxf(mx[h], s2[j][h]);
      }
    }
    vm = max_over_row_groups(vm);
    const float vnew = fmaxf(vref, vm);
    const float inv = vnew > 0.f ? __frcp_rn(vnew) : 0.f;
    const float vratio = vref * inv;  // 0 before the first step: o is 0 then
    vref = vnew;
    float osc[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const float mn = fmaxf(m2[h], max_over_row_groups(mx[h]));  // finite: token base is valid
      const float alpha = exp2_approx(m2[h] - mn);
      m2[h] = mn;
      lsum[h] *= alpha;
      osc[h] = alpha * vratio;
    }
#pragma unroll
    for (int m = 0; m < 8; ++m) {
      o[m][0] *= osc[0];
      o[m][1] *= osc[1];
      o[m][2] *= osc[0];
      o[m][3] *= osc[1];
    }
    // P^T B fragments: [2 i] tokens 16 i + 0..7, [2 i + 1] tokens 16 i + 8..15;
    // each weight is carried as the sum of two f16 values (ph + pl), which
    // leaves a relative error of about 2^-22
    uint32_t ph[4], pl[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float e0 = exp2_approx(s2[j][0] - m2[0]), e1 = exp2_approx(s2[j][1] - m2[1]);
      lsum[0] += e0;
      lsum[1] += e1;
      const float w = vsv[j] * inv;
      const float x0 = e0 * w, x1 = e1 * w;
      const uint32_t hi = f16x2_bits(x0, x1);
      const float2 hf2 = __half22float2(*reinterpret_cast<const __half2 *>(&hi));
      ph[j] = movmatrix_trans(hi);
      pl[j] = movmatrix_trans(f16x2_bits(x0 - hf2.x, x1 - hf2.y));
    }

    // ---- values: two 16-token k-steps x 8 head-dimension tiles
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const uint4 x0 = *reinterpret_cast<const uint4 *>(&st.v[16 * i + 2 * c][16 * r]);
      const uint4 x1 = *reinterpret_cast<const uint4 *>(&st.v[16 * i + 2 * c + 1][16 * r]);
      const uint4 x2 = *reinterpret_cast<const uint4 *>(&st.v[16 * i + 2 * c + 8][16 * r]);
      const uint4 x3 = *reinterpret_cast<const uint4 *>(&st.v[16 * i + 2 * c + 9][16 * r]);
      const uint32_t y0[4] = {x0.x, x0.y, x0.z, x0.w}, y1[4] = {x1.x, x1.y, x1.z, x1.w};
      const uint32_t y2[4] = {x2.x, x2.y, x2.z, x2.w}, y3[4] = {x3.x, x3.y, x3.z, x3.w};
#pragma unroll
      for (int n = 0; n < 4; ++n) {  // head dimensions 16 r + 4 n .. + 3
        const uint32_t lo01 = __byte_perm(y0[n], y1[n], 0x5140), hi01 = __byte_perm(y0[n], y1[n], 0x7362);
        const uint32_t lo89 = __byte_perm(y2[n], y3[n], 0x5140), hi89 = __byte_perm(y2[n], y3[n], 0x7362);
        uint32_t a0, a1, a2, a3, c0, c1, c2, c3;
        e4m3x4_f16(lo01, a0, a1);
        e4m3x4_f16(lo89, a2, a3);
        mma_16816(o[2 * n], a0, a1, a2, a3, ph[2 * i], ph[2 * i + 1]);
        mma_16816(o[2 * n], a0, a1, a2, a3, pl[2 * i], pl[2 * i + 1]);
        e4m3x4_f16(hi01, c0, c1);
        e4m3x4_f16(hi89, c2, c3);
        mma_16816(o[2 * n + 1], c0, c1, c2, c3, ph[2 * i], ph[2 * i + 1]);
        mma_16816(o[2 * n + 1], c0, c1, c2, c3, pl[2 * i], pl[2 * i + 1]);
      }
    }
    __syncwarp();  // the stage is rewritten by later steps
    slot = slot == kStages - 1 ? 0 : slot + 1;
  }
  cp_async_wait<0>();

  // ---- merge the four warps (the stage buffers are free now: reuse them for
  // the partial outputs), write this split's partial per query head
  lsum[0] = sum_over_row_groups(lsum[0]);
  lsum[1] = sum_over_row_groups(lsum[1]);
  __syncthreads();
  float(*red_o)[G][kD] = reinterpret_cast<float(*)[G][kD]>(attn_smem);
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int j = 2 * c + h;
    if (j < G) {
#pragma unroll
      for (int m = 0; m < 8; ++m) {
        red_o[warp][j][16 * r + 2 * m] = o[m][h] * vref;
        red_o[warp][j][16 * r + 2 * m + 1] = o[m][2 + h] * vref;
      }
      if (r == 0) {
        red_m[warp][j] = m2[h];
        red_l[warp][j] = lsum[h];
      }
    }
  }
  __syncthreads();
  for (int i = threadIdx.x; i < G * (kD + 2); i += blockDim.x) {
    const int j = i / (kD + 2), col = i - j * (kD + 2);
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kAttnWarps; ++w) M = fmaxf(M, red_m[w][j]);
    float val = 0.f;
    if (col < kD) {
      if (M != -INFINITY)
#pragma unroll
        for (int w = 0; w < kAttnWarps; ++w)
          if (red_m[w][j] != -INFINITY) val += red_o[w][j][col] * exp2f(red_m[w][j] - M);
    } else if (col == kD) {
      val = M;
    } else if (M != -INFINITY) {
#pragma unroll
      for (int w = 0; w < kAttnWarps; ++w)
        if (red_m[w][j] != -INFINITY) val += red_l[w][j] * exp2f(red_m[w][j] - M);
    }
    a.ws[(((int64_t)b * a.Hq + h0 + j) * a.nsplit + split) * kPart + col] = val;
  }
}

template <int G>
constexpr int attn_smem_bytes() {
  return (int)(sizeof(StepStage) * kStages * kAttnWarps);
}
static_assert(sizeof(StepStage) * kStages * kAttnWarps >= sizeof(float) * kAttnWarps * 8 * kD, "partial outputs fit the stages");

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
        const float w = exp2f(ms[k] - M);
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
  *reinterpret_cast<uint32_t *>(dst + 4 * lane) =
      fast_tile<MODE>(ts) ? encode4<MODE, true>(x.x, x.y, ts) : encode4<MODE>(x.x, x.y, ts);
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

int g_attn_blocks_per_sm[4] = {0, 0, 0, 0};  // G = 1, 2, 4, 8

int attn_blocks_per_sm(int G) {
  const int gi = G == 1 ? 0 : G == 2 ? 1 : G == 4 ? 2 : 3;
  if (g_attn_blocks_per_sm[gi] == 0) {
    int n = 0;
    cudaError_t e = cudaSuccess;
    if (prepare_attention() == FP8BQ_OK) {
      switch (gi) {
        case 0: e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, decode_attn_kernel<1>, kAttnWarps * 32, attn_smem_bytes<1>()); break;
        case 1: e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, decode_attn_kernel<2>, kAttnWarps * 32, attn_smem_bytes<2>()); break;
        case 2: e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, decode_attn_kernel<4>, kAttnWarps * 32, attn_smem_bytes<4>()); break;
        default: e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, decode_attn_kernel<8>, kAttnWarps * 32, attn_smem_bytes<8>()); break;
      }
    }
    if (e != cudaSuccess) (void)cudaGetLastError();
    g_attn_blocks_per_sm[gi] = std::max(1, n);
  }
  return g_attn_blocks_per_sm[gi];
}

// Splits of the sequence.  Measured on B200: about two blocks per SM keep
// HBM busy, and beyond that more (shorter) chunks only add fixed costs (the
// queries, the pipeline fill, the merge, the partials).  So fewer key/value
// heads than SMs are split into about 2 x SMs blocks in all (chunks of at
// least two passes of a block); otherwise heads stay whole unless up to four
// splits even out the waves of resident blocks: s minimizes waves(s) x
// (passes per chunk + 1).
int attn_splits(int64_t B, int64_t Hkv, int64_t S, int G) {
  const int64_t W = std::max<int64_t>(B * Hkv, 1);
  const int64_t sms = num_sms();
  const int64_t passes = (S + kChunkQuantum - 1) / kChunkQuantum;
  const int64_t max_splits = std::max<int64_t>(1, std::min<int64_t>(passes / 2, 4096));
  if (W < sms) return (int)std::min(max_splits, std::max<int64_t>(1, 2 * sms / W));
  const int64_t R = sms * attn_blocks_per_sm(G);
  int64_t best = 1, best_cost = INT64_MAX;
  for (int64_t s = 1; s <= std::min<int64_t>(4, max_splits); ++s) {
    const int64_t cost = (W * s + R - 1) / R * ((passes + s - 1) / s + 1);
    if (cost < best_cost) {
      best_cost = cost;
      best = s;
    }
  }
  return (int)best;
}

}  // namespace

size_t decode_attention_workspace_size(int64_t B, int64_t Hq, int64_t Hkv, int64_t S) {
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || S <= 0) return 0;
  return (size_t)B * Hq * attn_splits(B, Hkv, S, (int)(Hq / Hkv)) * kPart * sizeof(float);
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
  a.nsplit = attn_splits(B, Hkv, S, (int)(Hq / Hkv));
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
