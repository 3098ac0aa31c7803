// Decode-shaped (small M, memory-bound) block-scaled FP8 linear for sm_100a:
// Y[M,N] = q(X)[M,K] . W[N,K]^T with the activation quantized on the fly
// (1x128 tiles) and W pre-quantized (128x128 tiles).
//
// Method: "NVIDIA NeMo RL Achieves 48% Speedup With End-to-End FP8 Precision
// Training", section "Technical breakthrough": FP8 is applied in generation as
// well as in training, with block-wise E4M3 (activations 1x128, weights
// 128x128).  In generation the linear layers see a handful of tokens, so the
// time goes into streaming the weight from HBM.
//
// Design.  Two launches:
//   1. prologue: 1x128 quantization of X into the workspace (the same device
//      code as fp8bq_quant_act) and zeroing of the split-K counters;
//   2. the GEMM, with the operands swapped so that the tensor cores do useful
//      work at small M: the weight is the 128-row MMA operand and the tokens
//      are the MMA's N dimension (NT = M rounded up to 16, 32 or 64; rows
//      past M are TMA zero-fill).  For M > 64 the per-token promotion would
//      cost more than the weight stream, so step 2 is the prefill GEMM on the
//      quantized activation instead.  A unit of work is one 128-row
//      weight block times one contiguous range of K-blocks (split-K chosen on
//      the host so the units fill the SMs).  Per K-block: TMA loads of the
//      weight tile (16 KB), the activation-code tile and that K-block's row
//      scales into a deep stage ring; 4 x tcgen05.mma 128xNTx32 into one of
//      two TMEM buffers; the epilogue warps (weight row = TMEM lane, token =
//      column) add P * (sa[kb][token] * sw[nb][kb]) into FP32 registers.
//   A unit writes bf16 directly when the K range is not split; otherwise it
//   writes an FP32 partial to the workspace and bumps a per-weight-block
//   counter, and the unit that arrives last sums the partials in split order
//   (deterministic) and writes bf16.
#include <cuda_bf16.h>
#include <string.h>

#include <algorithm>

#include "device.cuh"
#include "internal.h"
#include "quant.cuh"

namespace fp8bq {
namespace {

constexpr int DBM = 128, DBK = 128;
constexpr int kDThreads = 384;
constexpr int kDLaunchRegs = 168;
constexpr int kDLowRegs = 56;
constexpr int kDHighRegs = 224;
static_assert(128 * kDLowRegs + 256 * kDHighRegs <= kDThreads * kDLaunchRegs, "register split");
constexpr int kMaxDecodeM = 256;
// Above this many tokens the swapped kernel's per-column promotion costs more
// than the weight stream: quantize into the workspace and run the prefill GEMM
// (128-row tiles, per-row scales) instead.
constexpr int kSwapMaxM = 64;
constexpr int kMaxSplit = 16;
constexpr int kDEpiWarps = 8;
constexpr int kStageBudget = 212992;

template <int NT>
struct DCfg {
  static constexpr int kABytes = DBM * DBK;  // weight tile
  static constexpr int kBBytes = NT * DBK;   // activation-code tile
  static constexpr int kSBytes = NT * 4;     // the K-block's activation scales
  static constexpr int kSSlot = (kSBytes + 127) / 128 * 128;
  static constexpr int kTx = kABytes + kBBytes + kSBytes;
  static constexpr int kFit = kStageBudget / (kABytes + kBBytes + kSSlot);
  static constexpr int kStages = kFit < 8 ? kFit : 8;
  static constexpr int kCW = NT / 2;         // token columns per epilogue warpgroup
  static constexpr int kTmemCols = 2 * NT < 32 ? 32 : 2 * NT;
  static constexpr int kCH = kCW < 32 ? kCW : 32;  // columns per TMEM load round
  static constexpr int kSmemBytes = kStages * (kABytes + kBBytes + kSSlot) + 256 + 1024;
  static_assert(kStages >= 3 && kSmemBytes <= 232448, "decode shared memory budget");
};

struct DecodeArgs {
  const float *sw;
  int32_t M, N, KB, NB;
  int32_t S;      // K-splits per weight block
  int32_t units;  // NB * S
  float *part;    // [S][M][N] partials (S > 1)
  int32_t *cnt;   // [NB] arrival counters, zeroed by the prologue
  uint16_t *y;    // bf16 bits
  int64_t ldy;
};

__device__ __forceinline__ uint16_t bf16_bits(float v) {
  __nv_bfloat16 b = __float2bfloat16_rn(v);
  return *reinterpret_cast<uint16_t *>(&b);
}

// Named barrier among the 256 epilogue threads that also ORs a predicate.
__device__ __forceinline__ bool epi_barrier_or(bool p) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred q, o;\n\t"
      "setp.ne.u32 q, %1, 0;\n\t"
      "bar.red.or.pred o, 1, 256, q;\n\t"
      "selp.u32 %0, 1, 0, o;\n\t}\n"
      : "=r"(r)
      : "r"((uint32_t)p)
      : "memory");
  return r != 0;
}

// CH consecutive TMEM columns of this warp's 32 lanes into r[0..CH).
template <int CH>
__device__ __forceinline__ void load_cols(uint32_t taddr, uint32_t *r) {
  if constexpr (CH == 8) {
    tmem_ld_32x32b_x8(taddr, r);
  } else if constexpr (CH == 16) {
    tmem_ld_32x32b_x16(taddr, r);
  } else {
#pragma unroll
    for (int c = 0; c < CH / 32; ++c) tmem_ld_32x32b_x32(taddr + 32 * c, *reinterpret_cast<uint32_t(*)[32]>(r + 32 * c));
  }
}

template <int NT>
__global__ void __launch_bounds__(kDThreads, 1)
    decode_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX,
                  const __grid_constant__ CUtensorMap tmS, const DecodeArgs args) {
  using C = DCfg<NT>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *sA = base;
  uint8_t *sB = sA + C::kStages * C::kABytes;
  uint8_t *sS = sB + C::kStages * C::kBBytes;  // kStages slots of kSSlot bytes (128-byte aligned)
  uint64_t *bars = reinterpret_cast<uint64_t *>(sS + C::kStages * C::kSSlot);
  uint64_t *full = bars;
  uint64_t *empty = bars + C::kStages;
  uint64_t *tfull = empty + C::kStages;
  uint64_t *tempty = tfull + 2;
  uint64_t *drain = tempty + 2;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(drain + 1);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
  volatile int *last_flag = abort_flag + 1;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int S = args.S, KB = args.KB;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1 + kDEpiWarps);  // MMA commit + every epilogue warp (they read the scales)
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], kDEpiWarps);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    *last_flag = 0;
    fence_mbarrier_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tensormap(&tmW);
    prefetch_tensormap(&tmX);
    prefetch_tensormap(&tmS);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp < 4) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kDLowRegs));
    if (warp == 0 && lane == 0) {
      // ---------------------------------------------------------------- producer
      int stage = 0;
      uint32_t phase = 0, armed = 0, armed_parity = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < args.units && ok; u += gridDim.x) {
        const int nb = u / S, kc = u - nb * S;
        const int kb0 = (int)((int64_t)kc * KB / S), kb1 = (int)((int64_t)(kc + 1) * KB / S);
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1, abort_flag, kSiteProducerEmpty)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&full[stage], C::kTx);
          tma_load_2d(sA + stage * C::kABytes, &tmW, &full[stage], kb * DBK, nb * DBM);
          tma_load_2d(sB + stage * C::kBBytes, &tmX, &full[stage], kb * DBK, 0);
          tma_load_2d(sS + stage * C::kSSlot, &tmS, &full[stage], 0, kb);
          armed |= 1u << stage;
          armed_parity = (armed_parity & ~(1u << stage)) | (phase << stage);
          if (++stage == C::kStages) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      if (!ok) {
        for (int s = 0; s < C::kStages; ++s)
          if (armed >> s & 1u) mbar_wait(&full[s], (armed_parity >> s) & 1u, nullptr, kSiteDrain);
      }
    } else if (warp == 1 && lane == 0) {
      // ---------------------------------------------------------------- MMA issuer
      const uint32_t idesc = idesc_f8f6f4_e4m3_f32(DBM, NT);
      int stage = 0, buf = 0;
      uint32_t phase = 0, bphase = 0;
      bool ok = true, issued = false;
      for (int u = blockIdx.x; u < args.units && ok; u += gridDim.x) {
        const int nb = u / S, kc = u - nb * S;
        const int kb0 = (int)((int64_t)kc * KB / S), kb1 = (int)((int64_t)(kc + 1) * KB / S);
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait(&tempty[buf], bphase ^ 1, abort_flag, kSiteMmaTmemEmpty) ||
              !mbar_wait(&full[stage], phase, abort_flag, kSiteMmaFull)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t d = tmem_base + (uint32_t)(buf * NT);
          const uint32_t a0 = smem_addr(sA + stage * C::kABytes);
          const uint32_t b0 = smem_addr(sB + stage * C::kBBytes);
#pragma unroll
          for (int k = 0; k < DBK / 32; ++k)
            mma_f8f6f4(d, smem_desc_k_sw128(a0 + 32 * k), smem_desc_k_sw128(b0 + 32 * k), idesc, k > 0 ? 1u : 0u);
          mma_commit(&empty[stage]);
          mma_commit(&tfull[buf]);
          issued = true;
          if (++stage == C::kStages) {
            stage = 0;
            phase ^= 1;
          }
          if (++buf == 2) {
            buf = 0;
            bphase ^= 1;
          }
        }
      }
      if (!ok && issued) {
        mma_commit(drain);
        mbar_wait(drain, 0, nullptr, kSiteDrain);
      }
    }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kDHighRegs));
    // ------------------------------------------------------------------ epilogue
    const int quarter = warp & 3;
    const int h = (warp - 4) >> 2;
    const int c0 = h * C::kCW;  // first token column of this warpgroup
    int stage = 0, buf = 0;
    uint32_t phase = 0, bphase = 0;
    bool ok = true;
    for (int u = blockIdx.x; u < args.units; u += gridDim.x) {
      const int nb = u / S, kc = u - nb * S;
      const int kb0 = (int)((int64_t)kc * KB / S), kb1 = (int)((int64_t)(kc + 1) * KB / S);
      const int n = nb * DBM + quarter * 32 + lane;  // weight row = output column
      const float *swp = args.sw + (int64_t)nb * KB;
      float acc[C::kCW];
#pragma unroll
      for (int j = 0; j < C::kCW; ++j) acc[j] = 0.f;
      float w0 = __ldg(swp + kb0), w1 = (kb0 + 1 < kb1) ? __ldg(swp + kb0 + 1) : 0.f;
      for (int kb = kb0; kb < kb1 && ok; ++kb) {
        const float w = w0;
        w0 = w1;
        if (kb + 2 < kb1) w1 = __ldg(swp + kb + 2);
        const bool got = mbar_wait(&tfull[buf], bphase, abort_flag, kSiteEpiTmemFull);
        if (!__all_sync(0xffffffffu, got)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t taddr = tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(buf * NT + c0);
        const float4 *sc4 = reinterpret_cast<const float4 *>(sS + stage * C::kSSlot) + c0 / 4;
#pragma unroll
        for (int c = 0; c < C::kCW / C::kCH; ++c) {
          uint32_t r[C::kCH];
          load_cols<C::kCH>(taddr + c * C::kCH, r);
          tmem_ld_wait();
          if (c == C::kCW / C::kCH - 1) {  // the TMEM buffer has been read
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&tempty[buf]);
          }
#pragma unroll
          for (int j = 0; j < C::kCH / 4; ++j) {
            const float4 s4 = sc4[c * C::kCH / 4 + j];
            float *a = &acc[c * C::kCH + 4 * j];
            a[0] = fmaf(__uint_as_float(r[4 * j + 0]), s4.x * w, a[0]);
            a[1] = fmaf(__uint_as_float(r[4 * j + 1]), s4.y * w, a[1]);
            a[2] = fmaf(__uint_as_float(r[4 * j + 2]), s4.z * w, a[2]);
            a[3] = fmaf(__uint_as_float(r[4 * j + 3]), s4.w * w, a[3]);
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[stage]);  // the stage's scales have been read
        if (++stage == C::kStages) {
          stage = 0;
          phase ^= 1;
        }
        if (++buf == 2) {
          buf = 0;
          bphase ^= 1;
        }
      }
      (void)phase;
      if (S == 1) {
        if (!ok) break;
        if (n < args.N) {
#pragma unroll
          for (int j = 0; j < C::kCW; ++j)
            if (c0 + j < args.M) args.y[(int64_t)(c0 + j) * args.ldy + n] = bf16_bits(acc[j]);
        }
        continue;
      }
      // split K: partial out, then the last unit of this weight block reduces
      if (ok && n < args.N) {
#pragma unroll
        for (int j = 0; j < C::kCW; ++j)
          if (c0 + j < args.M) args.part[((int64_t)kc * args.M + (c0 + j)) * args.N + n] = acc[j];
      }
      __threadfence();
      const bool stop1 = epi_barrier_or(!ok);
      if (stop1) break;
      if (warp == 4 && lane == 0) *last_flag = (atomicAdd(args.cnt + nb, 1) == S - 1) ? 1 : 0;
      epi_barrier_or(false);
      if (*last_flag) {
        // Sum the S partials in split order (the same order whichever unit
        // arrives last); this unit's own partial is still in registers.  The
        // loads of one split are independent, so all of them are in flight
        // together.
        __threadfence();
        float tot[C::kCW];
#pragma unroll
        for (int j = 0; j < C::kCW; ++j) tot[j] = 0.f;
        for (int s = 0; s < S; ++s) {
          if (s == kc) {
#pragma unroll
            for (int j = 0; j < C::kCW; ++j) tot[j] += acc[j];
          } else if (n < args.N) {
            const float *src = args.part + (int64_t)s * args.M * args.N + n;
#pragma unroll
            for (int j = 0; j < C::kCW; ++j)
              if (c0 + j < args.M) tot[j] += __ldcg(src + (int64_t)(c0 + j) * args.N);
          }
        }
        if (n < args.N) {
#pragma unroll
          for (int j = 0; j < C::kCW; ++j)
            if (c0 + j < args.M) args.y[(int64_t)(c0 + j) * args.ldy + n] = bf16_bits(tot[j]);
        }
      }
      if (epi_barrier_or(*abort_flag != 0)) break;  // also keeps last_flag stable until all have read it
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::kTmemCols);
  }
}

// Prologue: 1x128 quantization of X into the workspace, counters zeroed.
template <int MODE, bool VEC>
__global__ void __launch_bounds__(256) decode_prologue_kernel(const uint16_t *__restrict__ x, int64_t M, int64_t K,
                                                              int64_t ldx, uint8_t *__restrict__ q,
                                                              float *__restrict__ sa, int64_t ldsa,
                                                              int32_t *__restrict__ cnt, int ncnt) {
  if (blockIdx.x == 0 && blockIdx.y == 0)
    for (int i = threadIdx.x; i < ncnt; i += blockDim.x) cnt[i] = 0;
  if constexpr (VEC) qdev::quant_act_vec_block<MODE, 4>(blockIdx.x, blockIdx.y, x, M, K, ldx, q, K, sa, ldsa);
  else qdev::quant_act_scalar_block<MODE>(blockIdx.x, blockIdx.y, x, M, K, ldx, q, K, sa, ldsa);
}

struct Plan {
  int NT, S, NB, KB;
  int64_t ldsa;
  size_t off_q, off_sa, off_part, off_cnt, total;
};

size_t align256(size_t v) { return (v + 255) & ~size_t(255); }

int pick_nt(int64_t M) {
  if (M <= 16) return 16;
  if (M <= 32) return 32;
  return 64;
}

// Split-K count: minimise (weight bytes / SM-fill efficiency) + partial traffic.
int pick_split(int64_t M, int64_t N, int64_t K, int NB, int KB, int sms) {
  double best = 1e300;
  int best_s = 1;
  for (int s = 1; s <= std::min(KB, kMaxSplit); ++s) {
    const int64_t units = (int64_t)NB * s;
    const int64_t waves = (units + sms - 1) / sms;
    const double eff = (double)units / (double)(waves * sms);
    const double cost = (double)N * K / eff + (s > 1 ? 8.0 * s * M * N : 0.0);
    if (cost < best * (1.0 - 1e-9)) {
      best = cost;
      best_s = s;
    }
  }
  return best_s;
}

Plan make_plan(int64_t M, int64_t N, int64_t K) {
  Plan p;
  p.NT = M <= kSwapMaxM ? pick_nt(M) : 0;  // 0: the prefill GEMM
  p.NB = (int)((N + 127) / 128);
  p.KB = (int)(K / 128);
  p.S = p.NT ? pick_split(M, N, K, p.NB, p.KB, num_sms()) : 1;
  p.ldsa = (M + 3) / 4 * 4;
  p.off_q = 0;
  p.off_sa = align256((size_t)(M * K));
  p.off_part = p.off_sa + align256((size_t)p.KB * p.ldsa * 4);
  p.off_cnt = p.off_part + (p.S > 1 ? align256((size_t)p.S * M * N * 4) : 0);
  p.total = p.off_cnt + align256((size_t)p.NB * 4);
  return p;
}

int g_dready[3][64] = {{0}};

template <int NT>
fp8bq_status launch_decode_nt(const CUtensorMap &tW, const CUtensorMap &tX, const CUtensorMap &tS,
                              const DecodeArgs &a, cudaStream_t stream, int slot) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= 64) dev = 0;
  int &ready = g_dready[slot][dev];
  if (ready == -1) return FP8BQ_ERR_UNSUPPORTED;
  if (ready == 0) {
    cudaFuncAttributes fa;
    e = cudaFuncGetAttributes(&fa, decode_kernel<NT>);
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncGetAttributes(decode)");
    if (fa.numRegs != kDLaunchRegs) {
      ready = -1;
      return FP8BQ_ERR_UNSUPPORTED;
    }
    e = cudaFuncSetAttribute(decode_kernel<NT>, cudaFuncAttributeMaxDynamicSharedMemorySize, DCfg<NT>::kSmemBytes);
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(decode)");
    ready = 1;
  }
  const int grid = std::min(a.units, num_sms());
  decode_kernel<NT><<<grid, kDThreads, DCfg<NT>::kSmemBytes, stream>>>(tW, tX, tS, a);
  return check_launch("gemm_decode");
}

bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

}  // namespace

cudaError_t take_device_error_decode(unsigned long long *v) { return take_tu_device_error(v); }

size_t decode_workspace_size(int64_t M, int64_t N, int64_t K) {
  if (M <= 0 || N <= 0 || K <= 0 || M > kMaxDecodeM || K % 128 != 0) return 0;
  return make_plan(M, N, K).total;
}

fp8bq_status launch_gemm_decode(const void *x, int64_t ldx, const uint8_t *qw, int64_t ldw, const float *sw, void *y,
                                int64_t ldy, int64_t M, int64_t N, int64_t K, int mode, void *ws, size_t ws_bytes,
                                cudaStream_t stream) {
  if (M > kMaxDecodeM) return FP8BQ_ERR_UNSUPPORTED;
  const Plan p = make_plan(M, N, K);
  if (ws == nullptr || ws_bytes < p.total || !aligned(ws, 256)) return FP8BQ_ERR_WORKSPACE;
  uint8_t *wsb = static_cast<uint8_t *>(ws);
  uint8_t *q = wsb + p.off_q;
  float *sa = reinterpret_cast<float *>(wsb + p.off_sa);
  float *part = reinterpret_cast<float *>(wsb + p.off_part);
  int32_t *cnt = reinterpret_cast<int32_t *>(wsb + p.off_cnt);

  // 1. quantize X (and zero the counters)
  const uint16_t *xs = static_cast<const uint16_t *>(x);
  const bool vec = aligned(x, 16) && ldx % 8 == 0;  // K % 128 == 0 already
  if (vec) {
    dim3 grid((unsigned)((M + 63) / 64), (unsigned)p.KB);
    if (mode == FP8BQ_SCALE_FP32)
      decode_prologue_kernel<FP8BQ_SCALE_FP32, true><<<grid, 256, 0, stream>>>(xs, M, K, ldx, q, sa, p.ldsa, cnt, p.NB);
    else
      decode_prologue_kernel<FP8BQ_SCALE_POW2, true><<<grid, 256, 0, stream>>>(xs, M, K, ldx, q, sa, p.ldsa, cnt, p.NB);
  } else {
    dim3 grid((unsigned)((M + 15) / 16), (unsigned)p.KB);
    if (mode == FP8BQ_SCALE_FP32)
      decode_prologue_kernel<FP8BQ_SCALE_FP32, false><<<grid, 256, 0, stream>>>(xs, M, K, ldx, q, sa, p.ldsa, cnt, p.NB);
    else
      decode_prologue_kernel<FP8BQ_SCALE_POW2, false><<<grid, 256, 0, stream>>>(xs, M, K, ldx, q, sa, p.ldsa, cnt, p.NB);
  }
  fp8bq_status st = check_launch("gemm_decode prologue");
  if (st != FP8BQ_OK) return st;

  // 2. the GEMM
  if (p.NT == 0)
    return launch_gemm(q, K, sa, p.ldsa, qw, ldw, sw, y, ldy, M, N, K, mode, FP8BQ_GEMM_AUTO, stream);
  CUtensorMap tW, tX, tS;
  if (!make_tmap_2d(&tW, CU_TENSOR_MAP_DATA_TYPE_UINT8, qw, (uint64_t)K, (uint64_t)N, (uint64_t)ldw, DBK, DBM,
                    CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_tmap_2d(&tX, CU_TENSOR_MAP_DATA_TYPE_UINT8, q, (uint64_t)K, (uint64_t)M, (uint64_t)K, DBK,
                    (uint32_t)p.NT, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_tmap_2d(&tS, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, sa, (uint64_t)M, (uint64_t)p.KB, (uint64_t)p.ldsa * 4,
                    (uint32_t)p.NT, 1, CU_TENSOR_MAP_SWIZZLE_NONE))
    return FP8BQ_ERR_INVALID_ARG;
  DecodeArgs a;
  a.sw = sw;
  a.M = (int32_t)M;
  a.N = (int32_t)N;
  a.KB = p.KB;
  a.NB = p.NB;
  a.S = p.S;
  a.units = p.NB * p.S;
  a.part = part;
  a.cnt = cnt;
  a.y = static_cast<uint16_t *>(y);
  a.ldy = ldy;
  switch (p.NT) {
    case 16: return launch_decode_nt<16>(tW, tX, tS, a, stream, 0);
    case 32: return launch_decode_nt<32>(tW, tX, tS, a, stream, 1);
    default: return launch_decode_nt<64>(tW, tX, tS, a, stream, 2);
  }
}

}  // namespace fp8bq
