// Block-scaled FP8 GEMM with power-of-two scales on the tensor cores' native
// block scaling (tcgen05.mma kind::mxf8f6f4 .block_scale, UE8M0 scale factors
// in TMEM), for sm_100a.
//
// Method: "NVIDIA NeMo RL Achieves 48% Speedup With End-to-End FP8 Precision
// Training", section "Technical breakthrough" (block-wise E4M3, activations
// 1x128, weights 128x128) with the power-of-2 scaling factors of section "Why
// this matters for AI economics".
//
// With power-of-two scales sa = 2^ea and sw = 2^ew, every product
// qa * qw * sa * sw is exact in FP32 (barring overflow), so the scales can be
// applied inside the MMA instead of by promotion: the hardware multiplies each
// 32-deep K-slice by 2^(ea + ew) given UE8M0 exponents per row of A and per row
// of B.  The 1x128 activation scale becomes four equal UE8M0 values per row per
// K-block and the 128x128 weight scale the same value for all 128 rows of the
// weight block.  The accumulator then stays in TMEM for the whole K loop and
// the epilogue runs once per tile.  The result differs from the promotion path
// only in the order of the FP32 additions.
//
// Structure (persistent, 1 CTA per SM, 384 threads):
//   warp 0      TMA producer: A 128x128 B and B 256x128 B tiles per K-block,
//               4-stage ring.
//   warp 1      MMA issuer: per K-block copies the stage's scale factors into
//               TMEM (tcgen05.cp 32x128b.warpx4: SFA 4 columns, SFB 8 columns)
//               and issues 4 x tcgen05.mma 128x256x32 block_scale into the one
//               256-column accumulator.
//   warp 2      scale-factor producer: per K-block converts the 128 row scales
//               of A and the two weight-block scales of B to UE8M0 bytes in the
//               stage's 32x128b shared-memory layout (byte (r*16 + c*4 + k) =
//               scale of row r + 32c, K-slice k).
//   warps 4-11  epilogue: drain the accumulator (tcgen05.ld, then release it
//               to the next tile's MMAs at once), bf16 through 64-byte-swizzled
//               staging and TMA stores.
#include <cuda_bf16.h>

#include <algorithm>

#include "device.cuh"
#include "internal.h"

namespace fp8bq {
namespace {

constexpr int BM = 128, BN = 256, BK = 128;
constexpr int kStages = 4;
constexpr int kABytes = BM * BK;
constexpr int kBBytes = BN * BK;
constexpr int kSFABytes = 512;   // 32 rows x 16 bytes
constexpr int kSFBBytes = 1024;  // two 32x16-byte blocks (B rows 0-127, 128-255)
constexpr int kSFBytes = kSFABytes + kSFBBytes;
constexpr int kEpiWarps = 8;
constexpr int kEpiBufBytes = 32 * 64;  // 32 rows x 32 bf16, 64-byte swizzle
constexpr int kThreads = 384;
constexpr int kLaunchRegs = 168;
constexpr int kLowRegs = 56;
constexpr int kHighRegs = 224;
static_assert(128 * kLowRegs + 256 * kHighRegs <= kThreads * kLaunchRegs, "register split");
constexpr int kTmemCols = 512;
constexpr int kAccCols = BN;       // one 128 x 256 FP32 accumulator
constexpr int kSFCols = 12;        // per stage: SFA 4 + SFB 8 TMEM columns
constexpr int kSmemBytes =
    kStages * (kABytes + kBBytes) + kStages * kSFBytes + kEpiWarps * kEpiBufBytes + 256 + 1024;
static_assert(kSmemBytes <= 232448, "shared memory budget");
static_assert(kAccCols + kStages * kSFCols <= kTmemCols, "TMEM budget");

struct NativeArgs {
  const float *sa;
  const float *sw;    // ROWB: B row scales sw[kb * ldsw + n]; else 128x128 tile scales sw[nb * KB + kb]
  int64_t ldsa;
  int64_t ldsw;
  int32_t M, N, KB, NB;
  int32_t num_m, num_n;
  int32_t band, n_major;  // tile order (raster_tile)
};

__device__ __forceinline__ void tile_mn(int t, const NativeArgs &a, int &mb, int &nb) {
  raster_tile(t, a.num_m, a.num_n, a.band, a.n_major, mb, nb);
}

// UE8M0 of a power-of-two fp32 scale: its exponent field (2^-127, a binary32
// denormal, has field 0, which is UE8M0's 2^-127).  Replicated into 4 bytes.
__device__ __forceinline__ uint32_t ue8m0x4(float s) { return (__float_as_uint(s) >> 23 & 0xFFu) * 0x01010101u; }

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t *>(&v);
}

// ROWB: B's scales vary per B row (the weight-gradient GEMM, where B = X^T
// is 1x128-quantized along the tokens); otherwise one scale per 128x128 tile.
template <bool ROWB>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_native_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                       const __grid_constant__ CUtensorMap tmY, const NativeArgs args) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *sA = base;
  uint8_t *sB = sA + kStages * kABytes;
  uint8_t *sSF = sB + kStages * kBBytes;
  uint8_t *sEpi = sSF + kStages * kSFBytes;
  uint64_t *bars = reinterpret_cast<uint64_t *>(sEpi + kEpiWarps * kEpiBufBytes);
  uint64_t *full = bars;             // TMA bytes landed + scale factors written (count 2)
  uint64_t *empty = bars + kStages;  // MMAs done with the stage
  uint64_t *tfull = empty + kStages;  // accumulator complete
  uint64_t *tempty = tfull + 1;       // accumulator drained by the epilogue
  uint64_t *drain = tempty + 1;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(drain + 1);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int total = args.num_m * args.num_n;
  const int KB = args.KB;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 2);
      mbar_init(&empty[s], 1);
    }
    mbar_init(tfull, 1);
    mbar_init(tempty, kEpiWarps);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbarrier_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tensormap(&tmA);
    prefetch_tensormap(&tmB);
    prefetch_tensormap(&tmY);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp < 4) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kLowRegs));
    if (warp == 0 && lane == 0) {
      // ---------------------------------------------------------------- TMA producer
      int stage = 0;
      uint32_t phase = 0, armed = 0, armed_parity = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
        int mb, nb;
        tile_mn(t, args, mb, nb);
        for (int kb = 0; kb < KB; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1, abort_flag, kSiteProducerEmpty)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&full[stage], kABytes + kBBytes);
          tma_load_2d(sA + stage * kABytes, &tmA, &full[stage], kb * BK, mb * BM);
          tma_load_2d(sB + stage * kBBytes, &tmB, &full[stage], kb * BK, nb * BN);
          armed |= 1u << stage;
          armed_parity = (armed_parity & ~(1u << stage)) | (phase << stage);
          if (++stage == kStages) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      if (!ok) {
        for (int s = 0; s < kStages; ++s)
          if (armed >> s & 1u) mbar_wait(&full[s], (armed_parity >> s) & 1u, nullptr, kSiteDrain);
      }
    } else if (warp == 2) {
      // ---------------------------------------------------------------- scale factors
      // The CTA's (tile, K-block) steps in order; each step's scales are
      // loaded PD - 1 steps ahead (a ring of register sets), so their latency
      // (about a microsecond under the GEMM's memory load) hides behind the
      // steps before it.  Lane l writes A rows l + 32 c and B rows l + 32 c of
      // both 128-row halves; an absent row's scale loads as 0 (UE8M0 byte 0).
      constexpr int NBV = ROWB ? 8 : 2;
      const int my_tiles = (int)blockIdx.x < total ? (total - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;
      const int steps = my_tiles * KB;
      // the load cursor: tile lt (its position lmb, lnb) and K-block lkb of
      // the next step to load; the tile's position is worked out once per
      // tile, not per step (the raster's divisions would pace this warp)
      int lt = (int)blockIdx.x, lkb = 0, lmb = 0, lnb = 0;
      if (lt < total) tile_mn(lt, args, lmb, lnb);
      auto load = [&](float (&av)[4], float (&bv)[NBV]) {
        const float *sap = args.sa + (int64_t)lkb * args.ldsa + lmb * BM + lane;
        const int m = lmb * BM + lane;
#pragma unroll
        for (int c = 0; c < 4; ++c) av[c] = m + 32 * c < args.M ? __ldg(sap + 32 * c) : 0.f;
        if constexpr (ROWB) {
          const float *sbp = args.sw + (int64_t)lkb * args.ldsw;
          const int n0 = lnb * BN + lane;
#pragma unroll
          for (int c = 0; c < 8; ++c) bv[c] = n0 + 32 * c < args.N ? __ldg(sbp + n0 + 32 * c) : 0.f;
        } else {
          const int wb0 = lnb * 2, wb1 = lnb * 2 + 1;
          bv[0] = wb0 < args.NB ? __ldg(args.sw + (int64_t)wb0 * KB + lkb) : 0.f;
          bv[1] = wb1 < args.NB ? __ldg(args.sw + (int64_t)wb1 * KB + lkb) : 0.f;
        }
        if (++lkb == KB) {
          lkb = 0;
          lt += (int)gridDim.x;
          if (lt < total) tile_mn(lt, args, lmb, lnb);
        }
      };
      constexpr int PD = ROWB ? 2 : 4;  // eight B scales per step with ROWB: fewer steps ahead
      float av[PD][4], bv[PD][NBV];
#pragma unroll
      for (int p = 0; p < PD - 1; ++p)
        if (p < steps) load(av[p], bv[p]);
      float (&a0)[4] = av[0];
      float (&b0)[NBV] = bv[0];
      int stage = 0;
      uint32_t phase = 0;
      for (int s = 0; s < steps; ++s) {
        if (s + PD - 1 < steps) load(av[PD - 1], bv[PD - 1]);
        const bool got = mbar_wait(&empty[stage], phase ^ 1, abort_flag, kSiteProducerEmpty);
        if (!__all_sync(0xffffffffu, got)) break;
        uint8_t *sf = sSF + stage * kSFBytes;
        *reinterpret_cast<uint4 *>(sf + lane * 16) =
            make_uint4(ue8m0x4(a0[0]), ue8m0x4(a0[1]), ue8m0x4(a0[2]), ue8m0x4(a0[3]));
        if constexpr (ROWB) {
          *reinterpret_cast<uint4 *>(sf + kSFABytes + lane * 16) =
              make_uint4(ue8m0x4(b0[0]), ue8m0x4(b0[1]), ue8m0x4(b0[2]), ue8m0x4(b0[3]));
          *reinterpret_cast<uint4 *>(sf + kSFABytes + 512 + lane * 16) =
              make_uint4(ue8m0x4(b0[4]), ue8m0x4(b0[5]), ue8m0x4(b0[6]), ue8m0x4(b0[7]));
        } else {
          const uint32_t w0 = ue8m0x4(b0[0]), w1 = ue8m0x4(b0[1]);
          *reinterpret_cast<uint4 *>(sf + kSFABytes + lane * 16) = make_uint4(w0, w0, w0, w0);
          *reinterpret_cast<uint4 *>(sf + kSFABytes + 512 + lane * 16) = make_uint4(w1, w1, w1, w1);
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&full[stage]);
        if (++stage == kStages) {
          stage = 0;
          phase ^= 1;
        }
#pragma unroll
        for (int p = 0; p < PD - 1; ++p) {
#pragma unroll
          for (int c = 0; c < 4; ++c) av[p][c] = av[p + 1][c];
#pragma unroll
          for (int c = 0; c < NBV; ++c) bv[p][c] = bv[p + 1][c];
        }
      }
    } else if (warp == 1 && lane == 0) {
      // ---------------------------------------------------------------- MMA issuer
      int stage = 0;
      uint32_t phase = 0, tphase = 0;
      bool ok = true, issued = false;
      for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
        if (!mbar_wait(tempty, tphase ^ 1, abort_flag, kSiteMmaTmemEmpty)) {
          ok = false;
          break;
        }
        tphase ^= 1;
        tc_fence_after();
        for (int kb = 0; kb < KB; ++kb) {
          if (!mbar_wait(&full[stage], phase, abort_flag, kSiteMmaFull)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sfa_t = tmem_base + (uint32_t)(kAccCols + stage * kSFCols);
          const uint32_t sfb_t = sfa_t + 4;
          const uint32_t sf_s = smem_addr(sSF + stage * kSFBytes);
          tmem_cp_32x128b_warpx4(sfa_t, smem_desc_k_noswizzle_16B_rows(sf_s));
          tmem_cp_32x128b_warpx4(sfb_t, smem_desc_k_noswizzle_16B_rows(sf_s + kSFABytes));
          tmem_cp_32x128b_warpx4(sfb_t + 4, smem_desc_k_noswizzle_16B_rows(sf_s + kSFABytes + 512));
          const uint32_t a0 = smem_addr(sA + stage * kABytes);
          const uint32_t b0 = smem_addr(sB + stage * kBBytes);
#pragma unroll
          for (int k = 0; k < BK / 32; ++k)
            mma_mxf8f6f4(tmem_base, smem_desc_k_sw128(a0 + 32 * k), smem_desc_k_sw128(b0 + 32 * k),
                         idesc_mxf8f6f4_e4m3_ue8m0(BM, BN, (uint32_t)k, (uint32_t)k), sfa_t, sfb_t,
                         (kb > 0 || k > 0) ? 1u : 0u);
          mma_commit(&empty[stage]);
          issued = true;
          if (++stage == kStages) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (ok) mma_commit(tfull);
      }
      if (!ok && issued) {
        mma_commit(drain);
        mbar_wait(drain, 0, nullptr, kSiteDrain);
      }
    }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kHighRegs));
    // ------------------------------------------------------------------ epilogue
    const int ew = warp - 4;
    const int quarter = warp & 3;
    const int half = ew >> 2;
    uint8_t *ebuf = sEpi + ew * kEpiBufBytes;
    uint32_t tphase = 0;
    for (int t = blockIdx.x; t < total; t += gridDim.x) {
      int mb, nb;
      tile_mn(t, args, mb, nb);
      const bool got = mbar_wait(tfull, tphase, abort_flag, kSiteEpiTmemFull);
      if (!__all_sync(0xffffffffu, got)) break;
      tphase ^= 1;
      tc_fence_after();
      uint32_t r[128];
      const uint32_t taddr = tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(half * 128);
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld_32x32b_x32(taddr + 32 * c, *reinterpret_cast<uint32_t(*)[32]>(&r[32 * c]));
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_relaxed(tempty);  // the next tile's MMAs may overwrite the accumulator
#pragma unroll
      for (int c = 0; c < 4; ++c) {  // four 32-column chunks
        if (lane == 0) bulk_wait_group_read0();
        __syncwarp();
        uint8_t *rowp = ebuf + lane * 64;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const uint32_t *v = &r[32 * c + 8 * j];
          uint4 pk;
          pk.x = pack_bf16x2(__uint_as_float(v[0]), __uint_as_float(v[1]));
          pk.y = pack_bf16x2(__uint_as_float(v[2]), __uint_as_float(v[3]));
          pk.z = pack_bf16x2(__uint_as_float(v[4]), __uint_as_float(v[5]));
          pk.w = pack_bf16x2(__uint_as_float(v[6]), __uint_as_float(v[7]));
          *reinterpret_cast<uint4 *>(rowp + ((j ^ ((lane >> 1) & 3)) << 4)) = pk;
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          const int x = nb * BN + half * 128 + c * 32;
          const int y = mb * BM + quarter * 32;
          if (x < args.N && y < args.M) {
            tma_store_2d(&tmY, ebuf, x, y);
            bulk_commit_group();
          }
        }
      }
    }
    if (lane == 0) bulk_wait_group0();
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

template <bool ROWB>
fp8bq_status native_ready() {
  static DeviceOnce once;  // one per instantiation
  return once.get([](int) {
    cudaFuncAttributes fa;
    cudaError_t e = cudaFuncGetAttributes(&fa, gemm_native_kernel<ROWB>);
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncGetAttributes(gemm_native)");
    if (fa.numRegs != kLaunchRegs) return FP8BQ_ERR_UNSUPPORTED;
    e = cudaFuncSetAttribute(gemm_native_kernel<ROWB>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(gemm_native)");
    return FP8BQ_OK;
  });
}

}  // namespace

cudaError_t take_device_error_native(unsigned long long *v) { return take_tu_device_error(v); }

fp8bq_status launch_gemm_native(const uint8_t *qa, int64_t lda, const float *sa, int64_t ldsa, const uint8_t *qw,
                                int64_t ldw, const float *sw, void *y, int64_t ldy, int64_t M, int64_t N, int64_t K,
                                cudaStream_t stream) {
  CUtensorMap tA, tB, tY;
  if (!make_tmap_2d(&tA, CU_TENSOR_MAP_DATA_TYPE_UINT8, qa, (uint64_t)K, (uint64_t)M, (uint64_t)lda, BK, BM,
                    CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_tmap_2d(&tB, CU_TENSOR_MAP_DATA_TYPE_UINT8, qw, (uint64_t)K, (uint64_t)N, (uint64_t)ldw, BK, BN,
                    CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_tmap_2d(&tY, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, y, (uint64_t)N, (uint64_t)M, (uint64_t)ldy * 2, 32, 32,
                    CU_TENSOR_MAP_SWIZZLE_64B))
    return FP8BQ_ERR_INVALID_ARG;
  const fp8bq_status ready = native_ready<false>();
  if (ready != FP8BQ_OK) return ready;
  NativeArgs a;
  a.sa = sa;
  a.sw = sw;
  a.ldsa = ldsa;
  a.ldsw = 0;
  a.M = (int32_t)M;
  a.N = (int32_t)N;
  a.KB = (int32_t)(K / BK);
  a.NB = (int32_t)((N + 127) / 128);
  a.num_m = (int32_t)((M + BM - 1) / BM);
  a.num_n = (int32_t)((N + BN - 1) / BN);
  choose_raster(M, N, K, BM, BN, &a.band, &a.n_major);
  const int64_t tiles = (int64_t)a.num_m * a.num_n;
  const int grid = (int)std::min<int64_t>(tiles, num_sms());
  gemm_native_kernel<false><<<grid, kThreads, kSmemBytes, stream>>>(tA, tB, tY, a);
  return check_launch("gemm_native");
}

// The weight-gradient GEMM with power-of-two scales on the native block-scaled
// MMA: dW[N][K] = dY^T [N][M] . (X^T [K][M])^T, both operands' 1x128 scales
// along the tokens (A: sa[mb * ldsa + n], B: sb[mb * ldsb + k]).
fp8bq_status launch_gemm_native_wgrad(const uint8_t *qa, int64_t lda, const float *sa, int64_t ldsa,
                                      const uint8_t *qb, int64_t ldb, const float *sb, int64_t ldsb, void *y,
                                      int64_t ldy, int64_t N, int64_t K, int64_t M, cudaStream_t stream) {
  CUtensorMap tA, tB, tY;
  if (!make_tmap_2d(&tA, CU_TENSOR_MAP_DATA_TYPE_UINT8, qa, (uint64_t)M, (uint64_t)N, (uint64_t)lda, BK, BM,
                    CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_tmap_2d(&tB, CU_TENSOR_MAP_DATA_TYPE_UINT8, qb, (uint64_t)M, (uint64_t)K, (uint64_t)ldb, BK, BN,
                    CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_tmap_2d(&tY, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, y, (uint64_t)K, (uint64_t)N, (uint64_t)ldy * 2, 32, 32,
                    CU_TENSOR_MAP_SWIZZLE_64B))
    return FP8BQ_ERR_INVALID_ARG;
  const fp8bq_status ready = native_ready<true>();
  if (ready != FP8BQ_OK) return ready;
  NativeArgs a;
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
  gemm_native_kernel<true><<<grid, kThreads, kSmemBytes, stream>>>(tA, tB, tY, a);
  return check_launch("gemm_native_wgrad");
}

}  // namespace fp8bq
