// Block-scaled FP8 GEMM (FP32 promotion) on CTA pairs: the paired tcgen05
// MMA (cta_group::2) for sm_100a.
//
// Method: "NVIDIA NeMo RL Achieves 48% Speedup With End-to-End FP8 Precision
// Training", section "Technical breakthrough": linear layers in FP8 on
// block-wise quantized E4M3 operands (activations 1x128, weights 128x128),
// every 128-deep K-block's FP32 partial scaled by sa[kb][m] * sw[n/128][kb]
// and added in FP32.
//
// A cluster of two CTAs (one per SM of a TPC) computes a 256x256 output tile.
// CTA r loads rows [128r, 128r+128) of the tile's A block and rows
// [128r, 128r+128) of its B block (256 columns of the output) into its own
// shared memory; the first CTA issues tcgen05.mma.cta_group::2 (256x256x32),
// which reads both CTAs' tiles at the same offsets and writes each CTA's 128
// rows of the partial into that CTA's TMEM.  Compared with one SM computing
// 128x256 tiles, each SM's tensor core reads 8 KB of operands per 32-deep step
// instead of 12 KB, and a stage is 32 KB instead of 48 KB, so the ring is six
// stages deep.
//
// Synchronization (each CTA fetches its own tiles):
//   full[s]   in CTA 0: CTA 0's producer arms it with both CTAs' bytes; both
//             CTAs' TMA loads complete on it.
//   empty[s]  in both CTAs: the MMA's commit arrives on both (multicast).
//   tfull[b]  in both CTAs: the MMA's commit arrives on both (multicast).
//   tempty[b] in CTA 0: all 16 epilogue warps of the pair arrive (CTA 1's
//             remotely).
// Each CTA's epilogue is that of the one-SM kernel: 8 warps, each 32 TMEM
// lanes x 128 columns (one weight block), packed FP32 fma promotion, bf16 out
// through swizzled staging and TMA stores.
#include <cuda_bf16.h>

#include <algorithm>

#include "device.cuh"
#include "internal.h"

namespace fp8bq {
namespace {

constexpr int CBM = 128;                 // A rows per CTA
constexpr int PBM = 2 * CBM;             // rows per pair tile
constexpr int BK = 128;
constexpr int kABytes = CBM * BK;
constexpr int kEpiWarps = 8;
constexpr int kEpiBufBytes = 32 * 128;   // 32 rows x 64 bf16, 128-byte swizzle
constexpr int kThreads = 384;
constexpr int kLaunchRegs = 168;
constexpr int kLowRegs = 56;
constexpr int kHighRegs = 224;
static_assert(128 * kLowRegs + 256 * kHighRegs <= kThreads * kLaunchRegs, "register split");
constexpr int kTmemCols = 512;

// Tile shapes: PBN = 256 (two 256-column TMEM buffers) or PBN = 128 (four
// 128-column buffers, so the MMA can run three K-blocks ahead of the
// promotion warps instead of one).
template <int PBN>
struct PairCfg {
  static constexpr int CBN = PBN / 2;                 // B rows per CTA
  static constexpr int kBBytes = CBN * BK;
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kStages = PBN == 256 ? 6 : 8;
  static constexpr int kBufs = kTmemCols / PBN;       // TMEM accumulator buffers
  static constexpr int kWarpCols = PBN / 2;           // columns per epilogue warp
  static constexpr int kSmemBytes = kStages * kStageBytes + kEpiWarps * kEpiBufBytes + 256 + 1024;
  static_assert(kSmemBytes <= 232448, "shared memory budget");
  static_assert(2 * kStages + 2 * kBufs + 1 <= 28, "barrier area");
};

struct PairArgs {
  const float *sa;
  const float *sw;
  int64_t ldsa;
  int32_t M, N, KB, NB;
  int32_t num_m, num_n;  // pair tiles (256 x 256)
  int32_t band, n_major;  // tile order (raster_tile)
};

__device__ __forceinline__ void pair_tile(int t, const PairArgs &a, int &pm, int &nb) {
  raster_tile(t, a.num_m, a.num_n, a.band, a.n_major, pm, nb);
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t *>(&v);
}

// Leaves time for TMA loads still in flight on the error path (they complete
// in microseconds; the error path is taken only after a one-second wait).
__device__ __forceinline__ void settle() {
  for (int i = 0; i < 64; ++i) __nanosleep(1000);
}

template <int PBN>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                     const __grid_constant__ CUtensorMap tmY, const PairArgs args) {
  using C = PairCfg<PBN>;
  constexpr int CBN = C::CBN, kBBytes = C::kBBytes, kStageBytes = C::kStageBytes, kStages = C::kStages;
  constexpr int kBufs = C::kBufs, kWarpCols = C::kWarpCols;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *sA = base;
  uint8_t *sB = sA + kStages * kABytes;
  uint8_t *sEpi = sB + kStages * kBBytes;
  uint64_t *bars = reinterpret_cast<uint64_t *>(sEpi + kEpiWarps * kEpiBufBytes);
  uint64_t *full = bars;
  uint64_t *empty = full + kStages;
  uint64_t *tfull = empty + kStages;
  uint64_t *tempty = tfull + kBufs;
  uint64_t *drain = tempty + kBufs;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(drain + 1);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const int pair = (int)cluster_id_x(), npairs = (int)nclusters_x();
  const int total = args.num_m * args.num_n;
  const int KB = args.KB;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < kBufs; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], 2 * kEpiWarps);
    }
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
    tmem_alloc_pair(tmem_slot, kTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // both CTAs' barriers exist before any remote arrive or TMA completion
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp < 4) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kLowRegs));
    if (warp == 0 && lane == 0) {
      // ---------------------------------------------------------------- producer (both CTAs)
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int t = pair; t < total && ok; t += npairs) {
        int pm, nb;
        pair_tile(t, args, pm, nb);
        for (int kb = 0; kb < KB; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1, abort_flag, kSiteProducerEmpty)) {
            ok = false;
            break;
          }
          if (rank == 0) mbar_arrive_expect_tx(&full[stage], 2 * kStageBytes);
          const uint32_t bar0 = mapa_shared(smem_addr(&full[stage]), 0);
          tma_load_2d_pair(sA + stage * kABytes, &tmA, bar0, kb * BK, pm * PBM + (int)rank * CBM);
          tma_load_2d_pair(sB + stage * kBBytes, &tmB, bar0, kb * BK, nb * PBN + (int)rank * CBN);
          if (++stage == kStages) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      if (!ok) settle();
    } else if (warp == 1 && lane == 0 && rank == 0) {
      // ---------------------------------------------------------------- MMA issuer (first CTA)
      const uint32_t idesc = idesc_f8f6f4_e4m3_f32(PBM, PBN);
      int stage = 0, buf = 0;
      uint32_t phase = 0, bphase = 0;
      bool ok = true, issued = false;
      for (int t = pair; t < total && ok; t += npairs) {
        for (int kb = 0; kb < KB; ++kb) {
          if (!mbar_wait(&tempty[buf], bphase ^ 1, abort_flag, kSiteMmaTmemEmpty) ||
              !mbar_wait(&full[stage], phase, abort_flag, kSiteMmaFull)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t d = tmem_base + (uint32_t)(buf * PBN);
          const uint32_t a0 = smem_addr(sA + stage * kABytes);
          const uint32_t b0 = smem_addr(sB + stage * kBBytes);
#pragma unroll
          for (int k = 0; k < BK / 32; ++k)
            mma_f8f6f4_pair(d, smem_desc_k_sw128(a0 + 32 * k), smem_desc_k_sw128(b0 + 32 * k), idesc,
                            k > 0 ? 1u : 0u);
          mma_commit_pair_mc(&empty[stage], 0x3);
          mma_commit_pair_mc(&tfull[buf], 0x3);
          issued = true;
          if (++stage == kStages) {
            stage = 0;
            phase ^= 1;
          }
          if (++buf == kBufs) {
            buf = 0;
            bphase ^= 1;
          }
        }
      }
      if (!ok && issued) {  // TMEM and both CTAs' tiles must be quiescent before anyone leaves
        mma_commit_pair_mc(drain, 0x1);
        mbar_wait(drain, 0, nullptr, kSiteDrain);
      }
      if (!ok) settle();
    }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kHighRegs));
    // ------------------------------------------------------------------ promotion + epilogue (both CTAs)
    const int ew = warp - 4;
    const int quarter = warp & 3;
    const int half = ew >> 2;
    const int row = quarter * 32 + lane;
    uint8_t *ebuf = sEpi + ew * kEpiBufBytes;
    const uint32_t tempty0 = mapa_shared(smem_addr(&tempty[0]), 0);
    constexpr int kPairs = kWarpCols / 2;  // accumulator pairs per thread
    int buf = 0;
    uint32_t bphase = 0;
    for (int t = pair; t < total; t += npairs) {
      int pm, nb;
      pair_tile(t, args, pm, nb);
      const int r0 = pm * PBM + (int)rank * CBM;  // this CTA's first row
      const int m = r0 + row;
      const int wn = PBN == 256 ? nb * 2 + half : nb;  // the warp's weight block
      const bool live = m < args.M && wn < args.NB;
      const float *sa_p = args.sa + m;
      const float *sw_p = args.sw + (int64_t)wn * KB;
      float2 acc[kPairs];
#pragma unroll
      for (int j = 0; j < kPairs; ++j) acc[j] = make_float2(0.f, 0.f);
      float a0 = 0.f, w0 = 0.f, a1 = 0.f, w1 = 0.f;
      if (live) {
        a0 = __ldg(sa_p);
        w0 = __ldg(sw_p);
        if (KB > 1) {
          a1 = __ldg(sa_p + args.ldsa);
          w1 = __ldg(sw_p + 1);
        }
      }
      bool ok = true;
      for (int kb = 0; kb < KB; ++kb) {
        const float sc = a0 * w0;
        a0 = a1;
        w0 = w1;
        if (live && kb + 2 < KB) {
          a1 = __ldg(sa_p + (int64_t)(kb + 2) * args.ldsa);
          w1 = __ldg(sw_p + kb + 2);
        }
        const float2 sc2 = make_float2(sc, sc);
        const bool got = mbar_wait(&tfull[buf], bphase, abort_flag, kSiteEpiTmemFull);
        if (!__all_sync(0xffffffffu, got)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t taddr =
            tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(buf * PBN + half * kWarpCols);
#pragma unroll
        for (int c = 0; c < kWarpCols / 64; ++c) {
          uint32_t r[64];
          tmem_ld_32x32b_x32(taddr + 64 * c, *reinterpret_cast<uint32_t(*)[32]>(&r[0]));
          tmem_ld_32x32b_x32(taddr + 64 * c + 32, *reinterpret_cast<uint32_t(*)[32]>(&r[32]));
          tmem_ld_wait();
          if (c == kWarpCols / 64 - 1) {  // this warp's part of the buffer has been read
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
              if (rank == 0) mbar_arrive_relaxed(&tempty[buf]);
              else mbar_arrive_cluster_relaxed(tempty0 + (uint32_t)(buf * sizeof(uint64_t)));
            }
          }
#pragma unroll
          for (int j = 0; j < 32; ++j)
            acc[32 * c + j] =
                __ffma2_rn(make_float2(__uint_as_float(r[2 * j]), __uint_as_float(r[2 * j + 1])), sc2, acc[32 * c + j]);
        }
        if (++buf == kBufs) {
          buf = 0;
          bphase ^= 1;
        }
      }
      if (!ok) break;
#pragma unroll
      for (int c = 0; c < kWarpCols / 64; ++c) {
        if (lane == 0) bulk_wait_group_read0();
        __syncwarp();
        uint8_t *rowp = ebuf + lane * 128;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const float2 *a = &acc[c * 32 + j * 4];
          uint4 pk;
          pk.x = pack_bf16x2(a[0].x, a[0].y);
          pk.y = pack_bf16x2(a[1].x, a[1].y);
          pk.z = pack_bf16x2(a[2].x, a[2].y);
          pk.w = pack_bf16x2(a[3].x, a[3].y);
          *reinterpret_cast<uint4 *>(rowp + ((j ^ (lane & 7)) << 4)) = pk;
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          const int x = nb * PBN + half * kWarpCols + c * 64;
          const int y = r0 + quarter * 32;
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
  cluster_sync();  // the peer's MMAs and reads of this CTA's TMEM / shared memory are over
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, kTmemCols);
  }
}

std::atomic<int> g_pmax_clusters[2][kMaxDevices] = {};  // [tile shape][device], set once the kernel is ready

// Per-device set-up of the pair kernel: register count, shared-memory opt-in
// and the number of clusters of two that fit at once.
template <int PBN>
fp8bq_status pair_ready() {
  static DeviceOnce once;  // one per instantiation
  return once.get([](int dev) {
    constexpr int si = PBN == 256 ? 0 : 1;
    cudaFuncAttributes fa;
    if (cudaFuncGetAttributes(&fa, gemm_pair_kernel<PBN>) != cudaSuccess || fa.numRegs != kLaunchRegs ||
        cudaFuncSetAttribute(gemm_pair_kernel<PBN>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             PairCfg<PBN>::kSmemBytes) != cudaSuccess) {
      cudaGetLastError();
      return FP8BQ_ERR_UNSUPPORTED;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * 128);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = PairCfg<PBN>::kSmemBytes;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int nclusters = 0;
    if (cudaOccupancyMaxActiveClusters(&nclusters, gemm_pair_kernel<PBN>, &cfg) != cudaSuccess || nclusters < 1) {
      cudaGetLastError();
      return FP8BQ_ERR_UNSUPPORTED;
    }
    g_pmax_clusters[si][dev].store(nclusters, std::memory_order_relaxed);
    return FP8BQ_OK;
  });
}

template <int PBN>
fp8bq_status launch_pair(const uint8_t *qa, int64_t lda, const float *sa, int64_t ldsa, const uint8_t *qw,
                         int64_t ldw, const float *sw, void *y, int64_t ldy, int64_t M, int64_t N, int64_t K,
                         cudaStream_t stream) {
  const fp8bq_status ready = pair_ready<PBN>();
  if (ready != FP8BQ_OK) return ready;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  CUtensorMap tA, tB, tY;
  if (!make_tmap_2d(&tA, CU_TENSOR_MAP_DATA_TYPE_UINT8, qa, (uint64_t)K, (uint64_t)M, (uint64_t)lda, BK, CBM,
                    CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_tmap_2d(&tB, CU_TENSOR_MAP_DATA_TYPE_UINT8, qw, (uint64_t)K, (uint64_t)N, (uint64_t)ldw, BK,
                    PairCfg<PBN>::CBN, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_tmap_2d(&tY, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, y, (uint64_t)N, (uint64_t)M, (uint64_t)ldy * 2, 64, 32,
                    CU_TENSOR_MAP_SWIZZLE_128B))
    return FP8BQ_ERR_INVALID_ARG;
  PairArgs a;
  a.sa = sa;
  a.sw = sw;
  a.ldsa = ldsa;
  a.M = (int32_t)M;
  a.N = (int32_t)N;
  a.KB = (int32_t)(K / BK);
  a.NB = (int32_t)((N + 127) / 128);
  a.num_m = (int32_t)((M + PBM - 1) / PBM);
  a.num_n = (int32_t)((N + PBN - 1) / PBN);
  choose_raster(M, N, K, PBM, PBN, &a.band, &a.n_major);
  const int64_t tiles = (int64_t)a.num_m * a.num_n;
  const int si = PBN == 256 ? 0 : 1;
  const int pairs = (int)std::min<int64_t>(
      tiles, std::min(g_pmax_clusters[si][dev].load(std::memory_order_relaxed), num_sms() / 2));
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * pairs);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = PairCfg<PBN>::kSmemBytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, gemm_pair_kernel<PBN>, tA, tB, tY, a);
  if (e != cudaSuccess) return cuda_fail(e, "gemm_pair launch");
  return check_launch("gemm_pair");
}

}  // namespace

bool pair_gemm_available() { return pair_ready<256>() == FP8BQ_OK && pair_ready<128>() == FP8BQ_OK; }

cudaError_t take_device_error_pair(unsigned long long *v) { return take_tu_device_error(v); }

fp8bq_status launch_gemm_pair(const uint8_t *qa, int64_t lda, const float *sa, int64_t ldsa, const uint8_t *qw,
                              int64_t ldw, const float *sw, void *y, int64_t ldy, int64_t M, int64_t N, int64_t K,
                              int tile_n, cudaStream_t stream) {
  if (tile_n == 128) return launch_pair<128>(qa, lda, sa, ldsa, qw, ldw, sw, y, ldy, M, N, K, stream);
  return launch_pair<256>(qa, lda, sa, ldsa, qw, ldw, sw, y, ldy, M, N, K, stream);
}

}  // namespace fp8bq
