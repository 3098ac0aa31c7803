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
// The GEMM runs with the operands swapped so that the tensor cores do useful
// work at small M: the weight is the 128-row MMA operand and the tokens are
// the MMA's N dimension (NT = M rounded up to 16, 32 or 64).  A work item is a
// (128-row weight block nb, 128-deep K-block kb) pair: the weight tile (16 KB)
// comes through a TMA stage ring; 4 x tcgen05.mma 128xNTx32 go into one of
// eight TMEM buffers; the epilogue warps (weight row = TMEM lane, token =
// column) add P * (sa[kb][token] * sw[nb][kb]) into FP32 registers.
//
// Split over K in thread-block clusters: a cluster of S CTAs owns whole weight
// blocks (blocks c, c + C, c + 2C, ... for cluster c of C), and CTA rank r of
// the cluster takes K-blocks [r KB / S, (r + 1) KB / S) of each.  The host
// picks S (1..8) and C so that the largest per-CTA item count is smallest.
// At the end of a block every rank r > 0 leaves its FP32 partial in its own
// shared memory and signals rank 0, which adds the partials in rank order
// (over distributed shared memory: deterministic, no global atomics) and
// writes the bf16 result.
//
// The activation's 1x128 quantization (the device code of fp8bq_quant_act):
//   inside the same kernel when M <= 16 and a CTA's K range holds at most 256
//     1x128 tiles of X: the epilogue warps quantize them into shared memory in
//     the MMA's operand layout while the weight ring fills (one launch);
//   otherwise a prologue kernel writes the codes and scales to the workspace
//     and the producer loads them with TMA beside the weight tiles (M <= 64),
//     or the prologue is followed by the prefill GEMM (M > 64, where the
//     per-token promotion costs more than the weight stream).
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
constexpr int kSwapMaxM = 64;
constexpr int kResMaxM = 16;        // activation quantized inside the GEMM kernel up to this M ...
constexpr int kResMaxTiles = 256;   // ... when a CTA's K range holds at most this many 1x128 tiles of X
constexpr int kMaxResKB = 48;       // K-blocks of resident activation codes per CTA
constexpr int kMaxSplit = 8;        // CTAs of a cluster (split of K)
constexpr int kDEpiWarps = 8;
constexpr int kStageBudget = 212992;
constexpr int kSwSlots = 512;       // weight scales of a CTA's first work items, staged in shared memory

// QM < 0: activation codes and scales come from the workspace (TMA, beside the
// weight tiles); QM = FP8BQ_SCALE_FP32 / POW2: quantized in the kernel (NT = 16).
template <int NT, int QM>
struct DCfg {
  static constexpr bool kRes = QM >= 0;
  static constexpr int kABytes = DBM * DBK;                 // weight tile
  static constexpr int kBBytes = kRes ? 0 : NT * DBK;       // activation-code tile
  static constexpr int kSBytes = kRes ? 0 : NT * 4;         // the K-block's activation scales
  static constexpr int kSSlot = (kSBytes + 127) / 128 * 128;
  static constexpr int kTx = kABytes + kBBytes + kSBytes;
  static constexpr int kResBytes = kRes ? kMaxResKB * (NT * DBK + NT * 4) : 0;
  static constexpr int kPartBytes = NT * DBM * 4;           // a block's FP32 partial, for rank 0 of the cluster
  static constexpr int kFit = (kStageBudget - kResBytes - kPartBytes) / (kABytes + kBBytes + kSSlot);
  static constexpr int kStages = kFit < 8 ? kFit : 8;
  static constexpr int kCW = NT / 2;         // token columns per epilogue warpgroup
  // TMEM accumulator buffers: a work item's partial is only NT columns, so
  // eight of them fit and the MMA can run eight items ahead of the epilogue
  static constexpr int kTBufs = 8;
  static constexpr int kTmemCols = kTBufs * NT;   // 128, 256 or 512: a power of two
  static constexpr int kSmemBytes =
      kStages * (kABytes + kBBytes + kSSlot) + kResBytes + kPartBytes + kSwSlots * 4 + 512 + 1024;
  static_assert(!kRes || NT == kResMaxM, "resident activation codes only for NT = 16");
  static_assert(kStages >= 3 && kSmemBytes <= 232448, "decode shared memory budget");
};

struct DecodeArgs {
  const float *sw;
  int32_t M, N, KB, NB;
  int32_t split;      // CTAs per cluster (S)
  uint16_t *y;        // bf16 bits
  int64_t ldy;
  const uint16_t *x;  // resident quantization: bf16 activations [M][ldx]
  int64_t ldx;
};

// The work of CTA `rank` of cluster `cid` (of `ncl`): weight blocks cid,
// cid + ncl, ... and K-blocks [kb0, kb1) of each; item q is block
// nb0 + (q / nk) * ncl, K-block kb0 + q % nk.
struct Share {
  int nb0, ncl, kb0, kb1, nk, nblk, items;
  __device__ Share(const DecodeArgs &a, int cid, int ncls, int rank) {
    nb0 = cid;
    ncl = ncls;
    kb0 = (int)((int64_t)rank * a.KB / a.split);
    kb1 = (int)((int64_t)(rank + 1) * a.KB / a.split);
    nk = kb1 - kb0;
    nblk = cid < a.NB ? (a.NB - cid + ncls - 1) / ncls : 0;
    items = nblk * nk;
  }
  __device__ int nb(int q) const { return nb0 + (q / nk) * ncl; }
  __device__ int kb(int q) const { return kb0 + q % nk; }
};

__device__ __forceinline__ uint16_t bf16_bits(float v) {
  __nv_bfloat16 b = __float2bfloat16_rn(v);
  return *reinterpret_cast<uint16_t *>(&b);
}

// CH consecutive TMEM columns of this warp's 32 lanes into r[0..CH).
template <int CH>
__device__ __forceinline__ void load_cols(uint32_t taddr, uint32_t *r) {
  if constexpr (CH == 8) {
    tmem_ld_32x32b_x8(taddr, r);
  } else {
    tmem_ld_32x32b_x16(taddr, r);
  }
}

// One 1x128 tile of the activation (row m, K-block kb) quantized by a group of
// four lanes into a resident shared-memory tile of NT = 16 rows x 128 bytes in
// the MMA operand's 128-byte-swizzled layout (16-byte chunk c of row m at
// chunk position c ^ (m & 7)); lane qd of the group owns chunks qd, qd + 4,
// qd + 8, qd + 12 of the row, as fp8bq_quant_act's vector kernel does.
// Every lane of the warp calls it (the amax shuffles span the warp); lanes
// with have == false store nothing.  v: the lane's four 16-byte pieces of the
// row (pieces qd, qd + 4, qd + 8, qd + 12), loaded by the caller.
template <int MODE>
__device__ __forceinline__ void quant_row_tile_to_smem(bool have, const uint4 (&v)[4], int qd, uint8_t *tile, int m,
                                                       float *scale) {
  uint32_t am = max(max(qdev::absmax_bits8(v[0]), qdev::absmax_bits8(v[1])),
                    max(qdev::absmax_bits8(v[2]), qdev::absmax_bits8(v[3])));
  am = max(am, __shfl_xor_sync(0xffffffffu, am, 1));
  am = max(am, __shfl_xor_sync(0xffffffffu, am, 2));
  if (!have) return;
  const qdev::TileScale ts = qdev::tile_scale<MODE>(qdev::bits_to_amax(am));
  uint8_t *row = tile + m * 128;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const int e8 = j * 4 + qd;  // 8-element piece of the row
    const uint2 c = qdev::fast_tile<MODE>(ts) ? qdev::encode8<MODE, true>(v[j], ts) : qdev::encode8<MODE>(v[j], ts);
    *reinterpret_cast<uint2 *>(row + (((e8 >> 1) ^ (m & 7)) << 4) + (e8 & 1) * 8) = c;
  }
  if (qd == 0) *scale = ts.s;
}

template <int NT, int QM>
__global__ void __launch_bounds__(kDThreads, 1)
    decode_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX,
                  const __grid_constant__ CUtensorMap tmS, const DecodeArgs args) {
  using C = DCfg<NT, QM>;
  constexpr bool kRes = C::kRes;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *sA = base;
  uint8_t *sB = sA + C::kStages * C::kABytes;
  uint8_t *sS = sB + C::kStages * C::kBBytes;  // kStages slots of kSSlot bytes (128-byte aligned)
  uint8_t *sXr = sS + C::kStages * C::kSSlot;  // resident codes: kMaxResKB tiles of NT x 128 B
  float *sXs = reinterpret_cast<float *>(sXr + (kRes ? kMaxResKB * NT * DBK : 0));  // [kMaxResKB][NT]
  float *sPart = reinterpret_cast<float *>(sXr + C::kResBytes);  // [NT][128]: this CTA's partial of a block
  float *sSw = sPart + NT * DBM;                                  // [kSwSlots]: sw of items 0, 1, ...
  uint64_t *bars = reinterpret_cast<uint64_t *>(sSw + kSwSlots);
  uint64_t *full = bars;
  uint64_t *empty = bars + C::kStages;
  uint64_t *tfull = empty + C::kStages;
  uint64_t *tempty = tfull + C::kTBufs;
  uint64_t *drain = tempty + C::kTBufs;
  uint64_t *xready = drain + 1;
  uint64_t *red_full = xready + 1;  // rank 0: the other ranks' partials of the current block are in place
  uint64_t *red_free = red_full + 1;  // rank > 0: rank 0 has read this CTA's partial
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(red_free + 1);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int S = args.split;
  const int rank = S > 1 ? (int)cluster_ctarank() : 0;
  const Share sh(args, S > 1 ? (int)cluster_id_x() : (int)blockIdx.x, S > 1 ? (int)nclusters_x() : (int)gridDim.x,
                 rank);

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(&full[s], 1);
      // MMA commit, and with scales in the stage every epilogue warp too
      mbar_init(&empty[s], kRes ? 1 : 1 + kDEpiWarps);
    }
    for (int b = 0; b < C::kTBufs; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], kDEpiWarps);
    }
    mbar_init(drain, 1);
    mbar_init(xready, kDEpiWarps);
    mbar_init(red_full, (S - 1) * kDEpiWarps);
    mbar_init(red_free, kDEpiWarps);
    *abort_flag = 0;
    fence_mbarrier_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tensormap(&tmW);
    if constexpr (!kRes) {
      prefetch_tensormap(&tmX);
      prefetch_tensormap(&tmS);
    }
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  if (S > 1) cluster_sync();  // every CTA's barriers exist before any remote arrive
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp < 4) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kDLowRegs));
    if (warp == 0 && lane == 0) {
      // ---------------------------------------------------------------- producer
      int stage = 0;
      uint32_t phase = 0, armed = 0, armed_parity = 0;
      bool ok = true;
      for (int q = 0; q < sh.items; ++q) {
        const int nb = sh.nb(q), kb = sh.kb(q);
        if (!mbar_wait(&empty[stage], phase ^ 1, abort_flag, kSiteProducerEmpty)) {
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(&full[stage], C::kTx);
        tma_load_2d(sA + stage * C::kABytes, &tmW, &full[stage], kb * DBK, nb * DBM);
        if constexpr (!kRes) {
          tma_load_2d(sB + stage * C::kBBytes, &tmX, &full[stage], kb * DBK, 0);
          tma_load_2d(sS + stage * C::kSSlot, &tmS, &full[stage], 0, kb);
        }
        armed |= 1u << stage;
        armed_parity = (armed_parity & ~(1u << stage)) | (phase << stage);
        if (++stage == C::kStages) {
          stage = 0;
          phase ^= 1;
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
      if constexpr (kRes) ok = mbar_wait(xready, 0, abort_flag, kSiteMmaFull);  // the resident codes are written
      for (int q = 0; q < sh.items && ok; ++q) {
        if (!mbar_wait(&tempty[buf], bphase ^ 1, abort_flag, kSiteMmaTmemEmpty) ||
            !mbar_wait(&full[stage], phase, abort_flag, kSiteMmaFull)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d = tmem_base + (uint32_t)(buf * NT);
        const uint32_t a0 = smem_addr(sA + stage * C::kABytes);
        uint32_t b0 = 0;
        if constexpr (kRes) b0 = smem_addr(sXr + (sh.kb(q) - sh.kb0) * (NT * DBK));
        else b0 = smem_addr(sB + stage * C::kBBytes);
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
        if (++buf == C::kTBufs) {
          buf = 0;
          bphase ^= 1;
        }
      }
      if (!ok && issued) {
        mma_commit(drain);
        mbar_wait(drain, 0, nullptr, kSiteDrain);
      }
    }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kDHighRegs));
    const int et = threadIdx.x - 128;   // 0..255
    // the weight scale of every work item (sw is [NB][KB] row-major): read
    // once, not per item
    for (int q = et; q < kSwSlots && q < sh.items; q += 256)
      sSw[q] = __ldg(args.sw + (int64_t)sh.nb(q) * args.KB + sh.kb(q));
    if constexpr (!kRes) named_barrier_sync(1, 256);
    if constexpr (kRes) {
      // ------------------------------------------------------------ activation quantization
      const int nkb = sh.nk;
      // rows M..NT-1 of every tile are zero (the MMA reads all NT rows)
      for (int z = et; z < nkb * (NT - args.M) * 8; z += 256) {
        const int i = z / ((NT - args.M) * 8), rr = z - i * (NT - args.M) * 8;
        const int m = args.M + rr / 8, c = rr % 8;
        *reinterpret_cast<uint4 *>(sXr + i * (NT * DBK) + m * 128 + c * 16) = make_uint4(0, 0, 0, 0);
      }
      // and so are their scales (only those: rows below M get theirs from the
      // quantization below, which may run first in another warp)
      for (int z = et; z < nkb * (NT - args.M); z += 256) {
        const int i = z / (NT - args.M);
        sXs[i * NT + args.M + (z - i * (NT - args.M))] = 0.f;
      }
      __syncwarp();
      // tile (i, m) for i < nkb, m < M, four lanes each; groups never straddle a
      // warp.  Passes of 64 tiles; the loads of up to kChunk passes are issued
      // together so that their latencies overlap
      constexpr int kChunk = 4;
      const int grp = et >> 2, qd = et & 3;
      const int ntile = nkb * args.M;
      for (int c0 = 0; c0 < ntile; c0 += 64 * kChunk) {
        uint4 v[kChunk][4];
#pragma unroll
        for (int u = 0; u < kChunk; ++u) {
          const int t = c0 + 64 * u + grp;
          const int i = t / args.M, m = t - (t / args.M) * args.M;
          const uint16_t *xrow = args.x + (int64_t)m * args.ldx + (int64_t)(sh.kb0 + i) * DBK;
#pragma unroll
          for (int j = 0; j < 4; ++j) v[u][j] = t < ntile ? ld_nc_v4(xrow + (j * 4 + qd) * 8) : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int u = 0; u < kChunk; ++u) {
          const int t = c0 + 64 * u + grp;
          const bool have = t < ntile;
          const int i = have ? t / args.M : 0, m = have ? t - (t / args.M) * args.M : 0;
          quant_row_tile_to_smem<QM < 0 ? 0 : QM>(have, v[u], qd, sXr + i * (NT * DBK), m, sXs + i * NT + m);
        }
      }
      __syncwarp();
      fence_proxy_async_smem();
      named_barrier_sync(1, 256);  // every tile written (scales are read by all epilogue warps)
      if (lane == 0) mbar_arrive(xready);
    }
    // ------------------------------------------------------------------ epilogue
    const int quarter = warp & 3;
    const int h = (warp - 4) >> 2;
    const int c0 = h * C::kCW;          // first token column of this warpgroup
    const int r = quarter * 32 + lane;  // weight row within the block = output column
    int stage = 0, buf = 0;
    uint32_t bphase = 0, rphase = 0;
    float acc[C::kCW];
#pragma unroll
    for (int j = 0; j < C::kCW; ++j) acc[j] = 0.f;
    for (int q = 0; q < sh.items; ++q) {
      const int kb = sh.kb(q);
      const float w = q < kSwSlots ? sSw[q] : __ldg(args.sw + (int64_t)sh.nb(q) * args.KB + kb);
      const bool got = mbar_wait(&tfull[buf], bphase, abort_flag, kSiteEpiTmemFull);
      if (!__all_sync(0xffffffffu, got)) break;
      tc_fence_after();
      const uint32_t taddr = tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(buf * NT + c0);
      const float4 *sc4;
      if constexpr (kRes) sc4 = reinterpret_cast<const float4 *>(sXs + (kb - sh.kb0) * NT + c0);
      else sc4 = reinterpret_cast<const float4 *>(sS + stage * C::kSSlot) + c0 / 4;
      uint32_t v[C::kCW];
      if constexpr (C::kCW <= 16) {
        load_cols<C::kCW>(taddr, v);
      } else {
        load_cols<16>(taddr, v);
        load_cols<16>(taddr + 16, v + 16);
      }
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_relaxed(&tempty[buf]);
#pragma unroll
      for (int j = 0; j < C::kCW / 4; ++j) {
        const float4 s4 = sc4[j];
        acc[4 * j + 0] = fmaf(__uint_as_float(v[4 * j + 0]), s4.x * w, acc[4 * j + 0]);
        acc[4 * j + 1] = fmaf(__uint_as_float(v[4 * j + 1]), s4.y * w, acc[4 * j + 1]);
        acc[4 * j + 2] = fmaf(__uint_as_float(v[4 * j + 2]), s4.z * w, acc[4 * j + 2]);
        acc[4 * j + 3] = fmaf(__uint_as_float(v[4 * j + 3]), s4.w * w, acc[4 * j + 3]);
      }
      if constexpr (!kRes) {
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[stage]);  // the stage's scales have been read
      }
      if (++stage == C::kStages) stage = 0;
      if (++buf == C::kTBufs) {
        buf = 0;
        bphase ^= 1;
      }
      if (kb != sh.kb1 - 1) continue;
      // ----------------------------------------------- end of this CTA's part of a block
      const int n = sh.nb(q) * DBM + r;
      bool fine = true;
      if (S == 1) {
        if (n < args.N) {
#pragma unroll
          for (int j = 0; j < C::kCW; ++j)
            if (c0 + j < args.M) args.y[(int64_t)(c0 + j) * args.ldy + n] = bf16_bits(acc[j]);
        }
      } else if (rank > 0) {
        // hand the partial to rank 0 through this CTA's shared memory (once
        // rank 0 has read the previous block's)
        fine = mbar_wait_cluster(red_free, rphase ^ 1, abort_flag, kSiteEpiTmemFull);
#pragma unroll
        for (int j = 0; j < C::kCW; ++j) sPart[(c0 + j) * DBM + r] = acc[j];
        asm volatile("fence.acq_rel.cluster;" ::: "memory");
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(mapa_shared(smem_addr(red_full), 0));
        rphase ^= 1;
      } else {
        // rank 0: the sum over the ranks, in rank order
        fine = mbar_wait_cluster(red_full, rphase, abort_flag, kSiteEpiTmemFull);
        rphase ^= 1;
        if (__all_sync(0xffffffffu, fine)) {
          float sum[C::kCW];
#pragma unroll
          for (int j = 0; j < C::kCW; ++j) sum[j] = acc[j];
          for (int pr = 1; pr < S; ++pr) {
            const uint32_t src = mapa_shared(smem_addr(sPart + c0 * DBM + r), (uint32_t)pr);
            float t[C::kCW];
#pragma unroll
            for (int j = 0; j < C::kCW; ++j) t[j] = ld_shared_cluster_f32(src + (uint32_t)(j * DBM * 4));
#pragma unroll
            for (int j = 0; j < C::kCW; ++j) sum[j] += t[j];
          }
          __syncwarp();
          if (lane == 0)  // every rank's partial has been read: its buffer may be reused
            for (int pr = 1; pr < S; ++pr) mbar_arrive_cluster(mapa_shared(smem_addr(red_free), (uint32_t)pr));
          if (n < args.N) {
#pragma unroll
            for (int j = 0; j < C::kCW; ++j)
              if (c0 + j < args.M) args.y[(int64_t)(c0 + j) * args.ldy + n] = bf16_bits(sum[j]);
          }
        }
      }
      if (!__all_sync(0xffffffffu, fine)) break;
#pragma unroll
      for (int j = 0; j < C::kCW; ++j) acc[j] = 0.f;
    }
    // a rank > 0 keeps its shared memory until rank 0 has read its last partial
    if (S > 1 && rank > 0 && sh.nblk > 0) mbar_wait_cluster(red_free, rphase ^ 1, abort_flag, kSiteEpiTmemFull);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::kTmemCols);
  }
  if (S > 1) cluster_sync();  // no CTA leaves while another may still address its shared memory
}

// Prologue: 1x128 quantization of X into the workspace.
template <int MODE, bool VEC>
__global__ void __launch_bounds__(256) decode_prologue_kernel(const uint16_t *__restrict__ x, int64_t M, int64_t K,
                                                              int64_t ldx, uint8_t *__restrict__ q,
                                                              float *__restrict__ sa, int64_t ldsa) {
  if constexpr (VEC) qdev::quant_act_vec_block<MODE>(blockIdx.x, blockIdx.y, x, M, K, ldx, q, K, sa, ldsa);
  else qdev::quant_act_scalar_block<MODE>(blockIdx.x, blockIdx.y, x, M, K, ldx, q, K, sa, ldsa);
}

struct Plan {
  int NT, NB, KB, S, C;   // S CTAs per cluster, C clusters
  bool res;               // activation quantized inside the GEMM kernel (one launch)
  int64_t ldsa;
  size_t off_q, off_sa, total;
};

size_t align256(size_t v) { return (v + 255) & ~size_t(255); }

int pick_nt(int64_t M) {
  if (M <= 16) return 16;
  if (M <= 32) return 32;
  return 64;
}

// The split S (CTAs per cluster, each a contiguous K range of every block of
// its cluster) and the cluster count C that make the largest per-CTA item
// count ceil(NB / C) * ceil(KB / S) smallest with C * S <= SMs; ties go to
// the smaller S (fewer partials to add).
void pick_split(int NB, int KB, int sms, int *S, int *C) {
  int best = 0x7fffffff;
  *S = 1;
  *C = std::min(NB, sms);
  for (int s = 1; s <= kMaxSplit && s <= KB; ++s) {
    const int c = std::min(NB, sms / s);
    if (c < 1) break;
    const int items = ((NB + c - 1) / c) * ((KB + s - 1) / s);
    if (items < best) {
      best = items;
      *S = s;
      *C = c;
    }
  }
}

// vec: the activations allow 16-byte loads (x 16-byte aligned, ldx % 8 == 0).
Plan make_plan(int64_t M, int64_t N, int64_t K, bool vec) {
  Plan p;
  p.NT = M <= kSwapMaxM ? pick_nt(M) : 0;  // 0: the prefill GEMM
  p.NB = (int)((N + 127) / 128);
  p.KB = (int)(K / 128);
  pick_split(p.NB, p.KB, num_sms(), &p.S, &p.C);
  const int nk = (p.KB + p.S - 1) / p.S;    // K-blocks per CTA (at most)
  p.res = p.NT == kResMaxM && vec && nk <= kMaxResKB && nk * M <= kResMaxTiles;
  p.ldsa = (M + 3) / 4 * 4;
  p.off_q = 0;
  p.off_sa = align256((size_t)(M * K));
  p.total = p.res ? 0 : p.off_sa + align256((size_t)p.KB * p.ldsa * 4);
  return p;
}

template <int NT, int QM>
fp8bq_status launch_decode_nt(const CUtensorMap &tW, const CUtensorMap &tX, const CUtensorMap &tS,
                              const DecodeArgs &a, int clusters, cudaStream_t stream) {
  static DeviceOnce once;  // one per instantiation
  const fp8bq_status ready = once.get([](int) {
    cudaFuncAttributes fa;
    cudaError_t e = cudaFuncGetAttributes(&fa, decode_kernel<NT, QM>);
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncGetAttributes(decode)");
    if (fa.numRegs != kDLaunchRegs) return FP8BQ_ERR_UNSUPPORTED;
    e = cudaFuncSetAttribute(decode_kernel<NT, QM>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             DCfg<NT, QM>::kSmemBytes);
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(decode)");
    e = cudaFuncSetAttribute(decode_kernel<NT, QM>, cudaFuncAttributeNonPortableClusterSizeAllowed, 0);
    (void)e;
    return FP8BQ_OK;
  });
  if (ready != FP8BQ_OK) return ready;
  cudaLaunchConfig_t cfg = {};
  cfg.blockDim = dim3(kDThreads);
  cfg.dynamicSmemBytes = DCfg<NT, QM>::kSmemBytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)a.split;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = a.split > 1 ? 1 : 0;
  if (a.split > 1) {
    // no more clusters than can be resident at once (clusters live inside one
    // GPC, so C * S <= SMs alone does not guarantee it): a second wave of
    // clusters would double the time
    static std::atomic<int> max_active[kMaxDevices][kMaxSplit + 1] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    if (dev < 0 || dev >= kMaxDevices) return FP8BQ_ERR_UNSUPPORTED;
    int n = max_active[dev][a.split].load(std::memory_order_relaxed);
    if (n == 0) {
      cfg.gridDim = dim3((unsigned)(a.split * 256));
      e = cudaOccupancyMaxActiveClusters(&n, decode_kernel<NT, QM>, &cfg);
      if (e != cudaSuccess || n < 1) {
        cudaGetLastError();
        return e != cudaSuccess ? cuda_fail(e, "cudaOccupancyMaxActiveClusters(decode)") : FP8BQ_ERR_UNSUPPORTED;
      }
      max_active[dev][a.split].store(n, std::memory_order_relaxed);
    }
    clusters = std::min(clusters, n);
  }
  cfg.gridDim = dim3((unsigned)(clusters * a.split));
  cudaError_t e = cudaLaunchKernelEx(&cfg, decode_kernel<NT, QM>, tW, tX, tS, a);
  if (e != cudaSuccess) return cuda_fail(e, "gemm_decode launch");
  return check_launch("gemm_decode");
}

bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

}  // namespace

cudaError_t take_device_error_decode(unsigned long long *v) { return take_tu_device_error(v); }

size_t decode_workspace_size(int64_t M, int64_t N, int64_t K) {
  if (M <= 0 || N <= 0 || K <= 0 || M > kMaxDecodeM || K % 128 != 0) return 0;
  return make_plan(M, N, K, false).total;  // the larger of the two plans
}

fp8bq_status launch_gemm_decode(const void *x, int64_t ldx, const uint8_t *qw, int64_t ldw, const float *sw, void *y,
                                int64_t ldy, int64_t M, int64_t N, int64_t K, int mode, void *ws, size_t ws_bytes,
                                cudaStream_t stream) {
  if (M > kMaxDecodeM) return FP8BQ_ERR_UNSUPPORTED;
  const bool vec = aligned(x, 16) && ldx % 8 == 0;  // K % 128 == 0 already
  const Plan p = make_plan(M, N, K, vec);
  // the documented size (the larger plan's), whichever path this call takes
  const size_t need = make_plan(M, N, K, false).total;
  if (ws_bytes < need || (need > 0 && (ws == nullptr || !aligned(ws, 256)))) return FP8BQ_ERR_WORKSPACE;
  uint8_t *wsb = static_cast<uint8_t *>(ws);
  uint8_t *q = wsb + p.off_q;
  float *sa = reinterpret_cast<float *>(wsb + p.off_sa);
  const uint16_t *xs = static_cast<const uint16_t *>(x);

  // 1. quantize X into the workspace, unless the GEMM kernel does it
  if (!p.res) {
    if (vec) {
      dim3 grid((unsigned)((M + 63) / 64), (unsigned)p.KB);
      if (mode == FP8BQ_SCALE_FP32)
        decode_prologue_kernel<FP8BQ_SCALE_FP32, true><<<grid, 256, 0, stream>>>(xs, M, K, ldx, q, sa, p.ldsa);
      else
        decode_prologue_kernel<FP8BQ_SCALE_POW2, true><<<grid, 256, 0, stream>>>(xs, M, K, ldx, q, sa, p.ldsa);
    } else {
      dim3 grid((unsigned)((M + 15) / 16), (unsigned)p.KB);
      if (mode == FP8BQ_SCALE_FP32)
        decode_prologue_kernel<FP8BQ_SCALE_FP32, false><<<grid, 256, 0, stream>>>(xs, M, K, ldx, q, sa, p.ldsa);
      else
        decode_prologue_kernel<FP8BQ_SCALE_POW2, false><<<grid, 256, 0, stream>>>(xs, M, K, ldx, q, sa, p.ldsa);
    }
    fp8bq_status st = check_launch("gemm_decode prologue");
    if (st != FP8BQ_OK) return st;
    if (p.NT == 0)  // M > 64: the prefill GEMM on the quantized activation
      return launch_gemm(q, K, sa, p.ldsa, qw, ldw, sw, y, ldy, M, N, K, mode, FP8BQ_GEMM_AUTO, stream);
  }

  // 2. the GEMM, K split over the CTAs of each cluster
  CUtensorMap tW, tX, tS;
  if (!make_tmap_2d(&tW, CU_TENSOR_MAP_DATA_TYPE_UINT8, qw, (uint64_t)K, (uint64_t)N, (uint64_t)ldw, DBK, DBM,
                    CU_TENSOR_MAP_SWIZZLE_128B))
    return FP8BQ_ERR_INVALID_ARG;
  if (p.res) {
    tX = tW;  // not read by the kernel
    tS = tW;
  } else if (!make_tmap_2d(&tX, CU_TENSOR_MAP_DATA_TYPE_UINT8, q, (uint64_t)K, (uint64_t)M, (uint64_t)K, DBK,
                           (uint32_t)p.NT, CU_TENSOR_MAP_SWIZZLE_128B) ||
             !make_tmap_2d(&tS, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, sa, (uint64_t)M, (uint64_t)p.KB,
                           (uint64_t)p.ldsa * 4, (uint32_t)p.NT, 1, CU_TENSOR_MAP_SWIZZLE_NONE)) {
    return FP8BQ_ERR_INVALID_ARG;
  }
  DecodeArgs a;
  a.sw = sw;
  a.M = (int32_t)M;
  a.N = (int32_t)N;
  a.KB = p.KB;
  a.NB = p.NB;
  a.split = p.S;
  a.y = static_cast<uint16_t *>(y);
  a.ldy = ldy;
  a.x = xs;
  a.ldx = ldx;
  if (p.res)
    return mode == FP8BQ_SCALE_FP32 ? launch_decode_nt<16, FP8BQ_SCALE_FP32>(tW, tX, tS, a, p.C, stream)
                                    : launch_decode_nt<16, FP8BQ_SCALE_POW2>(tW, tX, tS, a, p.C, stream);
  switch (p.NT) {
    case 16: return launch_decode_nt<16, -1>(tW, tX, tS, a, p.C, stream);
    case 32: return launch_decode_nt<32, -1>(tW, tX, tS, a, p.C, stream);
    default: return launch_decode_nt<64, -1>(tW, tX, tS, a, p.C, stream);
  }
}

}  // namespace fp8bq
