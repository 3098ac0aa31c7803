// Decode-shaped (small M, memory-bound) block-scaled FP8 linear for sm_100a:
// Y[M,N] = q(X)[M,K] . W[N,K]^T with the activation quantized on the fly
// (1x128 tiles) and W pre-quantized (128x128 tiles).  This file holds the
// call's routing (the wide form of decode_wide.cu up to M = 64 by default,
// the prefill GEMM above), the prologue quantization kernel and the narrow
// form below, which FP8BQ_DECODE_KERNEL=narrow selects.
//
// Method: "NVIDIA NeMo RL Achieves 48% Speedup With End-to-End FP8 Precision
// Training", section "Technical breakthrough": FP8 is applied in generation as
// well as in training, with block-wise E4M3 (activations 1x128, weights
// 128x128).  In generation the linear layers see a handful of tokens, so the
// time goes into streaming the weight from HBM.
//
// The narrow form runs with the operands swapped so that the tensor cores do
// useful work at small M: the weight is the 128-row MMA operand and the tokens are
// the MMA's N dimension (NT = M rounded up to 16, 32 or 64).  A work item is a
// (128-row weight block nb, 128-deep K-block kb) pair: the weight tile (16 KB)
// comes through a TMA stage ring; 4 x tcgen05.mma 128xNTx32 go into one of
// eight TMEM buffers; the epilogue warps (weight row = TMEM lane, token =
// column) add P * (sa[kb][token] * sw[nb][kb]) into FP32 registers.
//
// Split over K in thread-block clusters: a cluster of S CTAs owns whole weight
// blocks (blocks c, c + C, c + 2C, ... for cluster c of C), and CTA rank r of
// the cluster takes K-blocks r, r + S, r + 2S, ... of each.  The host picks S
// (1..8) and C from a time model (the busiest CTA's items against the HBM's
// share, plus the cost of the cross-CTA sum).  At the end of a block every
// rank r > 0 leaves its FP32 partial in its own shared memory and signals
// rank 0, which adds the partials in rank order (over distributed shared
// memory: deterministic, no global atomics) and writes the bf16 result; rank
// 0 does so one block late, so that the wait for the other ranks overlaps its
// next block's items.
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
#include <stdlib.h>
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
constexpr int kWideMaxNTiles = 16;
constexpr int kResMaxM = 16;        // activation quantized inside the GEMM kernel up to this M ...
constexpr int kResMaxTiles = 256;   // ... when a CTA's K range holds at most this many 1x128 tiles of X
constexpr int kMaxSplit = 8;        // CTAs of a cluster (split of K)
// Split choice, in units of one work item's time: an SM's TMA stream of
// weight tiles runs at about one 16 KB tile per half microsecond whatever the
// number of stages in flight (so the busiest CTA's item count sets the time),
// and the cross-CTA sum of a split block costs about kRedItems.
constexpr int kRedItems = 2;
constexpr int kDEpiWarps = 8;
constexpr int kSmemCap = 232448;    // dynamic shared memory per CTA (227 KB)
constexpr int kMaxStages = 16;      // weight stages: as many as the shared memory left over holds
constexpr int kMinStages = 4;
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
  static constexpr int kStageBytes = kABytes + kBBytes + kSSlot;
  static constexpr int kTx = kABytes + kBBytes + kSBytes;
  static constexpr int kResTile = NT * DBK;                 // resident codes of one K-block
  static constexpr int kCW = NT / 2;         // token columns per epilogue warpgroup
  // TMEM accumulator buffers: a work item's partial is only NT columns, so
  // eight of them fit and the MMA can run eight items ahead of the epilogue
  static constexpr int kTBufs = 8;
  static constexpr int kTmemCols = kTBufs * NT;   // 128, 256 or 512: a power of two
  static_assert(!kRes || NT == kResMaxM, "resident activation codes only for NT = 16");

  // Shared memory: nst stages, then nres resident K-blocks of activation codes
  // (1024-byte aligned, the swizzle atom) and their scales, the slots for the
  // other ranks' partials, the staged weight scales and the barriers; 1024
  // bytes of alignment slack.
  static __host__ __device__ int res_code_bytes(int nres) { return (nres * kResTile + 1023) / 1024 * 1024; }
  static int smem_bytes(int nst, int nres, int slot_bytes) {
    return 1024 + nst * kStageBytes + res_code_bytes(nres) + nres * NT * 4 + slot_bytes + kSwSlots * 4 + 512;
  }
  // the most stages that fit beside the rest (0 if fewer than kMinStages)
  static int stages_for(int nres, int slot_bytes) {
    const int n = (kSmemCap - smem_bytes(0, nres, slot_bytes)) / kStageBytes;
    return n < kMinStages ? 0 : (n > kMaxStages ? kMaxStages : n);
  }
};

struct DecodeArgs {
  const float *sw;
  int32_t M, N, KB, NB;
  int32_t split;      // CTAs per cluster (S)
  int32_t nst;        // weight stages (kMinStages..kMaxStages)
  int32_t nres;       // resident K-blocks of activation codes (0 unless quantized in the kernel)
  uint16_t *y;        // bf16 bits
  int64_t ldy;
  const uint16_t *x;  // resident quantization: bf16 activations [M][ldx]
  int64_t ldx;
};

// The work of CTA `rank` of cluster `cid` (of `ncl`): weight blocks cid,
// cid + ncl, ... and of each the K-blocks rank, rank + S, rank + 2S, ...
// (interleaved, so that the S CTAs of a cluster stream neighbouring 128-byte
// pieces of the same weight rows at the same time); item q is block
// nb0 + (q / nk) * ncl, K-block kb0 + (q % nk) * S, at position q % nk of
// the CTA's part of the block.
struct Share {
  int nb0, ncl, kb0, ks, nk, nblk, items;
  __device__ Share(const DecodeArgs &a, int cid, int ncls, int rank) {
    nb0 = cid;
    ncl = ncls;
    kb0 = rank;
    ks = a.split;
    nk = (a.KB - rank + a.split - 1) / a.split;
    nblk = cid < a.NB ? (a.NB - cid + ncls - 1) / ncls : 0;
    items = nblk * nk;
  }
  __device__ int nb(int q) const { return nb0 + (q / nk) * ncl; }
  __device__ int pos(int q) const { return q % nk; }
  __device__ int kb(int q) const { return kb0 + (q % nk) * ks; }
  __device__ bool last(int q) const { return q % nk == nk - 1; }  // the CTA's last item of the block
};

// The cross-CTA sum of a split block (S > 1): every rank > 0 keeps its
// NT x 128 FP32 partial in its own shared memory (two buffers: consecutive
// blocks) and rank 0 reads them over distributed shared memory.
__host__ __device__ __forceinline__ int red_floats(int NT, int S) { return S <= 1 ? 0 : 2 * NT * DBM; }

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

template <int NT, int QM>
__global__ void __launch_bounds__(kDThreads, 1)
    decode_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX,
                  const __grid_constant__ CUtensorMap tmS, const DecodeArgs args) {
  using C = DCfg<NT, QM>;
  constexpr bool kRes = C::kRes;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int nst = args.nst;
  uint8_t *sA = base;
  uint8_t *sB = sA + nst * C::kABytes;
  uint8_t *sS = sB + nst * C::kBBytes;         // nst slots of kSSlot bytes (128-byte aligned)
  uint8_t *sXr = base + nst * C::kStageBytes;  // resident codes: nres tiles of NT x 128 B (1024-aligned)
  float *sXs = reinterpret_cast<float *>(sXr + C::res_code_bytes(args.nres));  // [nres][NT]
  // [2][NT][128]: this CTA's partials of blocks jb (buffer jb % 2), token column-major
  float *sRed = sXs + args.nres * NT;
  float *sSw = sRed + red_floats(NT, args.split);  // [kSwSlots]: sw of items 0, 1, ...
  uint64_t *bars = reinterpret_cast<uint64_t *>(sSw + kSwSlots);
  uint64_t *full = bars;
  uint64_t *empty = bars + kMaxStages;
  uint64_t *tfull = empty + kMaxStages;
  uint64_t *tempty = tfull + C::kTBufs;
  uint64_t *drain = tempty + C::kTBufs;
  uint64_t *xready = drain + 1;      // resident activation codes written
  uint64_t *red_full = xready + 1;  // [2] rank 0: the other ranks' partials of block jb are in buffer jb % 2
  uint64_t *red_free = red_full + 2;  // [2] rank > 0: rank 0 has read buffer jb % 2 (this CTA may write it)
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(red_free + 2);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int S = args.split;
  const int rank = S > 1 ? (int)cluster_ctarank() : 0;
  const Share sh(args, S > 1 ? (int)cluster_id_x() : (int)blockIdx.x, S > 1 ? (int)nclusters_x() : (int)gridDim.x,
                 rank);

  // The epilogue warps issue the first pass of the activation's loads (with
  // the activation quantized here) and the weight scales' loads before the
  // set-up below, so that they reach memory ahead of the weight stream and
  // overlap the set-up (the MMA cannot start before they are back).
  constexpr int kChunk = 4;     // passes of 64 1x128 tiles whose loads are issued together
  const int et = threadIdx.x - 128;   // epilogue thread 0..255
  const int grp = et >> 2, qd = et & 3;
  uint4 xv[kChunk][4];
  float swv[kSwSlots / 256];
  // the four lanes of tile t = c0 + 64 u + grp (K-block i = t / M, row m)
  auto load_pass = [&](int c0, uint4 (&v)[kChunk][4]) {
    const int ntile = sh.nk * args.M;
#pragma unroll
    for (int u = 0; u < kChunk; ++u) {
      const int t = c0 + 64 * u + grp;
      const int i = t / args.M, m = t - (t / args.M) * args.M;
      const uint16_t *xrow = args.x + (int64_t)m * args.ldx + (int64_t)(sh.kb0 + i * sh.ks) * DBK;
#pragma unroll
      for (int j = 0; j < 4; ++j) v[u][j] = t < ntile ? ld_nc_v4(xrow + (j * 4 + qd) * 8) : make_uint4(0, 0, 0, 0);
    }
  };
  if (warp >= 4) {
    if constexpr (kRes) load_pass(0, xv);
#pragma unroll
    for (int i = 0; i < kSwSlots / 256; ++i) {
      const int q = et + 256 * i;
      swv[i] = q < sh.items ? __ldg(args.sw + (int64_t)sh.nb(q) * args.KB + sh.kb(q)) : 0.f;
    }
  }

  if (threadIdx.x == 0) {
    for (int s = 0; s < nst; ++s) {
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
    for (int b = 0; b < 2; ++b) {
      mbar_init(&red_full[b], (S - 1) * kDEpiWarps);  // every epilogue warp of the other ranks
      mbar_init(&red_free[b], kDEpiWarps);
    }
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
      for (int q = 0; q < sh.items && ok; ++q) {
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
        if (++stage == nst) {
          stage = 0;
          phase ^= 1;
        }
      }
      if (!ok) {
        for (int s = 0; s < nst; ++s)
          if (armed >> s & 1u) mbar_wait(&full[s], (armed_parity >> s) & 1u, nullptr, kSiteDrain);
      }
    } else if (warp == 1 && lane == 0) {
      // ---------------------------------------------------------------- MMA issuer
      const uint32_t idesc = idesc_f8f6f4_e4m3_f32(DBM, NT);
      int stage = 0, buf = 0;
      uint32_t phase = 0, bphase = 0;
      bool ok = true, issued = false;
      if constexpr (kRes) ok = mbar_wait(xready, 0, abort_flag, kSiteMmaFull);  // the resident codes are written
      // The four K-steps of one item accumulate into one TMEM buffer, so each
      // waits for the one before; the tensor pipe is kept busy by issuing the
      // K-steps of up to kMmaGroup items interleaved (items whose weight tile
      // and TMEM buffer are already available join the first one).
      constexpr int kMmaGroup = 4;
      for (int q = 0; q < sh.items && ok;) {
        uint32_t d[kMmaGroup], a0[kMmaGroup], b0[kMmaGroup];
        int st_of[kMmaGroup], bf_of[kMmaGroup];
        int g = 0;
        for (; g < kMmaGroup && q + g < sh.items; ++g) {
          if (g == 0) {
            if (!mbar_wait(&tempty[buf], bphase ^ 1, abort_flag, kSiteMmaTmemEmpty) ||
                !mbar_wait(&full[stage], phase, abort_flag, kSiteMmaFull)) {
              ok = false;
              break;
            }
          } else if (!mbar_test_wait(&tempty[buf], bphase ^ 1) || !mbar_test_wait(&full[stage], phase)) {
            break;
          }
          d[g] = tmem_base + (uint32_t)(buf * NT);
          a0[g] = smem_addr(sA + stage * C::kABytes);
          if constexpr (kRes) b0[g] = smem_addr(sXr + sh.pos(q + g) * (NT * DBK));
          else b0[g] = smem_addr(sB + stage * C::kBBytes);
          st_of[g] = stage;
          bf_of[g] = buf;
          if (++stage == nst) {
            stage = 0;
            phase ^= 1;
          }
          if (++buf == C::kTBufs) {
            buf = 0;
            bphase ^= 1;
          }
        }
        if (!ok) break;
        tc_fence_after();
#pragma unroll
        for (int k = 0; k < DBK / 32; ++k)
#pragma unroll
          for (int i = 0; i < kMmaGroup; ++i)
            if (i < g)
              mma_f8f6f4(d[i], smem_desc_k_sw128(a0[i] + 32 * k), smem_desc_k_sw128(b0[i] + 32 * k), idesc,
                         k > 0 ? 1u : 0u);
#pragma unroll
        for (int i = 0; i < kMmaGroup; ++i) {
          if (i < g) {
            mma_commit(&empty[st_of[i]]);
            mma_commit(&tfull[bf_of[i]]);
          }
        }
        issued = true;
        q += g;
      }
      if (!ok && issued) {
        mma_commit(drain);
        mbar_wait(drain, 0, nullptr, kSiteDrain);
      }
    }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kDHighRegs));
    // the weight scale of every work item (sw is [NB][KB] row-major), read
    // once, not per item (loaded above)
    auto store_sw = [&]() {
#pragma unroll
      for (int i = 0; i < kSwSlots / 256; ++i)
        if (et + 256 * i < sh.items) sSw[et + 256 * i] = swv[i];
    };
    if constexpr (!kRes) {
      store_sw();
      named_barrier_sync(1, 256);
    }
    if constexpr (kRes) {
      // ------------------------------------------------------------ activation quantization
      // tile (i, m) for i < nk, m < M, four lanes each; groups never straddle a
      // warp.  Passes of 64 tiles, the loads of kChunk passes issued together
      // so that their latencies overlap (the first ones before the set-up)
      const int nkb = sh.nk;
      const int ntile = nkb * args.M;
      for (int c0 = 0; c0 < ntile || c0 == 0; c0 += 64 * kChunk) {
        uint4 v[kChunk][4];
        if (c0 == 0) {
#pragma unroll
          for (int u = 0; u < kChunk; ++u)
#pragma unroll
            for (int j = 0; j < 4; ++j) v[u][j] = xv[u][j];
          // rows M..NT-1 of every tile are zero (the MMA reads all NT rows),
          // and so are their scales (only those: rows below M get theirs from
          // the quantization, which may run first in another warp)
          for (int z = et; z < nkb * (NT - args.M) * 8; z += 256) {
            const int i = z / ((NT - args.M) * 8), rr = z - i * (NT - args.M) * 8;
            const int m = args.M + rr / 8, c = rr % 8;
            *reinterpret_cast<uint4 *>(sXr + i * (NT * DBK) + m * 128 + c * 16) = make_uint4(0, 0, 0, 0);
          }
          for (int z = et; z < nkb * (NT - args.M); z += 256) {
            const int i = z / (NT - args.M);
            sXs[i * NT + args.M + (z - i * (NT - args.M))] = 0.f;
          }
          store_sw();
        } else {
          load_pass(c0, v);
        }
#pragma unroll
        for (int u = 0; u < kChunk; ++u) {
          const int t = c0 + 64 * u + grp;
          const bool have = t < ntile;
          const int i = have ? t / args.M : 0, m = have ? t - (t / args.M) * args.M : 0;
          qdev::quant_row_tile_to_smem<QM < 0 ? 0 : QM>(have, v[u], qd, sXr + i * (NT * DBK), m, sXs + i * NT + m);
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
    uint32_t bphase = 0;
    float acc[C::kCW], prev[C::kCW];
#pragma unroll
    for (int j = 0; j < C::kCW; ++j) acc[j] = prev[j] = 0.f;
    auto store_y = [&](int jb, const float (&v)[C::kCW]) {
      const int n = (sh.nb0 + jb * sh.ncl) * DBM + r;
      if (n < args.N) {
#pragma unroll
        for (int j = 0; j < C::kCW; ++j)
          if (c0 + j < args.M) args.y[(int64_t)(c0 + j) * args.ldy + n] = bf16_bits(v[j]);
      }
    };
    // Rank 0: block jb's sum over the ranks, in rank order (its own partial
    // `own`, then ranks 1 .. S-1 from its slots jb % 2), written to Y.
    auto reduce = [&](int jb, const float (&own)[C::kCW]) -> bool {
      const int pb = jb & 1;
      const bool got = mbar_wait_cluster(&red_full[pb], (uint32_t)((jb >> 1) & 1), abort_flag, kSiteEpiTmemFull);
      if (!__all_sync(0xffffffffu, got)) return false;
      float sum[C::kCW];
#pragma unroll
      for (int j = 0; j < C::kCW; ++j) sum[j] = own[j];
      // the live token columns, eight at a time: every rank's loads issued
      // before the first add (one round trip), then added in rank order
      constexpr int kJC = C::kCW < 8 ? C::kCW : 8;
#pragma unroll
      for (int j0 = 0; j0 < C::kCW; j0 += kJC) {
        if (c0 + j0 >= args.M) break;
        float t[kMaxSplit - 1][kJC];
#pragma unroll
        for (int pr = 1; pr < kMaxSplit; ++pr) {
          if (pr >= S) break;
          const uint32_t src = mapa_shared(smem_addr(sRed + pb * (NT * DBM) + (c0 + j0) * DBM + r), (uint32_t)pr);
#pragma unroll
          for (int j = 0; j < kJC; ++j) t[pr - 1][j] = ld_shared_cluster_f32(src + (uint32_t)(j * DBM * 4));
        }
#pragma unroll
        for (int pr = 1; pr < kMaxSplit; ++pr) {
          if (pr >= S) break;
#pragma unroll
          for (int j = 0; j < kJC; ++j) sum[j0 + j] += t[pr - 1][j];
        }
      }
      // the partials have been read (their values are in registers): the
      // other ranks may fill the buffer again
      __syncwarp();
      if (lane == 0)
        for (int pr = 1; pr < S; ++pr)
          mbar_arrive_cluster_relaxed(mapa_shared(smem_addr(&red_free[pb]), (uint32_t)pr));
      store_y(jb, sum);
      return true;
    };
    bool alive = true;
    auto sw_of = [&](int q) -> float {
      return q < kSwSlots ? sSw[q] : __ldg(args.sw + (int64_t)sh.nb(q) * args.KB + sh.kb(q));
    };
    // acc[j] += P[j] * (sa[token j] * w) for one item's TMEM partial v
    auto promote = [&](const uint32_t (&v)[C::kCW], int pos, int st, float w) {
      const float4 *sc4;
      if constexpr (kRes) sc4 = reinterpret_cast<const float4 *>(sXs + pos * NT + c0);
      else sc4 = reinterpret_cast<const float4 *>(sS + st * C::kSSlot) + c0 / 4;
#pragma unroll
      for (int j = 0; j < C::kCW / 4; ++j) {
        const float4 s4 = sc4[j];
        acc[4 * j + 0] = fmaf(__uint_as_float(v[4 * j + 0]), s4.x * w, acc[4 * j + 0]);
        acc[4 * j + 1] = fmaf(__uint_as_float(v[4 * j + 1]), s4.y * w, acc[4 * j + 1]);
        acc[4 * j + 2] = fmaf(__uint_as_float(v[4 * j + 2]), s4.z * w, acc[4 * j + 2]);
        acc[4 * j + 3] = fmaf(__uint_as_float(v[4 * j + 3]), s4.w * w, acc[4 * j + 3]);
      }
    };
    auto load_item = [&](int b, uint32_t (&v)[C::kCW]) {
      const uint32_t taddr = tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(b * NT + c0);
      if constexpr (C::kCW <= 16) {
        load_cols<C::kCW>(taddr, v);
      } else {
        load_cols<16>(taddr, v);
        load_cols<16>(taddr + 16, v + 16);
      }
    };
    for (int q = 0; q < sh.items;) {
      const int pos = sh.pos(q);
      // two items of the same block at once: their TMEM loads share one wait
      // (the promotion still adds them in item order)
      const bool two = !sh.last(q) && q + 1 < sh.items;
      const int buf1 = buf + 1 == C::kTBufs ? 0 : buf + 1;
      const uint32_t bphase1 = buf + 1 == C::kTBufs ? bphase ^ 1 : bphase;
      const int stage1 = stage + 1 == nst ? 0 : stage + 1;
      const float w0 = sw_of(q), w1 = two ? sw_of(q + 1) : 0.f;
      bool got = mbar_wait(&tfull[buf], bphase, abort_flag, kSiteEpiTmemFull);
      if (two && got) got = mbar_wait(&tfull[buf1], bphase1, abort_flag, kSiteEpiTmemFull);
      if (!__all_sync(0xffffffffu, got)) {
        alive = false;
        break;
      }
      tc_fence_after();
      uint32_t v0[C::kCW], v1[C::kCW];
      load_item(buf, v0);
      if (two) load_item(buf1, v1);
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive_relaxed(&tempty[buf]);
        if (two) mbar_arrive_relaxed(&tempty[buf1]);
      }
      promote(v0, pos, stage, w0);
      if (two) promote(v1, pos + 1, stage1, w1);
      if constexpr (!kRes) {
        __syncwarp();
        if (lane == 0) {  // the stages' scales have been read
          mbar_arrive(&empty[stage]);
          if (two) mbar_arrive(&empty[stage1]);
        }
      }
      const int n_done = two ? 2 : 1;
      for (int i = 0; i < n_done; ++i) {
        if (++stage == nst) stage = 0;
        if (++buf == C::kTBufs) {
          buf = 0;
          bphase ^= 1;
        }
      }
      q += n_done;
      if (!sh.last(q - 1)) continue;
      // ----------------------------------------------- end of this CTA's part of block jb
      const int jb = (q - 1) / sh.nk;
      bool fine = true;
      if (S == 1) {
        store_y(jb, acc);
      } else if (rank > 0) {
        // hand the partial to rank 0 in buffer jb % 2, once rank 0 has read
        // block jb - 2 there
        const int pb = jb & 1;
        fine = mbar_wait_cluster(&red_free[pb], (uint32_t)(((jb >> 1) & 1) ^ 1), abort_flag, kSiteEpiTmemFull);
        if (__all_sync(0xffffffffu, fine)) {
#pragma unroll
          for (int j = 0; j < C::kCW; ++j) sRed[pb * (NT * DBM) + (c0 + j) * DBM + r] = acc[j];
          asm volatile("fence.acq_rel.cluster;" ::: "memory");
          __syncwarp();
          if (lane == 0) mbar_arrive_cluster(mapa_shared(smem_addr(&red_full[pb]), 0));
        }
      } else {
        // rank 0 adds up block jb - 1 now (its peers have had a block's time
        // to deliver their partials) and keeps block jb's own partial
        if (jb > 0) fine = reduce(jb - 1, prev);
#pragma unroll
        for (int j = 0; j < C::kCW; ++j) prev[j] = acc[j];
      }
      if (!__all_sync(0xffffffffu, fine)) {
        alive = false;
        break;
      }
#pragma unroll
      for (int j = 0; j < C::kCW; ++j) acc[j] = 0.f;
    }
    if (S > 1 && sh.nblk > 0 && alive && rank == 0) reduce(sh.nblk - 1, prev);  // the last block
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::kTmemCols);
  }
  if (S > 1) cluster_sync();  // no CTA leaves while another may still address its shared memory
}

// Prologue: 1x128 quantization of X into the workspace.  Launched as a
// programmatic dependent (it waits for the previous kernel before touching
// memory) and lets the GEMM kernel that follows start its set-up at once.
template <int MODE, bool VEC>
__global__ void __launch_bounds__(256) decode_prologue_kernel(const uint16_t *__restrict__ x, int64_t M, int64_t K,
                                                              int64_t ldx, uint8_t *__restrict__ q,
                                                              float *__restrict__ sa, int64_t ldsa) {
  pdl_launch_dependents();
  pdl_wait();
  if constexpr (VEC) qdev::quant_act_vec_block<MODE>(blockIdx.x, blockIdx.y, x, M, K, ldx, q, K, sa, ldsa);
  else qdev::quant_act_scalar_block<MODE>(blockIdx.x, blockIdx.y, x, M, K, ldx, q, K, sa, ldsa);
}

// Per-device set-up of the five kernel instantiations (shared-memory opt-in,
// register check) and the number of clusters of each size that can be
// resident at once (clusters live inside one GPC, so C * S <= SMs alone does
// not guarantee it; a second wave of clusters would double the time).
struct DecodeDevice {
  int max_clusters[kMaxSplit + 1];
};
DecodeDevice g_ddev[kMaxDevices];
DeviceOnce g_dsetup;

template <int NT, int QM>
fp8bq_status setup_kernel() {
  cudaFuncAttributes fa;
  cudaError_t e = cudaFuncGetAttributes(&fa, decode_kernel<NT, QM>);
  if (e != cudaSuccess) return cuda_fail(e, "cudaFuncGetAttributes(decode)");
  if (fa.numRegs != kDLaunchRegs) return FP8BQ_ERR_UNSUPPORTED;
  e = cudaFuncSetAttribute(decode_kernel<NT, QM>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemCap);
  if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(decode)");
  return FP8BQ_OK;
}

fp8bq_status decode_device(const DecodeDevice **out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  const fp8bq_status st = g_dsetup.get_for(dev, [](int d) -> fp8bq_status {
    fp8bq_status s = setup_kernel<16, FP8BQ_SCALE_FP32>();
    if (s == FP8BQ_OK) s = setup_kernel<16, FP8BQ_SCALE_POW2>();
    if (s == FP8BQ_OK) s = setup_kernel<16, -1>();
    if (s == FP8BQ_OK) s = setup_kernel<32, -1>();
    if (s == FP8BQ_OK) s = setup_kernel<64, -1>();
    if (s != FP8BQ_OK) return s;
    DecodeDevice &dd = g_ddev[d];
    dd.max_clusters[0] = 0;
    dd.max_clusters[1] = num_sms();
    for (int S = 2; S <= kMaxSplit; ++S) {
      // every instantiation runs one CTA per SM (its registers), so one query
      // at the largest shared-memory size stands for all
      cudaLaunchConfig_t cfg = {};
      cfg.blockDim = dim3(kDThreads);
      cfg.gridDim = dim3((unsigned)(S * 256));
      cfg.dynamicSmemBytes = kSmemCap;
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeClusterDimension;
      attr[0].val.clusterDim.x = (unsigned)S;
      attr[0].val.clusterDim.y = 1;
      attr[0].val.clusterDim.z = 1;
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      int n = 0;
      if (cudaOccupancyMaxActiveClusters(&n, decode_kernel<16, -1>, &cfg) != cudaSuccess) {
        cudaGetLastError();
        n = 0;  // clusters of this size are not used
      }
      dd.max_clusters[S] = n;
    }
    return FP8BQ_OK;
  });
  if (st == FP8BQ_OK) *out = &g_ddev[dev];
  return st;
}

struct Plan {
  int NT, NB, KB, S, C;   // S CTAs per cluster, C clusters
  bool res;               // activation quantized inside the GEMM kernel (one launch)
  int nres, nst, smem;    // resident K-blocks, weight stages, dynamic shared memory
  int64_t ldsa;
  size_t off_q, off_sa, total;
};

size_t align256(size_t v) { return (v + 255) & ~size_t(255); }

int pick_nt(int64_t M) {
  if (M <= 16) return 16;
  if (M <= 32) return 32;
  return 64;
}

// Workspace layout of the path with a prologue (codes [M][K], scales [KB][ldsa]).
void workspace_layout(int64_t M, int64_t K, Plan *p) {
  p->ldsa = (M + 3) / 4 * 4;
  p->off_q = 0;
  p->off_sa = align256((size_t)(M * K));
  p->total = p->off_sa + align256((size_t)(K / 128) * p->ldsa * 4);
}

// Shared memory of split S: nres resident K-blocks (0: none), rank 0's slots;
// false if fewer than kMinStages weight stages fit beside them.
template <int NT, int QM>
bool fit_smem(Plan *p, int S, int64_t M) {
  const int slot = red_floats(NT, S) * 4;
  p->nst = DCfg<NT, QM>::stages_for(p->nres, slot);
  p->smem = DCfg<NT, QM>::smem_bytes(p->nst, p->nres, slot);
  return p->nst > 0;
}

// The shared-memory layout of split S; false if none fits.
bool fit_split(Plan *p, int S, int64_t M, bool vec) {
  const int nk = (p->KB + S - 1) / S;  // K-blocks per CTA (at most)
  p->res = false;
  if (p->NT == kResMaxM && vec && nk * M <= kResMaxTiles) {
    p->nres = nk;
    p->res = fit_smem<16, FP8BQ_SCALE_FP32>(p, S, M);  // both modes lay shared memory out alike
    if (p->res) return true;
  }
  p->nres = 0;
  switch (p->NT) {
    case 16: return fit_smem<16, -1>(p, S, M);
    case 32: return fit_smem<32, -1>(p, S, M);
    default: return fit_smem<64, -1>(p, S, M);
  }
}

// The kernel a decode call runs.  FP8BQ_DECODE_KERNEL = narrow | wide | gemm
// in the environment forces one where the shape allows it (narrow and wide
// take M <= 64); unset or anything else is the default routing.
enum Route { kAuto = 0, kNarrow, kWide, kGemm };

Route route_override() {
  const char *v = getenv("FP8BQ_DECODE_KERNEL");
  if (v == nullptr) return kAuto;
  if (strcmp(v, "narrow") == 0) return kNarrow;
  if (strcmp(v, "wide") == 0) return kWide;
  if (strcmp(v, "gemm") == 0) return kGemm;
  return kAuto;
}

// vec: the activations allow 16-byte loads (x 16-byte aligned, ldx % 8 == 0).
// The split S (CTAs per cluster, each a contiguous K range of every block of
// its cluster) and the cluster count C (at most the resident clusters of that
// size) minimise the modelled time: the busiest CTA's items,
// ceil(NB / C) * ceil(KB / S), plus kRedItems per block when S > 1; ties go
// to the smaller S.  Only splits whose shared memory fits count.  narrow:
// this kernel for any M <= 64; otherwise p.NT = 0 (the prefill GEMM).
Plan make_plan(int64_t M, int64_t N, int64_t K, bool vec, const DecodeDevice &dd, bool narrow) {
  Plan p;
  p.S = p.C = 1;
  p.res = false;
  p.nres = p.nst = p.smem = 0;
  p.NT = narrow && M <= kSwapMaxM ? pick_nt(M) : 0;
  p.NB = (int)((N + 127) / 128);
  p.KB = (int)(K / 128);
  workspace_layout(M, K, &p);
  if (p.NT == 0) return p;
  int best = 0x7fffffff, bestS = 1;
  for (int s = 1; s <= kMaxSplit && s <= p.KB; ++s) {
    const int c = std::min(p.NB, std::min(dd.max_clusters[1] / s, dd.max_clusters[s]));
    if (c < 1 || !fit_split(&p, s, M, vec)) continue;
    const int blocks = (p.NB + c - 1) / c;
    const int cost = blocks * ((p.KB + s - 1) / s) + (s > 1 ? blocks * kRedItems : 0);
    if (cost < best) {
      best = cost;
      bestS = s;
    }
  }
  p.S = bestS;
  p.C = std::max(1, std::min(p.NB, std::min(dd.max_clusters[1] / bestS, dd.max_clusters[bestS])));
  fit_split(&p, bestS, M, vec);  // S = 1 always fits
  if (p.res) p.total = 0;
  return p;
}

template <int NT, int QM>
fp8bq_status launch_decode_nt(const CUtensorMap &tW, const CUtensorMap &tX, const CUtensorMap &tS,
                              const DecodeArgs &a, const Plan &p, cudaStream_t stream) {
  cudaLaunchConfig_t cfg = {};
  cfg.blockDim = dim3(kDThreads);
  cfg.gridDim = dim3((unsigned)(p.C * p.S));
  cfg.dynamicSmemBytes = (size_t)p.smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)p.S;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = p.S > 1 ? 1 : 0;
  cudaError_t e = cudaLaunchKernelEx(&cfg, decode_kernel<NT, QM>, tW, tX, tS, a);
  if (e != cudaSuccess) return cuda_fail(e, "gemm_decode launch");
  return check_launch("gemm_decode");
}

bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

}  // namespace

cudaError_t take_device_error_decode(unsigned long long *v) { return take_tu_device_error(v); }

size_t decode_workspace_size(int64_t M, int64_t N, int64_t K) {
  if (M <= 0 || N <= 0 || K <= 0 || M > kMaxDecodeM || K % 128 != 0) return 0;
  Plan p;
  workspace_layout(M, K, &p);  // the path with a prologue: the larger need
  return p.total;
}

fp8bq_status launch_gemm_decode(const void *x, int64_t ldx, const uint8_t *qw, int64_t ldw, const float *sw, void *y,
                                int64_t ldy, int64_t M, int64_t N, int64_t K, int mode, void *ws, size_t ws_bytes,
                                cudaStream_t stream) {
  if (M > kMaxDecodeM) return FP8BQ_ERR_UNSUPPORTED;
  const DecodeDevice *dd = nullptr;
  const fp8bq_status ready = decode_device(&dd);
  if (ready != FP8BQ_OK) return ready;
  const bool vec = aligned(x, 16) && ldx % 8 == 0;  // K % 128 == 0 already
  // the kernel: the wide form up to M = 64 (measured faster than the narrow
  // form and the prefill GEMM on every Llama-8B projection at M = 1, 16, 64)
  // and, for weights of at most kWideMaxNTiles 256-row tiles, up to M = 256
  // in groups of 64 tokens (o / down at M = 128: 17.3 / 30.5 us against the
  // GEMM's 22.4 / 58.8, whose few tiles leave most SMs idle); the prefill GEMM
  // otherwise (qkv / gate+up at M = 128: 21.8 / 28.8 us against 26.0 / 75.7)
  Route route = route_override();
  if (route == kAuto)
    route = M <= kSwapMaxM || (M <= kMaxDecodeM && (N + 255) / 256 <= kWideMaxNTiles) ? kWide : kGemm;
  DecodeWidePlan wp;
  bool wide = false;
  if (route == kWide) {
    const fp8bq_status ws_st = plan_decode_wide(M, N, K, vec, &wp);
    if (ws_st != FP8BQ_OK && ws_st != FP8BQ_ERR_UNSUPPORTED) return ws_st;
    wide = ws_st == FP8BQ_OK;  // else the prefill GEMM (M > 64)
  }
  const Plan p = make_plan(M, N, K, vec, *dd, route == kNarrow);
  // the documented size (the path with a prologue), whichever path this call takes
  const size_t need = decode_workspace_size(M, N, K);
  if (ws_bytes < need || (need > 0 && (ws == nullptr || !aligned(ws, 256)))) return FP8BQ_ERR_WORKSPACE;
  uint8_t *wsb = static_cast<uint8_t *>(ws);
  uint8_t *q = wsb + p.off_q;
  float *sa = reinterpret_cast<float *>(wsb + p.off_sa);
  const uint16_t *xs = static_cast<const uint16_t *>(x);

  // 1. quantize X into the workspace, unless the GEMM kernel does it
  if (!(wide ? wp.res : p.res)) {
    cudaLaunchConfig_t cfg = {};
    cfg.blockDim = dim3(256);
    cfg.gridDim = dim3((unsigned)(vec ? (M + 63) / 64 : (M + 15) / 16), (unsigned)p.KB);
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    auto kern = vec ? (mode == FP8BQ_SCALE_FP32 ? decode_prologue_kernel<FP8BQ_SCALE_FP32, true>
                                                : decode_prologue_kernel<FP8BQ_SCALE_POW2, true>)
                    : (mode == FP8BQ_SCALE_FP32 ? decode_prologue_kernel<FP8BQ_SCALE_FP32, false>
                                                : decode_prologue_kernel<FP8BQ_SCALE_POW2, false>);
    const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, xs, M, K, ldx, q, sa, p.ldsa);
    if (e != cudaSuccess) return cuda_fail(e, "gemm_decode prologue launch");
    fp8bq_status st = check_launch("gemm_decode prologue");
    if (st != FP8BQ_OK) return st;
    if (!wide && p.NT == 0)  // the prefill GEMM on the quantized activation
      return launch_gemm(q, K, sa, p.ldsa, qw, ldw, sw, y, ldy, M, N, K, mode, FP8BQ_GEMM_AUTO, stream);
  }
  if (wide) return launch_decode_wide(wp, xs, ldx, qw, ldw, sw, q, sa, p.ldsa, y, ldy, M, N, K, mode, stream);

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
  a.nst = p.nst;
  a.nres = p.nres;
  a.y = static_cast<uint16_t *>(y);
  a.ldy = ldy;
  a.x = xs;
  a.ldx = ldx;
  if (p.res)
    return mode == FP8BQ_SCALE_FP32 ? launch_decode_nt<16, FP8BQ_SCALE_FP32>(tW, tX, tS, a, p, stream)
                                    : launch_decode_nt<16, FP8BQ_SCALE_POW2>(tW, tX, tS, a, p, stream);
  switch (p.NT) {
    case 16: return launch_decode_nt<16, -1>(tW, tX, tS, a, p, stream);
    case 32: return launch_decode_nt<32, -1>(tW, tX, tS, a, p, stream);
    default: return launch_decode_nt<64, -1>(tW, tX, tS, a, p, stream);
  }
}

}  // namespace fp8bq
