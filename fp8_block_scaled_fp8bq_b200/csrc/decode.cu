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
// the MMA's N dimension (NT = M rounded up to 16, 32 or 64).  The NB x KB grid
// of (128-row weight block, 128-deep K-block) work items is cut, in
// weight-block-major order, into one contiguous equal share per CTA, so every
// SM streams the same number of weight bytes whatever NB is.  Per work item:
// the weight tile (16 KB) comes through a TMA stage ring; 4 x tcgen05.mma
// 128xNTx32 go into one of eight TMEM buffers; the epilogue warps (weight row =
// TMEM lane, token = column) add P * (sa[kb][token] * sw[nb][kb]) into FP32
// registers.  A weight block whose whole K range lies inside one share is
// written as bf16 at once.  A block cut between shares goes to FP32 partial
// slots in the workspace; each CTA that holds part of it then counts itself
// on the block's counter, and the last one to arrive adds all the partial
// slots in CTA order (deterministic) and writes the bf16 result, then resets
// the counter to 0 (so the workspace's counter area must be zero before the
// first call and is left zero by every call).
//
// The activation's 1x128 quantization (the device code of fp8bq_quant_act):
//   M <= 16: inside the same kernel.  Each CTA quantizes the K-blocks its share
//     touches (at most kMaxResKB) into shared memory, in the MMA's operand
//     layout, while the weight ring is filling: one launch per call;
//   16 < M <= 64: a prologue kernel writes the codes and scales to the
//     workspace and the GEMM's producer loads them with TMA beside the weight
//     tiles (two launches);
//   M > 64: the per-token promotion costs more than the weight stream, so the
//     prologue is followed by the prefill GEMM.
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
constexpr int kResMaxM = 16;        // activation quantized inside the GEMM kernel up to this M
constexpr int kMaxResKB = 48;       // K-blocks of resident activation codes per CTA
constexpr int kDEpiWarps = 8;
constexpr int kStageBudget = 212992;
constexpr int kMaxShares = 1024;    // CTAs of one call (counter area: kMaxShares ints)
constexpr size_t kCounterBytes = kMaxShares * 4;

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
  static constexpr int kFit = (kStageBudget - kResBytes) / (kABytes + kBBytes + kSSlot);
  static constexpr int kStages = kFit < 8 ? kFit : 8;
  static constexpr int kCW = NT / 2;         // token columns per epilogue warpgroup
  // TMEM accumulator buffers: a work item's partial is only NT columns, so
  // eight of them fit and the MMA can run eight items ahead of the epilogue
  static constexpr int kTBufs = 8;
  static constexpr int kTmemCols = kTBufs * NT;   // 128, 256 or 512: a power of two
  static constexpr int kSmemBytes = kStages * (kABytes + kBBytes + kSSlot) + kResBytes + 512 + 1024;
  static_assert(!kRes || NT == kResMaxM, "resident activation codes only for NT = 16");
  static_assert(kStages >= 3 && kSmemBytes <= 232448, "decode shared memory budget");
};

struct DecodeArgs {
  const float *sw;
  int32_t M, N, KB, NB;
  int64_t W;      // NB * KB work items
  int32_t G;      // CTAs (shares)
  float *part;    // [G][2][M][128] partial slots
  int *cnt;       // [kMaxShares] arrival counters of cut weight blocks (zero between calls)
  uint16_t *y;    // bf16 bits
  int64_t ldy;
  const uint16_t *x;  // resident quantization: bf16 activations [M][ldx]
  int64_t ldx;
};

// First work item of CTA c's share.
__host__ __device__ __forceinline__ int64_t share_begin(int64_t c, int64_t W, int64_t G) { return c * W / G; }

// The CTA whose share holds work item p.
__host__ __device__ __forceinline__ int64_t share_of(int64_t p, int64_t W, int64_t G) {
  int64_t c = p * G / W;
  while (c + 1 < G && share_begin(c + 1, W, G) <= p) ++c;
  while (c > 0 && share_begin(c, W, G) > p) --c;
  return c;
}

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
  uint64_t *bars = reinterpret_cast<uint64_t *>(sXr + C::kResBytes);
  uint64_t *full = bars;
  uint64_t *empty = bars + C::kStages;
  uint64_t *tfull = empty + C::kStages;
  uint64_t *tempty = tfull + C::kTBufs;
  uint64_t *drain = tempty + C::kTBufs;
  uint64_t *xready = drain + 1;
  uint64_t *fl_in = xready + 1;   // cut-block flush: all epilogue warps have written their partials
  uint64_t *fl_out = fl_in + 1;   // cut-block flush: the arrival has been counted
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(fl_out + 1);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
  volatile int *last_flag = abort_flag + 1;  // [2]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int KB = args.KB;
  const int64_t p_begin = share_begin(blockIdx.x, args.W, args.G);
  const int64_t p_end = share_begin(blockIdx.x + 1, args.W, args.G);
  // the K-blocks this share touches: slot i holds K-block (kb_first + i) % KB
  const int kb_first = (int)(p_begin % KB);
  const int nkb = (int)(p_end - p_begin < (int64_t)KB ? p_end - p_begin : (int64_t)KB);

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
    mbar_init(fl_in, kDEpiWarps);
    mbar_init(fl_out, 1);
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
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp < 4) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kDLowRegs));
    if (warp == 0 && lane == 0) {
      // ---------------------------------------------------------------- producer
      int stage = 0;
      uint32_t phase = 0, armed = 0, armed_parity = 0;
      bool ok = true;
      for (int64_t p = p_begin; p < p_end; ++p) {
        const int nb = (int)(p / KB), kb = (int)(p - (int64_t)nb * KB);
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
      for (int64_t p = p_begin; p < p_end && ok; ++p) {
        if (!mbar_wait(&tempty[buf], bphase ^ 1, abort_flag, kSiteMmaTmemEmpty) ||
            !mbar_wait(&full[stage], phase, abort_flag, kSiteMmaFull)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d = tmem_base + (uint32_t)(buf * NT);
        const uint32_t a0 = smem_addr(sA + stage * C::kABytes);
        uint32_t b0 = 0;
        if constexpr (kRes) {
          const int kb = (int)(p % KB);
          const int slot = kb - kb_first + (kb < kb_first ? KB : 0);
          b0 = smem_addr(sXr + slot * (NT * DBK));
        } else {
          b0 = smem_addr(sB + stage * C::kBBytes);
        }
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
    if constexpr (kRes) {
      // ------------------------------------------------------------ activation quantization
      // rows M..NT-1 of every tile are zero (the MMA reads all NT rows)
      for (int z = et; z < nkb * (NT - args.M) * 8; z += 256) {
        const int i = z / ((NT - args.M) * 8), rr = z - i * (NT - args.M) * 8;
        const int m = args.M + rr / 8, c = rr % 8;
        *reinterpret_cast<uint4 *>(sXr + i * (NT * DBK) + m * 128 + c * 16) = make_uint4(0, 0, 0, 0);
      }
      for (int z = et; z < nkb * NT; z += 256) sXs[z] = 0.f;
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
          const uint16_t *xrow = args.x + (int64_t)m * args.ldx + (int64_t)((kb_first + i) % KB) * DBK;
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
    uint32_t bphase = 0;
    int cut_nb[2] = {0, 0}, ncut = 0;  // weight blocks of this share that other shares hold too
    bool done = true;
    float acc[C::kCW];
#pragma unroll
    for (int j = 0; j < C::kCW; ++j) acc[j] = 0.f;
    // sw is [NB][KB] row-major, so work item p's weight scale is sw[p]; the
    // next two are loaded ahead
    float w0 = p_begin < p_end ? __ldg(args.sw + p_begin) : 0.f;
    float w1 = p_begin + 1 < p_end ? __ldg(args.sw + p_begin + 1) : 0.f;
    for (int64_t p = p_begin; p < p_end; ++p) {
      const int nb = (int)(p / KB), kb = (int)(p - (int64_t)nb * KB);
      const float w = w0;
      w0 = w1;
      if (p + 2 < p_end) w1 = __ldg(args.sw + p + 2);
      const bool got = mbar_wait(&tfull[buf], bphase, abort_flag, kSiteEpiTmemFull);
      if (!__all_sync(0xffffffffu, got)) {
        done = false;
        break;
      }
      tc_fence_after();
      const uint32_t taddr = tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(buf * NT + c0);
      const float4 *sc4;
      if constexpr (kRes) {
        const int slot = kb - kb_first + (kb < kb_first ? KB : 0);
        sc4 = reinterpret_cast<const float4 *>(sXs + slot * NT + c0);
      } else {
        sc4 = reinterpret_cast<const float4 *>(sS + stage * C::kSSlot) + c0 / 4;
      }
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
      // end of this weight block's run inside the share: flush it
      if (kb == KB - 1 || p + 1 == p_end) {
        const int64_t run0 = (p - kb > p_begin) ? p - kb : p_begin;  // first work item of the run
        const bool whole = (run0 == p - kb) && kb == KB - 1;
        const int n = nb * DBM + r;
        if (whole) {
          if (n < args.N) {
#pragma unroll
            for (int j = 0; j < C::kCW; ++j)
              if (c0 + j < args.M) args.y[(int64_t)(c0 + j) * args.ldy + n] = bf16_bits(acc[j]);
          }
        } else {
          // slot 0: the run holding the share's first item; slot 1: the last
          // run.  The block is counted and reduced after the share's last item.
          const int which = (run0 == p_begin) ? 0 : 1;
          float *dst = args.part + ((int64_t)(blockIdx.x * 2 + which) * args.M) * DBM + r;
#pragma unroll
          for (int j = 0; j < C::kCW; ++j)
            if (c0 + j < args.M) dst[(int64_t)(c0 + j) * DBM] = acc[j];
          cut_nb[ncut++] = nb;
        }
#pragma unroll
        for (int j = 0; j < C::kCW; ++j) acc[j] = 0.f;
      }
    }
    // Count this CTA on each cut block it holds; the last CTA to arrive adds
    // every sharing CTA's partial slot in CTA order.  (Hand-offs on bounded
    // mbarriers, so an abort elsewhere in the CTA cannot leave a warp waiting.)
    if (done && ncut > 0) {
      __threadfence();  // this thread's partial slots are visible to the other CTAs
      __syncwarp();
      if (lane == 0) mbar_arrive(fl_in);
      bool fine = true;
      if (et == 0) {
        fine = mbar_wait(fl_in, 0, abort_flag, kSiteEpiTmemFull);
        for (int i = 0; i < ncut; ++i) {
          int is_last = 0;
          if (fine) {
            const int64_t first = (int64_t)cut_nb[i] * KB;
            const int64_t cf = share_of(first, args.W, args.G), cl = share_of(first + KB - 1, args.W, args.G);
            const int prior = atomicAdd(args.cnt + cf, 1);
            is_last = prior == (int)(cl - cf);
            if (is_last) {
              __threadfence();
              args.cnt[cf] = 0;  // left zero for the next call (every arrival has been counted)
            }
          }
          last_flag[i] = is_last;
        }
        mbar_arrive(fl_out);
      }
      fine = mbar_wait(fl_out, 0, abort_flag, kSiteEpiTmemFull) && fine;
      if (__all_sync(0xffffffffu, fine)) {
        for (int i = 0; i < ncut; ++i) {
          if (!last_flag[i]) continue;
          const int nb = cut_nb[i];
          const int n = nb * DBM + r;
          const int64_t first = (int64_t)nb * KB;
          const int64_t cf = share_of(first, args.W, args.G), cl = share_of(first + KB - 1, args.W, args.G);
          float sum[C::kCW];
#pragma unroll
          for (int j = 0; j < C::kCW; ++j) sum[j] = 0.f;
          for (int64_t c = cf; c <= cl; ++c) {
            const int wc = share_begin(c, args.W, args.G) >= first ? 0 : 1;
            const float *src = args.part + ((c * 2 + wc) * args.M + c0) * DBM + r;
            float v[C::kCW];  // one CTA's slot: independent loads, issued together
#pragma unroll
            for (int j = 0; j < C::kCW; ++j) v[j] = (c0 + j < args.M) ? __ldcg(src + (int64_t)j * DBM) : 0.f;
#pragma unroll
            for (int j = 0; j < C::kCW; ++j) sum[j] += v[j];
          }
          if (n < args.N) {
#pragma unroll
            for (int j = 0; j < C::kCW; ++j)
              if (c0 + j < args.M) args.y[(int64_t)(c0 + j) * args.ldy + n] = bf16_bits(sum[j]);
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::kTmemCols);
  }
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
  int NT, NB, KB, G;
  bool res;     // activation quantized inside the GEMM kernel (one launch)
  int64_t W, ldsa;
  size_t off_q, off_sa, off_part, total;  // the counter area is [0, kCounterBytes)
};

size_t align256(size_t v) { return (v + 255) & ~size_t(255); }

int pick_nt(int64_t M) {
  if (M <= 16) return 16;
  if (M <= 32) return 32;
  return 64;
}

// vec: the activations allow 16-byte loads (x 16-byte aligned, ldx % 8 == 0).
Plan make_plan(int64_t M, int64_t N, int64_t K, bool vec) {
  Plan p;
  p.NT = M <= kSwapMaxM ? pick_nt(M) : 0;  // 0: the prefill GEMM
  p.NB = (int)((N + 127) / 128);
  p.KB = (int)(K / 128);
  p.W = (int64_t)p.NB * p.KB;
  p.G = (int)std::min<int64_t>(std::min<int64_t>(p.W, num_sms()), kMaxShares);
  const int64_t longest = (p.W + p.G - 1) / p.G;  // the largest share
  p.res = p.NT == kResMaxM && vec && std::min<int64_t>(longest, p.KB) <= kMaxResKB;
  p.ldsa = (M + 3) / 4 * 4;
  p.off_q = kCounterBytes;
  p.off_sa = p.off_q + (p.res ? 0 : align256((size_t)(M * K)));
  p.off_part = p.off_sa + (p.res ? 0 : align256((size_t)p.KB * p.ldsa * 4));
  p.total = p.off_part + (p.NT ? align256((size_t)p.G * 2 * M * DBM * 4) : 0);
  return p;
}

template <int NT, int QM>
fp8bq_status launch_decode_nt(const CUtensorMap &tW, const CUtensorMap &tX, const CUtensorMap &tS,
                              const DecodeArgs &a, cudaStream_t stream) {
  static DeviceOnce once;  // one per instantiation
  const fp8bq_status ready = once.get([](int) {
    cudaFuncAttributes fa;
    cudaError_t e = cudaFuncGetAttributes(&fa, decode_kernel<NT, QM>);
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncGetAttributes(decode)");
    if (fa.numRegs != kDLaunchRegs) return FP8BQ_ERR_UNSUPPORTED;
    e = cudaFuncSetAttribute(decode_kernel<NT, QM>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             DCfg<NT, QM>::kSmemBytes);
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(decode)");
    return FP8BQ_OK;
  });
  if (ready != FP8BQ_OK) return ready;
  decode_kernel<NT, QM><<<a.G, kDThreads, DCfg<NT, QM>::kSmemBytes, stream>>>(tW, tX, tS, a);
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
  if (ws == nullptr || ws_bytes < make_plan(M, N, K, false).total || !aligned(ws, 256)) return FP8BQ_ERR_WORKSPACE;
  uint8_t *wsb = static_cast<uint8_t *>(ws);
  uint8_t *q = wsb + p.off_q;
  float *sa = reinterpret_cast<float *>(wsb + p.off_sa);
  float *part = reinterpret_cast<float *>(wsb + p.off_part);
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

  // 2. the GEMM, with the cut weight blocks reduced by their last CTA
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
  a.W = p.W;
  a.G = p.G;
  a.part = part;
  a.cnt = reinterpret_cast<int *>(wsb);
  a.y = static_cast<uint16_t *>(y);
  a.ldy = ldy;
  a.x = xs;
  a.ldx = ldx;
  if (p.res)
    return mode == FP8BQ_SCALE_FP32 ? launch_decode_nt<16, FP8BQ_SCALE_FP32>(tW, tX, tS, a, stream)
                                    : launch_decode_nt<16, FP8BQ_SCALE_POW2>(tW, tX, tS, a, stream);
  switch (p.NT) {
    case 16: return launch_decode_nt<16, -1>(tW, tX, tS, a, stream);
    case 32: return launch_decode_nt<32, -1>(tW, tX, tS, a, stream);
    default: return launch_decode_nt<64, -1>(tW, tX, tS, a, stream);
  }
}

}  // namespace fp8bq
