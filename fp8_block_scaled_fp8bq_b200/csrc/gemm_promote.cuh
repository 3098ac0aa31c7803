// The promotion GEMM kernel for sm_100a (included by the translation units that
// instantiate it): block-scaled FP8 Y[M,N] = X[M,K] . W[N,K]^T with E4M3
// operands, 1x128 activation scales and 128x128 weight scales; its grouped
// (mixture-of-experts) form, where rows [offsets[e], offsets[e+1]) of the
// expert-sorted activations multiply expert e's weight; and two epilogues:
// bf16 Y, or the gated feed-forward activation of a gate+up projection
// followed by the 1x128 quantization of its result (SwiGLU epilogue below).
//
// Method: "NVIDIA NeMo RL Achieves 48% Speedup With End-to-End FP8 Precision
// Training", section "Technical breakthrough": the linear layers run in FP8 on
// block-wise quantized E4M3 operands (activations 1x128, weights 128x128);
// section "Real-world performance gains": the recipe also runs on a
// mixture-of-experts model.
//
// Promotion design (FP32 scales).  A scale varies with the row m (activation)
// and with the 128-column block of n (weight) and with the K-block, so it
// cannot be folded into the MMA.  Each 128-deep K-block's product
//   P_kb[m][n] = sum_{k in kb} qa[m][k] * qw[n][k]      (E4M3 x E4M3, exact in FP32)
// is produced by the tensor cores into TMEM, and the epilogue warps add
//   acc[m][n] += P_kb[m][n] * (sa[kb][m] * sw[n/128][kb])
// into FP32 registers.  The result is rounded to bf16 once.
//
// Structure (one persistent CTA per SM, 384 threads = 3 warpgroups):
//   warp 0      TMA producer: A (128x128 B) and B (256x128 B) tiles of each
//               K-block into a 4-stage shared-memory ring (128-byte swizzle).
//   warp 1      TMEM owner and MMA issuer: 4 x tcgen05.mma kind::f8f6f4
//               (128x256x32) per K-block into one of two 256-column TMEM
//               buffers; tcgen05.commit frees the smem stage and hands the
//               buffer to the epilogue.
//   warps 2-3   idle after the prologue (warpgroup 0 gives its registers to
//               the epilogue with setmaxnreg).
//   warps 4-11  promotion + epilogue (warpgroups 1 and 2): warp w reads TMEM
//               lanes 32*(w%4)..+31 (its 32 rows) and columns
//               [128*h, 128*h+128) with h = (w-4)/4, i.e. exactly one 128-wide
//               weight block, so each thread needs one scale product per
//               K-block and holds 128 FP32 accumulators (packed fma pairs).
//               After the last K-block the accumulators leave as bf16: TMA
//               stores (dense) or row-masked coalesced stores (grouped, where
//               a 128-row tile can run past its expert's last row).
// The MMA of K-block kb+1 overlaps the promotion of kb (two TMEM buffers), and
// the stores of one tile overlap the MMAs of the next.
//
// Grouped scheduling is on the device: every CTA reads offsets[0..E], builds
// the prefix of tile counts per expert in shared memory, and maps each tile
// id to (expert, 128-row block, 256-column block) by binary search, so no
// host synchronization is needed.  Tiles of one expert are consecutive (row
// blocks fastest), so concurrently running CTAs share that expert's weight
// tiles in L2.
#pragma once

#include <cuda_bf16.h>
#include <string.h>

#include <algorithm>

#include "device.cuh"
#include "internal.h"
#include "quant.cuh"

namespace fp8bq {
namespace {

constexpr int BM = 128, BN = 256, BK = 128;
constexpr int kStages = 4;
constexpr int kABytes = BM * BK;
constexpr int kBBytes = BN * BK;
constexpr int kStageBytes = kABytes + kBBytes;
constexpr int kEpiWarps = 8;
constexpr int kThreads = 128 + kEpiWarps * 32;
// Register split (setmaxnreg): the launch gives every thread kLaunchRegs; the
// producer/MMA warpgroup drops to kLowRegs and the two epilogue warpgroups
// rise to kHighRegs.  128 * kLowRegs + 256 * kHighRegs must not exceed
// 384 * kLaunchRegs (the build checks ptxas's count against kLaunchRegs, and
// the launcher checks it again at run time).
constexpr int kLaunchRegs = 168;
constexpr int kLowRegs = 56;
constexpr int kHighRegs = 224;
static_assert(128 * kLowRegs + 256 * kHighRegs <= kThreads * kLaunchRegs, "register split");
constexpr int kTmemCols = 2 * BN;
constexpr int kBarBytes = 256;
constexpr int kXAmaxBytes = kEpiWarps * 32 * 4;  // SwiGLU epilogue: partial amax per thread

// Epilogues: bf16 Y; SwiGLU + 1x128 quantization with FP32 or power-of-2
// scales; bf16 Y with 1x128 scales on B's rows instead of 128x128 tiles (the
// weight-gradient GEMM, both of whose operands are activation-like).
constexpr int kEpiBf16 = 0, kEpiSwigluFp32 = 1, kEpiSwigluPow2 = 2, kEpiBf16RowB = 3;

template <int EPI>
constexpr bool tma_store_epi() { return EPI == kEpiBf16 || EPI == kEpiBf16RowB; }

// Per-warp bf16 staging: dense = 32 rows x 64 columns in the TMA 128-byte
// swizzle; grouped = 32 rows x 32 columns in the TMA 64-byte swizzle (64-byte
// rows, 16-byte chunks XOR ((row >> 1) & 3), conflict-free for both the row
// writes and the warp's masked copy-out).
template <bool G>
struct Cfg {
  static constexpr int kEpiBufBytes = G ? 32 * 64 : 32 * 128;
  static constexpr int kSchedBytes = G ? 2 * (kMaxExperts + 1) * 4 : 0;
  static constexpr int kSmemBytes =
      kStages * kStageBytes + kEpiWarps * kEpiBufBytes + kBarBytes + kSchedBytes + kXAmaxBytes + 1024;
  static_assert(kSmemBytes <= 232448, "shared memory budget");
};

struct GemmArgs {
  const float *sa;
  const float *sw;
  int64_t ldsa;
  int32_t M, N, KB, NB;     // grouped: M = total rows
  int32_t num_m, num_n;     // dense tile grid; grouped: num_n only
  int32_t band, n_major;    // dense tile order (raster_tile)
  // grouped only
  const int32_t *offsets;   // [E+1], device
  int32_t E;
  uint16_t *y;              // output base for the masked stores (bf16 bits)
  int64_t ldy;
  int64_t ldsw;             // kEpiBf16RowB: B row scales sw[kb * ldsw + n]
  int32_t selftest;         // 1: the producer issues nothing (failure-detection self-test)
  // SwiGLU epilogue only: H codes [rows][ldqh], H scales [N/256][ldsh], optional bf16 H [rows][ldh]
  uint8_t *qh;
  int64_t ldqh;
  float *sh;
  int64_t ldsh;
  uint16_t *h;
  int64_t ldh;
};

// A tile: rows [row0, row_end) of the activations (row_end clips the last
// tile of a matrix or of an expert), 256-column block nb, expert e.
struct Tile {
  int e, row0, row_end, nb;
};

__device__ __forceinline__ Tile dense_tile(int t, const GemmArgs &a) {
  int mi, ni;
  raster_tile(t, a.num_m, a.num_n, a.band, a.n_major, mi, ni);
  Tile tl;
  tl.e = 0;
  tl.row0 = mi * BM;
  tl.row_end = a.M;
  tl.nb = ni;
  return tl;
}

// prefix[e] = tiles of experts before e (prefix[E] = total); offs = clamped offsets.
__device__ __forceinline__ Tile grouped_tile(int t, const GemmArgs &a, const int *prefix, const int *offs) {
  int lo = 0, hi = a.E - 1;  // last expert whose first tile is <= t (empty experts are skipped)
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (prefix[mid] <= t) lo = mid;
    else hi = mid - 1;
  }
  const int local = t - prefix[lo];
  const int mt_e = (offs[lo + 1] - offs[lo] + BM - 1) / BM;
  Tile tl;
  tl.e = lo;
  tl.nb = local / mt_e;
  tl.row0 = offs[lo] + (local - tl.nb * mt_e) * BM;
  tl.row_end = offs[lo + 1];
  return tl;
}

template <bool G>
__device__ __forceinline__ Tile tile_at(int t, const GemmArgs &a, const int *prefix, const int *offs) {
  if constexpr (G) return grouped_tile(t, a, prefix, offs);
  else return dense_tile(t, a);
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t *>(&v);
}

// Shared-memory carve-up and pipeline state common to the three roles.
struct Smem {
  uint8_t *a;        // kStages x [128 rows x 128 B], 128-byte swizzled
  uint8_t *b;        // kStages x [256 rows x 128 B], 128-byte swizzled
  uint8_t *epi;      // kEpiWarps x bf16 staging
  uint64_t *full;    // [kStages] TMA bytes landed
  uint64_t *empty;   // [kStages] MMAs done reading the stage
  uint64_t *tfull;   // [2] K-block partial ready in TMEM buffer
  uint64_t *tempty;  // [2] TMEM buffer read by all epilogue warps
  uint64_t *drain;   // MMA drain on the error path
  uint32_t *tmem_slot;
  volatile int *abort_flag;
  int *prefix;       // grouped: [E+1] tile prefix
  int *offs;         // grouped: [E+1] clamped offsets
  uint64_t *xbar;    // SwiGLU epilogue: [4] exchange barrier of the two warps of each row quarter
  float *xamax;      // SwiGLU epilogue: [kEpiWarps][32] partial amax
};

template <bool G>
__device__ __forceinline__ Smem carve(uint8_t *raw) {
  Smem s;
  uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(raw) + 1023) & ~uintptr_t(1023));
  s.a = base;
  s.b = base + kStages * kABytes;
  s.epi = s.b + kStages * kBBytes;
  uint64_t *bars = reinterpret_cast<uint64_t *>(s.epi + kEpiWarps * Cfg<G>::kEpiBufBytes);
  s.full = bars;
  s.empty = bars + kStages;
  s.tfull = bars + 2 * kStages;
  s.tempty = s.tfull + 2;
  s.drain = s.tempty + 2;
  s.tmem_slot = reinterpret_cast<uint32_t *>(s.drain + 1);
  s.abort_flag = reinterpret_cast<volatile int *>(s.tmem_slot + 1);
  s.xbar = bars + 16;
  s.prefix = reinterpret_cast<int *>(reinterpret_cast<uint8_t *>(bars) + kBarBytes);
  s.offs = s.prefix + (kMaxExperts + 1);
  s.xamax = reinterpret_cast<float *>(reinterpret_cast<uint8_t *>(bars) + kBarBytes + Cfg<G>::kSchedBytes);
  return s;
}

// Grouped prologue (one warp): clamp the offsets into [0, M] and make them
// nondecreasing (so offsets that break the contract cannot cause an
// out-of-bounds access), then the exclusive prefix of tiles per expert.
__device__ __forceinline__ void build_schedule(const Smem &S, const GemmArgs &a, int lane) {
  const int n = a.E + 1;
  const int per = (n + 31) / 32;
  const int i0 = min(lane * per, n), i1 = min(i0 + per, n);
  int run = 0;
  for (int i = i0; i < i1; ++i) {
    int v = __ldg(a.offsets + i);
    v = max(0, min(v, a.M));
    run = max(run, v);
    S.offs[i] = run;
  }
  // max-scan of the chunk maxima across lanes
  int incl = run;
#pragma unroll
  for (int d = 1; d < 32; d <<= 1) {
    const int o = __shfl_up_sync(0xffffffffu, incl, d);
    if (lane >= d) incl = max(incl, o);
  }
  int before = __shfl_up_sync(0xffffffffu, incl, 1);
  if (lane == 0) before = 0;
  for (int i = i0; i < i1; ++i) S.offs[i] = max(S.offs[i], before);
  __syncwarp();
  // tiles per expert and their exclusive prefix
  int sum = 0;
  for (int i = i0; i < i1 && i < a.E; ++i) sum += ((S.offs[i + 1] - S.offs[i] + BM - 1) / BM) * a.num_n;
  int excl = sum;
#pragma unroll
  for (int d = 1; d < 32; d <<= 1) {
    const int o = __shfl_up_sync(0xffffffffu, excl, d);
    if (lane >= d) excl += o;
  }
  excl -= sum;
  for (int i = i0; i < i1; ++i) {
    S.prefix[i] = excl;
    if (i < a.E) excl += ((S.offs[i + 1] - S.offs[i] + BM - 1) / BM) * a.num_n;
  }
}

template <bool G>
__device__ __forceinline__ int total_tiles(const Smem &S, const GemmArgs &a) {
  if constexpr (G) return S.prefix[a.E];
  else return a.num_m * a.num_n;
}

// TMA producer (one thread): stream the A and B tiles of every K-block of this
// CTA's tiles through the stage ring.
template <bool G>
__device__ __forceinline__ void run_producer(const Smem &S, const CUtensorMap *tmA, const CUtensorMap *tmB,
                                             const GemmArgs &args) {
  if (args.selftest) return;  // nothing arrives: the MMA issuer's bounded wait runs out
  const int total = total_tiles<G>(S, args);
  int stage = 0;
  uint32_t phase = 0, armed = 0, armed_parity = 0;
  bool ok = true;
  for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
    const Tile tl = tile_at<G>(t, args, S.prefix, S.offs);
    for (int kb = 0; kb < args.KB; ++kb) {
      if (!mbar_wait(&S.empty[stage], phase ^ 1, S.abort_flag, kSiteProducerEmpty)) {
        ok = false;
        break;
      }
      mbar_arrive_expect_tx(&S.full[stage], kStageBytes);
      tma_load_2d(S.a + stage * kABytes, tmA, &S.full[stage], kb * BK, tl.row0);
      if constexpr (G) tma_load_3d(S.b + stage * kBBytes, tmB, &S.full[stage], kb * BK, tl.nb * BN, tl.e);
      else tma_load_2d(S.b + stage * kBBytes, tmB, &S.full[stage], kb * BK, tl.nb * BN);
      armed |= 1u << stage;
      armed_parity = (armed_parity & ~(1u << stage)) | (phase << stage);
      if (++stage == kStages) {
        stage = 0;
        phase ^= 1;
      }
    }
  }
  if (!ok) {  // every load issued must land before the CTA may exit
    for (int s = 0; s < kStages; ++s)
      if (armed >> s & 1u) mbar_wait(&S.full[s], (armed_parity >> s) & 1u, nullptr, kSiteDrain);
  }
}

// MMA issuer (one thread): per K-block, four 128x256x32 E4M3 MMAs into a fresh
// TMEM buffer (the first one overwrites, the rest accumulate).
template <bool G>
__device__ __forceinline__ void run_mma(const Smem &S, uint32_t tmem_base, const GemmArgs &args) {
  const int total = total_tiles<G>(S, args);
  const uint32_t idesc = idesc_f8f6f4_e4m3_f32(BM, BN);
  int stage = 0, buf = 0;
  uint32_t phase = 0, bphase = 0;
  bool ok = true, issued = false;
  for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
    for (int kb = 0; kb < args.KB; ++kb) {
      if (!mbar_wait(&S.tempty[buf], bphase ^ 1, S.abort_flag, kSiteMmaTmemEmpty) ||
          !mbar_wait(&S.full[stage], phase, S.abort_flag, kSiteMmaFull)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t d = tmem_base + (uint32_t)(buf * BN);
      const uint32_t a0 = smem_addr(S.a + stage * kABytes);
      const uint32_t b0 = smem_addr(S.b + stage * kBBytes);
#pragma unroll
      for (int k = 0; k < BK / 32; ++k)
        mma_f8f6f4(d, smem_desc_k_sw128(a0 + 32 * k), smem_desc_k_sw128(b0 + 32 * k), idesc, k > 0 ? 1u : 0u);
      mma_commit(&S.empty[stage]);
      mma_commit(&S.tfull[buf]);
      issued = true;
      if (++stage == kStages) {
        stage = 0;
        phase ^= 1;
      }
      if (++buf == 2) {
        buf = 0;
        bphase ^= 1;
      }
    }
  }
  if (!ok && issued) {  // TMEM must be quiescent before it is freed
    mma_commit(S.drain);
    mbar_wait(S.drain, 0, nullptr, kSiteDrain);
  }
}

// ---------------------------------------------------------------------------
// SwiGLU + 1x128 quantization epilogue
// ---------------------------------------------------------------------------
// The gate+up weight is stored with its 128-row blocks interleaved (block 2j =
// gate rows of features [128j, 128j+128), block 2j+1 = up rows of the same
// features), so a 256-column output tile nb holds g (columns 0..127, epilogue
// half 0) and u (columns 128..255, half 1) of feature block j = nb, and one row
// of it is exactly one 1x128 tile of H = silu(g) * u.
//
// Per row quarter, warps (quarter, 0) and (quarter, 1) hold the same 32 rows.
// Warp `half` produces H for feature columns [64 half, 64 half + 64): it keeps
// its own 64 values there and receives the partner's 64 through its staging
// buffer (as bf16: the GEMM's output is bf16), in rounds of as many columns as
// the buffer holds.  The two warps then exchange their partial amax, both form
// the row's tile scale from the same value, and each encodes its 64 columns.
//
// H follows the unfused composition: g and u are the bf16-rounded GEMM
// outputs; silu(g) * u is evaluated in FP32 with the SFU exponential and the
// fast divide (relative error a few 2^-24, far below the bf16 step of H) and
// rounded to bf16 once; the codes and the scale are those of the 1x128
// activation quantizer applied to that bf16 H (the quantizer's own device code).
// Values travel as packed bf16 pairs (lower column in the low half).

__device__ __forceinline__ float swiglu_f32(float g, float u) {
  return __fmul_rn(__fdividef(g, __fadd_rn(1.f, __expf(-g))), u);
}

// Both warps of a row quarter meet here (all 64 threads arrive).  Bounded: on a
// timeout or an abort elsewhere in the CTA it returns false on every lane.
__device__ __forceinline__ bool pair_sync(uint64_t *bar, uint32_t &phase, volatile int *abort) {
  mbar_arrive(bar);
  const bool got = mbar_wait(bar, phase, abort, kSitePairExchange);
  phase ^= 1u;
  return __all_sync(0xffffffffu, got);
}

template <bool G, int MODE, int HALF>
__device__ __forceinline__ bool swiglu_epilogue(const Smem &S, const GemmArgs &a, const Tile &tl, float2 (&acc)[64],
                                                int ew, int quarter, int lane, uint32_t &xphase) {
  constexpr int RB = Cfg<G>::kEpiBufBytes / 32;  // exchange bytes per row: 128 (dense) or 64 (grouped)
  constexpr int XC = RB / 2;                     // bf16 columns per round
  constexpr int NCH = RB / 16;                   // 16-byte chunks per row
  constexpr int SWZ = RB == 128 ? 0 : 1;         // chunk c of row l sits at c ^ ((l >> SWZ) & (NCH - 1))
  constexpr int SEND = HALF ? 0 : 64;            // the columns the partner produces
  constexpr int KEEP = HALF * 64;                // the columns this warp produces
  const int partner = ew ^ 4;
  uint8_t *mine = S.epi + ew * Cfg<G>::kEpiBufBytes + lane * RB;
  const uint8_t *theirs = S.epi + partner * Cfg<G>::kEpiBufBytes + lane * RB;
  uint64_t *xb = &S.xbar[quarter];
  const int swz = (lane >> SWZ) & (NCH - 1);

  // own values of the produced columns, bf16-rounded (the GEMM's output), packed
  uint32_t hw[32];
#pragma unroll
  for (int j = 0; j < 32; ++j) hw[j] = pack_bf16x2(acc[KEEP / 2 + j].x, acc[KEEP / 2 + j].y);

#pragma unroll
  for (int r = 0; r < 64 / XC; ++r) {
    if (r > 0 && !pair_sync(xb, xphase, S.abort_flag)) return false;  // partner done reading round r-1
#pragma unroll
    for (int c = 0; c < NCH; ++c) {
      const float2 *p = &acc[(SEND + r * XC + 8 * c) / 2];
      uint4 pk;
      pk.x = pack_bf16x2(p[0].x, p[0].y);
      pk.y = pack_bf16x2(p[1].x, p[1].y);
      pk.z = pack_bf16x2(p[2].x, p[2].y);
      pk.w = pack_bf16x2(p[3].x, p[3].y);
      *reinterpret_cast<uint4 *>(mine + ((c ^ swz) << 4)) = pk;
    }
    if (!pair_sync(xb, xphase, S.abort_flag)) return false;
#pragma unroll
    for (int c = 0; c < NCH; ++c) {
      const uint4 v = *reinterpret_cast<const uint4 *>(theirs + ((c ^ swz) << 4));
      const uint32_t o[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int j = (r * XC + 8 * c) / 2 + i;  // pair index within the produced columns
        const uint32_t gw = HALF ? o[i] : hw[j];
        const uint32_t uw = HALF ? hw[j] : o[i];
        hw[j] = pack_bf16x2(swiglu_f32(bf16_lo(gw), bf16_lo(uw)), swiglu_f32(bf16_hi(gw), bf16_hi(uw)));
      }
    }
  }

  // the tile amax: this warp's 64 columns, then the partner's
  uint32_t am = 0;
#pragma unroll
  for (int j = 0; j < 32; ++j) am = __vmaxu2(am, hw[j] & 0x7FFF7FFFu);
  S.xamax[ew * 32 + lane] = qdev::bits_to_amax(max(am & 0xFFFFu, am >> 16));
  if (!pair_sync(xb, xphase, S.abort_flag)) return false;
  const float amax = fmaxf(S.xamax[ew * 32 + lane], S.xamax[partner * 32 + lane]);
  const qdev::TileScale ts = qdev::tile_scale<MODE>(amax);

  const int m = tl.row0 + quarter * 32 + lane;
  if (m < tl.row_end) {
    const int64_t col0 = (int64_t)tl.nb * 128 + KEEP;
    uint8_t *q = a.qh + (int64_t)m * a.ldqh + col0;
    if (qdev::fast_tile<MODE>(ts)) {
#pragma unroll
      for (int c = 0; c < 4; ++c) {  // 16 codes per store
        uint4 pk;
        pk.x = qdev::encode4<MODE, true>(hw[8 * c + 0], hw[8 * c + 1], ts);
        pk.y = qdev::encode4<MODE, true>(hw[8 * c + 2], hw[8 * c + 3], ts);
        pk.z = qdev::encode4<MODE, true>(hw[8 * c + 4], hw[8 * c + 5], ts);
        pk.w = qdev::encode4<MODE, true>(hw[8 * c + 6], hw[8 * c + 7], ts);
        *reinterpret_cast<uint4 *>(q + 16 * c) = pk;
      }
    } else {
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint4 pk;
        pk.x = qdev::encode4<MODE>(hw[8 * c + 0], hw[8 * c + 1], ts);
        pk.y = qdev::encode4<MODE>(hw[8 * c + 2], hw[8 * c + 3], ts);
        pk.z = qdev::encode4<MODE>(hw[8 * c + 4], hw[8 * c + 5], ts);
        pk.w = qdev::encode4<MODE>(hw[8 * c + 6], hw[8 * c + 7], ts);
        *reinterpret_cast<uint4 *>(q + 16 * c) = pk;
      }
    }
    if (HALF == 0) a.sh[(int64_t)tl.nb * a.ldsh + m] = ts.s;
    if (a.h != nullptr) {
      uint16_t *hp = a.h + (int64_t)m * a.ldh + col0;
#pragma unroll
      for (int c = 0; c < 8; ++c)
        *reinterpret_cast<uint4 *>(hp + 8 * c) = make_uint4(hw[4 * c], hw[4 * c + 1], hw[4 * c + 2], hw[4 * c + 3]);
    }
  }
  return true;
}

// Promotion + epilogue (one warp of the two epilogue warpgroups).
template <bool G, int EPI>
__device__ __forceinline__ void run_epilogue(const Smem &S, uint32_t tmem_base, const CUtensorMap *tmY,
                                             const GemmArgs &args, int warp, int lane) {
  const int total = total_tiles<G>(S, args);
  const int KB = args.KB;
  const int ew = warp - 4;
  const int quarter = warp & 3;  // TMEM lanes this warp may access
  const int half = ew >> 2;      // 128-column half of the tile = one weight block
  const int row = quarter * 32 + lane;
  uint8_t *ebuf = S.epi + ew * Cfg<G>::kEpiBufBytes;
  int buf = 0;
  uint32_t bphase = 0, xphase = 0;
  for (int t = blockIdx.x; t < total; t += gridDim.x) {
    const Tile tl = tile_at<G>(t, args, S.prefix, S.offs);
    const int m = tl.row0 + row;
    const int wn = tl.nb * 2 + half;
    const bool live = m < tl.row_end && wn < args.NB;
    const float *sa_p = args.sa + m;
    const float *sw_p = args.sw + ((int64_t)tl.e * args.NB + wn) * KB;
    // kEpiBf16RowB: the scale of B row n (output column n) for K-block kb is
    // sw[kb * ldsw + n].  Lane l loads the 4 scales of columns n0 + 4l .. +3 two
    // K-blocks ahead; per K-block the warp puts its 128 into the first 512
    // bytes of its staging buffer and every lane reads them back as broadcasts.
    const int64_t n0 = (int64_t)tl.nb * BN + half * 128;
    const bool bcol = EPI == kEpiBf16RowB && n0 + 4 * lane < args.N;
    const float *sb_p = args.sw + n0 + 4 * lane;
    float *slot = reinterpret_cast<float *>(ebuf);
    float4 b0 = make_float4(0.f, 0.f, 0.f, 0.f), b1 = b0;
    if constexpr (EPI == kEpiBf16RowB) {
      if (bcol) {
        b0 = __ldg(reinterpret_cast<const float4 *>(sb_p));
        if (KB > 1) b1 = __ldg(reinterpret_cast<const float4 *>(sb_p + args.ldsw));
      }
      if (lane == 0) bulk_wait_group_read0();  // the previous tile's store has left the buffer
      __syncwarp();
    }
    // 128 FP32 accumulators as 64 pairs: the promotion is a packed fma (two
    // lanes of FP32 per instruction).
    float2 acc[64];
#pragma unroll
    for (int j = 0; j < 64; ++j) acc[j] = make_float2(0.f, 0.f);
    // Scale factors are loaded two K-blocks before use so their latency is
    // hidden: (a0, w0) belong to kb, (a1, w1) to kb+1.
    // (With kEpiBf16RowB the tile factor is 1: B's scales enter per column.)
    constexpr bool kTileB = EPI != kEpiBf16RowB;
    float a0 = 0.f, w0 = kTileB ? 0.f : 1.f, a1 = 0.f, w1 = w0;
    if (live) {
      a0 = __ldg(sa_p);
      if (kTileB) w0 = __ldg(sw_p);
      if (KB > 1) {
        a1 = __ldg(sa_p + args.ldsa);
        if (kTileB) w1 = __ldg(sw_p + 1);
      }
    }
    bool ok = true;
    for (int kb = 0; kb < KB; ++kb) {
      const float sc = a0 * w0;
      a0 = a1;
      w0 = w1;
      if (live && kb + 2 < KB) {
        a1 = __ldg(sa_p + (int64_t)(kb + 2) * args.ldsa);
        if (kTileB) w1 = __ldg(sw_p + kb + 2);
      }
      const float2 sc2 = make_float2(sc, sc);
      if constexpr (EPI == kEpiBf16RowB) {
        __syncwarp();  // every lane has read the previous K-block's scales
        *reinterpret_cast<float4 *>(slot + 4 * lane) = b0;
        b0 = b1;
        if (bcol && kb + 2 < KB) b1 = __ldg(reinterpret_cast<const float4 *>(sb_p + (int64_t)(kb + 2) * args.ldsw));
        __syncwarp();
      }
      const bool got = mbar_wait(&S.tfull[buf], bphase, S.abort_flag, kSiteEpiTmemFull);
      if (!__all_sync(0xffffffffu, got)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t taddr = tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(buf * BN + half * 128);
#pragma unroll
      for (int c = 0; c < 2; ++c) {  // two 64-column halves, two loads in flight each
        uint32_t r[64];
        tmem_ld_32x32b_x32(taddr + 64 * c, *reinterpret_cast<uint32_t(*)[32]>(&r[0]));
        tmem_ld_32x32b_x32(taddr + 64 * c + 32, *reinterpret_cast<uint32_t(*)[32]>(&r[32]));
        tmem_ld_wait();
        if (c == 1) {  // the buffer has been read: hand it back to the MMA warp
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive_relaxed(&S.tempty[buf]);
        }
        if constexpr (EPI == kEpiBf16RowB) {
          // acc[n] += P[n] * (sa[m] * sb[n]): the scale product per column pair
#pragma unroll
          for (int j = 0; j < 32; j += 2) {
            const float4 sb4 = *reinterpret_cast<const float4 *>(slot + 64 * c + 2 * j);
            const float2 s01 = __fmul2_rn(sc2, make_float2(sb4.x, sb4.y));
            const float2 s23 = __fmul2_rn(sc2, make_float2(sb4.z, sb4.w));
            acc[32 * c + j] = __ffma2_rn(make_float2(__uint_as_float(r[2 * j]), __uint_as_float(r[2 * j + 1])), s01,
                                         acc[32 * c + j]);
            acc[32 * c + j + 1] = __ffma2_rn(make_float2(__uint_as_float(r[2 * j + 2]), __uint_as_float(r[2 * j + 3])),
                                             s23, acc[32 * c + j + 1]);
          }
        } else {
#pragma unroll
          for (int j = 0; j < 32; ++j)
            acc[32 * c + j] = __ffma2_rn(make_float2(__uint_as_float(r[2 * j]), __uint_as_float(r[2 * j + 1])), sc2,
                                         acc[32 * c + j]);
        }
      }
      if (++buf == 2) {
        buf = 0;
        bphase ^= 1;
      }
    }
    if (!ok) break;

    if constexpr (EPI == kEpiSwigluFp32 || EPI == kEpiSwigluPow2) {
      constexpr int MODE = EPI == kEpiSwigluPow2 ? FP8BQ_SCALE_POW2 : FP8BQ_SCALE_FP32;
      const bool done = half == 0 ? swiglu_epilogue<G, MODE, 0>(S, args, tl, acc, ew, quarter, lane, xphase)
                                  : swiglu_epilogue<G, MODE, 1>(S, args, tl, acc, ew, quarter, lane, xphase);
      if (!done) break;
    } else if constexpr (!G) {
      // bf16 out: two 64-column chunks through this warp's 4 KB staging buffer,
      // written in the 128-byte swizzled order the TMA store expects.
#pragma unroll
      for (int c = 0; c < 2; ++c) {
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
          const int x = tl.nb * BN + half * 128 + c * 64;
          const int y = tl.row0 + quarter * 32;
          if (x < args.N && y < args.M) {
            tma_store_2d(tmY, ebuf, x, y);
            bulk_commit_group();
          }
        }
      }
    } else {
      // bf16 out in four 32-column chunks through the staging buffer, whose
      // layout is the TMA's 64-byte swizzle.  A tile wholly inside its expert
      // leaves with TMA stores; a tile that runs past its expert's last row
      // is copied by the warp, 8 rows x 64 bytes per instruction, rows masked.
      const int rbase = tl.row0 + quarter * 32;
      const bool whole = tl.row0 + BM <= tl.row_end;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        if (lane == 0) bulk_wait_group_read0();  // an earlier TMA store has left the buffer
        __syncwarp();
        uint8_t *rowp = ebuf + lane * 64;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float2 *a = &acc[c * 16 + j * 4];
          uint4 pk;
          pk.x = pack_bf16x2(a[0].x, a[0].y);
          pk.y = pack_bf16x2(a[1].x, a[1].y);
          pk.z = pack_bf16x2(a[2].x, a[2].y);
          pk.w = pack_bf16x2(a[3].x, a[3].y);
          *reinterpret_cast<uint4 *>(rowp + ((j ^ ((lane >> 1) & 3)) << 4)) = pk;
        }
        const int n0 = tl.nb * BN + half * 128 + c * 32;
        if (whole) {
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0 && n0 < args.N) {
            tma_store_2d(tmY, ebuf, n0, rbase);
            bulk_commit_group();
          }
        } else {
          __syncwarp();
#pragma unroll
          for (int it = 0; it < 4; ++it) {
            const int r = it * 8 + (lane >> 2);
            const int p = lane & 3;
            const uint4 v = *reinterpret_cast<const uint4 *>(ebuf + r * 64 + ((p ^ ((r >> 1) & 3)) << 4));
            const int gr = rbase + r;
            const int gc = n0 + p * 8;
            if (gr < tl.row_end && gc < args.N)
              *reinterpret_cast<uint4 *>(args.y + (int64_t)gr * args.ldy + gc) = v;
          }
        }
      }
    }
  }
  if constexpr (tma_store_epi<EPI>()) {
    if (lane == 0) bulk_wait_group0();
  }
  __syncwarp();
}

template <bool G, int EPI>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_promote_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                        const __grid_constant__ CUtensorMap tmY, const GemmArgs args) {
  extern __shared__ uint8_t smem_raw[];
  const Smem S = carve<G>(smem_raw);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&S.full[s], 1);
      mbar_init(&S.empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&S.tfull[b], 1);
      mbar_init(&S.tempty[b], kEpiWarps);
    }
    mbar_init(S.drain, 1);
    for (int q = 0; q < 4; ++q) mbar_init(&S.xbar[q], 64);
    *S.abort_flag = 0;
    fence_mbarrier_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tensormap(&tmA);
    prefetch_tensormap(&tmB);
    if constexpr (tma_store_epi<EPI>()) prefetch_tensormap(&tmY);
  }
  if constexpr (G) {
    if (warp == 2) build_schedule(S, args, lane);
  }
  if (warp == 1) {
    tmem_alloc(S.tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *S.tmem_slot;

  // Each role's setmaxnreg sits inside the role's own branch, so the code of
  // the role is compiled under that role's register budget.
  if (warp < 4) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kLowRegs));
    if (warp == 0 && lane == 0) run_producer<G>(S, &tmA, &tmB, args);
    else if (warp == 1 && lane == 0) run_mma<G>(S, tmem_base, args);
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kHighRegs));
    run_epilogue<G, EPI>(S, tmem_base, &tmY, args, warp, lane);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

// Per-device one-time setup: opt in to the large shared-memory carve-up and
// confirm that the kernel was built with the register count the setmaxnreg
// split assumes (a smaller count would make setmaxnreg.inc wait forever).
template <bool G, int EPI>
fp8bq_status prepare_kernel() {
  static DeviceOnce once;  // one per instantiation
  return once.get([](int) {
    cudaFuncAttributes fa;
    cudaError_t e = cudaFuncGetAttributes(&fa, gemm_promote_kernel<G, EPI>);
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncGetAttributes(gemm)");
    if (fa.numRegs != kLaunchRegs) return FP8BQ_ERR_UNSUPPORTED;
    e = cudaFuncSetAttribute(gemm_promote_kernel<G, EPI>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             Cfg<G>::kSmemBytes);
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(gemm)");
    return FP8BQ_OK;
  });
}

}  // namespace
}  // namespace fp8bq
