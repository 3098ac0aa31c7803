// Decode-shaped block-scaled FP8 linear, wide form, for sm_100a:
// Y[M,N] = q(X)[M,K] . W[N,K]^T for M <= 256 tokens (in groups of 64), with
// the activation quantized in 1x128 tiles and W pre-quantized in 128x128
// tiles.
//
// Method: "NVIDIA NeMo RL Achieves 48% Speedup With End-to-End FP8 Precision
// Training", section "Technical breakthrough": FP8 is applied in generation as
// well as in training, with block-wise E4M3 (activations 1x128, weights
// 128x128).  A generation step's linear layers see a handful of tokens, so
// the time is the weight's stream from HBM.
//
// The tokens are the MMA's 128-row operand (A) and 256 weight rows its N
// dimension: one tcgen05.mma 128x256x32 covers twice the weight bytes of a
// 128-weight-row MMA at the same issue cost, so the MMA no longer paces the
// weight stream.  Only A's first NT rows (NT = M, or a group's 64 tokens,
// rounded up to 16, 32 or 64) hold tokens; the MMA reads the rest of its 128
// rows from whatever follows in shared memory (the layout keeps that window
// inside the allocation) and the matching accumulator rows (TMEM lanes
// NT..127) are never read back.
//
// A work item is (256-row weight tile t, 128-deep K-block kb): its 32 KB
// weight tile arrives by TMA, 4 MMAs accumulate into one of two 256-column
// TMEM buffers, and the epilogue warps of the token lanes (thread = token,
// 64 weight rows each) add P * (sa[kb][token] * sw[nb][kb]) into FP32
// registers, nb being the 128-row weight block of those rows.
//
// Split over K in thread-block clusters of S CTAs (S up to 16): cluster c
// owns blocks c, c + C, ... (a block is a weight tile and a group of up to 64
// tokens); rank r takes K-blocks r, r + S, ... of each.  At
// the end of a tile every rank sends each 4-column piece of its FP32 partial
// (NT x 256) to the rank that owns those columns (rank r owns slice r of the
// 256 columns), with st.async stores into the owner's shared memory that
// complete on the owner's mbarrier; the owner adds the S partials of its
// slice in rank order (deterministic) and writes those columns of Y.  No
// fence and no remote load is on that path, and the sum is spread over the
// cluster.
//
// The kernel is launched as a programmatic dependent of the previous kernel
// of the stream: its set-up (barriers, TMEM, cluster) overlaps that kernel's
// tail, and every global access comes after griddepcontrol.wait.
//
// The activation's codes either come from a quantization inside this kernel
// (M <= 16 and at most 64 1x128 tiles per CTA: worker warps write them in the
// operand layout while the weight ring fills) or from the workspace, written
// by a prologue kernel and loaded by TMA beside the weight tiles.
#include <cuda_bf16.h>
#include <string.h>

#include <algorithm>

#include "device.cuh"
#include "internal.h"
#include "quant.cuh"

namespace fp8bq {
namespace {

constexpr int WBN = 256, WBK = 128;
// Sixteen warps.  Warp w may read TMEM lanes 32 (w % 4) .. 32 (w % 4) + 31
// only, and tokens sit in lanes 0..NT-1 (NT <= 64: lane quarters 0 and 1), so
// warps 2 and 3 (quarters that never hold a token) are the TMA producer and
// the MMA issuer, and warp w of a token quarter takes weight columns
// 64 (w / 4) .. 64 (w / 4) + 63 of the tile: 64 FP32 accumulators per thread
// within the 128 registers a 512-thread CTA allows.  Warps 4..11 (the
// "workers") also quantize the activation, stage the weight scales and do the
// cross-CTA sum.
constexpr int kWThreads = 512;
constexpr int kWProducerWarp = 2;
constexpr int kWMmaWarp = 3;
constexpr int kWMaxM = 256;          // tokens; above 64 in groups of 64 (one block per weight tile and group)
constexpr int kWMaxSplit = 16;       // CTAs per cluster (above 8: the non-portable cluster sizes)
constexpr int kWSmemCap = 232448;    // dynamic shared memory per CTA (227 KB)
constexpr int kWMaxStages = 8;
constexpr int kWMinStages = 3;
constexpr int kWSwItems = 256;       // work items whose two weight scales are staged in shared memory
// 1x128 activation tiles per CTA quantized inside the kernel (one pass of the
// 256 worker threads, four per tile).  Measured: beyond one pass the prologue
// kernel is faster (the extra passes' loads wait behind the weight stream).
constexpr int kWResMaxTiles = 64;
// Split choice, in units of one work item (a 32 KB weight tile): the busiest
// CTA's items plus, for a split tile, about kWRedItems for the cross-CTA sum.
constexpr int kWRedItems = 1;

// Columns of a tile owned by each rank in the cross-CTA sum of a split of S:
// whole 8-column pieces (rank r: [r c, min(256, (r + 1) c)), c = this).
__host__ __device__ constexpr int slice_cols(int S) { return ((WBN + S - 1) / S + 7) / 8 * 8; }

// QM < 0: activation codes and scales from the workspace (TMA, in the weight
// stages); QM = FP8BQ_SCALE_FP32 / POW2: quantized in the kernel (NT = 16).
template <int NT, int QM>
struct WCfg {
  static constexpr bool kRes = QM >= 0;
  static constexpr int kWBytes = WBN * WBK;   // weight tile
  static constexpr int kXBytes = NT * WBK;    // the token rows of one K-block's A tile (a stage slot)
  static constexpr int kSBytes = NT * 4;      // the K-block's activation scales
  static constexpr int kSSlot = (kSBytes + 127) / 128 * 128;
  static constexpr int kTx = kWBytes + (kRes ? 0 : kXBytes + kSBytes);
  static constexpr int kQuarters = (NT + 31) / 32;   // TMEM lane quarters holding tokens
  static constexpr int kActWarps = 4 * kQuarters;    // token warps (four column quarters each)
  // workers: warps 4..11 (some of them token warps as well).  Measured: the
  // same role on the eight warps whose quarters hold no token was 0.3 to
  // 1.6 us slower per call at M = 1 and 2.
  static constexpr int kWorkWarps = 8;
  static constexpr int kWorkThreads = 32 * kWorkWarps;
  static __device__ __forceinline__ int work_slot(int w) { return w >= 4 && w < 12 ? w - 4 : -1; }
  static constexpr int kTmemCols = 2 * WBN;          // two accumulator buffers
  static_assert(!kRes || NT == 16, "activation quantized in the kernel only for NT = 16");
  static_assert(kXBytes % 1024 == 0, "A tiles start on the 1024-byte swizzle atom");

  // Shared memory (after up to 1024 bytes of alignment): the codes (nres
  // resident K-blocks, or one slot per stage) first, so that the 16 KB an A
  // descriptor spans from any code tile stays inside the weight stages that
  // follow; the weight stages; the activation scales; the receive buffer of
  // the cross-CTA sum (S > 1); the staged weight scales; the barriers.
  //
  // A resident K-block's codes: the M token rows rounded up to the 8-row
  // swizzle atom (the A window's further rows read the next K-blocks' codes).
  static __host__ __device__ int res_tile_bytes(int M) { return (M + 7) / 8 * 1024; }
  static __host__ __device__ int x_bytes(int nst, int nres, int M) {
    return kRes ? nres * res_tile_bytes(M) : nst * kXBytes;
  }
  static __host__ __device__ int s_bytes(int nst, int nres) { return kRes ? nres * NT * 4 : nst * kSSlot; }
  // [S][M][slice_cols(S)]: every rank's partial of this CTA's column slice
  static __host__ __device__ int recv_floats(int S, int M) { return S > 1 ? S * M * slice_cols(S) : 0; }
  static int smem_bytes(int nst, int nres, int S, int M) {
    return 1024 + x_bytes(nst, nres, M) + nst * kWBytes + s_bytes(nst, nres) + recv_floats(S, M) * 4 +
           kWSwItems * 2 * 4 + 512;
  }
  static int stages_for(int nres, int S, int M) {
    const int per = kWBytes + (kRes ? 0 : kXBytes + kSSlot);
    const int n = (kWSmemCap - smem_bytes(0, nres, S, M)) / per;
    return n < kWMinStages ? 0 : (n > kWMaxStages ? kWMaxStages : n);
  }
};

struct WideArgs {
  const float *sw;
  int32_t M, N, KB, NB;  // NB: 128-row weight blocks (rows of sw)
  int32_t NW;            // 256-row weight tiles
  int32_t MG;            // token groups of 64 rows (1 when M <= 64)
  int32_t split;         // CTAs per cluster (S)
  int32_t nst;           // weight stages
  int32_t nres;          // resident K-blocks of activation codes (0 unless quantized in the kernel)
  uint16_t *y;           // bf16 bits
  int64_t ldy;
  const uint16_t *x;     // in-kernel quantization: bf16 activations [M][ldx]
  int64_t ldx;
};

// A block is a (256-row weight tile, group of 64 tokens) pair, block b =
// tile * MG + group (the groups of a tile are neighbours, so the clusters
// streaming one weight tile for different tokens run at the same time and
// share it in L2).  The work of CTA `rank` of cluster `cid` (of `ncl`):
// blocks cid, cid + ncl, ... and of each the K-blocks rank, rank + S, ...
// (interleaved, so that the cluster's CTAs stream neighbouring pieces of the
// same weight rows at the same time); item q is block t0 + (q / nk) * ncl,
// K-block kb0 + (q % nk) * S.
struct WShare {
  int t0, ncl, kb0, ks, nk, nblk, items, mg;
  __device__ WShare(const WideArgs &a, int cid, int ncls, int rank) {
    t0 = cid;
    ncl = ncls;
    kb0 = rank;
    ks = a.split;
    nk = (a.KB - rank + a.split - 1) / a.split;
    mg = a.MG;
    const int nbt = a.NW * a.MG;
    nblk = cid < nbt ? (nbt - cid + ncls - 1) / ncls : 0;
    items = nblk * nk;
  }
  __device__ int blk(int q) const { return t0 + (q / nk) * ncl; }
  __device__ int tile(int q) const { return blk(q) / mg; }
  __device__ int tgroup(int q) const { return blk(q) % mg; }
  __device__ int pos(int q) const { return q % nk; }
  __device__ int kb(int q) const { return kb0 + (q % nk) * ks; }
};

__device__ __forceinline__ uint32_t bf16x2_bits(float lo, float hi) {
  __nv_bfloat162 b = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t *>(&b);
}

__device__ __forceinline__ uint16_t bf16_bits1(float v) {
  __nv_bfloat16 b = __float2bfloat16_rn(v);
  return *reinterpret_cast<uint16_t *>(&b);
}

// Eight consecutive output values of row `yr` at column n (n + 8 <= N: one
// 16-byte store; else the columns below N one by one).
__device__ __forceinline__ void store8(uint16_t *yr, int n, int N, const float *v) {
  if (n + 8 <= N) {
    uint4 p;
    p.x = bf16x2_bits(v[0], v[1]);
    p.y = bf16x2_bits(v[2], v[3]);
    p.z = bf16x2_bits(v[4], v[5]);
    p.w = bf16x2_bits(v[6], v[7]);
    *reinterpret_cast<uint4 *>(yr + n) = p;
  } else {
#pragma unroll
    for (int j = 0; j < 8; ++j)
      if (n + j < N) yr[n + j] = bf16_bits1(v[j]);
  }
}

template <int NT, int QM>
__global__ void __launch_bounds__(kWThreads, 1)
    decode_wide_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX,
                       const __grid_constant__ CUtensorMap tmS, const WideArgs args) {
  using C = WCfg<NT, QM>;
  constexpr bool kRes = C::kRes;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int nst = args.nst;
  const int S = args.split;
  uint8_t *sX = base;                                 // codes: nres resident tiles, or nst stage slots
  uint8_t *sW = sX + C::x_bytes(nst, args.nres, args.M);  // nst weight tiles
  const int xtile = C::res_tile_bytes(args.M);        // resident codes: bytes per K-block
  float *sSx = reinterpret_cast<float *>(sW + nst * C::kWBytes);  // [nres][NT], or nst slots of kSSlot bytes
  float *sR = reinterpret_cast<float *>(reinterpret_cast<uint8_t *>(sSx) + C::s_bytes(nst, args.nres));
  float *sSw = sR + C::recv_floats(S, min(args.M, NT));  // [kWSwItems][2]
  uint64_t *bars = reinterpret_cast<uint64_t *>(sSw + 2 * kWSwItems);
  uint64_t *full = bars;
  uint64_t *empty = bars + kWMaxStages;
  uint64_t *tfull = empty + kWMaxStages;
  uint64_t *tempty = tfull + 2;
  uint64_t *drain = tempty + 2;
  uint64_t *xready = drain + 1;   // the codes (if quantized here) and the staged weight scales are written
  uint64_t *rbar = xready + 1;    // every rank's partial of this CTA's slice has arrived (st.async bytes)
  uint64_t *pfree = rbar + 1;     // every rank has read its slice: this CTA may send the next tile's pieces
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(pfree + 1);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rank = S > 1 ? (int)cluster_ctarank() : 0;
  const WShare sh(args, S > 1 ? (int)cluster_id_x() : (int)blockIdx.x, S > 1 ? (int)nclusters_x() : (int)gridDim.x,
                  rank);
  const int wslot = C::work_slot(warp);
  const bool worker = wslot >= 0;
  const bool tokw = (warp & 3) < C::kQuarters && warp != kWProducerWarp && warp != kWMmaWarp;

  const int et = 32 * wslot + lane;  // worker thread 0 .. kWorkThreads - 1
  const int grp = et >> 2, qd = et & 3;
  // The activation's loads (when it is quantized here): tile t of the CTA's
  // nk * M <= 64 (K-block t / M, row t % M) by the four lanes of group t.
  uint4 xv[4];
  constexpr int kSwPer = (2 * kWSwItems + C::kWorkThreads - 1) / C::kWorkThreads;
  float swv[kSwPer];
  auto load_x = [&]() {
    const int t = grp;
    const int i = t / args.M, m = t - (t / args.M) * args.M;
    const uint16_t *xrow = args.x + (int64_t)m * args.ldx + (int64_t)(sh.kb0 + i * sh.ks) * WBK;
    const bool have = t < sh.nk * args.M;
#pragma unroll
    for (int j = 0; j < 4; ++j) xv[j] = have ? ld_nc_v4(xrow + (j * 4 + qd) * 8) : make_uint4(0, 0, 0, 0);
  };
  // weight scale of item q's half hh (0 for a half beyond the last weight row)
  auto sw_global = [&](int q, int hh) -> float {
    const int nb = 2 * sh.tile(q) + hh;
    return nb < args.NB ? __ldg(args.sw + (int64_t)nb * args.KB + sh.kb(q)) : 0.f;
  };
  pdl_launch_dependents();
  if (threadIdx.x == 0) {
    for (int s = 0; s < nst; ++s) {
      mbar_init(&full[s], 1);
      // the MMA's commit, and with the scales in the stage the token warps that read them
      mbar_init(&empty[s], kRes ? 1 : 1 + C::kActWarps);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], C::kActWarps);
    }
    mbar_init(drain, 1);
    mbar_init(xready, C::kWorkWarps);
    mbar_init(rbar, 1);                   // this CTA's expect_tx; the bytes come from every rank
    mbar_init(pfree, S * C::kWorkWarps);  // the workers of every rank
    *abort_flag = 0;
    fence_mbarrier_init();
  }
  if (warp == kWProducerWarp && lane == 0) {
    prefetch_tensormap(&tmW);
    if constexpr (!kRes) {
      prefetch_tensormap(&tmX);
      prefetch_tensormap(&tmS);
    }
  }
  if (warp == kWMmaWarp) {
    tmem_alloc(tmem_slot, C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  if (S > 1) cluster_sync();  // every CTA's barriers exist before any remote arrive
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // After the wait (the previous kernel of the stream has completed) global
  // memory is read and written; the workers issue the activation's loads and
  // the weight scales' loads first.
  pdl_wait();
  if (worker) {
    if constexpr (kRes) load_x();
#pragma unroll
    for (int i = 0; i < kSwPer; ++i) {
      const int z = et + C::kWorkThreads * i;
      swv[i] = z < 2 * kWSwItems && (z >> 1) < sh.items ? sw_global(z >> 1, z & 1) : 0.f;
    }
  }

  if (warp == kWProducerWarp) {
    if (lane == 0) {
      // ---------------------------------------------------------------- producer
      int stage = 0;
      uint32_t phase = 0, armed = 0, armed_parity = 0;
      bool ok = true;
      for (int q = 0; q < sh.items; ++q) {
        const int t = sh.tile(q), kb = sh.kb(q), r0 = 64 * sh.tgroup(q);
        if (!mbar_wait(&empty[stage], phase ^ 1, abort_flag, kSiteProducerEmpty)) {
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(&full[stage], C::kTx);
        tma_load_2d(sW + stage * C::kWBytes, &tmW, &full[stage], kb * WBK, t * WBN);
        if constexpr (!kRes) {
          tma_load_2d(sX + stage * C::kXBytes, &tmX, &full[stage], kb * WBK, r0);
          tma_load_2d(reinterpret_cast<uint8_t *>(sSx) + stage * C::kSSlot, &tmS, &full[stage], r0, kb);
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
    }
  } else if (warp == kWMmaWarp) {
    if (lane == 0) {
      // ---------------------------------------------------------------- MMA issuer
      const uint32_t idesc = idesc_f8f6f4_e4m3_f32(128, WBN);
      int stage = 0, buf = 0;
      uint32_t phase = 0, bphase = 0;
      bool ok = true, issued = false;
      if constexpr (kRes) ok = mbar_wait(xready, 0, abort_flag, kSiteMmaFull);  // the codes are written
      for (int q = 0; q < sh.items && ok; ++q) {
        if (!mbar_wait(&tempty[buf], bphase ^ 1, abort_flag, kSiteMmaTmemEmpty) ||
            !mbar_wait(&full[stage], phase, abort_flag, kSiteMmaFull)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d = tmem_base + (uint32_t)(buf * WBN);
        const uint32_t a0 = kRes ? smem_addr(sX + sh.pos(q) * xtile) : smem_addr(sX + stage * C::kXBytes);
        const uint32_t b0 = smem_addr(sW + stage * C::kWBytes);
#pragma unroll
        for (int k = 0; k < WBK / 32; ++k)
          mma_f8f6f4(d, smem_desc_k_sw128(a0 + 32 * k), smem_desc_k_sw128(b0 + 32 * k), idesc, k > 0 ? 1u : 0u);
        mma_commit(&empty[stage]);
        mma_commit(&tfull[buf]);
        issued = true;
        if (++stage == nst) {
          stage = 0;
          phase ^= 1;
        }
        if (++buf == 2) {
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
    if (worker) {
#pragma unroll
      for (int i = 0; i < kSwPer; ++i) {
        const int z = et + C::kWorkThreads * i;
        if (z < 2 * kWSwItems && (z >> 1) < sh.items) sSw[z] = swv[i];
      }
      if constexpr (kRes) {
        // ---------------------------------------------------------- activation quantization
        // tile (i, m) for i < nk, m < M, four lanes each (groups never
        // straddle a warp); a code tile's rows from M up to its 8-row atom
        // are left as they are: they only feed accumulator rows never read
        const int t = grp;
        const bool have = t < sh.nk * args.M;
        const int i = have ? t / args.M : 0, m = have ? t - (t / args.M) * args.M : 0;
        qdev::quant_row_tile_to_smem<QM < 0 ? 0 : QM>(have, xv, qd, sX + i * xtile, m, sSx + i * NT + m);
        __syncwarp();
        fence_proxy_async_smem();
      } else {
        __syncwarp();
      }
      if (lane == 0) mbar_arrive(xready);
    }
    // ------------------------------------------------------------------ epilogue
    const int quarter = warp & 3;
    const int g = warp >> 2;                    // weight columns 64 g .. 64 g + 63 of the tile
    const int m = quarter * 32 + lane;          // token = accumulator row (token warps)
    const int ms = m < NT ? m : NT - 1;         // its scale slot (lanes beyond NT read a valid one)
    int stage = 0, buf = 0;
    bool xw = false;  // xready seen
    uint32_t bphase = 0;
    float acc[64];
#pragma unroll
    for (int j = 0; j < 64; ++j) acc[j] = 0.f;
    bool alive = tokw || worker;
    auto sw_of = [&](int q) -> float { return q < kWSwItems ? sSw[2 * q + (g >> 1)] : sw_global(q, g >> 1); };
    // this rank's column slice of the cross-CTA sum
    const int cw = slice_cols(S);
    const int s0 = min(WBN, rank * cw), s1 = min(WBN, s0 + cw);
    const int nch = (s1 - s0) / 8;
    for (int jb = 0; jb < sh.nblk && alive; ++jb) {
      const int t = sh.tile(jb * sh.nk), r0 = 64 * sh.tgroup(jb * sh.nk);
      const int Mb = min(args.M - r0, 64);  // this block's tokens: rows r0 .. r0 + Mb - 1
      if (tokw) {
#pragma unroll 1
        for (int i = 0; i < sh.nk; ++i) {
          const int q = jb * sh.nk + i;
          const bool got = mbar_wait(&tfull[buf], bphase, abort_flag, kSiteEpiTmemFull);
          if (!__all_sync(0xffffffffu, got)) {
            alive = false;
            break;
          }
          tc_fence_after();
          // the activation scales and the weight scales are written
          const bool xok = xw || mbar_wait(xready, 0, abort_flag, kSiteEpiTmemFull);
          xw = true;
          if (!__all_sync(0xffffffffu, xok)) {
            alive = false;
            break;
          }
          float sx;
          if constexpr (kRes) sx = sSx[i * NT + ms];
          else sx = sSx[stage * (C::kSSlot / 4) + ms];
          const float s = sx * sw_of(q);
          if constexpr (!kRes) {
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[stage]);  // the stage's scales have been read
          }
          const uint32_t taddr = tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(buf * WBN + g * 64);
#pragma unroll
          for (int c = 0; c < 2; ++c) {
            uint32_t v[32];
            tmem_ld_32x32b_x32(taddr + 32 * c, v);
            tmem_ld_wait();
            if (c == 1) {
              tc_fence_before();
              __syncwarp();
              if (lane == 0) mbar_arrive_relaxed(&tempty[buf]);
            }
#pragma unroll
            for (int j = 0; j < 32; ++j) acc[32 * c + j] = fmaf(__uint_as_float(v[j]), s, acc[32 * c + j]);
          }
          if (++stage == nst) stage = 0;
          if (++buf == 2) {
            buf = 0;
            bphase ^= 1;
          }
        }
      }
      if (!alive) break;
      if (S == 1) {
        if (tokw && m < Mb) {
          uint16_t *yr = args.y + (int64_t)(r0 + m) * args.ldy;
          const int n0 = t * WBN + g * 64;
          if (n0 + 64 <= args.N) {
#pragma unroll
            for (int c = 0; c < 8; ++c) {
              uint4 pk;
              pk.x = bf16x2_bits(acc[8 * c + 0], acc[8 * c + 1]);
              pk.y = bf16x2_bits(acc[8 * c + 2], acc[8 * c + 3]);
              pk.z = bf16x2_bits(acc[8 * c + 4], acc[8 * c + 5]);
              pk.w = bf16x2_bits(acc[8 * c + 6], acc[8 * c + 7]);
              *reinterpret_cast<uint4 *>(yr + n0 + 8 * c) = pk;
            }
          } else {
#pragma unroll
            for (int j = 0; j < 64; ++j)
              if (n0 + j < args.N) yr[n0 + j] = bf16_bits1(acc[j]);
          }
        }
      } else {
        if (tokw) {
          // tile jb's pieces, once every rank has read its slice of tile jb - 1:
          // each 4-column piece to the rank that owns those columns
          const bool fine = jb == 0 || mbar_wait_cluster(pfree, (uint32_t)((jb - 1) & 1), abort_flag, kSiteEpiTmemFull);
          if (!__all_sync(0xffffffffu, fine)) {
            alive = false;
            break;
          }
          if (m < Mb) {
            const uint32_t row = smem_addr(sR + (rank * Mb + m) * cw);
            const uint32_t rb = smem_addr(rbar);
            int owner = (64 * g) / cw;
            int ob = owner * cw;
            uint32_t dst_row = mapa_shared(row, (uint32_t)owner), dst_bar = mapa_shared(rb, (uint32_t)owner);
#pragma unroll
            for (int c = 0; c < 16; ++c) {
              const int col = 64 * g + 4 * c;
              if (col >= ob + cw) {
                ++owner;
                ob += cw;
                dst_row = mapa_shared(row, (uint32_t)owner);
                dst_bar = mapa_shared(rb, (uint32_t)owner);
              }
              st_async_v4(dst_row + (uint32_t)(col - ob) * 4u,
                          make_float4(acc[4 * c], acc[4 * c + 1], acc[4 * c + 2], acc[4 * c + 3]), dst_bar);
            }
          }
        }
        if (worker) {
          // columns [s0, s1) of tile jb: the S partials added in rank order
          if (wslot == 0 && lane == 0) mbar_arrive_expect_tx(rbar, (uint32_t)(S * Mb * (s1 - s0) * 4));
          const bool got = mbar_wait_cluster(rbar, (uint32_t)(jb & 1), abort_flag, kSiteEpiTmemFull);
          if (!__all_sync(0xffffffffu, got)) {
            alive = false;
            break;
          }
          const int nbase = t * WBN;
          const int units = Mb * nch;
#pragma unroll 1
          for (int u = et; u < units; u += C::kWorkThreads) {
            const int mm = u / nch, col = s0 + 8 * (u - mm * nch);
            if (nbase + col >= args.N) continue;
            const float *src = sR + mm * cw + (col - s0);
            float sum[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) sum[j] = 0.f;
#pragma unroll 4
            for (int p = 0; p < S; ++p) {
              const float4 a = *reinterpret_cast<const float4 *>(src + p * (Mb * cw));
              const float4 b = *reinterpret_cast<const float4 *>(src + p * (Mb * cw) + 4);
              sum[0] += a.x;
              sum[1] += a.y;
              sum[2] += a.z;
              sum[3] += a.w;
              sum[4] += b.x;
              sum[5] += b.y;
              sum[6] += b.z;
              sum[7] += b.w;
            }
            store8(args.y + (int64_t)(r0 + mm) * args.ldy, nbase + col, args.N, sum);
          }
          // the slice has been read (its sums are stored): the ranks may send the next tile
          __syncwarp();
          if (lane < S) mbar_arrive_cluster_relaxed(mapa_shared(smem_addr(pfree), (uint32_t)lane));
        }
      }
#pragma unroll
      for (int j = 0; j < 64; ++j) acc[j] = 0.f;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kWMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::kTmemCols);
  }
  if (S > 1) cluster_sync();  // no CTA leaves while another may still write its shared memory
}

// Per-device set-up of the five instantiations (shared-memory and cluster-size
// opt-ins) and the number of clusters of each size that can
// be resident at once (clusters live inside one GPC, so C * S <= SMs alone
// does not guarantee it; a second wave would double the time).
struct WideDevice {
  int max_clusters[kWMaxSplit + 1];
};
WideDevice g_wdev[kMaxDevices];
DeviceOnce g_wsetup;

template <int NT, int QM>
fp8bq_status setup_wide_kernel() {
  cudaError_t e =
      cudaFuncSetAttribute(decode_wide_kernel<NT, QM>, cudaFuncAttributeMaxDynamicSharedMemorySize, kWSmemCap);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(decode_wide_kernel<NT, QM>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
  if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(decode_wide)");
  return FP8BQ_OK;
}

fp8bq_status wide_device(const WideDevice **out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  const fp8bq_status st = g_wsetup.get_for(dev, [](int d) -> fp8bq_status {
    fp8bq_status s = setup_wide_kernel<16, FP8BQ_SCALE_FP32>();
    if (s == FP8BQ_OK) s = setup_wide_kernel<16, FP8BQ_SCALE_POW2>();
    if (s == FP8BQ_OK) s = setup_wide_kernel<16, -1>();
    if (s == FP8BQ_OK) s = setup_wide_kernel<32, -1>();
    if (s == FP8BQ_OK) s = setup_wide_kernel<64, -1>();
    if (s != FP8BQ_OK) return s;
    WideDevice &wd = g_wdev[d];
    wd.max_clusters[0] = 0;
    wd.max_clusters[1] = num_sms();
    for (int S = 2; S <= kWMaxSplit; ++S) {
      // every instantiation runs one CTA per SM, so one query at the largest
      // shared-memory size stands for all
      cudaLaunchConfig_t cfg = {};
      cfg.blockDim = dim3(kWThreads);
      cfg.gridDim = dim3((unsigned)(S * 256));
      cfg.dynamicSmemBytes = kWSmemCap;
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeClusterDimension;
      attr[0].val.clusterDim.x = (unsigned)S;
      attr[0].val.clusterDim.y = 1;
      attr[0].val.clusterDim.z = 1;
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      int n = 0;
      if (cudaOccupancyMaxActiveClusters(&n, decode_wide_kernel<16, -1>, &cfg) != cudaSuccess) {
        cudaGetLastError();
        n = 0;  // clusters of this size are not used
      }
      wd.max_clusters[S] = n;
    }
    return FP8BQ_OK;
  });
  if (st == FP8BQ_OK) *out = &g_wdev[dev];
  return st;
}

// Shared memory of split S: resident codes when the activation is quantized
// in the kernel, else stage slots; false if fewer than kWMinStages fit.
bool fit_wide(DecodeWidePlan *p, int S, int64_t M, int KB, bool vec) {
  const int nk = (KB + S - 1) / S;
  p->res = false;
  if (p->NT == 16 && vec && nk * M <= kWResMaxTiles) {
    p->nres = nk;
    p->nst = WCfg<16, FP8BQ_SCALE_FP32>::stages_for(nk, S, (int)M);  // both modes lay shared memory out alike
    p->smem = WCfg<16, FP8BQ_SCALE_FP32>::smem_bytes(p->nst, nk, S, (int)M);
    p->res = p->nst > 0;
    if (p->res) return true;
  }
  p->nres = 0;
  const int mrows = (int)std::min<int64_t>(M, 64);  // a block's tokens at most
  switch (p->NT) {
    case 16:
      p->nst = WCfg<16, -1>::stages_for(0, S, mrows);
      p->smem = WCfg<16, -1>::smem_bytes(p->nst, 0, S, mrows);
      break;
    case 32:
      p->nst = WCfg<32, -1>::stages_for(0, S, mrows);
      p->smem = WCfg<32, -1>::smem_bytes(p->nst, 0, S, mrows);
      break;
    default:
      p->nst = WCfg<64, -1>::stages_for(0, S, mrows);
      p->smem = WCfg<64, -1>::smem_bytes(p->nst, 0, S, mrows);
      break;
  }
  return p->nst > 0;
}

template <int NT, int QM>
fp8bq_status launch_wide_nt(const CUtensorMap &tW, const CUtensorMap &tX, const CUtensorMap &tS, const WideArgs &a,
                            const DecodeWidePlan &p, cudaStream_t stream) {
  cudaLaunchConfig_t cfg = {};
  cfg.blockDim = dim3(kWThreads);
  cfg.gridDim = dim3((unsigned)(p.C * p.S));
  cfg.dynamicSmemBytes = (size_t)p.smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = (unsigned)p.S;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = p.S > 1 ? 2 : 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, decode_wide_kernel<NT, QM>, tW, tX, tS, a);
  if (e != cudaSuccess) return cuda_fail(e, "gemm_decode (wide) launch");
  return check_launch("gemm_decode (wide)");
}

}  // namespace

cudaError_t take_device_error_decode_wide(unsigned long long *v) { return take_tu_device_error(v); }

// The split S (CTAs per cluster) and cluster count C (at most the resident
// clusters of that size) that minimise the modelled time: the busiest CTA's
// items, ceil(NW / C) * ceil(KB / S), plus kWRedItems per tile when S > 1;
// ties go to the smaller S.  Only splits whose shared memory fits count.
fp8bq_status plan_decode_wide(int64_t M, int64_t N, int64_t K, bool vec, DecodeWidePlan *p) {
  if (M < 1 || M > kWMaxM || N < 1 || K < 128 || K % 128 != 0) return FP8BQ_ERR_UNSUPPORTED;
  const WideDevice *wd = nullptr;
  const fp8bq_status ready = wide_device(&wd);
  if (ready != FP8BQ_OK) return ready;
  p->NT = M <= 16 ? 16 : (M <= 32 ? 32 : 64);
  p->MG = (int)((M + 63) / 64);
  const int NBT = (int)((N + WBN - 1) / WBN) * p->MG;  // blocks: weight tiles x token groups
  const int KB = (int)(K / WBK);
  int best = 0x7fffffff, bestS = 0;
  for (int s = 1; s <= kWMaxSplit && s <= KB; ++s) {
    const int c = std::min(NBT, std::min(wd->max_clusters[1] / s, wd->max_clusters[s]));
    if (c < 1 || !fit_wide(p, s, M, KB, vec)) continue;
    const int blocks = (NBT + c - 1) / c;
    const int cost = blocks * ((KB + s - 1) / s) + (s > 1 ? blocks * kWRedItems : 0);
    if (cost < best) {
      best = cost;
      bestS = s;
    }
  }
  if (bestS == 0) return FP8BQ_ERR_UNSUPPORTED;
  p->S = bestS;
  p->C = std::min(NBT, std::min(wd->max_clusters[1] / bestS, wd->max_clusters[bestS]));
  fit_wide(p, bestS, M, KB, vec);
  return FP8BQ_OK;
}

fp8bq_status launch_decode_wide(const DecodeWidePlan &p, const uint16_t *x, int64_t ldx, const uint8_t *qw,
                                int64_t ldw, const float *sw, const uint8_t *q, const float *sa, int64_t ldsa,
                                void *y, int64_t ldy, int64_t M, int64_t N, int64_t K, int mode,
                                cudaStream_t stream) {
  CUtensorMap tW, tX, tS;
  if (!make_tmap_2d(&tW, CU_TENSOR_MAP_DATA_TYPE_UINT8, qw, (uint64_t)K, (uint64_t)N, (uint64_t)ldw, WBK, WBN,
                    CU_TENSOR_MAP_SWIZZLE_128B))
    return FP8BQ_ERR_INVALID_ARG;
  if (p.res) {
    tX = tW;  // not read by the kernel
    tS = tW;
  } else if (!make_tmap_2d(&tX, CU_TENSOR_MAP_DATA_TYPE_UINT8, q, (uint64_t)K, (uint64_t)M, (uint64_t)K, WBK,
                           (uint32_t)p.NT, CU_TENSOR_MAP_SWIZZLE_128B) ||
             !make_tmap_2d(&tS, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, sa, (uint64_t)M, (uint64_t)(K / WBK),
                           (uint64_t)ldsa * 4, (uint32_t)p.NT, 1, CU_TENSOR_MAP_SWIZZLE_NONE)) {
    return FP8BQ_ERR_INVALID_ARG;
  }
  WideArgs a;
  a.sw = sw;
  a.M = (int32_t)M;
  a.N = (int32_t)N;
  a.KB = (int32_t)(K / WBK);
  a.NB = (int32_t)((N + 127) / 128);
  a.NW = (int32_t)((N + WBN - 1) / WBN);
  a.MG = p.MG;
  a.split = p.S;
  a.nst = p.nst;
  a.nres = p.nres;
  a.y = static_cast<uint16_t *>(y);
  a.ldy = ldy;
  a.x = x;
  a.ldx = ldx;
  if (p.res)
    return mode == FP8BQ_SCALE_FP32 ? launch_wide_nt<16, FP8BQ_SCALE_FP32>(tW, tX, tS, a, p, stream)
                                    : launch_wide_nt<16, FP8BQ_SCALE_POW2>(tW, tX, tS, a, p, stream);
  switch (p.NT) {
    case 16: return launch_wide_nt<16, -1>(tW, tX, tS, a, p, stream);
    case 32: return launch_wide_nt<32, -1>(tW, tX, tS, a, p, stream);
    default: return launch_wide_nt<64, -1>(tW, tX, tS, a, p, stream);
  }
}

}  // namespace fp8bq
